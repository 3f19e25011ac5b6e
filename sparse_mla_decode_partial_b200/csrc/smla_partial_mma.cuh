// smla_partial_mma.cuh -- split-K partial pass with warp-level bf16 MMA.
//
// "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
// Decode", section "The Split-K Imperative": the decode kernel attends over
// the top-k candidate rows of the KV cache with tensor-core MMA; split-K cuts
// the top-k axis into NSPLIT chunks, one thread block each, and every block
// writes a partial output that a log-sum-exp combine merges later.
//
// One CTA = one (query token, split) and ALL of its heads, because every
// gathered 1152-byte latent row is shared by all heads: gathering it once per
// CTA is what keeps the pass at one HBM read per selected row.
//
// Warp roles (HG = head groups of 16 rows, the mma M dimension):
//   warp 4*HG      producer: resolves index -> page -> row, issues one 1-D
//                  bulk async copy (TMA engine, 1152 B) per row into a ring of
//                  NSTAGE tiles of NT rows, completes on an mbarrier.
//   warps 0..4HG-1 consumers, 4 per head group: S = Q K^T over 576 dims
//                  (each warp NT/4 columns), masked online softmax in fp32
//                  (exp2 domain, quad shuffles + one smem exchange per tile),
//                  P to smem as bf16, O += P C (each warp 128 of the 512
//                  output columns, fp32 registers).
// Shared-memory rows are 1168 B apart (1152 + 16) so that the 8 row addresses
// of every ldmatrix phase fall in distinct 16-byte bank groups.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "smla_ptx.cuh"

namespace smla {

constexpr int kDc = 512;
constexpr int kDr = 64;
constexpr int kD = kDc + kDr;
constexpr int kPage = 64;
constexpr int kRowBytes = kD * 2;                 // 1152
constexpr int kSmemRowBytes = kRowBytes + 16;     // 1168
constexpr float kLog2e = 1.4426950408889634f;     // log2(e)
constexpr float kLn2 = 0.69314718055994531f;      // ln(2)

// Source of the bulk copy for a padding slot: a row of zeros, so that masked
// slots hold finite values (their probability is 0, and 0 * finite = 0).
__device__ __align__(128) uint16_t g_zero_row[kD];

struct PartialParams {
    const __nv_bfloat16 *q;       // [B, T, H, 576]
    const __nv_bfloat16 *cache;   // [num_pages * 64, 576]
    long long num_pages;
    const int *page_table;        // [B, pt_stride]
    int pt_stride;
    const int *idx;               // [B, T, K]
    int B, T, H, K;
    float scale_log2;             // scale * log2(e)
    int nsplit;
    int kc;                       // ceil(K / nsplit)
    float *part_o;                // [B, T, H, S, 512]
    float *part_m;                // [B, T, H, S]
    float *part_lse;              // [B, T, H, S]
    __nv_bfloat16 *o;             // direct mode (S == 1): [B, T, H, 512]
    float *lse;                   // direct mode: [B, T, H]
};

template <int HG, int NT, int NSTAGE>
struct MmaCfg {
    static_assert(NT == 32 || NT == 64, "tile rows");
    static constexpr int kHeads = 16 * HG;
    static constexpr int kComputeWarps = 4 * HG;
    static constexpr int kThreads = (kComputeWarps + 1) * 32;
    static constexpr int kPStride = NT * 2 + 16;  // bytes per P row (conflict-free ldmatrix)
    static constexpr int kStageBytes = NT * kSmemRowBytes;
    static constexpr int kOffQ = 0;
    static constexpr int kOffKV = kOffQ + kHeads * kSmemRowBytes;
    static constexpr int kOffP = kOffKV + NSTAGE * kStageBytes;
    static constexpr int kOffRed = kOffP + HG * 16 * kPStride;   // float [HG][4][16]
    static constexpr int kOffL = kOffRed + HG * 4 * 16 * 4;       // float [HG][4][16]
    static constexpr int kOffHdr = kOffL + HG * 4 * 16 * 4;       // u64 [NSTAGE]
    static constexpr int kOffBar = kOffHdr + NSTAGE * 8;          // u64 full[], empty[], q
    static constexpr int kSmemBytes = kOffBar + (2 * NSTAGE + 1) * 8;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

template <int HG, int NT, int NSTAGE, bool DIRECT>
__global__ void __launch_bounds__(MmaCfg<HG, NT, NSTAGE>::kThreads, 1)
    smla_partial_mma_kernel(const PartialParams p) {
    using C = MmaCfg<HG, NT, NSTAGE>;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x;  // (b * T + t) * S + s
    const int s = unit % p.nsplit;
    const int bt = unit / p.nsplit;
    const int b = bt / p.T;
    const long long j0l = (long long)s * p.kc;
    const int j0 = (int)(j0l < p.K ? j0l : p.K);
    const int j1 = (int)((long long)j0 + p.kc < p.K ? (long long)j0 + p.kc : p.K);
    const int n_tiles = (j1 - j0 + NT - 1) / NT;
    bool dead = false;  // set once a bounded wait of this thread has timed out

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty = full + NSTAGE;
    uint64_t *qbar = full + 2 * NSTAGE;
    volatile uint64_t *hdr = reinterpret_cast<volatile uint64_t *>(smem + C::kOffHdr);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], C::kComputeWarps);
        }
        mbar_init(qbar, 1);
        fence_mbar_init();
    }
    // Head rows beyond H are zero (they are never written by a copy).
    {
        constexpr int kChunks = kSmemRowBytes / 16;
        const int n = (C::kHeads - p.H) * kChunks;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const int r = p.H + i / kChunks;
            *reinterpret_cast<uint4 *>(smem + C::kOffQ + r * kSmemRowBytes + (i % kChunks) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __syncthreads();

    if (warp == C::kComputeWarps) {
        // ============================================================ producer
        const __nv_bfloat16 *qsrc = p.q + (size_t)bt * p.H * kD;
        if (lane == 0) {
            mbar_expect_tx(qbar, (uint32_t)(p.H * kRowBytes));
            mbar_arrive(qbar);
        }
        __syncwarp();
        for (int h = lane; h < p.H; h += 32)
            bulk_g2s(smem + C::kOffQ + h * kSmemRowBytes, qsrc + (size_t)h * kD, kRowBytes, qbar);

        const int *idx_bt = p.idx + (size_t)bt * p.K;
        const int *pt_b = p.page_table + (size_t)b * p.pt_stride;
        const long long max_pos = (long long)p.pt_stride * kPage;
        const uint64_t policy = l2_policy_evict_first();
        constexpr int kSlots = NT / 32;
        const uint8_t *src[kSlots];
        bool valid[kSlots];

        auto resolve = [&](int tile) {
            int iv[kSlots];
#pragma unroll
            for (int k = 0; k < kSlots; ++k) {
                const int j = j0 + tile * NT + k * 32 + lane;
                iv[k] = (j < j1) ? __ldg(idx_bt + j) : -1;
            }
#pragma unroll
            for (int k = 0; k < kSlots; ++k) {
                const int i = iv[k];
                valid[k] = false;
                src[k] = reinterpret_cast<const uint8_t *>(g_zero_row);
                if (i != -1) {
                    bool bad = (i < 0) || ((long long)i >= max_pos);
                    if (!bad) {
                        const int page = __ldg(pt_b + (i >> 6));
                        bad = (page < 0) || ((long long)page >= p.num_pages);
                        if (!bad) {
                            valid[k] = true;
                            src[k] = reinterpret_cast<const uint8_t *>(p.cache) +
                                     ((size_t)page * kPage + (size_t)(i & (kPage - 1))) * kRowBytes;
                        }
                    }
                    if (bad) {
                        atomicOr(&g_status_flags, kFlagIndexRange);
                        atomicAdd(&g_bad_index_count, 1ull);
                    }
                }
            }
        };

        if (n_tiles > 0) resolve(0);
        for (int it = 0; it < n_tiles; ++it) {
            const int stage = it % NSTAGE;
            if (it >= NSTAGE) mbar_wait(&empty[stage], ((it / NSTAGE) - 1) & 1, dead);
            if (lane == 0) mbar_expect_tx(&full[stage], (uint32_t)(NT * kRowBytes));
            __syncwarp();
            uint8_t *dst = smem + C::kOffKV + stage * C::kStageBytes;
            uint64_t mask = 0;
#pragma unroll
            for (int k = 0; k < kSlots; ++k) {
                uint8_t *d = dst + (k * 32 + lane) * kSmemRowBytes;
                if (valid[k])
                    bulk_g2s_hint(d, src[k], kRowBytes, &full[stage], policy);
                else
                    bulk_g2s(d, src[k], kRowBytes, &full[stage]);
                mask |= (uint64_t)__ballot_sync(0xffffffffu, valid[k]) << (32 * k);
            }
            if (lane == 0) {
                hdr[stage] = mask;
                mbar_arrive(&full[stage]);  // release: hdr is visible to the waiters
            }
            if (it + 1 < n_tiles) resolve(it + 1);
        }
        // Copies still in flight must land before the CTA may exit.
        for (int it = (n_tiles > NSTAGE ? n_tiles - NSTAGE : 0); it < n_tiles; ++it)
            mbar_wait(&full[it % NSTAGE], (it / NSTAGE) & 1, dead);
        return;
    }

    // ================================================================ consumers
    const int g = warp >> 2;   // head group
    const int qw = warp & 3;   // quarter: S columns and O columns owned
    const int r0 = lane >> 2;  // fragment row (and r0 + 8)
    const int cq = lane & 3;   // fragment column pair
    constexpr int NTW = NT / 32;  // n8 tiles of S per warp
    const int col0 = qw * (NT / 4);

    float m_run0 = -INFINITY, m_run1 = -INFINITY;
    float l0 = 0.f, l1 = 0.f;
    float oacc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;

    const uint32_t q_base = smem_addr(smem + C::kOffQ) +
                            (16 * g + (lane & 15)) * kSmemRowBytes + (lane >> 4) * 16;
    uint8_t *pbuf = smem + C::kOffP + g * 16 * C::kPStride;
    const uint32_t p_base = smem_addr(pbuf) + (lane & 15) * C::kPStride + (lane >> 4) * 16;
    float *red = reinterpret_cast<float *>(smem + C::kOffRed) + g * 64;
    const uint32_t bar_id = 1 + g;

    mbar_wait(qbar, 0, dead);

    for (int it = 0; it < n_tiles; ++it) {
        const int stage = it % NSTAGE;
        mbar_wait(&full[stage], (it / NSTAGE) & 1, dead);
        const uint64_t vmask = hdr[stage];
        const uint32_t kv = smem_addr(smem + C::kOffKV + stage * C::kStageBytes);

        // ---- S = Q K^T, columns [col0, col0 + NT/4)
        float sacc[NTW][4];
#pragma unroll
        for (int n = 0; n < NTW; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
        uint32_t b_base;
        if (NTW == 2)
            b_base = kv + (col0 + (lane & 7) + ((lane >> 4) << 3)) * kSmemRowBytes +
                     ((lane >> 3) & 1) * 16;
        else
            b_base = kv + (col0 + (lane & 7)) * kSmemRowBytes + ((lane >> 3) & 1) * 16;
#pragma unroll 6
        for (int kk = 0; kk < kD / 16; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(q_base + kk * 32, a0, a1, a2, a3);
            if (NTW == 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b_base + kk * 32, b0, b1, b2, b3);
                mma_bf16_16816(sacc[0], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(sacc[NTW - 1], a0, a1, a2, a3, b2, b3);
            } else {
                uint32_t b0, b1;
                ldsm_x2(b_base + kk * 32, b0, b1);
                mma_bf16_16816(sacc[0], a0, a1, a2, a3, b0, b1);
            }
        }

        // ---- scale into the log2 domain, mask, row max of this warp's columns
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < NTW; ++n) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = col0 + 8 * n + 2 * cq + e;
                const bool ok = (vmask >> col) & 1ull;
                const float v0 = ok ? sacc[n][e] * p.scale_log2 : -INFINITY;
                const float v1 = ok ? sacc[n][2 + e] * p.scale_log2 : -INFINITY;
                sacc[n][e] = v0;
                sacc[n][2 + e] = v1;
                mx0 = fmaxf(mx0, v0);
                mx1 = fmaxf(mx1, v1);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        if (cq == 0) {
            red[qw * 16 + r0] = mx0;
            red[qw * 16 + r0 + 8] = mx1;
        }
        named_bar_sync(bar_id, 128);
        const float t0 = fmaxf(fmaxf(red[r0], red[16 + r0]), fmaxf(red[32 + r0], red[48 + r0]));
        const float t1 = fmaxf(fmaxf(red[8 + r0], red[24 + r0]), fmaxf(red[40 + r0], red[56 + r0]));
        const float mn0 = fmaxf(m_run0, t0);
        const float mn1 = fmaxf(m_run1, t1);
        const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
        const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
        const float al0 = exp2f(m_run0 - mu0);
        const float al1 = exp2f(m_run1 - mu1);
        m_run0 = mn0;
        m_run1 = mn1;

        // ---- P = exp2(s - m), row sums, P -> smem (bf16)
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int n = 0; n < NTW; ++n) {
            const float p00 = exp2f(sacc[n][0] - mu0), p01 = exp2f(sacc[n][1] - mu0);
            const float p10 = exp2f(sacc[n][2] - mu1), p11 = exp2f(sacc[n][3] - mu1);
            ps0 += p00 + p01;
            ps1 += p10 + p11;
            const int col = col0 + 8 * n + 2 * cq;
            *reinterpret_cast<uint32_t *>(pbuf + r0 * C::kPStride + col * 2) = pack_bf16x2(p00, p01);
            *reinterpret_cast<uint32_t *>(pbuf + (r0 + 8) * C::kPStride + col * 2) =
                pack_bf16x2(p10, p11);
        }
        l0 = l0 * al0 + ps0;
        l1 = l1 * al1 + ps1;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            oacc[n][0] *= al0;
            oacc[n][1] *= al0;
            oacc[n][2] *= al1;
            oacc[n][3] *= al1;
        }
        named_bar_sync(bar_id, 128);

        // ---- O[:, qw*128 .. +128] += P C
        const uint32_t v_base = kv + ((lane & 7) + ((lane >> 3) & 1) * 8) * kSmemRowBytes +
                                (qw * 128 + (lane >> 4) * 8) * 2;
#pragma unroll
        for (int kk = 0; kk < NT / 16; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(p_base + kk * 32, a0, a1, a2, a3);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(v_base + kk * 16 * kSmemRowBytes + np * 32, b0, b1, b2, b3);
                mma_bf16_16816(oacc[2 * np], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(oacc[2 * np + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
    }

    // ---- epilogue: full row sums, then partial (or final) outputs
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float *lred = reinterpret_cast<float *>(smem + C::kOffL) + g * 64;
    if (cq == 0) {
        lred[qw * 16 + r0] = l0;
        lred[qw * 16 + r0 + 8] = l1;
    }
    named_bar_sync(bar_id, 128);
    const float lt0 = lred[r0] + lred[16 + r0] + lred[32 + r0] + lred[48 + r0];
    const float lt1 = lred[8 + r0] + lred[24 + r0] + lred[40 + r0] + lred[56 + r0];

#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int h = 16 * g + r0 + 8 * half;
        if (h >= p.H) continue;
        const float lt = half ? lt1 : lt0;
        const float mr = half ? m_run1 : m_run0;
        const size_t row = (size_t)bt * p.H + h;
        if (!DIRECT) {
            float *dst = p.part_o + (row * p.nsplit + s) * kDc + qw * 128 + 2 * cq;
#pragma unroll
            for (int n = 0; n < 16; ++n)
                *reinterpret_cast<float2 *>(dst + 8 * n) =
                    make_float2(oacc[n][2 * half], oacc[n][2 * half + 1]);
            if (qw == 0 && cq == 0) {
                const size_t k = row * p.nsplit + s;
                p.part_m[k] = (lt > 0.f) ? mr * kLn2 : -INFINITY;
                p.part_lse[k] = (lt > 0.f) ? (mr + log2f(lt)) * kLn2 : -INFINITY;
            }
        } else {
            const float inv = (lt > 0.f) ? 1.f / lt : 0.f;
            __nv_bfloat16 *dst = p.o + row * kDc + qw * 128 + 2 * cq;
#pragma unroll
            for (int n = 0; n < 16; ++n)
                *reinterpret_cast<uint32_t *>(dst + 8 * n) =
                    pack_bf16x2(oacc[n][2 * half] * inv, oacc[n][2 * half + 1] * inv);
            if (qw == 0 && cq == 0) p.lse[row] = (lt > 0.f) ? (mr + log2f(lt)) * kLn2 : -INFINITY;
        }
    }
}

}  // namespace smla
