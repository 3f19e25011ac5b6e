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
// CTA is what keeps the pass at one HBM read per selected row.  Under the
// balanced schedule of the whole decode a CTA instead takes an equal run of
// 32-row tiles that may span two tokens; it walks those pieces (work items)
// in order, one partial slot per piece.
//
// Warp roles (HG = head groups of 16 rows, the mma M dimension):
//   warps 4*HG,    producers: every thread of the CTA first resolves the
//   4*HG+1         split's index entries to physical rows (index loads, then
//                  page-table loads, a batch in flight at once) into shared
//                  memory; then both producer warps issue every tile (one
//                  the rows of even slots, the other the odd ones), one 1-D
//                  bulk async copy (TMA engine, 1152 B) per row into a ring of
//                  NSTAGE tiles of NT rows, each tile completing on an
//                  mbarrier that counts both warps and their bytes.
//   warps 0..4HG-1 consumers, 4 per head group.  Each warp keeps the Q
//                  fragments of one quarter of the 576 dims in registers and
//                  computes that quarter's partial S = Q K^T for all NT rows
//                  of a tile (independent accumulators per n8 tile); the four
//                  partials meet once per tile in shared memory (double
//                  buffered: one named barrier per tile).  Every warp then
//                  holds the full S of its 16 heads, runs the masked online
//                  softmax in fp32 (exp2 domain, quad shuffles), turns P into
//                  A fragments in registers and accumulates O += P C for its
//                  128 of the 512 output columns in fp32 registers.
// Shared-memory rows are 1168 B apart (1152 + 16) so that the 8 row addresses
// of every ldmatrix phase fall in distinct 16-byte bank groups.
//
// Every partial kernel is launched as a programmatic dependent of what
// precedes it on the stream and waits (griddepcontrol.wait) before its first
// global access.  Its inputs (q, the indices, the page table) may therefore
// be written by the predecessor while this grid is already resident, so they
// are read with weak global loads (ld_input), which the wait makes see the
// predecessor's writes, never through the read-only path, whose contract is
// that the data stays unchanged for the kernel's lifetime.
// The cache rows arrive by cp.async.cg, bulk or tensor copies (all through L2).
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
constexpr int kResolveChunk = 2048;  // index entries resolved to rows ahead of the copies

// Sources of the bulk copies for padding slots: rows of zeros, so that masked
// slots hold finite values (their probability is 0, and 0 * finite = 0).
// Slot s of a tile copies zero row s: thousands of CTAs copying one shared row
// at once serialised on its few L2 lines.  (The cp.async gathers zero-fill
// padding slots without reading memory at all.)
constexpr int kZeroRows = 32;
__device__ __align__(128) uint16_t g_zero_rows[kZeroRows][kD];

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
    __nv_bfloat16 *o;             // direct mode (nsplit = 1): [B, T, H, 512]
    float *lse;                   // direct mode (nsplit = 1): [B, T, H]
    // Balanced schedule (pipelined kernels, whole decode only): CTA c of
    // `grid` takes tiles [c U / grid, (c+1) U / grid) of the flattened
    // (query token, 32-row tile) space, U = B T tpt.  0 = equal splits of kc.
    int balanced;
    int tpt;                      // 32-row tiles per query token, ceil(K / 32)
    int grid;
    long long n_units;            // U
    // Dense-context variant (tcgen05 kernel only; idx unused): query token
    // (b, t) attends to list entries [0, seq_lens[b * dense_t + t]), entry j
    // being position j.  Unit bt = b * T + g packs query tokens
    // [g * pack, min(dense_t, (g + 1) * pack)) of sequence b, dense_h heads
    // each, into the MMA's M rows (pack * dense_h <= 64).
    const int *seq_lens;          // [B, dense_t]; nullptr = sparse index lists
    int pack, dense_t, dense_h;
};

// One piece of a CTA's work: rows [j0, j1) of query token bt, written as
// partial slot `slot`.  `last`: the piece ends the token (balanced schedule),
// so its CTA also marks the token's unused slots empty.
struct WorkItem {
    int bt, j0, j1, slot;
    bool last;
};

// CTA that owns flattened tile u under the balanced schedule: the c with
// floor(c U / G) <= u < floor((c+1) U / G).
__device__ __forceinline__ int owner_cta(const PartialParams &p, long long u) {
    return (int)(((u + 1) * p.grid - 1) / p.n_units);
}

// Iterates the items of CTA c: start with u = item_begin(p, c).  Equal splits
// give one item, split s = c % nsplit of token c / nsplit.
__device__ __forceinline__ long long item_begin(const PartialParams &p, int c) {
    return p.balanced ? (long long)c * p.n_units / p.grid : 0;
}
__device__ __forceinline__ bool next_item(const PartialParams &p, int c, long long &u, WorkItem &w) {
    if (!p.balanced) {
        if (u != 0) return false;
        u = 1;
        const int s = c % p.nsplit;
        const long long j0 = (long long)s * p.kc;
        w.bt = c / p.nsplit;
        w.j0 = (int)(j0 < p.K ? j0 : p.K);
        w.j1 = (int)(j0 + p.kc < p.K ? j0 + p.kc : p.K);
        w.slot = s;
        w.last = false;
        return true;
    }
    const long long u_end = (long long)(c + 1) * p.n_units / p.grid;
    if (u >= u_end) return false;
    const long long bt = u / p.tpt;
    const long long tok_end = (bt + 1) * p.tpt;
    const long long ue = u_end < tok_end ? u_end : tok_end;
    w.bt = (int)bt;
    w.j0 = (int)((u - bt * p.tpt) * 32);
    const long long j1 = (ue - bt * p.tpt) * 32;
    w.j1 = (int)(j1 < p.K ? j1 : p.K);
    w.slot = c - owner_cta(p, bt * p.tpt);
    w.last = ue == tok_end;
    u = ue;
    return true;
}

// Balanced schedule: the CTA holding a token's last rows marks the slots no
// CTA wrote for that token (slot + 1 .. nsplit - 1) as empty, m = lse = -inf;
// the combine gives them weight 0 without reading their part_o.
__device__ __forceinline__ void mark_unused_slots(const PartialParams &p, const WorkItem &w, int tid,
                                                  int nthreads) {
    const int spare = p.nsplit - 1 - w.slot;
    if (!w.last || spare <= 0) return;
    for (int i = tid; i < p.H * spare; i += nthreads) {
        const size_t k = ((size_t)w.bt * p.H + i / spare) * p.nsplit + w.slot + 1 + i % spare;
        p.part_m[k] = -INFINITY;
        p.part_lse[k] = -INFINITY;
    }
}

// Index entries [j0 + base, j0 + base + n) of query token bt -> physical rows
// in rows_s[0, n) (-1 = masked), resolved by threads tid, tid + nthreads, ...
// of the caller with every load of a batch in flight at once.  Entries other
// than -1 that are out of range are counted.
template <int BATCH>
__device__ __forceinline__ void resolve_rows(const PartialParams &p, int bt, int j0, int base, int n,
                                             int *rows_s, int tid, int nthreads) {
    const int *idx_bt = p.idx + (size_t)bt * p.K + j0 + base;
    const int *pt_b = p.page_table + (size_t)(bt / p.T) * p.pt_stride;
    const long long max_pos = (long long)p.pt_stride * kPage;
    for (int b0 = 0; b0 < n; b0 += nthreads * BATCH) {
        int iv[BATCH];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int j = b0 + k * nthreads + tid;
            iv[k] = (j < n) ? ld_input(idx_bt + j) : -1;
        }
        int pg[BATCH];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int i = iv[k];
            pg[k] = (i >= 0 && (long long)i < max_pos) ? ld_input(pt_b + (i >> 6)) : -1;
        }
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int j = b0 + k * nthreads + tid;
            const int i = iv[k];
            int row = -1;
            if (i != -1) {
                const bool ok = (i >= 0) && ((long long)i < max_pos) && (pg[k] >= 0) &&
                                ((long long)pg[k] < p.num_pages);
                if (ok) {
                    row = pg[k] * kPage + (i & (kPage - 1));
                } else if (j < n) {
                    atomicOr(&g_status_flags, kFlagIndexRange);
                    atomicAdd(&g_bad_index_count, 1ull);
                }
            }
            if (j < n) rows_s[j] = row;
        }
    }
}

template <int HG, int NT, int NSTAGE>
struct MmaCfg {
    static_assert(NT == 16 || NT == 32 || NT == 64, "tile rows");
    static constexpr int kHeads = 16 * HG;
    static constexpr int kComputeWarps = 4 * HG;
    // Two producer warps share every tile's rows (slot s by warp s % 2): one
    // warp issues only about 22 GB/s of 1-D bulk copies, so a tile issued by
    // both lands in about half the time, and two per CTA (four per SM) keep
    // the TMA engine near the HBM rate.
    static constexpr int kProducerWarps = 2;
    static constexpr int kThreads = (kComputeWarps + kProducerWarps) * 32;
    static constexpr int kSRow = NT + 8;  // floats per S-partial row (32-byte pad: conflict-free float2)
    static constexpr int kStageBytes = NT * kSmemRowBytes;
    static constexpr int kQBytes = kHeads * kSmemRowBytes;
    static constexpr int kSPartBytes = HG * 2 * 4 * 16 * kSRow * 4;
    static constexpr int kOffQ = 0;  // Q rows, then (after Q is in registers) the S partials
    static constexpr int kOffKV = kOffQ + ((kQBytes > kSPartBytes ? kQBytes : kSPartBytes) + 127) / 128 * 128;
    static constexpr int kOffHdr = kOffKV + NSTAGE * kStageBytes;  // u64 [NSTAGE]
    static constexpr int kOffBar = kOffHdr + NSTAGE * 8;            // u64 full[], empty[]
    static constexpr int kOffRows = kOffBar + 2 * NSTAGE * 8;       // int [kResolveChunk]
    static constexpr int kSmemBytes = kOffRows + kResolveChunk * 4;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    // CTAs per SM the launch bounds ask for: two when a pair fits (more
    // producers per SM keep more row gathers in flight).
    static constexpr int kMinBlocks = (2 * (kSmemBytes + 1024) <= 233472 && kThreads <= 192) ? 2 : 1;
};

// Per-thread state and work of one consumer warp (4 warps per head group of
// 16 heads).  Each warp keeps the Q fragments of one quarter of the 576 dims
// in registers and computes that quarter's partial S for all NT rows of a tile
// (independent accumulators per n8 tile); the four partials meet once per tile
// in shared memory.  Every warp then holds the full S of its 16 heads, runs the
// masked online softmax in fp32 (exp2 domain, quad shuffles), turns P into A
// fragments in registers and accumulates O += P C for its 128 of the 512
// output columns in fp32 registers.
template <int NT, int HG>
struct MmaConsumer {
    static constexpr int NTS = NT / 8;          // n8 tiles of S (all NT columns)
    static constexpr int KQ = kD / 16 / 4;      // k16 steps of S per warp (9)
    static constexpr int kSRow = NT + 8;        // floats per S-partial row (32-B pad)
    int g, qw, lane, r0, cq;
    uint32_t qa[KQ][4];
    float oacc[16][4];
    float m_run0, m_run1, l0, l1;

    __device__ __forceinline__ void init(int warp, int lane_) {
        g = warp >> 2;     // head group
        qw = warp & 3;     // quarter: k range of S, and 128 output columns
        lane = lane_;
        r0 = lane >> 2;    // fragment row (and r0 + 8)
        cq = lane & 3;     // fragment column pair
        m_run0 = m_run1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int n = 0; n < 16; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
    }

    // This warp's 16 heads x 144 dims of Q with plain 16-byte loads (rows beyond
    // H are zero), parked in shared memory (rows 1168 B apart) and ldmatrix-ed
    // into A fragments.
    __device__ __forceinline__ void load_q(uint8_t *q_smem, const PartialParams &p, int bt) {
        const uint4 *qsrc = reinterpret_cast<const uint4 *>(p.q + (size_t)bt * p.H * kD);
        uint4 qv[9];
#pragma unroll
        for (int i = 0; i < 9; ++i) {
            const int c = lane + 32 * i;  // 16 rows x 18 chunks of 8 dims
            const int h = 16 * g + c / 18;
            qv[i] = (h < p.H) ? ld_input(qsrc + (size_t)h * (kD / 8) + KQ * 2 * qw + c % 18)
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 9; ++i) {
            const int c = lane + 32 * i;
            *reinterpret_cast<uint4 *>(q_smem + (16 * g + c / 18) * kSmemRowBytes +
                                       (KQ * 2 * qw + c % 18) * 16) = qv[i];
        }
        __syncwarp();
        const uint32_t q_base =
            smem_addr(q_smem) + (16 * g + (lane & 15)) * kSmemRowBytes + (lane >> 4) * 16;
#pragma unroll
        for (int kk = 0; kk < KQ; ++kk)
            ldsm_x4(q_base + (KQ * qw + kk) * 32, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
    }

    // One tile of NT rows (1168-B rows at shared address kv); vmask bit j = row j
    // valid; sp = this group's S-partial buffer for the tile (double buffered by
    // the caller so one named barrier per tile suffices).
    __device__ __forceinline__ void tile(uint32_t kv, uint64_t vmask, float *sp, float scale_log2) {
        // ---- partial S = Q K^T over this warp's 144 dims, all NT columns
        float sacc[NTS][4];
#pragma unroll
        for (int n = 0; n < NTS; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
        const uint32_t b_base = kv + ((lane & 7) + ((lane >> 4) << 3)) * kSmemRowBytes +
                                ((lane >> 3) & 1) * 16 + KQ * qw * 32;
#pragma unroll
        for (int kk = 0; kk < KQ; ++kk) {
#pragma unroll
            for (int np = 0; np < NTS / 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b_base + np * 16 * kSmemRowBytes + kk * 32, b0, b1, b2, b3);
                mma_bf16_16816(sacc[2 * np], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
                mma_bf16_16816(sacc[2 * np + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
            }
        }
#pragma unroll
        for (int n = 0; n < NTS; ++n) {
            float *d = sp + qw * 16 * kSRow + 8 * n + 2 * cq;
            *reinterpret_cast<float2 *>(d + r0 * kSRow) = make_float2(sacc[n][0], sacc[n][1]);
            *reinterpret_cast<float2 *>(d + (r0 + 8) * kSRow) = make_float2(sacc[n][2], sacc[n][3]);
        }
        named_bar_sync(1 + g, 128);

        // ---- full S (sum of the four k quarters), scaled to log2 units, masked
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < NTS; ++n) {
            float2 a = make_float2(0.f, 0.f), c = make_float2(0.f, 0.f);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float *src = sp + w * 16 * kSRow + 8 * n + 2 * cq;
                const float2 x = *reinterpret_cast<const float2 *>(src + r0 * kSRow);
                const float2 y = *reinterpret_cast<const float2 *>(src + (r0 + 8) * kSRow);
                a.x += x.x;
                a.y += x.y;
                c.x += y.x;
                c.y += y.y;
            }
            const int col = 8 * n + 2 * cq;
            const bool ok0 = (vmask >> col) & 1ull, ok1 = (vmask >> (col + 1)) & 1ull;
            sacc[n][0] = ok0 ? a.x * scale_log2 : -INFINITY;
            sacc[n][1] = ok1 ? a.y * scale_log2 : -INFINITY;
            sacc[n][2] = ok0 ? c.x * scale_log2 : -INFINITY;
            sacc[n][3] = ok1 ? c.y * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(sacc[n][0], sacc[n][1]));
            mx1 = fmaxf(mx1, fmaxf(sacc[n][2], sacc[n][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m_run0, mx0);
        const float mn1 = fmaxf(m_run1, mx1);
        const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0;
        const float mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
        const float al0 = fast_exp2(m_run0 - mu0);
        const float al1 = fast_exp2(m_run1 - mu1);
        m_run0 = mn0;
        m_run1 = mn1;

        // ---- P = exp2(s - m) straight into A fragments (k16 step j = n8 tiles 2j, 2j+1)
        uint32_t pa[NT / 16][4];
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int n = 0; n < NTS; ++n) {
            const float p00 = fast_exp2(sacc[n][0] - mu0), p01 = fast_exp2(sacc[n][1] - mu0);
            const float p10 = fast_exp2(sacc[n][2] - mu1), p11 = fast_exp2(sacc[n][3] - mu1);
            ps0 += p00 + p01;
            ps1 += p10 + p11;
            pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(p00, p01);
            pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p10, p11);
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

        // ---- O[:, qw*128 .. +128] += P C
        const uint32_t v_base = kv + ((lane & 7) + ((lane >> 3) & 1) * 8) * kSmemRowBytes +
                                (qw * 128 + (lane >> 4) * 8) * 2;
#pragma unroll
        for (int j = 0; j < NT / 16; ++j) {
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(v_base + j * 16 * kSmemRowBytes + np * 32, b0, b1, b2, b3);
                mma_bf16_16816(oacc[2 * np], pa[j][0], pa[j][1], pa[j][2], pa[j][3], b0, b1);
                mma_bf16_16816(oacc[2 * np + 1], pa[j][0], pa[j][1], pa[j][2], pa[j][3], b2, b3);
            }
        }
    }

    // Row sums (every warp of the group holds the same full sums), then the
    // unnormalised partial with m and lse, or (DIRECT) the final o and lse.
    template <bool DIRECT>
    __device__ __forceinline__ void epilogue(const PartialParams &p, int bt, int s) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int h = 16 * g + r0 + 8 * half;
            if (h >= p.H) continue;
            const float lt = half ? l1 : l0;
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
                if (qw == 0 && cq == 0)
                    p.lse[row] = (lt > 0.f) ? (mr + log2f(lt)) * kLn2 : -INFINITY;
            }
        }
    }
};

template <int HG, int NT, int NSTAGE, bool DIRECT>
__global__ void __launch_bounds__(MmaCfg<HG, NT, NSTAGE>::kThreads, MmaCfg<HG, NT, NSTAGE>::kMinBlocks)
    smla_partial_mma_kernel(const PartialParams p) {
    using C = MmaCfg<HG, NT, NSTAGE>;
    static_assert(NT == 32, "the balanced schedule counts 32-row tiles");
    static_assert(NSTAGE % 2 == 0, "the two producer warps own alternate stages");
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    bool dead = false;  // set once a bounded wait of this thread has timed out

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty = full + NSTAGE;
    volatile uint64_t *hdr = reinterpret_cast<volatile uint64_t *>(smem + C::kOffHdr);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&full[i], C::kProducerWarps);  // one arrival (+ its bytes) per producer warp
            mbar_init(&empty[i], C::kComputeWarps);
        }
        fence_mbar_init();
    }
    // The combine kernel is launched as a programmatic dependent: let it be
    // scheduled now; it waits for this grid's completion before reading.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // This grid is itself a programmatic dependent of what precedes it on the
    // stream: wait for that to complete before the first global access.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Every thread helps resolve the first chunk of the first item, so that
    // the first copies start after two memory round trips (one warp alone
    // took several microseconds for a 512-entry split).
    int *rows_s0 = reinterpret_cast<int *>(smem + C::kOffRows);
    {
        long long u0 = item_begin(p, cta);
        WorkItem w0;
        if (next_item(p, cta, u0, w0))
            resolve_rows<4>(p, w0.bt, w0.j0, 0, min(kResolveChunk, w0.j1 - w0.j0), rows_s0,
                            threadIdx.x, C::kThreads);
    }
    __syncthreads();

    if (warp >= C::kComputeWarps) {
        // ============================================================ producers
        const int pw = warp - C::kComputeWarps;  // issues the rows of slots s with s % 2 == pw
        const uint32_t bar_prod = 2 + HG;        // named barrier of the producer warps
        const uint64_t policy = l2_policy_evict_first();
        int *rows_s = reinterpret_cast<int *>(smem + C::kOffRows);
        constexpr int kResolveBatch = HG <= 2 ? 16 : 8;  // loads in flight per lane
        int it = 0;  // tile counter over all of this CTA's items (ring position)
        long long u = item_begin(p, cta);
        WorkItem w;
        bool first_chunk = true;  // resolved by the whole CTA above
        while (next_item(p, cta, u, w)) {
            const int len = w.j1 - w.j0;
            for (int base = 0; base < len; base += kResolveChunk) {
                const int n = min(kResolveChunk, len - base);
                // Resolve the whole chunk before its first copy: index loads,
                // then page-table loads, a batch per lane in flight at once.
                if (!first_chunk) {
                    named_bar_sync(bar_prod, 32 * C::kProducerWarps);  // rows_s free for rewriting
                    resolve_rows<kResolveBatch>(p, w.bt, w.j0, base, n, rows_s, 32 * pw + lane,
                                                32 * C::kProducerWarps);
                    named_bar_sync(bar_prod, 32 * C::kProducerWarps);  // rows_s complete
                }
                first_chunk = false;
                // Issue one bulk copy per row (or per padding slot, from its zero row).
                const int chunk_tiles = (n + NT - 1) / NT;
                for (int t = 0; t < chunk_tiles; ++t, ++it) {
                    const int stage = it % NSTAGE;
                    if (it >= NSTAGE) mbar_wait(&empty[stage], ((it / NSTAGE) - 1) & 1, dead);
                    constexpr int kMine = (NT - 1) / C::kProducerWarps + 1;  // slots per warp (NT even)
                    if (lane == 0) mbar_expect_tx(&full[stage], (uint32_t)(kMine * kRowBytes));
                    __syncwarp();
                    uint8_t *dst = smem + C::kOffKV + stage * C::kStageBytes;
                    uint64_t mask = 0;
#pragma unroll
                    for (int k = 0; k < (NT + 31) / 32; ++k) {
                        const int slot = k * 32 + lane;
                        const int r = t * NT + slot;
                        const int row = (slot < NT && r < n) ? rows_s[r] : -1;
                        uint8_t *d = dst + slot * kSmemRowBytes;
                        if (slot < NT && slot % C::kProducerWarps == pw) {
                            if (row >= 0)
                                bulk_g2s_hint(d, reinterpret_cast<const uint8_t *>(p.cache) +
                                                     (size_t)row * kRowBytes,
                                              kRowBytes, &full[stage], policy);
                            else
                                bulk_g2s(d, g_zero_rows[slot % kZeroRows], kRowBytes, &full[stage]);
                        }
                        mask |= (uint64_t)__ballot_sync(0xffffffffu, row >= 0) << (32 * k);
                    }
                    if (lane == 0) {
                        if (pw == 0) hdr[stage] = mask;
                        mbar_arrive(&full[stage]);  // release: hdr is visible to the waiters
                    }
                }
            }
        }
        // Copies still in flight must land before the CTA may exit.
        for (int k = (it > NSTAGE ? it - NSTAGE : 0); k < it; ++k)
            mbar_wait(&full[k % NSTAGE], (k / NSTAGE) & 1, dead);
        return;
    }

    // ================================================================ consumers
    // The Q region doubles as the split-k score exchange of every head group
    // (a group's exchange buffer overlaps the next group's Q rows), so Q is
    // (re)written only when all consumer warps are past their last exchange.
    float *spart_base = reinterpret_cast<float *>(smem + C::kOffQ);
    int it = 0;
    long long u = item_begin(p, cta);
    WorkItem w;
    bool first = true;
    while (next_item(p, cta, u, w)) {
        MmaConsumer<NT, HG> cons;
        cons.init(warp, lane);
        if (!first) named_bar_sync(1 + HG, 128 * HG);
        first = false;
        cons.load_q(smem + C::kOffQ, p, w.bt);
        named_bar_sync(1 + HG, 128 * HG);  // Q is in registers: the region is free
        float *spart = spart_base + cons.g * 2 * 4 * 16 * C::kSRow;
        const int n_tiles = (w.j1 - w.j0 + NT - 1) / NT;
        for (int t = 0; t < n_tiles; ++t, ++it) {
            const int stage = it % NSTAGE;
            mbar_wait(&full[stage], (it / NSTAGE) & 1, dead);
            cons.tile(smem_addr(smem + C::kOffKV + stage * C::kStageBytes), hdr[stage],
                      spart + (it & 1) * 4 * 16 * C::kSRow, p.scale_log2);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
        }
        cons.template epilogue<DIRECT>(p, w.bt, w.slot);
        if (!DIRECT && warp < 4) mark_unused_slots(p, w, threadIdx.x, 128);
    }
}

// ----------------------------------------------------------------------------
// Latency path: a split of at most 32 rows (one tile), as in single-request
// decode with a large NSPLIT.  There the pipelined kernel's chain -- index
// load, then page-table load, then 32 TMA row copies issued one after another,
// then the math -- is the whole cost.  This kernel instead loads the
// sequence's entire page-table row together with the indices and Q (one
// memory round trip), resolves the rows from shared memory, gathers the tile
// with 16-byte cp.async copies issued by every thread (one more round trip,
// no serial TMA queue) and runs the same consumer math on it.
constexpr int kSmallMaxPt = 8192;  // page-table entries kept in shared memory
constexpr int kSmallMaxRows = 64;  // rows per split the latency form takes


template <int HG, int TILES>
struct SmallCfg {
    static_assert(TILES == 1 || TILES == 2, "one or two 32-row tiles per split");
    static constexpr int NT = 32;
    static constexpr int kThreads = 128 * HG;
    static constexpr int kQBytes = 16 * HG * kSmemRowBytes;
    static constexpr int kSPartBytes = HG * 2 * 4 * 16 * (NT + 8) * 4;
    static constexpr int kOffQ = 0;  // Q rows, then the S partials
    static constexpr int kOffKV = ((kQBytes > kSPartBytes ? kQBytes : kSPartBytes) + 127) / 128 * 128;
    static constexpr int kOffRows = kOffKV + TILES * NT * kSmemRowBytes;  // int [32 TILES] rows, masks
    static constexpr int kOffPt = kOffRows + (NT + 4) * TILES * 4;      // int [pt_stride]
    static constexpr int kMaxSmemBytes = kOffPt + kSmallMaxPt * 4;
    static int smem_bytes(int pt_stride) { return kOffPt + pt_stride * 4; }
};

// TILES: 32-row tiles per split (a split of up to 64 rows still takes one
// round trip for its rows: both tiles are gathered at once).
template <int HG, int TILES, bool DIRECT>
__global__ void __launch_bounds__(SmallCfg<HG, TILES>::kThreads)
    smla_partial_small_kernel(const PartialParams p) {
    using C = SmallCfg<HG, TILES>;
    constexpr int NT = C::NT;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tid = threadIdx.x;
    const int unit = blockIdx.x;  // (b * T + t) * S + s
    const int s = unit % p.nsplit;
    const int bt = unit / p.nsplit;
    const int b = bt / p.T;
    const long long j0l = (long long)s * p.kc;
    const int j0 = (int)(j0l < p.K ? j0l : p.K);
    const int j1 = (int)((long long)j0 + p.kc < p.K ? (long long)j0 + p.kc : p.K);
    int *rows_s = reinterpret_cast<int *>(smem + C::kOffRows);  // [TILES * 32] rows, then masks
    int *pt_s = reinterpret_cast<int *>(smem + C::kOffPt);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // launched as a programmatic dependent: the predecessor on the stream
    // completes before the first global access
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // 1. page-table row, this split's indices and Q: all loads in flight at once
    const int *pt_b = p.page_table + (size_t)b * p.pt_stride;
    for (int i0 = 0; i0 < p.pt_stride; i0 += C::kThreads * 8) {
        int v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + k * C::kThreads + tid;
            v[k] = (i < p.pt_stride) ? ld_input(pt_b + i) : -1;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + k * C::kThreads + tid;
            if (i < p.pt_stride) pt_s[i] = v[k];
        }
    }
    int my_idx = -1;
    if (tid < NT * TILES && j0 + tid < j1) my_idx = ld_input(p.idx + (size_t)bt * p.K + j0 + tid);
    MmaConsumer<NT, HG> cons;
    cons.init(warp, lane);
    cons.load_q(smem + C::kOffQ, p, bt);
    __syncthreads();

    // 2. rows of tile w (warp w); out-of-range entries are masked and counted
    if (warp < TILES) {
        const int i = my_idx;
        int row = -1;
        if (i != -1) {
            const long long max_pos = (long long)p.pt_stride * kPage;
            bool ok = (i >= 0) && ((long long)i < max_pos);
            const int pg = ok ? pt_s[i >> 6] : -1;
            ok = ok && (pg >= 0) && ((long long)pg < p.num_pages);
            if (ok) {
                row = pg * kPage + (i & (kPage - 1));
            } else {
                atomicOr(&g_status_flags, kFlagIndexRange);
                atomicAdd(&g_bad_index_count, 1ull);
            }
        }
        rows_s[warp * NT + lane] = row;
        const uint32_t m = __ballot_sync(0xffffffffu, row >= 0);
        if (lane == 0) rows_s[NT * TILES + warp] = (int)m;
    }
    __syncthreads();

    // 3. gather: TILES x 32 rows x 72 chunks of 16 B, cp.async from every thread
    // Padding slots (no row) are zero-filled by the copy itself (source size
    // 0: nothing is read), so that they hold finite values.
    const uint8_t *cache = reinterpret_cast<const uint8_t *>(p.cache);
    uint8_t *kv = smem + C::kOffKV;
    for (int c = tid; c < TILES * NT * 72; c += C::kThreads) {
        const int r = c / 72, k = c - 72 * (c / 72);
        const int row = rows_s[r];
        const uint8_t *src = cache + (size_t)(row >= 0 ? row : 0) * kRowBytes + k * 16;
        const uint32_t nbytes = row >= 0 ? 16u : 0u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         smem_addr(kv + r * kSmemRowBytes + k * 16)),
                     "l"(src), "r"(nbytes)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    // 4. the tiles and the epilogue (the Q region now holds the S partials,
    //    double buffered by tile)
    float *spart = reinterpret_cast<float *>(smem + C::kOffQ) + cons.g * 2 * 4 * 16 * (NT + 8);
#pragma unroll
    for (int t = 0; t < TILES; ++t)
        cons.tile(smem_addr(kv + t * NT * kSmemRowBytes), (uint32_t)rows_s[NT * TILES + t],
                  spart + (t & 1) * 4 * 16 * (NT + 8), p.scale_log2);
    cons.template epilogue<DIRECT>(p, bt, s);
}

}  // namespace smla
