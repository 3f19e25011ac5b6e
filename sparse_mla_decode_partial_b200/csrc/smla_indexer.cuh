// smla_indexer.cuh -- the top-k indexer that produces the decode's index
// lists: index scores on the 5th-generation tensor core, then a per-token
// radix selection.
//
// "The Negative Result That Refined the Hunt: Disabling the MMA FlashMLA
// Kernel", section "The Context: A Systematic Bisection Campaign": an indexer
// kernel and a bf16 index-key path run ahead of the sparse decode kernel,
// which attends over the top-k candidate tokens ("The Moment of Truth ...",
// section "The Split-K Imperative").  The pages give no formula; the
// published DeepSeek sparse-attention indexer is the reading:
//     I[s] = sum_j w[j] * max(0, qI[j] . kI[row(s)])          (128-wide keys)
// and the selection is the min(K, n) largest scores over the visible
// positions [0, n), equal scores going to the smaller position, written as
// ascending positions then -1.
//
// Scores (smla_ix_score_kernel): one persistent CTA per SM walks an equal
// share of the (query token, 128-key tile) units.  A tile is two 64-key pages
// of the index-key cache, each moved by two TMA tile loads (64 keys x 64
// values, 128B swizzle) straight into the K-major layout of the MMA's A
// operand: the KEYS are M = 128, the index heads N (16, 32 or 64), K = 128
// (8 k-steps), so the accumulator holds one key per TMEM lane and the
// epilogue thread that owns a key reduces over its heads without talking to
// any other thread.  Warp roles: warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer, warps 4-7 epilogue (TMEM lanes 0-127).
// Selection (smla_ix_select_kernel): one CTA per query token; three radix
// passes (11, 11, 10 bits) over an order-preserving key of the fp32 score
// find the K-th largest score, then one ascending scan writes the positions
// above it and the first ones (by position) equal to it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "smla_tc_ptx.cuh"

namespace smla {

constexpr int kIxDim = 128;        // index-key width (bf16 values)
constexpr int kIxTile = 128;       // keys per unit: the MMA's M
constexpr int kIxMaxHeads = 64;    // index heads: the MMA's N (padded to 16, 32, 64)
constexpr int kIxStages = 4;       // key tiles in flight per CTA
constexpr int kIxSelectThreads = 1024;

struct IndexerParams {
    const int *page_table;   // [B, pt_stride]
    int pt_stride;
    long long num_pages;
    const int *n_vis;        // [B * T] visible positions of each query token
    const float *w;          // [B * T, HI] head weights
    int BT, T, HI, max_n, K;
    int *tile_start;         // [B * T + 1]: first unit of each token; [B * T] = all units
    float *scores;           // [B * T, score_stride]; NaN = not a candidate
    long long score_stride;
    int *out;                // [B * T, K]
};

// Visible positions of token u, clamped to [0, max_n].
__device__ __forceinline__ int ix_visible(const IndexerParams &p, int u) {
    return min(max(__ldg(p.n_vis + u), 0), p.max_n);
}

// ---------------------------------------------------------------- block scan (1024 threads)
// Inclusive sum over the block; *total receives the block's sum.  Every
// thread must call it; scratch holds 33 ints.
__device__ __forceinline__ int ix_block_scan(int v, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
    }
    if (lane == 31) scratch[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int x = lane < nwarps ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        scratch[lane] = x;  // inclusive warp totals
    }
    __syncthreads();
    if (warp > 0) v += scratch[warp - 1];
    *total = scratch[nwarps - 1];
    __syncthreads();  // scratch may be reused at once
    return v;
}

// ---------------------------------------------------------------- plan
// Units of work: token u has ceil(n_u / 128) key tiles; tile_start is their
// exclusive prefix sum.  A length outside [0, max_n] is clamped and counted.
__global__ void __launch_bounds__(1024) smla_ix_plan_kernel(const IndexerParams p) {
    __shared__ int scratch[33];
    int carry = 0;
    for (int base = 0; base < p.BT; base += blockDim.x) {
        const int u = base + threadIdx.x;
        int tiles = 0;
        if (u < p.BT) {
            const int raw = __ldg(p.n_vis + u);
            if (raw < 0 || raw > p.max_n) {
                atomicOr(&g_status_flags, kFlagIndexRange);
                atomicAdd(&g_bad_index_count, 1ull);
            }
            tiles = (min(max(raw, 0), p.max_n) + kIxTile - 1) / kIxTile;
        }
        int total;
        const int incl = ix_block_scan(tiles, scratch, &total);
        if (u < p.BT) p.tile_start[u] = carry + incl - tiles;
        carry += total;
    }
    if (threadIdx.x == 0) p.tile_start[p.BT] = carry;
}

// Token holding unit `unit` (tile_start ascending; tokens with no tile skipped).
__device__ __forceinline__ int ix_token_of(const IndexerParams &p, long long unit) {
    int lo = 0, hi = p.BT - 1;  // the last token with tile_start <= unit
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.tile_start + mid) <= unit) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------- TMA (tiled, no multicast)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 32 lanes x N consecutive 32-bit columns (N = 16, 32 or 64): thread i gets lane (base + i).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld32(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_cols<64>(uint32_t taddr, uint32_t (&r)[64]) {
    uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
    uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
    tmem_ld32(taddr, lo);
    tmem_ld32(taddr + 32, hi);
}

// ---------------------------------------------------------------- scores
template <int NPAD>
struct IxCfg {
    static_assert(NPAD == 16 || NPAD == 32 || NPAD == 64, "index heads per MMA");
    static constexpr int kThreads = 256;
    static constexpr int kBoxBytes = kIxTile * 128;        // 128 keys x 64 values
    static constexpr int kStageBytes = 2 * kBoxBytes;      // 32 KB: the tile's two 64-value boxes
    static constexpr int kQBoxBytes = NPAD * 128;
    static constexpr int kQBytes = 2 * kQBoxBytes;
    static constexpr int kOffStages = 0;
    static constexpr int kOffQ = kIxStages * kStageBytes;   // two query slots
    static constexpr int kOffBar = kOffQ + 2 * kQBytes;
    // full[S], empty[S], q_full[2], q_empty[2], acc_full[2], acc_empty[2]
    static constexpr int kNumBars = 2 * kIxStages + 8;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffW = kOffTmem + 16;              // fp32 [64] weights of the token
    static constexpr int kBytes = kOffW + kIxMaxHeads * 4;
    static constexpr int kSmemBytes = kBytes + 1024;         // alignment slack (1024-B atoms)
    static constexpr uint32_t kTmemCols = 128;               // two accumulators of 64 columns
};

template <int NPAD>
__global__ void __launch_bounds__(IxCfg<NPAD>::kThreads, 1)
    smla_ix_score_kernel(const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_q, const IndexerParams p) {
    using C = IxCfg<NPAD>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *full = bars, *empty = bars + kIxStages;
    uint64_t *q_full = bars + 2 * kIxStages, *q_empty = q_full + 2;
    uint64_t *acc_full = q_empty + 2, *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);
    float *w_s = reinterpret_cast<float *>(smem + C::kOffW);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kIxStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 128);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    const uint32_t sbase = smem_addr(smem);
    bool dead = false;

    // this CTA's units: an equal share of all (token, tile) units
    const long long n_units = __ldg(p.tile_start + p.BT);
    const long long u_begin = n_units * blockIdx.x / gridDim.x;
    const long long u_end = n_units * (blockIdx.x + 1) / gridDim.x;

    if (warp == 0) {
        // ============================================================ TMA producer
        if (lane == 0 && u_begin < u_end) {
            const uint64_t keep = l2_policy_evict_last();   // a query is read again per tile
            const uint64_t once = l2_policy_evict_first();  // keys are read once
            int tok = ix_token_of(p, u_begin), changes = -1;
            for (long long unit = u_begin, i = 0; unit < u_end; ++unit, ++i) {
                bool fresh = unit == u_begin;
                while (__ldg(p.tile_start + tok + 1) <= unit) {
                    ++tok;
                    fresh = true;
                }
                if (fresh) {  // the token's query heads into the next slot
                    ++changes;
                    const int sl = changes & 1, use = changes >> 1;
                    if (use >= 1) mbar_wait(&q_empty[sl], (use - 1) & 1, dead);
                    mbar_arrive_expect_tx(&q_full[sl], (uint32_t)C::kQBytes);
                    const uint32_t qd = sbase + C::kOffQ + sl * C::kQBytes;
                    tma_load_2d(qd, &map_q, 0, tok * p.HI, &q_full[sl], keep);
                    tma_load_2d(qd + C::kQBoxBytes, &map_q, 64, tok * p.HI, &q_full[sl], keep);
                }
                const int st = (int)(i % kIxStages);
                if (i >= kIxStages) mbar_wait(&empty[st], (int)((i / kIxStages) - 1) & 1, dead);
                const int tile = (int)(unit - __ldg(p.tile_start + tok));
                const int n = ix_visible(p, tok);
                const int *pt_b = p.page_table + (size_t)(tok / p.T) * p.pt_stride;
                int pages[2];
                uint32_t bytes = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int lp = 2 * tile + h;  // logical page
                    pages[h] = -1;
                    const int first = lp * 64;
                    if (first >= n) continue;     // no visible position on it
                    const int pg = lp < p.pt_stride ? __ldg(pt_b + lp) : -1;
                    if (pg >= 0 && (long long)pg < p.num_pages) {
                        pages[h] = pg;
                        bytes += 2 * 64 * 128;
                    } else {  // visible positions on a page no entry maps: not candidates
                        atomicOr(&g_status_flags, kFlagIndexRange);
                        atomicAdd(&g_bad_index_count, (unsigned long long)(min(n, first + 64) - first));
                    }
                }
                mbar_arrive_expect_tx(&full[st], bytes);
                const uint32_t dst = sbase + C::kOffStages + st * C::kStageBytes;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (pages[h] < 0) continue;
                    tma_load_2d(dst + h * 8192, &map_k, 0, pages[h] * 64, &full[st], once);
                    tma_load_2d(dst + C::kBoxBytes + h * 8192, &map_k, 64, pages[h] * 64, &full[st], once);
                }
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0 && u_begin < u_end) {
            constexpr uint32_t kIdesc = idesc_bf16_f32(kIxTile, NPAD, false, false);
            int tok = ix_token_of(p, u_begin), changes = -1;
            for (long long unit = u_begin, i = 0; unit < u_end; ++unit, ++i) {
                bool fresh = unit == u_begin;
                while (__ldg(p.tile_start + tok + 1) <= unit) {
                    ++tok;
                    fresh = true;
                }
                if (fresh) {
                    ++changes;
                    mbar_wait(&q_full[changes & 1], (changes >> 1) & 1, dead);
                }
                const int st = (int)(i % kIxStages), a = (int)(i & 1);
                mbar_wait(&full[st], (int)(i / kIxStages) & 1, dead);
                if (i >= 2) mbar_wait(&acc_empty[a], (int)((i >> 1) - 1) & 1, dead);
                tc_fence_after();
                const uint32_t ka = sbase + C::kOffStages + st * C::kStageBytes;
                const uint32_t qa = sbase + C::kOffQ + (changes & 1) * C::kQBytes;
#pragma unroll
                for (int kk = 0; kk < kIxDim / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    const uint64_t ad = smem_desc(ka + (kk >> 2) * C::kBoxBytes + koff, 16, 1024, kSwizzle128B);
                    const uint64_t bd = smem_desc(qa + (kk >> 2) * C::kQBoxBytes + koff, 16, 1024, kSwizzle128B);
                    umma_bf16(tmem + a * 64, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&empty[st]);
                umma_commit(&acc_full[a]);
                // the token's last unit here: its query slot may be refilled
                if (unit + 1 == u_end || __ldg(p.tile_start + tok + 1) <= unit + 1)
                    umma_commit(&q_empty[changes & 1]);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ============================================================ epilogue
        const int q4 = warp & 3;                 // TMEM lanes 32 q4 .. + 31
        const int row = 32 * q4 + lane;          // key of the tile
        const int et = threadIdx.x - 128;        // 0 .. 127
        int tok = u_begin < u_end ? ix_token_of(p, u_begin) : 0, w_tok = -1;
        for (long long unit = u_begin, i = 0; unit < u_end; ++unit, ++i) {
            while (__ldg(p.tile_start + tok + 1) <= unit) ++tok;
            if (tok != w_tok) {  // the token's head weights (0 past HI)
                named_bar_sync(1, 128);
                if (et < kIxMaxHeads) w_s[et] = et < p.HI ? __ldg(p.w + (size_t)tok * p.HI + et) : 0.f;
                named_bar_sync(1, 128);
                w_tok = tok;
            }
            const int a = (int)(i & 1);
            mbar_wait(&acc_full[a], (int)(i >> 1) & 1, dead);
            tc_fence_after();
            uint32_t x[NPAD];
            tmem_ld_cols<NPAD>(tmem + ((uint32_t)(32 * q4) << 16) + a * 64, x);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&acc_empty[a]);
            const int tile = (int)(unit - __ldg(p.tile_start + tok));
            const int s = tile * kIxTile + row;
            const int n = ix_visible(p, tok);
            if (s < n) {
                const int lp = s >> 6;
                const int pg = lp < p.pt_stride ? __ldg(p.page_table + (size_t)(tok / p.T) * p.pt_stride + lp) : -1;
                float score = __uint_as_float(0x7fffffffu);  // NaN: not a candidate
                if (pg >= 0 && (long long)pg < p.num_pages) {
                    float acc = 0.f;
#pragma unroll
                    for (int j = 0; j < NPAD; ++j)
                        acc = (j < p.HI) ? fmaf(w_s[j], fmaxf(__uint_as_float(x[j]), 0.f), acc) : acc;
                    score = acc;
                }
                p.scores[(size_t)tok * p.score_stride + s] = score;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- selection
// Order-preserving key of a score: larger score -> larger key; -0 and +0
// share one key; NaN (not a candidate) -> 0, below every real score.
__device__ __forceinline__ uint32_t ix_key(float f) {
    if (f != f) return 0u;
    if (f == 0.f) f = 0.f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kIxSelectThreads) smla_ix_select_kernel(const IndexerParams p) {
    __shared__ unsigned hist[2048];
    __shared__ int scratch[33];
    __shared__ int found[2];
    const int u = blockIdx.x, tid = threadIdx.x;
    const int n = ix_visible(p, u), K = p.K;
    const float *sc = p.scores + (size_t)u * p.score_stride;
    int *out = p.out + (size_t)u * K;

    // Three radix passes find the K-th largest key (thresh) and how many keys
    // equal to it are taken (need); with K or fewer candidates, all are.
    uint32_t prefix = 0, thresh = 0;
    int need = K, valid = 0;
    const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = shifts[pass], nb = 1 << widths[pass];
        for (int i = tid; i < 2048; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        const int hi_shift = shift + widths[pass];  // bits above this digit must match prefix
        for (int s = tid; s < n; s += blockDim.x) {
            const uint32_t key = ix_key(__ldg(sc + s));
            const bool match = key != 0u && (hi_shift >= 32 || (key >> hi_shift) == prefix);
            const uint32_t d = (key >> shift) & (uint32_t)(nb - 1);
            // aggregate equal digits within the warp (scores cluster in few buckets)
            const uint32_t peers = __match_any_sync(__activemask(), match ? d : 0xffffffffu);
            if (match && (__ffs(peers) - 1) == (tid & 31)) atomicAdd(&hist[d], (unsigned)__popc(peers));
        }
        __syncthreads();
        // bins from the top: thread i sums bins nb-1-2i and nb-2-2i
        int v = 0, b_hi = -1, b_lo = -1;
        if (2 * tid < nb) {
            b_hi = nb - 1 - 2 * tid;
            b_lo = b_hi - 1;
            v = (int)hist[b_hi] + (b_lo >= 0 ? (int)hist[b_lo] : 0);
        }
        int total;
        const int incl = ix_block_scan(v, scratch, &total);
        if (pass == 0) {
            valid = total;
            if (valid <= K) {  // every candidate is taken
                thresh = 0u;
                need = 0;
                break;
            }
        }
        const int excl = incl - v;
        if (b_hi >= 0 && excl < need && need <= incl) {
            const int h = (int)hist[b_hi];
            if (excl + h >= need) {
                found[0] = b_hi;
                found[1] = excl;
            } else {
                found[0] = b_lo;
                found[1] = excl + h;
            }
        }
        __syncthreads();
        prefix = (prefix << widths[pass]) | (uint32_t)found[0];
        need -= found[1];
        __syncthreads();
        if (pass == 2) thresh = prefix;
    }

    // Ascending scan: keys above thresh, and the first `need` equal to it.
    int eq_carry = 0, sel_carry = 0, total;
    for (int base = 0; base < n; base += blockDim.x) {
        const int s = base + tid;
        const uint32_t key = s < n ? ix_key(__ldg(sc + s)) : 0u;
        const int eq = (need > 0 && key == thresh) ? 1 : 0;
        const int eq_incl = ix_block_scan(eq, scratch, &total);
        const int eq_rank = eq_carry + eq_incl - eq;
        eq_carry += total;
        const int sel = (key > thresh || (eq && eq_rank < need)) ? 1 : 0;
        const int sel_incl = ix_block_scan(sel, scratch, &total);
        const int at = sel_carry + sel_incl - sel;
        if (sel && at < K) out[at] = s;
        sel_carry += total;
    }
    for (int i = min(sel_carry, K) + tid; i < K; i += blockDim.x) out[i] = -1;
}

}  // namespace smla
