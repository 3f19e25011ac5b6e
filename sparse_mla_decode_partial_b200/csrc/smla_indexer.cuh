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
// Selection (smla_ix_select_kernel): one CTA per query token; radix passes
// (8, 12, 12 bits) over an order-preserving key of the fp32 score find the
// K-th largest score -- the first over all scores, the others over the
// crossing bucket's candidates in shared memory -- then ordered scans of two
// position bitmaps write the positions above it and the first ones (by
// position) equal to it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "smla_tc_ptx.cuh"

namespace smla {

constexpr int kIxDim = 128;        // index-key width (bf16 values)
constexpr int kIxTile = 128;       // keys per unit: the MMA's M
constexpr int kIxMaxHeads = 64;    // index heads: the MMA's N (padded to 16, 32, 64)
constexpr int kIxStages = 5;       // key tiles in flight per CTA
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

// What a role needs to know about one unit, computed by one lane for a batch
// of 32 consecutive units (the dependent loads of 32 units then overlap).
// pg[h]: physical page of the tile's h-th page; -1 when none of its
// positions is visible, -2 when visible positions sit on a page no entry
// maps (not candidates; counted by the producer).
struct IxUnit {
    int tok, tile, n, pg0, pg1;
};

// `hint`: a token at or before the unit's (units are walked in order, and
// consecutive units rarely change token, so the advance is a step or two of
// cached loads).
__device__ __forceinline__ IxUnit ix_unit(const IndexerParams &p, long long unit, int hint) {
    IxUnit m;
    m.tok = hint;
    while (__ldg(p.tile_start + m.tok + 1) <= unit) ++m.tok;
    m.tile = (int)(unit - __ldg(p.tile_start + m.tok));
    m.n = ix_visible(p, m.tok);
    const int *pt_b = p.page_table + (size_t)(m.tok / p.T) * p.pt_stride;
    int pg[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int lp = 2 * m.tile + h;
        pg[h] = -1;
        if (lp * 64 < m.n) {
            const int v = lp < p.pt_stride ? __ldg(pt_b + lp) : -1;
            pg[h] = (v >= 0 && (long long)v < p.num_pages) ? v : -2;
        }
    }
    m.pg0 = pg[0];
    m.pg1 = pg[1];
    return m;
}

__device__ __forceinline__ IxUnit ix_unit_from(const IxUnit &m, int k) {
    IxUnit r;
    r.tok = __shfl_sync(0xffffffffu, m.tok, k);
    r.tile = __shfl_sync(0xffffffffu, m.tile, k);
    r.n = __shfl_sync(0xffffffffu, m.n, k);
    r.pg0 = __shfl_sync(0xffffffffu, m.pg0, k);
    r.pg1 = __shfl_sync(0xffffffffu, m.pg1, k);
    return r;
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
    // full[S], empty[S], q_full[2], q_empty[2], acc_full[A], acc_empty[A]
    static constexpr int kAcc = 4;                           // accumulators of 64 TMEM columns
    static constexpr int kNumBars = 2 * kIxStages + 4 + 2 * kAcc;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffW = kOffTmem + 16;              // fp32 [64] weights of the token
    static constexpr int kBytes = kOffW + kIxMaxHeads * 4;
    static constexpr int kSmemBytes = kBytes + 1024;         // alignment slack (1024-B atoms)
    static constexpr uint32_t kTmemCols = 64 * kAcc;
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
    uint64_t *acc_full = q_empty + 2, *acc_empty = acc_full + C::kAcc;
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
        }
        for (int i = 0; i < C::kAcc; ++i) {
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
        if (u_begin < u_end) {
            const uint64_t keep = l2_policy_evict_last();   // a query is read again per tile
            const uint64_t once = l2_policy_evict_first();  // keys are read once
            int prev_tok = -1, changes = -1;
            int hint = ix_token_of(p, u_begin);
            long long i = 0;
            for (long long ub = u_begin; ub < u_end; ub += 32) {
                const int cnt = (int)min(32ll, u_end - ub);
                const IxUnit mine = ix_unit(p, min(ub + lane, u_end - 1), hint);
                hint = __shfl_sync(0xffffffffu, mine.tok, cnt - 1);
                for (int k = 0; k < cnt; ++k, ++i) {
                    const IxUnit m = ix_unit_from(mine, k);
                    if (lane == 0) {
                        if (m.tok != prev_tok) {  // the token's query heads into the next slot
                            prev_tok = m.tok;
                            ++changes;
                            const int sl = changes & 1, use = changes >> 1;
                            if (use >= 1) mbar_wait(&q_empty[sl], (use - 1) & 1, dead);
                            mbar_arrive_expect_tx(&q_full[sl], (uint32_t)C::kQBytes);
                            const uint32_t qd = sbase + C::kOffQ + sl * C::kQBytes;
                            tma_load_2d(qd, &map_q, 0, m.tok * p.HI, &q_full[sl], keep);
                            tma_load_2d(qd + C::kQBoxBytes, &map_q, 64, m.tok * p.HI, &q_full[sl], keep);
                        }
                        const int st = (int)(i % kIxStages);
                        if (i >= kIxStages) mbar_wait(&empty[st], (int)((i / kIxStages) - 1) & 1, dead);
                        const int pgs[2] = {m.pg0, m.pg1};
                        uint32_t bytes = 0;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (pgs[h] >= 0) {
                                bytes += 2 * 64 * 128;
                            } else if (pgs[h] == -2) {  // visible positions no page entry maps
                                const int first = (2 * m.tile + h) * 64;
                                atomicOr(&g_status_flags, kFlagIndexRange);
                                atomicAdd(&g_bad_index_count, (unsigned long long)(min(m.n, first + 64) - first));
                            }
                        }
                        mbar_arrive_expect_tx(&full[st], bytes);
                        const uint32_t dst = sbase + C::kOffStages + st * C::kStageBytes;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (pgs[h] < 0) continue;
                            tma_load_2d(dst + h * 8192, &map_k, 0, pgs[h] * 64, &full[st], once);
                            tma_load_2d(dst + C::kBoxBytes + h * 8192, &map_k, 64, pgs[h] * 64, &full[st], once);
                        }
                    }
                    __syncwarp();
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
                const int st = (int)(i % kIxStages), a = (int)(i % C::kAcc);
                mbar_wait(&full[st], (int)(i / kIxStages) & 1, dead);
                if (i >= C::kAcc) mbar_wait(&acc_empty[a], (int)((i / C::kAcc) - 1) & 1, dead);
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
        int w_tok = -1;
        int hint = u_begin < u_end ? ix_token_of(p, u_begin) : 0;
        long long i = 0;
        for (long long ub = u_begin; ub < u_end; ub += 32) {
            const int cnt = (int)min(32ll, u_end - ub);
            const IxUnit mine = ix_unit(p, min(ub + lane, u_end - 1), hint);
            hint = __shfl_sync(0xffffffffu, mine.tok, cnt - 1);
            for (int k = 0; k < cnt; ++k, ++i) {
                const IxUnit m = ix_unit_from(mine, k);
                if (m.tok != w_tok) {  // the token's head weights (0 past HI)
                    named_bar_sync(1, 128);
                    if (et < kIxMaxHeads) w_s[et] = et < p.HI ? __ldg(p.w + (size_t)m.tok * p.HI + et) : 0.f;
                    named_bar_sync(1, 128);
                    w_tok = m.tok;
                }
                const int a = (int)(i % C::kAcc);
                mbar_wait(&acc_full[a], (int)(i / C::kAcc) & 1, dead);
                tc_fence_after();
                uint32_t x[NPAD];
                tmem_ld_cols<NPAD>(tmem + ((uint32_t)(32 * q4) << 16) + a * 64, x);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acc_empty[a]);
                const int s = m.tile * kIxTile + row;
                if (s < m.n) {
                    float score = __uint_as_float(0x7fffffffu);  // NaN: not a candidate
                    if ((row < 64 ? m.pg0 : m.pg1) >= 0) {
                        float acc = 0.f;
#pragma unroll
                        for (int j = 0; j < NPAD; ++j)
                            acc = (j < p.HI) ? fmaf(w_s[j], fmaxf(__uint_as_float(x[j]), 0.f), acc) : acc;
                        score = acc;
                    }
                    p.scores[(size_t)m.tok * p.score_stride + s] = score;
                }
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

// Shared memory of the selection kernel: the histograms (per-warp private
// ones for the first digit), the crossing bucket's candidates and two bitmaps
// over the visible positions (selected, equal to the threshold).
constexpr int kIxCandCap = 8192;    // candidates of the crossing bucket kept in shared memory
constexpr int kIxHistBytes = 32 * 256 * 4;  // 32 warps x 256 bins, or one 4096-bin histogram
__host__ __device__ constexpr int ix_select_smem_bytes(int max_n) {
    return kIxHistBytes + kIxCandCap * 8 + 2 * 4 * ((max_n + 31) / 32);
}
constexpr int kIxSelectMaxN = (232448 - kIxHistBytes - kIxCandCap * 8 - 1024) / 8 * 32;

// Warp-aggregated increment of hist[d] (lanes with the same digit add once).
__device__ __forceinline__ void ix_hist_add(unsigned *hist, bool match, uint32_t d) {
    const uint32_t peers = __match_any_sync(__activemask(), match ? d : 0xffffffffu);
    if (match && (__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[d], (unsigned)__popc(peers));
}

// Bucket of the histogram (nb bins) holding the need-th largest key counted
// from the top: writes (bucket, keys above it) to found[]; returns the total.
// Thread i sums bins nb-1-i*per .. nb-per-i*per (per = nb / blockDim.x).
__device__ __forceinline__ int ix_find_bucket(const unsigned *hist, int nb, int need, int *scratch,
                                              int *found) {
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    const int top = nb - 1 - (int)threadIdx.x * per;
    int v = 0;
    for (int k = 0; k < per; ++k)
        if (top - k >= 0) v += (int)hist[top - k];
    int total;
    const int incl = ix_block_scan(v, scratch, &total);
    int excl = incl - v;
    if (excl < need && need <= incl) {
        for (int k = 0; k < per && top - k >= 0; ++k) {
            const int h = (int)hist[top - k];
            if (excl + h >= need) {
                found[0] = top - k;
                found[1] = excl;
                break;
            }
            excl += h;
        }
    }
    __syncthreads();
    return total;
}

// Ordered scan of a bitmap of `words` words: calls emit(rank, position) for
// every set bit in ascending position order (rank = its index among set bits).
template <typename F>
__device__ __forceinline__ int ix_bitmap_scan(const uint32_t *bits, int words, int *scratch, F emit) {
    const int per = (words + blockDim.x - 1) / blockDim.x;
    const int w0 = min(words, (int)threadIdx.x * per), w1 = min(words, w0 + per);
    int cnt = 0;
    for (int i = w0; i < w1; ++i) cnt += __popc(bits[i]);
    int total;
    int rank = ix_block_scan(cnt, scratch, &total) - cnt;
    for (int i = w0; i < w1; ++i) {
        uint32_t m = bits[i];
        while (m) {
            const int b = __ffs(m) - 1;
            m &= m - 1;
            emit(rank++, 32 * i + b);
        }
    }
    return total;
}

// One CTA per query token.  Pass A (global): histogram of the top 8 bits of
// the key, one private histogram per warp (scores crowd into few buckets;
// shared bins would serialise the warps) -> the crossing bucket d0.  Pass B
// (global): positions with a digit above d0 are selected (bitmap); those in
// d0 become candidates in shared memory.  Two 12-bit radix passes over the
// candidates give the exact threshold key and how many keys equal to it are
// taken; the first of those by position are found by an ordered scan of an
// "equal" bitmap, and an ordered scan of the selection bitmap writes the
// output.  If d0 holds more than kIxCandCap keys, the finer passes and the
// marking read the global scores instead.
__global__ void __launch_bounds__(kIxSelectThreads) smla_ix_select_kernel(const IndexerParams p) {
    extern __shared__ __align__(16) uint8_t ix_smem[];
    unsigned *hist = reinterpret_cast<unsigned *>(ix_smem);
    uint32_t *cand_key = reinterpret_cast<uint32_t *>(ix_smem + kIxHistBytes);
    int *cand_pos = reinterpret_cast<int *>(ix_smem + kIxHistBytes + kIxCandCap * 4);
    uint32_t *sel_bits = reinterpret_cast<uint32_t *>(ix_smem + kIxHistBytes + kIxCandCap * 8);
    __shared__ int scratch[33];
    __shared__ int found[2];
    __shared__ int n_cand;
    const int u = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int n = ix_visible(p, u), K = p.K;
    const int words = (n + 31) / 32;
    uint32_t *eq_bits = sel_bits + words;
    const float *sc = p.scores + (size_t)u * p.score_stride;
    int *out = p.out + (size_t)u * K;
    constexpr int kIlp = 8;

    for (int i = tid; i < kIxHistBytes / 4; i += nt) hist[i] = 0;
    for (int i = tid; i < 2 * words; i += nt) sel_bits[i] = 0;
    if (tid == 0) n_cand = 0;
    __syncthreads();

    // ---- pass A: top 8 bits into this warp's own 256 bins
    unsigned *my_hist = hist + warp * 256;
    for (int base = 0; base < n; base += nt * kIlp) {
        uint32_t key[kIlp];
#pragma unroll
        for (int j = 0; j < kIlp; ++j) {
            const int s = base + j * nt + tid;
            key[j] = s < n ? ix_key(__ldg(sc + s)) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kIlp; ++j) ix_hist_add(my_hist, key[j] != 0u, key[j] >> 24);
    }
    __syncthreads();
    // fold the 32 private histograms into bins 0..255 of warp 0's
    if (tid < 256) {
        unsigned sum = 0;
        for (int w = 0; w < 32; ++w) sum += hist[w * 256 + tid];
        hist[tid] = sum;
    }
    __syncthreads();
    int need = K;
    const int valid = ix_find_bucket(hist, 256, need, scratch, found);
    const bool take_all = valid <= K;
    const uint32_t d0 = take_all ? 0u : (uint32_t)found[0];
    if (!take_all) need -= found[1];

    // ---- pass B: digits above d0 are in; d0's keys become candidates
    for (int base = 0; base < n; base += nt * kIlp) {
        uint32_t key[kIlp];
#pragma unroll
        for (int j = 0; j < kIlp; ++j) {
            const int s = base + j * nt + tid;
            key[j] = s < n ? ix_key(__ldg(sc + s)) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kIlp; ++j) {
            const int s = base + j * nt + tid;
            const uint32_t d = key[j] >> 24;
            const bool above = key[j] != 0u && (take_all || d > d0);
            const bool cand = key[j] != 0u && !take_all && d == d0;
            if (above) atomicOr(&sel_bits[s >> 5], 1u << (s & 31));
            // warp-aggregated append of the candidates
            const uint32_t cm = __ballot_sync(0xffffffffu, cand);
            int slot0 = 0;
            if (lane == 0 && cm) slot0 = atomicAdd(&n_cand, __popc(cm));
            slot0 = __shfl_sync(0xffffffffu, slot0, 0);
            if (cand) {
                const int c = slot0 + __popc(cm & ((1u << lane) - 1u));
                if (c < kIxCandCap) {
                    cand_key[c] = key[j];
                    cand_pos[c] = s;
                }
            }
        }
    }
    __syncthreads();

    if (!take_all) {
        // ---- the two finer 12-bit digits, over the candidates (or the global scores)
        const int m = n_cand;
        const bool in_smem = m <= kIxCandCap;
        uint32_t prefix = d0;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 12 : 0, hi_shift = shift + 12;
            for (int i = tid; i < 4096; i += nt) hist[i] = 0;
            __syncthreads();
            if (in_smem) {
                for (int c = tid; c < ((m + 31) & ~31); c += nt) {
                    const uint32_t key = c < m ? cand_key[c] : 0u;
                    ix_hist_add(hist, c < m && (key >> hi_shift) == prefix, (key >> shift) & 4095u);
                }
            } else {
                for (int base = 0; base < n; base += nt * kIlp) {
                    uint32_t key[kIlp];
#pragma unroll
                    for (int j = 0; j < kIlp; ++j) {
                        const int s = base + j * nt + tid;
                        key[j] = s < n ? ix_key(__ldg(sc + s)) : 0u;
                    }
#pragma unroll
                    for (int j = 0; j < kIlp; ++j)
                        ix_hist_add(hist, key[j] != 0u && (key[j] >> hi_shift) == prefix,
                                    (key[j] >> shift) & 4095u);
                }
            }
            __syncthreads();
            ix_find_bucket(hist, 4096, need, scratch, found);
            prefix = (prefix << 12) | (uint32_t)found[0];
            need -= found[1];
            __syncthreads();
        }
        const uint32_t thresh = prefix;
        // ---- mark: above the threshold -> selected; equal -> the "equal" bitmap
        if (in_smem) {
            for (int c = tid; c < m; c += nt) {
                const uint32_t key = cand_key[c];
                const int s = cand_pos[c];
                if (key > thresh) atomicOr(&sel_bits[s >> 5], 1u << (s & 31));
                else if (key == thresh) atomicOr(&eq_bits[s >> 5], 1u << (s & 31));
            }
        } else {
            for (int s = tid; s < n; s += nt) {
                const uint32_t key = ix_key(__ldg(sc + s));
                if (key == 0u || (key >> 24) != d0) continue;  // the bits above d0 are set already
                if (key > thresh) atomicOr(&sel_bits[s >> 5], 1u << (s & 31));
                else if (key == thresh) atomicOr(&eq_bits[s >> 5], 1u << (s & 31));
            }
        }
        __syncthreads();
        // ---- the first `need` equal keys by position
        ix_bitmap_scan(eq_bits, words, scratch, [&](int rank, int s) {
            if (rank < need) atomicOr(&sel_bits[s >> 5], 1u << (s & 31));
        });
        __syncthreads();
    }

    // ---- output: selected positions in ascending order, then -1
    const int taken = ix_bitmap_scan(sel_bits, words, scratch, [&](int rank, int s) {
        if (rank < K) out[rank] = s;
    });
    for (int i = min(taken, K) + tid; i < K; i += nt) out[i] = -1;
}

}  // namespace smla
