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
// Selection: a radix select on an order-preserving key of the fp32 score.
// The first digit (12 bits) is counted and its crossing bucket found over
// every position, split into chunks so that one long context keeps the whole
// device busy (smla_ix_hist_kernel); a second chunked pass selects the
// positions above that bucket (a position bitmap) and gathers those in it as
// candidates (smla_ix_mark_kernel); per token, two 10-bit digits over the
// candidates give the exact K-th largest key, and ordered scans of position
// bitmaps write the positions above it and the first ones (by position)
// equal to it (smla_ix_finish_kernel).
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
constexpr int kIxSelBins = 4096;   // selection: bins of the first digit (key >> 20)

// Selection state of one query token (in the selection scratch).
struct IxSelMeta {
    int d0;        // crossing bucket of the first digit
    int need;      // keys still to take from it
    int take_all;  // every candidate is selected (at most K of them)
    int count;     // entries appended to cand
    int pad[4];
};
static_assert(sizeof(IxSelMeta) == 32, "meta is 32 bytes");

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
    // selection scratch (see the selection section below)
    unsigned *sel_hist;      // [B * T, 4096]; the score kernel adds to it when non-null
    IxSelMeta *sel_meta;     // [B * T]
    uint32_t *sel_bits;      // [B * T, sel_words]
    uint2 *sel_cand;         // [B * T, max_n]: (key, position)
    int sel_words;
    int sel_chunks;          // chunks of kIxSelChunk positions per token
    int sel_prefetch;        // the scores are complete before the selection chain starts
    uint4 *zero;             // plan kernel: n_zero 16-byte words to clear (or null)
    long long n_zero;
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

// Inclusive sum over a group of NT threads (t = 0 .. NT-1, whole warps) that
// synchronise with sync(); *total receives the group's sum.  scratch holds
// NT / 32 ints.
template <int NT, typename Sync>
__device__ __forceinline__ int ix_group_scan(int v, int t, int *scratch, int *total, Sync sync) {
    const int lane = t & 31, warp = t >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
    }
    if (lane == 31) scratch[warp] = v;
    sync();
    int base = 0, tot = 0;
#pragma unroll
    for (int k = 0; k < NT / 32; ++k) {
        const int x = scratch[k];
        base += k < warp ? x : 0;
        tot += x;
    }
    *total = tot;
    sync();  // scratch may be reused at once
    return v + base;
}

// The crossing bucket of a token's first digit from its complete histogram
// (4096 bins, counted from the top): group thread t holds bins
// [4096 - per*(t+1), 4096 - per*t) in registers (ix_decide_load), then one
// group scan finds the bucket (ix_decide).  Writes (take_all, d0, need) to
// dec[] (shared); dec is complete after the group's next sync.
template <int NT>
__device__ __forceinline__ void ix_decide_load(const unsigned *gh, int t, uint32_t (&b)[4096 / NT]) {
    constexpr int kPer = 4096 / NT;
    static_assert(kPer % 4 == 0, "bins per thread load as uint4");
    const int lo = 4096 - kPer * (t + 1);
#pragma unroll
    for (int q = 0; q < kPer / 4; ++q) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(gh + lo) + q);
        b[4 * q] = v.x;
        b[4 * q + 1] = v.y;
        b[4 * q + 2] = v.z;
        b[4 * q + 3] = v.w;
    }
}

// The scan half of the above over bins already loaded by ix_decide_load.
template <int NT, typename Sync>
__device__ __forceinline__ void ix_decide(const uint32_t (&b)[4096 / NT], int K, int t, int *scratch,
                                          int *dec, Sync sync) {
    constexpr int kPer = 4096 / NT;
    const int lo = 4096 - kPer * (t + 1);
    int v = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) v += (int)b[k];
    int total;
    const int incl = ix_group_scan<NT>(v, t, scratch, &total, sync);
    if (total <= K) {
        if (t == 0) {
            dec[0] = 1;
            dec[1] = 0;
            dec[2] = 0;
        }
        return;
    }
    int excl = incl - v;
    if (excl < K && K <= incl) {
#pragma unroll
        for (int k = kPer - 1; k >= 0; --k) {    // from the highest bin down
            if (excl >= 0 && excl + (int)b[k] >= K) {
                dec[0] = 0;
                dec[1] = lo + k;
                dec[2] = K - excl;
                excl = -1;
            } else if (excl >= 0) {
                excl += (int)b[k];
            }
        }
    }
}

// Order-preserving key of a score: larger score -> larger key; -0 and +0
// share one key; NaN (not a candidate) -> 0, below every real score.
__device__ __forceinline__ uint32_t ix_key(float f) {
    if (f != f) return 0u;
    if (f == 0.f) f = 0.f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void ix_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void ix_pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- plan
// Units of work: token u has ceil(n_u / 128) key tiles; tile_start is their
// exclusive prefix sum (CTA 0).  A length outside [0, max_n] is clamped and
// counted.  Every CTA also clears its share of p.zero (the selection's
// histograms when the score kernel fills them).
__global__ void __launch_bounds__(1024) smla_ix_plan_kernel(const IndexerParams p) {
    __shared__ int scratch[33];
    ix_pdl_trigger();
    for (long long i = blockIdx.x * 1024ll + threadIdx.x; i < p.n_zero; i += (long long)gridDim.x * 1024)
        p.zero[i] = make_uint4(0u, 0u, 0u, 0u);
    if (blockIdx.x != 0) return;
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

// tile_start is written by the plan kernel, whose programmatic dependent (the
// score kernel) is resident while it runs: it is read with weak global loads
// (ld_input), never through the read-only path.  The caller's inputs (n_vis, w, the page
// table, the keys) are complete before the plan kernel starts.
//
// Token holding unit `unit` (tile_start ascending; tokens with no tile skipped).
__device__ __forceinline__ int ix_token_of(const IndexerParams &p, long long unit) {
    int lo = 0, hi = p.BT - 1;  // the last token with tile_start <= unit
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ld_input(p.tile_start + mid) <= unit) lo = mid; else hi = mid - 1;
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
    while (ld_input(p.tile_start + m.tok + 1) <= unit) ++m.tok;
    m.tile = (int)(unit - ld_input(p.tile_start + m.tok));
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
    static constexpr int kOffHist = kOffTmem + 16;            // u32 [4096]: selection digits of a token
    // head weights of the CTA's tokens (when they span at most kWTokens)
    static constexpr int kWTokens = 64;
    static constexpr int kOffW = kOffHist + kIxSelBins * 4;   // f32 [kWTokens][NPAD]
    static constexpr int kBytes = kOffW + kWTokens * NPAD * 4;
    static constexpr int kSmemBytes = kBytes + 1024;         // alignment slack (1024-B atoms)
    static constexpr uint32_t kTmemCols = 64 * kAcc;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

template <int NPAD>
__global__ void __launch_bounds__(IxCfg<NPAD>::kThreads, 1)
    smla_ix_score_kernel(const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_q, const IndexerParams p) {
    using C = IxCfg<NPAD>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    ix_pdl_trigger();
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *full = bars, *empty = bars + kIxStages;
    uint64_t *q_full = bars + 2 * kIxStages, *q_empty = q_full + 2;
    uint64_t *acc_full = q_empty + 2, *acc_empty = acc_full + C::kAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);

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
    ix_pdl_wait();   // the plan (and the cleared histograms) are complete
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    const uint32_t sbase = smem_addr(smem);
    bool dead = false;

    // this CTA's units: an equal share of all (token, tile) units
    const long long n_units = ld_input(p.tile_start + p.BT);
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
                while (ld_input(p.tile_start + tok + 1) <= unit) {
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
                // descriptors built once; a k-step adds a constant to the
                // address field (16-byte units, no carry below 2^18)
                const uint64_t ad0 = smem_desc(ka, 16, 1024, kSwizzle128B);
                const uint64_t bd0 = smem_desc(qa, 16, 1024, kSwizzle128B);
#pragma unroll
                for (int kk = 0; kk < kIxDim / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    const uint64_t ad = ad0 + (uint64_t)(((kk >> 2) * C::kBoxBytes + koff) >> 4);
                    const uint64_t bd = bd0 + (uint64_t)(((kk >> 2) * C::kQBoxBytes + koff) >> 4);
                    umma_bf16(tmem + a * 64, ad, bd, kIdesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&empty[st]);
                umma_commit(&acc_full[a]);
                // the token's last unit here: its query slot may be refilled
                if (unit + 1 == u_end || ld_input(p.tile_start + tok + 1) <= unit + 1)
                    umma_commit(&q_empty[changes & 1]);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ============================================================ epilogue
        const int q4 = warp & 3;                 // TMEM lanes 32 q4 .. + 31
        const int row = 32 * q4 + lane;          // key of the tile
        const int et = threadIdx.x - 128;        // 0 .. 127
        // The selection's first-digit counts of the current token gather in
        // shared memory and go to the token's global histogram when the token
        // changes (global atomics per key would pile onto a few hot bins).
        unsigned *hist_s = reinterpret_cast<unsigned *>(smem + C::kOffHist);
        const bool count = p.sel_hist != nullptr;
        int h_tok = -1;
        auto flush = [&]() {
            named_bar_sync(1, 128);
            unsigned *gh = p.sel_hist + (size_t)h_tok * kIxSelBins;
            for (int b = et; b < kIxSelBins; b += 128) {
                const unsigned v = hist_s[b];
                if (v) {
                    atomicAdd(gh + b, v);
                    hist_s[b] = 0u;
                }
            }
            named_bar_sync(1, 128);
        };
        if (count) {
            for (int b = et; b < kIxSelBins; b += 128) hist_s[b] = 0u;
            named_bar_sync(1, 128);
        }
        int w_tok = -1;
        float wr[NPAD];                          // the token's head weights (0 past HI)
        int hint = u_begin < u_end ? ix_token_of(p, u_begin) : 0;
        // The weights of every token this CTA touches (a contiguous span) wait
        // in shared memory, loaded once, so that a token change reads them
        // there instead of paying a memory round trip.
        float *w_s = reinterpret_cast<float *>(smem + C::kOffW);
        const int w_first = hint;
        const int w_last = u_begin < u_end ? ix_token_of(p, u_end - 1) : hint - 1;
        const bool w_staged = w_last - w_first < C::kWTokens;
        if (w_staged) {
            const int n = (w_last - w_first + 1) * NPAD;
            for (int i0 = 0; i0 < n; i0 += 128 * 8) {
                float v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int e = i0 + k * 128 + et, j = e % NPAD;
                    v[k] = (e < n && j < p.HI) ? __ldg(p.w + (size_t)(w_first + e / NPAD) * p.HI + j) : 0.f;
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (i0 + k * 128 + et < n) w_s[i0 + k * 128 + et] = v[k];
            }
            named_bar_sync(1, 128);
        }
        long long i = 0;
        for (long long ub = u_begin; ub < u_end; ub += 32) {
            const int cnt = (int)min(32ll, u_end - ub);
            const IxUnit mine = ix_unit(p, min(ub + lane, u_end - 1), hint);
            hint = __shfl_sync(0xffffffffu, mine.tok, cnt - 1);
            for (int k = 0; k < cnt; ++k, ++i) {
                const IxUnit m = ix_unit_from(mine, k);
                if (m.tok != w_tok) {
                    if (w_staged) {
                        const float4 *src = reinterpret_cast<const float4 *>(w_s + (m.tok - w_first) * NPAD);
#pragma unroll
                        for (int j = 0; j < NPAD / 4; ++j) {
                            const float4 x = src[j];
                            wr[4 * j] = x.x;
                            wr[4 * j + 1] = x.y;
                            wr[4 * j + 2] = x.z;
                            wr[4 * j + 3] = x.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < NPAD; ++j)
                            wr[j] = j < p.HI ? __ldg(p.w + (size_t)m.tok * p.HI + j) : 0.f;
                    }
                    w_tok = m.tok;
                    if (count) {
                        if (h_tok >= 0) flush();
                        h_tok = m.tok;
                    }
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
                        // four interleaved partial sums (heads j = r mod 4), added pairwise
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int j = 0; j < NPAD; ++j)
                            if (j < p.HI) acc[j & 3] = fmaf(wr[j], fmaxf(__uint_as_float(x[j]), 0.f), acc[j & 3]);
                        score = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                    }
                    p.scores[(size_t)m.tok * p.score_stride + s] = score;
                    if (count) {  // the selection's first digit, counted here
                        const uint32_t key = ix_key(score);
                        if (key != 0u) atomicAdd(&hist_s[key >> 20], 1u);
                    }
                }
            }
        }
        if (count && h_tok >= 0) flush();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- selection
// A per-call scratch (workspace):
//   hist   [BT][4096] u32    counts of the first digit (key >> 20)
//   meta   [BT]              crossing bucket, keys still needed, candidate count
//   bits   [BT][sel_words]   positions selected by the first digit
//   cand   [BT][max_n] uint2 (key, position) of those in the crossing bucket
// The histogram is filled by the score kernel's epilogue when the scores are
// computed here (smla_indexer_topk), else by smla_ix_hist_kernel over given
// scores (after smla_ix_clear_kernel).  smla_ix_mark_kernel then finds the
// crossing bucket and marks; hist and mark split every token into chunks of
// kIxSelChunk positions, one CTA per (token, chunk), so a long context is
// spread over the whole device.  smla_ix_finish_kernel (one CTA per token)
// resolves the remaining 20 bits over the candidates and writes the output.
// The kernels are chained by programmatic dependent launch: each calls
// griddepcontrol.wait before it touches what its predecessor writes.
constexpr int kIxSelThreads = 512;     // chunked passes
constexpr int kIxSelIlp = 16;          // positions per thread: one load round trip
constexpr int kIxSelChunk = kIxSelThreads * kIxSelIlp;
constexpr int kIxMarkSmemBytes = kIxSelChunk * 8;   // staged candidates
constexpr int kIxFinishThreads = 512;
constexpr int kIxCandCap = 8192;       // candidates the finish kernel holds in shared memory
constexpr int kIxFineBins = 1024;      // the two finer digits: 10 bits each


__host__ __device__ constexpr int ix_finish_smem_bytes(int max_n) {
    return kIxCandCap * 8 + kIxFineBins * 4 + 2 * 4 * ((max_n + 31) / 32);
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
// every set bit in ascending position order (rank = its index among set
// bits).  Each warp owns a contiguous run of words and reads it 32 words at
// a time (lane i the i-th word), so the reads are conflict-free.
template <typename F>
__device__ __forceinline__ int ix_bitmap_scan(const uint32_t *bits, int words, int *scratch, F emit) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int per = ((words + nw - 1) / nw + 31) & ~31;
    const int w0 = min(words, warp * per), w1 = min(words, w0 + per);
    int cnt = 0;
    for (int i = w0 + lane; i < w1; i += 32) cnt += __popc(bits[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    int total;
    const int incl = ix_block_scan(lane == 0 ? cnt : 0, scratch, &total);
    int base = __shfl_sync(0xffffffffu, incl, 0) - cnt;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        uint32_t m = i < w1 ? bits[i] : 0u;
        const int c = __popc(m);
        int x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int rank = base + x - c;
        base += __shfl_sync(0xffffffffu, x, 31);
        while (m) {
            const int b = __ffs(m) - 1;
            m &= m - 1;
            emit(rank++, 32 * i + b);
        }
    }
    return total;
}

// Zeroes the per-token histograms and meta (n16 16-byte words).
__global__ void __launch_bounds__(256) smla_ix_clear_kernel(uint4 *buf, long long n16) {
    ix_pdl_trigger();
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n16; i += (long long)gridDim.x * 256)
        buf[i] = make_uint4(0u, 0u, 0u, 0u);
}

// The (token, chunk) pair of a CTA of the chunked passes: a 1-D grid over
// B*T x sel_chunks, token-major, so that the CTAs with work (chunks below a
// token's length) are spread along the launch order.
struct IxChunk {
    int u, s0, s1;
};
__device__ __forceinline__ IxChunk ix_chunk(const IndexerParams &p) {
    const int u = blockIdx.x / p.sel_chunks;
    const int s0 = (blockIdx.x - u * p.sel_chunks) * kIxSelChunk;
    return {u, s0, min(ix_visible(p, u), s0 + kIxSelChunk)};
}

// The chunk's keys, one load round trip (lane-consecutive positions); coherent
// loads, since the score kernel may have written them while this grid was
// already resident.
// Every load is issued before any key is formed: the loads are volatile, so a
// branch on one loaded value between two loads would hold the next load back
// for a full round trip.
__device__ __forceinline__ void ix_load_chunk(const float *sc, const IxChunk &ck,
                                              uint32_t (&key)[kIxSelIlp]) {
    float v[kIxSelIlp];
#pragma unroll
    for (int j = 0; j < kIxSelIlp; ++j) {
        const int s = ck.s0 + j * kIxSelThreads + (int)threadIdx.x;
        v[j] = __ldcg(sc + min(s, ck.s1 - 1));   // ck.s1 > ck.s0: in range
    }
#pragma unroll
    for (int j = 0; j < kIxSelIlp; ++j) {
        const int s = ck.s0 + j * kIxSelThreads + (int)threadIdx.x;
        key[j] = s < ck.s1 ? ix_key(v[j]) : 0u;
    }
}

// Pass 1 over given scores, one CTA per (token, chunk): histogram of the
// first digit in shared memory, added into the token's global histogram.
// The scores are complete before the chain starts (stream order), so they
// are read before the wait; the global histogram (cleared by the
// predecessor) only after it.
__global__ void __launch_bounds__(kIxSelThreads) smla_ix_hist_kernel(const IndexerParams p) {
    __shared__ unsigned hist[kIxSelBins];
    ix_pdl_trigger();
    const int tid = threadIdx.x, nt = blockDim.x;
    const IxChunk ck = ix_chunk(p);
    if (ck.s0 >= ck.s1) return;
    uint32_t key[kIxSelIlp];
    ix_load_chunk(p.scores + (size_t)ck.u * p.score_stride, ck, key);
    for (int i = tid; i < kIxSelBins; i += nt) hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kIxSelIlp; ++j)
        if (key[j] != 0u) atomicAdd(&hist[key[j] >> 20], 1u);
    __syncthreads();
    ix_pdl_wait();
    unsigned *gh = p.sel_hist + (size_t)ck.u * kIxSelBins;
    for (int i = tid; i < kIxSelBins; i += nt) {
        const unsigned v = hist[i];
        if (v) atomicAdd(gh + i, v);
    }
}

// Pass 2, one CTA per (token, chunk): the crossing bucket from the token's
// histogram (every CTA of the token finds the same one; chunk 0 records it
// in meta); positions whose first digit is above it are selected (one bitmap
// word per warp step, written whole, so the bitmap needs no clearing); those
// in it are staged in shared memory and appended to the token's candidates
// with one reservation.  Scores are read before the wait only when they were
// complete before the chain started.
__global__ void __launch_bounds__(kIxSelThreads) smla_ix_mark_kernel(const IndexerParams p) {
    extern __shared__ __align__(16) uint8_t ix_smem[];
    uint2 *stage = reinterpret_cast<uint2 *>(ix_smem);
    __shared__ int scratch[kIxSelThreads / 32];
    __shared__ int dec[3];
    __shared__ int ccount, cbase;
    ix_pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31;
    const IxChunk ck = ix_chunk(p);
    if (ck.s0 >= ck.s1) return;
    const int u = ck.u;
    if (tid == 0) ccount = 0;
    const float *sc = p.scores + (size_t)u * p.score_stride;
    uint32_t key[kIxSelIlp];
    if (p.sel_prefetch) ix_load_chunk(sc, ck, key);
    ix_pdl_wait();
    // the histogram's loads go out first: the scan needs them before the keys
    uint32_t bins[kIxSelBins / kIxSelThreads];
    ix_decide_load<kIxSelThreads>(p.sel_hist + (size_t)u * kIxSelBins, tid, bins);
    if (!p.sel_prefetch) ix_load_chunk(sc, ck, key);
    IxSelMeta *meta = p.sel_meta + u;
    ix_decide<kIxSelThreads>(bins, p.K, tid, scratch, dec, [] { __syncthreads(); });
    __syncthreads();   // dec[] complete (written by one thread)
    if (ck.s0 == 0 && tid == 0) {
        meta->take_all = dec[0];
        meta->d0 = dec[1];
        meta->need = dec[2];
    }
    const bool take_all = dec[0] != 0;
    const uint32_t d0 = (uint32_t)dec[1];
    uint32_t *bits = p.sel_bits + (size_t)u * p.sel_words;
#pragma unroll
    for (int j = 0; j < kIxSelIlp; ++j) {
        const int s = ck.s0 + j * kIxSelThreads + tid;   // a warp covers 32 consecutive positions
        const uint32_t d = key[j] >> 20;
        const bool above = key[j] != 0u && (take_all || d > d0);
        const bool is_cand = key[j] != 0u && !take_all && d == d0;
        const uint32_t word = __ballot_sync(0xffffffffu, above);
        if (lane == 0 && s < ck.s1) bits[s >> 5] = word;
        const uint32_t cm = __ballot_sync(0xffffffffu, is_cand);
        if (cm) {
            int slot0 = 0;
            if (lane == 0) slot0 = atomicAdd(&ccount, __popc(cm));
            slot0 = __shfl_sync(0xffffffffu, slot0, 0);
            if (is_cand) stage[slot0 + __popc(cm & ((1u << lane) - 1u))] = make_uint2(key[j], (uint32_t)s);
        }
    }
    __syncthreads();
    const int m = ccount;
    if (m == 0) return;
    if (tid == 0) cbase = atomicAdd(&meta->count, m);
    __syncthreads();
    uint2 *cand = p.sel_cand + (size_t)u * p.max_n + cbase;
    for (int i = tid; i < m; i += kIxSelThreads) cand[i] = stage[i];
}

// Pass 3, one CTA per token: two 10-bit digits over the candidates (held in
// shared memory when they fit, else re-read) give the exact threshold key and
// how many keys equal to it are taken; the first of those by position come
// from an ordered scan of an "equal" bitmap; an ordered scan of the selection
// bitmap writes the output.
__global__ void __launch_bounds__(kIxFinishThreads) smla_ix_finish_kernel(const IndexerParams p) {
    extern __shared__ __align__(16) uint8_t ix_smem[];
    uint32_t *cand_key = reinterpret_cast<uint32_t *>(ix_smem);
    int *cand_pos = reinterpret_cast<int *>(ix_smem + kIxCandCap * 4);
    unsigned *hist = reinterpret_cast<unsigned *>(ix_smem + kIxCandCap * 8);
    uint32_t *sel = reinterpret_cast<uint32_t *>(ix_smem + kIxCandCap * 8 + kIxFineBins * 4);
    __shared__ int scratch[33];
    __shared__ int found[2];
    const int u = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int n = ix_visible(p, u), K = p.K;
    int *out = p.out + (size_t)u * K;
    ix_pdl_wait();
    if (n == 0) {
        for (int i = tid; i < K; i += nt) out[i] = -1;
        return;
    }
    const int words = (n + 31) / 32;
    uint32_t *eq = sel + words;
    const IxSelMeta meta = p.sel_meta[u];
    const uint32_t *gbits = p.sel_bits + (size_t)u * p.sel_words;
    const uint2 *gcand = p.sel_cand + (size_t)u * p.max_n;
    for (int i = tid; i < words; i += nt) {  // independent of meta: first
        sel[i] = gbits[i];
        eq[i] = 0u;
    }
    const int m = meta.take_all ? 0 : meta.count;
    const bool in_smem = m <= kIxCandCap;
    if (in_smem) {
        for (int c = tid; c < m; c += nt) {
            const uint2 e = gcand[c];
            cand_key[c] = e.x;
            cand_pos[c] = (int)e.y;
        }
    }
    if (!meta.take_all) {
        int need = meta.need, n_eq = 0;
        uint32_t prefix = (uint32_t)meta.d0;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 10 : 0, hi_shift = shift + 10;
            for (int i = tid; i < kIxFineBins; i += nt) hist[i] = 0;
            __syncthreads();
            for (int c = tid; c < m; c += nt) {
                const uint32_t key = in_smem ? cand_key[c] : gcand[c].x;
                if ((key >> hi_shift) == prefix) atomicAdd(&hist[(key >> shift) & 1023u], 1u);
            }
            __syncthreads();
            ix_find_bucket(hist, kIxFineBins, need, scratch, found);
            prefix = (prefix << 10) | (uint32_t)found[0];
            need -= found[1];
            if (pass == 1) n_eq = (int)hist[found[0] & (kIxFineBins - 1)];   // keys equal to the threshold
        }
        const uint32_t thresh = prefix;
        const bool all_eq = n_eq == need;   // no tie to break by position
        for (int c = tid; c < m; c += nt) {
            uint32_t key;
            int s;
            if (in_smem) {
                key = cand_key[c];
                s = cand_pos[c];
            } else {
                const uint2 e = gcand[c];
                key = e.x;
                s = (int)e.y;
            }
            if (key > thresh || (all_eq && key == thresh)) atomicOr(&sel[s >> 5], 1u << (s & 31));
            else if (key == thresh) atomicOr(&eq[s >> 5], 1u << (s & 31));
        }
        __syncthreads();
        if (!all_eq)
            ix_bitmap_scan(eq, words, scratch, [&](int rank, int s) {
                if (rank < need) atomicOr(&sel[s >> 5], 1u << (s & 31));
            });
    }
    __syncthreads();
    const int taken = ix_bitmap_scan(sel, words, scratch, [&](int rank, int s) {
        if (rank < K) out[rank] = s;
    });
    for (int i = min(taken, K) + tid; i < K; i += nt) out[i] = -1;
}

}  // namespace smla
