// smla_partial_tc.cuh -- split-K partial pass on the 5th-generation tensor
// core (tcgen05 + TMEM) for query tokens with up to 64 heads.
//
// "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
// Decode", section "The Split-K Imperative": tensor-core (MMA) attention over
// the top-k candidate rows, split-K over that axis, partials merged by LSE.
//
// A CTA walks a list of work items.  An item is a run of one query token's
// list entries written as one partial slot: with equal splits the CTA's one
// (token, split); under the balanced schedule of the whole decode an equal
// share of the flattened (token, 32-row tile) space, which may cover the end
// of one token and the start of the next ("The Occupancy Hypothesis ...",
// section "The Occupancy Insight": every SM should have blocks in flight).
// In dense mode an item packs up to 64 / H query tokens of one sequence.  All
// heads of an item are the MMA's M = 64 rows (heads past the item's real rows
// are zero rows of Q and are never written out).
//
// 512 threads (16 warps x 128 registers: the whole register file):
//   warps 0-3  softmax warpgroup: stages the item's Q into TMEM (the score
//              MMA's A operand) -- the next item's Q as soon as the last score
//              MMA of the current item has completed -- then per PAIR of
//              32-row tiles reads S from TMEM, masks, keeps a running max per
//              head with lazy rescaling (O is rescaled only when the max grows
//              by more than 2^8), writes P as bf16 into each tile's spent k_pe
//              box; at an item's end drains O (partials through the item's
//              last ring slot, whole 128-B segments per store) and hands that
//              slot back to the producers.
//   warps 4-14 producers: resolve list entries to cache rows, then gather each
//              32-row tile with 16-byte cp.async copies written straight into
//              the 128B-swizzled K-major layout (each warp instruction moves
//              4 rows x 128 B); completion reaches the tile's mbarrier through
//              cp.async.mbarrier.arrive.  Padding slots copy row 0 and are
//              masked.  A pair never spans two items: an item with an odd
//              tile count ends in a pair whose second tile is empty.
//   warp 15    TMEM owner + MMA issuer (one thread):
//                QK(pair): S[64 x 64] = Q[64 x 576] [K_2p K_2p+1]^T   36 x (M64 N64 K16), A in TMEM
//                PV(t):    O[64 x 512] += P_t[64 x 32] C_t[32 x 512]  2 x 2 x (M64 N256 K16)
//              An M64 N64 MMA costs ~45 cycles whatever N below 64, so a
//              pair's two tiles share one N = 64 score MMA per k-step.  The
//              issuer polls: QK goes out in four chunks of nine k-steps, and a
//              pair whose P is ready gets its PV issued between chunks, so its
//              ring slot is freed without waiting for the next pair's scores.
// Shared memory ring: three pair slots of 2 x 36864 B; box b (64 columns) of
// tile h of a slot at slot + 8192 b + 4096 h, rows 128 B apart.
// TMEM (512 columns; an M = 64 operand or accumulator occupies lanes 0-15 of
// each 32-lane sub-partition, or 16-31 at lane offset 16; an A operand in
// TMEM must sit at its accumulator's lanes):
//   lanes 0-15   cols [0,288)    Q, two bf16 per column (A of QK)
//                cols 288+64b    S of pair b (b = pair mod 3), columns 0-31
//                                its first tile, 32-63 its second
//   lanes 16-31  cols [0,512)    O
// Softmax thread (warp q, lane l): head 16q + l % 16; lanes l and l + 16 take
// the pair's first and second tile, and the first and second 32 of each 64
// columns of O.
#pragma once

#include <climits>
#include <cstdint>
#include <cuda_bf16.h>

#include "smla_partial_mma.cuh"
#include "smla_tc_ptx.cuh"

namespace smla {

constexpr int kMaxTcRows = 64;  // query rows (the MMA's M) of one CTA

struct TcCfg {
#ifndef SMLA_TC_PRODUCER_WARPS
#define SMLA_TC_PRODUCER_WARPS 11
#endif
    static constexpr int kProducerWarps = SMLA_TC_PRODUCER_WARPS;
    static constexpr int kMmaWarp = 4 + kProducerWarps;
    static constexpr int kThreads = 32 * (kMmaWarp + 1);
    static constexpr int kTileRows = 32;
    static constexpr int kSlots = 3;                        // pair slots in the ring
    static constexpr int kStages = 2 * kSlots;              // tiles in the ring
    static constexpr int kSBufs = 3;                        // S accumulators in TMEM
    static constexpr int kQkChunk = 9;                      // score k-steps per issue burst
    static constexpr int kBoxBytes = kTileRows * 128;       // 4096: 32 rows x 64 bf16
    static constexpr int kBoxStride = 2 * kBoxBytes;        // 8192: the pair's two tiles per box
    static constexpr int kStageBytes = 9 * kBoxBytes;       // 36864 per tile
    static constexpr int kOffKV = 0;                        // Q lives in TMEM: the ring starts at 0
    static constexpr int kOffRows = kOffKV + kStages * kStageBytes;  // 221184
    static constexpr int kOffBar = kOffRows + kResolveChunk * 4;     // 229376
    // kv_full[6], kv_empty[6], s_full[3], p_full[3], o_done[2], q_ready, o_free
    static constexpr int kNumBars = kStages + kStages + kSBufs + kSBufs + 2 + 1 + 1;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffHdr = kOffTmem + 16;           // u32 [kStages]
    static constexpr int kBytes = kOffHdr + 4 * kStages;
    static constexpr int kSmemBytes = kBytes + 1024;        // + alignment slack for 1024-B atoms
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kQCol = 0;
    static constexpr uint32_t kSCol = 288;
    static constexpr uint32_t kOLane = 16;
    __host__ __device__ static constexpr int tile_off(int stage) {  // tile base inside the ring
        return (stage >> 1) * 2 * kStageBytes + (stage & 1) * kBoxBytes;
    }
    static constexpr float kTau = 8.0f;                     // lazy-rescale threshold (log2 units)
};
static_assert(TcCfg::kSmemBytes <= 232448, "shared memory per CTA");
static_assert(TcCfg::kSCol + 64 * TcCfg::kSBufs <= TcCfg::kTmemCols, "TMEM columns");
static_assert(kResolveChunk % 64 == 0, "a resolve chunk holds whole pairs");

// One work item of the tcgen05 kernel (see the header comment).
struct TcItem {
    int bt, j0, j1, slot;
    bool last;            // balanced schedule: the item ends its token
    long long row0;       // global query row of M row 0
    int nrows;            // real M rows
    int b, tok0, ntok;    // sequence; dense: first packed token, tokens packed
    __device__ __forceinline__ int n_tiles() const { return (j1 - j0 + 31) / 32; }
    __device__ __forceinline__ int n_pairs() const { return (n_tiles() + 1) / 2; }
};

__device__ __forceinline__ bool tc_next_item(const PartialParams &p, int cta, long long &u,
                                             TcItem &it) {
    WorkItem w;
    if (!next_item(p, cta, u, w)) return false;
    it.bt = w.bt;
    it.j0 = w.j0;
    it.j1 = w.j1;
    it.slot = w.slot;
    it.last = w.last;
    it.b = w.bt / p.T;
    if (p.seq_lens != nullptr) {
        it.tok0 = (w.bt - it.b * p.T) * p.pack;
        it.ntok = min(p.pack, p.dense_t - it.tok0);
        it.row0 = ((long long)it.b * p.dense_t + it.tok0) * p.dense_h;
        it.nrows = it.ntok * p.dense_h;
    } else {
        it.tok0 = 0;
        it.ntok = 0;
        it.row0 = (long long)w.bt * p.H;
        it.nrows = p.H;
    }
    return true;
}

// Dense mode: the item's list is positions [0, n_unit), the longest visible
// length of its tokens, each clamped to [0, K].
__device__ __forceinline__ int tc_dense_extent(const PartialParams &p, const TcItem &it) {
    int n_unit = 0;
    for (int t = 0; t < it.ntok; ++t)
        n_unit = max(n_unit, min(max(__ldg(p.seq_lens + (size_t)it.b * p.dense_t + it.tok0 + t), 0), p.K));
    return n_unit;
}

// List entries [j0 + base, j0 + base + n) of an item -> cache rows in rows_s
// (threads tid, tid + nthreads, ...).  Dense mode: entry j is position j,
// visible up to n_unit.
__device__ __forceinline__ void tc_resolve(const PartialParams &p, const TcItem &it, int base, int n,
                                           int n_unit, int *rows_s, int tid, int nthreads) {
    if (p.seq_lens == nullptr) {
        resolve_rows<4>(p, it.bt, it.j0, base, n, rows_s, tid, nthreads);
        return;
    }
    const int *pt_b = p.page_table + (size_t)it.b * p.pt_stride;
    const long long max_pos = (long long)p.pt_stride * kPage;
    for (int j = tid; j < n; j += nthreads) {
        const int pos = it.j0 + base + j;
        int row = -1;
        if (pos < n_unit) {
            const int pg = (long long)pos < max_pos ? __ldg(pt_b + (pos >> 6)) : -1;
            if ((long long)pos < max_pos && pg >= 0 && (long long)pg < p.num_pages) {
                row = pg * kPage + (pos & (kPage - 1));
            } else {
                atomicOr(&g_status_flags, kFlagIndexRange);
                atomicAdd(&g_bad_index_count, 1ull);
            }
        }
        rows_s[j] = row;
    }
}

// Q of an item (rows past the item's real rows are zero) into TMEM lanes 0-15
// of each sub-partition, the QK MMA's A operand: row hrow at lane hrow % 16 of
// sub-partition hrow / 16, 32-bit column j = bf16 elements 2j, 2j+1.  Thread t
// of the warpgroup writes columns 64 i + 32 (t / 16) + [0, 32) for i < 4,
// then 256 + 16 (t / 16) + [0, 16).
__device__ __forceinline__ void tc_stage_q(const PartialParams &p, const TcItem &it, uint32_t t_lane,
                                           int hrow, int half) {
    const bool real = hrow < it.nrows;
    const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((size_t)it.row0 + (real ? hrow : 0)) * kD);
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
        uint32_t w[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint4 v = real ? __ldg(qrow + 16 * i + 8 * half + k) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * k] = v.x;
            w[4 * k + 1] = v.y;
            w[4 * k + 2] = v.z;
            w[4 * k + 3] = v.w;
        }
        tmem_st16x2_32(t_lane + TcCfg::kQCol + 64 * i, w);
    }
    uint32_t w[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint4 v = real ? __ldg(qrow + 64 + 4 * half + k) : make_uint4(0u, 0u, 0u, 0u);
        w[4 * k] = v.x;
        w[4 * k + 1] = v.y;
        w[4 * k + 2] = v.z;
        w[4 * k + 3] = v.w;
    }
    tmem_st16x2_16(t_lane + TcCfg::kQCol + 256, w);
}

template <bool DIRECT>
__global__ void __launch_bounds__(TcCfg::kThreads, 1)
    smla_partial_tc_kernel(const PartialParams p) {
    using C = TcCfg;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (128B-swizzle atoms are 8 rows x 128 B).
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const bool dense = p.seq_lens != nullptr;
    bool dead = false;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + C::kStages;
    uint64_t *s_full = bars + 2 * C::kStages;
    uint64_t *p_full = s_full + C::kSBufs;
    uint64_t *o_done = p_full + C::kSBufs;  // [pair parity]: PV of that pair complete
    uint64_t *q_ready = o_done + 2;         // phase k: the k-th item's Q is in TMEM
    uint64_t *o_free = q_ready + 1;         // phase k: the k-th item's O is drained
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);
    volatile uint32_t *hdr = reinterpret_cast<volatile uint32_t *>(smem + C::kOffHdr);
    int *rows_s = reinterpret_cast<int *>(smem + C::kOffRows);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            // 32 cp.async arrivals per producer warp + one plain arrive that
            // publishes the tile's validity mask
            mbar_init(&kv_full[i], 32 * C::kProducerWarps + 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < C::kSBufs; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
        }
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        mbar_init(q_ready, 4);
        mbar_init(o_free, 1);
        fence_mbar_init();
    }
    if (warp == C::kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // Every thread helps resolve the first chunk of the first item, so that
    // the first copies start after two memory round trips.
    {
        long long u0 = item_begin(p, cta);
        TcItem it0;
        if (tc_next_item(p, cta, u0, it0)) {
            const int n_unit = dense ? tc_dense_extent(p, it0) : 0;
            tc_resolve(p, it0, 0, min(kResolveChunk, it0.j1 - it0.j0), n_unit, rows_s, threadIdx.x,
                       C::kThreads);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);
    const uint32_t sbase = smem_addr(smem);

    if (warp >= 4 && warp < 4 + C::kProducerWarps) {
        // ============================================================ producers
        const int pw = warp - 4;
        const int ptid = threadIdx.x - 128;  // 0 .. 32 * kProducerWarps - 1
        constexpr int kPT = 32 * C::kProducerWarps;
        // Padding slots copy cache row 0 (always in range) and are masked to
        // probability 0 by the softmax, so they add 0 * row 0 to O.
        constexpr int kPadRow = 0;
        const uint8_t *cache = reinterpret_cast<const uint8_t *>(p.cache);
        const uint32_t bar_prod = 1;  // named barrier of the producer warps
        long long u = item_begin(p, cta);
        TcItem it;
        int gp = 0;               // pair counter over all items (ring position)
        bool first_chunk = true;  // resolved by the whole CTA
        while (tc_next_item(p, cta, u, it)) {
            int n_unit = 0;
            if (dense) {
                n_unit = tc_dense_extent(p, it);
                // split 0 counts a length outside [0, K] once per token
                for (int t = 0; t < it.ntok; ++t) {
                    const int raw = __ldg(p.seq_lens + (size_t)it.b * p.dense_t + it.tok0 + t);
                    if (it.slot == 0 && ptid == t && (raw < 0 || raw > p.K)) {
                        atomicOr(&g_status_flags, kFlagIndexRange);
                        atomicAdd(&g_bad_index_count, 1ull);
                    }
                }
            }
            const int len = it.j1 - it.j0;
            for (int base = 0; base < len; base += kResolveChunk) {
                const int n = min(kResolveChunk, len - base);
                if (!first_chunk) {
                    named_bar_sync(bar_prod, kPT);  // rows_s free for rewriting
                    tc_resolve(p, it, base, n, n_unit, rows_s, ptid, kPT);
                    named_bar_sync(bar_prod, kPT);  // rows_s complete
                }
                first_chunk = false;
                const int chunk_tiles = (n + C::kTileRows - 1) / C::kTileRows;
                for (int cp = 0; cp < (chunk_tiles + 1) / 2; ++cp, ++gp) {
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        const int stage = 2 * (gp % C::kSlots) + h;
                        if (gp >= C::kSlots) mbar_wait(&kv_empty[stage], ((gp / C::kSlots) - 1) & 1, dead);
                        const int t = 2 * cp + h;  // tile of the chunk; t == chunk_tiles: empty
                        if (t < chunk_tiles) {
                            uint8_t *dst = smem + C::kOffKV + C::tile_off(stage);
                            // 72 warp instructions per tile, each 4 rows x 128 B; warp pw
                            // takes every kProducerWarps-th from i = pw
#pragma unroll 2
                            for (int i = pw; i < 72; i += C::kProducerWarps) {
                                const int seg = 4 * i + (lane >> 3);  // 0..287: row r, column box
                                const int r = seg / 9, box = seg - 9 * r, ch = lane & 7;
                                const int j = t * C::kTileRows + r;
                                const int row = (j < n) ? rows_s[j] : -1;
                                const uint8_t *src = cache + (size_t)(row >= 0 ? row : kPadRow) * kRowBytes +
                                                     box * 128 + ch * 16;
                                const uint32_t d =
                                    smem_addr(dst + box * C::kBoxStride + r * 128 + ((ch ^ (r & 7)) << 4));
                                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src)
                                             : "memory");
                            }
                        }
                        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                                         smem_addr(&kv_full[stage]))
                                     : "memory");
                        if (pw == 0) {
                            const int j = t * C::kTileRows + lane;
                            const uint32_t vmask =
                                __ballot_sync(0xffffffffu, t < chunk_tiles && j < n && rows_s[j] >= 0);
                            if (lane == 0) {
                                hdr[stage] = vmask;
                                mbar_arrive(&kv_full[stage]);  // release: hdr is visible to the waiters
                            }
                        }
                    }
                }
            }
        }
        // Copies still in flight must land before the CTA may exit.
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == C::kMmaWarp) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 64, false, false);
            constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256, false, true);
            // total pairs of this CTA
            int total = 0;
            {
                long long uc = item_begin(p, cta);
                TcItem tmp;
                while (tc_next_item(p, cta, uc, tmp)) total += tmp.n_pairs();
            }
            // QK cursor and PV cursor walk the same pair sequence
            long long uq = item_begin(p, cta), uv = item_begin(p, cta);
            TcItem iq, iv;
            bool hq = tc_next_item(p, cta, uq, iq), hv = tc_next_item(p, cta, uv, iv);
            int q_item = 0, q_pair = 0, v_item = 0, v_pair = 0;
            int qk_next = 0, pv_next = 0, qk_chunk = 0;
            bool idle = false;
            uint64_t idle_since = 0;
            while (pv_next < total && !dead) {
                bool progressed = false;
                // ---- PV first: a pair whose P is written frees its ring slot
                if (hv && pv_next < qk_next &&
                    mbar_test_wait(&p_full[pv_next % C::kSBufs], (pv_next / C::kSBufs) & 1) &&
                    (v_pair > 0 || v_item == 0 || mbar_test_wait(o_free, (v_item - 1) & 1))) {
                    tc_fence_after();
                    const int gp = pv_next;
                    const int n_tiles = iv.n_tiles();
                    const bool last_pair = v_pair == iv.n_pairs() - 1;
                    for (int h = 0; h < 2 && 2 * v_pair + h < n_tiles; ++h) {
                        const int stage = 2 * (gp % C::kSlots) + h;
                        const uint32_t kv_addr = sbase + C::kOffKV + C::tile_off(stage);
                        const uint32_t p_addr = kv_addr + 8 * C::kBoxStride;
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint32_t acc = (v_pair > 0 || h > 0 || kk > 0) ? 1u : 0u;
                            const uint64_t a = smem_desc(p_addr + kk * 32, 16, 512, kSwizzle64B);
                            const uint64_t blo = smem_desc(kv_addr + kk * 2048, C::kBoxStride, 1024,
                                                           kSwizzle128B);
                            const uint64_t bhi = smem_desc(kv_addr + 4 * C::kBoxStride + kk * 2048,
                                                           C::kBoxStride, 1024, kSwizzle128B);
                            umma_bf16(tmem + (C::kOLane << 16), a, blo, kIdescPV, acc);
                            umma_bf16(tmem + (C::kOLane << 16) + 256, a, bhi, kIdescPV, acc);
                        }
                    }
                    // an item's last pair keeps its slot: the softmax warps drain
                    // O through it and hand it back themselves
                    if (!last_pair) {
                        umma_commit(&kv_empty[2 * (gp % C::kSlots)]);
                        umma_commit(&kv_empty[2 * (gp % C::kSlots) + 1]);
                    }
                    umma_commit(&o_done[gp & 1]);
                    ++pv_next;
                    if (++v_pair == iv.n_pairs()) {
                        v_pair = 0;
                        ++v_item;
                        hv = tc_next_item(p, cta, uv, iv);
                    }
                    progressed = true;
                }
                // ---- one chunk of a pair's score MMAs
                if (hq && qk_next < total && qk_next < pv_next + C::kSBufs) {
                    const int gp = qk_next;
                    bool ready = true;
                    if (qk_chunk == 0) {
                        ready = (q_pair > 0 || mbar_test_wait(q_ready, q_item & 1)) &&
                                mbar_test_wait(&kv_full[2 * (gp % C::kSlots)], (gp / C::kSlots) & 1) &&
                                mbar_test_wait(&kv_full[2 * (gp % C::kSlots) + 1], (gp / C::kSlots) & 1);
                        if (ready) {
                            // The tiles were written by cp.async (generic proxy); the
                            // MMA reads them through the async proxy.  An empty
                            // second tile holds stale rows: their scores are masked.
                            fence_proxy_async_smem();
                            tc_fence_after();
                        }
                    }
                    if (ready) {
                        const uint32_t kv_addr = sbase + C::kOffKV + C::tile_off(2 * (gp % C::kSlots));
                        const uint32_t d = tmem + C::kSCol + 64 * (gp % C::kSBufs);
#pragma unroll 3
                        for (int kk = qk_chunk * C::kQkChunk; kk < (qk_chunk + 1) * C::kQkChunk; ++kk) {
                            const uint32_t koff = (kk & 3) * 32;  // 16-element step inside the 128-B row
                            const uint32_t a = tmem + C::kQCol + 8 * kk;  // 16 bf16 = 8 columns of Q
                            const uint64_t bd = smem_desc(kv_addr + (kk >> 2) * C::kBoxStride + koff,
                                                          16, 1024, kSwizzle128B);
                            umma_bf16_ts(d, a, bd, kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        if (++qk_chunk == 36 / C::kQkChunk) {
                            umma_commit(&s_full[gp % C::kSBufs]);
                            qk_chunk = 0;
                            ++qk_next;
                            if (++q_pair == iq.n_pairs()) {
                                q_pair = 0;
                                ++q_item;
                                hq = tc_next_item(p, cta, uq, iq);
                            }
                        }
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = false;
                } else if (!idle) {
                    idle = true;
                    idle_since = global_timer_ns();
                } else if (global_timer_ns() - idle_since > kWaitLimitNs) {
                    atomicOr(&g_status_flags, kFlagTimeout);  // give up: every other wait is bounded too
                    dead = true;
                }
            }
        }
        __syncwarp();
    } else {
        // ============================================================ softmax warpgroup
        const int q4 = warp;          // TMEM sub-partition (lanes 32*q4 .. +31)
        const int hrow = 16 * q4 + (lane & 15);
        const int half = lane >> 4;
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q4) << 16);            // lanes 0-15: Q, S
        const uint32_t t_o = tmem + ((uint32_t)(32 * q4 + C::kOLane) << 16);  // lanes 16-31: O

        long long u = item_begin(p, cta);
        TcItem it;
        bool have = tc_next_item(p, cta, u, it);
        if (have) {
            tc_stage_q(p, it, t_lane, hrow, half);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        int gp = 0, k = 0;
        while (have) {
            long long un = u;
            TcItem next;
            const bool has_next = tc_next_item(p, cta, un, next);
            if (has_next) {  // the next item's Q into L2 ahead of its staging
                const uint8_t *qn = reinterpret_cast<const uint8_t *>(p.q + (size_t)next.row0 * kD);
                for (int i = threadIdx.x; i < next.nrows * 9; i += 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(qn + (size_t)i * 128));
            }
            const int n_tiles = it.n_tiles(), n_pairs = it.n_pairs();
            // dense: list entries visible to query row hrow (rows past the
            // item's real rows see none); sparse: no per-row limit
            int lim = INT_MAX;
            if (dense)
                lim = hrow < it.nrows ? min(max(__ldg(p.seq_lens + (size_t)it.b * p.dense_t + it.tok0 +
                                                      hrow / p.dense_h), 0), p.K)
                                      : 0;
            float m_ref = -INFINITY;  // running reference max of head hrow (log2 units)
            float l_acc = 0.f;        // this thread's tile's share of the sum of P of head hrow

            for (int pr = 0; pr < n_pairs; ++pr, ++gp) {
                const int t0 = 2 * pr;
                const bool has1 = t0 + 1 < n_tiles;
                const int st0 = 2 * (gp % C::kSlots);
                mbar_wait(&s_full[gp % C::kSBufs], (gp / C::kSBufs) & 1, dead);
                tc_fence_after();
                // S of the pair (TMEM lanes 0-15): thread t gets head hrow's scores
                // against tile t0 + t / 16 (columns 32 (t / 16) + [0, 32)), so the
                // two threads of a head split the pair's 64 columns
                uint32_t sv[32];
                tmem_ld16x2_32(t_lane + C::kSCol + 64 * (gp % C::kSBufs), sv);
                tmem_ld_wait();
                if (pr == n_pairs - 1 && has_next) {
                    // every score MMA of this item has completed: the next
                    // item's Q may replace this one in TMEM
                    tc_stage_q(p, next, t_lane, hrow, half);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(q_ready);
                }
                mbar_wait(&kv_full[st0], (gp / C::kSlots) & 1, dead);
                uint32_t vm = hdr[st0];
                mbar_wait(&kv_full[st0 + 1], (gp / C::kSlots) & 1, dead);
                const uint32_t vm1 = hdr[st0 + 1];
                if (half) vm = vm1;  // an empty second tile: every column masked
                if (dense) {  // this row's causal limit, as a mask over this tile's columns
                    const int r = lim - (it.j0 + (t0 + half) * C::kTileRows);
                    vm &= r >= 32 ? 0xffffffffu : (r <= 0 ? 0u : (1u << r) - 1u);
                }
                // scores in log2 units, padding -> -inf; selects, not branches
                float mt = -INFINITY;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float x = ((vm >> j) & 1u) ? __uint_as_float(sv[j]) * p.scale_log2 : -INFINITY;
                    sv[j] = __float_as_uint(x);
                    mt = fmaxf(mt, x);
                }
                // the pair's max of head hrow; both threads of the head then keep
                // the same reference max (same inputs, same steps)
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                float alpha = 1.f;
                if (mt > m_ref + C::kTau) {
                    alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mt);
                    m_ref = mt;
                }
                // Rescale the head's row of O when its max jumped (warp-collective
                // TMEM access; alpha = 1 for the other heads).
                const bool need = (pr >= 1) && (alpha != 1.f);
                if (__any_sync(0xffffffffu, need)) {
                    // O must hold PV of the previous pair before it is rescaled.
                    // PV of the pair after it needs this pair's P, so the parity
                    // wait cannot alias.
                    mbar_wait(&o_done[(gp - 1) & 1], ((gp - 1) >> 1) & 1, dead);
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 512; c += 64) {  // thread t: columns c + 32 (t / 16) + [0, 32)
                        uint32_t orr[32];
                        tmem_ld16x2_32(t_o + c, orr);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
                        tmem_st16x2_32(t_o + c, orr);
                    }
                    tmem_st_wait();
                }
                {
                    const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
                    float ps = 0.f;
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float a0 = fast_exp2(__uint_as_float(sv[2 * j]) - mu);  // exp2(-inf) = 0
                        const float a1 = fast_exp2(__uint_as_float(sv[2 * j + 1]) - mu);
                        ps += a0 + a1;
                        pk[j] = pack_bf16x2(a0, a1);
                    }
                    if (half == 0 || has1) {
                        // this tile's P (64 heads x 32 rows, bf16) in its spent k_pe
                        // box, K-major 64B swizzle
                        uint8_t *pbase = smem + C::kOffKV + C::tile_off(st0 + half) + 8 * C::kBoxStride;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4 *>(pbase + hrow * 64 + ((c ^ ((hrow >> 1) & 3)) << 4)) =
                                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    }
                    l_acc = l_acc * alpha + ps;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[gp % C::kSBufs]);
            }

            // ---- end of the item: O (unnormalised) and m, lse of head hrow
            const int gp_last = gp - 1;  // the item's last pair (n_pairs == 0: none)
            const float l_tot = l_acc + __shfl_xor_sync(0xffffffffu, l_acc, 16);
            if (n_pairs > 0) {
                mbar_wait(&o_done[gp_last & 1], (gp_last >> 1) & 1, dead);
                tc_fence_after();
            }
            const bool write = hrow < it.nrows;
            const size_t row = (size_t)it.row0 + hrow;
            // O of head hrow from TMEM lanes 16-31: thread t holds columns
            // c + 32 (t / 16) + [0, 32) per step.  Partials leave through shared
            // memory so that each store instruction writes whole 128-B row
            // segments.  Per warp, 32 lane-rows of 32 floats at a 144-B pitch
            // (conflict-free both ways), in the item's last ring slot: its
            // tiles have been consumed and the producers wait for it.
            constexpr int kPitch = 36;
            const int slot_base = C::tile_off(n_pairs > 0 ? 2 * (gp_last % C::kSlots) : 0);
            float *stage = reinterpret_cast<float *>(smem + C::kOffKV + slot_base) + warp * (32 * kPitch);
#pragma unroll 1
            for (int c = 0; c < 512; c += 64) {
                uint32_t orr[32];
                if (n_pairs > 0) {
                    tmem_ld16x2_32(t_o + c, orr);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) orr[j] = 0u;
                }
                const int col = c + 32 * half;
                if (!DIRECT) {
                    float4 *mine = reinterpret_cast<float4 *>(stage + lane * kPitch);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        mine[j] = make_float4(__uint_as_float(orr[4 * j]), __uint_as_float(orr[4 * j + 1]),
                                              __uint_as_float(orr[4 * j + 2]), __uint_as_float(orr[4 * j + 3]));
                    __syncwarp();
                    // eight lanes per lane-row, four lane-rows per instruction
#pragma unroll
                    for (int kq = 0; kq < 8; ++kq) {
                        const int lr = 4 * kq + (lane >> 3);  // lane-row: lane lr's head and columns
                        const int ch = lane & 7;              // 16-B chunk of its 128-B segment
                        const int hr = 16 * q4 + (lr & 15);
                        if (hr < it.nrows) {
                            const float4 v = *reinterpret_cast<const float4 *>(stage + lr * kPitch + 4 * ch);
                            *reinterpret_cast<float4 *>(p.part_o + (((size_t)it.row0 + hr) * p.nsplit + it.slot) * kDc +
                                                        c + 32 * (lr >> 4) + 4 * ch) = v;
                        }
                    }
                    __syncwarp();
                } else if (write) {
                    const float inv = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + row * kDc + col);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_uint4(
                            pack_bf16x2(__uint_as_float(orr[8 * j]) * inv, __uint_as_float(orr[8 * j + 1]) * inv),
                            pack_bf16x2(__uint_as_float(orr[8 * j + 2]) * inv, __uint_as_float(orr[8 * j + 3]) * inv),
                            pack_bf16x2(__uint_as_float(orr[8 * j + 4]) * inv, __uint_as_float(orr[8 * j + 5]) * inv),
                            pack_bf16x2(__uint_as_float(orr[8 * j + 6]) * inv, __uint_as_float(orr[8 * j + 7]) * inv));
                }
            }
            if (write && half == 0) {
                const float lse_v = (l_tot > 0.f) ? (m_ref + log2f(l_tot)) * kLn2 : -INFINITY;
                if (!DIRECT) {
                    const size_t kx = row * p.nsplit + it.slot;
                    p.part_m[kx] = (l_tot > 0.f) ? m_ref * kLn2 : -INFINITY;
                    p.part_lse[kx] = lse_v;
                } else {
                    p.lse[row] = lse_v;
                }
            }
            if (!DIRECT) {
                WorkItem wi;
                wi.bt = it.bt;
                wi.j0 = it.j0;
                wi.j1 = it.j1;
                wi.slot = it.slot;
                wi.last = it.last;
                mark_unused_slots(p, wi, threadIdx.x, 128);
            }
            // O is read out and the staging slot is free: the next item's PV
            // may overwrite O, the producers may refill the slot
            tc_fence_before();
            named_bar_sync(2, 128);
            if (threadIdx.x == 0) {
                mbar_arrive(o_free);
                if (n_pairs > 0) {
                    mbar_arrive(&kv_empty[2 * (gp_last % C::kSlots)]);
                    mbar_arrive(&kv_empty[2 * (gp_last % C::kSlots) + 1]);
                }
            }
            it = next;
            u = un;
            have = has_next;
            ++k;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == C::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace smla
