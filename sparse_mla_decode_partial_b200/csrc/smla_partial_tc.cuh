// smla_partial_tc.cuh -- split-K partial pass on the 5th-generation tensor
// core (tcgen05 + TMEM) for query tokens with up to 64 heads.
//
// "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
// Decode", section "The Split-K Imperative": tensor-core (MMA) attention over
// the top-k candidate rows, split-K over that axis, partials merged by LSE.
//
// One CTA = one (query token, split), all heads (M = 64 rows of the MMA;
// heads >= H are zero rows of Q and are never written out), or in dense mode
// up to 64 / H query tokens of one sequence.  512 threads (16 warps x 128
// registers: the whole register file):
//   warps 0-3  softmax warpgroup: stages Q into TMEM once (it is the QK
//              MMA's A operand), then per PAIR of 32-row tiles reads S from
//              TMEM (tcgen05.ld), masks, keeps a running max per head with
//              lazy rescaling (O is only rescaled when the max grows by more
//              than 2^8), writes P as bf16 into each tile's spent k_pe box,
//              and finally drains O (partials through shared memory, whole
//              128-B segments per store).
//   warps 4-14 producers: resolve the split's indices to rows (as the mma
//              kernel does), then gather each 32-row tile with 16-byte
//              cp.async copies written straight into the 128B-swizzled
//              K-major layout (each warp instruction moves 4 rows x 128 B,
//              coalesced); completion reaches the tile's mbarrier through
//              cp.async.mbarrier.arrive.  Padding slots are zero-filled (nothing read) and are
//              masked.  In dense mode a tile of 32 consecutive cache rows
//              moves instead with nine TMA tile loads (32 rows x 64 values,
//              128B swizzle) on the same barrier.
//   warp 15    TMEM owner + MMA issuer (one thread):
//                QK(pair): S[64 x 64] = Q[64 x 576] [K_2p K_2p+1]^T   36 x (M64 N64 K16), A in TMEM
//                PV(t):    O[64 x 512] += P_t[64 x 32] C_t[32 x 512]  2 x 2 x (M64 N256 K16)
//              A tcgen05 MMA costs at least ~46 cycles whatever its size
//              below M64 N64 (M64 N32 costs the same as M64 N64), so the
//              two tiles of a pair share one N = 64 score MMA per k-step: the
//              ring keeps the pair's tiles side by side in every 64-column
//              box.  The 36 score MMAs of a pair go out as one burst from
//              descriptors built once per pair (rebuilding them per MMA, or
//              splitting the burst, left the tensor pipe waiting).  The
//              issuer polls: a pair's QK goes out as soon as both
//              tiles have landed, its PV as soon as its P is ready.
// Like the other partial kernels it is a programmatic dependent of what
// precedes it on the stream: it waits before touching global memory or tensor
// memory, and reads q, the indices, the lengths and the page table with weak
// global loads (ld_input), never through the read-only path.
// Shared memory ring: three pair slots of 2 x 36864 B (Q is not in shared
// memory); box b (64 columns) of tile h of a slot at slot + 8192 b + 4096 h,
// rows 128 B apart.
// TMEM (512 columns; an M = 64 operand or accumulator occupies lanes 0-15 of
// each 32-lane sub-partition, or 16-31 when addressed at lane offset 16; an A
// operand in TMEM must sit at its accumulator's lanes):
//   lanes 0-15   cols [0,288)    Q, two bf16 per column (A of QK)
//                cols 288+64b    S of pair b (b = pair parity, double
//                                buffered), columns 0-31 its first tile,
//                                32-63 its second
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
    static constexpr int kStages = 6;                       // tiles in the ring (3 pair slots)
    static constexpr int kBoxBytes = kTileRows * 128;       // 4096: 32 rows x 64 bf16
    static constexpr int kBoxStride = 2 * kBoxBytes;        // 8192: the pair's two tiles per box
    static constexpr int kStageBytes = 9 * kBoxBytes;       // 36864 per tile
    static constexpr int kOffKV = 0;                        // Q lives in TMEM: the ring starts at 0
    static constexpr int kOffRows = kOffKV + kStages * kStageBytes;  // 221184
    static constexpr int kOffBar = kOffRows + kResolveChunk * 4;     // 229376
    // barriers: kv_full[6], kv_empty[6], s_full[2], p_full[2], o_done[2], q_ready
    static constexpr int kNumBars = kStages + kStages + 2 + 2 + 2 + 1;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffHdr = kOffTmem + 16;           // u32 [kStages]
    static constexpr int kBytes = kOffHdr + 4 * kStages;
    static constexpr int kSmemBytes = kBytes + 1024;        // + alignment slack for 1024-B atoms
    static constexpr uint32_t kTmemCols = 512;
    // TMEM: Q (the QK MMA's A operand, two bf16 per column) at lanes 0-15 of
    // each sub-partition, columns [0, 288); S of a pair at the same lanes (an
    // A operand in TMEM must share the accumulator's lanes), columns 288 +
    // 64 * parity; O at lanes 16-31, columns [0, 512).
    static constexpr uint32_t kQCol = 0;
    static constexpr uint32_t kSCol = 288;
    static constexpr uint32_t kOLane = 16;
    __host__ __device__ static constexpr int tile_off(int stage) {  // tile base inside the ring
        return (stage >> 1) * 2 * kStageBytes + (stage & 1) * kBoxBytes;
    }
    static constexpr float kTau = 8.0f;                     // lazy-rescale threshold (log2 units)
};
static_assert(TcCfg::kSmemBytes <= 232448, "shared memory per CTA");

template <bool DIRECT>
__global__ void __launch_bounds__(TcCfg::kThreads, 1)
    smla_partial_tc_kernel(const PartialParams p, const __grid_constant__ CUtensorMap map_kv) {
    using C = TcCfg;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (128B-swizzle atoms are 8 rows x 128 B).
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x;  // (b * T + t) * S + s
    const int s = unit % p.nsplit;
    const int bt = unit / p.nsplit;
    const int b = bt / p.T;
    const long long j0l = (long long)s * p.kc;
    const int j0 = (int)(j0l < p.K ? j0l : p.K);
    const int j1 = (int)((long long)j0 + p.kc < p.K ? (long long)j0 + p.kc : p.K);
    const int n_tiles = (j1 - j0 + C::kTileRows - 1) / C::kTileRows;
    const int n_pairs = (n_tiles + 1) / 2;
    bool dead = false;
    // Query rows of this unit: global row of M row 0, and how many M rows are
    // real.  Sparse: the H heads of token bt.  Dense: the packed tokens' heads.
    const bool dense = p.seq_lens != nullptr;
    long long row0 = (long long)bt * p.H;
    int nrows = p.H;
    int tok0 = 0, ntok = 0;  // dense: first token of the unit (within sequence b), tokens in it
    if (dense) {
        tok0 = (bt - b * p.T) * p.pack;
        ntok = min(p.pack, p.dense_t - tok0);
        row0 = ((long long)b * p.dense_t + tok0) * p.dense_h;
        nrows = ntok * p.dense_h;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + C::kStages;
    uint64_t *s_full = bars + 2 * C::kStages;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_done = p_full + 2;  // [pair parity]: PV of that pair complete
    uint64_t *q_ready = o_done + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);
    volatile uint32_t *hdr = reinterpret_cast<volatile uint32_t *>(smem + C::kOffHdr);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            // 32 cp.async arrivals per producer warp + one plain arrive that
            // publishes the tile's validity mask
            mbar_init(&kv_full[i], 32 * C::kProducerWarps + 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
        }
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        mbar_init(q_ready, 4);
        fence_mbar_init();
    }
    // Launched as a programmatic dependent of whatever precedes it on the
    // stream: everything above touches only shared memory; from here on the
    // kernel reads global memory and takes tensor memory, so it first waits
    // for its predecessor to complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == C::kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
        const int *idx_bt = dense ? nullptr : p.idx + (size_t)bt * p.K + j0;
        // dense: the unit's list is positions [0, n_unit), the longest visible
        // length of its tokens (each clamped to [0, K]; split 0 counts a
        // length outside that range once per token)
        int n_unit = 0;
        if (dense) {
            for (int t = 0; t < ntok; ++t) {
                const int raw = ld_input(p.seq_lens + (size_t)b * p.dense_t + tok0 + t);
                n_unit = max(n_unit, min(max(raw, 0), p.K));
                if (s == 0 && ptid == t && (raw < 0 || raw > p.K)) {
                    atomicOr(&g_status_flags, kFlagIndexRange);
                    atomicAdd(&g_bad_index_count, 1ull);
                }
            }
        }
        const int *pt_b = p.page_table + (size_t)b * p.pt_stride;
        const long long max_pos = (long long)p.pt_stride * kPage;
        // Padding slots are zero-filled by the copy itself (source size 0:
        // nothing is read; the address stays that of row 0, always in range)
        // and are masked to probability 0 by the softmax.
        constexpr int kPadRow = 0;
        int *rows_s = reinterpret_cast<int *>(smem + C::kOffRows);
        const uint8_t *cache = reinterpret_cast<const uint8_t *>(p.cache);
        const uint32_t bar_prod = 1;  // named barrier of the producer warps
        const uint64_t evict_first = l2_policy_evict_first();  // rows are read once
        const uint32_t sbase_p = smem_addr(smem);
        const int len = j1 - j0;
        int it = 0;
        for (int base = 0; base < len; base += kResolveChunk) {
            const int n = min(kResolveChunk, len - base);
            named_bar_sync(bar_prod, 32 * C::kProducerWarps);  // rows_s free for rewriting
            for (int b0 = 0; b0 < n; b0 += kPT * 16) {
                int iv[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int j = b0 + k * kPT + ptid;
                    if (dense) {
                        const int pos = j0 + base + j;
                        iv[k] = (j < n && pos < n_unit) ? pos : -1;
                    } else {
                        iv[k] = (j < n) ? ld_input(idx_bt + base + j) : -1;
                    }
                }
                int pg[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int i = iv[k];
                    pg[k] = (i >= 0 && (long long)i < max_pos) ? ld_input(pt_b + (i >> 6)) : -1;
                }
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int j = b0 + k * kPT + ptid;
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
            named_bar_sync(bar_prod, 32 * C::kProducerWarps);  // rows_s complete
            const int chunk_tiles = (n + C::kTileRows - 1) / C::kTileRows;
            for (int t = 0; t < chunk_tiles; ++t, ++it) {
                const int stage = it % C::kStages;
                if (it >= C::kStages) mbar_wait(&kv_empty[stage], ((it / C::kStages) - 1) & 1, dead);
                uint8_t *dst = smem + C::kOffKV + C::tile_off(stage);
                // Dense lists walk whole pages: a tile of 32 consecutive cache rows
                // moves with nine TMA tile loads (32 rows x 64 values, 128B
                // swizzle) straight into the tile's boxes; the thread issuing them
                // adds their bytes to the barrier before its own arrival.
                bool bulk = false;
                if (dense && (t + 1) * C::kTileRows <= n) {
                    const int r0 = rows_s[t * C::kTileRows];
                    bulk = r0 >= 0 && rows_s[t * C::kTileRows + C::kTileRows - 1] == r0 + C::kTileRows - 1;
                    if (bulk && ptid == 0) {
                        mbar_expect_tx(&kv_full[stage], (uint32_t)C::kStageBytes);
#pragma unroll 1
                        for (int box = 0; box < 9; ++box)
                            tma_load_2d(sbase_p + C::kOffKV + C::tile_off(stage) + box * C::kBoxStride,
                                        &map_kv, box * 64, r0, &kv_full[stage], evict_first);
                    }
                }
                // 72 warp instructions per tile, each 4 rows x 128 B; warp pw takes every
                // kProducerWarps-th from i = pw
#pragma unroll 2
                for (int i = bulk ? 72 : pw; i < 72; i += C::kProducerWarps) {
                    const int seg = 4 * i + (lane >> 3);  // 0..287: row r, column box
                    const int r = seg / 9, box = seg - 9 * r, ch = lane & 7;
                    const int j = t * C::kTileRows + r;
                    const int row = (j < n) ? rows_s[j] : -1;
                    const uint8_t *src = cache + (size_t)(row >= 0 ? row : kPadRow) * kRowBytes +
                                         box * 128 + ch * 16;
                    const uint32_t d = smem_addr(dst + box * C::kBoxStride + r * 128 + ((ch ^ (r & 7)) << 4));
                    const uint32_t nbytes = row >= 0 ? 16u : 0u;
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(nbytes)
                                 : "memory");
                }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                                 smem_addr(&kv_full[stage]))
                             : "memory");
                if (pw == 0) {
                    const int j = t * C::kTileRows + lane;
                    const uint32_t vmask = __ballot_sync(0xffffffffu, j < n && rows_s[j] >= 0);
                    if (lane == 0) {
                        hdr[stage] = vmask;
                        mbar_arrive(&kv_full[stage]);  // release: hdr is visible to the waiters
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
            mbar_wait(q_ready, 0, dead);
            tc_fence_after();
            // Issue whatever is ready: a pair's QK as soon as its tiles have
            // landed (and its S buffer is free), a pair's PV as soon as its P
            // is written.  PV never waits behind the next pair's loads, so a
            // finished pair frees its slot immediately.  (Issuing blocks while
            // the tensor pipe is busy; splitting QK into chunks so that a
            // ready PV could slip in between measured no faster: it only moves
            // the wait onto the other slot.)
            int qk_next = 0, qk_landed = 0, pv_next = 0;
            bool idle = false;
            uint64_t idle_since = 0;
            while (pv_next < n_pairs && !dead) {
                bool progressed = false;
                if (qk_next < n_pairs && qk_next < pv_next + 2) {
                    const int tiles_in_pair = min(2, n_tiles - 2 * qk_next);
                    while (qk_landed < tiles_in_pair) {
                        const int t = 2 * qk_next + qk_landed;
                        if (!mbar_test_wait(&kv_full[t % C::kStages], (t / C::kStages) & 1)) break;
                        ++qk_landed;
                    }
                    if (qk_landed == tiles_in_pair) {
                        // The tiles were written by cp.async (generic proxy); the
                        // MMA reads them through the async proxy.  A pair with one
                        // tile reads a stale second half: its scores are masked.
                        fence_proxy_async_smem();
                        tc_fence_after();
                        const uint32_t kv_addr = sbase + C::kOffKV + C::tile_off((2 * qk_next) % C::kStages);
                        const uint32_t d = tmem + C::kSCol + 64 * (qk_next & 1);
                        // One descriptor built per pair; each k-step adds a constant
                        // to its address field (16-byte units; the ring's addresses
                        // stay below 2^18, so the 14-bit field never carries).  Building
                        // the descriptor inside the issue loop held back-to-back MMA
                        // issue: mixed took 60.4 us against 54.2 us this way.
                        const uint64_t bd0 = smem_desc(kv_addr, 16, 1024, kSwizzle128B);
#pragma unroll
                        for (int kk = 0; kk < 36; ++kk) {
                            // box kk / 4, 16-element step kk % 4 inside the 128-B row
                            const uint64_t bd = bd0 + (uint64_t)(((kk >> 2) * C::kBoxStride + (kk & 3) * 32) >> 4);
                            umma_bf16_ts(d, tmem + C::kQCol + 8 * kk, bd, kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&s_full[qk_next & 1]);
                        ++qk_next;
                        qk_landed = 0;
                        progressed = true;
                    }
                }
                if (pv_next < qk_next && mbar_test_wait(&p_full[pv_next & 1], (pv_next >> 1) & 1)) {
                    tc_fence_after();
                    const int pp = pv_next;
                    for (int t = 2 * pp; t < 2 * pp + 2 && t < n_tiles; ++t) {
                        const int stage = t % C::kStages;
                        const uint32_t kv_addr = sbase + C::kOffKV + C::tile_off(stage);
                        const uint32_t p_addr = kv_addr + 8 * C::kBoxStride;
                        const uint64_t a0 = smem_desc(p_addr, 16, 512, kSwizzle64B);
                        const uint64_t b0 = smem_desc(kv_addr, C::kBoxStride, 1024, kSwizzle128B);
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                            const uint64_t a = a0 + (uint64_t)((kk * 32) >> 4);
                            const uint64_t blo = b0 + (uint64_t)((kk * 2048) >> 4);
                            const uint64_t bhi = b0 + (uint64_t)((4 * C::kBoxStride + kk * 2048) >> 4);
                            umma_bf16(tmem + (C::kOLane << 16), a, blo, kIdescPV, acc);
                            umma_bf16(tmem + (C::kOLane << 16) + 256, a, bhi, kIdescPV, acc);
                        }
                        umma_commit(&kv_empty[stage]);
                    }
                    umma_commit(&o_done[pp & 1]);
                    ++pv_next;
                    progressed = true;
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

        // ---- stage Q (rows past the unit's real rows are zero) into TMEM, the
        // QK MMA's A operand: row hrow at lane hrow % 16 of this sub-partition,
        // 32-bit column j = bf16 elements 2j, 2j+1 (the row's own word order).
        // Thread t writes columns 64 i + 32 (t / 16) + [0, 32) for i < 4, then
        // 256 + 16 (t / 16) + [0, 16).
        {
            const bool real = hrow < nrows;
            const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((size_t)row0 + (real ? hrow : 0)) * kD);
#pragma unroll 1
            for (int i = 0; i < 4; ++i) {
                uint32_t w[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 v = real ? ld_input(qrow + 16 * i + 8 * half + k) : make_uint4(0u, 0u, 0u, 0u);
                    w[4 * k] = v.x;
                    w[4 * k + 1] = v.y;
                    w[4 * k + 2] = v.z;
                    w[4 * k + 3] = v.w;
                }
                tmem_st16x2_32(t_lane + C::kQCol + 64 * i, w);
            }
            {
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint4 v = real ? ld_input(qrow + 64 + 4 * half + k) : make_uint4(0u, 0u, 0u, 0u);
                    w[4 * k] = v.x;
                    w[4 * k + 1] = v.y;
                    w[4 * k + 2] = v.z;
                    w[4 * k + 3] = v.w;
                }
                tmem_st16x2_16(t_lane + C::kQCol + 256, w);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }

        // dense: list entries visible to query row hrow (rows past the unit's
        // real rows see none); sparse: no per-row limit
        int lim = INT_MAX;
        if (dense)
            lim = hrow < nrows ? min(max(ld_input(p.seq_lens + (size_t)b * p.dense_t + tok0 +
                                               hrow / p.dense_h), 0), p.K)
                               : 0;
        float m_ref = -INFINITY;  // running reference max of head hrow (log2 units)
        float l_acc = 0.f;        // this thread's tile's share of the sum of P of head hrow

        for (int pr = 0; pr < n_pairs; ++pr) {
            const int t0 = 2 * pr;
            const bool has1 = t0 + 1 < n_tiles;
            mbar_wait(&s_full[pr & 1], (pr >> 1) & 1, dead);
            tc_fence_after();
            // S of the pair (TMEM lanes 0-15): thread t gets head hrow's scores
            // against tile t0 + t / 16 (columns 32 (t / 16) + [0, 32)), so the
            // two threads of a head split the pair's 64 columns
            uint32_t sv[32];
            tmem_ld16x2_32(t_lane + C::kSCol + 64 * (pr & 1), sv);
            tmem_ld_wait();
            mbar_wait(&kv_full[t0 % C::kStages], (t0 / C::kStages) & 1, dead);
            uint32_t vm = hdr[t0 % C::kStages];
            uint32_t vm1 = 0;
            if (has1) {
                mbar_wait(&kv_full[(t0 + 1) % C::kStages], ((t0 + 1) / C::kStages) & 1, dead);
                vm1 = hdr[(t0 + 1) % C::kStages];
            }
            if (half) vm = vm1;  // an absent second tile: every column masked
            if (dense) {  // this row's causal limit, as a mask over this tile's columns
                const int r = lim - (j0 + (t0 + half) * C::kTileRows);
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
                // O must hold PV of pair pr-1 before it is rescaled.  The tensor
                // pipe runs in issue order and QK(pr) went out after PV(pr-2), so
                // PV(pr-3) is done and this parity wait cannot alias.
                mbar_wait(&o_done[(pr - 1) & 1], ((pr - 1) >> 1) & 1, dead);
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
                    uint8_t *pbase = smem + C::kOffKV + C::tile_off((t0 + half) % C::kStages) + 8 * C::kBoxStride;
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
            if (lane == 0) mbar_arrive(&p_full[pr & 1]);
        }

        // ---- epilogue: O (unnormalised) and m, lse of head hrow
        const float l_tot = l_acc + __shfl_xor_sync(0xffffffffu, l_acc, 16);
        if (n_pairs > 0) {
            mbar_wait(&o_done[(n_pairs - 1) & 1], ((n_pairs - 1) >> 1) & 1, dead);
            tc_fence_after();
        }
        const bool write = hrow < nrows;
        const size_t row = (size_t)row0 + hrow;
        // O of head hrow from TMEM lanes 16-31: thread t holds columns
        // c + 32 (t / 16) + [0, 32) per step.  Partials leave through shared
        // memory so that each store instruction writes whole 128-B row
        // segments (a direct store would touch 16 rows at once).  Per warp, 32
        // lane-rows of 32 floats at a 144-B pitch (conflict-free both ways),
        // in the ring: every tile has been consumed by now.
        constexpr int kPitch = 36;
        float *stage = reinterpret_cast<float *>(smem + C::kOffKV) + warp * (32 * kPitch);
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
                for (int k = 0; k < 8; ++k) {
                    const int lr = 4 * k + (lane >> 3);  // lane-row: lane lr's head and columns
                    const int ch = lane & 7;             // 16-B chunk of its 128-B segment
                    const int hr = 16 * q4 + (lr & 15);
                    if (hr < nrows) {
                        const float4 v = *reinterpret_cast<const float4 *>(stage + lr * kPitch + 4 * ch);
                        *reinterpret_cast<float4 *>(p.part_o + (((size_t)row0 + hr) * p.nsplit + s) * kDc +
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
                const size_t k = row * p.nsplit + s;
                p.part_m[k] = (l_tot > 0.f) ? m_ref * kLn2 : -INFINITY;
                p.part_lse[k] = lse_v;
            } else {
                p.lse[row] = lse_v;
            }
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
