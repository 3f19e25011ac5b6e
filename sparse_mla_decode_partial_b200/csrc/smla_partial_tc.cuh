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
//   warps 0-3  softmax warpgroup: stages Q (128B-swizzled) once, then per
//              PAIR of 32-row tiles reads S from TMEM (tcgen05.ld), masks,
//              keeps a running max per head with lazy rescaling (O is only
//              rescaled when the max grows by more than 2^8), writes P as bf16
//              into each tile's spent k_pe box, and finally drains O
//              (partials through shared memory, whole 128-B segments per
//              store).
//   warps 4-14 producers: resolve the split's indices to rows (as the mma
//              kernel does), then gather each 32-row tile with 16-byte
//              cp.async copies written straight into the 128B-swizzled
//              K-major layout (each warp instruction moves 4 rows x 128 B,
//              coalesced); completion reaches the tile's mbarrier through
//              cp.async.mbarrier.arrive.  Padding slots copy row 0 and are
//              masked.
//   warp 15    TMEM owner + MMA issuer (one thread):
//                QK(pair): S[64 x 64] = Q[64 x 576] [K_2p K_2p+1]^T   36 x (M64 N64 K16)
//                PV(t):    O[64 x 512] += P_t[64 x 32] C_t[32 x 512]  2 x 2 x (M64 N256 K16)
//              A tcgen05 MMA costs at least ~46 cycles whatever its size
//              below M64 N64 (M64 N32 costs the same as M64 N64), so the
//              two tiles of a pair share one N = 64 score MMA per k-step: the
//              ring keeps the pair's tiles side by side in every 64-column
//              box.  The issuer polls: a pair's QK goes out as soon as both
//              tiles have landed, its PV as soon as its P is ready.
// Shared memory ring: two pair slots of 2 x 36864 B; box b (64 columns) of
// tile h of a slot at slot + 8192 b + 4096 h, rows 128 B apart.
// TMEM (512 columns; M = 64 accumulators occupy lanes 0-15 of each 32-lane
// sub-partition, or 16-31 when addressed at lane offset 16):
//   cols [0,256)   lane off 0: O[:, 0:256]     lane off 16: O[:, 256:512]
//   cols 256+64b   lane off 0: S of pair b (b = pair parity, double buffered),
//                  columns 0-31 its first tile, 32-63 its second
// Softmax thread (warp q, lane l): lanes 0-15 own head 16q + l and do the
// pair's softmax; lane l + 16 rescales the second half of the same head's O.
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
    static constexpr int kStages = 4;                       // tiles in the ring (2 pair slots)
    static constexpr int kBoxBytes = kTileRows * 128;       // 4096: 32 rows x 64 bf16
    static constexpr int kBoxStride = 2 * kBoxBytes;        // 8192: the pair's two tiles per box
    static constexpr int kStageBytes = 9 * kBoxBytes;       // 36864 per tile
    static constexpr int kQBoxBytes = 64 * 128;             // 8192
    static constexpr int kOffQ = 0;                         // 9 x 8192
    static constexpr int kOffKV = 9 * kQBoxBytes;           // 73728
    static constexpr int kOffRows = kOffKV + kStages * kStageBytes;  // 221184
    static constexpr int kOffBar = kOffRows + kResolveChunk * 4;     // 229376
    // barriers: kv_full[4], kv_empty[4], s_full[2], p_full[2], o_done[2], q_ready
    static constexpr int kNumBars = 4 + 4 + 2 + 2 + 2 + 1;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kOffHdr = kOffTmem + 16;           // u32 [4]
    static constexpr int kBytes = kOffHdr + 16;
    static constexpr int kSmemBytes = kBytes + 1024;        // + alignment slack for 1024-B atoms
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kSCol = 256;
    __host__ __device__ static constexpr int tile_off(int stage) {  // tile base inside the ring
        return (stage >> 1) * 2 * kStageBytes + (stage & 1) * kBoxBytes;
    }
    static constexpr float kTau = 8.0f;                     // lazy-rescale threshold (log2 units)
};
static_assert(TcCfg::kSmemBytes <= 232448, "shared memory per CTA");

template <bool DIRECT>
__global__ void __launch_bounds__(TcCfg::kThreads, 1)
    smla_partial_tc_kernel(const PartialParams p) {
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
    uint64_t *kv_empty = bars + 4;
    uint64_t *s_full = bars + 8;
    uint64_t *p_full = bars + 10;
    uint64_t *o_done = bars + 12;  // [pair parity]: PV of that pair complete
    uint64_t *q_ready = bars + 14;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmem);
    volatile uint32_t *hdr = reinterpret_cast<volatile uint32_t *>(smem + C::kOffHdr);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) {
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
                const int raw = __ldg(p.seq_lens + (size_t)b * p.dense_t + tok0 + t);
                n_unit = max(n_unit, min(max(raw, 0), p.K));
                if (s == 0 && ptid == t && (raw < 0 || raw > p.K)) {
                    atomicOr(&g_status_flags, kFlagIndexRange);
                    atomicAdd(&g_bad_index_count, 1ull);
                }
            }
        }
        const int *pt_b = p.page_table + (size_t)b * p.pt_stride;
        const long long max_pos = (long long)p.pt_stride * kPage;
        // Padding slots copy cache row 0 (always in range) and are masked to
        // probability 0 by the softmax, so they add 0 * row 0 to O.
        constexpr int kPadRow = 0;
        int *rows_s = reinterpret_cast<int *>(smem + C::kOffRows);
        const uint8_t *cache = reinterpret_cast<const uint8_t *>(p.cache);
        const uint32_t bar_prod = 1;  // named barrier of the producer warps
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
                        iv[k] = (j < n) ? __ldg(idx_bt + base + j) : -1;
                    }
                }
                int pg[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int i = iv[k];
                    pg[k] = (i >= 0 && (long long)i < max_pos) ? __ldg(pt_b + (i >> 6)) : -1;
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
                // 72 warp instructions per tile, each 4 rows x 128 B; warp pw takes every
                // kProducerWarps-th from i = pw
#pragma unroll 2
                for (int i = pw; i < 72; i += C::kProducerWarps) {
                    const int seg = 4 * i + (lane >> 3);  // 0..287: row r, column box
                    const int r = seg / 9, box = seg - 9 * r, ch = lane & 7;
                    const int j = t * C::kTileRows + r;
                    const int row = (j < n) ? rows_s[j] : -1;
                    const uint8_t *src = cache + (size_t)(row >= 0 ? row : kPadRow) * kRowBytes +
                                         box * 128 + ch * 16;
                    const uint32_t d = smem_addr(dst + box * C::kBoxStride + r * 128 + ((ch ^ (r & 7)) << 4));
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
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
            const uint32_t q_addr = sbase + C::kOffQ;
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
#pragma unroll 4
                        for (int kk = 0; kk < 36; ++kk) {
                            const uint32_t koff = (kk & 3) * 32;  // 16-element step inside the 128-B row
                            const uint64_t a = smem_desc(q_addr + (kk >> 2) * C::kQBoxBytes + koff, 16,
                                                         1024, kSwizzle128B);
                            const uint64_t bd = smem_desc(kv_addr + (kk >> 2) * C::kBoxStride + koff,
                                                          16, 1024, kSwizzle128B);
                            umma_bf16(d, a, bd, kIdescQK, kk > 0 ? 1u : 0u);
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
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk) {
                            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                            const uint64_t a = smem_desc(p_addr + kk * 32, 16, 512, kSwizzle64B);
                            const uint64_t blo = smem_desc(kv_addr + kk * 2048, C::kBoxStride, 1024,
                                                           kSwizzle128B);
                            const uint64_t bhi = smem_desc(kv_addr + 4 * C::kBoxStride + kk * 2048,
                                                           C::kBoxStride, 1024, kSwizzle128B);
                            umma_bf16(tmem, a, blo, kIdescPV, acc);
                            umma_bf16(tmem + (16u << 16), a, bhi, kIdescPV, acc);
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
        const int tid = threadIdx.x;  // 0..127
        const int q4 = warp;          // TMEM sub-partition (lanes 32*q4 .. +31)
        const int hrow = 16 * q4 + (lane & 15);
        const int half = lane >> 4;

        // ---- stage Q (heads x 576, zero rows beyond H) as 9 swizzled 64-column boxes
        {
            const uint4 *qsrc = reinterpret_cast<const uint4 *>(p.q + (size_t)row0 * kD);
            for (int c0 = 0; c0 < 64 * 72; c0 += 128 * 12) {
                uint4 v[12];
#pragma unroll
                for (int k = 0; k < 12; ++k) {
                    const int c = c0 + k * 128 + tid;
                    const int h = c / 72;
                    v[k] = (c < 64 * 72 && h < nrows) ? __ldg(qsrc + (size_t)h * 72 + (c % 72))
                                                     : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int k = 0; k < 12; ++k) {
                    const int c = c0 + k * 128 + tid;
                    if (c < 64 * 72) {
                        const int h = c / 72, k16 = c % 72;
                        const int box = k16 >> 3, ch = k16 & 7;
                        *reinterpret_cast<uint4 *>(smem + C::kOffQ + box * C::kQBoxBytes + h * 128 +
                                                   ((ch ^ (h & 7)) << 4)) = v[k];
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }

        // dense: list entries visible to query row hrow (rows past the unit's
        // real rows see none); sparse: no per-row limit
        int lim = INT_MAX;
        if (dense)
            lim = hrow < nrows ? min(max(__ldg(p.seq_lens + (size_t)b * p.dense_t + tok0 +
                                               hrow / p.dense_h), 0), p.K)
                               : 0;
        float m_ref = -INFINITY;  // running reference max of head hrow (log2 units)
        float l_acc = 0.f;        // sum of P of head hrow relative to m_ref (lanes 0-15; 0 elsewhere)
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q4) << 16);

        for (int pr = 0; pr < n_pairs; ++pr) {
            const int t0 = 2 * pr;
            const bool has1 = t0 + 1 < n_tiles;
            mbar_wait(&s_full[pr & 1], (pr >> 1) & 1, dead);
            tc_fence_after();
            // S of the pair: lanes 0-15 hold head hrow, columns 0-31 tile t0,
            // 32-63 tile t0+1 (lanes 16-31 read unused TMEM lanes, ignored)
            uint32_t s0[32], s1[32];
            tmem_ld32(t_lane + C::kSCol + 64 * (pr & 1), s0);
            tmem_ld32(t_lane + C::kSCol + 64 * (pr & 1) + 32, s1);
            tmem_ld_wait();
            mbar_wait(&kv_full[t0 % C::kStages], (t0 / C::kStages) & 1, dead);
            uint32_t vm0 = hdr[t0 % C::kStages];
            uint32_t vm1 = 0;
            if (has1) {
                mbar_wait(&kv_full[(t0 + 1) % C::kStages], ((t0 + 1) / C::kStages) & 1, dead);
                vm1 = hdr[(t0 + 1) % C::kStages];
            }
            if (dense) {  // this row's causal limit, as a mask over the pair's columns
                const int r0 = lim - (j0 + t0 * C::kTileRows);
                const int r1 = r0 - C::kTileRows;
                vm0 &= r0 >= 32 ? 0xffffffffu : (r0 <= 0 ? 0u : (1u << r0) - 1u);
                vm1 &= r1 >= 32 ? 0xffffffffu : (r1 <= 0 ? 0u : (1u << r1) - 1u);
            }
            const bool owner = half == 0;  // lanes 0-15 run the softmax of head hrow
            // scores in log2 units, padding (and an absent second tile) -> -inf;
            // selects, not branches
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float x0 = ((vm0 >> j) & 1u) ? __uint_as_float(s0[j]) * p.scale_log2 : -INFINITY;
                const float x1 = ((vm1 >> j) & 1u) ? __uint_as_float(s1[j]) * p.scale_log2 : -INFINITY;
                s0[j] = __float_as_uint(x0);
                s1[j] = __float_as_uint(x1);
                mt = fmaxf(mt, fmaxf(x0, x1));
            }
            if (!owner) mt = -INFINITY;
            float alpha = 1.f;
            if (owner && mt > m_ref + C::kTau) {
                alpha = (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - mt);
                m_ref = mt;
            }
            alpha = __shfl_sync(0xffffffffu, alpha, lane & 15);  // lane l+16 rescales O[:, 256:512]
            // Rescale this thread's half row of O when its head's max jumped
            // (warp-collective TMEM access; alpha = 1 for the other threads).
            const bool need = (pr >= 1) && (alpha != 1.f);
            if (__any_sync(0xffffffffu, need)) {
                // O must hold PV of pair pr-1 before it is rescaled.  The tensor
                // pipe runs in issue order and QK(pr) went out after PV(pr-2), so
                // PV(pr-3) is done and this parity wait cannot alias.
                mbar_wait(&o_done[(pr - 1) & 1], ((pr - 1) >> 1) & 1, dead);
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t orr[32];
                    tmem_ld32(t_lane + c, orr);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
                    tmem_st32(t_lane + c, orr);
                }
                tmem_st_wait();
            }
            if (owner) {
                const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
                float ps = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t r0 = h ? s1[2 * j] : s0[2 * j], r1 = h ? s1[2 * j + 1] : s0[2 * j + 1];
                        const float a0 = fast_exp2(__uint_as_float(r0) - mu);  // exp2(-inf) = 0
                        const float a1 = fast_exp2(__uint_as_float(r1) - mu);
                        ps += a0 + a1;
                        pk[j] = pack_bf16x2(a0, a1);
                    }
                    if (h == 1 && !has1) continue;
                    // P tile (64 heads x 32 rows, bf16) in the tile's spent k_pe box,
                    // K-major 64B swizzle
                    uint8_t *pbase = smem + C::kOffKV + C::tile_off((t0 + h) % C::kStages) + 8 * C::kBoxStride;
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
        // Partials leave through shared memory so that each store instruction
        // writes whole 128-B row segments: lane L holds 32 columns of its own
        // row, and a direct store would touch 32 rows (32 lines) at once.
        // Per warp, 32 lane-rows of 32 floats at a 144-B pitch (conflict-free
        // both ways) in the Q region, which no MMA reads any more.
        constexpr int kPitch = 36;
        float *stage = reinterpret_cast<float *>(smem + C::kOffQ) + warp * (32 * kPitch);
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
            uint32_t orr[32];
            if (n_pairs > 0) {
                tmem_ld32(t_lane + c, orr);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) orr[j] = 0u;
            }
            const int col = 256 * half + c;
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
                    const int lr = 4 * k + (lane >> 3);  // lane-row: lane lr's row and half
                    const int ch = lane & 7;             // 16-B chunk of its 128-B segment
                    const int hr = 16 * q4 + (lr & 15);
                    if (hr < nrows) {
                        const float4 v = *reinterpret_cast<const float4 *>(stage + lr * kPitch + 4 * ch);
                        *reinterpret_cast<float4 *>(p.part_o + (((size_t)row0 + hr) * p.nsplit + s) * kDc +
                                                    256 * (lr >> 4) + c + 4 * ch) = v;
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
