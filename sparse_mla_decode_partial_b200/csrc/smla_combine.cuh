// smla_combine.cuh -- log-sum-exp combine of split-K partials.
//
// "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
// Decode", section "The Split-K Imperative": each split block writes a partial
// attention output, later merged by a log-sum-exp combine kernel.  Per
// (b, t, h), with m_s the reference point of split s and lse_s its log-sum-exp:
//   M = max_s m_s,  L = sum_s exp(lse_s - M),
//   o = sum_s exp(m_s - M) O_s / L,  lse = M + ln L;  every split empty: 0, -inf.
// A split with m_s = -inf is empty and its O_s is never used (the balanced
// schedule of the whole decode leaves such slots unwritten).
//
// One 512-thread CTA per (b, t, h): 4 groups of 128 threads, thread c of a
// group owning output columns 4c..4c+3.  Splits are taken in batches of
// 4 x kCombineDepth; in a batch every thread issues all its loads (partial
// rows, m, lse) before using any, so a batch costs one memory round trip.
// A running maximum rescales the accumulators between batches.
//
// For few splits (S <= 8) a second form gives each (b, t, h) one warp: lane l
// owns columns 4l + 128j (j < 4, coalesced float4 rows) and issues every load
// of every split at once, so thousands of units finish in one wave.
//
// Both are launched as programmatic dependents of the partial pass: they may
// be scheduled while that grid still runs, and wait on griddepcontrol before
// touching memory.  The partials are read with coherent L2 loads (__ldcg),
// never the read-only path: that data is written by the grid that runs
// concurrently, so no load of it may be treated as invariant and scheduled
// ahead of the wait.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "smla_ptx.cuh"

namespace smla {

constexpr int kCombineThreads = 512;
constexpr int kCombineGroups = 4;
constexpr int kCombineDepth = 16;  // splits per group per batch

__global__ void __launch_bounds__(kCombineThreads)
    smla_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_m,
                        const float *__restrict__ part_lse, int nsplit,
                        __nv_bfloat16 *__restrict__ o, float *__restrict__ lse) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float red_m[kCombineGroups];
    __shared__ float red_l[kCombineGroups];
    __shared__ float4 red_acc[kCombineGroups - 1][128];

    const size_t u = blockIdx.x;
    const int g = threadIdx.x >> 7;
    const int c = threadIdx.x & 127;
    const float *pm = part_m + u * nsplit;
    const float *pl = part_lse + u * nsplit;
    const float4 *po = reinterpret_cast<const float4 *>(part_o + u * (size_t)nsplit * 512) + c;

    float M = -INFINITY;  // running max over all batches (identical in every thread)
    float L = 0.f;        // this group's sum of exp(lse_s - M)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);

    for (int s0 = 0; s0 < nsplit; s0 += kCombineGroups * kCombineDepth) {
        float mv[kCombineDepth], lv[kCombineDepth];
        float4 v[kCombineDepth];
#pragma unroll
        for (int k = 0; k < kCombineDepth; ++k) {
            const int s = s0 + g * kCombineDepth + k;
            if (s < nsplit) {
                mv[k] = __ldcg(pm + s);
                lv[k] = __ldcg(pl + s);
                v[k] = __ldcg(po + (size_t)s * 128);
            } else {
                mv[k] = -INFINITY;
                lv[k] = -INFINITY;
                v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float mb = -INFINITY;
#pragma unroll
        for (int k = 0; k < kCombineDepth; ++k) mb = fmaxf(mb, mv[k]);
        if (c == 0) red_m[g] = mb;
        __syncthreads();
        mb = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
        __syncthreads();  // red_m is rewritten by the next batch
        const float Mn = fmaxf(M, mb);
        if (Mn == -INFINITY) continue;  // nothing valid so far
        const float r = (M == -INFINITY) ? 0.f : expf(M - Mn);
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
        L *= r;
#pragma unroll
        for (int k = 0; k < kCombineDepth; ++k) {
            // An empty slot (m = -inf) contributes nothing, whatever its part_o
            // holds (selects, so that stale bits there never reach acc).
            const bool on = mv[k] != -INFINITY;
            const float w = on ? expf(mv[k] - Mn) : 0.f;
            acc.x = on ? fmaf(w, v[k].x, acc.x) : acc.x;
            acc.y = on ? fmaf(w, v[k].y, acc.y) : acc.y;
            acc.z = on ? fmaf(w, v[k].z, acc.z) : acc.z;
            acc.w = on ? fmaf(w, v[k].w, acc.w) : acc.w;
            if (lv[k] != -INFINITY) L += expf(lv[k] - Mn);
        }
        M = Mn;
    }

    if (g > 0) red_acc[g - 1][c] = acc;
    if (c == 0) red_l[g] = L;
    __syncthreads();
    if (g != 0) return;
    uint2 *dst = reinterpret_cast<uint2 *>(o + u * 512) + c;
    if (M == -INFINITY) {
        *dst = make_uint2(0u, 0u);
        if (c == 0) lse[u] = -INFINITY;
        return;
    }
#pragma unroll
    for (int k = 0; k < kCombineGroups - 1; ++k) {
        const float4 a = red_acc[k][c];
        acc.x += a.x;
        acc.y += a.y;
        acc.z += a.z;
        acc.w += a.w;
    }
    const float Lt = (red_l[0] + red_l[1]) + (red_l[2] + red_l[3]);
    const float inv = 1.f / Lt;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    *dst = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
    if (c == 0) lse[u] = M + logf(Lt);
}

// Column-quarter form (S > 8): one 512-thread CTA per (b, t, h) and 128 of
// its 512 output columns, so a (b, t, h) is combined by four CTAs on four SMs
// and each CTA pulls a quarter of the partial bytes.  16 groups of 32 threads;
// thread c of a group owns columns 4c..4c+3 of the quarter; group g takes
// splits g, g+16, ... (kCombineQDepth per batch, all loads of a batch in
// flight at once).  Every quarter computes M and L itself (they are scalars).
constexpr int kCombineQGroups = 16;
constexpr int kCombineQDepth = 4;

__global__ void __launch_bounds__(kCombineThreads)
    smla_combine_quarter_kernel(const float *__restrict__ part_o, const float *__restrict__ part_m,
                                const float *__restrict__ part_lse, int nsplit,
                                __nv_bfloat16 *__restrict__ o, float *__restrict__ lse) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float red_m[kCombineQGroups];
    __shared__ float red_l[kCombineQGroups];
    __shared__ float4 red_acc[kCombineQGroups - 1][32];

    const size_t u = blockIdx.x >> 2;
    const int quarter = blockIdx.x & 3;
    const int g = threadIdx.x >> 5;
    const int c = threadIdx.x & 31;
    const float *pm = part_m + u * nsplit;
    const float *pl = part_lse + u * nsplit;
    const float4 *po = reinterpret_cast<const float4 *>(part_o + u * (size_t)nsplit * 512) + quarter * 32 + c;

    float M = -INFINITY;  // running max over all batches (identical in every thread)
    float L = 0.f;        // this group's sum of exp(lse_s - M)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);

    for (int s0 = 0; s0 < nsplit; s0 += kCombineQGroups * kCombineQDepth) {
        float mv[kCombineQDepth], lv[kCombineQDepth];
        float4 v[kCombineQDepth];
#pragma unroll
        for (int k = 0; k < kCombineQDepth; ++k) {
            const int sp = s0 + g + kCombineQGroups * k;
            if (sp < nsplit) {
                mv[k] = __ldcg(pm + sp);
                lv[k] = __ldcg(pl + sp);
                v[k] = __ldcg(po + (size_t)sp * 128);
            } else {
                mv[k] = -INFINITY;
                lv[k] = -INFINITY;
                v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float mb = -INFINITY;
#pragma unroll
        for (int k = 0; k < kCombineQDepth; ++k) mb = fmaxf(mb, mv[k]);
        if (c == 0) red_m[g] = mb;
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kCombineQGroups; ++k) mb = fmaxf(mb, red_m[k]);
        __syncthreads();  // red_m is rewritten by the next batch
        const float Mn = fmaxf(M, mb);
        if (Mn == -INFINITY) continue;  // nothing valid so far
        const float r = (M == -INFINITY) ? 0.f : expf(M - Mn);
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
        L *= r;
#pragma unroll
        for (int k = 0; k < kCombineQDepth; ++k) {
            const bool on = mv[k] != -INFINITY;  // empty slot: part_o is not used
            const float w = on ? expf(mv[k] - Mn) : 0.f;
            acc.x = on ? fmaf(w, v[k].x, acc.x) : acc.x;
            acc.y = on ? fmaf(w, v[k].y, acc.y) : acc.y;
            acc.z = on ? fmaf(w, v[k].z, acc.z) : acc.z;
            acc.w = on ? fmaf(w, v[k].w, acc.w) : acc.w;
            if (lv[k] != -INFINITY) L += expf(lv[k] - Mn);
        }
        M = Mn;
    }

    if (g > 0) red_acc[g - 1][c] = acc;
    if (c == 0) red_l[g] = L;
    __syncthreads();
    if (g != 0) return;
    uint2 *dst = reinterpret_cast<uint2 *>(o + u * 512 + quarter * 128) + c;
    if (M == -INFINITY) {
        *dst = make_uint2(0u, 0u);
        if (quarter == 0 && c == 0) lse[u] = -INFINITY;
        return;
    }
    float Lt = 0.f;
#pragma unroll
    for (int k = 0; k < kCombineQGroups; ++k) Lt += red_l[k];
#pragma unroll
    for (int k = 0; k < kCombineQGroups - 1; ++k) {
        const float4 a = red_acc[k][c];
        acc.x += a.x;
        acc.y += a.y;
        acc.z += a.z;
        acc.w += a.w;
    }
    const float inv = 1.f / Lt;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    *dst = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
    if (quarter == 0 && c == 0) lse[u] = M + logf(Lt);
}

constexpr int kCombineWarpUnits = 4;  // units (warps) per CTA of the warp form

template <int SMAX>
__global__ void __launch_bounds__(32 * kCombineWarpUnits)
    smla_combine_warp_kernel(const float *__restrict__ part_o, const float *__restrict__ part_m,
                             const float *__restrict__ part_lse, int nsplit, int n_units,
                             __nv_bfloat16 *__restrict__ o, float *__restrict__ lse) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const long long u = (long long)blockIdx.x * kCombineWarpUnits + (threadIdx.x >> 5);
    if (u >= n_units) return;
    const float *pm = part_m + u * nsplit;
    const float *pl = part_lse + u * nsplit;
    const float4 *po = reinterpret_cast<const float4 *>(part_o + u * (long long)nsplit * 512) + lane;

    float mv[SMAX], lv[SMAX];
    float4 v[SMAX][4];
#pragma unroll
    for (int s = 0; s < SMAX; ++s) {
        if (s < nsplit) {
            mv[s] = __ldcg(pm + s);
            lv[s] = __ldcg(pl + s);
#pragma unroll
            for (int j = 0; j < 4; ++j) v[s][j] = __ldcg(po + s * 128 + j * 32);
        } else {
            mv[s] = -INFINITY;
            lv[s] = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) v[s][j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < SMAX; ++s) M = fmaxf(M, mv[s]);
    uint2 *dst = reinterpret_cast<uint2 *>(o + u * 512) + lane;
    if (M == -INFINITY) {
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j * 32] = make_uint2(0u, 0u);
        if (lane == 0) lse[u] = -INFINITY;
        return;
    }
    float L = 0.f;
    float4 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < SMAX; ++s) {
        if (lv[s] != -INFINITY) L += expf(lv[s] - M);
        const bool on = mv[s] != -INFINITY;  // empty slot: part_o is not used
        const float w = on ? expf(mv[s] - M) : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[j].x = on ? fmaf(w, v[s][j].x, acc[j].x) : acc[j].x;
            acc[j].y = on ? fmaf(w, v[s][j].y, acc[j].y) : acc[j].y;
            acc[j].z = on ? fmaf(w, v[s][j].z, acc[j].z) : acc[j].z;
            acc[j].w = on ? fmaf(w, v[s][j].w, acc[j].w) : acc[j].w;
        }
    }
    const float inv = 1.f / L;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x * inv, acc[j].y * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z * inv, acc[j].w * inv);
        dst[j * 32] = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
    }
    if (lane == 0) lse[u] = M + logf(L);
}

// Self-test of the bounded waits (smla_selftest_wait_timeout): one warp waits
// on a fresh mbarrier that nothing ever arrives at, through the same
// mbar_wait the kernels use, with the given limit.  The wait gives up, raises
// the timeout flag and the kernel returns.
__global__ void __launch_bounds__(32) smla_selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    bool dead = false;
    mbar_wait(&bar, 0, dead, limit_ns);
}

// Copy of the per-step inputs of smla_decode_host from pinned host memory
// (addressed through its device alias) into the workspace's staging area.
// Every read crosses the host link, so its latency (about a microsecond)
// dominates a small step: the three regions are flattened into one item
// space (16-byte vectors where the source allows them, then 4-byte words for
// a tail) and each thread issues the loads of all its items, up to
// kIngestDepth of them, before it stores any.  A step whose items fit the
// grid's threads then costs one round trip, not one per region.
struct IngestRegion {
    const uint8_t *src;
    uint8_t *dst;
    size_t bytes;  // multiple of 4
};
struct IngestArgs {
    IngestRegion r[3];
};
constexpr int kIngestThreads = 256;
constexpr int kIngestDepth = 4;  // items in flight per thread

// Item counts of one region: n16 vectors (none when the source is not
// 16-byte aligned) followed by the remaining 4-byte words.
__device__ __forceinline__ void ingest_counts(const IngestRegion &r, size_t &n16, size_t &n) {
    n16 = (reinterpret_cast<uintptr_t>(r.src) & 15) ? 0 : r.bytes / 16;
    n = n16 + (r.bytes - n16 * 16) / 4;
}

__global__ void __launch_bounds__(kIngestThreads) smla_ingest_kernel(const IngestArgs a) {
    // the partial pass is launched as a programmatic dependent: let it be
    // scheduled now (it waits for this grid's completion before reading)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    size_t n16[3], end[3];
    size_t total = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        size_t n;
        ingest_counts(a.r[k], n16[k], n);
        total += n;
        end[k] = total;
    }
    const size_t nthreads = (size_t)gridDim.x * blockDim.x;
    for (size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < total;
         i0 += nthreads * kIngestDepth) {
        uint4 v[kIngestDepth];
        uint8_t *dst[kIngestDepth];
        bool wide[kIngestDepth];
#pragma unroll
        for (int j = 0; j < kIngestDepth; ++j) {
            const size_t i = i0 + (size_t)j * nthreads;
            dst[j] = nullptr;
            wide[j] = false;
            if (i < total) {
                const int k = i < end[0] ? 0 : (i < end[1] ? 1 : 2);
                const size_t local = i - (k == 0 ? 0 : end[k - 1]);
                const IngestRegion &r = a.r[k];
                if (local < n16[k]) {
                    v[j] = reinterpret_cast<const uint4 *>(r.src)[local];
                    dst[j] = r.dst + local * 16;
                    wide[j] = true;
                } else {
                    const size_t off = n16[k] * 16 + (local - n16[k]) * 4;
                    v[j].x = *reinterpret_cast<const uint32_t *>(r.src + off);
                    dst[j] = r.dst + off;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kIngestDepth; ++j) {
            if (dst[j] == nullptr) continue;
            if (wide[j])
                *reinterpret_cast<uint4 *>(dst[j]) = v[j];
            else
                *reinterpret_cast<uint32_t *>(dst[j]) = v[j].x;
        }
    }
}

}  // namespace smla
