// smla_combine.cuh -- log-sum-exp combine of split-K partials.
//
// "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
// Decode", section "The Split-K Imperative": each split block writes a partial
// attention output, later merged by a log-sum-exp combine kernel.  Per
// (b, t, h), with m_s the reference point of split s and lse_s its log-sum-exp:
//   M = max_s m_s,  L = sum_s exp(lse_s - M),
//   o = sum_s exp(m_s - M) O_s / L,  lse = M + ln L;  every split empty: 0, -inf.
// One 128-thread CTA per (b, t, h); thread i owns output columns 4i..4i+3 and
// streams the S partial rows with 16-byte loads.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace smla {

constexpr int kCombineThreads = 128;

__device__ __forceinline__ float block_reduce_max_128(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

__device__ __forceinline__ float block_reduce_sum_128(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    return (red[0] + red[1]) + (red[2] + red[3]);
}

__global__ void __launch_bounds__(kCombineThreads)
    smla_combine_kernel(const float *__restrict__ part_o, const float *__restrict__ part_m,
                        const float *__restrict__ part_lse, int nsplit,
                        __nv_bfloat16 *__restrict__ o, float *__restrict__ lse) {
    extern __shared__ float w_s[];  // [nsplit] combine weights
    __shared__ float red[4];
    const size_t u = blockIdx.x;
    const int tid = threadIdx.x;
    const float *pm = part_m + u * nsplit;
    const float *pl = part_lse + u * nsplit;

    float M = -INFINITY;
    for (int s = tid; s < nsplit; s += kCombineThreads) M = fmaxf(M, pm[s]);
    M = block_reduce_max_128(M, red);

    uint2 *dst = reinterpret_cast<uint2 *>(o + u * 512) + tid;
    if (M == -INFINITY) {
        *dst = make_uint2(0u, 0u);
        if (tid == 0) lse[u] = -INFINITY;
        return;
    }
    float L = 0.f;
    for (int s = tid; s < nsplit; s += kCombineThreads) {
        const float v = pl[s];
        if (v != -INFINITY) L += expf(v - M);
    }
    L = block_reduce_sum_128(L, red);
    const float invL = 1.f / L;
    for (int s = tid; s < nsplit; s += kCombineThreads) {
        const float m = pm[s];
        w_s[s] = (m == -INFINITY) ? 0.f : expf(m - M) * invL;
    }
    __syncthreads();

    const float4 *src = reinterpret_cast<const float4 *>(part_o + u * (size_t)nsplit * 512) + tid;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int s = 0;
    for (; s + 4 <= nsplit; s += 4) {
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = __ldg(src + (size_t)(s + k) * 128);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float w = w_s[s + k];
            acc.x = fmaf(w, v[k].x, acc.x);
            acc.y = fmaf(w, v[k].y, acc.y);
            acc.z = fmaf(w, v[k].z, acc.z);
            acc.w = fmaf(w, v[k].w, acc.w);
        }
    }
    for (; s < nsplit; ++s) {
        const float4 v = __ldg(src + (size_t)s * 128);
        const float w = w_s[s];
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    *dst = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
    if (tid == 0) lse[u] = M + logf(L);
}

}  // namespace smla
