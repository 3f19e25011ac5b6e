// smla_dense.cuh -- the dense-context (KV-split verify) variant's first step.
//
// "The Occupancy Hypothesis: How One Kernel Parameter Unlocked 1.8x Decode
// Speedup on Blackwell", sections "The Occupancy Insight" and "The Broader
// Context": the speculative-decoding verify kernel attends each query token
// to its whole visible KV sequence and divides that sequence into NSPLIT
// splits, each a partial pass, merged by a reduce.  That is the sparse path
// with the index list of query token (b, t) set to every position
// 0 .. seq_lens[b, t] - 1.  This kernel writes those lists into the
// workspace; the partial kernels, the combine and the NSPLIT heuristic then
// run unchanged.
#pragma once

#include <cstdint>

#include "smla_ptx.cuh"

namespace smla {

// idx[bt * K + j] = j if j < seq_lens[bt] else -1, for bt < n_bt, j < K.
// A length outside [0, K] is clamped to that range, raises kFlagIndexRange
// and counts once in g_bad_index_count.  Grid-stride, one entry per thread and
// iteration: consecutive threads write consecutive words.
__global__ void __launch_bounds__(256) smla_dense_index_kernel(const int32_t *__restrict__ seq_lens,
                                                               long long n_bt, int K,
                                                               int32_t *__restrict__ idx) {
    const long long total = n_bt * (long long)K;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const long long bt = e / K;
        const int j = (int)(e - bt * K);
        const int n_raw = __ldg(seq_lens + bt);
        const int n = min(max(n_raw, 0), K);
        if (j == 0 && n != n_raw) {
            atomicOr(&g_status_flags, kFlagIndexRange);
            atomicAdd(&g_bad_index_count, 1ull);
        }
        idx[e] = j < n ? j : -1;
    }
}

}  // namespace smla
