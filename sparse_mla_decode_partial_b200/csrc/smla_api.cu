// smla_api.cu -- host side of the C ABI declared in include/smla.h: argument
// checks, the NSPLIT heuristic, workspace carving and kernel launches.
// Every entry point returns a status; nothing throws across the ABI.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <set>
#include <utility>

#include "smla.h"

// Tile shape of the mma kernel for H <= 16 (two CTAs per SM either way).
#ifndef SMLA_MMA_TILE_ROWS
#define SMLA_MMA_TILE_ROWS 32
#define SMLA_MMA_STAGES 2
#endif
#include "smla_combine.cuh"
#include "smla_partial_mma.cuh"
#include "smla_partial_tc.cuh"
#include "smla_indexer.cuh"

namespace {

using smla::PartialParams;

thread_local char g_last_error[256] = "";

smla_status cuda_fail(cudaError_t e) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return SMLA_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Per (device, kernel) one-time opt-in to large dynamic shared memory.
cudaError_t ensure_smem_attr(const void *kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static std::mutex mu;
    static std::set<std::pair<int, const void *>> done;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, kernel);
    if (done.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert(key);
    return e;
}

int current_device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// Kernel choice of launch_partial, as the schedule needs it.
bool uses_latency_kernel(int H, int K, int kc, int pt_stride) {
    return H <= 32 && K > 0 && kc <= smla::kSmallMaxRows && pt_stride <= smla::kSmallMaxPt;
}

// NSPLIT model ("The Occupancy Hypothesis ...", sections "The Occupancy
// Insight" and "The Broader Context": more blocks in flight hide memory
// latency, and the best NSPLIT depends on SMs, heads, batch and query
// length).  Cost in units of "one CTA gathering one 1152-B row at its share
// of HBM bandwidth":
//     waves(S) * (kFixedRows + ceil(K / S))     wave-quantised gather time
//   + scratch(S)                                partials written, re-read
// S is capped so that every split keeps at least kMinRowsPerSplit rows.
constexpr double kFixedRows = 48.0;     // per-CTA latency: launch, Q load, index chase
constexpr double kScratchWeight = 0.5;  // partials mostly stay in L2
constexpr int kMinRowsPerSplit = 32;
constexpr double kBalancedMargin = 0.15;
constexpr double kPartialBytesPerHead = (smla::kDc + 2) * 4.0;

int nsplit_model(int B, int T, int H, int K, int sm_count) {
    const long long base = (long long)B * T;
    int s_max = (K + kMinRowsPerSplit - 1) / kMinRowsPerSplit;
    if (s_max < 1) s_max = 1;
    if (s_max > SMLA_MAX_NSPLIT) s_max = SMLA_MAX_NSPLIT;
    while (s_max > 1 && base * s_max > INT_MAX) --s_max;
    // partial CTAs resident per SM: two for H <= 16 (the mma kernel's 2-stage
    // form fits twice), one otherwise (shared memory)
    const double slots = (double)sm_count * (H <= 16 ? 2.0 : 1.0);
    double best = 0.0;
    int best_s = 1;
    for (int s = 1; s <= s_max; ++s) {
        const double ctas = (double)base * s;
        const double waves = std::ceil(ctas / slots);
        const double rows = std::ceil((double)K / s);
        double t = waves * (kFixedRows + rows);
        if (s > 1) t += kScratchWeight * ctas * H * kPartialBytesPerHead * 2.0 / smla::kRowBytes / slots;
        if (s == 1 || t < best * (1.0 - 1e-9)) {
            best = t;
            best_s = s;
        }
    }
    // Balanced schedule (see use_balanced): one full wave of `slots` CTAs with
    // equal rows, about base + slots pieces in all (each costs kFixedRows and
    // writes one partial per head).  A CTA that moves from one token to the
    // next stalls its pipeline, which the model does not see (measured: 5-15%
    // of the pass), so the balanced choice must win by kBalancedMargin.
    const long long s_bal = (long long)std::ceil((double)slots / (double)base) + 1;
    const double units = (double)base * ((K + 31) / 32);
    if (H <= 32 && s_bal >= 2 && s_bal <= s_max && units >= 4.0 * slots &&
        !uses_latency_kernel(H, K, (K + (int)s_bal - 1) / (int)s_bal, 0)) {
        const double pieces = (double)base + slots;
        double t = kFixedRows * pieces / slots + units * 32.0 / slots;
        t += kScratchWeight * pieces * H * kPartialBytesPerHead * 2.0 / smla::kRowBytes / slots;
        if (t < best * (1.0 - kBalancedMargin)) best_s = (int)s_bal;
    }
    return best_s;
}

smla_status check_decode_args(const void *q, const void *kv_cache, int64_t num_pages,
                              const int32_t *page_table, int pt_stride, const int32_t *idx,
                              int B, int T, int H, int K, int page_size, float scale) {
    if (B < 0 || T < 0 || H < 0 || K < 0) return SMLA_ERR_INVALID_ARG;
    if (page_size != SMLA_PAGE_SIZE) return SMLA_ERR_UNSUPPORTED;
    if (H > SMLA_MAX_HEADS) return SMLA_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (q == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(q, 16)) return SMLA_ERR_MISALIGNED;
    if (K > 0) {
        if (kv_cache == nullptr || page_table == nullptr || idx == nullptr) return SMLA_ERR_INVALID_ARG;
        if (num_pages < 1 || pt_stride < 1) return SMLA_ERR_INVALID_ARG;
        if (num_pages > SMLA_MAX_PAGES) return SMLA_ERR_UNSUPPORTED;
        if (!aligned(kv_cache, 16) || !aligned(page_table, 4) || !aligned(idx, 4))
            return SMLA_ERR_MISALIGNED;
    }
    if ((long long)B * T * H > INT_MAX) return SMLA_ERR_INVALID_ARG;
    return SMLA_OK;
}

// Launch of a partial-pass kernel as a programmatic dependent of whatever
// precedes it on the stream (the host entry point's copy kernel, a previous
// decode, a user's kernel): its grid may be scheduled as soon as the
// predecessor lets it, and every partial kernel executes griddepcontrol.wait
// before its first global memory access and before it takes tensor memory.
// With no programmatic predecessor the wait returns at once.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), int grid, int threads, size_t smem,
                             cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int HG, int NT, int NS, bool DIRECT>
smla_status launch_mma(const PartialParams &p, int grid, cudaStream_t st) {
    using C = smla::MmaCfg<HG, NT, NS>;
    const void *fn = reinterpret_cast<const void *>(&smla::smla_partial_mma_kernel<HG, NT, NS, DIRECT>);
    cudaError_t e = ensure_smem_attr(fn, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_dependent(smla::smla_partial_mma_kernel<HG, NT, NS, DIRECT>, grid, C::kThreads,
                         C::kSmemBytes, st, p);
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

}  // namespace
smla_status encode_cache_tiles(CUtensorMap *map, const void *cache, int64_t num_pages);
namespace {

template <bool DIRECT>
smla_status launch_tc(const PartialParams &p, int grid, cudaStream_t st) {
    const void *fn = reinterpret_cast<const void *>(&smla::smla_partial_tc_kernel<DIRECT>);
    cudaError_t e = ensure_smem_attr(fn, smla::TcCfg::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e);
    // dense lists load whole half-pages by TMA; sparse lists never use the map
    CUtensorMap map;
    std::memset(&map, 0, sizeof map);
    if (p.seq_lens != nullptr && p.K > 0) {
        const smla_status s = encode_cache_tiles(&map, p.cache, p.num_pages);
        if (s != SMLA_OK) return s;
    }
    e = launch_dependent(smla::smla_partial_tc_kernel<DIRECT>, grid, smla::TcCfg::kThreads,
                         smla::TcCfg::kSmemBytes, st, p, map);
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

template <int HG, int TILES, bool DIRECT>
smla_status launch_small(const PartialParams &p, int grid, cudaStream_t st) {
    using C = smla::SmallCfg<HG, TILES>;
    const void *fn = reinterpret_cast<const void *>(&smla::smla_partial_small_kernel<HG, TILES, DIRECT>);
    cudaError_t e = ensure_smem_attr(fn, C::kMaxSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_dependent(smla::smla_partial_small_kernel<HG, TILES, DIRECT>, grid, C::kThreads,
                         C::smem_bytes(p.pt_stride), st, p);
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

template <bool DIRECT>
smla_status launch_partial(const PartialParams &p, cudaStream_t st) {
    const long long grid = p.balanced ? (long long)p.grid : (long long)p.B * p.T * p.nsplit;
    if (grid > INT_MAX) return SMLA_ERR_INVALID_ARG;
    // one or two tiles per split: the latency path (see smla_partial_small_kernel)
    if (!p.balanced && uses_latency_kernel(p.H, p.K, p.kc, p.pt_stride)) {
        if (p.kc <= 32)
            return p.H <= 16 ? launch_small<1, 1, DIRECT>(p, (int)grid, st)
                             : launch_small<2, 1, DIRECT>(p, (int)grid, st);
        return p.H <= 16 ? launch_small<1, 2, DIRECT>(p, (int)grid, st)
                         : launch_small<2, 2, DIRECT>(p, (int)grid, st);
    }
    if (p.H > 32) return launch_tc<DIRECT>(p, (int)grid, st);
    if (p.H > 16) return launch_mma<2, 32, 4, DIRECT>(p, (int)grid, st);
    return launch_mma<1, SMLA_MMA_TILE_ROWS, SMLA_MMA_STAGES, DIRECT>(p, (int)grid, st);
}

PartialParams make_params(const void *q, const void *kv_cache, int64_t num_pages,
                          const int32_t *page_table, int pt_stride, const int32_t *idx, int B,
                          int T, int H, int K, float scale, int nsplit) {
    PartialParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.cache = static_cast<const __nv_bfloat16 *>(kv_cache);
    p.num_pages = num_pages;
    p.page_table = page_table;
    p.pt_stride = pt_stride;
    p.idx = idx;
    p.B = B;
    p.T = T;
    p.H = H;
    p.K = K;
    p.scale_log2 = scale * smla::kLog2e;
    p.nsplit = nsplit;
    p.kc = (K + nsplit - 1) / nsplit;
    return p;
}

// Partial CTAs resident per SM for the pipelined kernels (their launch bounds).
int resident_per_sm(int H) {
    if (H > 32) return 1;  // tcgen05 kernel: one CTA per SM (shared memory, TMEM)
    if (H > 16) return smla::MmaCfg<2, 32, 4>::kMinBlocks;
    return smla::MmaCfg<1, SMLA_MMA_TILE_ROWS, SMLA_MMA_STAGES>::kMinBlocks;
}

// Balanced schedule ("The Occupancy Hypothesis ...", section "The Occupancy
// Insight": the grid should keep every SM busy).  With S slots per token the
// equal split launches B*T*S CTAs, which leaves a partly filled last wave
// whenever B*T*S is not a multiple of the resident CTAs R.  The balanced
// schedule launches exactly R CTAs, each taking an equal share of the
// flattened (token, 32-row tile) space; a token then spans at most
// ceil(R / (B*T)) + 1 CTAs, each writing one of its S slots.  Used when it
// fits in S slots and each CTA gets at least 4 tiles.  The tcgen05 kernel
// (H > 32) keeps equal splits: its gather is bound by the device-wide 16-byte
// cp.async rate, not by the SMs it occupies (a balanced form measured no
// faster).
bool use_balanced(int B, int T, int H, int K, int nsplit, int pt_stride, int sms, int *grid) {
    if (nsplit < 2 || K <= 0 || H > 32) return false;
    const int kc = (K + nsplit - 1) / nsplit;
    if (uses_latency_kernel(H, K, kc, pt_stride)) return false;
    const long long bt = (long long)B * T;
    const long long resident = (long long)sms * resident_per_sm(H);
    const long long units = bt * ((K + 31) / 32);
    if (bt * nsplit <= resident) return false;             // equal splits fit one wave
    if ((long long)(nsplit - 1) * bt < resident) return false;  // a token could need > S slots
    if (units < 4 * resident) return false;
    *grid = (int)resident;
    return true;
}

smla_status launch_combine(const float *part_o, const float *part_m, const float *part_lse, int B,
                           int T, int H, int nsplit, void *o, float *lse, cudaStream_t st) {
    const long long units = (long long)B * T * H;
    if (units == 0) return SMLA_OK;
    if (units > INT_MAX) return SMLA_ERR_INVALID_ARG;
    // Programmatic dependent launch: the combine grid may be scheduled while
    // the partial pass still runs; the kernel waits (griddepcontrol.wait) for
    // its predecessor to complete before reading anything.
    cudaLaunchConfig_t cfg = {};
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    __nv_bfloat16 *ob = static_cast<__nv_bfloat16 *>(o);
    cudaError_t e;
    if (nsplit <= 8) {
        // one warp per (b, t, h), every load in flight at once
        cfg.gridDim = dim3((unsigned)((units + smla::kCombineWarpUnits - 1) / smla::kCombineWarpUnits));
        cfg.blockDim = dim3(32 * smla::kCombineWarpUnits);
        const int n = (int)units;
        if (nsplit <= 2)
            e = cudaLaunchKernelEx(&cfg, smla::smla_combine_warp_kernel<2>, part_o, part_m, part_lse,
                                   nsplit, n, ob, lse);
        else if (nsplit <= 4)
            e = cudaLaunchKernelEx(&cfg, smla::smla_combine_warp_kernel<4>, part_o, part_m, part_lse,
                                   nsplit, n, ob, lse);
        else
            e = cudaLaunchKernelEx(&cfg, smla::smla_combine_warp_kernel<8>, part_o, part_m, part_lse,
                                   nsplit, n, ob, lse);
    } else if (units <= INT_MAX / 4) {
        // four CTAs per (b, t, h), one per 128-column quarter
        cfg.gridDim = dim3((unsigned)(units * 4));
        cfg.blockDim = dim3(smla::kCombineThreads);
        e = cudaLaunchKernelEx(&cfg, smla::smla_combine_quarter_kernel, part_o, part_m, part_lse,
                               nsplit, ob, lse);
    } else {
        cfg.gridDim = dim3((unsigned)units);
        cfg.blockDim = dim3(smla::kCombineThreads);
        e = cudaLaunchKernelEx(&cfg, smla::smla_combine_kernel, part_o, part_m, part_lse, nsplit, ob,
                               lse);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

int smla_version(void) { return 100; }

const char *smla_last_error(void) { return g_last_error; }

const char *smla_status_string(smla_status status) {
    switch (status) {
        case SMLA_OK: return "SMLA_OK";
        case SMLA_ERR_INVALID_ARG: return "SMLA_ERR_INVALID_ARG: invalid argument";
        case SMLA_ERR_UNSUPPORTED: return "SMLA_ERR_UNSUPPORTED: unsupported shape or page size";
        case SMLA_ERR_MISALIGNED: return "SMLA_ERR_MISALIGNED: pointer alignment";
        case SMLA_ERR_WORKSPACE_TOO_SMALL: return "SMLA_ERR_WORKSPACE_TOO_SMALL: workspace too small";
        case SMLA_ERR_INDEX_RANGE: return "SMLA_ERR_INDEX_RANGE: index entry out of range";
        case SMLA_ERR_CUDA: return "SMLA_ERR_CUDA: CUDA error (see smla_last_error)";
        case SMLA_ERR_TIMEOUT: return "SMLA_ERR_TIMEOUT: a kernel wait timed out";
    }
    return "unknown smla_status";
}

int smla_choose_nsplit(int B, int T, int H, int K, int sm_count) {
    if (const char *env = std::getenv("SMLA_NSPLIT")) {
        char *end = nullptr;
        const long v = std::strtol(env, &end, 10);
        if (end != env && v > 0) return (int)(v > SMLA_MAX_NSPLIT ? SMLA_MAX_NSPLIT : v);
    }
    if (B <= 0 || T <= 0 || H <= 0 || K <= 0) return 1;
    if (sm_count <= 0) sm_count = current_device_sms();
    return nsplit_model(B, T, H, K, sm_count);
}

size_t smla_workspace_bytes(int B, int T, int H, int nsplit) {
    if (B < 0 || T < 0 || H < 0 || nsplit < 1 || nsplit > SMLA_MAX_NSPLIT) return 0;
    const size_t n = (size_t)B * T * H * nsplit;
    return round256(n * smla::kDc * sizeof(float)) + 2 * round256(n * sizeof(float));
}

smla_status smla_decode_partial(const void *q, const void *kv_cache, int64_t num_pages,
                                const int32_t *page_table, int pt_stride, const int32_t *topk_idx,
                                int B, int T, int H, int K, int page_size, float scale, int nsplit,
                                float *part_o, float *part_m, float *part_lse, void *stream) {
    smla_status st = check_decode_args(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B,
                                       T, H, K, page_size, scale);
    if (st != SMLA_OK) return st;
    if (nsplit < 1 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (part_o == nullptr || part_m == nullptr || part_lse == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(part_o, 16) || !aligned(part_m, 4) || !aligned(part_lse, 4))
        return SMLA_ERR_MISALIGNED;
    PartialParams p = make_params(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B, T, H,
                                  K, scale, nsplit);
    p.part_o = part_o;
    p.part_m = part_m;
    p.part_lse = part_lse;
    return launch_partial<false>(p, static_cast<cudaStream_t>(stream));
}

smla_status smla_lse_combine(const float *part_o, const float *part_m, const float *part_lse,
                             int B, int T, int H, int nsplit, void *o, float *lse, void *stream) {
    if (B < 0 || T < 0 || H < 0) return SMLA_ERR_INVALID_ARG;
    if (nsplit < 1 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (!part_o || !part_m || !part_lse || !o || !lse) return SMLA_ERR_INVALID_ARG;
    if (!aligned(part_o, 16) || !aligned(part_m, 4) || !aligned(part_lse, 4) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return SMLA_ERR_MISALIGNED;
    return launch_combine(part_o, part_m, part_lse, B, T, H, nsplit, o, lse,
                          static_cast<cudaStream_t>(stream));
}

namespace {

// The partial pass of the whole decode into the workspace (nsplit >= 2):
// equal splits, or the balanced schedule when it applies.
smla_status decode_partial_pass(const void *q, const void *kv_cache, int64_t num_pages,
                                const int32_t *page_table, int pt_stride, const int32_t *topk_idx,
                                int B, int T, int H, int K, float scale, int nsplit, void *workspace,
                                size_t workspace_bytes, cudaStream_t s, PartialParams *out) {
    if (workspace_bytes < smla_workspace_bytes(B, T, H, nsplit)) return SMLA_ERR_WORKSPACE_TOO_SMALL;
    if (workspace == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SMLA_ERR_MISALIGNED;
    PartialParams p = make_params(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B, T, H,
                                  K, scale, nsplit);
    const size_t n = (size_t)B * T * H * nsplit;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t off_m = round256(n * smla::kDc * sizeof(float));
    const size_t off_l = off_m + round256(n * sizeof(float));
    p.part_o = reinterpret_cast<float *>(ws);
    p.part_m = reinterpret_cast<float *>(ws + off_m);
    p.part_lse = reinterpret_cast<float *>(ws + off_l);
    int grid = 0;
    if (use_balanced(B, T, H, K, nsplit, pt_stride, current_device_sms(), &grid)) {
        p.balanced = 1;
        p.grid = grid;
        p.tpt = (K + 31) / 32;
        p.n_units = (long long)B * T * p.tpt;
    }
    *out = p;
    return launch_partial<false>(p, s);
}

}  // namespace

smla_status smla_decode(const void *q, const void *kv_cache, int64_t num_pages,
                        const int32_t *page_table, int pt_stride, const int32_t *topk_idx, int B,
                        int T, int H, int K, int page_size, float scale, int nsplit,
                        void *workspace, size_t workspace_bytes, void *o, float *lse,
                        void *stream) {
    smla_status st = check_decode_args(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B,
                                       T, H, K, page_size, scale);
    if (st != SMLA_OK) return st;
    if (nsplit < 0 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (o == nullptr || lse == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(o, 16) || !aligned(lse, 4)) return SMLA_ERR_MISALIGNED;
    if (nsplit == 0) nsplit = smla_choose_nsplit(B, T, H, K, 0);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (nsplit == 1) {
        PartialParams p = make_params(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B, T,
                                      H, K, scale, nsplit);
        p.o = static_cast<__nv_bfloat16 *>(o);
        p.lse = lse;
        return launch_partial<true>(p, s);
    }
    PartialParams p{};
    st = decode_partial_pass(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B, T, H, K,
                             scale, nsplit, workspace, workspace_bytes, s, &p);
    if (st != SMLA_OK) return st;
    return launch_combine(p.part_o, p.part_m, p.part_lse, B, T, H, nsplit, o, lse, s);
}

smla_status smla_decode_partial_ws(const void *q, const void *kv_cache, int64_t num_pages,
                                   const int32_t *page_table, int pt_stride,
                                   const int32_t *topk_idx, int B, int T, int H, int K,
                                   int page_size, float scale, int nsplit, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    smla_status st = check_decode_args(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B,
                                       T, H, K, page_size, scale);
    if (st != SMLA_OK) return st;
    if (nsplit < 2 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    PartialParams p{};
    return decode_partial_pass(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B, T, H, K,
                               scale, nsplit, workspace, workspace_bytes,
                               static_cast<cudaStream_t>(stream), &p);
}

// ---------------------------------------------------------------------------
// Allocation-free decode.  The split-K partials go to a scratch array that the
// library owns in device memory (one copy per device that loads this module).
// In host code `g_noalloc_scratch` names a host-side stand-in, not a device
// address, so each device's real address is looked up with
// cudaGetSymbolAddress while that device is current, and only that address is
// handed to the kernels.  The address belongs to the device's current context:
// it is cached together with that context and looked up again when the
// context changes (a cudaDeviceReset() creates a new primary context).
static __device__ __align__(256) uint8_t g_noalloc_scratch[SMLA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

// cuCtxGetCurrent, reached through the runtime (no link against the driver
// library); null if the driver does not provide it.
PFN_cuCtxGetCurrent_v4000 ctx_getter() {
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
        (void)cudaGetLastError();
    });
    return fn;
}

// Device address of this device's scratch array in its current context
// (looked up on first use and again whenever the context has changed).
smla_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return SMLA_ERR_UNSUPPORTED;
    // The thread's current context: null until the runtime has made the
    // device's primary context current in this thread (then the address is
    // simply looked up again, which also makes it current).
    PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_getter();
    auto current_ctx = [get_ctx]() {
        CUcontext c = nullptr;
        if (get_ctx == nullptr || get_ctx(&c) != CUDA_SUCCESS) c = nullptr;
        return c;
    };
    const CUcontext ctx = current_ctx();
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || g_noalloc_ctx[dev] != ctx) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_ptr[dev] = ptr;
        g_noalloc_ctx[dev] = current_ctx();
    }
    *out = g_noalloc_ptr[dev];
    return SMLA_OK;
}
}  // namespace

smla_status smla_decode_noalloc(const void *q, const void *kv_cache, int64_t num_pages,
                                const int32_t *page_table, int pt_stride, const int32_t *topk_idx,
                                int B, int T, int H, int K, int page_size, float scale, int nsplit,
                                void *o, float *lse, void *stream) {
    smla_status st = check_decode_args(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B,
                                       T, H, K, page_size, scale);
    if (st != SMLA_OK) return st;
    if (nsplit < 0 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (nsplit == 0) {
        // the heuristic's split count, lowered until its partials fit the
        // scratch array (S = 1 needs none)
        nsplit = smla_choose_nsplit(B, T, H, K, 0);
        while (nsplit > 1 && smla_workspace_bytes(B, T, H, nsplit) > SMLA_NOALLOC_SCRATCH_BYTES)
            --nsplit;
    }
    const size_t need = nsplit > 1 ? smla_workspace_bytes(B, T, H, nsplit) : 0;
    if (need > SMLA_NOALLOC_SCRATCH_BYTES) {
        std::snprintf(g_last_error, sizeof g_last_error,
                      "smla_decode_noalloc: %zu bytes of split-K scratch needed for nsplit=%d, "
                      "the built-in scratch holds %u",
                      need, nsplit, (unsigned)SMLA_NOALLOC_SCRATCH_BYTES);
        return SMLA_ERR_WORKSPACE_TOO_SMALL;
    }
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != SMLA_OK) return st;
    return smla_decode(q, kv_cache, num_pages, page_table, pt_stride, topk_idx, B, T, H, K,
                       page_size, scale, nsplit, scratch, SMLA_NOALLOC_SCRATCH_BYTES, o, lse,
                       stream);
}

// ---------------------------------------------------------------------------
// Decode with per-step data in pinned host memory (see include/smla.h).
namespace {

// Device alias of pinned host memory, or nullptr when `ptr` is not pinned host
// memory that the current device can address.
void *host_alias(const void *ptr) {
    if (ptr == nullptr) return nullptr;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
        (void)cudaGetLastError();  // an unregistered pointer is not an error state
        return nullptr;
    }
    if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
    return a.devicePointer;
}

struct HostStaging {
    size_t base, q, idx, pt, total;  // byte offsets and sizes inside the workspace
};

HostStaging host_staging(int B, int T, int H, int K, int pt_stride, int nsplit) {
    HostStaging h{};
    h.base = nsplit > 1 ? smla_workspace_bytes(B, T, H, nsplit) : 0;
    const size_t q_bytes = (size_t)B * T * H * smla::kD * 2;
    const size_t idx_bytes = (size_t)B * T * K * 4;
    h.q = round256(h.base);
    h.idx = h.q + round256(q_bytes);
    h.pt = h.idx + round256(idx_bytes);
    h.total = h.pt + round256((size_t)B * pt_stride * 4);
    return h;
}

}  // namespace

size_t smla_workspace_host_bytes(int B, int T, int H, int K, int pt_stride, int nsplit) {
    if (B < 0 || T < 0 || H < 0 || K < 0 || pt_stride < 0 || nsplit < 1 || nsplit > SMLA_MAX_NSPLIT)
        return 0;
    return host_staging(B, T, H, K, pt_stride, nsplit).total;
}

smla_status smla_decode_host(const void *q_host, const void *kv_cache, int64_t num_pages,
                             const int32_t *page_table_host, int pt_stride,
                             const int32_t *topk_idx_host, int B, int T, int H, int K,
                             int page_size, float scale, int nsplit, void *workspace,
                             size_t workspace_bytes, void *o_host, float *lse_host, void *stream) {
    // Every check smla_decode makes on its arguments runs here first, on the
    // host pointers, so that a failed check launches nothing (not even the
    // copy kernel).
    smla_status st0 = check_decode_args(q_host, kv_cache, num_pages, page_table_host, pt_stride,
                                        topk_idx_host, B, T, H, K, page_size, scale);
    if (st0 != SMLA_OK) return st0;
    if (pt_stride < 0) return SMLA_ERR_INVALID_ARG;
    if (nsplit < 0 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (o_host == nullptr || lse_host == nullptr) return SMLA_ERR_INVALID_ARG;
    if (nsplit == 0) nsplit = smla_choose_nsplit(B, T, H, K, 0);
    // every host pointer must be pinned and visible to the device: checked
    // here, before anything is launched
    void *q_d = host_alias(q_host);
    void *o_d = host_alias(o_host);
    void *lse_d = host_alias(lse_host);
    void *pt_d = K > 0 ? host_alias(page_table_host) : nullptr;
    void *idx_d = K > 0 ? host_alias(topk_idx_host) : nullptr;
    if (q_d == nullptr || o_d == nullptr || lse_d == nullptr || (K > 0 && (pt_d == nullptr || idx_d == nullptr))) {
        std::snprintf(g_last_error, sizeof g_last_error,
                      "smla_decode_host: q, page_table, topk_idx, o and lse must be pinned host memory");
        return SMLA_ERR_INVALID_ARG;
    }
    if (!aligned(q_host, 16) || !aligned(o_host, 16) || !aligned(lse_host, 4) ||
        (K > 0 && (!aligned(page_table_host, 4) || !aligned(topk_idx_host, 4))))
        return SMLA_ERR_MISALIGNED;
    const HostStaging hs = host_staging(B, T, H, K, pt_stride, nsplit);
    if (workspace_bytes < hs.total) return SMLA_ERR_WORKSPACE_TOO_SMALL;
    if (workspace == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SMLA_ERR_MISALIGNED;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    smla::IngestArgs a{};
    a.r[0] = {static_cast<const uint8_t *>(q_d), ws + hs.q, (size_t)B * T * H * smla::kD * 2};
    if (K > 0) {
        a.r[1] = {static_cast<const uint8_t *>(idx_d), ws + hs.idx, (size_t)B * T * K * 4};
        a.r[2] = {static_cast<const uint8_t *>(pt_d), ws + hs.pt, (size_t)B * pt_stride * 4};
    }
    // one item per thread while the step is small (a single round trip over
    // the host link), at most one CTA per SM beyond that
    size_t items = 0;  // the kernel's item count (ingest_counts)
    for (const smla::IngestRegion &r : a.r) {
        const size_t n16 = aligned(r.src, 16) ? r.bytes / 16 : 0;
        items += n16 + (r.bytes - n16 * 16) / 4;
    }
    const unsigned blocks = (unsigned)std::min<size_t>(
        (items + smla::kIngestThreads - 1) / smla::kIngestThreads, (size_t)current_device_sms());
    smla::smla_ingest_kernel<<<blocks, smla::kIngestThreads, 0, st>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    return smla_decode(ws + hs.q, kv_cache, num_pages, reinterpret_cast<const int32_t *>(ws + hs.pt),
                       pt_stride, reinterpret_cast<const int32_t *>(ws + hs.idx), B, T, H, K, page_size,
                       scale, nsplit, workspace, hs.base, o_d, static_cast<float *>(lse_d), stream);
}

// ---------------------------------------------------------------------------
// Dense-context decode (see include/smla.h).  The tcgen05 kernel reads the
// visible lengths itself (entry j of a list is position j) and packs up to
// 64 / H query tokens of a sequence into the M rows of one pass over the
// rows; the combine then runs over the usual [B, T, H, S] partials.
namespace {

struct DensePlan {
    int pack;   // query tokens per unit
    int units;  // units per sequence
    int nsplit;
};

DensePlan dense_plan(int B, int T, int H, int K, int nsplit) {
    DensePlan d{};
    const int gmax = std::max(1, std::min(T, smla::kMaxTcRows / std::max(H, 1)));
    d.units = (T + gmax - 1) / gmax;
    d.pack = (T + d.units - 1) / d.units;  // the same number of passes, balanced units
    // one CTA per SM (the tcgen05 kernel): the heuristic's H > 32 model
    d.nsplit = nsplit > 0 ? nsplit : smla_choose_nsplit(B, d.units, smla::kMaxTcRows, K, 0);
    return d;
}

smla_status check_dense_args(const void *q, const void *kv_cache, int64_t num_pages,
                             const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                             int B, int T, int H, int K, int page_size, float scale, int nsplit) {
    smla_status st = check_decode_args(q, kv_cache, num_pages, page_table, pt_stride, seq_lens, B,
                                       T, H, K, page_size, scale);
    if (st != SMLA_OK) return st;
    if (nsplit < 0 || nsplit > SMLA_MAX_NSPLIT) return SMLA_ERR_INVALID_ARG;
    if (B > 0 && T > 0 && H > 0 && seq_lens == nullptr) return SMLA_ERR_INVALID_ARG;
    return SMLA_OK;
}

PartialParams dense_params(const void *q, const void *kv_cache, int64_t num_pages,
                           const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                           int B, int T, int H, int K, float scale, const DensePlan &d) {
    PartialParams p = make_params(q, kv_cache, num_pages, page_table, pt_stride, nullptr, B,
                                  d.units, d.pack * H, K, scale, d.nsplit);
    p.seq_lens = seq_lens;
    p.pack = d.pack;
    p.dense_t = T;
    p.dense_h = H;
    return p;
}

}  // namespace

size_t smla_dense_workspace_bytes(int B, int T, int H, int K, int nsplit) {
    if (B < 0 || T < 0 || H < 0 || K < 0 || nsplit < 1 || nsplit > SMLA_MAX_NSPLIT) return 0;
    return nsplit > 1 ? smla_workspace_bytes(B, T, H, nsplit) : 0;
}

int smla_dense_nsplit(int B, int T, int H, int K) {
    if (B <= 0 || T <= 0 || H <= 0 || H > SMLA_MAX_HEADS || K <= 0) return 1;
    return dense_plan(B, T, H, K, 0).nsplit;
}

smla_status smla_decode_dense_partial(const void *q, const void *kv_cache, int64_t num_pages,
                                      const int32_t *page_table, int pt_stride,
                                      const int32_t *seq_lens, int B, int T, int H, int K,
                                      int page_size, float scale, int nsplit, float *part_o,
                                      float *part_m, float *part_lse, void *stream) {
    smla_status st = check_dense_args(q, kv_cache, num_pages, page_table, pt_stride, seq_lens, B,
                                      T, H, K, page_size, scale, nsplit);
    if (st != SMLA_OK) return st;
    if (nsplit < 1) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (part_o == nullptr || part_m == nullptr || part_lse == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(part_o, 16) || !aligned(part_m, 4) || !aligned(part_lse, 4))
        return SMLA_ERR_MISALIGNED;
    const DensePlan d = dense_plan(B, T, H, K, nsplit);
    if ((long long)B * d.units * d.nsplit > INT_MAX) return SMLA_ERR_INVALID_ARG;
    PartialParams p = dense_params(q, kv_cache, num_pages, page_table, pt_stride, seq_lens, B, T,
                                   H, K, scale, d);
    p.part_o = part_o;
    p.part_m = part_m;
    p.part_lse = part_lse;
    return launch_tc<false>(p, B * d.units * d.nsplit, static_cast<cudaStream_t>(stream));
}

smla_status smla_decode_dense(const void *q, const void *kv_cache, int64_t num_pages,
                              const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                              int B, int T, int H, int K, int page_size, float scale, int nsplit,
                              void *workspace, size_t workspace_bytes, void *o, float *lse,
                              void *stream) {
    smla_status st = check_dense_args(q, kv_cache, num_pages, page_table, pt_stride, seq_lens, B,
                                      T, H, K, page_size, scale, nsplit);
    if (st != SMLA_OK) return st;
    if (B == 0 || T == 0 || H == 0) return SMLA_OK;
    if (o == nullptr || lse == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(o, 16) || !aligned(lse, 4)) return SMLA_ERR_MISALIGNED;
    DensePlan d = dense_plan(B, T, H, K, nsplit);
    // Split boundaries on whole pages: every 32-row tile is then half a page
    // of consecutive cache rows, which the kernel moves by TMA.  Kc rounds up
    // to 64 positions, and ceil(K / Kc) <= nsplit splits remain.
    const int kc64 = K > 0 ? ((K + d.nsplit - 1) / d.nsplit + 63) / 64 * 64 : 0;
    if (K > 0) d.nsplit = (K + kc64 - 1) / kc64;
    if ((long long)B * d.units * d.nsplit > INT_MAX) return SMLA_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    PartialParams p = dense_params(q, kv_cache, num_pages, page_table, pt_stride, seq_lens, B, T,
                                   H, K, scale, d);
    if (K > 0) p.kc = kc64;
    const int grid = B * d.units * d.nsplit;
    if (d.nsplit == 1) {
        p.o = static_cast<__nv_bfloat16 *>(o);
        p.lse = lse;
        return launch_tc<true>(p, grid, s);
    }
    if (workspace_bytes < smla_workspace_bytes(B, T, H, d.nsplit)) return SMLA_ERR_WORKSPACE_TOO_SMALL;
    if (workspace == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SMLA_ERR_MISALIGNED;
    const size_t n = (size_t)B * T * H * d.nsplit;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t off_m = round256(n * smla::kDc * sizeof(float));
    const size_t off_l = off_m + round256(n * sizeof(float));
    p.part_o = reinterpret_cast<float *>(ws);
    p.part_m = reinterpret_cast<float *>(ws + off_m);
    p.part_lse = reinterpret_cast<float *>(ws + off_l);
    st = launch_tc<false>(p, grid, s);
    if (st != SMLA_OK) return st;
    return launch_combine(p.part_o, p.part_m, p.part_lse, B, T, H, d.nsplit, o, lse, s);
}

smla_status smla_selftest_wait_timeout(unsigned long long limit_ns, void *stream) {
    if (limit_ns < 1000ull || limit_ns > 1000000000ull) return SMLA_ERR_INVALID_ARG;
    smla::smla_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

smla_status smla_check_device(int clear, unsigned long long *n_bad_index, void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned int flags = 0;
    unsigned long long count = 0;
    e = cudaMemcpyFromSymbol(&flags, smla::g_status_flags, sizeof flags);
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&count, smla::g_bad_index_count, sizeof count);
    if (e == cudaSuccess && clear) {
        const unsigned int zf = 0;
        const unsigned long long zc = 0;
        e = cudaMemcpyToSymbol(smla::g_status_flags, &zf, sizeof zf);
        if (e == cudaSuccess) e = cudaMemcpyToSymbol(smla::g_bad_index_count, &zc, sizeof zc);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    if (n_bad_index) *n_bad_index = count;
    if (flags & smla::kFlagTimeout) return SMLA_ERR_TIMEOUT;
    if (flags & smla::kFlagIndexRange) return SMLA_ERR_INDEX_RANGE;
    return SMLA_OK;
}

// ---------------------------------------------------------------------------
// Top-k indexer (see include/smla.h and smla_indexer.cuh).
}  // extern "C"

static_assert(smla::ix_finish_smem_bytes(SMLA_INDEXER_MAX_N) <= 232448, "selection bitmaps must fit shared memory");

namespace {

// cuTensorMapEncodeTiled, reached through the runtime (no link against the
// driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        (void)cudaGetLastError();
    });
    return fn;
}

// 2-D bf16 tensor of `rows` rows of 128 values (256-byte rows), read in boxes
// of 64 values x box_rows rows with the 128-byte swizzle.
smla_status encode_rows128(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return SMLA_ERR_CUDA;
    }
    const cuuint64_t dims[2] = {(cuuint64_t)smla::kIxDim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)smla::kIxDim * 2};
    const cuuint32_t box[2] = {64u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed: %d", (int)r);
        return SMLA_ERR_CUDA;
    }
    return SMLA_OK;
}

}  // namespace

// The latent cache as a 2-D bf16 tensor [num_pages * 64 rows, 576], read in
// boxes of 32 rows x 64 values with the 128-byte swizzle.
smla_status encode_cache_tiles(CUtensorMap *map, const void *cache, int64_t num_pages) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return SMLA_ERR_CUDA;
    }
    const cuuint64_t dims[2] = {(cuuint64_t)smla::kD, (cuuint64_t)num_pages * smla::kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)smla::kRowBytes};
    const cuuint32_t box[2] = {64u, (cuuint32_t)smla::TcCfg::kTileRows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(cache), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed: %d", (int)r);
        return SMLA_ERR_CUDA;
    }
    return SMLA_OK;
}

namespace {

smla_status check_indexer_args(const void *q_index, const float *w, const void *k_index,
                               int64_t num_pages, const int32_t *page_table, int pt_stride,
                               const int32_t *n_vis, int B, int T, int HI, int max_n,
                               int page_size) {
    if (B < 0 || T < 0 || HI < 1 || max_n < 0) return SMLA_ERR_INVALID_ARG;
    if (page_size != SMLA_PAGE_SIZE) return SMLA_ERR_UNSUPPORTED;
    if (HI > SMLA_INDEXER_MAX_HEADS || max_n > SMLA_INDEXER_MAX_N) return SMLA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0) return SMLA_OK;
    if ((long long)B * T > SMLA_INDEXER_MAX_TOKENS) return SMLA_ERR_UNSUPPORTED;
    if ((long long)B * T * HI > INT_MAX) return SMLA_ERR_INVALID_ARG;
    if (!q_index || !w || !n_vis) return SMLA_ERR_INVALID_ARG;
    if (!aligned(q_index, 16) || !aligned(w, 4) || !aligned(n_vis, 4)) return SMLA_ERR_MISALIGNED;
    if (max_n > 0) {
        if (!k_index || !page_table || num_pages < 1 || pt_stride < 1) return SMLA_ERR_INVALID_ARG;
        if (num_pages > SMLA_MAX_PAGES) return SMLA_ERR_UNSUPPORTED;
        if (!aligned(k_index, 16) || !aligned(page_table, 4)) return SMLA_ERR_MISALIGNED;
    }
    return SMLA_OK;
}

size_t ix_plan_bytes(int B, int T) { return round256(((size_t)B * T + 1) * sizeof(int)); }

// Selection scratch: [hist | meta] (cleared per call), the position bitmap
// and the candidate list.
size_t ix_select_zeroed_bytes(int B, int T) {
    return (size_t)B * T * (smla::kIxSelBins * sizeof(unsigned) + sizeof(smla::IxSelMeta));
}
size_t ix_select_bytes(int B, int T, int max_n) {
    const size_t bt = (size_t)B * T, words = ((size_t)max_n + 31) / 32;
    return round256(ix_select_zeroed_bytes(B, T)) + round256(bt * words * sizeof(uint32_t)) +
           round256(bt * max_n * sizeof(uint2));
}

cudaLaunchConfig_t pdl_config(cudaStream_t st, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// Plan + scores into `scores` (row stride `stride` floats).  With sel_ws
// (the selection scratch), the plan kernel also clears its histograms and
// the score kernel fills them.
smla_status launch_ix_scores(const void *q_index, const float *w, const void *k_index,
                             int64_t num_pages, const int32_t *page_table, int pt_stride,
                             const int32_t *n_vis, int B, int T, int HI, int max_n, int *plan,
                             float *scores, long long stride, void *sel_ws, cudaStream_t st) {
    smla::IndexerParams p{};
    p.page_table = page_table;
    p.pt_stride = pt_stride;
    p.num_pages = num_pages;
    p.n_vis = n_vis;
    p.w = w;
    p.BT = B * T;
    p.T = T;
    p.HI = HI;
    p.max_n = max_n;
    p.tile_start = plan;
    p.scores = scores;
    p.score_stride = stride;
    int plan_grid = 1;
    if (sel_ws != nullptr && max_n > 0) {
        p.sel_hist = static_cast<unsigned *>(sel_ws);
        p.zero = static_cast<uint4 *>(sel_ws);
        p.n_zero = (long long)(ix_select_zeroed_bytes(B, T) / 16);
        plan_grid = (int)std::min<long long>(std::max<long long>(1, (p.n_zero + 1023) / 1024),
                                             current_device_sms());
    }
    smla::smla_ix_plan_kernel<<<plan_grid, 1024, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
    if (max_n == 0) return SMLA_OK;
    const int npad = HI <= 16 ? 16 : (HI <= 32 ? 32 : 64);
    CUtensorMap map_k, map_q;
    smla_status s = encode_rows128(&map_k, k_index, (uint64_t)num_pages * SMLA_PAGE_SIZE, 64u);
    if (s != SMLA_OK) return s;
    s = encode_rows128(&map_q, q_index, (uint64_t)B * T * HI, (uint32_t)npad);
    if (s != SMLA_OK) return s;
    const void *fn;
    int smem;
    if (npad == 16) {
        fn = reinterpret_cast<const void *>(&smla::smla_ix_score_kernel<16>);
        smem = smla::IxCfg<16>::kSmemBytes;
    } else if (npad == 32) {
        fn = reinterpret_cast<const void *>(&smla::smla_ix_score_kernel<32>);
        smem = smla::IxCfg<32>::kSmemBytes;
    } else {
        fn = reinterpret_cast<const void *>(&smla::smla_ix_score_kernel<64>);
        smem = smla::IxCfg<64>::kSmemBytes;
    }
    e = ensure_smem_attr(fn, smem);
    if (e != cudaSuccess) return cuda_fail(e);
    // the score kernel may start while the plan runs; it waits for it in-kernel
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(st, attr);
    cfg.gridDim = dim3((unsigned)current_device_sms());
    cfg.blockDim = dim3(smla::IxCfg<16>::kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    if (npad == 16)
        e = cudaLaunchKernelEx(&cfg, smla::smla_ix_score_kernel<16>, map_k, map_q, p);
    else if (npad == 32)
        e = cudaLaunchKernelEx(&cfg, smla::smla_ix_score_kernel<32>, map_k, map_q, p);
    else
        e = cudaLaunchKernelEx(&cfg, smla::smla_ix_score_kernel<64>, map_k, map_q, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

// The selection chain over scores (row stride `stride`).  hist_filled: the
// score kernel filled the histograms just before (smla_indexer_topk), so
// the clear and histogram kernels are skipped and the scores are read only
// after the wait.
smla_status launch_ix_select(const float *scores, long long stride, const int32_t *n_vis, int B,
                             int T, int max_n, int K, void *workspace, int32_t *out, bool hist_filled,
                             cudaStream_t st) {
    smla::IndexerParams p{};
    p.n_vis = n_vis;
    p.BT = B * T;
    p.T = T;
    p.max_n = max_n;
    p.K = K;
    p.scores = const_cast<float *>(scores);
    p.score_stride = stride;
    p.out = out;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t bt = (size_t)B * T;
    p.sel_hist = reinterpret_cast<unsigned *>(ws);
    p.sel_meta = reinterpret_cast<smla::IxSelMeta *>(ws + bt * smla::kIxSelBins * sizeof(unsigned));
    p.sel_words = (max_n + 31) / 32;
    const size_t off_bits = round256(ix_select_zeroed_bytes(B, T));
    p.sel_bits = reinterpret_cast<uint32_t *>(ws + off_bits);
    p.sel_cand = reinterpret_cast<uint2 *>(ws + off_bits + round256(bt * p.sel_words * sizeof(uint32_t)));
    p.sel_chunks = (max_n + smla::kIxSelChunk - 1) / smla::kIxSelChunk;
    // The chain: [clear, hist,] mark, finish; every kernel after the first
    // may start early and waits on its predecessor in-kernel.
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(st, attr);
    cudaError_t e;
    if (max_n > 0) {
        cfg.gridDim = dim3((unsigned)((long long)p.BT * p.sel_chunks));
        cfg.blockDim = dim3(smla::kIxSelThreads);
        if (!hist_filled) {
            const long long n16 = (long long)(ix_select_zeroed_bytes(B, T) / 16);
            const long long blocks = std::min<long long>((n16 + 255) / 256, 4ll * current_device_sms());
            smla::smla_ix_clear_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<uint4 *>(ws), n16);
            e = cudaGetLastError();
            if (e != cudaSuccess) return cuda_fail(e);
            cfg.dynamicSmemBytes = 0;
            e = cudaLaunchKernelEx(&cfg, smla::smla_ix_hist_kernel, p);
            if (e != cudaSuccess) return cuda_fail(e);
            p.sel_prefetch = 1;
        }
        e = ensure_smem_attr(reinterpret_cast<const void *>(&smla::smla_ix_mark_kernel),
                             smla::kIxMarkSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e);
        cfg.dynamicSmemBytes = smla::kIxMarkSmemBytes;
        e = cudaLaunchKernelEx(&cfg, smla::smla_ix_mark_kernel, p);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    e = ensure_smem_attr(reinterpret_cast<const void *>(&smla::smla_ix_finish_kernel),
                         smla::ix_finish_smem_bytes(SMLA_INDEXER_MAX_N));
    if (e != cudaSuccess) return cuda_fail(e);
    cfg.gridDim = dim3((unsigned)p.BT);
    cfg.blockDim = dim3(smla::kIxFinishThreads);
    cfg.dynamicSmemBytes = smla::ix_finish_smem_bytes(max_n);
    e = cudaLaunchKernelEx(&cfg, smla::smla_ix_finish_kernel, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? SMLA_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

size_t smla_indexer_workspace_bytes(int B, int T, int max_n) {
    if (B < 0 || T < 0 || max_n < 0) return 0;
    return ix_plan_bytes(B, T) + round256((size_t)B * T * max_n * sizeof(float)) +
           ix_select_bytes(B, T, max_n);
}

size_t smla_indexer_select_workspace_bytes(int B, int T, int max_n) {
    if (B < 0 || T < 0 || max_n < 0) return 0;
    return ix_select_bytes(B, T, max_n);
}

smla_status smla_indexer_scores(const void *q_index, const float *w, const void *k_index,
                                int64_t num_pages, const int32_t *page_table, int pt_stride,
                                const int32_t *n_vis, int B, int T, int HI, int max_n,
                                int page_size, void *workspace, size_t workspace_bytes,
                                float *scores, void *stream) {
    smla_status st = check_indexer_args(q_index, w, k_index, num_pages, page_table, pt_stride,
                                        n_vis, B, T, HI, max_n, page_size);
    if (st != SMLA_OK) return st;
    if (B == 0 || T == 0 || max_n == 0) return SMLA_OK;
    if (scores == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(scores, 4)) return SMLA_ERR_MISALIGNED;
    if (workspace_bytes < ix_plan_bytes(B, T)) return SMLA_ERR_WORKSPACE_TOO_SMALL;
    if (workspace == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SMLA_ERR_MISALIGNED;
    return launch_ix_scores(q_index, w, k_index, num_pages, page_table, pt_stride, n_vis, B, T, HI,
                            max_n, static_cast<int *>(workspace), scores, max_n, nullptr,
                            static_cast<cudaStream_t>(stream));
}

smla_status smla_indexer_select(const float *scores, const int32_t *n_vis, int B, int T, int max_n,
                                int K, void *workspace, size_t workspace_bytes, int32_t *topk_idx,
                                void *stream) {
    if (B < 0 || T < 0 || max_n < 0 || K < 1) return SMLA_ERR_INVALID_ARG;
    if (max_n > SMLA_INDEXER_MAX_N) return SMLA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0) return SMLA_OK;
    if ((long long)B * T > SMLA_INDEXER_MAX_TOKENS) return SMLA_ERR_UNSUPPORTED;
    if (!n_vis || !topk_idx || (max_n > 0 && !scores)) return SMLA_ERR_INVALID_ARG;
    if (!aligned(n_vis, 4) || !aligned(topk_idx, 4) || !aligned(scores, 4)) return SMLA_ERR_MISALIGNED;
    if (workspace_bytes < ix_select_bytes(B, T, max_n)) return SMLA_ERR_WORKSPACE_TOO_SMALL;
    if (workspace == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SMLA_ERR_MISALIGNED;
    return launch_ix_select(scores, max_n, n_vis, B, T, max_n, K, workspace, topk_idx, false,
                            static_cast<cudaStream_t>(stream));
}

smla_status smla_indexer_topk(const void *q_index, const float *w, const void *k_index,
                              int64_t num_pages, const int32_t *page_table, int pt_stride,
                              const int32_t *n_vis, int B, int T, int HI, int max_n, int K,
                              int page_size, void *workspace, size_t workspace_bytes,
                              int32_t *topk_idx, void *stream) {
    smla_status st = check_indexer_args(q_index, w, k_index, num_pages, page_table, pt_stride,
                                        n_vis, B, T, HI, max_n, page_size);
    if (st != SMLA_OK) return st;
    if (K < 1) return SMLA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return SMLA_OK;
    if (topk_idx == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 4)) return SMLA_ERR_MISALIGNED;
    if (workspace_bytes < smla_indexer_workspace_bytes(B, T, max_n)) return SMLA_ERR_WORKSPACE_TOO_SMALL;
    if (workspace == nullptr) return SMLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return SMLA_ERR_MISALIGNED;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *plan = reinterpret_cast<int *>(ws);
    float *scores = reinterpret_cast<float *>(ws + ix_plan_bytes(B, T));
    void *sel_ws = ws + ix_plan_bytes(B, T) + round256((size_t)B * T * max_n * sizeof(float));
    st = launch_ix_scores(q_index, w, k_index, num_pages, page_table, pt_stride, n_vis, B, T, HI,
                          max_n, plan, scores, max_n, sel_ws, s);
    if (st != SMLA_OK) return st;
    return launch_ix_select(scores, max_n, n_vis, B, T, max_n, K, sel_ws, topk_idx, true, s);
}

}  // extern "C"
