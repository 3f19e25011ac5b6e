/*
 * smla.h -- C ABI of the split-K sparse MLA decode library (libsmla.so).
 *
 * The operation.  For every query token (b, t) and head h, attend over the
 * top-k latent KV rows that idx[b, t, :] selects from a paged cache:
 *
 *   row r        = [ c_r (512 bf16) | k_pe_r (64 bf16) ]        (576 bf16, 1152 B)
 *   q[b,t,h]     = [ q_nope (512 bf16) | q_pe (64 bf16) ]
 *   s_j          = scale * ( q_nope . c_r + q_pe . k_pe_r )       r = row of idx[b,t,j]
 *   o[b,t,h]     = sum_j softmax(s)_j * c_r                       (512 values)
 *   lse[b,t,h]   = ln sum_j exp(s_j)
 *
 * Sources.  "The Moment of Truth: Validating Split-K Parallelization for
 * Blackwell MLA Decode", section "The Split-K Imperative": the sparse MLA
 * decode kernel attends over top-k candidate tokens retrieved from the KV
 * cache; split-K partitions that top-k axis across thread blocks, each block
 * computing a partial attention output, and a log-sum-exp combine kernel
 * merges them.  "The Occupancy Hypothesis: How One Kernel Parameter Unlocked
 * 1.8x Decode Speedup on Blackwell", sections "The Occupancy Insight" and
 * "The Broader Context": NSPLIT multiplies the grid; its best value depends
 * on SM count, heads, batch and query length.  The pages print no formula,
 * dimension or index convention; the definition above is the standard
 * absorbed-MLA decode reading, and the conventions below are this library's.
 *
 * Index convention.  idx holds logical token positions of sequence b.  A
 * position i maps to physical cache row
 *     page_table[b * pt_stride + i / 64] * 64 + i % 64.
 * -1 is padding and contributes nothing.  Any other entry with i < 0,
 * i >= pt_stride * 64, or whose page entry is outside [0, num_pages), is also
 * treated as padding and counted in a device-side counter that
 * smla_check_device() reports as SMLA_ERR_INDEX_RANGE.  Duplicate entries
 * each count once.  A token with no valid entry gets o = 0, lse = -inf.
 *
 * Split convention.  With S = nsplit, Kc = ceil(K / S): split s covers index
 * positions [s*Kc, min(K, (s+1)*Kc)).  Trailing splits may be short or empty.
 * This is exactly what smla_decode_partial writes.  The whole-decode entry
 * points may instead cover a token with at most S pieces of unequal length
 * (see smla_decode); their results differ only in rounding order.
 *
 * Common rules for every entry point:
 *  - All pointers are DEVICE pointers on the current device, owned by the
 *    caller, except the per-step buffers of smla_decode_host (pinned host
 *    memory).  The library allocates no device memory at run time; it keeps a
 *    small host-side cache of per-device kernel attributes and, for
 *    smla_decode_noalloc, one static device array per GPU.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Arguments are checked on the host before
 *    anything is launched; a failed check launches nothing.
 *  - The first kernel of a decode is launched as a programmatic dependent
 *    of the stream's previous work: its grid may be scheduled early, but it
 *    waits for that work to complete before it touches global memory.  This
 *    keeps stream order for every predecessor that is itself ordered (any
 *    kernel launched without the programmatic attribute, a copy, an event).
 *  - q, kv_cache, part_o, o and workspace must be 16-byte aligned; int32 and
 *    fp32 arrays 4-byte aligned.  Otherwise SMLA_ERR_MISALIGNED.
 *  - Dimensions are fixed at 512 + 64 and page_size must be 64; heads per
 *    query token at most 64; num_pages at most SMLA_MAX_PAGES.  Otherwise
 *    SMLA_ERR_UNSUPPORTED.
 *  - B, T, H or K equal to 0 are legal (K = 0: every o = 0, lse = -inf).
 *  - K (an index list's width, the dense variant's longest visible length,
 *    the indexer's selection width) must be at most SMLA_MAX_K: the host's
 *    split arithmetic (ceil(K / nsplit), rounded up to whole pages, plus K)
 *    and the kernels' fill loops are 32-bit.  This is a precondition the
 *    library does not check; the Python binding refuses larger K.
 *  - Output buffers are the caller's and must hold the element counts each
 *    entry point lists (o [B, T, H, 512], lse [B, T, H], the partials
 *    [B, T, H, nsplit(, 512)], the indexer's [B, T, K] and [B, T, max_n]);
 *    the library writes through the pointers without knowing their extent.
 *  - A CUDA error at launch returns SMLA_ERR_CUDA; smla_last_error() gives
 *    its text.  No entry point throws, aborts or exits.
 *  - Entry points may be called from several host threads on different
 *    streams at once.
 */
#ifndef SMLA_H_
#define SMLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SMLA_DC 512        /* latent (value) width */
#define SMLA_DR 64         /* shared RoPE key width */
#define SMLA_D 576         /* cache row width in bf16 elements */
#define SMLA_PAGE_SIZE 64  /* tokens per cache page */
#define SMLA_MAX_HEADS 64
#define SMLA_MAX_NSPLIT 1024
#define SMLA_MAX_PAGES 33554431 /* cache rows must be addressable as int32 */
#define SMLA_MAX_K 1073741760   /* 2^30 - 64: largest K (a precondition, see below) */

typedef enum {
    SMLA_OK = 0,
    SMLA_ERR_INVALID_ARG = 1,
    SMLA_ERR_UNSUPPORTED = 2,
    SMLA_ERR_MISALIGNED = 3,
    SMLA_ERR_WORKSPACE_TOO_SMALL = 4,
    SMLA_ERR_INDEX_RANGE = 5,
    SMLA_ERR_CUDA = 6,
    SMLA_ERR_TIMEOUT = 7
} smla_status;

/*
 * NSPLIT heuristic (host only, no CUDA call unless sm_count <= 0).
 * "The Occupancy Hypothesis ...", section "The Broader Context": the right
 * NSPLIT depends on SM count, heads per rank, batch size and query length;
 * section "The Occupancy Insight": more blocks in flight hide memory latency.
 * One CTA serves all heads of one (b, t, split), so the grid is B*T*NSPLIT
 * CTAs.  The heuristic picks the NSPLIT in [1, min(SMLA_MAX_NSPLIT, ceil(K/32))]
 * that minimises a model of wave count x rows per CTA plus per-CTA overhead
 * and the split-K scratch traffic, with two resident CTAs per SM for H <= 16
 * and one otherwise.  It also prices smla_decode's balanced schedule (one
 * full wave of equal CTAs, ceil(SMs x resident / (B*T)) + 1 slots, H <= 32)
 * and returns that slot count only when the model favours it by more than 15%.
 * sm_count <= 0 queries the current device.  If the environment variable SMLA_NSPLIT holds a positive integer,
 * that value is returned instead (clamped to [1, SMLA_MAX_NSPLIT]).
 * Returns >= 1; returns 1 for degenerate sizes.
 */
int smla_choose_nsplit(int B, int T, int H, int K, int sm_count);

/*
 * Bytes of workspace smla_decode needs for this shape and nsplit (>= 1):
 * part_o, part_m and part_lse, each rounded up to 256 bytes.
 * Returns 0 for invalid arguments.
 */
size_t smla_workspace_bytes(int B, int T, int H, int nsplit);

/*
 * Split-K partial pass ("The Split-K Imperative": each block computes a
 * partial attention output over its chunk of the top-k axis).
 *
 *   q          bf16  [B, T, H, 576]                 device, 16-B aligned
 *   kv_cache   bf16  [num_pages, 64, 576]           device, 16-B aligned
 *   page_table int32 [B, pt_stride]                 device
 *   topk_idx   int32 [B, T, K], -1 = padding        device
 *   scale      softmax scale applied to the full 576-wide dot product
 *   nsplit     S in [1, SMLA_MAX_NSPLIT]
 * Outputs (fp32, device, caller-owned):
 *   part_o   [B, T, H, S, 512]  sum_j exp(s_j - part_m) c_j   (unnormalised)
 *   part_m   [B, T, H, S]       the reference point part_o is scaled by: at
 *                               most 8 ln 2 below the split's maximum score
 *                               and never above it (the tcgen05 kernel moves
 *                               it only when a score exceeds it by more than
 *                               that; the others keep the exact maximum);
 *                               -inf for a split with no valid entry
 *   part_lse [B, T, H, S]       ln sum_j exp(s_j) over the split (-inf if empty)
 * so part_o * exp(part_m - part_lse) is the split's normalised output.
 * An empty split writes part_o = 0, part_m = part_lse = -inf.
 */
smla_status smla_decode_partial(const void *q, const void *kv_cache, int64_t num_pages,
                                const int32_t *page_table, int pt_stride,
                                const int32_t *topk_idx, int B, int T, int H, int K,
                                int page_size, float scale, int nsplit, float *part_o,
                                float *part_m, float *part_lse, void *stream);

/*
 * LSE combine ("The Split-K Imperative": partial outputs merged by a
 * log-sum-exp combine kernel).  Per (b, t, h):
 *   M = max_s part_m,  L = sum_s exp(part_lse_s - M)
 *   o = sum_s exp(part_m_s - M) part_o_s / L     -> bf16 [B, T, H, 512]
 *   lse = M + ln L                               -> fp32 [B, T, H]
 * All splits empty: o = 0, lse = -inf.  Inputs as written by
 * smla_decode_partial with the same B, T, H, nsplit.
 */
smla_status smla_lse_combine(const float *part_o, const float *part_m, const float *part_lse,
                             int B, int T, int H, int nsplit, void *o, float *lse,
                             void *stream);

/*
 * Whole decode: partial pass then combine, on one stream.  nsplit = 0 picks
 * smla_choose_nsplit(B, T, H, K, <current device SMs>).  The workspace holds
 * the partials; it must be at least smla_workspace_bytes(B, T, H, S) for the
 * S actually used (size it with the value smla_choose_nsplit returns), else
 * SMLA_ERR_WORKSPACE_TOO_SMALL.  With S = 1 the partial pass writes o and
 * lse directly and the workspace is not touched (it may then be NULL).
 * S is the number of partial slots per query token.  When an equal split
 * into S chunks would leave a partly filled last wave of CTAs (pipelined
 * kernels, H <= 32), the call instead covers each token's top-k axis with at
 * most S contiguous pieces of unequal length, so that exactly one wave of
 * CTAs carries equal work; the LSE combine is exact for any partition, so
 * only the rounding order differs from smla_decode_partial's equal split.
 * The workspace contents on entry do not matter.
 *   o   bf16 [B, T, H, 512] device, 16-B aligned
 *   lse fp32 [B, T, H]      device
 */
smla_status smla_decode(const void *q, const void *kv_cache, int64_t num_pages,
                        const int32_t *page_table, int pt_stride, const int32_t *topk_idx,
                        int B, int T, int H, int K, int page_size, float scale, int nsplit,
                        void *workspace, size_t workspace_bytes, void *o, float *lse,
                        void *stream);

/*
 * The partial pass of smla_decode alone (nsplit >= 2): the same kernel,
 * schedule and workspace layout smla_decode uses -- equal splits, or the
 * balanced schedule's pieces in nsplit slots per token -- with the partials
 * left in the workspace.  The workspace holds, at offsets 0, round256(n * 512
 * * 4) and that plus round256(n * 4) with n = B*T*H*nsplit, part_o
 * [B,T,H,nsplit,512], part_m and part_lse [B,T,H,nsplit]; smla_lse_combine on
 * them completes the decode (it ignores a slot with part_m = -inf).  Splitting
 * the decode this way lets a caller schedule other work between the two
 * launches or time the partial pass alone.  Arguments and errors as for
 * smla_decode.
 */
smla_status smla_decode_partial_ws(const void *q, const void *kv_cache, int64_t num_pages,
                                   const int32_t *page_table, int pt_stride,
                                   const int32_t *topk_idx, int B, int T, int H, int K,
                                   int page_size, float scale, int nsplit, void *workspace,
                                   size_t workspace_bytes, void *stream);

/*
 * Checked mode: synchronises `stream`, then reads the current device's
 * sticky error state, optionally clearing it.  *n_bad_index (may be NULL)
 * receives the number of out-of-range index entries seen since the last
 * clear (each counted once per query token).  Returns SMLA_ERR_TIMEOUT if a
 * kernel gave up a bounded wait, else SMLA_ERR_INDEX_RANGE if any entry was
 * out of range, else SMLA_OK (or SMLA_ERR_CUDA).
 */
smla_status smla_check_device(int clear, unsigned long long *n_bad_index, void *stream);

/*
 * Whole decode with no caller-provided workspace and no allocation.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory at the moment they decode: code running
 * inside a region that must not call cudaMalloc (an allocator that is itself
 * being serviced, a memory pool that is locked or exhausted, a host process
 * that only ever receives device pointers from someone else), or plain C
 * callers with no allocator of their own.  It behaves like smla_decode with
 * the same arguments minus the workspace: the split-K partials live instead in
 * one scratch array of SMLA_NOALLOC_SCRATCH_BYTES that the library itself
 * holds in device memory on every GPU that loads it, until the process exits.
 *
 *  - q, kv_cache, page_table, topk_idx, o, lse: as for smla_decode (device,
 *    caller-owned).  nsplit = 0 picks the heuristic's value, lowered to the
 *    largest split count whose partials fit the scratch array.
 *  - If smla_workspace_bytes(B, T, H, S) for the split count actually used is
 *    larger than SMLA_NOALLOC_SCRATCH_BYTES, the call launches nothing and
 *    returns SMLA_ERR_WORKSPACE_TOO_SMALL (smla_last_error() says how many
 *    bytes were needed); pass a smaller nsplit or use smla_decode.
 *  - The first call on each device looks up that device's copy of the scratch
 *    array (cudaGetSymbolAddress, with the device current); make that first
 *    call before starting any stream capture.  The call itself never calls
 *    cudaMalloc, cudaFree or an allocating library routine.  The array is,
 *    however, part of the library's device code image: CUDA maps that image
 *    (code plus the 16 MiB array) into device memory when it loads the module
 *    on a device, which under lazy module loading (the CUDA 12 default)
 *    happens at the library's first launch or symbol lookup on that device --
 *    possibly inside the first smla_decode_noalloc call.  A caller that may
 *    not see device memory change at all inside its critical region should
 *    make one call (of any library entry point that launches work) on each
 *    device beforehand.  Later calls change no device memory reservation.
 *  - The looked-up address is kept per device together with the context it
 *    belongs to, and looked up again when the device's current context has
 *    changed (after a cudaDeviceReset(), the next call runs in the new
 *    primary context and finds its array there).
 *  - All calls on a device share the one array and it keeps whatever the last
 *    call left in it; nothing in it has to start at zero, because every split
 *    the combine reads is written first by the same call.  Calls whose work
 *    overlaps on the GPU (different streams, or host threads racing on one
 *    device) race on the array and produce wrong results: serialise them.
 */
#define SMLA_NOALLOC_SCRATCH_BYTES (16u << 20)
smla_status smla_decode_noalloc(const void *q, const void *kv_cache, int64_t num_pages,
                                const int32_t *page_table, int pt_stride,
                                const int32_t *topk_idx, int B, int T, int H, int K,
                                int page_size, float scale, int nsplit, void *o, float *lse,
                                void *stream);

/*
 * Whole decode for per-step data that lives in host memory.
 *
 * The pages have no counterpart to this entry point; it serves decode loops
 * whose query vectors, top-k indices and page tables are produced on the host
 * each step and whose outputs are consumed there.  q, page_table, topk_idx, o
 * and lse are PINNED host memory (cudaHostAlloc / cudaMallocHost /
 * cudaHostRegister, which on a unified-addressing system the GPU can address
 * directly); kv_cache and workspace are device memory as for smla_decode.
 * One small copy kernel pulls q, the indices and the page table over the
 * host link into a staging area at the end of the workspace, then the decode
 * runs as smla_decode does and writes o and lse straight into the host
 * buffers.  This avoids the per-transfer latency of separate copies.  The
 * copy kernel issues all of a thread's loads before its stores (one round trip
 * over the host link for a small step), and the decode's first kernel is its
 * programmatic dependent, so that kernel's launch overlaps the copy.
 *
 *  - workspace_bytes must be at least smla_workspace_host_bytes(B, T, H, K,
 *    pt_stride, nsplit) for the nsplit actually used (0 picks the heuristic's
 *    value), else SMLA_ERR_WORKSPACE_TOO_SMALL.
 *  - Any host pointer that is not pinned host memory visible to the current
 *    device returns SMLA_ERR_INVALID_ARG before anything is launched.
 *  - Asynchronous on `stream`: the host may read o and lse after
 *    synchronising the stream, and must not rewrite q, page_table or topk_idx
 *    before then.
 */
size_t smla_workspace_host_bytes(int B, int T, int H, int K, int pt_stride, int nsplit);
smla_status smla_decode_host(const void *q_host, const void *kv_cache, int64_t num_pages,
                             const int32_t *page_table_host, int pt_stride,
                             const int32_t *topk_idx_host, int B, int T, int H, int K,
                             int page_size, float scale, int nsplit, void *workspace,
                             size_t workspace_bytes, void *o_host, float *lse_host, void *stream);

/*
 * Dense-context decode: the KV-split verify variant.
 *
 * "The Occupancy Hypothesis: How One Kernel Parameter Unlocked 1.8x Decode
 * Speedup on Blackwell", sections "The Road to This Experiment", "The
 * Occupancy Insight" and "The Broader Context": the speculative-decoding
 * verify kernel attends each of q_len query tokens to its whole visible KV
 * sequence (46K tokens there), split into NSPLIT chunks, each a partial pass,
 * merged by a reduce.  Here query token (b, t) attends to the positions
 * 0 .. seq_lens[b*T + t] - 1 of sequence b, mapped through the page table
 * like a sparse index: the sparse definition with the index list of every
 * visible position.  For causal verify of T draft tokens appended at the end
 * of a sequence of n tokens, seq_lens[b*T + t] = n - T + t + 1.
 *
 * The partial kernel packs up to 64 / H query tokens of one sequence into the
 * 64 query rows of one tcgen05 pass over the rows, each row masked at its own
 * length, so a row read from HBM serves all of them.
 *
 *  - seq_lens  int32 [B, T], device memory, each in [0, K].  A length outside
 *              that range is clamped to it and raises SMLA_ERR_INDEX_RANGE in
 *              smla_check_device (counted once per query token).
 *  - K         the longest visible length.  smla_decode_dense rounds the
 *              split length ceil(K / nsplit) up to whole pages (64 positions)
 *              and uses the ceil(K / that) <= nsplit splits it needs, so that
 *              every 32-row tile is half a page of consecutive cache rows;
 *              smla_decode_dense_partial keeps split s at positions
 *              [s Kc, (s+1) Kc), Kc = ceil(K / nsplit), as for an index list
 *              of width K.
 *  - nsplit    0 picks smla_dense_nsplit(B, T, H, K).
 *  - Other arguments, layouts and outputs are those of smla_decode.  A
 *    visible position that no page maps is masked and counted once per
 *    position and packed group of query tokens.
 *  - workspace_bytes must be at least smla_dense_workspace_bytes(B, T, H, K,
 *    nsplit) for the nsplit used (the split-K partials; 0 for nsplit 1), else
 *    SMLA_ERR_WORKSPACE_TOO_SMALL; a workspace not 16-byte aligned gives
 *    SMLA_ERR_MISALIGNED.
 *
 * smla_decode_dense_partial runs the partial pass alone (nsplit >= 1) and
 * writes part_o / part_m / part_lse exactly as smla_decode_partial does for
 * the equivalent index lists; smla_lse_combine merges them.
 */
int smla_dense_nsplit(int B, int T, int H, int K);
size_t smla_dense_workspace_bytes(int B, int T, int H, int K, int nsplit);
smla_status smla_decode_dense(const void *q, const void *kv_cache, int64_t num_pages,
                              const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                              int B, int T, int H, int K, int page_size, float scale, int nsplit,
                              void *workspace, size_t workspace_bytes, void *o, float *lse,
                              void *stream);
smla_status smla_decode_dense_partial(const void *q, const void *kv_cache, int64_t num_pages,
                                      const int32_t *page_table, int pt_stride,
                                      const int32_t *seq_lens, int B, int T, int H, int K,
                                      int page_size, float scale, int nsplit, float *part_o,
                                      float *part_m, float *part_lse, void *stream);

/*
 * Self-test of the bounded waits (no counterpart on the pages).  Every wait in
 * the library's kernels gives up after a time limit, raises a sticky timeout
 * flag and lets the kernel return, so a broken pipeline never hangs the GPU.
 * This launches one warp that waits on a barrier nothing arrives at, through
 * the same wait routine, with limit_ns in [1e3, 1e9]; afterwards
 * smla_check_device() reports SMLA_ERR_TIMEOUT (and clears it when asked).
 * SMLA_ERR_INVALID_ARG for a limit outside the range.
 */
smla_status smla_selftest_wait_timeout(unsigned long long limit_ns, void *stream);

/*
 * Top-k indexer: the step that produces topk_idx for the decode.
 *
 * "The Negative Result That Refined the Hunt: Disabling the MMA FlashMLA
 * Kernel", section "The Context: A Systematic Bisection Campaign": the
 * deployment runs an indexer kernel and a bf16 index-key path ahead of the
 * sparse MLA decode kernel, which attends over the top-k candidate tokens
 * ("The Moment of Truth ...", section "The Split-K Imperative").  The pages
 * give no formula; this library follows the published DeepSeek
 * sparse-attention indexer.  For query token (b, t) and each visible
 * position s in [0, n_vis[b*T + t]) of sequence b:
 *
 *   logit_j(s) = q_index[b,t,j,:] . k_index[row(s), :]     128 bf16 values, fp32 sum
 *   I(s)       = sum_j w[b,t,j] * max(0, logit_j(s))        j < HI, fp32
 *
 * with row(s) = page_table[b*pt_stride + s/64]*64 + s%64 (the latent cache's
 * page table; the index-key cache is paged the same way).  The selection is
 * the min(K, number of candidates) positions with the largest I; equal scores
 * go to the smaller position.  topk_idx[b, t, :] lists the selected positions
 * in ascending order, then -1 up to width K -- the index-list convention of
 * smla_decode.
 *
 *   q_index    bf16 [B, T, HI, 128]       device, 16-B aligned
 *   w          fp32 [B, T, HI]            device
 *   k_index    bf16 [num_pages, 64, 128]  device, 16-B aligned
 *   page_table int32 [B, pt_stride]       device
 *   n_vis      int32 [B, T]               device: visible positions per query token
 *   HI         index heads, 1..SMLA_INDEXER_MAX_HEADS
 *   max_n      an upper bound on n_vis (sizes the score buffer and the work),
 *              at most SMLA_INDEXER_MAX_N; a length outside [0, max_n] is
 *              clamped and counted
 *   K          selection width >= 1
 *   B * T      at most SMLA_INDEXER_MAX_TOKENS
 * A visible position whose page entry is outside [0, num_pages), or past
 * pt_stride*64, is not a candidate; it is counted (SMLA_ERR_INDEX_RANGE in
 * smla_check_device).  Scores that are NaN are not candidates either.
 *
 * smla_indexer_topk runs both steps; its workspace must hold
 * smla_indexer_workspace_bytes(B, T, max_n) bytes (a per-token tile plan,
 * the fp32 scores and the selection scratch).  The two steps are also
 * exported:
 *   smla_indexer_scores writes I(s) into scores [B, T, max_n] (fp32, row
 *     stride max_n) for every visible s; a position that is not a candidate
 *     gets NaN; entries at s >= n_vis are not written.  Its workspace needs
 *     only the tile plan, which smla_indexer_workspace_bytes(B, T, 0) bytes
 *     cover.
 *   smla_indexer_select applies the selection rule to given scores of that
 *     layout (NaN = not a candidate; -0 and +0 are equal).  Its workspace
 *     must hold smla_indexer_select_workspace_bytes(B, T, max_n) bytes: per
 *     token a 16 KiB digit histogram, a position bitmap and a candidate list
 *     of max_n positions.  Scratch only: nothing carries over between calls.
 * Workspaces are device memory, 16-B aligned, owned by the caller and in use
 * until the call's work on `stream` completes.
 * Asynchronous on `stream`; errors as for the decode entry points.
 */
#define SMLA_INDEXER_DIM 128
#define SMLA_INDEXER_MAX_HEADS 64
#define SMLA_INDEXER_MAX_TOKENS 1048576
#define SMLA_INDEXER_MAX_N 524288   /* visible positions per query token */
size_t smla_indexer_workspace_bytes(int B, int T, int max_n);
size_t smla_indexer_select_workspace_bytes(int B, int T, int max_n);
smla_status smla_indexer_topk(const void *q_index, const float *w, const void *k_index,
                              int64_t num_pages, const int32_t *page_table, int pt_stride,
                              const int32_t *n_vis, int B, int T, int HI, int max_n, int K,
                              int page_size, void *workspace, size_t workspace_bytes,
                              int32_t *topk_idx, void *stream);
smla_status smla_indexer_scores(const void *q_index, const float *w, const void *k_index,
                                int64_t num_pages, const int32_t *page_table, int pt_stride,
                                const int32_t *n_vis, int B, int T, int HI, int max_n,
                                int page_size, void *workspace, size_t workspace_bytes,
                                float *scores, void *stream);
smla_status smla_indexer_select(const float *scores, const int32_t *n_vis, int B, int T,
                                int max_n, int K, void *workspace, size_t workspace_bytes,
                                int32_t *topk_idx, void *stream);

/* Static text for a status code. */
const char *smla_status_string(smla_status status);

/* Text of the last CUDA error seen by this host thread ("" if none). */
const char *smla_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int smla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SMLA_H_ */
