/*
 * dsa_decode.h -- C ABI of libdsa.so: the decode/verify step of a DeepSeek
 * Sparse Attention (DSA) layer with a GQA-4 backbone, on one NVIDIA B200.
 *
 * The step (NaiveAI research page, naive.ai/en/research):
 *   1. Indexer scan.  "Technical Details > Model Architecture": a lightweight
 *      indexer scores the full history.  "Hybrid SWA-DSA Architecture": the
 *      indexer has 16 query heads.  The page does not print the scoring rule;
 *      this library uses the DSA indexer's form
 *          I[t,s] = scale[s] * sum_{j<16} w[t,j] * ReLU(q_idx[t,j,:] . k_idx[s,:])
 *      over 64-dim keys (scale = 1 unless a per-token scale is given).
 *   2. Causal top-k.  "Hybrid SWA-DSA Architecture": DSA selects the top
 *      2,048 tokens.  Query t sits at position pos[t] and may select
 *      s in [0, pos[t]].  If pos[t] + 1 <= topk every visible position is
 *      selected; otherwise the topk largest scores, equal scores going to the
 *      lower position, which makes the result unique.  "AI-Centered R&D in
 *      Practice" requires bitwise-identical results run to run; every kernel
 *      here is deterministic.
 *   3. Sparse attention.  "Hybrid SWA-DSA Architecture": GQA with four KV
 *      groups; "NaiveRT > Optimizing inside the kernel": eight query heads
 *      per GPU under TP8, i.e. 64 query heads.  For head h (group g = h / 16)
 *          out[t,h,:] = sum_{s in S_t} softmax_s(q[t,h,:] . K[s,g,:] / sqrt(128)) V[s,g,:]
 *      over the selected set S_t only.
 *
 * Conventions for every entry point:
 *   - Device pointers unless stated otherwise.  The caller owns every buffer;
 *     the library keeps no pointer after a call returns.  Outputs must not
 *     alias inputs.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: results are valid once the stream reaches
 *     that point.  No entry point synchronises, except dsa_device_status.
 *   - Arguments are checked on the host before any launch; a failed check
 *     returns DSA_ERR_INVALID_ARG (or DSA_ERR_UNSUPPORTED for a shape this
 *     build does not handle) and launches nothing; dsa_last_error() then
 *     describes it.  Kernels never trap: an anomaly found on the device (an
 *     out-of-range selected index given to dsa_sparse_attn, a bounded wait that
 *     ran out) sets a device error word that dsa_device_status reports.
 *   - Inputs with NaN (an E4M3 code S.1111.111, a NaN bf16) give unspecified
 *     output values but never an out-of-bounds access.
 */
#ifndef DSA_DECODE_H
#define DSA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *dsa_stream_t;

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1, /* a null pointer, bad shape, stride, alignment, dtype, pos or topk */
    DSA_ERR_UNSUPPORTED = 2, /* head shape or size outside what this build implements */
    DSA_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch, allocation, ...) */
    DSA_ERR_DEVICE = 4       /* a kernel reported an anomaly (see dsa_device_status) */
} dsa_status_t;

typedef enum {
    DSA_BF16 = 0,     /* bfloat16, 2 bytes */
    DSA_FP8_E4M3 = 1, /* OCP FP8 E4M3, 1 byte */
    DSA_F32 = 2,      /* IEEE binary32 */
    DSA_I32 = 3       /* int32 */
} dsa_dtype_t;

/* A strided tensor view.  Strides are in elements; the innermost dimension must
 * have stride 1 and every other stride must keep rows 16-byte aligned.  `scale`
 * is read only for the indexer key cache: a per-token fp32 scale [L] (device),
 * or NULL for 1. */
typedef struct {
    void *data;
    int32_t dtype;      /* dsa_dtype_t */
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];
    const float *scale;
} dsa_tensor_t;

/* Shapes (T = query tokens, 1..8; L = cached positions, including the query
 * tokens' own; topk in 1..2048):
 *   q            [T][64][128]      bf16, contiguous        backbone queries (post-RoPE)
 *   q_idx        [T][16][64]       bf16, contiguous        indexer queries
 *   w_idx        [T][16]           f32, contiguous         indexer head weights
 *   k_idx_cache  [L][64]           bf16 or fp8-e4m3, row stride >= 64 and a multiple
 *                                  of 16 bytes; optional per-token scale [L] f32 (> 0)
 *   kv_cache     [L][2][4][128]    bf16; per token the K rows of the 4 groups, then
 *                                  the V rows; token stride >= 1024 elements and a
 *                                  multiple of 8; inner dims contiguous
 *   pos          HOST int32 [T],   0 <= pos[t] < L
 *   out          [T][64][128]      bf16, contiguous        attention output
 *   sel_idx      [T][topk]         int32, row stride >= topk: the selected positions of
 *                                  query t in ascending order, then -1 padding
 * All device base addresses must be 16-byte aligned. */

/* Bytes of workspace dsa_decode_ws needs for these sizes (0 if they are invalid).
 * Workspace contract (dsa_decode_ws, dsa_topk_from_scores, dsa_sparse_attn and
 * the other calls that take a workspace): the caller owns the memory; its first
 * DSA_WS_CTRL_BYTES bytes are the control region -- grid-barrier words,
 * per-query flags and a launch counter in the first 1024 bytes, then two radix
 * histograms that successive launches alternate between -- which must be zero
 * before the workspace's first use (one cudaMemsetAsync when it is created).  Every call leaves it ready for the next one (barrier and
 * per-query words back at zero, the histogram the next call uses cleared), so
 * later calls need no reset.  A launch that finds its barrier or per-query
 * words non-zero flags DSA_ERR_DEVICE (error word bit 0x8) and skips the
 * work that depends on them.  One workspace serves one call at a time: calls that may overlap on the
 * GPU need separate workspaces. */
#define DSA_WS_CTRL_BYTES 263168
DSA_API size_t dsa_workspace_bytes(int32_t T, int64_t L, int32_t topk);

/* The whole step: indexer scan, causal top-k, sparse attention -- two kernel
 * launches on `stream` (the indexer, then the cooperative top-k/attention
 * kernel as its programmatic dependent).  Takes its
 * workspace stream-ordered (cudaMallocAsync, a zeroing of its control words,
 * cudaFreeAsync, all on `stream`), so it
 * must not be captured into a CUDA graph on a device without memory-pool
 * support; use dsa_decode_ws for graphs. */
DSA_API dsa_status_t dsa_decode(const dsa_tensor_t *q, const dsa_tensor_t *q_idx, const dsa_tensor_t *w_idx,
                        const dsa_tensor_t *k_idx_cache, const dsa_tensor_t *kv_cache,
                        const int32_t *pos, int32_t topk, dsa_tensor_t *out, dsa_tensor_t *sel_idx,
                        dsa_stream_t stream);

/* Same as dsa_decode with a caller-provided device workspace of at least
 * dsa_workspace_bytes(T, L, topk) bytes, 256-byte aligned.  Makes no allocation
 * and no synchronisation, so it can be captured in a CUDA graph (pos is read
 * on the host at call time and baked into the launches). */
DSA_API dsa_status_t dsa_decode_ws(const dsa_tensor_t *q, const dsa_tensor_t *q_idx, const dsa_tensor_t *w_idx,
                           const dsa_tensor_t *k_idx_cache, const dsa_tensor_t *kv_cache,
                           const int32_t *pos, int32_t topk, dsa_tensor_t *out, dsa_tensor_t *sel_idx,
                           dsa_stream_t stream, void *workspace, size_t workspace_bytes);

/* dsa_decode_ws with an attention sink: `sink` is a per-head logit [64] f32
 * (device, 16-byte aligned, not NULL) that joins each head's softmax denominator
 * with no value row.  NaiveAI research page, "Hybrid SWA-DSA Architecture":
 * both attention types of the model carry a sink bias. */
DSA_API dsa_status_t dsa_decode_sink_ws(const dsa_tensor_t *q, const dsa_tensor_t *q_idx,
                                        const dsa_tensor_t *w_idx, const dsa_tensor_t *k_idx_cache,
                                        const dsa_tensor_t *kv_cache, const int32_t *pos, int32_t topk,
                                        const float *sink, dsa_tensor_t *out, dsa_tensor_t *sel_idx,
                                        dsa_stream_t stream, void *workspace, size_t workspace_bytes);

/* dsa_decode_ws with the query positions in device memory: pos_device is int32
 * [T] (T = q's first dimension), read by the kernel at launch, so one CUDA graph
 * of the step serves every decode position (write the next positions into the
 * buffer, replay).  The work is split over the whole cache [0, L) instead of the
 * positions known on the host, and the short-context bypass does not apply.  A
 * position outside [0, L) is clamped and flags DSA_ERR_DEVICE (bit 16).  sink is
 * NULL or as in dsa_decode_sink_ws.  NaiveAI research page, "The execution
 * model": rounds of the decoding loop advance on the device without the host. */
DSA_API dsa_status_t dsa_decode_devpos_ws(const dsa_tensor_t *q, const dsa_tensor_t *q_idx,
                                          const dsa_tensor_t *w_idx, const dsa_tensor_t *k_idx_cache,
                                          const dsa_tensor_t *kv_cache, const int32_t *pos_device, int32_t topk,
                                          const float *sink, dsa_tensor_t *out, dsa_tensor_t *sel_idx,
                                          dsa_stream_t stream, void *workspace, size_t workspace_bytes);

/* Short-context bypass (on by default): when every query of a step sees at most
 * topk positions (pos[t] + 1 <= topk), the top-k selects everything, so the step
 * skips the indexer and the selection and takes the visible positions directly.
 * Results are identical either way; 0 turns the bypass off (process-wide).
 * NaiveAI research page, "A faster microbenchmark is not a faster model", weighs
 * the same trade at 200 and 2,200 tokens. */
DSA_API void dsa_set_short_context_bypass(int32_t enable);

/* Sliding-window decode: attention of q [T][64][128] bf16 over the last
 * min(pos[t] + 1, window) positions of kv_cache (the same [L][2][4][128] bf16
 * layout and GQA grouping as the sparse step), 1 <= window <= 2048, optional
 * sink as in dsa_decode_sink_ws (NULL for none); out [T][64][128] bf16.
 * Workspace: dsa_workspace_bytes(T, L, window), control words as described
 * there.  NaiveAI research page, "Hybrid SWA-DSA Architecture": the SWA layers
 * attend over a 128-token window. */
DSA_API dsa_status_t dsa_swa_decode(const dsa_tensor_t *q, const dsa_tensor_t *kv_cache, const int32_t *pos,
                                    int32_t window, const float *sink, dsa_tensor_t *out, dsa_stream_t stream,
                                    void *workspace, size_t workspace_bytes);

/* Stage 1 alone: scores [T][ld] f32 (ld >= L, a multiple of 4).  scores[t][s] is
 * I[t,s] for s <= pos[t] and -inf for s > pos[t].  The sum is taken in fp32
 * (tensor-core dot products, then a fixed-order weighted sum over heads).
 * NaiveAI research page, "Technical Details > Model Architecture": the
 * lightweight indexer scores every cached position (it still scans the full
 * history); "Hybrid SWA-DSA Architecture": 16 indexer query heads. */
DSA_API dsa_status_t dsa_index_scores(const dsa_tensor_t *q_idx, const dsa_tensor_t *w_idx,
                              const dsa_tensor_t *k_idx_cache, const int32_t *pos, float *scores,
                              int64_t ld, dsa_stream_t stream);

/* Stage 2 alone: causal top-k of caller scores [T][ld] (f32, ld >= L, a multiple
 * of 4; entries s > pos[t] are ignored).  -0 and +0 compare equal.  Writes sel_idx
 * [T][sel_ld] (sel_ld >= topk).  Workspace: dsa_workspace_bytes(T, L, topk).
 * NaiveAI research page, "Hybrid SWA-DSA Architecture": DSA keeps the top
 * 2,048 positions of the indexer's scores; "AI-Centered R&D in Practice":
 * bitwise-reproducible results, hence the lower-position tie rule. */
DSA_API dsa_status_t dsa_topk_from_scores(const float *scores, int32_t T, int64_t L, int64_t ld,
                                  const int32_t *pos, int32_t topk, int32_t *sel_idx, int64_t sel_ld,
                                  dsa_stream_t stream, void *workspace, size_t workspace_bytes);

/* Stage 2 without any allocation: the same computation and arguments as
 * dsa_topk_from_scores, minus the workspace.  It is for callers that cannot
 * allocate device memory when they run this step: code inside a CUDA graph
 * capture or a real-time decode loop that forbids allocation after start-up,
 * or a host whose device memory is entirely owned by another allocator.  The
 * paper has no counterpart; this is an interface choice of this library.
 * Its scratch is a static device array of about 17.3 MB inside libdsa.so; every
 * GPU that loads the library holds it until the process exits.
 *   - Limits: T <= 8 and L <= 262144 scores per query; larger L returns
 *     DSA_ERR_INVALID_ARG (say "exceeds the no-allocation scratch limit").
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call outside any
 *     stream capture.
 *   - Every call shares the one array and clears the parts that must start at
 *     zero; calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on it and must be serialised by the caller. */
DSA_API dsa_status_t dsa_topk_from_scores_noalloc(const float *scores, int32_t T, int64_t L, int64_t ld,
                                                  const int32_t *pos, int32_t topk, int32_t *sel_idx,
                                                  int64_t sel_ld, dsa_stream_t stream);

/* Stage 3 alone: attention of q over the rows listed in sel_idx [T][topk]
 * (entries < 0 are skipped; an entry outside [0, pos[t]] is skipped and flags
 * DSA_ERR_DEVICE).  `sink` is NULL or a per-head logit [64] f32 (device) that
 * joins each head's softmax denominator with no value row (an attention sink).
 * Workspace: dsa_workspace_bytes(T, L, topk).  NaiveAI research page,
 * "Technical Details > Model Architecture": the backbone attends only to the
 * selected subset; "Hybrid SWA-DSA Architecture": GQA with four KV groups and
 * a sink bias. */
DSA_API dsa_status_t dsa_sparse_attn(const dsa_tensor_t *q, const dsa_tensor_t *kv_cache,
                             const dsa_tensor_t *sel_idx, const int32_t *pos, const float *sink,
                             dsa_tensor_t *out, dsa_stream_t stream, void *workspace,
                             size_t workspace_bytes);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: DSA_OK, DSA_ERR_DEVICE (an anomaly was flagged since the last
 * call), or DSA_ERR_CUDA (the stream reported an error). */
DSA_API dsa_status_t dsa_device_status(dsa_stream_t stream);

/* Static description of a status code. */
DSA_API const char *dsa_status_str(dsa_status_t status);

/* Detail of the last failed call on this host thread ("" if none). */
DSA_API const char *dsa_last_error(void);

/* Number of kernels this library has launched in this process (all devices). */
DSA_API uint64_t dsa_launch_count(void);

/* Profiling hook for the calling host thread.  With n == 5, dsa_decode and
 * dsa_decode_ws record five cudaEvent_t on their stream: events[0] before the
 * first launch, events[1] between the indexer kernel and the cooperative
 * top-k/attention kernel (when the indexer runs; the event then stands between
 * them in the stream, so the second kernel's launch no longer overlaps the
 * first's tail), events[2], events[3] and events[4] at the end of the call.
 * n == 0 disables; any other n is ignored. */
DSA_API void dsa_set_stage_events(void *const *events, int32_t n);

/* Failure-detection test hook for the calling host thread (one launch only).
 * The next cooperative-kernel launch from this thread makes each of its waits
 * between blocks (the grid barrier where there is one, the per-query counters)
 * wait for one arrival more than its grid makes: a block that never comes.  Every wait then runs into its bound after limit_cycles SM clocks
 * (1000 <= limit_cycles <= 2e9, the normal bound), sets the wait-timeout bit
 * (1) of the device error word and skips the work that depended on the
 * barrier; the launch still ends normally and leaves the workspace control
 * words at zero, so the next call runs as usual.  Only waits between blocks are
 * affected; waits for a block's own copies in flight keep their normal bound.
 * NaiveAI research page, "NaiveRT > A DSA layer: from 29 kernels to one": the
 * cooperative top-k/attention kernel depends on synchronisation between its
 * CTAs, which is what a bounded wait guards.  Returns DSA_ERR_INVALID_ARG for a limit
 * outside the range. */
DSA_API dsa_status_t dsa_debug_fail_next_barriers(int64_t limit_cycles);

/* Profiling hook for the calling host thread: when device_buffer is not NULL,
 * every launch records, per block b and slot k < 32, the GPU global timer (ns)
 * into ((uint64_t*)device_buffer)[b * 32 + k] at the phase boundaries of the
 * step: 0 start, 1 indexer scan done (both from the indexer kernel when it
 * runs), 31 start of the cooperative kernel, 2/3 candidate extraction (after
 * its grid barrier where there is one), 4/5 the per-query selection (blocks
 * 0..T-1 only), 6 first attention item starts (after its query's selection), 7
 * attention done, 9 merge done, 30 end; slots 28, 27 and 29 hold the SM clock counter at the start of
 * the first kernel, at the start of the cooperative kernel and at the end.  The
 * buffer must hold dsa_step_grid(...) * 32 entries.  NULL disables. */
DSA_API void dsa_set_step_trace(void *device_buffer);

/* Blocks of the step kernel on the current device (one per SM); 0 on error. */
DSA_API int32_t dsa_step_grid(int32_t fp8_keys);

#ifdef __cplusplus
}
#endif
#endif /* DSA_DECODE_H */
