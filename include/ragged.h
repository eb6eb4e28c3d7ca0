/*
 * ragged.h - C ABI of the pack -> attend -> unpack pipeline for token-pruned
 * Vision Transformers, after "Dispatch-Aware Ragged Attention for Pruned
 * Vision Transformers" (arXiv 2604.15408).
 *
 * The pipeline has three steps:
 *   1. pack:   per-image keep masks -> cu_seqlens, and the surviving token
 *              rows (CLS always kept) gathered into one flat ragged buffer;
 *   2. attend: bidirectional multi-head softmax attention over every
 *              variable-length sequence of that buffer, with no causal mask,
 *              no KV cache and no padding;
 *   3. unpack: extract each sequence's CLS row, or scatter rows back to their
 *              dense positions.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers named as device buffers are device memory of the current CUDA
 *    device, owned by the caller.  The library allocates nothing per call and
 *    keeps no pointer after returning.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is only enqueued: no call synchronises with the device,
 *    except ragged_get_device_status and ragged_pipeline with
 *    RAGGED_PIPELINE_SYNC, which say so.
 *  - Every call returns a ragged_status.  Argument errors are detected on the
 *    host before anything is enqueued; nothing is launched then and
 *    ragged_last_error() describes the problem.  A launch failure reported by
 *    the CUDA runtime returns RAGGED_ERR_CUDA.  Problems only the device can
 *    see (inconsistent cu_seqlens, a bounded wait that gave up) set bits of a
 *    per-device status word read by ragged_get_device_status; the affected
 *    sequence is skipped rather than read or written out of bounds.
 *  - Calls may be captured into a CUDA graph; none of them synchronises or
 *    allocates.
 *  - Sizes are int64_t; lengths and offsets inside cu_seqlens are int32, so
 *    B * L_full must stay below 2^31.
 */
#ifndef RAGGED_H
#define RAGGED_H

#include <stdint.h>

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(RAGGED_BUILD) && defined(__GNUC__)
#define RAGGED_API __attribute__((visibility("default")))
#else
#define RAGGED_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ragged_status {
    RAGGED_OK = 0,
    RAGGED_ERR_INVALID_ARG = 1, /* null pointer, negative size, misalignment, ... */
    RAGGED_ERR_UNSUPPORTED = 2, /* valid request outside what is implemented    */
    RAGGED_ERR_CUDA = 3,        /* the CUDA runtime reported an error           */
    RAGGED_ERR_DEVICE = 4       /* reserved for device-side failures            */
} ragged_status;

typedef enum ragged_dtype {
    RAGGED_F16 = 0,  /* IEEE binary16                     */
    RAGGED_BF16 = 1, /* bfloat16                          */
    RAGGED_F32 = 2   /* IEEE binary32 (FFMA check path)   */
} ragged_dtype;

/* Bits of the per-device status word (ragged_get_device_status). */
#define RAGGED_DEV_BAD_SEQLENS 0x1u /* cu_seqlens decreasing, or a length > max_seqlen */
#define RAGGED_DEV_TIMEOUT 0x2u     /* a bounded device-side wait gave up              */

/* Largest L_full accepted by pack/unpack and max_seqlen by attention. */
#define RAGGED_MAX_TOKENS 16384

/*
 * ragged_pack - survivor bookkeeping and gather (step 1).
 * Paper: radpulse article, section "Integrated pack pipeline, 2.24x
 * end-to-end" (cu_seqlens computed first, survivors copied with coalesced
 * copies into a contiguous flat tensor) and its section on the FA2 dispatch
 * ceiling (survivors packed into a contiguous ragged buffer for a varlen API).
 *
 *   dense       device, [B, L_full] rows of row_bytes bytes, contiguous,
 *               16-byte aligned.  Read only.
 *   B, L_full   images and dense tokens per image; 0 <= B <= 65535 (above:
 *               RAGGED_ERR_UNSUPPORTED), 1 <= L_full <= RAGGED_MAX_TOKENS.
 *   row_bytes   bytes per token row; a positive multiple of 16.
 *   keep        device, uint8 [B, L_full], any alignment.  Nonzero keeps the
 *               token.  Token 0 (CLS) is kept whatever keep[b, 0] says.
 *   packed      device, capacity B * L_full rows of row_bytes, 16-byte
 *               aligned.  On completion rows 0..T-1 hold the survivors, image
 *               by image, each image's survivors in ascending token order
 *               (so CLS of image b is row cu_seqlens[b]).  Rows >= T are not
 *               written.
 *   cu_seqlens  device, int32 [B + 1]: cu[0] = 0, cu[b+1] = cu[b] + L_b where
 *               L_b >= 1 is the survivor count of image b; T = cu[B].
 *   src_idx     device int32 [B * L_full] or NULL: for each packed row t,
 *               the flat dense row b * L_full + j it was copied from.
 * B == 0 writes cu_seqlens[0] = 0 and nothing else.
 */
RAGGED_API ragged_status ragged_pack(const void *dense, int64_t B, int64_t L_full, int64_t row_bytes,
                          const uint8_t *keep, void *packed, int32_t *cu_seqlens,
                          int32_t *src_idx, void *stream);

/*
 * ragged_attn_fwd - ragged bidirectional attention (step 2).
 * Paper: abstract (lightweight bidirectional attention kernel over ragged
 * ViT sequences) and radpulse section "Bypassing the binding" (no causal
 * mask, no KV cache, no softmax_lse workspace).  For every sequence b (rows
 * cu[b] .. cu[b+1]-1) and head h:
 *        O_b,h = softmax(scale * Q_b,h K_b,h^T) V_b,h
 * over the L_b rows of that sequence only.  Accumulation and softmax are in
 * fp32; the output is rounded to nearest even in the input format.
 *
 *   q, k, v        device; element (t, h, c) of each is at
 *                  base[t * tok_stride + h * head_stride + c].  Separate
 *                  tensors or the three slices of one fused [T, 3, H, 64]
 *                  buffer.  16-byte aligned.
 *   tok_stride, head_stride   in elements; each times the element size must
 *                  be a multiple of 16 bytes.
 *   cu_seqlens     device int32 [B + 1], non-decreasing, cu[0] = 0 (as
 *                  written by ragged_pack).  Read on the device only.
 *   B              number of sequences, 0 .. 65535 (0 is a no-op; above:
 *                  RAGGED_ERR_UNSUPPORTED).
 *   max_seqlen     host-side upper bound on every L_b (e.g. L_full), 1 ..
 *                  RAGGED_MAX_TOKENS.  Sizes the launch; a sequence longer
 *                  than this is skipped and RAGGED_DEV_BAD_SEQLENS is set.
 *                  Small launches (few sequences x heads) with max_seqlen up
 *                  to 640, and max_seqlen up to 64, keep each sequence's K
 *                  and V resident in shared memory (one load burst, keys split
 *                  across warps); other launches stream K/V tiles.
 *   H, head_dim    heads (>= 1) and head dimension (only 64 is implemented:
 *                  other values return RAGGED_ERR_UNSUPPORTED).
 *   scale          softmax scale, positive and finite; usually 1/sqrt(head_dim).
 *   dtype          format of q, k, v, out and cls_out.
 *   out            device, element (t, h, c) at out[t * out_tok_stride + h *
 *                  head_dim + c]; out_tok_stride >= H * head_dim, times the
 *                  element size a multiple of 16 bytes.  16-byte aligned.
 *   cls_out        device [B, H * head_dim] contiguous, or NULL: receives
 *                  row cu[b] of out for every b (the CLS extraction of step
 *                  3 fused into the attention epilogue).
 */
RAGGED_API ragged_status ragged_attn_fwd(const void *q, const void *k, const void *v, int64_t tok_stride,
                              int64_t head_stride, const int32_t *cu_seqlens, int64_t B,
                              int64_t max_seqlen, int64_t H, int64_t head_dim, float scale,
                              ragged_dtype dtype, void *out, int64_t out_tok_stride,
                              void *cls_out, void *stream);

/* Attention kernels (ragged_set_attn_kernel). */
#define RAGGED_ATTN_AUTO 0       /* per launch shape (default): RESIDENT for launches too
                                    small to fill the GPU or single-tile sequences,
                                    PERSISTENT for launches of at least 8 (sequence,
                                    128-query tile, head) items per SM (B <= 1024),
                                    TCGEN05 for other long sequences, STREAMING otherwise */
#define RAGGED_ATTN_STREAMING 1  /* mma.sync, K/V tiles streamed, any max_seqlen            */
#define RAGGED_ATTN_RESIDENT 2   /* mma.sync, whole sequence in shared memory, <= 640 keys */
#define RAGGED_ATTN_TCGEN05 3    /* tcgen05.mma with TMEM accumulators, K/V streamed, one
                                    CTA per (128-query tile, head, sequence)               */
#define RAGGED_ATTN_PERSISTENT 4 /* tcgen05.mma, persistent CTAs with a TMA load warp;
                                    B <= 1024, H <= 1023, max_seqlen <= 2047 * 128 and
                                    B * H * ceil(max_seqlen / 128) at most 1024 items per
                                    CTA (two CTAs per SM); otherwise RAGGED_ATTN_TCGEN05   */

/*
 * ragged_set_attn_kernel - process-wide choice of the f16/bf16 attention
 * kernel used by ragged_attn_fwd (and by the split mode of ragged_pipeline).
 * All kernels compute the same operation to the same tolerance; the choice
 * only changes speed.  Returns the previous choice, or -1 (and changes
 * nothing) for an unknown value.  A launch whose max_seqlen exceeds what the
 * chosen kernel holds (640 keys for RAGGED_ATTN_RESIDENT) returns
 * RAGGED_ERR_UNSUPPORTED.  The fp32 check path
 * has a single kernel.
 */
RAGGED_API int32_t ragged_set_attn_kernel(int32_t kernel);

/*
 * ragged_mask_l2 - Threshold-l2 keep mask (a device-side mask producer).
 * Paper: radpulse section "Integrated pack pipeline" (the pipeline is
 * independent of the pruning method; Threshold-l2 is among those named).  The
 * pages give no rule; the reading: token j of image b is kept when the
 * Euclidean norm of its feature vector is at least tau, and CLS always.
 *
 *   x           device, token (b, j) is the C elements starting at element
 *               (b * L_full + j) * tok_stride; f16, bf16 or f32 (dtype),
 *               aligned to its element size.  Read only.
 *   B, L_full   B >= 0 images (B = 0 is a no-op), 1 <= L_full <= RAGGED_MAX_TOKENS,
 *               B * L_full < 2^31 (else RAGGED_ERR_UNSUPPORTED).  One launch
 *               covers up to 65,535 images; larger batches take several,
 *               enqueued in order on the stream.
 *   C           elements per token, 1 <= C <= 2^24; tok_stride >= C.
 *   tau         threshold, not NaN.
 *   keep        device uint8 [B, L_full]: 1 kept, 0 dropped (an input for
 *               ragged_pack / ragged_pipeline).
 * The decision is exact, whatever the order of summation: a token is kept
 * when sum(x_c^2) >= tau^2 in exact arithmetic, CLS always.  With tau <= 0
 * every token is kept except those with a NaN element, which are always
 * dropped; a token with an infinite element (and no NaN) is always kept.  A
 * sum within a relative 2^-29 of the exact one (fp32 squares with error-free
 * two-sum accumulation for f16 / bf16 rows on 16-byte boundaries with C a
 * multiple of 8 up to 8192, else fp64) settles the bit unless it lies within
 * a relative 2^-26 of tau^2; there one lane forms the sum exactly, as an
 * integer multiple of 2^-298, which costs O(C) serial steps for that token.
 */
RAGGED_API ragged_status ragged_mask_l2(const void *x, int64_t B, int64_t L_full, int64_t C, int64_t tok_stride,
                                        ragged_dtype dtype, double tau, uint8_t *keep, void *stream);

/*
 * ragged_pack_topk - score top-k selection fused into pack: one launch
 * produces the keep decision, cu_seqlens and the packed rows.
 * Paper: as ragged_pack, and the mask-producer reading above: image b keeps
 * CLS and the k_b - 1 other tokens with the highest scores (ties: the lower
 * index; NaN ranks below every number); k_b = keep_count[b] clamped to
 * [1, L_full], so cu[b + 1] = cu[b] + k_b.
 *
 *   dense, B, L_full, row_bytes, packed, cu_seqlens, src_idx: as ragged_pack.
 *   scores      device float32 [B, L_full], 4-byte aligned; scores[b, 0]
 *               (CLS) is not used.
 *   keep_count  device int32 [B]: survivors per image, CLS included.
 *   keep_out    device uint8 [B, L_full] or NULL: receives the selection
 *               (for ragged_unpack).
 * Each CTA sorts its image's scores in shared memory (a bitonic network over
 * L_full rounded up to a power of two); -0 and +0 tie, NaNs of any payload
 * tie.  L_full is limited to 8192 here (RAGGED_ERR_UNSUPPORTED above it).
 */
RAGGED_API ragged_status ragged_pack_topk(const void *dense, int64_t B, int64_t L_full, int64_t row_bytes,
                                          const float *scores, const int32_t *keep_count, void *packed,
                                          int32_t *cu_seqlens, int32_t *src_idx, uint8_t *keep_out, void *stream);

/*
 * ragged_unpack_cls - CLS extraction (step 3).
 * Paper: radpulse section "Integrated pack pipeline" (after attention and the
 * MLP run on the packed tokens, the CLS token is extracted).
 *
 *   packed      device, rows of row_bytes, contiguous, 16-byte aligned.
 *   cu_seqlens  device int32 [B + 1].
 *   row_bytes   positive multiple of 16.
 *   cls_out     device [B] rows of row_bytes: cls_out[b] = packed[cu[b]].
 */
RAGGED_API ragged_status ragged_unpack_cls(const void *packed, const int32_t *cu_seqlens, int64_t B,
                                int64_t row_bytes, void *cls_out, void *stream);

/*
 * ragged_unpack - scatter back (step 3, full form).
 * Paper: the pipeline's last step, "scatter the result back, or extract the
 * CLS rows" (the pack-attend-unpack pipeline of the abstract), and radpulse
 * section "Integrated pack pipeline" (survivors kept in a flat tensor whose
 * rows map back to their images).  The inverse of ragged_pack's gather: dense_out[b, j] = packed[cu[b] + r]
 * for the r-th survivor j of image b (same keep mask, CLS always kept).  Rows
 * of dropped tokens are left untouched.
 *
 *   packed      device, rows of row_bytes, 16-byte aligned.
 *   cu_seqlens  device int32 [B + 1] from ragged_pack on the same keep mask.
 *   keep        device uint8 [B, L_full].
 *   dense_out   device [B, L_full] rows of row_bytes, 16-byte aligned.
 *   B, L_full, row_bytes   limits as for ragged_pack.
 */
RAGGED_API ragged_status ragged_unpack(const void *packed, const int32_t *cu_seqlens, const uint8_t *keep,
                            int64_t B, int64_t L_full, int64_t row_bytes, void *dense_out,
                            void *stream);

/* ragged_pipeline modes (flags). */
#define RAGGED_PIPELINE_AUTO 0u  /* choose per shape (see below)                  */
#define RAGGED_PIPELINE_FUSED 1u /* one launch: pack, attention and CLS together    */
#define RAGGED_PIPELINE_SPLIT 2u /* two launches: ragged_pack, then ragged_attn_fwd */
#define RAGGED_PIPELINE_SYNC 4u  /* return after the work has finished on `stream`  */

/*
 * ragged_pipeline - pack -> attend -> CLS in one host call.
 * Paper: radpulse section "Integrated pack pipeline, 2.24x end-to-end"
 * (cu_seqlens, survivor copy, attention, CLS extraction), and the abstract's
 * pack-attend-unpack pipeline.
 *
 * dense_qkv is one fused [B, L_full, 3, H, head_dim] buffer (q, k, v along
 * the third axis) in `dtype`.  Outputs: cu_seqlens [B + 1]; out [T, H,
 * head_dim] (capacity B * L_full rows, token stride H * head_dim); cls_out
 * [B, H * head_dim] unless NULL; packed_qkv [B * L_full (capacity), 3, H,
 * head_dim] (the survivors' rows, as ragged_pack writes them).
 *
 * Fused mode (f16 / bf16, L_full <= 640): a single launch in which every CTA
 * ranks its image's keep mask, gathers its rows straight from dense_qkv and
 * writes cu_seqlens, out and cls_out; packed_qkv is optional there (NULL: the
 * packed q/k/v is not materialised).  Split mode: ragged_pack into packed_qkv
 * (required) followed by ragged_attn_fwd.  AUTO picks the fused mode when it
 * is available and B is small enough that every CTA counting the survivors of
 * the images before its own stays cheap; otherwise the split mode.  Results
 * are identical in both modes.  Requirements as for ragged_pack and
 * ragged_attn_fwd, with max_seqlen = L_full and scale positive and finite.
 *
 * RAGGED_PIPELINE_SYNC (may be combined with either mode) makes the call wait
 * for the enqueued work (cudaStreamSynchronize on `stream`) before returning,
 * for callers that want the results on return without a second call; it is
 * the only form of any entry point besides ragged_get_device_status that
 * synchronises, and it must not be used during stream capture.
 */
RAGGED_API ragged_status ragged_pipeline(const void *dense_qkv, const uint8_t *keep, int64_t B,
                                         int64_t L_full, int64_t H, int64_t head_dim, float scale,
                                         ragged_dtype dtype, void *packed_qkv, int32_t *cu_seqlens,
                                         void *out, void *cls_out, uint32_t flags, void *stream);

/* Bytes of the fixed device scratch behind ragged_pipeline_noalloc (16 MiB). */
#define RAGGED_NOALLOC_SCRATCH_BYTES (16ll << 20)

/*
 * ragged_pipeline_noalloc - ragged_pipeline in its two-launch form, for
 * callers that must not allocate device memory.  The paper has no
 * counterpart: it is a packaging of the same pack and attention launches.
 *
 * Who needs it: a plugin hosted by a framework or inference server whose own
 * allocator owns all of device memory (a cudaMalloc behind its back breaks
 * its accounting or fails), code that runs while some thread captures a CUDA
 * graph in global capture mode (cudaMalloc is then an error), and services
 * that fix their device footprint when they start.  Such a caller can still
 * hand in its inputs and outputs, but not the packed q/k/v that the
 * two-launch pipeline passes from pack to attention.
 *
 * Here that intermediate lives in a fixed array of RAGGED_NOALLOC_SCRATCH_BYTES
 * bytes inside the library's device image.  Every GPU on which the library's
 * kernels are loaded holds it until the process exits.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 *   Arguments as ragged_pipeline, without packed_qkv and flags: dense_qkv
 *   [B, L_full, 3, H, head_dim], keep, cu_seqlens [B + 1], out (capacity
 *   B * L_full rows, token stride H * head_dim), cls_out (or NULL), stream.
 *   Results are identical to ragged_pipeline with RAGGED_PIPELINE_SPLIT.
 *
 * Limit: B * L_full * 3 * H * head_dim * element size must not exceed
 * RAGGED_NOALLOC_SCRATCH_BYTES (every token may survive); larger requests
 * return RAGGED_ERR_UNSUPPORTED before anything is enqueued.
 *
 * The first call on a device looks up the array's device address for that
 * device (cudaGetSymbolAddress, with that device current) and caches it; make
 * that first call before any stream capture.  All calls share the one array
 * and it keeps what the last call left there; nothing in it needs to start at
 * zero, since pack writes every row that attention then reads.  Two calls
 * whose work overlaps on the GPU (different streams, or different host
 * threads, without ordering between them) race on the array and may return
 * wrong results: order them on one stream or with events.
 */
RAGGED_API ragged_status ragged_pipeline_noalloc(const void *dense_qkv, const uint8_t *keep, int64_t B,
                                                 int64_t L_full, int64_t H, int64_t head_dim, float scale,
                                                 ragged_dtype dtype, int32_t *cu_seqlens, void *out,
                                                 void *cls_out, void *stream);

/*
 * A pipeline call recorded once as a CUDA graph that the library owns, so that
 * each later call is one graph launch, and with RAGGED_PIPELINE_SYNC the wait
 * for it too, in a single call.  Paper: radpulse section "Bypassing the
 * binding" and its section on the FA2 dispatch ceiling (the fixed host cost of
 * a varlen call is argument handling, allocation and the launch path; here a
 * call is one crossing into this library and one graph launch).
 *
 * ragged_pipeline_graph_create records ragged_pipeline with these arguments
 * (flags without RAGGED_PIPELINE_SYNC) on `stream`, which must be a created
 * stream, not the legacy default one.  It first runs the call once outside
 * the recording (so it validates the arguments and does the per-device set-up;
 * the outputs are written), then records it and instantiates the graph.  The
 * graph objects are allocated here, once.  Every launch reads and writes the
 * same buffers, with the same sizes; the buffers must stay valid until the
 * graph is destroyed.  *graph_out is NULL on failure.
 *
 * ragged_pipeline_graph_launch launches it on `stream` (any stream of the same
 * device); flags is 0 or RAGGED_PIPELINE_SYNC, which also waits for it
 * (cudaStreamSynchronize) before returning.  Launching allocates nothing.
 *
 * ragged_pipeline_graph_destroy frees the graph (NULL is a no-op).
 */
typedef struct ragged_pipeline_graph ragged_pipeline_graph;

RAGGED_API ragged_status ragged_pipeline_graph_create(const void *dense_qkv, const uint8_t *keep, int64_t B,
                                                      int64_t L_full, int64_t H, int64_t head_dim, float scale,
                                                      ragged_dtype dtype, void *packed_qkv, int32_t *cu_seqlens,
                                                      void *out, void *cls_out, uint32_t flags, void *stream,
                                                      ragged_pipeline_graph **graph_out);
RAGGED_API ragged_status ragged_pipeline_graph_launch(ragged_pipeline_graph *graph, void *stream, uint32_t flags);
RAGGED_API ragged_status ragged_pipeline_graph_destroy(ragged_pipeline_graph *graph);

/*
 * ragged_get_device_status - read and clear the status word of the current
 * device.  Synchronises with `stream` (the only call that does).  *host_out
 * receives the RAGGED_DEV_* bits set since the previous read.
 */
RAGGED_API ragged_status ragged_get_device_status(uint32_t *host_out, void *stream);

/* Static description of a status code. */
RAGGED_API const char *ragged_status_string(ragged_status status);

/* Description of the last error returned on the calling host thread. */
RAGGED_API const char *ragged_last_error(void);

/* ABI version of the library (bumped when a signature changes). */
RAGGED_API int32_t ragged_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RAGGED_H */
