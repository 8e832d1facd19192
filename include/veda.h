/*
 * veda.h -- C ABI of libveda: Veda-style learned block-sparse attention for
 * video diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * What the library computes (the pages state it in prose only):
 *   1. Tile pooling + selector projection.  A lightweight predictor scores
 *      blocks of the attention map; its trainable parts are a query and a key
 *      projection per layer, applied to tile-pooled Q and K (tao.media,
 *      "Affine launches MiniMax-H3 video studio and SN120 sparse attention
 *      competition", sections "Training the Selector, Not the Generator" and
 *      "How the SN120 Competition Works").  Pooling = the mean over the
 *      tokens that exist in a tile (a short last tile is averaged over its
 *      own tokens); projection = pooled row vector times W[h] ([d, r]).
 *   2. Tile scoring: s[i][j] = qhat_i . khat_j (raw dot product).
 *   3. Fixed-budget selection: per (batch, head, query tile) keep the
 *      `budget` key tiles of highest score, ties to the lowest tile index,
 *      emitted in ascending order (budgets: same article, section "How the
 *      SN120 Competition Works"; 32 reference + 32 video tiles chosen
 *      independently: veyrul.com, "Veda R2VA for MiniMax-H3", second
 *      paragraph).
 *   4. Block-sparse attention: each video query attends to every token of
 *      its query tile's kept video tiles, kept reference tiles, and every
 *      dense (text / VLM / audio) token, with one softmax over that set
 *      (same veyrul.com paragraph: text, VLM and audio attention stay dense).
 *      Tokens past the end of a segment are not keys.
 *
 * Conventions (all entry points):
 *   - Every pointer argument except `ws` sizes is a DEVICE pointer owned by
 *     the caller; the library allocates no device memory, and its only global
 *     state is per device and context (the streams and events that
 *     veda_attn_host reuses, the static array of veda_select_tiles_noalloc),
 *     so concurrent calls on different workspaces are safe.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream); calls return after enqueueing, without synchronising.
 *   - Argument errors are detected on the host before anything is launched
 *     and returned synchronously.  Errors found on the device (an index out
 *     of range, a bounded wait that ran out) are recorded in a sticky status
 *     word inside the workspace and returned by veda_check_status().
 *   - Layouts: activations are [B, n_tokens, H, d] with d contiguous and the
 *     other three strides given in ELEMENTS; every base pointer must be
 *     16-byte aligned and every stride * element size a multiple of 16 bytes.
 *     Selector weights are contiguous [H, d, r] in the problem's dtype.
 *     Kept-tile indices are contiguous int32 [B, H, n_q_tiles, budget].
 *     The attention output is contiguous [B, n_video_tokens, H, d] in the
 *     problem's dtype; the optional log-sum-exp is contiguous fp32
 *     [B, H, n_video_tokens] (natural log, of the scaled logits).
 */
#ifndef VEDA_H
#define VEDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VEDA_ABI_VERSION 1

#if defined(__GNUC__)
#define VEDA_API __attribute__((visibility("default")))
#else
#define VEDA_API
#endif

typedef struct CUstream_st* veda_stream_t; /* == cudaStream_t */

typedef enum {
    VEDA_OK = 0,
    VEDA_ERR_INVALID_ARG = -1,  /* bad pointer, size, stride, alignment or budget      */
    VEDA_ERR_UNSUPPORTED = -2,  /* valid but not implemented (d, tile, r, dtype, size) */
    VEDA_ERR_WORKSPACE = -3,    /* workspace NULL, misaligned or too small             */
    VEDA_ERR_CUDA = -4,         /* a CUDA launch or driver call failed                 */
    VEDA_ERR_TIMEOUT = -5,      /* device: a bounded wait ran out (kernel returned)    */
    VEDA_ERR_BAD_INDEX = -6,    /* device: a kept-tile index was outside its segment   */
    VEDA_ERR_FORMAT = -7,       /* a selector artifact is malformed or off its layout  */
    VEDA_ERR_IO = -8            /* a selector artifact could not be opened or read     */
} veda_status;

typedef enum { VEDA_F32 = 0, VEDA_BF16 = 1 } veda_dtype;

/* Problem flags. */
#define VEDA_FLAG_SIMT_ATTENTION 1u /* run attention on the fp32 SIMT kernel even
                                       where the tensor-core kernel applies (bf16,
                                       d = 128, tile = 128): a cross-check path  */
#define VEDA_FLAG_TEST_SHORT_WAITS 2u /* test hook for the failure path: the
                                       pipeline waits of the tensor-core kernels
                                       (attention, tile selection) give up after
                                       ~64 clocks, so the call stops early,
                                       frees its resources and reports
                                       VEDA_ERR_TIMEOUT through
                                       veda_check_status(); its output is then
                                       undefined.  No effect on the kernels
                                       without waits (pool + project, SIMT
                                       score, top-k, SIMT attention). */
#define VEDA_FLAG_UNFUSED_SELECTION 4u /* compute the tile scores with the fp32
                                       SIMT kernel instead of the tensor cores
                                       (a cross-check path; also used when
                                       r > 64) */
#define VEDA_FLAG_ONCHIP_SELECTION 8u /* select each row's top-k on chip while
                                       the tensor cores recompute its scores,
                                       writing no score matrix (see
                                       veda_score_topk_tiles); otherwise the
                                       tensor-core scores are written to the
                                       workspace and the warp-per-row top-k
                                       kernel selects from them */

/* One key/value segment, [B, n_tokens, H, d] (d contiguous). */
typedef struct {
    const void* k;
    const void* v;
    int64_t n_tokens;   /* 0: segment absent (ref / dense only) */
    int64_t stride_b;   /* element strides of k and v (shared) */
    int64_t stride_tok;
    int64_t stride_h;
    int32_t budget;     /* sparse segments: kept tiles per (query tile, head),
                           1 <= budget <= ceil(n_tokens / tile).
                           dense segment: must be 0. */
    int32_t reserved;
} veda_segment;

/* One attention layer call.  Queries are the video tokens (q has
 * video.n_tokens tokens); query tile i covers the same tokens as video key
 * tile i. */
typedef struct {
    int32_t B, H;
    int32_t d;          /* head dim: 64 or 128 */
    int32_t tile;       /* tokens per tile (query and key): 64 or 128 */
    int32_t r;          /* selector width: 1..128, multiple of 4 */
    veda_dtype dtype;   /* of q, k, v, weights and output */
    float softmax_scale;/* 0: 1/sqrt(d) */
    uint32_t flags;     /* VEDA_FLAG_* */
    const void* q;
    int64_t q_stride_b, q_stride_tok, q_stride_h;
    veda_segment video; /* sparse, required */
    veda_segment ref;   /* sparse visual-reference segment, optional */
    veda_segment dense; /* always-attended text / VLM / audio keys, optional */
} veda_problem;

/* Bytes of device workspace the calls below need for this problem (pooled
 * projections, tile scores and the status word).  The workspace must be
 * 256-byte aligned and prepared once with veda_workspace_init(). */
VEDA_API veda_status veda_workspace_size(const veda_problem* p, size_t* bytes);

/* Zero the workspace's status word (enqueued on `stream`).  Call once after
 * allocating a workspace; veda_check_status() re-arms it after each read. */
VEDA_API veda_status veda_workspace_init(void* ws, size_t ws_bytes, veda_stream_t stream);

/* Steps 1-3: pool + project Q and K, score every key tile, keep the top
 * `budget` per (b, h, query tile) for the video segment and, when present,
 * independently for the reference segment.  Steps 2-3 run as
 * veda_score_topk_tiles describes.
 *   w_q, w_k   [H, d, r] device, problem dtype
 *   idx_video  [B, H, n_q_tiles, video.budget] int32 out (ascending rows)
 *   idx_ref    [B, H, n_q_tiles, ref.budget]   int32 out; NULL iff no reference */
VEDA_API veda_status veda_select_tiles(const veda_problem* p, const void* w_q, const void* w_k,
                              int32_t* idx_video, int32_t* idx_ref,
                              void* ws, size_t ws_bytes, veda_stream_t stream);

/* Step 4: attention over the caller's kept tiles plus every dense token.
 *   idx_video / idx_ref: as produced by veda_select_tiles (any order is
 *   accepted; an index outside its segment is skipped and flagged as
 *   VEDA_ERR_BAD_INDEX in the status word).
 *   out [B, video.n_tokens, H, d] problem dtype; lse [B, H, video.n_tokens]
 *   fp32 or NULL. */
VEDA_API veda_status veda_block_sparse_attn(const veda_problem* p, const int32_t* idx_video,
                                   const int32_t* idx_ref, void* out, float* lse,
                                   void* ws, size_t ws_bytes, veda_stream_t stream);

/* Dense-query rows: queries that are not video tokens (text, VLM, audio or
 * reference tokens of a joint-attention layer) attend densely to every token
 * of every segment of the problem -- all video tiles, all reference tiles
 * and every dense token -- with one softmax (veyrul.com, "Veda R2VA for
 * MiniMax-H3", second paragraph: text, VLM conditioning and audio attention
 * stay dense; only the video and reference key tiles are selected).  The
 * problem's budgets are not used.
 *   q_rows   [B, n_rows, H, d] device, problem dtype, d contiguous; element
 *            strides (q_stride_*) are multiples of 16 bytes, q_rows 16-byte
 *            aligned; n_rows in [1, 2^30]
 *   out      [B, n_rows, H, d] problem dtype (16-byte aligned); lse
 *            [B, H, n_rows] fp32 or NULL
 *   ws       a workspace of this problem: its status word takes device-side
 *            errors, and with few (b, h, query tile) units the key lists are
 *            split over several CTAs and the ranges' partial results are kept
 *            in the workspace's scratch (overwriting what a selection call
 *            left there) before one merge; a workspace too small for them
 *            just runs unsplit.  Do not share it with a call in flight.
 * Errors: VEDA_ERR_INVALID_ARG for a bad pointer, stride or row count, as
 * for the other calls; device-side errors go to the status word. */
VEDA_API veda_status veda_dense_query_attn(const veda_problem* p, const void* q_rows, int64_t n_rows,
                                  int64_t q_stride_b, int64_t q_stride_tok, int64_t q_stride_h,
                                  void* out, float* lse, void* ws, size_t ws_bytes, veda_stream_t stream);

/* Steps 1-4 on HOST buffers, with the host<->device copies pipelined.
 * The heads are processed in groups of heads_per_group: while one group's
 * selection and attention run, the next group's Q/K/V and weights are
 * copied in and the previous group's output, LSE and kept tiles are copied
 * out, on three streams forked from and joined back to `stream` (each head
 * is independent of the others, so a group is a complete problem of its
 * own).  Results equal veda_attn's.  The three streams and their events are
 * made once per device (and again after a device reset) and reused by every
 * call; concurrent calls on one device enqueue in turn on them.
 *   p              the problem with HOST pointers; Q and every segment packed
 *                  [B, n, H, d] (stride_h = d, stride_tok = H d, stride_b =
 *                  n H d); page-locked host memory lets the copies overlap
 *   w_q, w_k       HOST [H, d, r]
 *   idx_video/ref  HOST [B, H, n_q_tiles, budget] int32 out, or idx_video
 *                  NULL to skip them (idx_ref NULL iff no reference)
 *   out, lse       HOST [B, video.n_tokens, H, d] / [B, H, video.n_tokens]
 *                  fp32 (lse may be NULL)
 *   dev_buf        caller-owned DEVICE buffer of veda_attn_host_buffer_size
 *                  bytes, 256-byte aligned; its first 256 bytes are a status
 *                  block: initialise it with veda_workspace_init and read
 *                  device-side errors with veda_check_status(dev_buf).
 * Returns after enqueueing.  VEDA_ERR_UNSUPPORTED for host tensors that are
 * not packed; VEDA_ERR_WORKSPACE for a short or misaligned dev_buf. */
VEDA_API veda_status veda_attn_host_buffer_size(const veda_problem* p, int32_t heads_per_group, size_t* bytes);
VEDA_API veda_status veda_attn_host(const veda_problem* p, const void* w_q, const void* w_k, int32_t* idx_video,
                           int32_t* idx_ref, void* out, float* lse, int32_t heads_per_group, void* dev_buf,
                           size_t dev_bytes, veda_stream_t stream);

/* Steps 1-4 in one call (selection, then attention on the selected tiles),
 * stream-ordered, no host synchronisation.  idx_video / idx_ref receive the
 * kept tiles as in veda_select_tiles. */
VEDA_API veda_status veda_attn(const veda_problem* p, const void* w_q, const void* w_k,
                      int32_t* idx_video, int32_t* idx_ref, void* out, float* lse,
                      void* ws, size_t ws_bytes, veda_stream_t stream);

/* The three stages of veda_select_tiles, exposed for timing and testing.
 * They communicate through the workspace; call them in this order. */
/* Step 1 for Q, video K and (if present) reference K. */
VEDA_API veda_status veda_pool_project(const veda_problem* p, const void* w_q, const void* w_k,
                              void* ws, size_t ws_bytes, veda_stream_t stream);
/* Step 2: fp32 tile scores of every sparse segment into the workspace. */
VEDA_API veda_status veda_score_tiles(const veda_problem* p, void* ws, size_t ws_bytes,
                             veda_stream_t stream);
/* Step 3: top-k of the workspace scores into idx_video / idx_ref. */
VEDA_API veda_status veda_topk_tiles(const veda_problem* p, int32_t* idx_video, int32_t* idx_ref,
                            void* ws, size_t ws_bytes, veda_stream_t stream);
/* Steps 2-3 (what veda_select_tiles runs after veda_pool_project).  The
 * tile scores are computed on the tensor cores from the projections in the
 * workspace, as three bf16 parts per value whose six leading products give
 * fp32 accuracy.  By default they are written to the workspace and the
 * step-3 kernel selects from them.  With VEDA_FLAG_ONCHIP_SELECTION the same
 * kernel selects each row's top-k on chip while it recomputes the row's
 * scores pass by pass, writing no score matrix; rows whose on-chip
 * selection cannot finish (a score band wider than its buffer, or a NaN) get
 * their scores written to the workspace and go through the step-3 kernel.
 * With r > 64 or VEDA_FLAG_UNFUSED_SELECTION the scores come from the fp32
 * SIMT kernel. */
VEDA_API veda_status veda_score_topk_tiles(const veda_problem* p, int32_t* idx_video, int32_t* idx_ref,
                                           void* ws, size_t ws_bytes, veda_stream_t stream);

/* Tile selection without a workspace, for callers that cannot allocate
 * device memory when they call: a serving engine that plans all memory up
 * front and forbids allocation once requests flow, a plugin whose enqueue
 * hook may not allocate, or a latency-critical loop that cannot afford the
 * device synchronisation cudaMalloc implies.  The pages have no counterpart
 * of this call; it exists only for such callers.
 *   Computes exactly what veda_select_tiles() computes with
 *   VEDA_FLAG_UNFUSED_SELECTION (the same pool + project, fp32 score and
 *   top-k kernels), with
 *   its scratch in a 64 MiB array that this library reserves statically on
 *   every GPU that uses it and keeps until the process exits.  The problem is
 *   processed one batch entry and one group of heads at a time; a problem
 *   where the scores of a single head do not fit (about 4000 key tiles at
 *   r = 64) returns VEDA_ERR_WORKSPACE without launching anything.
 *   The call allocates nothing.  Its first call on each device looks up the
 *   array's device address (cudaGetSymbolAddress) and caches it under the
 *   current context's id, so make that first call before capturing the
 *   stream into a CUDA graph; after cudaDeviceReset (or any new context on
 *   the device) the next call looks the address up again, and a failed
 *   lookup is retried on the next call.  All calls share the one array,
 *   which keeps the last call's contents: calls that can overlap on the GPU
 *   (different streams without ordering) race with each other; calls on one
 *   stream are ordered and safe.  Errors are reported through the return
 *   code only (these selection kernels record no device-side errors, and
 *   there is no workspace status word to read).
 *   Arguments as for veda_select_tiles(), without ws / ws_bytes. */
VEDA_API veda_status veda_select_tiles_noalloc(const veda_problem* p, const void* w_q, const void* w_k,
                                               int32_t* idx_video, int32_t* idx_ref, veda_stream_t stream);

/* Read-only views of the workspace (device pointers), for tests:
 *   which = 0: qhat [B,H,n_q_tiles,r] fp32     1: khat video [B,H,n_q_tiles,r]
 *           2: khat ref [B,H,n_ref_tiles,r]    3: scores video [B,H,n_q_tiles,ld]
 *           4: scores ref [B,H,n_q_tiles,ld]
 *           5 / 6: int32 rows the fused selection (video / reference) left
 *              to the step-3 kernel: [0] = count, then the row ids
 * *ld receives the row stride (elements) of the score matrices (>= n tiles;
 * 1 for which = 5, 6). */
VEDA_API veda_status veda_workspace_view(const veda_problem* p, void* ws, size_t ws_bytes, int which,
                                const void** ptr, int64_t* ld);

/* Synchronise `stream`, return the sticky device status recorded in `ws`
 * since the last check (VEDA_OK if none), and reset it. */
VEDA_API veda_status veda_check_status(void* ws, veda_stream_t stream);

/* Static, human-readable name of a status code. */
VEDA_API const char* veda_status_string(veda_status s);

/* ---- selector artifacts --------------------------------------------------
 * The trained selector projections ship as a safetensors file: the published
 * competition artifact holds exactly 100 float16 tensors, the query and key
 * projections of 50 layers, each of shape (56, 384, 128), in at most
 * 560,000,000 bytes, with metadata that names the miner's hotkey
 * (tao.media, "Affine launches MiniMax-H3 video studio...", section "How the
 * SN120 Competition Works").  The R2VA predictor is stored in FP8 and
 * dequantised to BF16 at load (veyrul.com, "Veda R2VA for MiniMax-H3",
 * second paragraph); no scale format is published, so FP8 (E4M3) tensors are
 * read with a caller-given scale.  A tensor of shape (H, d, r) is the
 * [H, d, r] weight layout that veda_select_tiles takes.
 * All of this is host code: the caller copies converted tensors to the
 * device.  The reader owns its memory until veda_selector_close. */
typedef struct veda_selector veda_selector;

/* Read and check a safetensors file: header length, JSON header, dtypes
 * (F16, BF16, F32, F8_E4M3), shapes, and byte ranges that tile the data
 * section exactly.  VEDA_ERR_IO: cannot be read; VEDA_ERR_FORMAT: malformed. */
VEDA_API veda_status veda_selector_open(const char* path, veda_selector** out);
VEDA_API void veda_selector_close(veda_selector* s);

/* Check the published layout: exactly n_tensors tensors, each F16 or
 * F8_E4M3 with shape shape[0..ndim), the file at most max_file_bytes
 * (<= 0: no limit), and (if required_meta_key is not NULL) a non-empty
 * metadata value under that key.  VEDA_ERR_FORMAT when anything differs. */
VEDA_API veda_status veda_selector_check(const veda_selector* s, int32_t n_tensors, const int64_t* shape,
                                int32_t ndim, int64_t max_file_bytes, const char* required_meta_key);

/* Tensors are indexed 0..count-1 in data-section order. */
VEDA_API int32_t veda_selector_count(const veda_selector* s);
VEDA_API veda_status veda_selector_find(const veda_selector* s, const char* name, int32_t* index);
/* name / dtype point into the reader (valid until close); shape receives ndim
 * (<= 8) extents.  Any output pointer may be NULL. */
VEDA_API veda_status veda_selector_info(const veda_selector* s, int32_t index, const char** name,
                               const char** dtype, int32_t* ndim, int64_t* shape);
/* The metadata value under `key`, or NULL. */
VEDA_API const char* veda_selector_metadata(const veda_selector* s, const char* key);
/* Tensor `index`, times `scale` (> 0; 1 for F16 / BF16 / F32 data), into host
 * `dst` as fp32 or bf16 (round to nearest, ties to even), row-major in the
 * stored shape.  dst_bytes must hold every element. */
VEDA_API veda_status veda_selector_read(const veda_selector* s, int32_t index, veda_dtype out_dtype, float scale,
                               void* dst, size_t dst_bytes);

#ifdef __cplusplus
}
#endif
#endif /* VEDA_H */
