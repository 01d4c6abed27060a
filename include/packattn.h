/*
 * packattn.h -- C ABI of the B200 (sm_100a) packed variable-length attention library.
 *
 * The one operation: packed variable-length bidirectional multi-head attention,
 * forward.  Images of different native resolutions are patchified (patch 16) and
 * concatenated into one token stream; cu_seqlens = [0, L0, L0+L1, ...] splits
 * the stream into segments, and each token attends only to the tokens of its
 * own segment, with no padding (Mage-Flow page, section "Packing + Flash
 * Attention varlen": q, k, v of shape [total_tokens, num_heads, head_dim], one
 * cu_seqlens for queries and keys, max_seqlen, causal = False).  Per segment i,
 * head h and query row r of that segment (SparseAttn page, section 3.1):
 *
 *     s_j      = scale * q[r,h,:] . k[j,h,:]          for j in [cu_i, cu_{i+1})
 *     out[r,h] = sum_j softmax(s)_j * v[j,h,:]
 *     lse[r,h] = log(sum_j exp(s_j))                  (natural log)
 *
 * All functions are thread-safe.  No function allocates or synchronises on the
 * hot path once the workspace of the (device, stream) pair is large enough.
 */
#ifndef PACKATTN_H_
#define PACKATTN_H_

#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes.  Negative values are errors. */
enum pa_status {
  PA_OK = 0,
  PA_ERR_NULL = -1,         /* a required pointer is NULL */
  PA_ERR_ALIGN = -2,        /* q, k, v or out not 16-byte aligned; lse or cu_seqlens not 4-byte aligned */
  PA_ERR_HEAD_DIM = -3,     /* head_dim is not 64 or 128 */
  PA_ERR_SHAPE = -4,        /* heads < 1, batch < 0, total_tokens < 0, batch == 0 with tokens, sizes too large */
  PA_ERR_CU_SEQLENS = -5,   /* device: cu_seqlens[0] != 0, decreasing, or cu_seqlens[batch] != total_tokens */
  PA_ERR_MAX_SEQLEN = -6,   /* max_seqlen < 1 with tokens (host), or a segment longer than max_seqlen (device) */
  PA_ERR_TIMEOUT = -7,      /* device: a pipeline wait exceeded its limit; the kernel stopped early */
  PA_ERR_CUDA = -8,         /* a CUDA runtime call or a kernel launch failed */
  PA_ERR_SCALE = -9,        /* scale is not finite */
  PA_ERR_NOT_DEVICE = -10,  /* q, k, v, out, lse or cu_seqlens is not device memory of one GPU */
  PA_ERR_NOALLOC_LIMIT = -11 /* pa_varlen_attn_fwd_noalloc: batch above its 1024-segment maximum */
};

/*
 * pa_varlen_attn_fwd -- enqueue the packed varlen attention forward on `stream`.
 *
 *   q, k, v      device, bf16, [total_tokens, heads, head_dim], contiguous (row
 *                stride heads*head_dim elements), 16-byte aligned.  Read only.
 *   cu_seqlens   device, int32, [batch + 1], non-decreasing, cu_seqlens[0] = 0,
 *                cu_seqlens[batch] = total_tokens.  Zero-length segments are
 *                allowed and produce nothing.
 *   batch        number of segments (images), >= 0.
 *   total_tokens T, >= 0.
 *   heads        H >= 1.      head_dim  d in {64, 128}.
 *   max_seqlen   an upper bound of every segment length (>= 1 when T > 0).
 *   scale        finite multiplier of q.k (1/sqrt(d) for standard attention).
 *   out          device, bf16, [total_tokens, heads, head_dim], 16-byte aligned,
 *                written (rounded once, to nearest even).
 *   lse          device, fp32, [total_tokens, heads], natural-log log-sum-exp of
 *                the scaled scores of each row.
 *   stream       a cudaStream_t (NULL = the legacy default stream).
 *
 * Ownership: the caller owns every buffer and the stream; all buffers must stay
 * alive until the enqueued work completes.  The library owns only a small
 * workspace per (device, stream) (schedule, per-segment tensor maps, status
 * word), grown stream-ordered and freed by pa_release_workspace.
 *
 * Errors: argument problems the host can see return a negative pa_status at
 * once and enqueue nothing.  batch == 0 or total_tokens == 0 returns PA_OK and
 * enqueues nothing.  Problems only the device can see (cu_seqlens, a segment
 * longer than max_seqlen, a wait timeout) are recorded in the status word of the
 * (device, stream) pair; out and lse are then undefined.  Read them with
 * pa_get_error.  Launch failures return PA_ERR_CUDA.
 *
 * Results are bitwise deterministic from run to run.
 */
PA_API int pa_varlen_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                              int32_t batch, int32_t total_tokens, int32_t heads, int32_t head_dim,
                              int32_t max_seqlen, float scale, void* out, float* lse, void* stream);

/*
 * pa_varlen_attn_bwd -- enqueue the gradients of pa_varlen_attn_fwd on `stream`:
 * dq, dk, dv from q, k, v, the forward's out and lse, and dout = dL/dout.
 * (Chain rule through the row softmax of the forward definition, SparseAttn page,
 * section 3.1; P recomputed from the saved log-sum-exp as in the blockwise
 * algorithm of the GigaPath-Flash page, sections 3.2 / 4.2.)  Per segment, head,
 * query row r and key j of the segment:
 *     P_rj  = exp(scale * q_r . k_j - lse_r),     D_r = dout_r . out_r,
 *     dS_rj = P_rj (dout_r . v_j - D_r),
 *     dq_r  = scale * sum_j dS_rj k_j,   dk_j = scale * sum_r dS_rj q_r,
 *     dv_j  = sum_r P_rj dout_r.
 *
 *   q, k, v, out, dout   device, bf16, [total_tokens, heads, head_dim], contiguous,
 *                        16-byte aligned; out and lse as pa_varlen_attn_fwd wrote
 *                        them for the same q, k, v, cu_seqlens and scale.
 *   lse                  device, fp32, [total_tokens, heads], 4-byte aligned.
 *   cu_seqlens, batch, total_tokens, heads, head_dim, max_seqlen, scale:
 *                        as for pa_varlen_attn_fwd.
 *   dq, dk, dv           device, bf16, [total_tokens, heads, head_dim], 16-byte
 *                        aligned, written (each rounded once to nearest even).
 *
 * Ownership, workspace and errors: as for pa_varlen_attn_fwd.  The workspace of
 * the (device, stream) pair also holds an fp32 dq accumulator of
 * 4 * total_tokens * heads * head_dim bytes.  dk and dv are bitwise
 * deterministic; dq sums fp32 partials of different key tiles in whatever order
 * they arrive, so its last bits may differ from run to run.
 */
PA_API int pa_varlen_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                              const void* dout, const int32_t* cu_seqlens, int32_t batch, int32_t total_tokens,
                              int32_t heads, int32_t head_dim, int32_t max_seqlen, float scale, void* dq, void* dk,
                              void* dv, void* stream);

/*
 * pa_qkv_rope_fwd -- the fused QKV projection in front of the attention (Mage-Flow
 * page, "DiT Block" data flow: x -> [Q,K,V] projection -> RoPE -> attention, and
 * "fusion strategy one": one GEMM with the stacked weight, its output split into
 * q, k, v), enqueued on `stream`:
 *     qkv = x W_qkv^T;  q, k, v = the [T, H, d] slices of qkv (rows of W_qkv: the
 *     H*d rows of q, then of k, then of v, head-major);
 *     q, k rotated by the rotary embedding (rotate-half pairs (c, c + d/2),
 *     theta_i = rope_theta^(-2i/d)) at each token's position inside its own image.
 *
 *   x            device, bf16, [total_tokens, hidden], row-major, 16-byte aligned.
 *   w_qkv        device, bf16, [3 * heads * head_dim, hidden], row-major (the
 *                layout of a linear layer's weight), 16-byte aligned.
 *   cu_seqlens   device, int32, [batch + 1], as for pa_varlen_attn_fwd (only read
 *                when rope_theta > 0; positions restart at every segment).
 *   hidden       C, a multiple of 8.   heads H >= 1.   head_dim d in {64, 128}.
 *   max_seqlen   an upper bound of every segment length (>= 1 when rotating).
 *   rope_theta   base of the rotary frequencies; <= 0 disables the rotation.
 *   q, k, v      device, bf16, [total_tokens, heads, head_dim], 16-byte aligned,
 *                written (rounded once to nearest even after the rotation).
 *
 * Workspace: token positions in the (device, stream) workspace and a table of
 * (cos, sin) per (position, frequency), computed in fp64 and kept per (device,
 * stream) until max_seqlen grows or head_dim / rope_theta change.  Errors: as for
 * pa_varlen_attn_fwd; invalid cu_seqlens or a segment longer than max_seqlen are
 * recorded in the status word (pa_get_error).
 */
PA_API int pa_qkv_rope_fwd(const void* x, const void* w_qkv, const int32_t* cu_seqlens, int32_t batch,
                           int32_t total_tokens, int32_t hidden, int32_t heads, int32_t head_dim,
                           int32_t max_seqlen, float rope_theta, void* q, void* k, void* v, void* stream);

/*
 * pa_linear_fwd -- y = x W^T on `stream` (the attention's output projection,
 * Mage-Flow page, "DiT Block" data flow: attention -> output projection).
 *   x [rows, in_features], W [out_features, in_features], y [rows, out_features]:
 *   device, bf16, row-major, 16-byte aligned; in_features a multiple of 8,
 *   out_features a multiple of 32.  fp32 accumulation, y rounded once.
 */
PA_API int pa_linear_fwd(const void* x, const void* w, int32_t rows, int32_t in_features, int32_t out_features,
                         void* y, void* stream);

/*
 * FP8 (E4M3) variant of the forward, head_dim 128 (FPS Attention slides of the
 * Mage-Flow talk: attention on FP8 operands with Q and K quantised per tensor, V per
 * channel and the softmax weights P per tensor).  Two calls: the quantiser, then the
 * attention on its output.
 *
 * pa_fp8_vt_keys -- keys per row of the transposed V buffer for a pack of `batch`
 * segments and `total_tokens` tokens: 16*ceil(total_tokens/16) + 16*batch (-1 if
 * an argument is negative).  Segment s of the pack occupies keys
 * [16*ceil(cu[s]/16) + 16*s, + L_s) of every row, so that each starts on a
 * 16-byte boundary (the TMA copy rule); the keys between segments are never read.
 */
PA_API int64_t pa_fp8_vt_keys(int32_t batch, int32_t total_tokens);

/*
 * pa_fp8_quantize_qkv -- quantise bf16 q, k, v to E4M3 on `stream`.
 *   q, k, v      device, bf16, [total_tokens, heads, 128], 16-byte aligned (read).
 *   cu_seqlens   device, int32, [batch + 1], as for pa_varlen_attn_fwd (the layout
 *                of v8t depends on it; it is not validated here).
 *   q8, k8       device, [total_tokens, heads, 128] bytes, 16-byte aligned (written).
 *   v8t          device, [heads*128][pa_fp8_vt_keys(batch, total_tokens)] bytes,
 *                16-byte aligned: v8 transposed per (head, channel) row, segment
 *                by segment as pa_fp8_vt_keys describes (only the segments' keys
 *                are written).
 *   scales       device, fp32, [4 + heads*128], 16-byte aligned (written):
 *                [0] s_q, [1] s_k, [2..3] zero, [4 + h*128 + c] s_v of (h, c).
 * With a = the absolute maximum of a group (the whole q; the whole k; the column
 * (h, c) of v over all tokens): mult = 448 / a, s = a / 448 (fp32, correctly
 * rounded; both 1 when a = 0) and code = E4M3(fp32(x * mult)), rounded to nearest
 * even and clamped to +-448.  x = s * value(code) is the dequantised input.
 * Workspace: the absolute maxima, in the (device, stream) workspace.  Errors:
 * PA_ERR_HEAD_DIM unless head_dim = 128; otherwise as for pa_varlen_attn_fwd.
 * Inputs with NaN give undefined codes.
 */
PA_API int pa_fp8_quantize_qkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                               int32_t batch, int32_t total_tokens, int32_t heads, int32_t head_dim, void* q8,
                               void* k8, void* v8t, float* scales, void* stream);

/*
 * pa_fp8_quantize_qkv_delayed -- the same quantisation in one pass over q, k, v, with
 * the scales taken from given maxima instead of this call's (delayed scaling: the
 * maxima of the previous step of a training or serving loop; the pages fix the
 * granularity -- q, k per tensor, v per channel -- not where the maxima come from).
 *   amax_in      device, fp32, [4 + heads*128], 4-byte aligned (read): a_q at [0],
 *                a_k at [1], a of v's column (h, c) at [4 + h*128 + c]; finite and
 *                non-negative (as amax_out holds them).  mult, s and code follow from
 *                these a exactly as in pa_fp8_quantize_qkv; an input above its a is
 *                clamped to the code of +-448.
 *   amax_out     device, fp32, [4 + heads*128], 4-byte aligned (written): the absolute
 *                maxima of this call's q, k and v columns, in amax_in's layout (exact:
 *                the largest |bf16| of each group, widened), for the next call.  Must
 *                not overlap amax_in (PA_ERR_SHAPE).
 * Other arguments as for pa_fp8_quantize_qkv.  Workspace: none.  With batch = 0 or
 * total_tokens = 0, amax_out is zeroed and nothing else is written.  Errors:
 * PA_ERR_NULL for a null amax_in or amax_out; otherwise as pa_fp8_quantize_qkv.
 */
PA_API int pa_fp8_quantize_qkv_delayed(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                       int32_t batch, int32_t total_tokens, int32_t heads, int32_t head_dim,
                                       const float* amax_in, float* amax_out, void* q8, void* k8, void* v8t,
                                       float* scales, void* stream);

/*
 * pa_varlen_attn_fwd_fp8 -- the packed varlen attention forward on the quantiser's
 * output (q8, k8, v8t, scales as pa_fp8_quantize_qkv writes them; the same pack,
 * heads and cu_seqlens).  Computes, with x = scale * s_q * s_k * (q8 . k8) per key,
 *     out[r,h,c] = s_v[h,c] * sum_j P8_j v8[j,h,c] / sum_j P8_j,
 *     lse[r,h]   = log sum_j exp(x_j),
 * where P8_j is E4M3 of exp(x_j - m) times a power of two (m: a running maximum of
 * the row), i.e. softmax weights rounded to E4M3 relative to the row's largest
 * ones.  out bf16 [total_tokens, heads, 128], lse fp32 [total_tokens, heads] as for
 * pa_varlen_attn_fwd; other arguments, ownership, workspace and errors likewise
 * (PA_ERR_HEAD_DIM unless head_dim = 128; q8, k8, v8t, scales 16-byte aligned).
 */
PA_API int pa_varlen_attn_fwd_fp8(const void* q8, const void* k8, const void* v8t, const float* scales,
                                  const int32_t* cu_seqlens, int32_t batch, int32_t total_tokens, int32_t heads,
                                  int32_t head_dim, int32_t max_seqlen, float scale, void* out, float* lse,
                                  void* stream);

/*
 * pa_get_error -- synchronise `stream`, return the first device-side error
 * recorded for the calling device and `stream` since the last call (PA_OK if
 * none) and clear it.  Returns PA_ERR_CUDA if the synchronisation fails.
 */
PA_API int pa_get_error(void* stream);

/* A short English description of a pa_status code (static storage). */
PA_API const char* pa_status_string(int code);

/* Library version as major*10000 + minor*100 + patch. */
PA_API int pa_version(void);

/* Frees every workspace (synchronises the device of each).  Later calls re-create them. */
PA_API void pa_release_workspace(void);

/*
 * pa_set_short_packing -- short-segment packing in pa_varlen_attn_fwd and
 * pa_varlen_attn_fwd_noalloc (on by default).  A native-resolution pack of small
 * images (Mage-Flow page, section "Packing + Flash Attention varlen", and its
 * padding / bucketing / packing table) has many segments of at most 128 tokens.
 * With packing on, the scheduler cuts runs of consecutive such segments, in
 * packing order, into shared 128-row tiles that hold whole segments (two tiles
 * per work item); inside a tile every query row sees only the keys of its own
 * segment, so the result is the same block-diagonal attention (the wasted block
 * work of the Fusion page, section 3.5, shrinks).  With packing off every
 * non-empty segment has tiles of its own.  Both settings compute the same
 * definition; they differ in the order of nothing but which rows share a tile.
 * Affects calls enqueued afterwards; thread-safe.
 */
PA_API void pa_set_short_packing(int on);

/*
 * pa_schedule_stats -- the tile ledger of the last call of pa_varlen_attn_fwd,
 * pa_varlen_attn_fwd_fp8 or pa_varlen_attn_bwd on the calling thread's current
 * device and `stream` (synchronises `stream`).
 * Writes 6 values to `out` (host memory):
 *   out[0] work items, out[1] units (segments alone + groups of short segments;
 *          the FP8 forward and the backward take every non-empty segment alone),
 *   out[2] 128 x 128 score tiles computed over all heads,
 *   out[3] useful (query, key) pairs over all heads = heads * sum_i L_i^2,
 *   out[4] groups of short segments, out[5] segments inside groups.
 * Useful pairs / (score tiles * 16384) is the tile utilisation of the call (the
 * block-level waste account of the Fusion page, section 3.5).  Returns PA_OK,
 * PA_ERR_NULL (out is NULL), PA_ERR_NOT_DEVICE (no forward call on this
 * device and stream yet) or PA_ERR_CUDA.  Not for pa_varlen_attn_fwd_noalloc.
 */
PA_API int pa_schedule_stats(void* stream, int64_t* out);

/*
 * pa_set_wait_limit_ms -- limit of every pipeline wait inside the kernels, in
 * milliseconds (default 4000).  After the limit a kernel records
 * PA_ERR_TIMEOUT, stops issuing work, drains what it has in flight and returns.
 * Values < 1 are clamped to 1.  Affects launches enqueued afterwards.
 */
PA_API void pa_set_wait_limit_ms(int ms);

/*
 * pa_selftest_wait_timeout -- enqueue a one-warp kernel on `stream` that waits,
 * through the same bounded-wait routine as the attention kernel, on a barrier
 * that nothing completes, with a limit of `limit_us` microseconds.  The kernel
 * returns normally and records PA_ERR_TIMEOUT in the status word of the
 * (device, stream) pair, which pa_get_error then reports.  Used to test the
 * failure path without faulting or hanging the GPU.  Returns PA_OK or PA_ERR_CUDA.
 */
PA_API int pa_selftest_wait_timeout(uint32_t limit_us, void* stream);

/*
 * Kernel timing for measurement.  While enabled, pa_varlen_attn_fwd records a
 * pair of CUDA events on its stream around the attention kernel (not the
 * schedule kernel) and launches it without overlapping the schedule kernel
 * (no programmatic dependent launch), so the events bracket it alone;
 * pa_varlen_attn_bwd records a pair around its main kernel (not the prep,
 * schedule and dq conversion kernels).  pa_profile_read synchronises on the last recorded event,
 * writes the summed attention-kernel time in milliseconds and the number of
 * launches timed, and clears the record.  Returns PA_OK or PA_ERR_CUDA.
 */
PA_API void pa_profile_enable(int on);
PA_API int pa_profile_read(double* total_ms, int32_t* launches);

/*
 * pa_varlen_attn_fwd_noalloc -- the same forward as pa_varlen_attn_fwd (same
 * kernels, same results bit for bit), for callers that must not allocate
 * device memory.  None of the pages defines this entry point: it is a service
 * of this library and has no counterpart in the method.
 *
 * Who needs it: code whose device memory belongs to someone else -- a framework
 * whose caching allocator or pre-reserved arena owns nearly all of the GPU (a
 * cudaMalloc there fails or fragments memory the owner cannot see), a plug-in
 * whose enqueue is called in a context that forbids allocation, or a serving
 * loop that must not allocate after warm-up.  Such a caller already owns q, k,
 * v, cu_seqlens, out and lse; the one thing pa_varlen_attn_fwd adds is its own
 * workspace (schedule, per-segment tensor maps, status word), grown with
 * cudaMallocAsync.  This entry point uses instead a fixed 400 KiB array that is
 * part of the library's device image: every GPU that loads the library holds it
 * until the process exits.  The call allocates nothing (no cudaMalloc,
 * cudaMallocAsync, cudaFree or allocating library routine).
 *
 *   Arguments q ... lse and stream: as for pa_varlen_attn_fwd.
 *   batch        at most 1024 segments; a larger batch returns
 *                PA_ERR_NOALLOC_LIMIT and enqueues nothing.
 *   status       optional device int32 (4-byte aligned, same GPU).  The call
 *                sets it to 0 on `stream`, and the kernels record there a
 *                device-side error (PA_ERR_CU_SEQLENS, PA_ERR_MAX_SEQLEN,
 *                PA_ERR_TIMEOUT) of this call; read it after the stream has
 *                finished.  With NULL a status word inside the fixed array is
 *                used (cleared by each call) and such errors are not reported.
 *                pa_get_error does not see this entry point's errors.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and sets the kernels'
 * shared-memory attributes; that first call may also make the CUDA runtime load
 * the library's kernels onto the device.  Make it before any stream capture.
 *
 * Sharing: all calls on one GPU use the same array, which keeps the contents of
 * the last call; each call clears the status word and rewrites everything else
 * before reading it.  Calls whose work overlaps on that GPU (different streams,
 * or different host threads without ordering between their streams) race on
 * the array and give undefined results: order them on one stream or with
 * events.  Host-side use is thread-safe.
 */
PA_API int pa_varlen_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                      int32_t batch, int32_t total_tokens, int32_t heads, int32_t head_dim,
                                      int32_t max_seqlen, float scale, void* out, float* lse, int32_t* status,
                                      void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PACKATTN_H_ */
