/*
 * mla.h - C ABI of the VideoMLA latent-KV attention library for NVIDIA B200 (sm_100a).
 *
 * The library implements the attention hot path of VideoMLA ("VideoMLA: Low-Rank Latent KV
 * Cache for Minute-Scale Autoregressive Video Diffusion"): multi-head latent attention over a
 * rolling, frame-granular sliding-window cache that stores, per token, only a content latent
 * c_KV (d_c scalars) and one head-shared, unrotated positional key k_R (d_rope scalars).
 * Sources, cited by page and section:
 *   [M]  hyper.ai summary of VideoMLA (English edition), "Method"; identical to the Chinese
 *        edition's "方法" section.
 *   [A]  chatpaper abstract of the paper, English abstract.
 *   [F1] ai-papers.net article "VideoMLAとは？", the paragraph after Figure 1 (Wan2.1-1.3B base,
 *        192-wide content latent, 3,072 -> 224 cached scalars per token).
 *   [I]  hyper.ai summary, "Introduction" (rolling key-value cache; chunk-wise students).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer named as device memory must be a device (or managed) pointer on the current
 *   device, 16-byte aligned, to a dense row-major array of the stated shape.  "T" is the
 *   configuration's element type: bfloat16 (MLA_BF16) or float32 (MLA_FP32).
 * - The caller owns every buffer.  The library never allocates device memory, never
 *   synchronises the device or a stream, and keeps no pointer after a call returns.  The one
 *   exception is mla_attention_fwd_static_scratch: it uses a fixed array built into the library
 *   (reserved on every device that loads it) and keeps that array's device address (below).
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All work is
 *   enqueued on it, asynchronously.  The forward path's kernels are launched with programmatic
 *   stream serialisation: each may begin its set-up while the previous kernel on the stream
 *   drains and waits for that kernel's completion before it touches memory, so stream order is
 *   kept.  Setting the environment variable MLA_NO_PDL (read once per process) launches them
 *   plainly.
 * - Arguments are checked on the host before anything is launched.  A rejected call returns a
 *   non-zero mla_status, launches nothing and leaves every buffer untouched;
 *   mla_last_error() then describes the problem.  A launch that fails returns MLA_ERR_CUDA.
 * - Errors that only the device can see (a bounded wait inside a kernel that ran out) are
 *   written to the optional `dev_status` word (see mla_attention_fwd); kernels never trap.
 * - Entry points are thread-safe; mla_last_error() is per host thread.  Again the exception is
 *   mla_attention_fwd_static_scratch: its calls share one array per device, so calls whose work
 *   overlaps on the GPU race (below).
 *
 * Token order.  A chunk holds chunk_frames latent frames of frame_h x frame_w tokens; tokens
 * are ordered by frame, then row h, then column w.  Positions used by 3D-RoPE are
 * (t, h, w) = (absolute latent-frame index since the rollout began, row, column).  Frame
 * indices are int32: every entry point that takes first_frame rejects, with
 * MLA_ERR_INVALID_ARG, a first_frame below 0 or one with first_frame + chunk_frames above
 * INT32_MAX (mla_rope3d without a frame table: + rows_per_sample / tpf).
 */
#ifndef MLA_LATENT_KV_ATTN_H_
#define MLA_LATENT_KV_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 1

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,    /* a null pointer, a bad size or an inconsistent configuration */
  MLA_ERR_UNSUPPORTED = 2,    /* a valid request the library does not implement */
  MLA_ERR_ALIGNMENT = 3,      /* a pointer that is not 16-byte aligned */
  MLA_ERR_CUDA = 4,           /* a CUDA runtime or driver call failed */
  MLA_ERR_DEVICE_TIMEOUT = 5, /* value a kernel writes to dev_status when a bounded wait ran out */
  MLA_ERR_WORKSPACE = 6,      /* workspace missing or smaller than required */
  MLA_ERR_DEVICE_CHECK = 7    /* value a kernel of the MLA_DEBUG build writes to dev_status when
                                 an input's contents break the call's contract (a ring slot whose
                                 frame is empty or outside the chunk's window); the release build
                                 does not make these checks */
} mla_status;

typedef enum mla_dtype { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype;

/* Which kernels serve a call.  MLA_PATH_AUTO picks the tensor-core (tcgen05/TMA) kernels when
 * the shape allows (bf16; for attention d_c in {128, 192, 256}, d_rope in {16, 32, 64} and,
 * with the W_UV epilogue, d_head = 128) and the CUDA-core kernels otherwise; attention runs one
 * CTA per head and query tile.  MLA_PATH_TC_SINGLE is the same choice (kept for callers that
 * name it).  MLA_PATH_TC_PAIR runs attention, for an even head count and d_c in {128, 192}, on
 * the CTA-pair kernel instead, in which two CTAs (two heads of one query tile) execute every MMA
 * together and share each key tile (correct, but slower than the one-CTA kernel on this part;
 * for measurements); other calls as AUTO.  MLA_PATH_SIMT forces the CUDA-core kernels (every
 * dtype and shape; slow but simple, used as a cross-check). */
typedef enum mla_kernel_path {
  MLA_PATH_AUTO = 0,
  MLA_PATH_SIMT = 1,
  MLA_PATH_TC_SINGLE = 2,
  MLA_PATH_TC_PAIR = 3
} mla_kernel_path;

/* Layer shape, frame geometry and rollout geometry ([M], [F1]).
 * D = d_c + d_rope is the cached width per token; tpf = frame_h * frame_w;
 * n_q = chunk_frames * tpf query tokens per sample; the ring holds window_frames * tpf tokens
 * per sample.  3D-RoPE: axis a in (t, h, w) owns rope_pairs_a adjacent channel pairs of the
 * d_rope channels (t band first); pair i of axis a turns by pos_a * rope_base^(-i/rope_pairs_a);
 * (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).  The pages only say "3D-RoPE"; this is the
 * reading adopted.  softmax_scale multiplies q.k before the softmax (1/sqrt(d_head + d_rope)
 * in every preset). */
typedef struct mla_config {
  int32_t d_model;        /* token width of x                                  (Wan: 1536) */
  int32_t n_heads;        /* H                                                 (Wan: 12)   */
  int32_t d_head;         /* per-head width of k_nope, v and the output        (Wan: 128)  */
  int32_t d_c;            /* content latent width                              (Wan: 192)  */
  int32_t d_rope;         /* positional key width, = 2*(sum of rope pairs)     (Wan: 32)   */
  int32_t d_cq;           /* query latent width                                (Wan: 512)  */
  int32_t rope_pairs_t;   /* rotary pairs on the temporal axis                 (Wan: 4)    */
  int32_t rope_pairs_h;   /* rotary pairs on the row axis                      (Wan: 6)    */
  int32_t rope_pairs_w;   /* rotary pairs on the column axis                   (Wan: 6)    */
  float rope_base;        /* rotary base                                       (10000)     */
  float softmax_scale;    /* score scale                                       (1/sqrt(160)) */
  int32_t frame_h;        /* latent frame height in tokens                     (Wan: 30)   */
  int32_t frame_w;        /* latent frame width in tokens                      (Wan: 52)   */
  int32_t chunk_frames;   /* C: frames generated per chunk                                 */
  int32_t window_frames;  /* W: frames the ring keeps; chunk_frames <= window_frames       */
  int32_t batch;          /* B: independent samples, each with its own ring                */
  int32_t dtype;          /* mla_dtype of every T array                                    */
  int32_t kernel_path;    /* mla_kernel_path                                               */
} mla_config;

/* Returns a static, human-readable name of a status code. */
const char* mla_status_string(int32_t status);

/* Returns a description of the last error raised on the calling host thread ("" if none). */
const char* mla_last_error(void);

/* Returns MLA_ABI_VERSION of the loaded library. */
int32_t mla_abi_version(void);

/* Checks a configuration without touching the device.  Errors: MLA_ERR_INVALID_ARG for
 * non-positive sizes, d_rope != 2*(pairs), odd d_rope, chunk_frames > window_frames or an unknown
 * dtype/path. */
mla_status mla_config_check(const mla_config* cfg);

/* --------------------------------------------------------------------------------------------
 * mla_cache_append: joint down-projection and ring-buffer append.  [M]: a joint down-projection
 * turns every token into the content latent that the cache keeps, and W_R^K turns it into the
 * one positional key all heads share, cached before any rotation; [A]: the window of cached
 * frames has a fixed size; [I]: the cache rolls forward chunk by chunk.
 *
 *   mode & MLA_PROJECT : chunk_lat[b, n, :] = [W_down^KV x[b, n] || W_R^K x[b, n]]   (T, fp32 acc.)
 *   mode & MLA_APPEND  : for each frame f = first_frame + j, j < chunk_frames:
 *                          slot = f mod window_frames,
 *                          cache[b, slot*tpf + i, :] = chunk_lat[b, j*tpf + i, :]   (exact copy)
 *                          slot_frame[b, slot] = f
 *   MLA_PROJECT_AND_APPEND does both (the ring gets the same rounded values as chunk_lat).
 *
 *   x          device T [B, n_q, d_model]      (read if mode & MLA_PROJECT)
 *   w_dkv_kr   device T [d_c + d_rope, d_model] rows 0..d_c-1 = W_down^KV, rows d_c.. = W_R^K
 *   chunk_lat  device T [B, n_q, D]            written by PROJECT, read by APPEND
 *   cache      device T [B, window_frames*tpf, D]  the ring (read/written only by APPEND)
 *   slot_frame device int32 [B, window_frames] absolute frame held by each slot; -1 = empty.
 *              The caller initialises it to -1 before the first chunk.
 *   first_frame >= 0: absolute index of the chunk's first frame.
 * Append a chunk only after its own attention (the ring slots it overwrites may still be in the
 * window of that chunk).  Errors: MLA_ERR_INVALID_ARG (null pointer needed by mode, bad mode,
 * first_frame < 0), MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
#define MLA_PROJECT 1
#define MLA_APPEND 2
#define MLA_PROJECT_AND_APPEND 3
mla_status mla_cache_append(const mla_config* cfg, const void* x, const void* w_dkv_kr,
                            void* chunk_lat, void* cache, int32_t* slot_frame,
                            int32_t first_frame, int32_t mode, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_rope3d: in-place 3D-RoPE ([M]: the unrotated positional key is rotated by 3D-RoPE at
 * attention time; the positional query is rotated; [F1]: 3-D rotary position encoding).
 *
 *   data        device T [n_samples, rows_per_sample, row_width]; for every row, n_vec vectors
 *               of d_rope channels start at columns col_offset + v*vec_stride (v < n_vec) and are
 *               rotated in place (fp32 math, one rounding to T).
 *   Row r of a sample is token i = r mod tpf of frame slot fi = r / tpf, so (h, w) =
 *   (i / frame_w, i mod frame_w) and t = frame_table[sample*frame_table_stride + fi] when
 *   frame_table (device int32) is non-null, else first_frame + fi.  Rows whose t is negative
 *   (an empty ring slot) are left unchanged.  rows_per_sample must be a multiple of tpf.
 * Errors: MLA_ERR_INVALID_ARG (sizes, vectors beyond row_width), MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_rope3d(const mla_config* cfg, void* data, int32_t n_samples,
                      int32_t rows_per_sample, int32_t row_width, int32_t col_offset,
                      int32_t n_vec, int32_t vec_stride, const int32_t* frame_table,
                      int32_t frame_table_stride, int32_t first_frame, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_key_positions: the integer (t, h, w) of every key a chunk attends to, in the order
 * mla_attention_fwd walks them: ring slots 0 .. n_valid_frames*tpf - 1 (t from slot_frame), then
 * the chunk's own n_q tokens (t = first_frame + j).  Which keys are attended is the window rule
 * of [A]/[I]: the valid ring frames plus the whole chunk, bidirectionally.
 *   slot_frame device int32 [B, window_frames]; pos_out device int32 [B, n_keys, 3] with
 *   n_keys = (n_valid_frames + chunk_frames)*tpf.  0 <= n_valid_frames <= window_frames.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_key_positions(const mla_config* cfg, const int32_t* slot_frame,
                             int32_t n_valid_frames, int32_t first_frame, int32_t* pos_out,
                             void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_compose_query_weights: weight absorption of the key up-projection into the query path.
 * The content score q_nope_h . (W_UK_h c_KV) equals (W_UK_h^T W_UQ_h c_Q) . c_KV, so attention
 * can run on the latent directly.  (The pages define the two-part score [M]; absorption is exact
 * algebra, not a statement of the pages.)
 *   w_uq  device T [H, d_head, d_cq]   per-head content-query up-projection (q_nope = W_UQ_h c_Q)
 *   w_uk  device T [H, d_head, d_c]    per-head key up-projection
 *   w_qr  device T [H, d_rope, d_cq]   per-head positional-query projection
 *   w_qcat device T [H, D, d_cq]       out: rows 0..d_c-1 = W_UK_h^T W_UQ_h (fp32 accumulation,
 *                                      one rounding to T), rows d_c.. = W_QR_h (copied)
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_compose_query_weights(const mla_config* cfg, const void* w_uq, const void* w_uk,
                                     const void* w_qr, void* w_qcat, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_query_proj: the query path ([M]: query latent c_Q derived from x; head-specific positional
 * query computed from c_Q and rotated), in absorbed form.
 *   c_q[b, n]      = W_down^Q x[b, n]                                  (T, fp32 accumulation)
 *   q[b, n, h, :]  = [ w_qcat[h, 0:d_c] c_q  ||  RoPE3D(w_qcat[h, d_c:D] c_q, pos(b, n)) ]
 * pos(b, n) = (first_frame + n / tpf, row, column) of chunk token n.  q is not scaled.
 *   x      device T [B, n_q, d_model]     w_dq  device T [d_cq, d_model]
 *   w_qcat device T [H, D, d_cq] (from mla_compose_query_weights)
 *   c_q    device T [B, n_q, d_cq] (out)  q     device T [B, n_q, H, D] (out)
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_query_proj(const mla_config* cfg, const void* x, const void* w_dq,
                          const void* w_qcat, void* c_q, void* q, int32_t first_frame,
                          void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_project_chunk: every projection of a chunk's tokens in one pass over x: the query path of
 * mla_query_proj and the joint KV down-projection of mla_cache_append(MLA_PROJECT) ([M]: the
 * query latent c_Q and the content latent c_KV are both down-projections of the token x, and
 * k_R is W_R^K x).  The results equal those two calls:
 *   c_q[b, n]        = W_down^Q x[b, n]
 *   chunk_lat[b, n]  = [W_down^KV x[b, n] || W_R^K x[b, n]]
 *   q[b, n, h, :]    = [ w_qcat[h, 0:d_c] c_q  ||  RoPE3D(w_qcat[h, d_c:D] c_q, pos(b, n)) ]
 *   x      device T [B, n_q, d_model]
 *   w_x    device T [d_cq + D, d_model]: rows 0..d_cq-1 = W_down^Q, rows d_cq..d_cq+d_c-1 =
 *          W_down^KV, rows d_cq+d_c.. = W_R^K (the three down-projections stacked)
 *   w_qcat device T [H, D, d_cq] (from mla_compose_query_weights)
 *   c_q    device T [B, n_q, d_cq] (out)   q device T [B, n_q, H, D] (out)
 *   chunk_lat device T [B, n_q, D] (out)
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_project_chunk(const mla_config* cfg, const void* x, const void* w_x,
                             const void* w_qcat, void* c_q, void* q, void* chunk_lat,
                             int32_t first_frame, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_project_latents: the two down-projections of mla_project_chunk without the query heads
 * ([M]: the query latent c_Q and the content latent c_KV are down-projections of the token x,
 * k_R = W_R^K x), in one pass over x:
 *   c_q[b, n]       = W_down^Q x[b, n]                       device T [B, n_q, d_cq] (out)
 *   chunk_lat[b, n] = [W_down^KV x[b, n] || W_R^K x[b, n]]   device T [B, n_q, D]    (out)
 *   x device T [B, n_q, d_model]; w_x device T [d_cq + D, d_model] as in mla_project_chunk.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_project_latents(const mla_config* cfg, const void* x, const void* w_x, void* c_q,
                               void* chunk_lat, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_project_latents_rotated: mla_project_latents that also prepares the rotated positional
 * keys of the chunk's attention ([M]: k_R is cached unrotated and rotated by 3D-RoPE when the
 * chunk's attention runs), so that mla_attention_fwd_from_cq_prerotated needs no rotation pass.
 * Into `workspace` (the layout of mla_attention_workspace_bytes(cfg, n_valid_frames)) it writes
 * RoPE3D of every chunk token's k_R, as chunk_lat stores it, at the token's position (frame
 * first_frame + frame within the chunk), and the zero padding after the chunk; with
 * rotate_ring = 1 also RoPE3D of ring slots 0 .. n_valid_frames*tpf - 1 (t from slot_frame) and
 * the ring part's padding, exactly as mla_rotate_ring_keys does; with rotate_ring = 0 the ring
 * part is left as it is (a frozen ring whose keys mla_rotate_ring_keys rotated already).  On the
 * tensor-core path (bf16, d_cq and d_cq + d_c multiples of 32, d_rope in {16, 32, 64}) this is
 * one kernel: the projection GEMM's epilogue writes the chunk's rotated keys and its idle
 * epilogue warps rotate the ring's while the first tile's MMAs run; otherwise the projection
 * GEMMs and the rotation pass run one after the other, with the same results.
 *   x, w_x, c_q, chunk_lat   as in mla_project_latents
 *   cache, slot_frame        as in mla_attention_fwd (cache may be NULL when rotate_ring = 0 or
 *                            n_valid_frames = 0)
 *   n_valid_frames, first_frame  of the chunk's attention call
 *   workspace, workspace_bytes   the attention call's workspace, 256-byte aligned
 *   dev_status               as in mla_attention_fwd (MLA_DEBUG builds check the ring slots), or
 *                            NULL
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_WORKSPACE, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_project_latents_rotated(const mla_config* cfg, const void* x, const void* w_x,
                                       void* c_q, void* chunk_lat, const void* cache,
                                       const int32_t* slot_frame, int32_t n_valid_frames,
                                       int32_t first_frame, int32_t rotate_ring, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status,
                                       void* stream);

/* mla_attention_uses_tensor_cores: 1 if mla_attention_fwd with this configuration (and with the
 * W_UV epilogue when with_w_uv != 0) runs the tcgen05 tensor-core kernel, 0 if it runs the
 * CUDA-core kernel, -1 for an invalid configuration.  The tensor-core kernel covers bf16 with
 * d_c in {128, 192, 256} and d_rope in {16, 32, 64} (and d_head = 128 with W_UV) unless
 * kernel_path forces the CUDA-core path.  Host-only; launches nothing. */
int32_t mla_attention_uses_tensor_cores(const mla_config* cfg, int32_t with_w_uv);

/* --------------------------------------------------------------------------------------------
 * mla_attention_workspace_bytes: device scratch mla_attention_fwd needs for a call with the
 * given number of valid ring frames (rotated positional keys of every attended key, tile-padded).
 * Returns 0 for an invalid configuration.
 * ------------------------------------------------------------------------------------------ */
size_t mla_attention_workspace_bytes(const mla_config* cfg, int32_t n_valid_frames);

/* --------------------------------------------------------------------------------------------
 * mla_attention_fwd: latent-space multi-head attention of one chunk against the ring plus
 * itself ([M]: the score of head h combines q_nope.k_nope and q_rope.k_rope; per-head keys and
 * values are reconstructed from c_KV only when needed; [A]: sliding window).
 * Keys: ring slots 0 .. n_valid_frames*tpf - 1 (their frames from slot_frame), then the chunk's
 * own tokens; every query of the chunk sees every one of these keys (block-causal across chunks,
 * bidirectional inside the chunk).  For key m with latent L_m = [c_m || k_R,m]:
 *   K'_m   = [c_m || RoPE3D(k_R,m, pos_m)]
 *   s      = softmax_scale * q[b, n, h, :] . K'_m
 *   p      = softmax over m (fp32)
 *   O_lat  = sum_m p c_m                                   (the value of head h is W_UV_h c_m)
 *   out    = W_UV_h O_lat  (if w_uv != NULL)  else  O_lat
 *
 *   q          device T [B, n_q, H, D]         from mla_query_proj
 *   chunk_lat  device T [B, n_q, D]            the chunk's own latents (MLA_PROJECT)
 *   cache      device T [B, window_frames*tpf, D] the ring; slots >= n_valid_frames*tpf unused
 *   slot_frame device int32 [B, window_frames]
 *   n_valid_frames  0..window_frames, first_frame >= 0
 *   w_uv       device T [H, d_head, d_c] or NULL
 *   out        device T [B, n_q, H*d_head] (w_uv given; heads concatenated in head order)
 *              or device T [B, n_q, H, d_c] (w_uv NULL)
 *   lse        device float [B, H, n_q] natural-log softmax denominators of the scaled scores,
 *              or NULL
 *   workspace  device scratch of >= mla_attention_workspace_bytes(cfg, n_valid_frames) bytes,
 *              256-byte aligned; its contents on entry do not matter
 *   dev_status device int32 word or NULL.  The caller sets it to 0; a kernel writes
 *              MLA_ERR_DEVICE_TIMEOUT there if one of its bounded waits ran out (results are then
 *              undefined).  The host reads it after synchronising.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_WORKSPACE, MLA_ERR_UNSUPPORTED,
 * MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_attention_fwd(const mla_config* cfg, const void* q, const void* chunk_lat,
                             const void* cache, const int32_t* slot_frame,
                             int32_t n_valid_frames, int32_t first_frame, const void* w_uv,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_attention_fwd_from_cq: mla_attention_fwd with the absorbed query heads computed inside the
 * attention kernel from the query latent ([M]: the head-specific queries are computed from
 * c_Q, the positional one rotated by 3D-RoPE).  Each CTA forms its own tile of
 *   q[b, n, h, :] = [ w_qcat[h, 0:d_c] c_q[b, n] || RoPE3D(w_qcat[h, d_c:D] c_q[b, n], pos(b, n)) ]
 * (fp32 accumulation, rounded once to bf16, exactly as mla_query_proj stores it) and attends
 * with it; q never goes through device memory.  Results equal mla_query_proj followed by
 * mla_attention_fwd on the same inputs.
 *   c_q    device T [B, n_q, d_cq]   (mla_project_latents)
 *   w_qcat device T [H, D, d_cq]     (mla_compose_query_weights)
 *   the other arguments, results and the workspace as in mla_attention_fwd.
 * Needs the tensor-core path: bf16, d_c in {128, 192}, d_rope in {16, 32, 64} with
 * d_c + d_rope <= 256, d_cq a multiple of 64 (and d_head = 128 with w_uv); otherwise
 * MLA_ERR_UNSUPPORTED (use mla_project_chunk and mla_attention_fwd).  Errors: those of
 * mla_attention_fwd and MLA_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_attention_fwd_from_cq(const mla_config* cfg, const void* c_q, const void* w_qcat,
                                     const void* chunk_lat, const void* cache,
                                     const int32_t* slot_frame, int32_t n_valid_frames,
                                     int32_t first_frame, const void* w_uv, void* out, float* lse,
                                     void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream);
/* mla_attention_fwd_from_cq_cached_ring: mla_attention_fwd_from_cq for a workspace whose ring
 * part already holds the rotated ring keys (mla_rotate_ring_keys, same cache, slot_frame and
 * n_valid_frames, unchanged since), as mla_attention_fwd_cached_ring is to mla_attention_fwd:
 * only the chunk's own positional keys are rotated.  Arguments, results and errors as in
 * mla_attention_fwd_from_cq. */
mla_status mla_attention_fwd_from_cq_cached_ring(
    const mla_config* cfg, const void* c_q, const void* w_qcat, const void* chunk_lat,
    const void* cache, const int32_t* slot_frame, int32_t n_valid_frames, int32_t first_frame,
    const void* w_uv, void* out, float* lse, void* workspace, size_t workspace_bytes,
    int32_t* dev_status, void* stream);
/* mla_attention_fwd_from_cq_prerotated: mla_attention_fwd_from_cq for a workspace that already
 * holds every rotated positional key of the call (mla_project_latents_rotated with the same
 * chunk_lat, cache, slot_frame, n_valid_frames and first_frame, none changed since): the
 * attention kernel alone runs, with no rotation pass.  Results are bit-identical to
 * mla_attention_fwd_from_cq.  Arguments, results and errors as in mla_attention_fwd_from_cq. */
mla_status mla_attention_fwd_from_cq_prerotated(
    const mla_config* cfg, const void* c_q, const void* w_qcat, const void* chunk_lat,
    const void* cache, const int32_t* slot_frame, int32_t n_valid_frames, int32_t first_frame,
    const void* w_uv, void* out, float* lse, void* workspace, size_t workspace_bytes,
    int32_t* dev_status, void* stream);

/* --------------------------------------------------------------------------------------------
 * Frozen-ring attention.  While a chunk is denoised in several steps, every step attends to the
 * same ring ([I]: the rolling cache only moves on once a chunk is finished), so the rotation of
 * the ring's positional keys ([M]: k_R is cached unrotated and rotated by 3D-RoPE when attention
 * runs) gives the same values at every step.  These two calls split mla_attention_fwd so that
 * rotation is done once per ring state:
 *
 * mla_rotate_ring_keys: writes RoPE3D(k_R) of ring slots 0 .. n_valid_frames*tpf - 1 (t from
 *   slot_frame) into the ring part of an attention workspace (layout of
 *   mla_attention_workspace_bytes(cfg, n_valid_frames)).  Arguments as in mla_attention_fwd.
 *   Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_WORKSPACE, MLA_ERR_CUDA.
 *
 * mla_attention_fwd_cached_ring: mla_attention_fwd for a workspace whose ring part already holds
 *   the rotated ring keys written by mla_rotate_ring_keys with the same cache, slot_frame and
 *   n_valid_frames, none of which may have changed since; only the chunk's own positional keys
 *   are rotated.  Results are bit-identical to mla_attention_fwd.  Arguments, results and errors
 *   are those of mla_attention_fwd.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_rotate_ring_keys(const mla_config* cfg, const void* cache,
                                const int32_t* slot_frame, int32_t n_valid_frames,
                                void* workspace, size_t workspace_bytes, void* stream);
mla_status mla_attention_fwd_cached_ring(const mla_config* cfg, const void* q,
                                         const void* chunk_lat, const void* cache,
                                         const int32_t* slot_frame, int32_t n_valid_frames,
                                         int32_t first_frame, const void* w_uv, void* out,
                                         float* lse, void* workspace, size_t workspace_bytes,
                                         int32_t* dev_status, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_attention_fwd_static_scratch: mla_attention_fwd without the workspace arguments, for
 * callers that cannot allocate device memory.  The paper has no counterpart to this call; it
 * exists for deployment.  Some callers have no way to hand the library a scratch buffer:
 * plugins whose host framework gives them only their input and output buffers, and services
 * that forbid device allocation after start-up.  This call keeps its scratch (the rotated
 * positional keys of the attended keys) in a fixed 16 MiB array compiled into the library, and
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Arguments, results and errors are those of mla_attention_fwd.  A call whose scratch,
 *     mla_attention_workspace_bytes(cfg, n_valid_frames), exceeds 16 MiB (16777216 bytes) is
 *     rejected with MLA_ERR_WORKSPACE before anything is launched.
 *   - Every device that loads the library keeps those 16 MiB reserved until the process exits.
 *   - The first call in a CUDA context (normally: the first call on a device) looks up the
 *     array's device address with cudaGetSymbolAddress, with that device current, and caches it
 *     for that context; make that first call before any stream capture begins.  A device reset
 *     or another context gives a new context, whose first call looks the address up again.
 *   - All calls share the one array per device.  Calls whose kernels overlap on the GPU (on
 *     different streams, or from different host threads) race on it and give wrong results;
 *     order them on one stream.  Each call rewrites every part of the array it reads, so what an
 *     earlier call left there does not matter.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_attention_fwd_static_scratch(const mla_config* cfg, const void* q,
                                            const void* chunk_lat, const void* cache,
                                            const int32_t* slot_frame, int32_t n_valid_frames,
                                            int32_t first_frame, const void* w_uv, void* out,
                                            float* lse, int32_t* dev_status, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_attention_bwd: gradients of mla_attention_fwd without the W_UV epilogue, for training
 * ([M]: the latent students are trained through these layers).  With G = dL/dO_lat and the
 * forward's definitions (K'_m = [c_m || RoPE3D(k_R,m)], s = scale q.K'_m, p = exp(s - lse),
 * O_lat = sum_m p c_m):
 *   dP = G . c_m,  Delta = G . O_lat,  dS = p (dP - Delta)
 *   d_q[b, n, h]      = scale sum_m dS K'_m                         (w.r.t. q as given: its
 *                                                                     positional part rotated)
 *   d latent of key m = [ sum_{h,n} (p G + scale dS q[:d_c])  ||  RoPE3D^T(scale sum dS q[d_c:]) ]
 * i.e. w.r.t. the latents as stored (k_R unrotated; the transpose of a rotation is the rotation
 * by the opposite angle).  Keys are walked as in mla_attention_fwd.
 *   q, chunk_lat, cache, slot_frame, n_valid_frames, first_frame: as given to the forward
 *   o_lat     device T [B, n_q, H, d_c]   the forward's latent output (w_uv = NULL)
 *   lse       device float [B, H, n_q]    the forward's lse
 *   d_o_lat   device T [B, n_q, H, d_c]   dL/dO_lat
 *   d_q       device T [B, n_q, H, D]     out
 *   d_chunk_lat device T [B, n_q, D]      out: gradient of the chunk's latents
 *   d_cache   device T [B, W*tpf, D]      out: rows 0 .. n_valid_frames*tpf - 1 (the attended
 *                                         ring slots) are written, the others left untouched;
 *                                         may be NULL when n_valid_frames == 0
 *   workspace device scratch of >= mla_attention_bwd_workspace_bytes(cfg, n_valid_frames)
 *             bytes, 256-byte aligned; contents on entry do not matter
 *   dev_status device int32 word or NULL, as in mla_attention_fwd (bounded waits of the
 *             tensor-core kernels)
 * Probabilities are recomputed from q, the keys and lse.  bf16 with d_c 192, d_rope 32 and n_q a
 * multiple of 4 runs on the tensor cores (P and dS rounded to bf16 as MMA operands, fp32
 * accumulation); other shapes, fp32 and MLA_PATH_SIMT on CUDA cores in fp32.  Errors:
 * MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_WORKSPACE, MLA_ERR_UNSUPPORTED
 * (d_c + d_rope > 512), MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
size_t mla_attention_bwd_workspace_bytes(const mla_config* cfg, int32_t n_valid_frames);
mla_status mla_attention_bwd(const mla_config* cfg, const void* q, const void* chunk_lat,
                             const void* cache, const int32_t* slot_frame,
                             int32_t n_valid_frames, int32_t first_frame, const void* o_lat,
                             const float* lse, const void* d_o_lat, void* d_q,
                             void* d_chunk_lat, void* d_cache, void* workspace,
                             size_t workspace_bytes, int32_t* dev_status, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_out_proj: value up-projection of latent outputs and the optional output projection
 * ([M]: v_{t,h} is reconstructed from c_KV by W_UV_h; the output projection is the usual
 * attention-layer output map, which the pages do not describe).
 *   o[b, n, h*d_head:(h+1)*d_head] = W_UV_h o_lat[b, n, h]        (T, fp32 accumulation)
 *   y[b, n] = W_O o[b, n]                                          (only if w_o and y non-null)
 *   o_lat device T [B, n_q, H, d_c]   w_uv device T [H, d_head, d_c]   o device T [B, n_q, H*d_head]
 *   w_o   device T [d_model, H*d_head] or NULL                        y device T [B, n_q, d_model]
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_out_proj(const mla_config* cfg, const void* o_lat, const void* w_uv,
                        const void* w_o, void* o, void* y, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_selftest_wait_timeout: checks, without faulting anything, that a kernel of this library
 * whose bounded wait runs out reports it.  It launches one thread that waits, with the same
 * bounded-wait routine the tensor-core kernels use, on a barrier that nothing ever completes;
 * after about limit_us microseconds (1 .. 1e6) the wait gives up and the kernel writes
 * MLA_ERR_DEVICE_TIMEOUT to *dev_status (device int32) and exits.  The caller zeroes
 * *dev_status first and reads it after synchronising.  For failure-handling tests only.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_selftest_wait_timeout(int32_t* dev_status, int32_t limit_us, void* stream);

/* --------------------------------------------------------------------------------------------
 * Self-tests of the library's own approximations (for tests only).  Each evaluates, on the
 * device, the very function the kernels use, so that a test can hold it to its error bound.
 * All arrays are device memory, 4-byte aligned; n >= 0 elements.  Errors: MLA_ERR_INVALID_ARG,
 * MLA_ERR_ALIGNMENT, MLA_ERR_CUDA.
 *
 * mla_selftest_exp2: for every x[i] (float): y_poly[i] = the softmax's FMA-pipe 2^x (degree-3
 *   interpolant of 2^f at the Chebyshev nodes of [-1/2, 1/2], f = x - rint(x), scaled by 2^rint(x)
 *   through the exponent field; arguments below -125 are clamped to -125), evaluated in pairs as
 *   the softmax does; y_sfu[i] = the SFU's ex2.approx.ftz(x); y_exp2f[i] = CUDA's exp2f(x).
 * mla_selftest_sincos: sin and cos of angle[i] as 3D-RoPE computes them (reduction by 2 pi in two
 *   float constants, then the hardware sine/cosine on [-pi, pi]).
 * mla_selftest_rope_angles: for positions pos[i] = (t, h, w) (device int32 [n, 3]) and every
 *   rotary pair j of cfg ([M] 3D-RoPE, reading of mla_config): angle[i, j] (float [n, d_rope/2])
 *   as the kernels compute it, and its sine and cosine (sin_out, cos_out, float [n, d_rope/2]).
 * ------------------------------------------------------------------------------------------ */
mla_status mla_selftest_exp2(const float* x, float* y_poly, float* y_sfu, float* y_exp2f,
                             int32_t n, void* stream);
mla_status mla_selftest_sincos(const float* angle, float* sin_out, float* cos_out, int32_t n,
                               void* stream);
mla_status mla_selftest_rope_angles(const mla_config* cfg, const int32_t* pos, int32_t n,
                                    float* angle, float* sin_out, float* cos_out, void* stream);

/* --------------------------------------------------------------------------------------------
 * mla_probe_sm_clock: measures the SM clock on the device, for reports of achieved throughput
 * (it reads counters only and changes no setting).  Launches n_ctas CTAs of one warp (one per
 * SM when n_ctas <= the SM count and nothing else runs); thread 0 of each reads its SM's cycle
 * counter and the global nanosecond timer, spins on the timer for spin_us microseconds and
 * reads both again.  out (device uint64 [n_ctas, 4]) receives, per CTA: the SM id, the cycles
 * and the nanoseconds elapsed, 0; the SM clock in MHz is 1000 * cycles / nanoseconds.
 * 1 <= n_ctas <= 4096, 1 <= spin_us <= 1e5.  Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT,
 * MLA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------ */
mla_status mla_probe_sm_clock(unsigned long long* out, int32_t n_ctas, int32_t spin_us,
                              void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MLA_LATENT_KV_ATTN_H_ */
