/*
 * vmla.h -- C ABI of libvmla.so: VideoMLA latent-KV chunk attention on B200 (sm_100a).
 *
 * The method (VideoMLA: Low-Rank Latent KV Cache for Minute-Scale
 * Autoregressive Video Diffusion; cited below by page and section):
 *   [paperlayer]  summary on paperlayer.ai: §3 Method, §4, App. C.1, D.1-D.5, E, F
 *   [gist.it]     technical summary on gist.science (Italian), "Metodologia" 1-4
 *
 * Every token of a fixed sliding window of latent video frames is cached as a
 * shared content latent c_KV = W_dkv x (d_latent scalars) plus one head-shared
 * positional key k_R = W_kr x (d_rope scalars), stored before its 3D rotary
 * embedding [gist.it pt. 1, 3; paperlayer §3, App. D.5].  A chunk of new
 * frames attends over the whole window, itself included, with per-head queries
 * split into a content part (d_nope) and a 3D-rotated positional part (d_rope)
 * [paperlayer App. D.3-D.4].
 *
 * Conventions shared by every call
 * --------------------------------
 * - Memory.  The caller owns every device buffer (cache, workspace, weights,
 *   activations, outputs) and passes raw device pointers.  The library owns
 *   only its host-side handle; it never allocates device memory.  Device
 *   pointers must be 16-byte aligned.
 * - Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   Compute calls only enqueue work on it and return; nothing synchronises
 *   except vmla_device_status() and vmla_profile_read().
 * - Layout.  Row-major, contiguous, batch outermost.  dtype VMLA_BF16 means
 *   weights, x, q and the caches are bf16 (accumulation is fp32); VMLA_FP32
 *   means float.  Attention outputs are float32 in both cases.
 * - Errors.  Every call validates its arguments on the host and returns a
 *   vmla_status; nothing is enqueued when it is not VMLA_OK.  A launch
 *   failure reported by CUDA returns VMLA_ERR_CUDA.  Device-side faults that
 *   the kernels detect themselves (a pipeline wait that ran out of time, an
 *   index outside its buffer) are recorded in a device status word that
 *   vmla_device_status() reads.
 * - Threads.  A handle is not thread-safe; distinct handles are independent.
 */
#ifndef VMLA_H_
#define VMLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VMLA_ABI_VERSION 3

typedef enum vmla_status {
  VMLA_OK = 0,
  VMLA_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size, misaligned pointer */
  VMLA_ERR_UNSUPPORTED_SHAPE = 2, /* shape has no kernel for this dtype (see vmla_config_check) */
  VMLA_ERR_OUT_OF_RANGE = 3,      /* layer index, frame count or a RoPE position >= 1024 out of range */
  VMLA_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed */
  VMLA_ERR_DEVICE_TIMEOUT = 5,    /* a kernel gave up on a pipeline wait (device status word) */
  VMLA_ERR_STATE = 6,             /* frame sequence not allowed (skips or rewinds), buffers not bound */
  VMLA_ERR_DEVICE_BOUNDS = 7,     /* a kernel found an index outside its buffer (device status word) */
  VMLA_ERR_DEVICE_RANGE = 8       /* a kernel produced a value past the range of its storage type: a per-head
                                     query, key or value above 65504 in the fp16 reconstruct-once
                                     workspace (device status word) */
} vmla_status;

typedef enum vmla_dtype { VMLA_BF16 = 0, VMLA_FP32 = 1 } vmla_dtype;

/* How vmla_chunk_attention evaluates the same scores and outputs. */
typedef enum vmla_design {
  VMLA_DESIGN_AUTO = 0,        /* the design measured fastest that meets the accuracy gate:
                                  VMLA_BF16: RECON_ONCE from 192 latent dims on (and for the splits the
                                  absorbed kernel does not take), ABSORBED at 64 and 128.  VMLA_FP32
                                  always evaluates the absorbed form.  vmla_workspace_bytes(AUTO)
                                  covers the RECON_ONCE workspace whenever AUTO takes it; with a
                                  smaller workspace bound, AUTO stays ABSORBED up to 256 latent dims */
  VMLA_DESIGN_ABSORBED = 1,    /* W_uk folded into the query, MQA over [c_KV | k_R], W_uv after the
                                  softmax-weighted sum [paperlayer App. E] */
  VMLA_DESIGN_RECONSTRUCT = 2, /* per KV tile, per-head K/V rebuilt from c_KV on the tensor core and kept
                                  in shared memory, then d_head attention [gist.it pt. 2; paperlayer §3
                                  On-demand reconstruction]; VMLA_BF16 with d_latent 64, 128 or 192
                                  (VMLA_ERR_UNSUPPORTED_SHAPE otherwise), no extra workspace */
  VMLA_DESIGN_RECON_ONCE = 3   /* per-head K/V of the whole window rebuilt once into the workspace, then
                                  d_head attention; the rebuilt K/V, the per-head queries and the
                                  probabilities are fp16 (rounding 2^-11 against bf16's 2^-8), and a
                                  value past fp16's range is reported (VMLA_ERR_DEVICE_RANGE) */
} vmla_design;

/* When the positional key gets its 3D rotation. */
typedef enum vmla_rope_mode {
  VMLA_ROPE_AT_READ = 0,  /* stored unrotated, rotated at attention time with window-relative frame
                             indices: t = the frame's position in the window, oldest first (sink
                             frames first) [paperlayer App. D.5, App. E] */
  VMLA_ROPE_AT_APPEND = 1 /* rotated at append with the absolute frame index (scores are identical
                             without a sink frame, RoPE depends on offsets only) */
} vmla_rope_mode;

typedef struct vmla_config {
  int d_model;           /* D, width of x (1536) */
  int n_heads;           /* n_h (12) */
  int d_nope;            /* per-head content dims of q and k (96) */
  int d_rope;            /* positional dims, = 2*(rope_pairs[0]+rope_pairs[1]+rope_pairs[2]) (32) */
  int d_latent;          /* d_c, width of c_KV (192) */
  int d_value;           /* per-head value / output dims (128) */
  int rope_pairs[3];     /* complex pairs of the t, h, w axes ((6,5,5), [paperlayer App. D.3]) */
  int rope_base_dims[3]; /* B_a in w_{a,i} = theta^(-2i/B_a); 0 means 2*rope_pairs[a] */
  float rope_theta;      /* 10000 */
  int grid_h, grid_w;    /* latent frame grid; tokens per frame T_f = grid_h*grid_w (30 x 52 = 1560) */
  int window_frames;     /* W: ring capacity in frames, sink and current chunk included (21; 7 with a sink) */
  int chunk_frames;      /* largest n_frames of an attention call (3) */
  int batch;             /* independent rings (one per sample) */
  int layers;            /* layers held by one handle's caches */
  vmla_dtype dtype;
  vmla_rope_mode rope_mode;
  float softmax_rescale_log2; /* online softmax: a row's running max is raised only when a key tile's
                                 max exceeds it by more than 2^this (8 by default); 0 raises it on
                                 every increase.  Results are the same; only the amount of O
                                 rescaling work differs. */
  int sink_frames;       /* S: the first S frames of a rollout stay in the ring for good (slots 0..S-1);
                            later frames rotate FIFO through the other W-S slots.  Keys take
                            window-relative t: the sink 0..S-1, the local frames S.. in order
                            [paperlayer App. D.4: one sink latent frame + six recent ones; App. D.5
                            re-indexing].  0 (default): plain FIFO window.  Needs rope_mode
                            VMLA_ROPE_AT_READ and chunk_frames <= W-S; no dense cache. */
} vmla_config;

typedef struct vmla_handle vmla_handle;

/* Name of a status code (static string, never NULL). */
const char* vmla_status_string(vmla_status status);

/* Text of the CUDA error (name: description), or of the tensor-map encoding
 * failure, behind the last VMLA_ERR_CUDA this thread received; "" before any.
 * The pointer stays valid until the thread's next failing call. */
const char* vmla_last_error_detail(void);

/* VMLA_ABI_VERSION of the loaded library. */
int vmla_abi_version(void);

/* Fill *cfg with one Wan2.1-T2V-1.3B attention layer [paperlayer §4, App. C.1, D.1-D.3]:
 * D=1536, 12 heads, d_nope=96, d_rope=32 in (6,5,5) pairs, d_c=192, d_value=128,
 * 30x52 grid, W=21 frames, chunks of 3 frames, batch 1, 1 layer, bf16, RoPE at read,
 * softmax_rescale_log2 = 8. */
vmla_status vmla_config_init(vmla_config* cfg);

/* VMLA_OK when every field is consistent and a kernel exists for it:
 * VMLA_FP32 accepts any positive sizes (d_latent + d_rope <= 1024, d_value <= 1024, up to 64
 * rotary pairs);
 * VMLA_BF16 needs d_model a multiple of 64, d_nope + d_rope = d_value = 128 and d_latent one of
 * 64, 128, 192, 256, 384, 512 (VMLA_DESIGN_ABSORBED up to 256, VMLA_DESIGN_RECONSTRUCT up to 192),
 * with d_rope = 32 for every design, or d_rope = 16 (d_latent <= 256) or 64 (d_latent <= 192) for
 * the absorbed design only: the other designs, the dense cache, the folded mixer, the query-latent
 * path and the allocation-free call return VMLA_ERR_UNSUPPORTED_SHAPE for those splits.
 * Other shapes run with VMLA_FP32.
 * grid_h, grid_w, window_frames must be < 1024 (RoPE range, [paperlayer App. C.1]). */
vmla_status vmla_config_check(const vmla_config* cfg);

/* Bytes of the caller-allocated caches of one handle (all layers and samples):
 *   ckv:  [layers][batch][window_frames*T_f][d_latent]
 *   kr:   [layers][batch][window_frames*T_f][d_rope]
 *   dense_kv (the per-head comparison layout, 2*n_heads*d_value scalars per token):
 *         [layers][batch][window_frames*T_f][2][n_heads][d_value]  (keys, then values)
 * Any output pointer may be NULL. */
vmla_status vmla_cache_bytes(const vmla_config* cfg, size_t* ckv_bytes, size_t* kr_bytes, size_t* dense_kv_bytes);

/* Bytes of device workspace that vmla_bind() needs for calls with `design`
 * (and for the dense calls, whatever design). */
vmla_status vmla_workspace_bytes(const vmla_config* cfg, vmla_design design, size_t* bytes);

/* Where the intermediates of a chunk attention call live inside the workspace, as byte offsets
 * (for inspection and stage-by-stage checks; the workspace's contents after a call are those of
 * the last call that wrote them):
 *   [VMLA_WS_KR_ROT]  the window's positional keys rotated with window-relative t
 *                     [batch][W*T_f][d_rope] (RoPE at read only; ring-slot order; ABSORBED and
 *                     RECONSTRUCT: RECON_ONCE rotates them inside the reconstruction)
 *   [VMLA_WS_QT]      absorbed queries [batch][n_heads][n_q][d_latent + d_rope] (ABSORBED)
 *   [VMLA_WS_QD]      per-head queries with the positional part rotated [batch][n_heads][n_q][d_nope + d_rope]
 *                     (RECONSTRUCT, RECON_ONCE and the dense calls)
 *   [VMLA_WS_RECON]   the window's per-head keys and values [batch][W*T_f][2][n_heads][d_value] (RECON_ONCE)
 * n_q = chunk_frames * T_f; dtype-sized elements.  `n` >= VMLA_WS_COUNT. */
enum { VMLA_WS_KR_ROT = 0, VMLA_WS_QT = 1, VMLA_WS_QD = 2, VMLA_WS_RECON = 3, VMLA_WS_COUNT = 4 };
vmla_status vmla_workspace_offsets(const vmla_config* cfg, size_t* offsets, int n);

/* The angular frequency of each rotary pair, t pairs first, then h, then w
 * (w_{a,i} = theta^(-2i/B_a), i = 0..pairs_a-1 [paperlayer App. D.3]), as float. n >= pair count. */
vmla_status vmla_rope_frequencies(const vmla_config* cfg, float* freqs, int n);

/* Create / destroy a handle (host memory only; no CUDA call). */
vmla_status vmla_create(const vmla_config* cfg, vmla_handle** out);
vmla_status vmla_destroy(vmla_handle* h);

/* Attach the caller's latent caches and workspace (sizes from vmla_cache_bytes /
 * vmla_workspace_bytes).  Resets every layer's frame counter to 0.  The cache
 * contents need no initialisation: no kernel reads a slot before it is written. */
vmla_status vmla_bind(vmla_handle* h, void* ckv, void* kr, void* workspace, size_t workspace_bytes);

/* Attach the caller's dense per-head cache (only for the vmla_dense_* calls). */
vmla_status vmla_dense_bind(vmla_handle* h, void* dense_kv);

/* Latent cache write [gist.it pt. 1, 3; paperlayer §3 Shared low-rank KV cache]:
 *   [c_KV | k_R] = W_down x for n_frames frames, written into the ring slots of
 *   frames first_frame .. first_frame+n_frames-1 (slot of frame f = f mod W: the
 *   oldest frame is evicted, FIFO [paperlayer App. D.4]).  k_R is stored unrotated
 *   (VMLA_ROPE_AT_READ) or rotated with the absolute frame index (VMLA_ROPE_AT_APPEND).
 * x:      [batch][n_frames*T_f][d_model]
 * w_down: [d_latent + d_rope][d_model]  (rows of W_dkv, then rows of W_kr)
 * Frame rule per layer (F = frames appended so far): first_frame == F appends a new
 * chunk; first_frame + n_frames == F rewrites the newest frames (the next denoising
 * pass of the same chunk).  Anything else is VMLA_ERR_STATE.  1 <= n_frames <= W. */
vmla_status vmla_cache_append(vmla_handle* h, int layer, const void* x, const void* w_down, int64_t first_frame,
                              int n_frames, void* stream);

/* Chunk attention over the window [paperlayer App. D.3-D.5, App. E]:
 *   for query i of frame first_frame + i/T_f and head h,
 *     out[i, h*d_value:(h+1)*d_value] = sum_j softmax_j(s_ij) W_uv,h c_j,
 *     s_ij = ( q_nope,ih . W_uk,h c_j  +  RoPE(q_rope,ih) . RoPE(k_R,j) ) / sqrt(d_nope + d_rope)
 *   over every key j of the window frames [max(0, F-W), F) -- with sink frames, the first S
 *   frames of the rollout and the newest W-S -- (no mask: the chunk is the newest frames and
 *   sees itself).
 * q:    [batch][n_frames*T_f][n_heads][d_nope + d_rope]  (per head: content, then positional)
 * w_uk: [n_heads][d_nope][d_latent]   w_uv: [n_heads][d_value][d_latent]
 * out:  [batch][n_frames*T_f][n_heads*d_value], float32 for both dtypes (a bf16 rounding of the
 *       output alone would take two thirds of a 3e-2*RMS max-error budget: max |out| is about 5 RMS)
 * The chunk must be the newest appended frames: first_frame + n_frames == F,
 * 1 <= n_frames <= chunk_frames; otherwise VMLA_ERR_STATE.
 * Everything is enqueued on `stream`; VMLA_DESIGN_RECON_ONCE prepares the per-head queries on a
 * stream of the handle's own (created at its first such call), forked from `stream` by an event
 * and joined back into it before the attention kernel, so the call stays ordered on `stream`
 * (and can be captured in a CUDA graph from it). */
vmla_status vmla_chunk_attention(vmla_handle* h, int layer, const void* q, const void* w_uk, const void* w_uv,
                                 void* out, int64_t first_frame, int n_frames, vmla_design design, void* stream);

/* The dense per-head comparison [gist.it problem statement; paperlayer App. C.1]:
 * the same keys and values, cached as 2*n_heads*d_value scalars per token.
 * vmla_dense_cache_append writes k_h = [W_uk,h c | RoPE(k_R)] (rotated with the
 * absolute frame index) and v_h = W_uv,h c into dense_kv, with c and k_R = W_down x
 * as in vmla_cache_append (same frame rule, tracked separately from the latent
 * cache).  vmla_dense_chunk_attention runs d_head attention per head on it, with
 * the query's positional part rotated by the absolute frame index; out is float32 as above. */
vmla_status vmla_dense_cache_append(vmla_handle* h, int layer, const void* x, const void* w_down, const void* w_uk,
                                    const void* w_uv, int64_t first_frame, int n_frames, void* stream);
vmla_status vmla_dense_chunk_attention(vmla_handle* h, int layer, const void* q, void* out, int64_t first_frame,
                                       int n_frames, void* stream);

/* One denoising pass of a chunk, end to end from HOST memory: copy x and q from
 * (preferably pinned) host buffers into the caller's device staging buffers, append,
 * attend, copy out back to the host buffer.  The two input copies run on a stream of the
 * handle's own, each ordered after the previous call's last use of its staging buffer (x_dev:
 * the append; q_dev: the kernel that prepares the queries, the first kernel of the attention), so
 * consecutive calls overlap them with compute; append and
 * attention are enqueued on `stream`, which waits for the inputs.  The absorbed and the
 * reconstruct-once attention run as one launch per group of heads that fills the GPU once, and each
 * group's output columns
 * go back to out_host on a third stream while the next group computes; `stream` waits for the
 * last of those copies (other designs copy the output back on `stream`).  The host buffers
 * must stay valid, and out_host is complete, once `stream` reaches this point.
 * Shapes as above. */
vmla_status vmla_chunk_step_host(vmla_handle* h, int layer, const void* x_host, const void* q_host,
                                 void* out_host, const void* w_down, const void* w_uk, const void* w_uv,
                                 void* x_dev, void* q_dev, void* out_dev, int64_t first_frame, int n_frames,
                                 vmla_design design, void* stream);

/* Host-side view of the window after `frames_appended` frames (the same for every layer): for
 * each window frame -- the sink frames, then the local frames oldest first -- its absolute index,
 * its ring slot (frame mod W without a sink) and the frame index t its keys are rotated with:
 * with VMLA_ROPE_AT_READ the window-relative t (computed from the slot, as the window-RoPE kernel
 * does), with VMLA_ROPE_AT_APPEND the absolute frame index (the append rotated the keys with it).
 * `capacity` is the length of the
 * three arrays (any may be NULL); *n gets the number of window frames; VMLA_ERR_INVALID_ARG when
 * capacity < *n. */
vmla_status vmla_window(const vmla_handle* h, int64_t frames_appended, int32_t* frame, int32_t* slot,
                        int32_t* t_local, int capacity, int* n);

/* Frames appended so far to a layer's latent cache (resume a rollout exactly). */
vmla_status vmla_state_get(const vmla_handle* h, int layer, int64_t* frames_appended);
vmla_status vmla_state_set(vmla_handle* h, int layer, int64_t frames_appended);

/* Synchronise `stream`, read and clear the library's device status word:
 * VMLA_OK, VMLA_ERR_DEVICE_TIMEOUT, VMLA_ERR_DEVICE_BOUNDS or VMLA_ERR_DEVICE_RANGE; *flags (may
 * be NULL) gets the raw bits. */
vmla_status vmla_device_status(vmla_handle* h, void* stream, uint32_t* flags);

/* Per-stage CUDA-event timing of the kernels each call launches, recorded on the
 * stream each launches on.  Stages: 0 append, 1 rope, 2 query preparation (q-absorb; the
 * per-head queries, which reconstruct-once runs on the handle's side stream beside the
 * reconstruction, so their time there spans the overlap), 3 attention (absorbed), 4 attention
 * (reconstruct), 5 dense append, 6 dense attention (also the reconstruct-once attention),
 * 7 reconstruct-once (the reconstruction), 8 folded output mixer.
 * vmla_profile_read synchronises, then returns the summed milliseconds and the
 * launch count of one stage since profiling was enabled. */
vmla_status vmla_profile_enable(vmla_handle* h, int enable);
vmla_status vmla_profile_read(vmla_handle* h, int stage, double* total_ms, int* launches);

/* Work split of the bf16 append kernel (the down-projection GEMM [c_KV | k_R] =
 * W_down x of the paperlayer paper, Sec. 3): a persistent kernel over work items
 * (column part of [c_KV | k_R], one or two 128-row tiles of x).  `n_split` column
 * parts: 0 chooses per call (two when the row tiles alone would leave SMs idle,
 * and always when d_latent > 224; three when d_latent > 480), 1 or 2 forces it.
 * `row_tiles` 128-row tiles per item: 0 or 1 takes one, 2 shares every W_down
 * stage between two MMA chains (fewer L2 reads of W_down per row, but the item's
 * epilogue no longer overlaps the next item's MMAs: slower on the Wan-1.3B layer
 * at batch 1 to 64); two apply only where the call runs one column part.  `max_ctas`
 * caps the grid (0: one CTA per SM); a small cap makes each CTA run many items.
 * Every split gives the same bits.  n_split = 1 with d_latent > 224 makes later
 * appends return VMLA_ERR_UNSUPPORTED_SHAPE.  Host only; VMLA_ERR_INVALID_ARG for
 * n_split or row_tiles outside 0..2, both 2, or a negative cap. */
vmla_status vmla_set_append_tiling(vmla_handle* h, int n_split, int row_tiles, int max_ctas);

/* The value path absorbed all the way into the layer's output mixer [paperlayer App. E]:
 * with B_h = W_O,h W_uv,h (W_O,h the d_value columns of W_O that read head h),
 *   out = sum_h B_h o~_h,   o~_h = softmax-weighted latents of head h (d_latent wide),
 * one GEMM with K = n_heads * d_latent in place of the per-head W_uv,h and W_O.
 * vmla_fold_output_weights writes w_fold [d_out][n_heads*d_latent] (bf16) from
 * w_o [d_out][n_heads*d_value] and w_uv [n_heads][d_value][d_latent] (bf16, fp32 sums;
 * a one-time weight preparation).  vmla_chunk_attention_folded is vmla_chunk_attention
 * with VMLA_DESIGN_ABSORBED followed by that GEMM: o~ is handed over as a bf16 pair
 * (rounded part + residual, in the workspace), out is [batch][n_frames*T_f][d_out] fp32.
 * VMLA_BF16 with d_latent <= 256 and d_out a multiple of 128, else
 * VMLA_ERR_UNSUPPORTED_SHAPE; frame rules and errors as vmla_chunk_attention. */
vmla_status vmla_fold_output_weights(const vmla_config* cfg, const void* w_o, const void* w_uv, void* w_fold,
                                     int d_out, void* stream);
vmla_status vmla_chunk_attention_folded(vmla_handle* h, int layer, const void* q, const void* w_uk,
                                        const void* w_fold, int d_out, void* out, int64_t first_frame,
                                        int n_frames, void* stream);

/* The content path absorbed into the query latent [paperlayer App. E; §4: d_q = 768]:
 * with q_h = [W_uq,h c_Q | W_qr,h c_Q] the per-head queries of the query latent c_Q,
 *   q~_h = [A_h c_Q | RoPE(W_qr,h c_Q)],   A_h = W_uk,h^T W_uq,h  (d_latent x d_q),
 * so the query never exists per head.  vmla_fold_query_weights writes w_qabs
 * [n_heads][d_latent + d_rope][d_q] = [A_h ; W_qr,h] (bf16, fp32 sums; one-time weight
 * preparation) from w_uq [n_heads][d_nope][d_q], w_qr [n_heads][d_rope][d_q] and w_uk.
 * vmla_chunk_attention_qlatent is vmla_chunk_attention with VMLA_DESIGN_ABSORBED whose
 * query step is one GEMM over K = d_q from c_Q [batch][n_frames*T_f][d_q] (bf16).
 * VMLA_BF16 with d_latent 64, 128 or 192 and d_q a multiple of 64, else
 * VMLA_ERR_UNSUPPORTED_SHAPE; frame rules and errors as vmla_chunk_attention. */
vmla_status vmla_fold_query_weights(const vmla_config* cfg, const void* w_uq, const void* w_qr, const void* w_uk,
                                    int d_q, void* w_qabs, void* stream);
vmla_status vmla_chunk_attention_qlatent(vmla_handle* h, int layer, const void* c_q, const void* w_qabs, int d_q,
                                         const void* w_uv, void* out, int64_t first_frame, int n_frames,
                                         void* stream);

/* Allocation-free chunk attention.  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- for example a
 * plugin inside another runtime that is handed only its input and output
 * buffers and owns no allocator, or a latency-critical loop in which a
 * cudaMalloc (which can synchronise the device) is not allowed.  It needs no
 * handle and no workspace.
 *
 * It computes exactly what vmla_chunk_attention computes with
 * VMLA_DESIGN_ABSORBED (same kernels, same arguments and layouts; VMLA_BF16
 * only, the shapes that design takes), for the window of a layer that has
 * `frames_appended` frames in it.
 * `ckv` and `kr` are the caches of all layers as laid out by vmla_cache_bytes.
 * Its scratch (the window's rotated positional keys and the absorbed queries:
 * batch*W*T_f*d_rope*2 bytes, rounded up to 256, plus batch*n_heads*n_frames*T_f*
 * (d_latent + d_rope)*2 bytes) lives in a fixed 32 MiB array inside the library
 * that every GPU which loads the library holds until the process exits;
 * larger calls return VMLA_ERR_OUT_OF_RANGE and enqueue nothing.  The call
 * makes no cudaMalloc or cudaFree and calls no allocating routine.
 * - The first call on each device looks up the array's device address (with
 *   that device current) and keeps it; make that first call before any
 *   stream capture begins.
 * - Every call shares the one array, which keeps the last call's contents.
 *   Nothing in it has to start at zero: each call writes every scratch byte it
 *   reads.  Calls that overlap on the GPU (two streams, or two threads) race
 *   on the array: order them on one stream.
 * Returns as vmla_chunk_attention; device-side errors go to the same device
 * status word (read with vmla_device_status). */
vmla_status vmla_chunk_attention_noalloc(const vmla_config* cfg, int layer, const void* ckv, const void* kr,
                                         int64_t frames_appended, const void* q, const void* w_uk,
                                         const void* w_uv, void* out, int64_t first_frame, int n_frames,
                                         void* stream);

/* Self-test of the polynomial exp2 that the attention kernels evaluate on the
 * FMA pipe for part of each softmax tile (the rest goes to the MUFU unit):
 * y[i] = 2^x[i] for n (even) fp32 values in device memory, both arrays 8-byte
 * aligned.  Relative error <= 7.5e-5 for x >= -125; below that the result is at
 * most 2^-124.  VMLA_ERR_INVALID_ARG for odd n or misaligned arrays. */
vmla_status vmla_selftest_exp2(const float* x, float* y, int64_t n, void* stream);

/* Self-test of the bounded pipeline waits: launches one CTA that waits on an
 * mbarrier nothing arrives at, for at most `limit_ns` nanoseconds (<= 1e9), then
 * returns.  The device status word must afterwards report VMLA_ERR_DEVICE_TIMEOUT. */
vmla_status vmla_selftest_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* VMLA_H_ */
