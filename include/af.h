/*
 * af.h -- C ABI of the B200 affine-autoregressive-flow library (libaf.so).
 *
 * The operations are those of STARFlow-V ("STARFlow-V: End-to-End Video
 * Generative Modeling with Autoregressive Normalizing Flows", CVPR 2026 paper
 * notes, papernotes.org):
 *   - the affine AF block z = (x - mu(x*m)) / sigma(x*m), sigma > 0, m the
 *     self-exclusive causal mask (section "Key design 1: global-local
 *     architecture", affine-flow equation), with log|det dz/dx| = -sum log sigma
 *     (the change of variables behind L_NF, section "Loss / training strategy");
 *   - its inverse by video-aware block-wise Jacobi iteration
 *     x^(k+1) = mu(x^(k)*m) + sigma(x^(k)*m) * z, blocks of B tokens in
 *     sequence, parallel inside a block, finished blocks kept in a KV cache,
 *     warm start from the previous frame's converged x, stop when
 *     ||x^(k+1)-x^(k)||^2 / ||x^(k+1)||^2 < tau (section "Key design 3:
 *     video-aware block-wise Jacobi iteration");
 *   - stacks of T blocks of alternating direction, inverted last to first
 *     (section "Key design 1": T >= 3 alternating blocks).
 *
 * Model inside one AF block (the pages only say "causal Transformer"; the
 * readings taken): the input at sequence position p is x_{p-1} (zero at p=0),
 * i.e. the self-exclusive mask as a one-token shift; h = x_in W_in^T + b_in +
 * P_space[p mod frame_len] + P_time[p div frame_len]; `layers` pre-LN blocks
 * (LayerNorm eps 1e-5, causal multi-head attention j <= i with scale
 * 1/sqrt(d/heads), exact-erf GELU MLP of width mlp_ratio*d); final LayerNorm;
 * head [mu | s] = h W_head^T + b_head with sigma = exp(s).  Direction R2L
 * reverses each sample's token order before the block and restores it after.
 *
 * Conventions for every call below:
 *   - x, z: float32 [batch, L, C] row-major, logdet: float32 [batch],
 *     iters: int32; all are caller-owned DEVICE pointers.  x and z never alias.
 *   - ws: caller-owned device workspace of at least af_workspace_bytes(...)
 *     bytes, 256-byte aligned.  The library allocates nothing per call.
 *   - Every call only enqueues work on `stream` (a cudaStream_t, passed as
 *     void*) and returns.  The returned status covers argument checks and
 *     launch errors; device-side failures (a bounded wait that timed out) are
 *     reported by af_device_error().
 *   - Results are deterministic: the same inputs give the same bits.
 */
#ifndef AF_H_
#define AF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AF_OK = 0,
  AF_ERR_ARG = 1,        /* a bad argument: nothing was enqueued */
  AF_ERR_CUDA = 2,       /* a CUDA call failed; af_last_error_string() tells which */
  AF_ERR_WORKSPACE = 3,  /* ws is null, misaligned or smaller than af_workspace_bytes() */
  AF_NOT_CONVERGED = 4,  /* from af_last_convergence(): some block hit max_iter */
  AF_ERR_DEVICE = 5      /* from af_device_error(): a kernel gave up a bounded wait */
} af_status;

typedef enum { AF_L2R = 0, AF_R2L = 1 } af_dir;
typedef enum { AF_FP32 = 0, AF_BF16 = 1 } af_dtype;

/* Shape of one AF block.  max_len = frame_len * max_frames bounds L.
 * Every config needs positive sizes, d % heads == 0, C % 8 == 0, d % 4 == 0.
 * AF_BF16 also requires C % 64 == 0, d % 128 == 0, (mlp_ratio * d) % 128 == 0
 * and d / heads in {64, 128} (the tensor-core tile shapes);
 * AF_FP32 requires d / heads in {16, 32, 64, 128}. */
typedef struct {
  int C, d, heads, layers, mlp_ratio;
  int frame_len, max_frames;
  af_dtype dtype;
} af_config;

typedef struct af_model af_model;

/* Number of float32 host tensors af_model_create() expects: 4 + 12*layers + 4,
 * in this order ([out, in] row-major matrices):
 *   W_in [d,C], b_in [d], P_space [frame_len,d], P_time [max_frames,d],
 *   per layer: ln1_g [d], ln1_b [d], W_qkv [3d,d] (q;k;v rows, heads as
 *     consecutive d/heads slices), b_qkv [3d], W_o [d,d], b_o [d],
 *     ln2_g [d], ln2_b [d], W_1 [fd,d], b_1 [fd], W_2 [d,fd], b_2 [d]
 *     (fd = mlp_ratio*d),
 *   lnf_g [d], lnf_b [d], W_head [2C,d] (rows 0..C-1 give mu, C..2C-1 give s),
 *   b_head [2C]. */
int af_num_tensors(const af_config* cfg);

/* Copies the weights to the current CUDA device (rounded to bf16, nearest
 * even, for AF_BF16) and returns an opaque model that owns them.  `tensors`
 * are HOST pointers; the call is synchronous.  AF_ERR_ARG on a bad config. */
af_status af_model_create(const af_config* cfg, const float* const* tensors, int n_tensors,
                          af_model** out);
af_status af_model_destroy(af_model* m);

/* Workspace bytes for a call on `batch` sequences of L tokens whose Jacobi
 * blocks hold at most B tokens (pass B = L for af_forward; B need not divide
 * L).  Includes the KV cache of all layers over L positions.  The same
 * workspace serves every block of a stack made of models with the same
 * config.  0 on bad arguments. */
size_t af_workspace_bytes(const af_model* m, int batch, int L, int B);

/* Forward pass of one AF block: z and logdet (= -sum_{i,c} s_{i,c} per
 * sample) from x.  Requires 1 <= L <= max_len. */
af_status af_forward(const af_model* m, const float* x, int batch, int L, af_dir dir,
                     float* z, float* logdet, void* ws, size_t ws_bytes, void* stream);

/* Block-wise Jacobi inverse of one AF block.  Requires L % B == 0,
 * max_iter >= 1, tau >= 0 and finite.  Block b starts from z_b, or, when
 * warm_start != 0, from the previous frame's converged state ("Key design
 * 3": a new frame is warm-started from the previous frame's converged x):
 * the token at working-order position p starts from the converged x at
 * p - k*frame_len, the same spatial position in the most recent finished
 * frame (smallest k >= 1 landing before the block), and from z where no
 * frame before it has finished.  With B = frame_len this is "block b starts
 * from block b-1's final x".  A sample leaves the iteration of a block at
 * the first update whose residual is < tau (0/0 counts as converged);
 * iters[s * (L/B) + b] counts the updates computed.  All iterations, tests
 * and block changes run on the device: one graph launch per call (after one
 * small kernel that writes the block table into ws), no host round trip per
 * iteration. */
af_status af_inverse_jacobi(const af_model* m, const float* z, int batch, int L, af_dir dir,
                            int B, float tau, int max_iter, int warm_start, float* x,
                            int32_t* iters, void* ws, size_t ws_bytes, void* stream);

/* T blocks applied in order t = 0..T-1 (directions dirs[t]); logdet sums the
 * blocks' logdets.  All models must share one af_config. */
af_status flow_stack_forward(const af_model* const* blocks, const af_dir* dirs, int T,
                             const float* x, int batch, int L, float* z, float* logdet,
                             void* ws, size_t ws_bytes, void* stream);

/* Inverse of flow_stack_forward: Jacobi-inverts t = T-1 .. 0.
 * iters is [T, batch, L/B] (block t's counts at offset t*batch*(L/B)). */
af_status flow_stack_inverse(const af_model* const* blocks, const af_dir* dirs, int T,
                             const float* z, int batch, int L, int B, float tau, int max_iter,
                             int warm_start, float* x, int32_t* iters, void* ws,
                             size_t ws_bytes, void* stream);

/* Block-wise Jacobi inverse with a schedule of block sizes, over a range of
 * blocks (section "Key findings": runtime is U-shaped in the block size, and
 * the method uses a smaller block for the first frame and larger ones after;
 * "A complete example": I2V / V2V generation continues a sequence whose
 * first frames are observed).  block_sizes[0 .. n_blocks-1] (HOST array,
 * each >= 1, summing to L) cut the sequence into consecutive blocks; the
 * call inverts blocks b_begin .. b_end-1 (0 <= b_begin < b_end <= n_blocks)
 * with the rules of af_inverse_jacobi (warm start per frame as described
 * there), writing x and iters[s * n_blocks + b] of those blocks only.
 * ws needs af_workspace_bytes(m, batch, L, largest block).  When
 * b_begin > 0, x must already hold the final values of the blocks before
 * b_begin, and ws the K/V of the positions before block b_begin - 1 -- as
 * left by an earlier call on the same ws that ended at b_begin, or by
 * af_prefix_encode of those positions (the first update of block b_begin
 * recomputes block b_begin - 1's K/V from x).  af_last_convergence counts
 * accumulate over calls and restart with a call whose b_begin is 0. */
af_status af_inverse_jacobi_schedule(const af_model* m, const float* z, int batch, int L, af_dir dir,
                                     const int* block_sizes, int n_blocks, int b_begin, int b_end, float tau,
                                     int max_iter, int warm_start, float* x, int32_t* iters, void* ws,
                                     size_t ws_bytes, void* stream);

/* Flow-encode of observed tokens ("A complete example": I2V / V2V -- the
 * flow's forward pass writes the observed frames into the KV cache, no
 * separate encoder): writes the K/V of working-order positions
 * 0 .. n_tokens-1, computed from x, into the cache of a workspace laid out
 * for (batch, L, B) (size af_workspace_bytes(m, batch, L, B)), ready for
 * af_inverse_jacobi_schedule to continue at the block starting at n_tokens
 * (x must then hold the observed tokens too).  Runs passes of at most 2B
 * positions each; writes nothing but the cache and workspace scratch.
 * Requires 1 <= n_tokens <= L. */
af_status af_prefix_encode(const af_model* m, const float* x, int batch, int L, af_dir dir, int B, int n_tokens,
                           void* ws, size_t ws_bytes, void* stream);

/* Streaming generation past the model's length ("A complete example": a
 * sliding window over the deep flow -- after a chunk of latents is
 * produced, f_D is re-run on the last `overlap` latents to rebuild the KV
 * cache, and the next frames are generated).  z, x: [batch, n_frames *
 * frame_len, C], any n_frames; direction L->R, one frame per Jacobi block.
 * Window w covers `window` frames (<= max_frames) starting at frame
 * s_w = w * (window - overlap) (the last window may be shorter); it runs at
 * the model's positions 0 .. window*frame_len - 1.  Its first `overlap`
 * frames (after the first window) are the previous window's output,
 * flow-encoded into the cache (af_prefix_encode); the rest are generated by
 * block-Jacobi (tau, max_iter, warm_start as in af_inverse_jacobi).
 * iters [batch, n_frames] holds each frame's count from the window that
 * generated it.  ws: af_stream_workspace_bytes(m, batch, window) (a
 * window's workspace plus staging of its x and z).  0 <= overlap < window. */
size_t af_stream_workspace_bytes(const af_model* m, int batch, int window);
af_status af_inverse_jacobi_stream(const af_model* m, const float* z, int batch, int n_frames, int window, int overlap,
                                   float tau, int max_iter, int warm_start, float* x, int32_t* iters, void* ws,
                                   size_t ws_bytes, void* stream);

/* Bytes of the shallow-side workspace of flow_pipeline_inverse for T shallow
 * blocks (config of `shallow`), `batch` videos, frames of frame_len tokens,
 * `group` frames per shallow call; 0 on a bad argument. */
size_t flow_pipeline_workspace_bytes(const af_model* shallow, int T, int batch, int frame_len, int group);

/* Pipelined deep -> shallow decoding ("Key design 3": the deep flow
 * f_D runs without pause while the shallow blocks f_S consume its output
 * frame by frame; end-to-end latency is set by the deep block):
 * x = f_S^{-1}(f_D^{-1}(z)) with f_S applied to each frame on its own.
 * f_D^{-1} (`deep`, direction L->R, blocks of B tokens, tau, max_iter_deep,
 * warm_start) runs on stream_deep, one frame's blocks per graph launch.
 * Frames are handed to the shallow side in groups of `group` consecutive
 * frames (the last group may be shorter; 1 <= group <= L / frame_len): when
 * the deep flow has finished a group, an event lets stream_shallow run the
 * T-block stack inverse of the group's frames of every video as one batch of
 * batch * group one-frame samples (blocks shallow[0..T-1], directions
 * shallow_dirs, one Jacobi block per frame, no warm start, tau,
 * max_iter_shallow) while the deep flow moves on.  group 1 hands over every
 * frame at once (the shortest tail after the deep flow ends); larger groups
 * run fewer, larger shallow calls beside it.  z, x: [batch, L, C];
 * frame_len = the deep model's frame_len (the shallow models must accept
 * frames of that length and C); L % frame_len == 0 and frame_len % B == 0.
 * iters_deep [batch, L/B], iters_shallow [T, batch, L/frame_len].  ws_deep:
 * af_workspace_bytes(deep, batch, L, B); ws_shallow:
 * flow_pipeline_workspace_bytes(shallow[0], T, batch, frame_len, group).  The
 * two streams may be the same stream (no overlap).  On return all work is
 * enqueued; stream_deep waits for the last group's shallow work, so
 * synchronising stream_deep covers the whole call.  The result is
 * bit-identical to af_inverse_jacobi followed by flow_stack_inverse of each
 * group's frames as one batch. */
af_status flow_pipeline_inverse(const af_model* deep, const af_model* const* shallow, const af_dir* shallow_dirs, int T,
                                const float* z, int batch, int L, int B, float tau, int max_iter_deep,
                                int max_iter_shallow, int warm_start, int group, float* x, int32_t* iters_deep,
                                int32_t* iters_shallow, void* ws_deep, size_t ws_deep_bytes, void* ws_shallow,
                                size_t ws_shallow_bytes, void* stream_deep, void* stream_shallow);

/* The flow-score-matching denoiser s_phi ("Key design 2": a light causal
 * Transformer trained to regress sigma * grad log p of the flow at the noisy
 * sample, with one frame of look-ahead, s_phi(x_{<=n+1}) ~ (sigma grad log
 * p)_n; it refines the flow's slightly noisy output).  Same af_config and
 * tensor order as af_model_create except the head: W_head [C, d], b_head [C]
 * (plain outputs, no (mu, s) pairs).  Readings (the pages give only "8-layer
 * Transformer, width of the shallow blocks"): the input is x_noisy itself
 * (no shift); h = x W_in^T + b_in + P_space[p mod frame_len] + P_time[p div
 * frame_len]; pre-LN layers as in the AF block, with attention by frames of
 * frame_len tokens -- in the first layer a token of frame n attends every
 * token of frames <= n + 1, in later layers frames <= n -- so frame n's
 * output depends on frames <= n + 1 exactly; final LayerNorm and head give
 * s_phi.  AF_BF16 / AF_FP32 as for the AF block; an AF_BF16 denoiser also
 * needs C % 128 == 0 or C % 192 == 0 (its head has C outputs).  The model
 * can only be used with af_denoise (the flow calls reject it). */
int af_denoiser_num_tensors(const af_config* cfg);
af_status af_denoiser_create(const af_config* cfg, const float* const* tensors, int n_tensors,
                             af_model** out);

/* x = x_noisy + sigma * s_phi(x_noisy) (the Tweedie step with s_phi ~ sigma
 * grad log p), x_noisy and x [batch, L, C], L <= max_len, sigma finite.
 * ws: af_workspace_bytes(m, batch, L, L). */
af_status af_denoise(const af_model* m, const float* x_noisy, int batch, int L, float sigma, float* x, void* ws,
                     size_t ws_bytes, void* stream);

/* af_forward for callers that cannot allocate device memory -- a host that
 * owns the whole GPU memory through its own allocator, or a plugin that is
 * handed only its input and output buffers, and so cannot provide a
 * workspace.  No counterpart in the paper.  Same arguments and
 * results as af_forward minus the workspace: the call runs in a scratch array
 * inside the library, 32 MiB per device, held by every GPU that loads libaf.so
 * until the process exits.  Returns AF_ERR_WORKSPACE (with a message in
 * af_last_error_string) when af_workspace_bytes(m, batch, L, L) exceeds
 * 32 MiB.  The first call on a device looks up the array's address; make it
 * before any stream capture.  Calls share the array: calls whose GPU work
 * overlaps (other streams, other threads) race; serialise them.  Allocates
 * nothing and launches its kernels directly on `stream`. */
af_status af_forward_noalloc(const af_model* m, const float* x, int batch, int L, af_dir dir,
                             float* z, float* logdet, void* stream);

/* Synchronises `stream` and reports how many (sample, block) pairs of the
 * last inverse call on this workspace (of the calls since the last one that
 * started at block 0, for af_inverse_jacobi_schedule) stopped at max_iter
 * without passing the test: AF_OK if none, AF_NOT_CONVERGED otherwise
 * (*n_unconverged set). */
af_status af_last_convergence(void* ws, int* n_unconverged, void* stream);

/* Failure detection: every wait of the tensor-core kernels' pipelines (on a
 * TMA load, an MMA, a buffer hand-off between warps) is bounded.  A wait that
 * runs past `seconds` (default 2) makes its CTA abort: every role stops, the
 * loads and MMAs already in flight are waited for (each with its own 2 s
 * bound), tensor memory is freed, and the model's error word is set for
 * af_device_error.  The results of that call are then undefined; later calls
 * are unaffected.  Applies to calls enqueued after it (graphs captured with
 * another limit are captured anew).  AF_ERR_ARG unless 0 < seconds <= 60.
 * No counterpart in the paper. */
af_status af_set_wait_limit(af_model* m, double seconds);

/* Synchronises the device and returns AF_ERR_DEVICE (and clears the word)
 * if any kernel of this model gave up a bounded wait; *code is a bit mask of
 * where: 1 a GEMM pipeline wait, 4 an attention pipeline wait, 2 a drain
 * after an abort that did not see its in-flight work complete in time. */
af_status af_device_error(const af_model* m, int* code);

const char* af_status_string(af_status s);
const char* af_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* AF_H_ */
