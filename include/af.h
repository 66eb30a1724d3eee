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
 *     warm start from the previous block's converged x, stop when
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

/* Workspace bytes for a call on `batch` sequences of L tokens with Jacobi
 * block size B (pass B = L for af_forward).  Includes the KV cache of all
 * layers over L positions.  The same workspace serves every block of a
 * stack made of models with the same config.  0 on bad arguments. */
size_t af_workspace_bytes(const af_model* m, int batch, int L, int B);

/* Forward pass of one AF block: z and logdet (= -sum_{i,c} s_{i,c} per
 * sample) from x.  Requires 1 <= L <= max_len. */
af_status af_forward(const af_model* m, const float* x, int batch, int L, af_dir dir,
                     float* z, float* logdet, void* ws, size_t ws_bytes, void* stream);

/* Block-wise Jacobi inverse of one AF block.  Requires L % B == 0,
 * max_iter >= 1, tau >= 0 and finite.  Block b starts from z_b, or, when
 * warm_start != 0 and b > 0, from block b-1's final x.  A sample leaves the
 * iteration of a block at the first update whose residual is < tau (0/0
 * counts as converged); iters[s * (L/B) + b] counts the updates computed.
 * All iterations, tests and block changes run on the device: one graph
 * launch per call, no host round trip per iteration. */
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
 * last inverse call on this workspace stopped at max_iter without passing
 * the test: AF_OK if none, AF_NOT_CONVERGED otherwise (*n_unconverged set). */
af_status af_last_convergence(void* ws, int* n_unconverged, void* stream);

/* Synchronises the device and returns AF_ERR_DEVICE (and clears the flag)
 * if any kernel of this model gave up a bounded wait; *code says where. */
af_status af_device_error(const af_model* m, int* code);

const char* af_status_string(af_status s);
const char* af_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* AF_H_ */
