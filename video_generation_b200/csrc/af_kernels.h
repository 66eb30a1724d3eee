// af_kernels.h -- host-side launchers of libaf's kernels (internal, C++ linkage).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include "af_common.cuh"

namespace af {

// Launches with programmatic stream serialization when g_pdl is set, so that
// a kernel's launch and set-up overlap the tail of the kernel before it.  The
// calling thread sets it from its model before enqueueing (each model keeps
// its own setting: on by default, AF_PDL=0 in the environment turns it off,
// and a model whose capture refused programmatic edges turns it off for
// itself).
extern thread_local int g_pdl;
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
  cudaLaunchConfig_t c = {};
  c.gridDim = grid;
  c.blockDim = block;
  c.dynamicSmemBytes = smem;
  c.stream = st;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[0].val.programmaticStreamSerializationAllowed = g_pdl;
  c.attrs = a;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, kern, static_cast<KArgs>(args)...);
}

// ---- small kernels (af_kernels.cu) -----------------------------------------
// All row-wise kernels read the live row count from ctl->M and are launched
// for `m_max` rows.
void launch_ctl_forward(Ctl* ctl, int batch, int L, cudaStream_t st);
// shift = 1: the input of position p is x_{p-1} (zero at p = 0), the
// self-exclusive mask of an AF block; shift = 0: x_p itself (the denoiser).
template <typename T>
void launch_gather(const Ctl* ctl, const float* x, int L, int C, int dir, int shift, T* xin, int m_max,
                   cudaStream_t st);
template <typename T>
void launch_layernorm(const Ctl* ctl, const float* h, const float* g, const float* b, T* out,
                      int d, int m_max, cudaStream_t st);
void launch_logdet_finalize(const float* part, int batch, int L, int G, float* logdet,
                            int accumulate, cudaStream_t st);
// Jacobi driver (af_kernels.cu).  The block table (af_common.cuh) is written
// from kernel arguments in chunks of kTabChunk start positions.
constexpr int kTabChunk = 1000;
void launch_table_write(int* btab, const int* starts, int nb, int b_begin, int b_end, cudaStream_t st);
void launch_set_range(int* btab, int b_begin, int b_end, cudaStream_t st);
void launch_call_init(Ctl* ctl, const int* btab, int reset_nonconv, cudaStream_t st);
// vtail: layer 0's V cache (bf16 path) whose masked tail rows the block's
// attention reads, layer l's at kv_stride bytes further; null for fp32.
// B_max: the largest block of the table (sizes the grid); F: frame length.
void launch_block_init(Ctl* ctl, const int* btab, int* active, const float* z, float* x, int batch, int L, int C,
                       int B_max, int F, int dir, int warm, bf16* vtail, size_t kv_stride, int layers, int d,
                       cudaGraphConditionalHandle inner, cudaStream_t st);
void launch_jacobi_step(Ctl* ctl, const int* btab, int* active, const float* part, int batch, int G, float tau,
                        int max_iter, int32_t* iters, cudaGraphConditionalHandle inner, cudaStream_t st);
void launch_block_advance(Ctl* ctl, const int* btab, cudaGraphConditionalHandle outer, cudaStream_t st);
// Row layout of a pass over positions p0 .. p0+R-1 with no head output
// (flow-encode into the cache), zeroing the masked V tail past it.
void launch_set_pass(Ctl* ctl, int p0, int R, int batch, bf16* vtail, size_t kv_stride, int layers, int Lc, int d,
                     cudaStream_t st);

// ---- fp32 SIMT path (af_kernels.cu) -----------------------------------------
void launch_gemm_simt(int epi, const float* A, const float* W, int N, int K, int m_max,
                      const EpiArgs& e, cudaStream_t st);
void launch_head_simt(const float* A, const float* W, int N, int K, int m_max, const EpiArgs& e,
                      cudaStream_t st);
// Attention masks (both paths): token-causal when mask_frame is 0, else by
// frames of mask_frame tokens with mask_ahead frames of look-ahead.
void launch_attn_simt(const Ctl* ctl, const float* q, const float* kc, const float* vc, float* o,
                      int batch, int Lc, int d, int heads, int m_max, int mask_frame, int mask_ahead,
                      cudaStream_t st);

// ---- tensor-core bf16 path ---------------------------------------------------
// TMA descriptor of a row-major bf16 matrix [rows, cols] tiled as boxes of
// [box_rows, 64 columns] with 128-byte swizzle (af_gemm_tc.cu).
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int box_rows);
// TMA descriptor of the output of a TMA epilogue: fp32 h or bf16 u [rows, cols]
// in boxes of 32 rows x 16 columns, 64-byte (fp32) or 32-byte (bf16) swizzle.
bool make_tmap_out(CUtensorMap* map, const void* base, bool f32, int rows, int cols);
// C[M, N] = A[M, K] W[N, K]^T with epilogue `epi`, K % 64 == 0.  `pick` =
// BN * 10 + CG from gemm_tc_pick (N % BN == 0); tmA boxes are 128 rows, tmB
// boxes BN / CG rows; tmC (make_tmap_out) is the output of EPI_RESID (h),
// EPI_PART (the split-K partials, ksplit * kpart_rows rows), EPI_GELU (u) and
// EPI_QKV (q), tmC2 / tmC3 the K / V cache of EPI_QKV ([batch * Lc, d]); tmC2
// is h for EPI_PART (added into directly when the pass's tiles leave no room
// for a second split); unused ones may be null.
void launch_gemm_tc(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap* tmC,
                    const CUtensorMap* tmC2, const CUtensorMap* tmC3, int pick, int N, int K, int m_max,
                    const EpiArgs& e, int* err, int num_sms, cudaStream_t st);
int gemm_tc_pick(int N, int m_max, int num_sms, int unit, int max_bn);
// tiles of a GEMM with tile shape `pick` (gemm_tc_pick) over m_rows rows
int gemm_tc_tiles(int pick, int N, int m_rows);
// h[r, :] += bias + sum over s < *ks of part[s * rows + r, :] for r < ctl->M
// (the split-K partials of a residual GEMM, summed in split order); nothing
// when *ks is 0 (the GEMM ran unsplit and added into h itself)
void launch_split_sum(const Ctl* ctl, const float* part, int rows, int N, const int* ks, const float* bias, float* h,
                      int m_max, cudaStream_t st);

// Causal attention over the KV cache on tcgen05 (af_attn_tc.cu).  Each pass
// splits its live key range into at most nsplit_max splits (attn_tc_splits
// gives the most a call on a cache of Lc positions can use); with
// nsplit_max > 1, opart [nsplit_max, m_max, d] and mlpart [nsplit_max, m_max,
// heads, 2] hold the partials.  False if a tensor map cannot be encoded.
int attn_tc_splits(int batch, int heads, int r_max, int Lc, int num_sms);
bool launch_attn_tc2(const Ctl* ctl, const bf16* q, const bf16* kc, const bf16* vc, bf16* o, float* opart,
                     float* mlpart, int nsplit_max, int batch, int Lc, int d, int heads, int r_max, int m_max,
                     int num_sms, uint64_t wait_ns, int mask_frame, int mask_ahead, int l2_keep, int* err,
                     cudaStream_t st);

}  // namespace af
