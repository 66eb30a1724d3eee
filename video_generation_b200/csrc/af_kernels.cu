// af_kernels.cu -- row-wise kernels, the Jacobi driver kernels and the fp32 SIMT path.
//
// Jacobi driver ("STARFlow-V ... paper notes", key design 3): the inverse of an
// AF block runs as one CUDA graph with two nested device-side WHILE loops.
// The outer loop walks the blocks of B tokens in sequence; the inner loop runs
// Jacobi updates x^(k+1) = mu(x^(k)*m) + sigma(x^(k)*m) * z of the current
// block until every sample's residual ||x^(k+1)-x^(k)||^2 / ||x^(k+1)||^2 is
// below tau or max_iter updates ran.  The kernels below keep the iteration
// counter, the per-sample convergence flags and the loop conditions in device
// memory, so no iteration returns to the host.
#include "af_kernels.h"

namespace af {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Deterministic block sum (fixed shuffle tree, then warps in index order).
__device__ float block_sum(float v) {
  __shared__ float red[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (w == 0) {
    t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_sum(t);
  }
  return t;   // valid in thread 0
}

int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return (int)g;
}

// ------------------------------------------------------------------ control

__global__ void k_ctl_forward(Ctl* ctl, int batch, int L) {
  pdl_trigger();
  pdl_wait();
  ctl->P = 0; ctl->p0 = 0; ctl->R = L; ctl->M = batch * L; ctl->B = L;
  ctl->block = 0; ctl->iter = 0; ctl->n_active = 0;
}

// Block table of a call (af_common.cuh): written in chunks of kTabChunk
// entries from kernel arguments, so that writing it needs no host memory
// copy and can be captured.
struct TabChunk { int v[kTabChunk]; };
__global__ void k_table_write(int* btab, int first, int n, TabChunk ch, int nb, int b_begin, int b_end) {
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < n; i += blockDim.x) btab[BT_STARTS + first + i] = ch.v[i];
  if (threadIdx.x == 0 && first == 0) {
    btab[BT_NB] = nb;
    btab[BT_BEGIN] = b_begin;
    btab[BT_END] = b_end;
  }
}

__global__ void k_set_range(int* btab, int b_begin, int b_end) {
  pdl_trigger();
  pdl_wait();
  btab[BT_BEGIN] = b_begin;
  btab[BT_END] = b_end;
}

// Start of a call's block loop.  The count of unconverged (sample, block)
// pairs restarts with a call whose range starts at block 0 and accumulates
// over calls that continue a sequence.
__global__ void k_call_init(Ctl* ctl, const int* btab, int reset_nonconv) {
  pdl_trigger();
  pdl_wait();
  ctl->block = btab[BT_BEGIN];
  if (reset_nonconv && btab[BT_BEGIN] == 0) ctl->nonconv = 0;
}

// Zero the V rows r0 .. (end of the 64-key tile holding r0 - 1) of every layer
// and sample (bf16 cache): the tensor-core attention reads whole key tiles,
// and although the causal mask gives keys not yet written probability 0,
// 0 * V must be finite.  `vtail` is layer 0's V cache, layer l's is kv_stride
// bytes further; positions are per sample (Lc of them).
__device__ void zero_vtail(bf16* vtail, size_t kv_stride, int layers, int batch, int Lc, int d, int r0) {
  const int r1 = min(((r0 + 63) >> 6) << 6, Lc);
  if (r1 <= r0) return;
  const int dv = d >> 3;                                   // 16-byte units per row
  const long long nz = (long long)layers * batch * (r1 - r0) * dv;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nz;
       i += (long long)gridDim.x * blockDim.x) {
    const int u = (int)(i % dv);
    long long rest = i / dv;
    const int r = r0 + (int)(rest % (r1 - r0));
    rest /= (r1 - r0);
    const int s = (int)(rest % batch);
    const int l = (int)(rest / batch);
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<char*>(vtail) + (size_t)l * kv_stride +
                                          (((size_t)s * Lc + r) * d) * sizeof(bf16)) + u;
    *dst = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Start of Jacobi block b = ctl->block (positions P .. Q-1 of the table):
// the row layout of the first update (block b-1 rides along to commit its
// K/V), fresh per-sample flags, and the starting guess: z, or with warm start
// the previous frame's converged state ("STARFlow-V ... paper notes", key
// design 3) -- position p takes the converged x of p - k*F, the same spatial
// position in the most recent finished frame (smallest k >= 1 with
// p - k*F < P), or z where no frame before it has finished.  With a bf16
// cache (vtail != null) it also zeroes the masked V tail (zero_vtail) past Q.
__global__ void k_block_init(Ctl* ctl, const int* btab, int* active, const float* __restrict__ z, float* x,
                             int batch, int L, int C, int F, int dir, int warm, bf16* vtail, size_t kv_stride,
                             int layers, int d, cudaGraphConditionalHandle inner) {
  pdl_trigger();
  pdl_wait();
  const int b = ctl->block;
  const int P = btab[BT_STARTS + b], Q = btab[BT_STARTS + b + 1];
  const int B = Q - P;
  const int nvec = C >> 2;
  const long long n = (long long)batch * B * nvec;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int cv = (int)(i % nvec);
    const long long st = i / nvec;
    const int t = (int)(st % B);
    const int s = (int)(st / B);
    const int p = P + t;
    const size_t dst = ((size_t)s * L + tok_of(p, L, dir)) * C + cv * 4;
    const int src = p - (t / F + 1) * F;
    float4 v;
    if (warm && src >= 0)
      v = *reinterpret_cast<const float4*>(x + ((size_t)s * L + tok_of(src, L, dir)) * C + cv * 4);
    else
      v = *reinterpret_cast<const float4*>(z + dst);
    *reinterpret_cast<float4*>(x + dst) = v;
  }
  if (vtail) zero_vtail(vtail, kv_stride, layers, batch, L, d, Q);
  if (blockIdx.x == 0) {
    for (int s = threadIdx.x; s < batch; s += blockDim.x) active[s] = 1;
    if (threadIdx.x == 0) {
      const int p0 = b > 0 ? btab[BT_STARTS + b - 1] : P;
      ctl->P = P;
      ctl->B = B;
      ctl->p0 = p0;
      ctl->R = Q - p0;
      ctl->M = batch * (Q - p0);
      ctl->iter = 0;
      ctl->n_active = batch;
      ctl->done = 0;
      cudaGraphSetConditional(inner, 1u);
    }
  }
}

// End of one Jacobi update: per-sample residual from the head's partial sums
// (one CTA per sample, fixed summation order), the stopping test, the
// iteration counters; the last CTA to finish sets the inner loop condition.
__global__ void __launch_bounds__(512) k_jacobi_step(Ctl* ctl, const int* btab, int* active,
                                                     const float* __restrict__ part, int batch, int G, float tau,
                                                     int max_iter, int32_t* iters,
                                                     cudaGraphConditionalHandle inner) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_last;
  const int s = blockIdx.x;
  const int R = ctl->R, p0 = ctl->p0, P = ctl->P, B = ctl->B, iter = ctl->iter, blk = ctl->block;
  const int nblocks = btab[BT_NB];
  if (active[s]) {                                     // uniform over the CTA
    const float2* p = reinterpret_cast<const float2*>(part + ((size_t)s * R + (P - p0)) * G * 2);
    const int n = B * G;
    float num = 0.f, den = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const float2 v = p[i];
      num += v.x;
      den += v.y;
    }
    num = block_sum(num);
    den = block_sum(den);
    if (threadIdx.x == 0) {
      iters[(size_t)s * nblocks + blk] = iter + 1;
      const bool conv = (den == 0.f) ? (num == 0.f) : (num / den < tau);
      if (conv) active[s] = 0;
    }
  }
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&ctl->done, 1) == batch - 1;
  }
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    __threadfence();
    int na = 0;
    for (int i = 0; i < batch; ++i) na += *((volatile int*)active + i);
    ctl->done = 0;
    ctl->iter = iter + 1;
    ctl->n_active = na;
    const bool cont = na > 0 && iter + 1 < max_iter;
    if (!cont) ctl->nonconv += na;
    ctl->p0 = P;
    ctl->R = B;
    ctl->M = batch * B;
    cudaGraphSetConditional(inner, cont ? 1u : 0u);
  }
}

__global__ void k_block_advance(Ctl* ctl, const int* btab, cudaGraphConditionalHandle outer) {
  pdl_trigger();
  pdl_wait();
  const int b = ctl->block + 1;
  ctl->block = b;
  cudaGraphSetConditional(outer, b < btab[BT_END] ? 1u : 0u);
}

// A pass over positions p0 .. p0+R-1 of every sample whose rows give no head
// output (P = p0 + R): the flow-encode of observed tokens into the KV cache.
// Zeroes the masked V tail past the pass, like a block init.
__global__ void k_set_pass(Ctl* ctl, int p0, int R, int batch, bf16* vtail, size_t kv_stride, int layers, int Lc,
                           int d) {
  pdl_trigger();
  pdl_wait();
  if (vtail) zero_vtail(vtail, kv_stride, layers, batch, Lc, d, p0 + R);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    ctl->P = p0 + R;
    ctl->p0 = p0;
    ctl->R = R;
    ctl->M = batch * R;
    ctl->B = R;
  }
}

// ------------------------------------------------------------------ row-wise

// Self-exclusive mask as a one-token shift: the input of position p is
// x_{p-1} (zero at p = 0), read through the direction flip; without the shift
// (the denoiser) the input of p is x_p.
template <typename T>
__global__ void k_gather(const Ctl* ctl, const float* __restrict__ x, int L, int C, int dir, int shift, T* xin) {
  pdl_trigger();
  pdl_wait();
  const int M = ctl->M, R = ctl->R, p0 = ctl->p0;
  const int nvec = C >> 2;
  const long long n = (long long)M * nvec;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(i / nvec);
    const int c = (int)(i - (long long)row * nvec) * 4;
    const int s = row / R;
    const int p = p0 + (row - s * R);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p >= shift) v = *reinterpret_cast<const float4*>(x + ((size_t)s * L + tok_of(p - shift, L, dir)) * C + c);
    store4(xin + (size_t)row * C + c, v.x, v.y, v.z, v.w);
  }
}

// LayerNorm (eps 1e-5), one warp per two rows, fp32 statistics (two passes
// over registers: mean, then the centred variance).  NV = d / 128 float4 per
// lane and row; both rows' loads are issued before any arithmetic.
template <typename T, int NV>
__global__ void __launch_bounds__(256) k_layernorm_reg(const Ctl* ctl, const float* __restrict__ h,
                                                       const float* __restrict__ g, const float* __restrict__ b,
                                                       T* out, int d) {
  pdl_trigger();
  pdl_wait();
  const int wg = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int M = ctl->M;
  const int r0 = 2 * wg;
  if (r0 >= M) return;
  const bool two = r0 + 1 < M;
  float4 v[2][NV];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float4* hr = reinterpret_cast<const float4*>(h + (size_t)(two ? r0 + k : r0) * d);
#pragma unroll
    for (int i = 0; i < NV; ++i) v[k][i] = hr[lane + 32 * i];
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (k == 1 && !two) break;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) sum += (v[k][i].x + v[k][i].y) + (v[k][i].z + v[k][i].w);
    const float mean = warp_sum(sum) / d;
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float a = v[k][i].x - mean, bb = v[k][i].y - mean, c = v[k][i].z - mean, e = v[k][i].w - mean;
      sq += (a * a + bb * bb) + (c * c + e * e);
    }
    const float rstd = 1.0f / sqrtf(warp_sum(sq) / d + 1e-5f);
    T* orow = out + (size_t)(r0 + k) * d;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = (lane + 32 * i) * 4;
      const float4 gg = *reinterpret_cast<const float4*>(g + c);
      const float4 bv = *reinterpret_cast<const float4*>(b + c);
      store4(orow + c, (v[k][i].x - mean) * rstd * gg.x + bv.x, (v[k][i].y - mean) * rstd * gg.y + bv.y,
             (v[k][i].z - mean) * rstd * gg.z + bv.z, (v[k][i].w - mean) * rstd * gg.w + bv.w);
    }
  }
}

// Split-K sum of a residual GEMM: h += bias + part[0] + part[1] + ... in split
// order (deterministic), float4 per thread, grid-stride over the live rows.
__global__ void __launch_bounds__(256) k_split_sum(const Ctl* ctl, const float* __restrict__ part, int rows, int N,
                                                   const int* __restrict__ ks_ptr, const float* __restrict__ bias,
                                                   float* h) {
  pdl_trigger();
  pdl_wait();
  const int M = ctl->M, ks = *ks_ptr, n4 = N / 4;
  if (ks == 0) return;                                  // the GEMM added into h itself
  const long long total = (long long)M * n4;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / n4), c = (int)(i - (long long)r * n4);
    // every load issued before the first add (at most 4 splits, the host's
    // cap; the absent ones add +0)
    float4* hp = reinterpret_cast<float4*>(h + (size_t)r * N) + c;
    float4 p[4];
#pragma unroll
    for (int sp = 0; sp < 4; ++sp)
      p[sp] = sp < ks ? __ldcg(reinterpret_cast<const float4*>(part + ((size_t)sp * rows + r) * N) + c)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 v = reinterpret_cast<const float4*>(bias)[c];
    float4 o = *hp;
#pragma unroll
    for (int sp = 0; sp < 4; ++sp) {
      v.x += p[sp].x; v.y += p[sp].y; v.z += p[sp].z; v.w += p[sp].w;
    }
    o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
    *hp = o;
  }
}

template <typename T>
__global__ void k_layernorm_gen(const Ctl* ctl, const float* __restrict__ h, const float* __restrict__ g,
                                const float* __restrict__ b, T* out, int d) {
  pdl_trigger();
  pdl_wait();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (row >= ctl->M) return;
  const float* hr = h + (size_t)row * d;
  float sum = 0.f;
  for (int c = lane; c < d; c += 32) sum += hr[c];
  const float mean = warp_sum(sum) / d;
  float sq = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float a = hr[c] - mean;
    sq += a * a;
  }
  const float rstd = 1.0f / sqrtf(warp_sum(sq) / d + 1e-5f);
  for (int c = lane; c < d; c += 32) out[(size_t)row * d + c] = to_act<T>((hr[c] - mean) * rstd * g[c] + b[c]);
}

// logdet[s] = -sum of s over the sample's rows and head groups (fixed order).
__global__ void __launch_bounds__(512) k_logdet_finalize(const float* __restrict__ part, int L, int G,
                                                         float* logdet, int accumulate) {
  pdl_trigger();
  pdl_wait();
  const int s = blockIdx.x;
  const float4* p = reinterpret_cast<const float4*>(part + (size_t)s * L * G * 2);
  const int n = L * G / 2;                     // float4 = two (sum, unused) pairs
  float acc = 0.f;
#pragma unroll 4
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float4 v = p[i];
    acc += v.x + v.z;
  }
  if ((L * G) & 1) {
    if (threadIdx.x == 0) acc += part[((size_t)s * L * G + L * G - 1) * 2];
  }
  acc = block_sum(acc);
  if (threadIdx.x == 0) logdet[s] = accumulate ? logdet[s] - acc : -acc;
}

// ------------------------------------------------------------------ fp32 SIMT path

// C = A W^T, 64x64 tile, BK 16, 256 threads of 4x4 outputs.
template <int EPI>
__global__ void __launch_bounds__(256) k_gemm_simt(const float* __restrict__ A, const float* __restrict__ W,
                                                   int N, int K, EpiArgs e) {
  pdl_trigger();
  pdl_wait();
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int M = e.ctl->M;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (m0 >= M) return;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = tid; i < 64 * 16; i += 256) {
      const int r = i >> 4, k = i & 15;
      As[k][r] = (m0 + r < M && k0 + k < K) ? A[(size_t)(m0 + r) * K + k0 + k] : 0.f;
      Ws[k][r] = (n0 + r < N && k0 + k < K) ? W[(size_t)(n0 + r) * K + k0 + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[k][ty * 4 + i]; w[i] = Ws[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int col = n0 + tx * 4;
  if (col >= N) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty * 4 + i;
    if (row < M) epi4<EPI, float>(e, row, col, acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
  }
}

// Head in fp32: one thread per (row, 16-column group), then the shared affine epilogue.
__global__ void k_head_simt(const float* __restrict__ A, const float* __restrict__ W, int N, int K, EpiArgs e) {
  pdl_trigger();
  pdl_wait();
  const int G = N >> 4;
  const int M = e.ctl->M;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * G) return;
  const int row = i / G, g = i - row * G;
  const float* a = A + (size_t)row * K;
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float* w = W + (size_t)(g * 16 + j) * K;
    float s = 0.f;
    for (int k = 0; k < K; ++k) s = fmaf(a[k], w[k], s);
    v[j] = s;
  }
  head_group(e, row, g * 16, v);
}

// Causal attention in fp32: one warp per (row, head); lanes take keys
// j = lane, lane+32, ... <= p with a running max / sum, merged at the end.
template <int HD>
__global__ void __launch_bounds__(256) k_attn_simt(const Ctl* ctl, const float* __restrict__ q,
                                                   const float* __restrict__ kc, const float* __restrict__ vc,
                                                   float* o, int Lc, int d, int heads, int mF, int ahead) {
  pdl_trigger();
  pdl_wait();
  __shared__ float qs[8][HD];
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * 8 + wib;
  const int M = ctl->M;
  if (gw >= M * heads) return;
  const int row = gw / heads, hh = gw - row * heads;
  const int R = ctl->R, s = row / R, p = ctl->p0 + (row - s * R);
  const float scale = 1.0f / sqrtf((float)HD);
  for (int i = lane; i < HD; i += 32) qs[wib][i] = q[(size_t)row * d + hh * HD + i];
  __syncwarp();
  const float* K = kc + (size_t)s * Lc * d + hh * HD;
  const float* V = vc + (size_t)s * Lc * d + hh * HD;
  float m = -INFINITY, l = 0.f, acc[HD];
#pragma unroll
  for (int i = 0; i < HD; ++i) acc[i] = 0.f;
  int last = p;                                         // the row's last key (mask, see af_kernels.h)
  if (mF) last = min((p / mF + 1 + ahead) * mF, Lc) - 1;
  for (int j = lane; j <= last; j += 32) {
    float sc = 0.f;
#pragma unroll
    for (int i = 0; i < HD; ++i) sc = fmaf(qs[wib][i], K[(size_t)j * d + i], sc);
    sc *= scale;
    const float mn = fmaxf(m, sc);
    const float corr = expf(m - mn), pj = expf(sc - mn);
    l = l * corr + pj;
#pragma unroll
    for (int i = 0; i < HD; ++i) acc[i] = fmaf(pj, V[(size_t)j * d + i], acc[i] * corr);
    m = mn;
  }
  const float mx = warp_max(m);
  const float f = (m == -INFINITY) ? 0.f : expf(m - mx);
  const float lt = warp_sum(l * f);
#pragma unroll
  for (int i = 0; i < HD; ++i) {
    const float a = warp_sum(acc[i] * f);
    if (lane == (i & 31)) o[(size_t)row * d + hh * HD + i] = a / lt;
  }
}

}  // namespace

// ------------------------------------------------------------------ launchers

void launch_ctl_forward(Ctl* ctl, int batch, int L, cudaStream_t st) {
  launch_k(k_ctl_forward, dim3(1), dim3(1), 0, st, ctl, batch, L);
}
void launch_call_init(Ctl* ctl, const int* btab, int reset_nonconv, cudaStream_t st) {
  launch_k(k_call_init, dim3(1), dim3(1), 0, st, ctl, btab, reset_nonconv);
}

void launch_table_write(int* btab, const int* starts, int nb, int b_begin, int b_end, cudaStream_t st) {
  for (int first = 0; first <= nb; first += kTabChunk) {
    TabChunk ch;
    const int n = (nb + 1 - first) < kTabChunk ? (nb + 1 - first) : kTabChunk;
    for (int i = 0; i < n; ++i) ch.v[i] = starts[first + i];
    launch_k(k_table_write, dim3(1), dim3(256), 0, st, btab, first, n, ch, nb, b_begin, b_end);
  }
}

void launch_set_range(int* btab, int b_begin, int b_end, cudaStream_t st) {
  launch_k(k_set_range, dim3(1), dim3(1), 0, st, btab, b_begin, b_end);
}

void launch_set_pass(Ctl* ctl, int p0, int R, int batch, bf16* vtail, size_t kv_stride, int layers, int Lc, int d,
                     cudaStream_t st) {
  const long long work = vtail ? (long long)layers * batch * 64 * (d / 8) : 1;
  launch_k(k_set_pass, dim3(grid_for(work, kThreads)), dim3(kThreads), 0, st, ctl, p0, R, batch, vtail, kv_stride,
           layers, Lc, d);
}

template <typename T>
void launch_gather(const Ctl* ctl, const float* x, int L, int C, int dir, int shift, T* xin, int m_max,
                   cudaStream_t st) {
  launch_k(k_gather<T>, dim3(grid_for((long long)m_max * (C / 4), kThreads)), dim3(kThreads), 0, st, ctl, x, L, C, dir,
           shift, xin);
}
template void launch_gather<float>(const Ctl*, const float*, int, int, int, int, float*, int, cudaStream_t);
template void launch_gather<bf16>(const Ctl*, const float*, int, int, int, int, bf16*, int, cudaStream_t);

template <typename T>
void launch_layernorm(const Ctl* ctl, const float* h, const float* g, const float* b, T* out, int d,
                      int m_max, cudaStream_t st) {
  const int grid = (m_max + 7) / 8, grid2 = (m_max + 15) / 16;
  switch (d % 128 == 0 ? d / 128 : 0) {
    case 2: launch_k(k_layernorm_reg<T, 2>, dim3(grid2), dim3(256), 0, st, ctl, h, g, b, out, d); break;
    case 4: launch_k(k_layernorm_reg<T, 4>, dim3(grid2), dim3(256), 0, st, ctl, h, g, b, out, d); break;
    case 6: launch_k(k_layernorm_reg<T, 6>, dim3(grid2), dim3(256), 0, st, ctl, h, g, b, out, d); break;
    case 8: launch_k(k_layernorm_reg<T, 8>, dim3(grid2), dim3(256), 0, st, ctl, h, g, b, out, d); break;
    case 16: launch_k(k_layernorm_reg<T, 16>, dim3(grid2), dim3(256), 0, st, ctl, h, g, b, out, d); break;
    default: launch_k(k_layernorm_gen<T>, dim3(grid), dim3(256), 0, st, ctl, h, g, b, out, d); break;
  }
}
template void launch_layernorm<float>(const Ctl*, const float*, const float*, const float*, float*, int, int, cudaStream_t);
template void launch_layernorm<bf16>(const Ctl*, const float*, const float*, const float*, bf16*, int, int, cudaStream_t);

void launch_split_sum(const Ctl* ctl, const float* part, int rows, int N, const int* ks, const float* bias, float* h,
                      int m_max, cudaStream_t st) {
  const long long work = (long long)m_max * (N / 4);
  long long blocks = (work + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  launch_k(k_split_sum, dim3((unsigned)blocks), dim3(256), 0, st, ctl, part, rows, N, ks, bias, h);
}

void launch_logdet_finalize(const float* part, int batch, int L, int G, float* logdet, int accumulate,
                            cudaStream_t st) {
  launch_k(k_logdet_finalize, dim3(batch), dim3(512), 0, st, part, L, G, logdet, accumulate);
}

void launch_block_init(Ctl* ctl, const int* btab, int* active, const float* z, float* x, int batch, int L, int C,
                       int B_max, int F, int dir, int warm, bf16* vtail, size_t kv_stride, int layers, int d,
                       cudaGraphConditionalHandle inner, cudaStream_t st) {
  const long long work = (long long)batch * B_max * (C / 4) + (vtail ? (long long)layers * batch * 64 * (d / 8) : 0);
  launch_k(k_block_init, dim3(grid_for(work, kThreads)), dim3(kThreads), 0, st, ctl, btab, active, z, x, batch, L,
           C, F, dir, warm, vtail, kv_stride, layers, d, inner);
}

void launch_jacobi_step(Ctl* ctl, const int* btab, int* active, const float* part, int batch, int G, float tau,
                        int max_iter, int32_t* iters, cudaGraphConditionalHandle inner, cudaStream_t st) {
  launch_k(k_jacobi_step, dim3(batch), dim3(512), 0, st, ctl, btab, active, part, batch, G, tau, max_iter, iters,
           inner);
}

void launch_block_advance(Ctl* ctl, const int* btab, cudaGraphConditionalHandle outer, cudaStream_t st) {
  launch_k(k_block_advance, dim3(1), dim3(1), 0, st, ctl, btab, outer);
}

void launch_gemm_simt(int epi, const float* A, const float* W, int N, int K, int m_max, const EpiArgs& e,
                      cudaStream_t st) {
  dim3 grid((N + 63) / 64, (m_max + 63) / 64);
  switch (epi) {
    case EPI_INPROJ: launch_k(k_gemm_simt<EPI_INPROJ>, dim3(grid), dim3(256), 0, st, A, W, N, K, e); break;
    case EPI_QKV: launch_k(k_gemm_simt<EPI_QKV>, dim3(grid), dim3(256), 0, st, A, W, N, K, e); break;
    case EPI_RESID: launch_k(k_gemm_simt<EPI_RESID>, dim3(grid), dim3(256), 0, st, A, W, N, K, e); break;
    case EPI_GELU: launch_k(k_gemm_simt<EPI_GELU>, dim3(grid), dim3(256), 0, st, A, W, N, K, e); break;
    default: launch_k(k_gemm_simt<EPI_RAW>, dim3(grid), dim3(256), 0, st, A, W, N, K, e); break;
  }
}

void launch_head_simt(const float* A, const float* W, int N, int K, int m_max, const EpiArgs& e,
                      cudaStream_t st) {
  const long long n = (long long)m_max * (N / 16);
  launch_k(k_head_simt, dim3((int)((n + 127) / 128)), dim3(128), 0, st, A, W, N, K, e);
}

void launch_attn_simt(const Ctl* ctl, const float* q, const float* kc, const float* vc, float* o, int batch,
                      int Lc, int d, int heads, int m_max, int mask_frame, int mask_ahead, cudaStream_t st) {
  (void)batch;
  const int grid = (int)(((long long)m_max * heads + 7) / 8);
  const int F = mask_frame, A = mask_ahead;
  switch (d / heads) {
    case 16: launch_k(k_attn_simt<16>, dim3(grid), dim3(256), 0, st, ctl, q, kc, vc, o, Lc, d, heads, F, A); break;
    case 32: launch_k(k_attn_simt<32>, dim3(grid), dim3(256), 0, st, ctl, q, kc, vc, o, Lc, d, heads, F, A); break;
    case 64: launch_k(k_attn_simt<64>, dim3(grid), dim3(256), 0, st, ctl, q, kc, vc, o, Lc, d, heads, F, A); break;
    default: launch_k(k_attn_simt<128>, dim3(grid), dim3(256), 0, st, ctl, q, kc, vc, o, Lc, d, heads, F, A); break;
  }
}

}  // namespace af
