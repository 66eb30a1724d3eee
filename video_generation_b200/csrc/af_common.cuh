// af_common.cuh -- device-side types shared by every kernel of libaf.
//
// Row convention.  One "pass" of an AF block runs its Transformer over a set
// of rows.  Row r belongs to sample s = r / R and sits at sequence position
// p = p0 + r % R of the working order (the order after the direction flip).
// The forward pass uses p0 = 0, R = L.  A Jacobi iteration of block b
// (positions P .. P+B-1) uses p0 = P, R = B, except its first iteration for
// b > 0, which also carries block b-1 (p0 = its first position, R = both
// blocks' tokens) so that block b-1's K/V are recomputed from its final x and
// written to the cache in the same pass (the KV-cache commit of "STARFlow-V
// ... paper notes", key design 3).  Rows at p < P produce no (mu, s) output.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace af {

typedef __nv_bfloat16 bf16;

// Device-resident control block of a call (lives at the head of the workspace).
struct Ctl {
  int P;          // positions < P are final (their K/V are in the cache)
  int p0;         // first position of this pass's rows
  int R;          // rows per sample in this pass
  int M;          // batch * R
  int block;      // Jacobi block index
  int iter;       // updates computed so far in this block
  int n_active;   // samples still iterating in this block
  int nonconv;    // (sample, block) pairs that stopped at max_iter unconverged
  int done;       // CTAs of the current Jacobi step that finished their sample
  int B;          // tokens of the current Jacobi block
};

// Block table of a Jacobi call (in the workspace, written before the call's
// graph runs): the schedule of block sizes as start positions, and the range
// of blocks the call inverts.  Blocks need not be equal ("STARFlow-V ...
// paper notes", key findings: a smaller block for the first frame, larger
// ones later).
enum : int { BT_NB = 0, BT_BEGIN = 1, BT_END = 2, BT_STARTS = 4 };
// btab[BT_NB] = number of blocks nb, btab[BT_BEGIN] / btab[BT_END] = the range
// [begin, end) of blocks this call inverts, btab[BT_STARTS + i] = first
// position of block i (i = 0 .. nb; the last entry is L).
__host__ __device__ inline size_t btab_ints(int L) { return (size_t)BT_STARTS + (size_t)L + 1; }

// Bits OR-ed into the model's device error word: a pipeline wait that ran
// past the limit in a GEMM or in attention, and a drain after an abort that
// did not see its in-flight loads or MMAs complete within its own bound.
enum : int { ERR_NONE = 0, ERR_GEMM_WAIT = 1, ERR_DRAIN = 2, ERR_ATTN_WAIT = 4 };

enum Epi : int {
  EPI_INPROJ = 0,   // h = acc + b_in + pos(p)                          (fp32 h)
  EPI_QKV = 1,      // q / K-cache / V-cache = acc + b_qkv               (act type)
  EPI_RESID = 2,    // h += acc + b                                      (fp32 h)
  EPI_GELU = 3,     // u = gelu(acc + b)                                 (act type)
  EPI_HEAD = 4,     // affine map from interleaved (mu_c, s_c) columns   (fp32 x/z)
  EPI_RAW = 5,      // out32 = acc                                       (fp32 scratch)
  EPI_DENOISE = 6,  // x = x_noisy + sigma * (acc + b), plain columns    (fp32 x)
  EPI_PART = 7      // kpart[split] = acc over the split's k-blocks      (fp32 scratch)
};

// Everything an epilogue may touch.  Pointers not used by a kind stay null.
struct EpiArgs {
  const Ctl* ctl;
  const float* bias;       // [N]
  float* h;                // [Mmax, d] residual stream (fp32)
  void* out;               // EPI_GELU: [Mmax, N];  EPI_QKV: q [Mmax, d]
  float* out32;            // EPI_RAW: [Mmax, ldo]
  int ldo;                 // row stride of `out` (EPI_GELU) and `out32` (EPI_RAW)
  void* kc;                // EPI_QKV: this layer's K cache [batch][Lc][d]
  void* vc;                // EPI_QKV: this layer's V cache [batch][Lc][d]
  int Lc;                  // cache positions per sample
  int d;
  const float* pos_space;  // [frame_len, d]
  const float* pos_time;   // [max_frames, d]
  int frame_len;
  // head
  int head_mode;           // 0 forward (z, logdet partials), 1 Jacobi update, 2 denoise (x + sigma * s)
  float sigma;             // head_mode 2: the noise level
  int L, C, dir;
  const float* xin_f;      // forward: x (read)          inverse: z (read)
  float* xout_f;           // forward: z (write)         inverse: x (read + write)
  const int* active;       // inverse: per-sample flag
  float* part;             // [Mmax, 2C/16, 2] per-(row, 16-column group) partial sums
  uint64_t wait_ns;        // tensor-core kernels: limit of a pipeline wait before the CTA aborts
  int l2_keep;             // TMA outputs (residual adds, GELU) stored with an L2 evict_last policy
  // EPI_PART (split-K of a residual GEMM): at most ksplit splits; split s of a
  // tile stores its partial at rows s * kpart_rows + row of the partial map;
  // the splits used are written to *ks_out for the kernel that sums them (0
  // when one split: the epilogue then adds acc + b into h as EPI_RESID does)
  int ksplit;
  int kpart_rows;
  int* ks_out;
};

__device__ __forceinline__ int tok_of(int p, int L, int dir) { return dir ? (L - 1 - p) : p; }

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

template <typename T> __device__ __forceinline__ T to_act(float v);
template <> __device__ __forceinline__ float to_act<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 to_act<bf16>(float v) { return __float2bfloat16_rn(v); }

template <typename T> __device__ __forceinline__ float from_act(T v);
template <> __device__ __forceinline__ float from_act<float>(float v) { return v; }
template <> __device__ __forceinline__ float from_act<bf16>(bf16 v) { return __bfloat162float(v); }

// Store 4 consecutive values (16-byte aligned destination for float, 8 for bf16).
__device__ __forceinline__ void store4(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(bf16* dst, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = u;
}

// The head epilogue for one row and one 16-column group = 8 channels whose
// (mu_c, s_c) sit at columns (2c, 2c+1).  Forward: z = (x - mu) exp(-s) and the
// group's sum of s.  Inverse: x_new = mu + exp(s) z for active samples, with
// the group's sum of (x_new - x_old)^2 and of x_new^2.
__device__ __forceinline__ void head_group(const EpiArgs& e, int row, int col0, const float* v) {
  const Ctl* ctl = e.ctl;
  const int R = ctl->R;
  const int s = row / R;
  const int p = ctl->p0 + (row - s * R);
  if (e.head_mode == 2) {
    // denoiser: 16 plain channels, out = x_noisy + sigma * (acc + b)
    const size_t base = ((size_t)s * e.L + p) * e.C + col0;
#pragma unroll
    for (int j = 0; j < 16; ++j) e.xout_f[base + j] = fmaf(e.sigma, v[j] + e.bias[col0 + j], e.xin_f[base + j]);
    return;
  }
  if (p < ctl->P) return;                       // commit rows give no output
  const int tok = tok_of(p, e.L, e.dir);
  const int c0 = col0 >> 1;
  const size_t base = ((size_t)s * e.L + tok) * e.C + c0;
  const int G = (2 * e.C) >> 4;
  float* part = e.part + ((size_t)row * G + (col0 >> 4)) * 2;
  if (e.head_mode == 0) {
    float ssum = 0.f;
    float zz[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float mu = v[2 * j] + e.bias[col0 + 2 * j];
      const float sl = v[2 * j + 1] + e.bias[col0 + 2 * j + 1];
      zz[j] = (e.xin_f[base + j] - mu) * expf(-sl);
      ssum += sl;
    }
#pragma unroll
    for (int j = 0; j < 8; j += 4) store4(e.xout_f + base + j, zz[j], zz[j + 1], zz[j + 2], zz[j + 3]);
    part[0] = ssum;
    part[1] = 0.f;
  } else {
    if (!e.active[s]) { part[0] = 0.f; part[1] = 0.f; return; }
    float num = 0.f, den = 0.f;
    float xn[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float mu = v[2 * j] + e.bias[col0 + 2 * j];
      const float sl = v[2 * j + 1] + e.bias[col0 + 2 * j + 1];
      xn[j] = fmaf(expf(sl), e.xin_f[base + j], mu);
      const float dx = xn[j] - e.xout_f[base + j];
      num = fmaf(dx, dx, num);
      den = fmaf(xn[j], xn[j], den);
    }
#pragma unroll
    for (int j = 0; j < 8; j += 4) store4(e.xout_f + base + j, xn[j], xn[j + 1], xn[j + 2], xn[j + 3]);
    part[0] = num;
    part[1] = den;
  }
}

// Apply epilogue kind EPI to 4 consecutive columns col..col+3 of one row.
template <int EPI, typename T>
__device__ __forceinline__ void epi4(const EpiArgs& e, int row, int col, float a0, float a1,
                                     float a2, float a3) {
  if (EPI == EPI_RAW) {
    store4(e.out32 + (size_t)row * e.ldo + col, a0, a1, a2, a3);
    return;
  }
  const float4 b = *reinterpret_cast<const float4*>(e.bias + col);
  a0 += b.x; a1 += b.y; a2 += b.z; a3 += b.w;
  if (EPI == EPI_INPROJ) {
    const Ctl* ctl = e.ctl;
    const int R = ctl->R;
    const int s = row / R;
    const int p = ctl->p0 + (row - s * R);
    const float4 ps = *reinterpret_cast<const float4*>(e.pos_space + (size_t)(p % e.frame_len) * e.d + col);
    const float4 pt = *reinterpret_cast<const float4*>(e.pos_time + (size_t)(p / e.frame_len) * e.d + col);
    store4(e.h + (size_t)row * e.d + col, a0 + ps.x + pt.x, a1 + ps.y + pt.y, a2 + ps.z + pt.z,
           a3 + ps.w + pt.w);
  } else if (EPI == EPI_RESID) {
    float4* hp = reinterpret_cast<float4*>(e.h + (size_t)row * e.d + col);
    float4 hv = *hp;
    hv.x += a0; hv.y += a1; hv.z += a2; hv.w += a3;
    *hp = hv;
  } else if (EPI == EPI_GELU) {
    store4(reinterpret_cast<T*>(e.out) + (size_t)row * e.ldo + col, gelu_erf(a0), gelu_erf(a1),
           gelu_erf(a2), gelu_erf(a3));
  } else if (EPI == EPI_QKV) {
    const int d = e.d;
    if (col < d) {
      store4(reinterpret_cast<T*>(e.out) + (size_t)row * d + col, a0, a1, a2, a3);
    } else {
      const Ctl* ctl = e.ctl;
      const int R = ctl->R;
      const int s = row / R;
      const int p = ctl->p0 + (row - s * R);
      T* dst = reinterpret_cast<T*>(col < 2 * d ? e.kc : e.vc);
      const int cc = col < 2 * d ? col - d : col - 2 * d;
      store4(dst + ((size_t)s * e.Lc + p) * d + cc, a0, a1, a2, a3);
    }
  }
}

// Programmatic dependent launch: every kernel lets its dependents launch as
// soon as all of its CTAs are running, and waits for its predecessors'
// results (griddepcontrol.wait) before reading anything they wrote.  Both are
// no-ops for a kernel launched without a programmatic dependency.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bounded wait helper: true while `t0` + limit_ns has not passed.
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Packed fp32x2 arithmetic of sm_100 (two lanes of one 64-bit register).
__device__ __forceinline__ uint64_t u64_of(float2 v) { return *reinterpret_cast<uint64_t*>(&v); }
__device__ __forceinline__ float2 f2_of(uint64_t v) { return *reinterpret_cast<float2*>(&v); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(u64_of(a)), "l"(u64_of(b)), "l"(u64_of(c)));
  return f2_of(d);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(u64_of(a)), "l"(u64_of(b)));
  return f2_of(d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(u64_of(a)), "l"(u64_of(b)));
  return f2_of(d);
}
__device__ __forceinline__ float2 splat(float a) { return make_float2(a, a); }

}  // namespace af
