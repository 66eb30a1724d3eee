// af_attn.cu -- causal multi-head attention over the KV cache, bf16 operands,
// fp32 softmax statistics and accumulation.
//
// Query row r of sample s sits at position p = p0 + r % R and attends keys
// 0..p of the sample's cache (the cache already holds this pass's own K/V,
// written by the QKV GEMM epilogue), i.e. softmax(q k^T / sqrt(hd), j <= p) v:
// the finished blocks of the block-wise Jacobi schedule ("STARFlow-V ... paper
// notes", key design 3) are read from the cache, the rows of the current block
// causally among themselves.
//
// One CTA = 4 warps = 64 query rows of one (sample, head); key tiles of 64
// stream through shared memory (cp.async, double buffered, XOR-swizzled rows)
// and only tiles at or below the CTA's last query position are visited.
#include "af_kernels.h"

namespace af {
namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0 source bytes: the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled [rows][HD] bf16 tile.
template <int HD> __device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * HD * 2 + ((c ^ (r & 7)) << 4));
}

template <int HD>
__global__ void __launch_bounds__(128) k_attn_mma(const Ctl* ctl, const bf16* __restrict__ q,
                                                  const bf16* __restrict__ kc, const bf16* __restrict__ vc,
                                                  bf16* __restrict__ o, int Lc, int d) {
  constexpr int CH = HD / 8;                 // 16-byte chunks per row
  constexpr int TILE_BYTES = 64 * HD * 2;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TILE_BYTES;             // 2 buffers
  uint8_t* sV = sm + 3 * TILE_BYTES;         // 2 buffers

  const int R = ctl->R, p0 = ctl->p0;
  const int qt = blockIdx.x, hh = blockIdx.y, s = blockIdx.z;
  const int r_begin = qt * 64;
  if (r_begin >= R) return;
  const int r_end = min(r_begin + 64, R);
  const int kmax = p0 + r_end - 1;           // last key any row of this CTA may see
  const int nkt = kmax / 64 + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bf16* qbase = q + (size_t)s * R * d + hh * HD;
  const bf16* kbase = kc + (size_t)s * Lc * d + hh * HD;
  const bf16* vbase = vc + (size_t)s * Lc * d + hh * HD;

  // Q tile (rows beyond R zero-filled)
  for (int i = tid; i < 64 * CH; i += 128) {
    const int r = i / CH, c = i % CH;
    const bool ok = r_begin + r < R;
    cp_async16(smem_u32(sQ + swz<HD>(r, c)), qbase + (size_t)(ok ? r_begin + r : 0) * d + c * 8, ok);
  }
  auto load_kv = [&](int kt, int buf) {
    for (int i = tid; i < 64 * CH; i += 128) {
      const int r = i / CH, c = i % CH;
      const int j = kt * 64 + r;
      const bool ok = j <= kmax;
      const size_t off = (size_t)(ok ? j : 0) * d + c * 8;
      cp_async16(smem_u32(sK + buf * TILE_BYTES + swz<HD>(r, c)), kbase + off, ok);
      cp_async16(smem_u32(sV + buf * TILE_BYTES + swz<HD>(r, c)), vbase + off, ok);
    }
  };
  load_kv(0, 0);
  cp_commit();

  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);   // log2(e) / sqrt(hd)
  const int qrow0 = warp * 16 + (lane >> 2);                  // tile-local rows qrow0, qrow0 + 8
  const int qpos0 = p0 + r_begin + qrow0, qpos1 = qpos0 + 8;

  uint32_t qa[HD / 16][4];
  float oacc[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) load_kv(kt + 1, buf ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = kk * 2 + (lane >> 4);
        ldsm_x4(smem_u32(sQ + swz<HD>(r, c)), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    const uint8_t* tK = sK + buf * TILE_BYTES;
    const uint8_t* tV = sV + buf * TILE_BYTES;
    // S = Q K^T for this warp's 16 rows and the tile's 64 keys
    float sacc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int c = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(tK + swz<HD>(r, c)), b0, b1, b2, b3);
        mma16816(sacc[2 * np], qa[kk], b0, b1);
        mma16816(sacc[2 * np + 1], qa[kk], b2, b3);
      }
    }
    // causal mask on tiles that reach past the CTA's first query position
    const bool need_mask = kt * 64 + 63 > p0 + r_begin;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = kt * 64 + n * 8 + (lane & 3) * 2 + e;
        float v0 = sacc[n][e] * sl2, v1 = sacc[n][2 + e] * sl2;
        if (need_mask) {
          if (j > qpos0) v0 = -INFINITY;
          if (j > qpos1) v1 = -INFINITY;
        }
        sacc[n][e] = v0;
        sacc[n][2 + e] = v1;
        mx0 = fmaxf(mx0, v0);
        mx1 = fmaxf(mx1, v1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = (mn0 == -INFINITY) ? 1.f : exp2f(m0 - mn0);
    const float c1 = (mn1 == -INFINITY) ? 1.f : exp2f(m1 - mn1);
    const float b0s = (mn0 == -INFINITY) ? 0.f : mn0, b1s = (mn1 == -INFINITY) ? 0.f : mn1;
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pa[4][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float e0 = exp2f(sacc[n][0] - b0s), e1 = exp2f(sacc[n][1] - b0s);
      const float e2 = exp2f(sacc[n][2] - b1s), e3 = exp2f(sacc[n][3] - b1s);
      rs0 += e0 + e1;
      rs1 += e2 + e3;
      // accumulator layout of n-tiles (2kk, 2kk+1) is the A-fragment layout of key chunk kk
      pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(e0, e1);
      pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(e2, e3);
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) {
      oacc[i][0] *= c0; oacc[i][1] *= c0;
      oacc[i][2] *= c1; oacc[i][3] *= c1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = np * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(tV + swz<HD>(r, c)), b0, b1, b2, b3);
        mma16816(oacc[2 * np], a, b0, b1);
        mma16816(oacc[2 * np + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }
  // normalise and store
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int ra = r_begin + qrow0, rb = ra + 8;
  bf16* obase = o + (size_t)s * R * d + hh * HD;
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) {
    const int col = i * 8 + (lane & 3) * 2;
    if (ra < R) *reinterpret_cast<uint32_t*>(obase + (size_t)ra * d + col) = pack_bf16(oacc[i][0] * inv0, oacc[i][1] * inv0);
    if (rb < R) *reinterpret_cast<uint32_t*>(obase + (size_t)rb * d + col) = pack_bf16(oacc[i][2] * inv1, oacc[i][3] * inv1);
  }
}

}  // namespace

void launch_attn_tc(const Ctl* ctl, const bf16* q, const bf16* kc, const bf16* vc, bf16* o, int batch, int Lc,
                    int d, int heads, int r_max, cudaStream_t st) {
  dim3 grid((r_max + 63) / 64, heads, batch);
  if (d / heads == 64) {
    constexpr int smem = 5 * 64 * 64 * 2;
    static bool attr = false;
    if (!attr) { cudaFuncSetAttribute(k_attn_mma<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); attr = true; }
    k_attn_mma<64><<<grid, 128, smem, st>>>(ctl, q, kc, vc, o, Lc, d);
  } else {
    constexpr int smem = 5 * 64 * 128 * 2;
    static bool attr = false;
    if (!attr) { cudaFuncSetAttribute(k_attn_mma<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); attr = true; }
    k_attn_mma<128><<<grid, 128, smem, st>>>(ctl, q, kc, vc, o, Lc, d);
  }
}

}  // namespace af
