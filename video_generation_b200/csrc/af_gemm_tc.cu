// af_gemm_tc.cu -- bf16 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// C[M, N] = A[M, K] W[N, K]^T, both operands K-major bf16, fp32 accumulation in
// tensor memory, followed by one of the fused epilogues of af_common.cuh
// (bias + position add, QKV scatter into the KV cache, residual add, GELU,
// or the affine (mu, s) head).  These are the dense contractions of the AF
// block's causal Transformer: input projection, QKV, attention output
// projection, the two MLP matrices and the (mu, log-sigma) head.
//
// Design (one persistent CTA per SM, 256 threads):
//   warp 0      TMA producer: 128x64 A tile + BNx64 W tile per stage,
//               128-byte swizzle, mbarrier transaction counts.
//   warp 1      owns 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=BN, K=16) into one of two accumulators and commits
//               to the stage's "empty" barrier and the accumulator's "full".
//   warps 4..7  epilogue: tcgen05.ld 32 lanes x 16 columns per warp, apply
//               the fused epilogue, release the accumulator.
// With two accumulators the epilogue of tile i overlaps the MMAs of tile i+1.
// No cluster, no multicast: each CTA loads its own tiles.
// Every wait is bounded (2 s); on expiry the CTA raises its abort flag, drains
// its in-flight copies and MMAs, frees TMEM and reports ERR_GEMM_WAIT.
#include <cudaTypedefs.h>
#include "af_kernels.h"

namespace af {
namespace {

constexpr int BM = 128, BK = 64;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int BN> struct TcCfg {
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 192 ? 5 : 6);
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t NBARS = 2 * STAGES + 5;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + NBARS * 8 + 16;
  // instruction descriptor: F32 accumulate, BF16 A and B, both K-major, N>>3, M>>4
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(BM >> 4) << 24);
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `bar` with parity `parity`; false once the CTA has
// aborted or 2 s have passed (which aborts the CTA).
__device__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// Shared-memory matrix descriptor of a K-major tile written by TMA with
// 128-byte swizzle: rows of 64 bf16 (128 B), 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int BN, int EPI>
__global__ void __launch_bounds__(256, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int N, int K,
              EpiArgs e, int* err) {
  using Cfg = TcCfg<BN>;
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * Cfg::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * Cfg::B_BYTES);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  volatile int* abort_flag = &s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = e.ctl->M;
  const int tiles_m = (M + BM - 1) / BM, tiles_n = N / BN;
  const int ntiles = tiles_m * tiles_n;
  const int kbn = K / BK;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S), tempty0 = smem_u32(bars + 2 * S + 2);
  const uint32_t drain = smem_u32(bars + 2 * S + 4);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, 128);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int mb = t % tiles_m, nb = t / tiles_m;
        bool ok = true;
        for (int kb = 0; kb < kbn; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_expect_tx(full0 + 8 * stage, Cfg::STAGE_BYTES);
          tma_load_2d(smem_u32(sA + stage * Cfg::A_BYTES), &tmA, full0 + 8 * stage, kb * BK, mb * BM);
          tma_load_2d(smem_u32(sB + stage * Cfg::B_BYTES), &tmB, full0 + 8 * stage, kb * BK, nb * BN);
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // drain: the last load of every stage has landed before the CTA exits
      const long long n = issued < S ? issued : S;
      for (long long j = 1; j <= n; ++j) {
        const long long idx = issued - j;
        const int st = (int)(idx % S);
        const uint32_t ph = (uint32_t)((idx / S) & 1);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try(full0 + 8 * st, ph)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) { atomicExch(err, ERR_GEMM_DRAIN); break; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
        const int acc = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (!mbar_wait(tempty0 + 8 * acc, (use & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < kbn; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = sw128_desc(smem_u32(sA + stage * Cfg::A_BYTES));
          const uint64_t db = sw128_desc(smem_u32(sB + stage * Cfg::B_BYTES));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), Cfg::IDESC, (kb | k) != 0);
          umma_commit(empty0 + 8 * stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * acc);
      }
      // drain: every MMA issued by this thread has completed
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try(drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) { atomicExch(err, ERR_GEMM_DRAIN); break; }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 4;
    int i = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
      const int acc = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      if (!mbar_wait(tfull0 + 8 * acc, use & 1u, abort_flag)) break;
      tc_fence_after();
      const int mb = t % tiles_m, nb = t / tiles_m;
      const int row = mb * BM + ew * 32 + lane;
      const int n0 = nb * BN;
      const uint32_t taddr = tmem + (uint32_t)(acc * BN) + ((uint32_t)(ew * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld16(taddr + c, v);
        tmem_ld16(taddr + c + 16, v + 16);
        tmem_wait_ld();
        if (row < M) {
          if (EPI == EPI_HEAD) {
            head_group(e, row, n0 + c, v);
            head_group(e, row, n0 + c + 16, v + 16);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              epi4<EPI, bf16>(e, row, n0 + c + 4 * j, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (threadIdx.x == 0 && s_abort) atomicExch(err, ERR_GEMM_WAIT);
}

template <int BN, int EPI>
void launch_bn_epi(const CUtensorMap& tmA, const CUtensorMap& tmB, int N, int K, int m_max, const EpiArgs& e,
                   int* err, int num_sms, cudaStream_t st) {
  using Cfg = TcCfg<BN>;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_gemm_tc<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
    attr = true;
  }
  const int tiles = ((m_max + BM - 1) / BM) * (N / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  k_gemm_tc<BN, EPI><<<grid, 256, Cfg::SMEM, st>>>(tmA, tmB, N, K, e, err);
}

template <int BN>
void launch_bn(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, int N, int K, int m_max,
               const EpiArgs& e, int* err, int num_sms, cudaStream_t st) {
  switch (epi) {
    case EPI_INPROJ: launch_bn_epi<BN, EPI_INPROJ>(tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
    case EPI_QKV: launch_bn_epi<BN, EPI_QKV>(tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
    case EPI_RESID: launch_bn_epi<BN, EPI_RESID>(tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
    case EPI_GELU: launch_bn_epi<BN, EPI_GELU>(tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
    default: launch_bn_epi<BN, EPI_HEAD>(tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

bool make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile width: the candidate (dividing N) with the fewest column-waves of
// work, ceil(tiles / SMs) * BN; ties go to the wider tile.
int gemm_tc_pick_bn(int N, int m_max, int num_sms) {
  const int cands[3] = {256, 192, 128};
  int best = 0;
  long long best_cost = 0;
  for (int bn : cands) {
    if (N % bn) continue;
    const long long tiles = (long long)((m_max + BM - 1) / BM) * (N / bn);
    const long long cost = ((tiles + num_sms - 1) / num_sms) * bn;
    if (!best || cost < best_cost) { best = bn; best_cost = cost; }
  }
  return best;
}

void launch_gemm_tc(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, int bn, int N, int K, int m_max,
                    const EpiArgs& e, int* err, int num_sms, cudaStream_t st) {
  switch (bn) {
    case 256: launch_bn<256>(epi, tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
    case 192: launch_bn<192>(epi, tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
    default: launch_bn<128>(epi, tmA, tmB, N, K, m_max, e, err, num_sms, st); break;
  }
}

}  // namespace af
