// af_gemm_tc.cu -- bf16 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// C[M, N] = A[M, K] W[N, K]^T, both operands K-major bf16, fp32 accumulation in
// tensor memory, followed by one of the fused epilogues of af_common.cuh
// (bias + position add, QKV scatter into the KV cache, residual add, GELU,
// or the affine (mu, s) head).  These are the dense contractions of the AF
// block's causal Transformer: input projection, QKV, attention output
// projection, the two MLP matrices and the (mu, log-sigma) head.  A residual
// GEMM whose tiles would leave SM pairs idle runs split-K (EPI_PART): each
// unit is a (tile, half of K) pair that stores its fp32 partial by TMA, and
// a separate kernel sums the partials into h in split order.
//
// Design (persistent CTAs, one per SM, 384 or 640 threads):
//   warp 0      TMA producer: per stage two k-blocks (the last stage of a
//               tile one when K / 64 is odd), each a 128x64 A tile and a
//               (BN/CG)x64 W tile, 128-byte swizzle, one mbarrier
//               transaction count per stage.  Two k-blocks per barrier
//               round trip rather than one measured 1% faster on the
//               768-wide layers and 3.7% on the 2048-wide ones.
//   warp 1      owns 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128*CG, N=BN, K=16) into one of two accumulators and
//               commits to the stage's "empty" barrier and the accumulator's
//               "full".  CG = 2 pairs two SMs of a 2-CTA cluster on one
//               256-row tile (cta_group::2): each CTA loads its own 128 rows
//               of A and half of W, the leader issues the MMAs and its commits
//               reach both CTAs.  No TMA load uses cluster multicast.
//   warps 4..   epilogue, two or four warps per TMEM lane quarter (each takes
//               a column group of the tile), tcgen05.ld 32 lanes x 16 columns
//               at a time.  Residual add, GELU and QKV stage the result in
//               the output tensor map's swizzle and leave by TMA (bulk
//               reduce-add into h, bulk stores of u, q and the K / V cache);
//               the position add transposes through shared memory for
//               row-coalesced stores; the head works thread = row.
// With two accumulators the epilogue of tile i overlaps the MMAs of tile i+1.
// Every wait is bounded (2 s); on expiry the CTA raises its abort flag, drains
// its in-flight copies and MMAs, frees TMEM and reports ERR_GEMM_WAIT.
#include <cudaTypedefs.h>
#include "af_kernels.h"

namespace af {
namespace {

constexpr int BM = 128, BK = 64;
// Epilogue warps: 16 (4 per TMEM lane quarter), 8 for the position-add
// epilogue, which also reads two rows of positions (more registers per
// thread).  Block = producer, MMA, 2 spare, epilogue.
template <int EPI> struct EpiShape {
  static constexpr int WARPS = EPI == EPI_INPROJ ? 8 : 16;
  static constexpr int THREADS = (4 + WARPS) * 32;
  // residual add, GELU and QKV leave through TMA: each warp stages 32 rows x
  // 16 columns (one slot, reused once the previous bulk copy has read it) in
  // the output tensor map's swizzle and issues a bulk reduce-add (h += tile) or
  // a bulk store (u, q, K / V cache); one slot rather than two leaves room for
  // one more operand stage (a measured 1.4% on the 768-wide layers)
  static constexpr bool TMA_OUT = EPI == EPI_RESID || EPI == EPI_GELU || EPI == EPI_QKV || EPI == EPI_PART;
  static constexpr bool F32_OUT = EPI == EPI_RESID || EPI == EPI_PART;
  static constexpr uint32_t SLOT = F32_OUT ? 32 * 16 * 4 : 32 * 16 * 2;
};
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kMaxDevices = 64;

template <int BN, int CG, int EPI> struct TcCfg {
  // CG = CTAs per MMA: 1, or 2 for the SM-pair MMA (tile of 256 rows, each CTA
  // holding 128 rows of A and BN/2 rows of W).
  static constexpr int EPI_WARPS = EpiShape<EPI>::WARPS;
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = (BN / CG) * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  // per epilogue warp: a 32 x 16 fp32 transpose tile, 16-byte chunks
  // XOR-swizzled, or one TMA staging slot
  static constexpr uint32_t EPI_BYTES =
      EpiShape<EPI>::TMA_OUT ? EPI_WARPS * EpiShape<EPI>::SLOT : EPI_WARPS * 32 * 16 * 4;
  // KS k-blocks per stage, as many stages as the remaining shared memory
  // holds (at most 4)
  static constexpr int KS = 2;
  static constexpr int STAGES_FIT = (int)((232448u - 1024u - 512u - EPI_BYTES) / (KS * STAGE_BYTES));
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static constexpr uint32_t NBARS = 2 * STAGES + 6;
  static constexpr int THREADS = EpiShape<EPI>::THREADS;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * KS * STAGE_BYTES + EPI_BYTES + NBARS * 8 + 16;
  static_assert(STAGES >= 2 && SMEM <= 232448, "GEMM shared memory");
  // instruction descriptor: F32 accumulate, BF16 A and B, both K-major, N>>3, M>>4
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)((BM * CG) >> 4) << 24);
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
// The CTA's abort flag and the limit of its pipeline waits (the model's
// wait limit, 2 s by default; the drains after an abort keep kWaitLimitNs).
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// try_wait whose acquire covers writes released at cluster scope (by the
// other CTA of an SM pair)
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// complete-tx of `bytes` on a barrier of this CTA: stands in for a load that
// was counted on the barrier but never issued
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// The CTA's abort flag, the limit of its pipeline waits (the model's wait
// limit, 2 s by default; the drains after an abort keep kWaitLimitNs) and, on
// an SM pair, the other CTA's abort flag (shared::cluster address, else 0),
// raised with this CTA's so that the pair gives up together.
struct Abort {
  volatile int* flag;
  uint64_t limit_ns;
  uint32_t peer_flag;
};
// Wait for the phase of `bar` with parity `parity`; false once the CTA has
// aborted or the wait limit has passed (which aborts the CTA).
__device__ bool mbar_wait(uint32_t bar, uint32_t parity, const Abort& ab) {
  if (mbar_try(bar, parity)) return true;
  // slow path: every poll (a try_wait may itself block for a while) checks
  // the CTA's abort flag and the time
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (*ab.flag) return false;
    if (globaltimer_ns() - t0 > ab.limit_ns) {
      *ab.flag = 1;
      if (ab.peer_flag) st_cluster_u32(ab.peer_flag, 1u);
      return false;
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

// ---- SM-pair (cta_group::2) helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
// commit of the pair's MMAs, arriving on the barrier at this offset in both CTAs
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU of two values, with erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (Hastings):
// erf(u) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-u^2), t = 1 / (1 + p u),
// u >= 0, |error| <= 1.5e-7 -- far below the bf16 rounding of the MLP
// activations it feeds.  GELU(v) = v/2 + (v/2) sign(v) erf(|v| / sqrt 2).
// The fp32 SIMT path keeps erff.
__device__ __forceinline__ float2 gelu2_as7126(float2 v) {
  const float2 u = fmul2(make_float2(fabsf(v.x), fabsf(v.y)), splat(0.70710678118654752f));
  const float2 den = ffma2(u, splat(0.3275911f), splat(1.0f));
  const float2 t = make_float2(rcp_approx(den.x), rcp_approx(den.y));
  float2 q = ffma2(t, splat(1.061405429f), splat(-1.453152027f));
  q = ffma2(t, q, splat(1.421413741f));
  q = ffma2(t, q, splat(-0.284496736f));
  q = ffma2(t, q, splat(0.254829592f));
  q = fmul2(q, t);
  const float2 w = fmul2(fmul2(u, u), splat(-1.4426950408889634f));   // -u^2 log2(e)
  const float2 e = make_float2(ex2_approx(w.x), ex2_approx(w.y));
  const float2 erf_abs = ffma2(fmul2(q, e), splat(-1.0f), splat(1.0f));
  const float2 erf_s = make_float2(copysignf(erf_abs.x, v.x), copysignf(erf_abs.y, v.y));
  const float2 hv = fmul2(v, splat(0.5f));
  return ffma2(hv, erf_s, hv);
}

// TMA bulk writes of a staged tile (one thread), tracked as bulk async-groups.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
// The same with an L2 cache policy (createpolicy): outputs the next kernel
// reads at once are kept in L2 with evict_last.
__device__ __forceinline__ void tma_reduce_add_2d_hint(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                                       uint64_t pol) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, uint32_t src, int c0, int c1, uint64_t pol) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "l"(pol)
               : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most one group still reading its shared-memory source
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }


template <int BN, int EPI, int CG>
__global__ void __launch_bounds__(EpiShape<EPI>::THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
              const __grid_constant__ CUtensorMap tmC3, int N, int K, EpiArgs e, int* err) {
  using Cfg = TcCfg<BN, CG, EPI>;
  constexpr int S = Cfg::STAGES;
  constexpr int TM = BM * CG;               // accumulator rows per tile (both CTAs)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  constexpr int KS = Cfg::KS;
  uint8_t* sB = smem + S * KS * Cfg::A_BYTES;
  float* sEpi = reinterpret_cast<float*>(sB + S * KS * Cfg::B_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * KS * Cfg::B_BYTES + Cfg::EPI_BYTES);
  // bars: full[S], empty[S], tfull[2], tempty[2], drain, peer_done
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ uint32_t s_peer_issued;      // leader: loads the pair's second CTA issued
  volatile int* abort_flag = &s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;   // 0 = the pair's leader (issues the MMAs)
  const Abort ab{abort_flag, e.wait_ns, CG == 2 ? map_to_rank(smem_u32(&s_abort), rank ^ 1u) : 0u};
  const int unit = CG == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int nunits = CG == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int tiles_n = N / BN;
  const int kbn = K / BK;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t tfull0 = smem_u32(bars + 2 * S), tempty0 = smem_u32(bars + 2 * S + 2);
  const uint32_t drain = smem_u32(bars + 2 * S + 4);
  const uint32_t peer_done = smem_u32(bars + 2 * S + 5);

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_peer_issued = 0;
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, Cfg::EPI_WARPS * 32 * CG);
    }
    mbar_init(drain, 1);
    mbar_init(peer_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    if (EpiShape<EPI>::TMA_OUT) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmC)) : "memory");
    if (EPI == EPI_QKV) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmC2)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmC3)) : "memory");
    }
  }
  if (warp == 1) {
    if (CG == 2) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                   "r"(512));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                   "r"(512));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();   // the peer's barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t full_lead = CG == 2 ? map_to_rank(full0, 0) : full0;
  const uint32_t tempty_lead = CG == 2 ? map_to_rank(tempty0, 0) : tempty0;
  pdl_wait();                      // the A operand and the row count come from upstream
  const int M = e.ctl->M;
  const int tiles_m = (M + TM - 1) / TM;
  const int ntiles = tiles_m * tiles_n;
  // split-K (EPI_PART): as many splits as idle units allow, at most ksplit,
  // each an even number of k-blocks (whole stages) and at least 8 of them;
  // unit work w = split * ntiles + tile over k-blocks [split * kbs, + kbs)
  int ks = 1;
  if (EPI == EPI_PART) {
    ks = ntiles > 0 ? nunits / ntiles : 1;
    if (ks > e.ksplit) ks = e.ksplit;
    while (ks > 1 && (kbn % (KS * ks) != 0 || kbn / ks < 8)) --ks;
    if (ks < 1) ks = 1;
    // one split: the epilogue adds into h itself (ks_out 0: nothing to sum)
    if (blockIdx.x == 0 && threadIdx.x == 0) *e.ks_out = ks > 1 ? ks : 0;
  }
  const bool part_store = EPI == EPI_PART && ks > 1;      // warp-uniform
  const int kbs = kbn / ks;
  const int nwork = ntiles * ks;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int w = unit; w < nwork; w += nunits) {
        const int t = w % ntiles, kb0 = (w / ntiles) * kbs;
        const int mb = t % tiles_m, nb = t / tiles_m;
        const int arow = mb * TM + (int)rank * BM;
        const int brow = nb * BN + (int)rank * (BN / CG);
        bool ok = true;
        for (int kb = kb0; kb < kb0 + kbs; kb += KS) {
          const int nk = kb0 + kbs - kb < KS ? kb0 + kbs - kb : KS;
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, ab)) { ok = false; break; }
          if (rank == 0) mbar_expect_tx(full0 + 8 * stage, CG * nk * Cfg::STAGE_BYTES);
          for (int j = 0; j < nk; ++j) {
            const int sl = stage * KS + j;
            if (CG == 2) {
              tma_load_2d_pair(smem_u32(sA + sl * Cfg::A_BYTES), &tmA, full_lead + 8 * stage, (kb + j) * BK, arow);
              tma_load_2d_pair(smem_u32(sB + sl * Cfg::B_BYTES), &tmB, full_lead + 8 * stage, (kb + j) * BK, brow);
            } else {
              tma_load_2d(smem_u32(sA + sl * Cfg::A_BYTES), &tmA, full0 + 8 * stage, (kb + j) * BK, arow);
              tma_load_2d(smem_u32(sB + sl * Cfg::B_BYTES), &tmB, full0 + 8 * stage, (kb + j) * BK, brow);
            }
          }
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (CG == 2 && rank != 0) {
        // The second CTA's loads complete on the leader's full barriers: it
        // tells the leader how many it issued (its own abort, or the leader's,
        // may have stopped it at a different k-block than the leader), and the
        // leader's drain covers them before the pair leaves together (cluster
        // barrier at the end).
        st_cluster_u32(map_to_rank(smem_u32(&s_peer_issued), 0), (uint32_t)issued);
        mbar_arrive_cluster(map_to_rank(peer_done, 0));
      } else {
        // drain: the last load of every stage has landed before the CTA exits.
        // On an SM pair a stage's full barrier counts both CTAs' bytes: a
        // stage only the second CTA loaded gets the leader's arrival with the
        // second CTA's bytes, and a stage the leader armed for both but the
        // second CTA never loaded gets those bytes completed by hand.  Both
        // CTAs walk the same units, ceil(kbs / KS) stages each, so stage idx
        // is stage idx % spt of its unit and holds that stage's k-blocks.
        const int spt = (kbs + KS - 1) / KS;
        long long hi = issued, peer = issued;
        bool have_peer = true;
        if (CG == 2) {
          const uint64_t limit = ab.limit_ns + kWaitLimitNs;   // the second CTA's own waits end first
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_cluster(peer_done, 0)) {
            if (globaltimer_ns() - t0 > limit) { atomicOr(err, ERR_DRAIN); have_peer = false; break; }
          }
          if (have_peer) peer = (long long)s_peer_issued;
          if (peer > hi) hi = peer;
        }
        for (long long idx = (hi > S ? hi - S : 0); idx < hi && have_peer; ++idx) {
          const int st = (int)(idx % S);
          const uint32_t ph = (uint32_t)((idx / S) & 1);
          const int pos = (int)(idx % spt);
          const uint32_t peer_bytes = (uint32_t)(kbs - pos * KS < KS ? kbs - pos * KS : KS) * Cfg::STAGE_BYTES;
          if (CG == 2 && idx >= issued) mbar_expect_tx(full0 + 8 * st, peer_bytes);
          if (CG == 2 && idx < issued && idx >= peer) mbar_complete_tx(full0 + 8 * st, peer_bytes);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try(full0 + 8 * st, ph)) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) { atomicOr(err, ERR_DRAIN); break; }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issuer (leader only)
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      for (int w = unit; w < nwork; w += nunits, ++i) {
        const int kb0 = (w / ntiles) * kbs;
        const int acc = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (!mbar_wait(tempty0 + 8 * acc, (use & 1u) ^ 1u, ab)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = kb0; kb < kb0 + kbs; kb += KS) {
          const int nk = kb0 + kbs - kb < KS ? kb0 + kbs - kb : KS;
          if (!mbar_wait(full0 + 8 * stage, phase, ab)) { ok = false; break; }
          tc_fence_after();
          for (int j = 0; j < nk; ++j) {
            const int sl = stage * KS + j;
            const uint64_t da = sw128_desc(smem_u32(sA + sl * Cfg::A_BYTES));
            const uint64_t db = sw128_desc(smem_u32(sB + sl * Cfg::B_BYTES));
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint32_t accum = ((kb - kb0 + j) | k) != 0;
              if (CG == 2) umma_bf16_pair(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), Cfg::IDESC, accum);
              else umma_bf16(d_tmem, da + (uint64_t)(2 * k), db + (uint64_t)(2 * k), Cfg::IDESC, accum);
            }
          }
          if (CG == 2) umma_commit_pair(empty0 + 8 * stage);
          else umma_commit(empty0 + 8 * stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (CG == 2) umma_commit_pair(tfull0 + 8 * acc);
        else umma_commit(tfull0 + 8 * acc);
      }
      // drain: every MMA issued by this thread has completed
      if (CG == 2) umma_commit_pair_local(drain);
      else umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try(drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) { atomicOr(err, ERR_DRAIN); break; }
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    // Warp 4+ew owns TMEM lane quarter q = ew % 4 (rows 32q..32q+31 of the
    // tile) and column group ew / 4, read 16 columns at a time.
    const int ew = warp - 4;
    const int q = ew & 3, hf = ew >> 2;                 // lane quarter, column group
    constexpr int HALF = BN / (Cfg::EPI_WARPS / 4);     // columns per warp
    if constexpr (EpiShape<EPI>::TMA_OUT) {
      // Thread = row: each 16-column chunk read from TMEM gets its bias (and
      // GELU) and is written, in the output tensor map's swizzle, to the warp's
      // staging slot; lane 0 then sends the 32 x 16 tile with a TMA
      // bulk reduce-add into h (each element gets exactly one add, so the result
      // is deterministic) or a bulk store into u or q.  Rows past the last real
      // row land in workspace rows no kernel reads; rows past the buffer are
      // clipped.  K and V rows go to the cache at (sample, position): a warp's
      // 32 rows are one TMA store when they lie in one sample, else each thread
      // stores its row (a few slices per call straddle two samples).
      constexpr uint32_t SLOT = EpiShape<EPI>::SLOT;
      constexpr int NCH = HALF / 16;
      uint8_t* stg = reinterpret_cast<uint8_t*>(sEpi) + ew * SLOT;
      const int R = e.ctl->R, p0 = e.ctl->p0;
      const uint64_t keep_pol = e.l2_keep ? policy_evict_last() : 0ull;
      int i = 0;
      for (int w = unit; w < nwork; w += nunits, ++i) {
        const int t = w % ntiles;
        const int acc = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        const int mb = t % tiles_m, nb = t / tiles_m;
        const int row0 = mb * TM + (int)rank * BM + q * 32;
        // EPI_PART: the split's partial rows
        const int orow0 = EPI == EPI_PART ? (w / ntiles) * e.kpart_rows + row0 : row0;
        const int n0 = nb * BN + hf * HALF;
        const uint32_t taddr = tmem + (uint32_t)(acc * BN + hf * HALF) + ((uint32_t)(q * 32) << 16);
        // QKV: a 16-column chunk lies in one of q, K, V (16 divides d); the K
        // and V rows of this warp go to the cache at (sample, position)
        int ycache = 0;
        bool cache_ok = true;                           // warp-uniform
        if (EPI == EPI_QKV) {
          const int s0 = row0 / R;
          cache_ok = row0 + 31 < M && (row0 + 31) / R == s0;
          ycache = s0 * e.Lc + p0 + (row0 - s0 * R);
        }
        // the bias of the first chunk is loaded before waiting for the accumulator,
        // each later chunk's while the previous one is processed
        // (split-K partials take no bias: the kernel that sums them adds it)
        float4 bnext[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          bnext[jj] = part_store ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<const float4*>(e.bias + n0)[jj];
        // the wait's outcome is made warp-uniform before the .aligned TMEM loads
        if (!__all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * acc, use & 1u, ab))) break;
        tc_fence_after();
        float vb[2][16];
        tmem_ld16(taddr, vb[0]);
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          float4 b4[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) b4[jj] = bnext[jj];
          if (k + 1 < NCH) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              bnext[jj] = part_store ? make_float4(0.f, 0.f, 0.f, 0.f)
                                     : reinterpret_cast<const float4*>(e.bias + n0 + (k + 1) * 16)[jj];
          }
          tmem_wait_ld();
          if (k + 1 < NCH) {
            tmem_ld16(taddr + (k + 1) * 16, vb[(k + 1) & 1]);
          } else {
            // every TMEM read of this tile is done: release the accumulator
            tc_fence_before();
            if (CG == 2) mbar_arrive_cluster(tempty_lead + 8 * acc);
            else mbar_arrive(tempty0 + 8 * acc);
          }
          const float* v = vb[k & 1];
          const int col = n0 + k * 16;
          const int which = EPI == EPI_QKV ? col / e.d : 0;  // 0 q, 1 K, 2 V
          const bool tma_ok = which == 0 || cache_ok;       // warp-uniform
          uint8_t* slot = stg;
          if (lane == 0) bulk_wait_read0();             // the slot's previous tile has been read
          __syncwarp();
          if (EpiShape<EPI>::F32_OUT) {
            // fp32 rows of 64 B, 64-byte swizzle: 16-byte unit j of row r at j ^ ((r >> 1) & 3)
            uint8_t* rp = slot + lane * 64;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const float4 bb = b4[jj];
              *reinterpret_cast<float4*>(rp + ((jj ^ ((lane >> 1) & 3)) << 4)) =
                  make_float4(v[4 * jj] + bb.x, v[4 * jj + 1] + bb.y, v[4 * jj + 2] + bb.z, v[4 * jj + 3] + bb.w);
            }
          } else {
            // bf16 rows of 32 B, 32-byte swizzle: 16-byte unit j of row r at j ^ ((r >> 2) & 1)
            uint32_t pk[8];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const float4 bb = b4[jj];
              float2 g0 = fadd2(make_float2(v[4 * jj], v[4 * jj + 1]), make_float2(bb.x, bb.y));
              float2 g1 = fadd2(make_float2(v[4 * jj + 2], v[4 * jj + 3]), make_float2(bb.z, bb.w));
              if (EPI == EPI_GELU) {
                g0 = gelu2_as7126(g0);
                g1 = gelu2_as7126(g1);
              }
              __nv_bfloat162 lo = __floats2bfloat162_rn(g0.x, g0.y), hi = __floats2bfloat162_rn(g1.x, g1.y);
              pk[2 * jj] = *reinterpret_cast<uint32_t*>(&lo);
              pk[2 * jj + 1] = *reinterpret_cast<uint32_t*>(&hi);
            }
            if (tma_ok) {
              uint8_t* rp = slot + lane * 32;
              const int sw = (lane >> 2) & 1;
              *reinterpret_cast<uint4*>(rp + (sw << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              *reinterpret_cast<uint4*>(rp + ((1 ^ sw) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            } else if (row0 + lane < M) {
              // a K / V slice straddling two samples: this thread's row, direct
              const int r = row0 + lane, sm = r / R;
              bf16* cache = reinterpret_cast<bf16*>(which == 1 ? e.kc : e.vc);
              uint4* dst = reinterpret_cast<uint4*>(cache + ((size_t)sm * e.Lc + p0 + (r - sm * R)) * e.d +
                                                    (col - which * e.d));
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
          if (tma_ok) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              if (part_store && e.l2_keep) tma_store_2d_hint(&tmC, smem_u32(slot), col, orow0, keep_pol);
              else if (part_store) tma_store_2d(&tmC, smem_u32(slot), col, orow0);
              else if (EPI == EPI_PART && e.l2_keep) tma_reduce_add_2d_hint(&tmC2, smem_u32(slot), col, row0, keep_pol);
              else if (EPI == EPI_PART) tma_reduce_add_2d(&tmC2, smem_u32(slot), col, row0);
              else if (e.l2_keep && EPI == EPI_RESID) tma_reduce_add_2d_hint(&tmC, smem_u32(slot), col, row0, keep_pol);
              else if (EPI == EPI_RESID) tma_reduce_add_2d(&tmC, smem_u32(slot), col, row0);
              else if (e.l2_keep && EPI == EPI_GELU) tma_store_2d_hint(&tmC, smem_u32(slot), col, row0, keep_pol);
              else if (EPI == EPI_GELU || which == 0) tma_store_2d(&tmC, smem_u32(slot), col - which * e.d, row0);
              else tma_store_2d(which == 1 ? &tmC2 : &tmC3, smem_u32(slot), col - which * e.d, ycache);
              bulk_commit();
            }
          }
        }
      }
      if (lane == 0) bulk_wait_all();                   // the bulk writes are complete before the CTA exits
      __syncwarp();
    } else {
      // Position add (input projection) and the affine head.  For the position
      // add a 16-column chunk read from TMEM (thread = row) is transposed
      // through a swizzled 32 x 16 staging tile, so that lane l stores row
      // 8 it + l / 4, columns 4 (l % 4) .. + 3: each store covers eight 64-byte
      // row segments.  The head keeps thread = row.  Row -> (sample, position)
      // and the row pointers are computed once per tile.
      static_assert(EPI == EPI_INPROJ || EPI == EPI_HEAD || EPI == EPI_DENOISE, "epilogue without a TMA path");
      float* stg = sEpi + ew * 32 * 16;
      const int rl = lane >> 2, cq = lane & 3;
      const int sw_w = (lane >> 1) & 3;            // swizzle of the row this lane writes
      const int sw_r = (rl >> 1) & 3;              // swizzle of the rows this lane reads
      const Ctl* ctl = e.ctl;
      const int R = ctl->R, p0 = ctl->p0;
      int i = 0;
      for (int t = unit; t < ntiles; t += nunits, ++i) {
        const int acc = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        const int mb = t % tiles_m, nb = t / tiles_m;
        const int row0 = mb * TM + (int)rank * BM + q * 32;
        const int n0 = nb * BN + hf * HALF;
        const uint32_t taddr = tmem + (uint32_t)(acc * BN + hf * HALF) + ((uint32_t)(q * 32) << 16);
        // position add: the 4 rows this lane stores and their position rows
        float* rowp[4];
        const float* pos_s[4];
        const float* pos_t[4];
        if (EPI == EPI_INPROJ) {
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int r = row0 + it * 8 + rl;
            const int sm = r / R;
            const int p = p0 + (r - sm * R);
            rowp[it] = e.h + (size_t)r * e.d;
            pos_s[it] = e.pos_space + (size_t)(p % e.frame_len) * e.d;
            pos_t[it] = e.pos_time + (size_t)(p / e.frame_len) * e.d;
          }
        }
        // head: one row per thread, hoisted (sample, position, token) and row pointers
        bool head_out = false, head_act = false;
        const float* hin = nullptr;
        float* hout = nullptr;
        float* hpart = nullptr;
        if (EPI == EPI_HEAD || EPI == EPI_DENOISE) {
          const int r = row0 + lane;
          const int sm = r / R;
          const int p = p0 + (r - sm * R);
          head_out = r < M && p >= ctl->P;
          const size_t base = ((size_t)sm * e.L + tok_of(p, e.L, e.dir)) * e.C;
          hin = e.xin_f + base;
          hout = e.xout_f + base;
          hpart = e.part + (size_t)r * ((2 * e.C) >> 4) * 2;
          head_act = head_out && (EPI == EPI_DENOISE || e.head_mode == 0 || e.active[sm]);
        }
        // Loads that do not depend on the accumulator are issued before waiting
        // for it (bias, and the first chunk's position / x rows), and every
        // chunk's TMEM load and global loads are in flight while the previous
        // chunk is processed.
        constexpr int NCH = HALF / 16;
        float4 bias4[NCH];
#pragma unroll
        for (int k = 0; k < NCH; ++k) bias4[k] = *reinterpret_cast<const float4*>(e.bias + n0 + k * 16 + cq * 4);
        float4 pre[2][4], pre2[2][4];
        auto load_rows = [&](int k, float4* dst, float4* dst2) {
          if (EPI == EPI_DENOISE) {                         // 16 plain channels
            if (head_act) {
              const float4* src = reinterpret_cast<const float4*>(hin + n0 + k * 16);
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) dst[qq] = src[qq];
            }
            return;
          }
          if (EPI == EPI_HEAD) {
            if (head_act) {
              const int c0 = (n0 + k * 16) >> 1;
              dst[0] = *reinterpret_cast<const float4*>(hin + c0);
              dst[1] = *reinterpret_cast<const float4*>(hin + c0 + 4);
              if (e.head_mode == 1) {
                dst2[0] = *reinterpret_cast<const float4*>(hout + c0);
                dst2[1] = *reinterpret_cast<const float4*>(hout + c0 + 4);
              }
            }
            return;
          }
          const int col = n0 + k * 16 + cq * 4;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            if (row0 + it * 8 + rl < M) {
              dst[it] = *reinterpret_cast<const float4*>(pos_s[it] + col);
              dst2[it] = *reinterpret_cast<const float4*>(pos_t[it] + col);
            }
          }
        };
        load_rows(0, pre[0], pre2[0]);
        // the wait's outcome is made warp-uniform before the .aligned TMEM loads
        if (!__all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * acc, use & 1u, ab))) break;
        tc_fence_after();
        float vb[2][16];
        tmem_ld16(taddr, vb[0]);
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          const int c = k * 16;
          tmem_wait_ld();
          if (k + 1 < NCH) {
            tmem_ld16(taddr + c + 16, vb[(k + 1) & 1]);
            load_rows(k + 1, pre[(k + 1) & 1], pre2[(k + 1) & 1]);
          }
          const float* v = vb[k & 1];
          if (EPI == EPI_DENOISE) {
            // denoiser: x = x_noisy + sigma * (s_phi + b) for 16 plain channels
            if (!head_out) continue;
            const int col0 = n0 + c;
            const float4* xn4 = pre[k & 1];
            float4* o4 = reinterpret_cast<float4*>(hout + col0);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float4 bb = *reinterpret_cast<const float4*>(e.bias + col0 + 4 * qq);
              o4[qq] = make_float4(fmaf(e.sigma, v[4 * qq] + bb.x, xn4[qq].x), fmaf(e.sigma, v[4 * qq + 1] + bb.y, xn4[qq].y),
                                   fmaf(e.sigma, v[4 * qq + 2] + bb.z, xn4[qq].z), fmaf(e.sigma, v[4 * qq + 3] + bb.w, xn4[qq].w));
            }
            continue;
          }
          if (EPI == EPI_HEAD) {
            // 8 channels whose (mu_c, s_c) sit at columns (2c, 2c+1)
            const int col0 = n0 + c;
            float2* part = reinterpret_cast<float2*>(hpart) + (col0 >> 4);
            if (!head_out) continue;
            if (!head_act) { *part = make_float2(0.f, 0.f); continue; }
            const float* xi = reinterpret_cast<const float*>(pre[k & 1]);
            float r8[8];
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const float mu = v[2 * jj] + e.bias[col0 + 2 * jj];
              const float sl = v[2 * jj + 1] + e.bias[col0 + 2 * jj + 1];
              if (e.head_mode == 0) {
                r8[jj] = (xi[jj] - mu) * expf(-sl);            // z = (x - mu) exp(-s)
                a0 += sl;
              } else {
                r8[jj] = fmaf(expf(sl), xi[jj], mu);           // x_new = mu + exp(s) z
                const float dx = r8[jj] - reinterpret_cast<const float*>(pre2[k & 1])[jj];
                a0 = fmaf(dx, dx, a0);
                a1 = fmaf(r8[jj], r8[jj], a1);
              }
            }
            const int c0 = col0 >> 1;
            *reinterpret_cast<float4*>(hout + c0) = make_float4(r8[0], r8[1], r8[2], r8[3]);
            *reinterpret_cast<float4*>(hout + c0 + 4) = make_float4(r8[4], r8[5], r8[6], r8[7]);
            *part = make_float2(a0, a1);
            continue;
          }
          float4* srow = reinterpret_cast<float4*>(stg + lane * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) srow[j ^ sw_w] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          __syncwarp();
          float4 a[4];
#pragma unroll
          for (int it = 0; it < 4; ++it) a[it] = reinterpret_cast<const float4*>(stg + (it * 8 + rl) * 16)[cq ^ sw_r];
          __syncwarp();
          const int col = n0 + c + cq * 4;
          const float4 bb = bias4[k];
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            if (row0 + it * 8 + rl < M) {
              const float4 ps = pre[k & 1][it], pt = pre2[k & 1][it];
              *reinterpret_cast<float4*>(rowp[it] + col) =
                  make_float4(a[it].x + bb.x + ps.x + pt.x, a[it].y + bb.y + ps.y + pt.y,
                              a[it].z + bb.z + ps.z + pt.z, a[it].w + bb.w + ps.w + pt.w);
            }
          }
        }
        tc_fence_before();
        if (CG == 2) mbar_arrive_cluster(tempty_lead + 8 * acc);
        else mbar_arrive(tempty0 + 8 * acc);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();   // the leader's MMAs (writing both TMEMs) are drained
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    else asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(err, ERR_GEMM_WAIT);
}

template <int BN, int EPI, int CG>
void launch_bn_epi(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmC2,
                   const CUtensorMap& tmC3, int N, int K, int m_max, const EpiArgs& e,
                   int* err, int num_sms, cudaStream_t st) {
  using Cfg = TcCfg<BN, CG, EPI>;
  // the shared-memory opt-in and the co-resident cluster count are per device
  static int units_of_dev[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  int& max_units = units_of_dev[dev];
  if (!max_units) {
    cudaFuncSetAttribute(k_gemm_tc<BN, EPI, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
    max_units = num_sms / CG;
    if (CG == 2) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * max_units);
      q.blockDim = dim3(Cfg::THREADS);
      q.dynamicSmemBytes = Cfg::SMEM;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = 2; a[0].val.clusterDim.y = 1; a[0].val.clusterDim.z = 1;
      q.attrs = a;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, k_gemm_tc<BN, EPI, CG>, &q) == cudaSuccess && clusters > 0 &&
          clusters < max_units)
        max_units = clusters;
    }
  }
  const int tiles = ((m_max + BM * CG - 1) / (BM * CG)) * (N / BN) * (EPI == EPI_PART ? e.ksplit : 1);
  const int units = tiles > max_units ? max_units : tiles;
  if (CG == 1) {
    launch_k(k_gemm_tc<BN, EPI, 1>, dim3(units), dim3(Cfg::THREADS), Cfg::SMEM, st, tmA, tmB, tmC, tmC2, tmC3, N, K, e, err);
  } else {
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(2 * units);
    c.blockDim = dim3(Cfg::THREADS);
    c.dynamicSmemBytes = Cfg::SMEM;
    c.stream = st;
    cudaLaunchAttribute a[2];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = 2; a[0].val.clusterDim.y = 1; a[0].val.clusterDim.z = 1;
    a[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[1].val.programmaticStreamSerializationAllowed = g_pdl;
    c.attrs = a;
    c.numAttrs = 2;
    cudaLaunchKernelEx(&c, k_gemm_tc<BN, EPI, CG>, tmA, tmB, tmC, tmC2, tmC3, N, K, e, err);
  }
}

template <int BN, int CG>
void launch_bn(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmC2,
               const CUtensorMap& tmC3, int N, int K, int m_max,
               const EpiArgs& e, int* err, int num_sms, cudaStream_t st) {
  switch (epi) {
    case EPI_INPROJ: launch_bn_epi<BN, EPI_INPROJ, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
    case EPI_QKV: launch_bn_epi<BN, EPI_QKV, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
    case EPI_RESID: launch_bn_epi<BN, EPI_RESID, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
    case EPI_GELU: launch_bn_epi<BN, EPI_GELU, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
    case EPI_HEAD: launch_bn_epi<BN, EPI_HEAD, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
    case EPI_PART: launch_bn_epi<BN, EPI_PART, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
    default: launch_bn_epi<BN, EPI_DENOISE, CG>(tmA, tmB, tmC, tmC2, tmC3, N, K, m_max, e, err, num_sms, st); break;
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

bool make_tmap_out(CUtensorMap* map, const void* base, bool f32, int rows, int cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * es};
  cuuint32_t box[2] = {16u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            f32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile shape: SM-pair MMAs (256-row tiles) when there are at least 256 rows,
// and the width (<= max_bn, dividing N, and `unit` when non-zero) with the
// least work per unit, ceil(tiles / units) * BN, weighted by the shared-memory
// traffic a narrower tile spends per flop (operand bytes per MMA flop grow as
// 1/BN + 1/256: x1.15 at 192, x1.3 at 128, a measured trade-off against wave
// quantisation); ties go to the wider tile.  Returns BN * 10 + CG.
int gemm_tc_pick(int N, int m_max, int num_sms, int unit, int max_bn) {
  const int cands[3] = {256, 192, 128};
  const int weight[3] = {100, 115, 130};
  const int cg = m_max >= 256 ? 2 : 1;
  const int units = num_sms / cg;
  int best = 0;
  long long best_cost = 0;
  for (int i = 0; i < 3; ++i) {
    const int bn = cands[i];
    if (N % bn || (unit && unit % bn) || bn > max_bn) continue;
    const long long tiles = (long long)((m_max + BM * cg - 1) / (BM * cg)) * (N / bn);
    const long long cost = ((tiles + units - 1) / units) * bn * weight[i];
    if (!best || cost < best_cost) { best = bn; best_cost = cost; }
  }
  return best ? best * 10 + cg : 0;
}

int gemm_tc_tiles(int pick, int N, int m_rows) {
  const int bn = pick / 10, cg = pick % 10;
  return bn ? ((m_rows + BM * cg - 1) / (BM * cg)) * (N / bn) : 0;
}

void launch_gemm_tc(int epi, const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap* tmC,
                    const CUtensorMap* tmC2, const CUtensorMap* tmC3, int pick, int N, int K, int m_max,
                    const EpiArgs& e, int* err, int num_sms, cudaStream_t st) {
  const int bn = pick / 10, cg = pick % 10;
  // only the TMA epilogues read them
  const CUtensorMap& tmC_ = tmC ? *tmC : tmA;
  const CUtensorMap& tmC2_ = tmC2 ? *tmC2 : tmA;
  const CUtensorMap& tmC3_ = tmC3 ? *tmC3 : tmA;
  if (cg == 2) {
    switch (bn) {
      case 256: launch_bn<256, 2>(epi, tmA, tmB, tmC_, tmC2_, tmC3_, N, K, m_max, e, err, num_sms, st); break;
      case 192: launch_bn<192, 2>(epi, tmA, tmB, tmC_, tmC2_, tmC3_, N, K, m_max, e, err, num_sms, st); break;
      default: launch_bn<128, 2>(epi, tmA, tmB, tmC_, tmC2_, tmC3_, N, K, m_max, e, err, num_sms, st); break;
    }
  } else {
    switch (bn) {
      case 256: launch_bn<256, 1>(epi, tmA, tmB, tmC_, tmC2_, tmC3_, N, K, m_max, e, err, num_sms, st); break;
      case 192: launch_bn<192, 1>(epi, tmA, tmB, tmC_, tmC2_, tmC3_, N, K, m_max, e, err, num_sms, st); break;
      default: launch_bn<128, 1>(epi, tmA, tmB, tmC_, tmC2_, tmC3_, N, K, m_max, e, err, num_sms, st); break;
    }
  }
}

}  // namespace af
