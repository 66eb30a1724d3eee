// af_attn_tc.cu -- causal multi-head attention over the KV cache on the 5th-
// generation tensor cores (tcgen05, sm_100a).
//
// Query row r of sample s sits at position p = p0 + r % R and attends keys
// 0..p of the sample's cache: softmax(q k^T / sqrt(hd), j <= p) v.  The
// finished blocks of the block-wise Jacobi schedule are read from the cache
// and the current block's rows attend causally among themselves ("STARFlow-V
// ... paper notes", key design 3: finished blocks feed a KV cache).
//
// Persistent CTAs (one per SM) walk a static list of work items: 128 query rows
// of one (sample, head) against the key tiles of one split of the key range,
// 128 keys per tile.  Q and the O accumulator are double-buffered across items
// so the next item's loads and MMAs overlap the current item's softmax.
//   warp 0      TMA: Q once (128 x hd), then K and V tiles (128 keys x hd)
//               into a 2-3 stage ring; 128-byte swizzle.
//   warp 1      one thread issues S_j = Q K_j^T (M=128, N=128, K=hd) into one
//               of two TMEM buffers, and O += P_j V_j (M=128, N=hd, K=128)
//               into the TMEM accumulator; V is consumed in its natural
//               [key][hd] layout as an MN-major operand.
//   warps 4-11  softmax, two warps per TMEM lane quarter, each owning half of
//               a row's 128 scores and half of its hd outputs: pass 1 takes
//               the row max (halves exchanged through shared memory), pass 2
//               writes P = exp2(t - m) as bf16 into a swizzled shared tile.
//               The running max is raised lazily: O (in TMEM) and the row sum
//               are rescaled only when the max grows by more than 2^8, which
//               keeps every P below 256 and the result exact.
// With several splits, each writes an unnormalised (o, m, l) partial and
// k_attn_combine merges them.  Every wait is bounded (2 s); on expiry the CTA
// drains, frees TMEM and reports ERR_ATTN_WAIT.
#include "af_kernels.h"

namespace af {
namespace {

constexpr int BQ = 128, BKV = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;

template <int HD> struct AttnCfg {
  static constexpr int KCH = HD / 64;                     // 64-wide column boxes per row
  static constexpr uint32_t BOX = 128 * 64 * 2;           // one 128-row x 64-col bf16 box: 16 KB
  static constexpr uint32_t Q_BYTES = KCH * BOX;
  static constexpr uint32_t KV_BYTES = KCH * BOX;         // K or V tile
  static constexpr int STAGES = HD == 64 ? 3 : 2;
  static constexpr int QBUF = HD == 64 ? 2 : 1;            // Q buffers across work items
  static constexpr int PB = HD == 64 ? 2 : 1;              // P tiles (softmax j+1 overlaps P_j V_j)
  static constexpr uint32_t P_BYTES = 2 * BOX;            // one P tile: 128 rows x 128 keys
  static constexpr size_t SMEM = 1024 + QBUF * Q_BYTES + (size_t)STAGES * 2 * KV_BYTES + PB * P_BYTES +
                                 3 * 2 * 128 * 4 + (2 * STAGES + 27) * 8 + 64;
  // S = Q K^T: M 128, N 128, both K-major
  static constexpr uint32_t IDESC_S = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BKV >> 3) << 17) |
                                      ((uint32_t)(BQ >> 4) << 24);
  // O += P V: M 128, N hd, A (P) K-major, B (V) MN-major
  static constexpr uint32_t IDESC_O = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(HD >> 3) << 17) | ((uint32_t)(BQ >> 4) << 24);
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
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
// K-major, 128-byte swizzle: rows of 64 bf16, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major, 128-byte swizzle: 64 contiguous elements of N per row, one row per
// K index, 8-row groups 1024 B apart (SBO), 64-wide N boxes `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
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
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 2^x on the special-function unit (flush-to-zero; 2^-inf = +0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct AttnArgs {
  const Ctl* ctl;
  bf16* o;           // [Mmax, d] output (nsplit == 1)
  float* opart;      // [nsplit, Mmax, d] unnormalised partial outputs (nsplit > 1)
  float* mlpart;     // [nsplit, Mmax, heads, 2] running max (log2 units) and row sum
  int Lc, d, heads, nsplit, tiles_per_split, m_max, batch;
};

template <int HD>
__global__ void __launch_bounds__(384, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, AttnArgs g, int* err) {
  using Cfg = AttnCfg<HD>;
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int QB = Cfg::QBUF;
  uint8_t* sQ = smem;                                         // QB buffers
  uint8_t* sK = sQ + QB * Cfg::Q_BYTES;
  uint8_t* sV = sK + S * Cfg::KV_BYTES;
  constexpr int PB = Cfg::PB;
  uint8_t* sP = sV + S * Cfg::KV_BYTES;                       // PB tiles
  float* red = reinterpret_cast<float*>(sP + PB * Cfg::P_BYTES);  // [2 tiles][2 halves][128], then [2 halves][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 3 * 2 * 128);
  // bars: kv_full[S], kv_empty[S], q_full[2], q_empty[2], s_full[2], s_free[2], p_full[2], o_done[2],
  //       o_free[2], drain, pair[4 quarters][2 tiles], fin[4]
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  volatile int* abort_flag = &s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();

  const uint32_t kvf0 = smem_u32(bars), kve0 = smem_u32(bars + S);
  const uint32_t qf0 = smem_u32(bars + 2 * S), qe0 = smem_u32(bars + 2 * S + 2);
  const uint32_t sfull0 = smem_u32(bars + 2 * S + 4), sfree0 = smem_u32(bars + 2 * S + 6);
  const uint32_t pfull0 = smem_u32(bars + 2 * S + 8), odone0 = smem_u32(bars + 2 * S + 10);
  const uint32_t ofree0 = smem_u32(bars + 2 * S + 12), drain = smem_u32(bars + 2 * S + 14);
  const uint32_t pair0 = smem_u32(bars + 2 * S + 15), fin0 = smem_u32(bars + 2 * S + 23);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < S; ++i) {
      mbar_init(kvf0 + 8 * i, 1);
      mbar_init(kve0 + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(qf0 + 8 * i, 1);
      mbar_init(qe0 + 8 * i, 1);
      mbar_init(sfull0 + 8 * i, 1);
      mbar_init(sfree0 + 8 * i, 256);
      mbar_init(ofree0 + 8 * i, 256);
      mbar_init(pfull0 + 8 * i, 256);
      mbar_init(odone0 + 8 * i, 1);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(pair0 + 8 * i, 64);
    for (int i = 0; i < 4; ++i) mbar_init(fin0 + 8 * i, 64);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS = tmem, tO = tmem + 2 * BKV;              // S buffers at 0 and 128, O buffers at 256, 256 + hd
  pdl_wait();                                                 // q, the cache and the row layout come from upstream
  const Ctl* ctl = g.ctl;
  const int R = ctl->R, p0 = ctl->p0;
  const int q_tiles = (R + BQ - 1) / BQ;
  const int n_items = q_tiles * g.heads * g.batch * g.nsplit;

  // Work item -> (query tile, head, sample, key split) and its key-tile range.
  // The query tile varies slowest and the last (causally heaviest) tiles come
  // first, so CTAs taking items round-robin get a balanced mix of work.
  struct Item { int qt, hh, s, split, q_begin, t0, nt; };
  const int per_qt = g.heads * g.batch * g.nsplit;
  auto item_of = [&](int it) {
    Item x;
    x.qt = q_tiles - 1 - it / per_qt;
    int r = it % per_qt;
    x.hh = r % g.heads;
    r /= g.heads;
    x.split = r % g.nsplit;
    x.s = r / g.nsplit;
    x.q_begin = x.qt * BQ;
    const int q_end = min(x.q_begin + BQ, R);
    const int ntiles = (p0 + q_end - 1) / BKV + 1;          // key tiles up to the last needed key
    x.t0 = x.split * g.tiles_per_split;
    x.nt = min(ntiles, x.t0 + g.tiles_per_split) - x.t0;
    return x;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      int gi = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const Item x = item_of(it);
        if (x.nt <= 0) continue;
        const int qb = gi % QB;
        if (gi >= QB && !mbar_wait(qe0 + 8 * qb, (uint32_t)(((gi - QB) / QB) & 1), abort_flag)) break;
        mbar_expect_tx(qf0 + 8 * qb, Cfg::Q_BYTES);
#pragma unroll
        for (int kc = 0; kc < Cfg::KCH; ++kc)
          tma_load_2d(smem_u32(sQ + qb * Cfg::Q_BYTES + kc * Cfg::BOX), &tmQ, qf0 + 8 * qb, x.hh * HD + kc * 64,
                      x.s * R + x.q_begin);
        for (int j = 0; j < x.nt; ++j) {
          if (!mbar_wait(kve0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_expect_tx(kvf0 + 8 * stage, 2 * Cfg::KV_BYTES);
          const int key0 = (x.t0 + j) * BKV;
#pragma unroll
          for (int kc = 0; kc < Cfg::KCH; ++kc) {
            tma_load_2d(smem_u32(sK + stage * Cfg::KV_BYTES + kc * Cfg::BOX), &tmK, kvf0 + 8 * stage,
                        x.hh * HD + kc * 64, x.s * g.Lc + key0);
            tma_load_2d(smem_u32(sV + stage * Cfg::KV_BYTES + kc * Cfg::BOX), &tmV, kvf0 + 8 * stage,
                        x.hh * HD + kc * 64, x.s * g.Lc + key0);
          }
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        ++gi;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0, pstage = 0;
      uint32_t phase = 0;
      int gt = 0, gi = 0;                                     // global tile and item counters
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const Item x = item_of(it);
        if (x.nt <= 0) continue;
        const int qb = gi % QB, ob = gi & 1;
        if (!mbar_wait(qf0 + 8 * qb, (uint32_t)((gi / QB) & 1), abort_flag)) break;
        if (gi >= 2 && !mbar_wait(ofree0 + 8 * ob, (uint32_t)(((gi - 2) >> 1) & 1), abort_flag)) break;
        tc_fence_after();
        const uint32_t dO = tO + ob * HD;
        auto issue_pv = [&](int j, int gtile) -> bool {       // O += P_j V_j
          const int pb = gtile % PB;
          if (!mbar_wait(pfull0 + 8 * pb, (uint32_t)((gtile / PB) & 1), abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < BKV / 16; ++ks) {
            const uint64_t da = desc_k(smem_u32(sP + pb * Cfg::P_BYTES + (ks >> 2) * Cfg::BOX + (ks & 3) * 32));
            const uint64_t db = desc_mn(smem_u32(sV + pstage * Cfg::KV_BYTES + ks * 16 * 128), Cfg::BOX);
            umma(dO, da, db, Cfg::IDESC_O, (j > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(odone0 + 8 * pb);
          umma_commit(kve0 + 8 * pstage);
          if (++pstage == S) pstage = 0;
          return true;
        };
        for (int j = 0; j < x.nt; ++j) {
          const int gtile = gt + j;
          if (!mbar_wait(kvf0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          const int b = gtile & 1;
          if (gtile >= 2 && !mbar_wait(sfree0 + 8 * b, (uint32_t)(((gtile - 2) >> 1) & 1), abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint32_t off = (ks >> 2) * Cfg::BOX + (ks & 3) * 32;
            umma(tS + b * BKV, desc_k(smem_u32(sQ + qb * Cfg::Q_BYTES + off)),
                 desc_k(smem_u32(sK + stage * Cfg::KV_BYTES + off)), Cfg::IDESC_S, ks > 0 ? 1u : 0u);
          }
          umma_commit(sfull0 + 8 * b);
          if (j == x.nt - 1) umma_commit(qe0 + 8 * qb);       // the item's Q is no longer read
          if (++stage == S) { stage = 0; phase ^= 1u; }
          if (j >= 1 && !issue_pv(j - 1, gtile - 1)) { ok = false; break; }
        }
        if (!ok || !issue_pv(x.nt - 1, gt + x.nt - 1)) break;
        gt += x.nt;
        ++gi;
      }
      umma_commit(drain);
      const uint64_t tw = globaltimer_ns();
      while (!mbar_try(drain, 0)) {
        if (globaltimer_ns() - tw > kWaitLimitNs) { atomicExch(err, ERR_ATTN_WAIT); break; }
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------------- softmax
    const int ew = warp - 4;
    const int q = ew & 3, hf = ew >> 2;
    const int row = q * 32 + lane;                            // 0..127 within the query tile
    const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int gt = 0, gi = 0;
    bool alive = true;
    for (int it = blockIdx.x; alive && it < n_items; it += gridDim.x) {
      const Item x = item_of(it);
      const int rloc = x.q_begin + row;
      const size_t mrow = (size_t)x.s * R + rloc;
      if (x.nt <= 0) {
        // nothing to attend in this split: an empty partial (m = -inf, l = 0)
        if (hf == 0 && rloc < R) {
          float* ml = g.mlpart + (((size_t)x.split * g.m_max + mrow) * g.heads + x.hh) * 2;
          ml[0] = -INFINITY;
          ml[1] = 0.f;
        }
        continue;
      }
      const int qpos = p0 + rloc;
      const int qpos_min = p0 + x.q_begin;
      const int ob = gi & 1;
      float m_use = -INFINITY, l = 0.f;
      int j = 0;
      for (; j < x.nt; ++j) {
        const int gtile = gt + j;
        const int b = gtile & 1;
        // every wait's outcome is made warp-uniform before any .aligned TMEM access
        if (!__all_sync(0xffffffffu, mbar_wait(sfull0 + 8 * b, (uint32_t)((gtile >> 1) & 1), abort_flag))) break;
        tc_fence_after();
        const int key0 = (x.t0 + j) * BKV + hf * 64;
        const bool need_mask = (x.t0 + j) * BKV + BKV - 1 > qpos_min;
        const uint32_t sa = tS + b * BKV + hf * 64 + lane_off;
        // pass 1: row max.  The scores stay in registers for pass 2; the max is
        // taken on raw scores and scaled once (the scale is positive).
        float v[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16) tmem_ld16(sa + c, v + c);
        tmem_wait_ld();
        float mraw = -INFINITY;
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (key0 + i <= qpos) mraw = fmaxf(mraw, v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) mraw = fmaxf(mraw, v[i]);
        }
        float mx = mraw * sl2;
        float* rd = red + (b * 2) * 128;
        rd[hf * 128 + row] = mx;
        mbar_arrive(pair0 + 8 * (q * 2 + b));
        if (!__all_sync(0xffffffffu, mbar_wait(pair0 + 8 * (q * 2 + b), (uint32_t)((gtile >> 1) & 1), abort_flag))) break;
        mx = fmaxf(mx, rd[(1 - hf) * 128 + row]);
        const float m_new = fmaxf(m_use, mx);
        // raise the running max lazily; rows decide alone, the TMEM rescale of O
        // runs for the whole warp when any of its rows needs it (factor 1 for the rest)
        float corr = 1.f;
        if (m_new > m_use + kRescaleLog2 || m_use == -INFINITY) {
          if (m_use != -INFINITY) corr = exp2f(m_use - m_new);
          l *= corr;
          m_use = m_new;
        }
        if (j >= 1 && __any_sync(0xffffffffu, corr != 1.f)) {
          // O holds tiles 0..j-1: wait for P_{j-1} V_{j-1}
          const int gp = gtile - 1;
          if (!__all_sync(0xffffffffu, mbar_wait(odone0 + 8 * (gp % PB), (uint32_t)((gp / PB) & 1), abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD / 2; c += 16) {
            float v[16];
            const uint32_t oa = tO + ob * HD + hf * (HD / 2) + c + lane_off;
            tmem_ld16(oa, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= corr;
            tmem_st16(oa, v);
          }
          tmem_wait_st();
        }
        // the P tile this tile writes was last read by tile gtile - PB
        const int pb = gtile % PB;
        if (gtile >= PB &&
            !__all_sync(0xffffffffu, mbar_wait(odone0 + 8 * pb, (uint32_t)(((gtile - PB) / PB) & 1), abort_flag)))
          break;
        // pass 2: P = 2^(s * scale - m) in bf16 into the swizzled P tile, row sums;
        // masked keys are exactly 0
        const float nmb = (m_use == -INFINITY) ? 0.f : -m_use;
        uint8_t* prow = sP + pb * Cfg::P_BYTES + hf * Cfg::BOX + row * 128;
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            float e0 = ex2_approx(fmaf(v[c + i], sl2, nmb));
            float e1 = ex2_approx(fmaf(v[c + i + 1], sl2, nmb));
            if (need_mask) {
              if (key0 + c + i > qpos) e0 = 0.f;
              if (key0 + c + i + 1 > qpos) e1 = 0.f;
            }
            l += e0 + e1;
            pk[i >> 1] = pack_bf16(e0, e1);
          }
          const int u0 = c >> 3;                             // 16-byte units u0, u0+1 of this row
          *reinterpret_cast<uint4*>(prow + (((u0) ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(prow + (((u0 + 1) ^ (row & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(pfull0 + 8 * pb);
        mbar_arrive(sfree0 + 8 * b);
      }
      // item epilogue: wait for its last O, combine the halves' row sums, write out
      const int glast = gt + x.nt - 1;
      const bool ok = __all_sync(0xffffffffu, (j == x.nt) && mbar_wait(odone0 + 8 * (glast % PB),
                                                                        (uint32_t)((glast / PB) & 1), abort_flag));
      tc_fence_after();
      float* rl = red + 4 * 128;                               // past both row-max slots
      rl[hf * 128 + row] = l;
      mbar_arrive(fin0 + 8 * q);
      const bool ok2 = __all_sync(0xffffffffu, mbar_wait(fin0 + 8 * q, (uint32_t)(gi & 1), abort_flag));
      const float lt = l + rl[(1 - hf) * 128 + row];
      const bool valid = ok && ok2 && rloc < R;
#pragma unroll
      for (int c = 0; c < HD / 2; c += 16) {
        float v[16];
        tmem_ld16(tO + ob * HD + hf * (HD / 2) + c + lane_off, v);
        tmem_wait_ld();
        const int col = x.hh * HD + hf * (HD / 2) + c;
        if (!valid) continue;
        if (g.nsplit == 1) {
          const float inv = 1.f / lt;
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) pk[i >> 1] = pack_bf16(v[i] * inv, v[i + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(g.o + mrow * g.d + col);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          float4* dst = reinterpret_cast<float4*>(g.opart + ((size_t)x.split * g.m_max + mrow) * g.d + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      if (valid && g.nsplit > 1 && hf == 0) {
        float* ml = g.mlpart + (((size_t)x.split * g.m_max + mrow) * g.heads + x.hh) * 2;
        ml[0] = m_use;
        ml[1] = lt;
      }
      // the O buffer and the row-sum slots are free for the item after next
      tc_fence_before();
      mbar_arrive(ofree0 + 8 * ob);
      alive = ok && ok2;
      gt += x.nt;
      ++gi;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (threadIdx.x == 0 && s_abort) atomicExch(err, ERR_ATTN_WAIT);
}

// Merge the splits' partials: o = sum_i 2^(m_i - m) o_i / sum_i 2^(m_i - m) l_i.
template <int HD>
__global__ void __launch_bounds__(256) k_attn_combine(AttnArgs g) {
  pdl_trigger();
  pdl_wait();
  const int wg = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int M = g.ctl->M;
  if (wg >= M * g.heads) return;
  const int row = wg / g.heads, hh = wg - row * g.heads;
  float mx = -INFINITY;
  for (int i = 0; i < g.nsplit; ++i) mx = fmaxf(mx, g.mlpart[(((size_t)i * g.m_max + row) * g.heads + hh) * 2]);
  constexpr int PER = HD / 32;
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  float lsum = 0.f;
  for (int i = 0; i < g.nsplit; ++i) {
    const float* ml = g.mlpart + (((size_t)i * g.m_max + row) * g.heads + hh) * 2;
    if (ml[0] == -INFINITY) continue;
    const float w = exp2f(ml[0] - mx);
    lsum += w * ml[1];
    const float* op = g.opart + ((size_t)i * g.m_max + row) * g.d + hh * HD;
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] = fmaf(w, op[lane + 32 * k], acc[k]);
  }
  const float inv = 1.f / lsum;
#pragma unroll
  for (int k = 0; k < PER; ++k) g.o[(size_t)row * g.d + hh * HD + lane + 32 * k] = __float2bfloat16_rn(acc[k] * inv);
}

template <int HD>
void launch_hd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& g, int batch,
               int r_max, int* err, cudaStream_t st) {
  using Cfg = AttnCfg<HD>;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_attn_tc<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
    attr = true;
  }
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const long long items = (long long)((r_max + BQ - 1) / BQ) * g.heads * batch * g.nsplit;
  const int grid = (int)(items < sms ? items : sms);
  launch_k(k_attn_tc<HD>, dim3(grid), dim3(384), Cfg::SMEM, st, tq, tk, tv, g, err);
  if (g.nsplit > 1) {
    const long long warps = (long long)g.m_max * g.heads;
    launch_k(k_attn_combine<HD>, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0, st, g);
  }
}

}  // namespace

int attn_tc_splits(int batch, int heads, int r_max, int Lc, int num_sms) {
  const int q_tiles = (r_max + BQ - 1) / BQ;
  const long long ctas = (long long)q_tiles * heads * batch;
  if (ctas >= 2LL * num_sms) return 1;
  const int key_tiles = (Lc + BKV - 1) / BKV;
  int n = (key_tiles + 15) / 16;
  if (n < 1) n = 1;
  if (n > 64) n = 64;
  return n;
}

bool launch_attn_tc2(const Ctl* ctl, const bf16* q, const bf16* kc, const bf16* vc, bf16* o, float* opart,
                     float* mlpart, int nsplit, int batch, int Lc, int d, int heads, int r_max, int m_max, int* err,
                     cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16(&tq, q, m_max, d, 128) || !make_tmap_bf16(&tk, kc, batch * Lc, d, 128) ||
      !make_tmap_bf16(&tv, vc, batch * Lc, d, 128))
    return false;
  AttnArgs g;
  g.ctl = ctl;
  g.o = o;
  g.opart = opart;
  g.mlpart = mlpart;
  g.Lc = Lc;
  g.d = d;
  g.heads = heads;
  g.nsplit = nsplit;
  const int key_tiles = (Lc + BKV - 1) / BKV;
  g.tiles_per_split = (key_tiles + nsplit - 1) / nsplit;
  g.m_max = m_max;
  g.batch = batch;
  if (d / heads == 64) launch_hd<64>(tq, tk, tv, g, batch, r_max, err, st);
  else launch_hd<128>(tq, tk, tv, g, batch, r_max, err, st);
  return true;
}

}  // namespace af
