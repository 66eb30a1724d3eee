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
// of one (sample, head) against the 64-key tiles of one split of the key
// range.  A CTA's items alternate between two groups, each a complete pipeline
// with its own producer, MMA issuer, softmax warps and shared-memory buffers;
// the groups share only the tensor core, the exponential units and (disjoint
// columns of) TMEM, so one group's exponentials overlap the other's loads,
// row maxima, MMA waits and output.  Per group:
//   warp 0 / 2  TMA: the item's Q (128 x hd; the next item's Q is prefetched
//               when two buffers fit), then per tile K into a short ring (read
//               only by S = Q K^T) and V into its own ring; 128-byte swizzle.
//   warp 1 / 3  one thread issues S_t = Q K_t^T (M=128, N=64, K=hd) into the
//               group's TMEM S as soon as the softmax has taken S_{t-1} into
//               registers, and O += P_{t-1} V_{t-1} (M=128, N=hd, K=64) into
//               its TMEM O once that P is written; V is consumed in its
//               natural [key][hd] layout (MN-major).
//   warps 4-7 / 8-11  softmax: one thread per query row holds the tile's 64
//               scores in registers, takes the row max, and writes P =
//               exp2(t - m) as bf16 into one of the group's two swizzled P
//               tiles with the row sum kept in fp32.  Warps whose 32 rows are
//               all outside the sample, and 16-key chunks that the causal mask
//               removes for all of a warp's rows, skip the arithmetic (masked
//               chunks are written as zeros).  The running max is raised
//               lazily: O (in TMEM) and the row sum are rescaled only when the
//               max grows by more than 2^8, which keeps every P below 256 and
//               the result exact.
// With several splits, each writes an unnormalised (o, m, l) partial and
// k_attn_combine merges them.  Every wait is bounded (2 s); on expiry the CTA
// drains, frees TMEM and reports ERR_ATTN_WAIT.
#include "af_kernels.h"

namespace af {
namespace {

constexpr int BQ = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kAttnThreads = 384;

template <int HD> struct AttnCfg {
  static constexpr int BKV = 64;                          // keys per tile
  static constexpr int KCH = HD / 64;                     // 64-column boxes per q / k / v row
  static constexpr uint32_t QBOX = BQ * 128;              // 128 rows x 64 bf16: 16 KB
  static constexpr uint32_t KVBOX = BKV * 128;            // BKV rows x 64 bf16
  static constexpr uint32_t Q_BYTES = KCH * QBOX;
  static constexpr uint32_t KV_BYTES = KCH * KVBOX;       // one K or one V tile
  // Per group: QB Q buffers (the next item's Q prefetched when two fit), a K
  // ring (a K tile is read only by its S = Q K^T), a V ring (held until P V)
  // and PB P tiles.
  // hd 128 keeps one P tile, so that its V ring (the cache of a long video
  // is read from HBM) can hold two tiles.
  static constexpr int QB = HD == 64 ? 2 : 1;
  static constexpr int PB = HD == 64 ? 2 : 1;
  static constexpr int SK = 2, SV = HD == 64 ? 4 : 2;
  static constexpr uint32_t P_BYTES = QBOX;               // 128 rows x 64 keys
  static constexpr uint32_t GROUP_BYTES = QB * Q_BYTES + (SK + SV) * KV_BYTES + PB * P_BYTES;
  // barriers per group: QF[QB] QE[QB] KF[SK] KE[SK] VF[SV] VE[SV] SF SR PF[2] OD[2] OR DRAIN
  static constexpr int GBARS = 2 * QB + 2 * SK + 2 * SV + 8;
  static constexpr size_t SMEM = 1024 + 2 * (size_t)GROUP_BYTES + 2 * GBARS * 8;
  // S = Q K^T: M 128, N BKV, both K-major
  static constexpr uint32_t IDESC_S = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BKV >> 3) << 17) |
                                      ((uint32_t)(BQ >> 4) << 24);
  // O += P V: M 128, N hd, A (P) K-major, B (V) MN-major
  static constexpr uint32_t IDESC_O = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(HD >> 3) << 17) | ((uint32_t)(BQ >> 4) << 24);
};
static_assert(AttnCfg<64>::SMEM <= 232448 && AttnCfg<128>::SMEM <= 232448, "attention shared memory");

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
// The CTA's abort flag and the limit of its pipeline waits (the model's
// wait limit, 2 s by default; the drains after an abort keep kWaitLimitNs).
struct Abort {
  volatile int* flag;
  uint64_t limit_ns;
};
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
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_fast(uint32_t bar, uint32_t parity, const Abort& ab) {
  return mbar_try(bar, parity) || mbar_wait(bar, parity, ab);
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

// TMA bulk store of a staged tile (one thread), tracked as a bulk async-group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
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
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Which keys a query attends: token-causal (key <= query position) when F is
// 0; otherwise by frames of F tokens -- every key of the query's frame and of
// the `ahead` frames after it, never past the sequence (Lc positions).  The
// last attended key is nondecreasing in the query position.
struct KeyMask {
  int F, ahead, Lc;
  __host__ __device__ __forceinline__ int limit(int p) const {
    if (F == 0) return p;
    const int e = (p / F + 1 + ahead) * F;
    return (e < Lc ? e : Lc) - 1;
  }
};

struct AttnArgs {
  const Ctl* ctl;
  bf16* o;           // [Mmax, d] output (one split)
  float* opart;      // [nsplit_max, Mmax, d] unnormalised partial outputs (several splits)
  float* mlpart;     // [nsplit_max, Mmax, heads, 2] running max (log2 units) and row sum
  int Lc, d, heads, nsplit_max, m_max, batch, sms;
  uint64_t wait_ns;  // limit of a pipeline wait before the CTA aborts
  KeyMask km;        // which keys a query attends
  int l2_keep;       // output stored with an L2 evict_last policy (read by the next GEMM at once)
};

// Key splits of a pass, decided from the rows the pass really has (ctl->R
// query rows per sample at positions p0 ..) rather than from the cache's
// length: a pass whose (query tile, head, sample) items already give every SM
// one runs unsplit; otherwise the live key range (keys 0 .. p0 + R - 1) is cut
// into up to nsplit_max splits of at least kMinSplitTiles 64-key tiles, aiming
// at about one item per SM.  (Two per SM, one per pipeline of a CTA, was
// measured 4% slower on the deep flow's 390-row passes: the two pipelines of a
// CTA share its SM, and more splits mean more partials for the combine kernel
// to read.)  The attention kernel and the combine kernel evaluate this from
// the same control block, so they agree.
constexpr int kMinSplitTiles = 8;
constexpr int kMaxSplits = 32;
constexpr int kMaxDevices = 64;
struct SplitPlan { int q_tiles, nsplit, tps; };
__host__ __device__ __forceinline__ SplitPlan split_plan(int R, int p0, int heads, int batch, int nsplit_max,
                                                         int sms, int bkv, const KeyMask& km) {
  SplitPlan sp;
  sp.q_tiles = (R + BQ - 1) / BQ;
  const int live = km.limit(p0 + R - 1) / bkv + 1;        // key tiles up to the last key any row needs
  const int base = sp.q_tiles * heads * batch;
  int n = 1;
  if (nsplit_max > 1 && base < sms) {
    const int want = (sms + base - 1) / base;
    const int by_len = (live + kMinSplitTiles - 1) / kMinSplitTiles;
    n = want < by_len ? want : by_len;
    if (n > nsplit_max) n = nsplit_max;
    if (n < 1) n = 1;
  }
  sp.tps = (live + n - 1) / n;
  sp.nsplit = (live + sp.tps - 1) / sp.tps;
  return sp;
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, AttnArgs g,
              int* err) {
  using Cfg = AttnCfg<HD>;
  constexpr int BKV = Cfg::BKV, QB = Cfg::QB, PB = Cfg::PB, SK = Cfg::SK, SV = Cfg::SV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  volatile int* abort_flag = &s_abort;
  const Abort ab{abort_flag, g.wait_ns};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // group of this warp: warps 0, 1 and 4-7 serve group 0; warps 2, 3 and 8-11 group 1
  const int grp = warp < 4 ? (warp >> 1) : ((warp - 4) >> 2);
  pdl_trigger();

  // this group's shared memory: [Q buffers][K ring][V ring][P tiles]
  uint8_t* gs = smem + grp * Cfg::GROUP_BYTES;
  uint8_t* sQ = gs;
  uint8_t* sK = sQ + QB * Cfg::Q_BYTES;
  uint8_t* sV = sK + SK * Cfg::KV_BYTES;
  uint8_t* sP = sV + SV * Cfg::KV_BYTES;
  const uint32_t bars0 = smem_u32(smem + 2 * Cfg::GROUP_BYTES);
  const uint32_t gb = bars0 + 8u * (uint32_t)(grp * Cfg::GBARS);
  const uint32_t QF = gb, QE = QF + 8 * QB, KF = QE + 8 * QB, KE = KF + 8 * SK, VF = KE + 8 * SK,
                 VE = VF + 8 * SV, SF = VE + 8 * SV, SR = SF + 8, PF = SR + 8, OD = PF + 16, OR = OD + 16,
                 DRAIN = OR + 8;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < 2 * Cfg::GBARS; ++i) {
      // arrival counts: SR, PF and OR take one arrival per softmax thread of the group
      const int k = i % Cfg::GBARS;
      const int sr = 2 * QB + 2 * SK + 2 * SV + 1;
      const bool many = k == sr || k == sr + 1 || k == sr + 2 || k == sr + 5;
      mbar_init(bars0 + 8 * i, many ? 128 : 1);
    }
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
  // TMEM columns: S of groups 0 and 1 at 0 and BKV, O of groups 0 and 1 at 2 BKV and 2 BKV + hd
  const uint32_t tS = tmem + grp * BKV, tO = tmem + 2 * BKV + grp * HD;
  pdl_wait();                                                 // q, the cache and the row layout come from upstream
  const Ctl* ctl = g.ctl;
  const int R = ctl->R, p0 = ctl->p0;
  const SplitPlan plan = split_plan(R, p0, g.heads, g.batch, g.nsplit_max, g.sms, BKV, g.km);
  const int q_tiles = plan.q_tiles, nsplit = plan.nsplit, tps = plan.tps;
  const int n_items = q_tiles * g.heads * g.batch * nsplit;

  // Work item -> (query tile, head, sample, key split) and its key-tile range.
  // Query tiles end at R, R - 128, ...: the ragged tile is the first one, whose
  // few rows need only the first keys (its rows before 0 are padding).  The
  // query tile varies slowest and the last (causally heaviest) tiles come
  // first, so CTAs taking items round-robin get a balanced mix of work.
  struct Item { int qt, hh, s, split, q_begin, t0, nt; };
  const int per_qt = g.heads * g.batch * nsplit;
  const int pad = q_tiles * BQ - R;
  auto item_of = [&](int it) {
    Item x;
    x.qt = q_tiles - 1 - it / per_qt;
    int r = it % per_qt;
    x.hh = r % g.heads;
    r /= g.heads;
    x.split = r % nsplit;
    x.s = r / nsplit;
    x.q_begin = x.qt * BQ - pad;
    const int q_end = x.q_begin + BQ;
    const int ntiles = g.km.limit(p0 + q_end - 1) / BKV + 1;   // key tiles up to the last needed key
    x.t0 = x.split * tps;
    x.nt = min(ntiles, x.t0 + tps) - x.t0;
    return x;
  };
  // Each pipeline (group g of CTA c) is one of 2 * gridDim.x slots, s =
  // g * gridDim.x + c.  Items (heaviest first) are dealt to the slots in
  // rounds, forward in even rounds and backward in odd ones, so that a slot
  // that took one of the heaviest items of a round takes one of the lightest
  // of the next.  A group's k-th call (k = g, g + 2, ...) is round k / 2;
  // every role of a group walks the same items.
  const int n_slots = 2 * (int)gridDim.x;
  const int my_slot = grp * (int)gridDim.x + (int)blockIdx.x;
  auto global_item = [&](int k) {
    const int r = k >> 1;
    return r * n_slots + ((r & 1) ? n_slots - 1 - my_slot : my_slot);
  };

  if (warp < 4 && (warp & 1) == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA producer of the group
      int iw = 0, kst = 0, vst = 0;
      uint32_t kph = 0, vph = 0;
      long long nq = 0, nk = 0, nv = 0;                       // loads issued per ring
      bool ok = true;
      for (int k = grp; ok; k += 2) {
        const int it = global_item(k);
        if (it >= n_items) break;
        const Item x = item_of(it);
        if (x.nt <= 0) continue;
        // Q buffer iw % QB is free once item iw - QB's last S has been computed.
        // 32-row quarters; group 1 stores them in reverse order, so that on the
        // diagonal its light quarters share a sub-partition with group 0's
        // heavy ones (a softmax warp serves TMEM lanes 32 (warp % 4) ..).
        const int qb = iw % QB;
        if (iw >= QB && !mbar_wait(QE + 8 * qb, (uint32_t)(((iw / QB) - 1) & 1), ab)) break;
        mbar_expect_tx(QF + 8 * qb, Cfg::Q_BYTES);
#pragma unroll
        for (int kc = 0; kc < Cfg::KCH; ++kc)
#pragma unroll
          for (int qq = 0; qq < 4; ++qq)
            tma_load_2d(smem_u32(sQ + qb * Cfg::Q_BYTES + kc * Cfg::QBOX + (grp ? 3 - qq : qq) * 4096), &tmQ,
                        QF + 8 * qb, x.hh * HD + kc * 64, x.s * R + x.q_begin + 32 * qq);
        ++nq;
        for (int j = 0; j < x.nt; ++j) {
          const int krow = x.s * g.Lc + (x.t0 + j) * BKV;
          if (!mbar_wait(KE + 8 * kst, kph ^ 1u, ab)) { ok = false; break; }
          mbar_expect_tx(KF + 8 * kst, Cfg::KV_BYTES);
#pragma unroll
          for (int kc = 0; kc < Cfg::KCH; ++kc)
            tma_load_2d(smem_u32(sK + kst * Cfg::KV_BYTES + kc * Cfg::KVBOX), &tmK, KF + 8 * kst, x.hh * HD + kc * 64,
                        krow);
          ++nk;
          if (++kst == SK) { kst = 0; kph ^= 1u; }
          if (!mbar_wait(VE + 8 * vst, vph ^ 1u, ab)) { ok = false; break; }
          mbar_expect_tx(VF + 8 * vst, Cfg::KV_BYTES);
#pragma unroll
          for (int kc = 0; kc < Cfg::KCH; ++kc)
            tma_load_2d(smem_u32(sV + vst * Cfg::KV_BYTES + kc * Cfg::KVBOX), &tmV, VF + 8 * vst, x.hh * HD + kc * 64,
                        krow);
          ++nv;
          if (++vst == SV) { vst = 0; vph ^= 1u; }
        }
        ++iw;
      }
      if (*abort_flag) {
        // After an abort nothing consumes the loads still in flight: the latest
        // load of every stage of each ring lands before the CTA frees its
        // shared memory (one 2 s limit for the whole drain).
        const uint64_t t0 = globaltimer_ns();
        auto drain_ring = [&](uint32_t full0, int stages, long long issued) {
          const long long n = issued < stages ? issued : stages;
          for (long long jj = 1; jj <= n; ++jj) {
            const long long idx = issued - jj;
            const uint32_t bar = full0 + 8u * (uint32_t)(idx % stages);
            const uint32_t ph = (uint32_t)((idx / stages) & 1);
            while (!mbar_try(bar, ph)) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicOr(err, ERR_DRAIN);
                return;
              }
            }
          }
        };
        drain_ring(QF, QB, nq);
        drain_ring(KF, SK, nk);
        drain_ring(VF, SV, nv);
      }
    }
  } else if (warp < 4) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer of the group
      // Per tile t: S_t = Q K_t^T as soon as the group has taken S_{t-1} into
      // registers, then O += P_{t-1} V_{t-1} once that P is written.
      // Descriptors are formed once; a step adds its offset (16-byte units).
      const uint64_t dq = desc_k(smem_u32(sQ)), dk = desc_k(smem_u32(sK)), dp = desc_k(smem_u32(sP));
      const uint64_t dv = desc_mn(smem_u32(sV), Cfg::KVBOX);
      int iw = 0, kst = 0, vst = 0, t = 0;
      uint32_t kph = 0, vph = 0;
      // the tile whose P*V is pending: V stage and phase, tile within its item, item
      bool pend = false;
      int p_vst = 0, p_vph = 0, p_j = 0, p_iw = 0;
      bool ok = true;
      auto issue_pv = [&]() -> bool {
        const int u = t - 1, pb = u % PB;
        // an item's first P*V overwrites O: the group has read the previous item's O
        if (p_j == 0 && p_iw >= 1 && !wait_fast(OR, (uint32_t)((p_iw - 1) & 1), ab)) return false;
        if (!wait_fast(PF + 8 * pb, (uint32_t)((u / PB) & 1), ab)) return false;
        if (!wait_fast(VF + 8 * p_vst, (uint32_t)p_vph, ab)) return false;
        tc_fence_after();
        const uint64_t a0 = dp + (uint64_t)(pb * (Cfg::P_BYTES >> 4));
        const uint64_t b0 = dv + (uint64_t)(p_vst * (Cfg::KV_BYTES >> 4));
#pragma unroll
        for (int ks = 0; ks < BKV / 16; ++ks)
          umma(tO, a0 + (uint64_t)(ks * 2), b0 + (uint64_t)(ks * (2048 >> 4)), Cfg::IDESC_O, (p_j > 0 || ks > 0) ? 1u : 0u);
        umma_commit(OD + 8 * pb);
        umma_commit(VE + 8 * p_vst);                         // V tile no longer read
        return true;
      };
      for (int k = grp; ok; k += 2) {
        const int it = global_item(k);
        if (it >= n_items) break;
        const Item x = item_of(it);
        if (x.nt <= 0) continue;
        const int qb = iw % QB;
        if (!wait_fast(QF + 8 * qb, (uint32_t)((iw / QB) & 1), ab)) { ok = false; break; }
        const uint64_t aq = dq + (uint64_t)(qb * (Cfg::Q_BYTES >> 4));
        for (int j = 0; j < x.nt; ++j) {
          if (!wait_fast(KF + 8 * kst, kph, ab)) { ok = false; break; }
          if (t >= 1 && !wait_fast(SR, (uint32_t)((t - 1) & 1), ab)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bk = dk + (uint64_t)(kst * (Cfg::KV_BYTES >> 4));
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint64_t off = (uint64_t)((ks >> 2) * (Cfg::QBOX >> 4) + (ks & 3) * 2);
            const uint64_t offk = (uint64_t)((ks >> 2) * (Cfg::KVBOX >> 4) + (ks & 3) * 2);
            umma(tS, aq + off, bk + offk, Cfg::IDESC_S, ks > 0 ? 1u : 0u);
          }
          umma_commit(SF);
          umma_commit(KE + 8 * kst);                         // K tile no longer read
          if (j == x.nt - 1) umma_commit(QE + 8 * qb);       // the item's Q is no longer read
          if (++kst == SK) { kst = 0; kph ^= 1u; }
          if (pend && !issue_pv()) { ok = false; break; }
          pend = true;
          p_vst = vst;
          p_vph = (int)vph;
          p_j = j;
          p_iw = iw;
          if (++vst == SV) { vst = 0; vph ^= 1u; }
          ++t;
        }
        // the item's last P*V at once: the group's epilogue waits for it
        if (ok && pend && !issue_pv()) ok = false;
        pend = false;
        ++iw;
      }
      umma_commit(DRAIN);
      const uint64_t tw0 = globaltimer_ns();
      while (!mbar_try(DRAIN, 0)) {
        if (globaltimer_ns() - tw0 > kWaitLimitNs) { atomicOr(err, ERR_DRAIN); break; }
      }
    }
  } else {
    // -------------------------------------------------------------------- softmax of the group
    const int w = grp;
    const int q = warp & 3;                                   // TMEM lane quarter (warp % 4)
    const int quarter = w ? 3 - q : q;                        // the query rows it holds
    const int row = quarter * 32 + lane;                      // 0..127 within the query tile
    const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t tSw = tS + lane_off, tOw = tO + lane_off;
    uint8_t* prow0 = sP + (q * 32 + lane) * 128;             // P row = TMEM lane
    const int sw = lane & 7;                                  // 128-byte swizzle of this row
    int tw = 0;                                               // tiles this group has consumed
    int stg_buf = -1;                                         // P tile holding this warp's output staging
    bool alive = true;
    for (int k = w; alive; k += 2) {
      const int it = global_item(k);
      if (it >= n_items) break;
      const Item x = item_of(it);
      const int rloc = x.q_begin + row;
      if (x.nt <= 0) {
        // nothing to attend in this split: an empty partial (m = -inf, l = 0)
        if (rloc >= 0 && rloc < R) {
          const size_t mrow = (size_t)x.s * R + rloc;
          float* ml = g.mlpart + (((size_t)x.split * g.m_max + mrow) * g.heads + x.hh) * 2;
          ml[0] = -INFINITY;
          ml[1] = 0.f;
        }
        continue;
      }
      // the last key of this row and the lowest / highest of the warp's rows
      const int qpos = g.km.limit(p0 + rloc);
      const int wrow0 = x.q_begin + quarter * 32;             // the warp's first row
      const bool wvalid = wrow0 + 31 >= 0 && wrow0 < R;       // warp-uniform
      const int qlo = g.km.limit(p0 + max(wrow0, 0)), qhi = g.km.limit(p0 + min(wrow0 + 31, R - 1));
      float m_use = -INFINITY;
      float2 l2 = make_float2(0.f, 0.f);
      int j = 0;
      for (; j < x.nt; ++j) {
        // every wait's outcome is made warp-uniform before any .aligned TMEM access
        if (!__all_sync(0xffffffffu, mbar_wait(SF, (uint32_t)(tw & 1), ab))) break;
        tc_fence_after();
        const int key0 = (x.t0 + j) * BKV;
        // the row's scores move to registers and S is released at once, so the
        // next tile's S = Q K^T overlaps this tile's exponentials
        float v[BKV];
        if (wvalid) {
#pragma unroll
          for (int c = 0; c < BKV; c += 16) tmem_ld16(tSw + c, v + c);
          tmem_wait_ld();
        }
        tc_fence_before();
        mbar_arrive(SR);
        float corr = 1.f;
        if (wvalid) {
          // row max on raw scores (the scale is positive), causal keys only
          float mraw = -INFINITY;
#pragma unroll
          for (int c = 0; c < BKV; c += 16) {
            const int kc0 = key0 + c;
            if (kc0 > qhi) continue;                          // masked for every row of the warp
            if (kc0 + 15 <= qlo) {
#pragma unroll
              for (int i = 0; i < 16; ++i) mraw = fmaxf(mraw, v[c + i]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (kc0 + i <= qpos) mraw = fmaxf(mraw, v[c + i]);
            }
          }
          const float m_new = fmaxf(m_use, mraw * sl2);
          // raise the running max lazily; rows decide alone, the TMEM rescale of O
          // runs for the whole warp when any of its rows needs it (factor 1 for the rest)
          if (m_new > m_use + kRescaleLog2 || m_use == -INFINITY) {
            if (m_use != -INFINITY) corr = exp2f(m_use - m_new);
            l2 = fmul2(l2, splat(corr));
            m_use = m_new;
          }
        }
        // P tile tw % PB is free once the group's P*V of tile tw - PB has completed
        const int pb = tw % PB;
        if (tw >= PB &&
            !__all_sync(0xffffffffu, mbar_wait(OD + 8 * pb, (uint32_t)(((tw / PB) - 1) & 1), ab)))
          break;
        uint8_t* prow = prow0 + pb * Cfg::P_BYTES;
        if (pb == stg_buf) {
          // the output staging of the previous item must have been read by its TMA stores
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
          stg_buf = -1;
        }
        if (wvalid) {
          // P = 2^(s * scale - m) in bf16, masked keys exactly 0
          const float2 nmb = splat((m_use == -INFINITY) ? 0.f : -m_use);
#pragma unroll
          for (int c = 0; c < BKV; c += 16) {
            const int kc0 = key0 + c;
            uint32_t pk[8];
            if (kc0 > qhi) {
#pragma unroll
              for (int i = 0; i < 8; ++i) pk[i] = 0u;
            } else {
              const bool partial = kc0 + 15 > qlo;
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                float2 t = ffma2(make_float2(v[c + i], v[c + i + 1]), splat(sl2), nmb);
                if (partial) {
                  if (kc0 + i > qpos) t.x = -INFINITY;           // 2^-inf = +0
                  if (kc0 + i + 1 > qpos) t.y = -INFINITY;
                }
                const float2 e = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                l2 = fadd2(l2, e);
                pk[i >> 1] = pack_bf16(e.x, e.y);
              }
            }
            const int u0 = c >> 3;                            // 16-byte units u0, u0 + 1 of this row
            *reinterpret_cast<uint4*>(prow + ((u0 ^ sw) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(prow + (((u0 + 1) ^ sw) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if (j >= 1 && __any_sync(0xffffffffu, corr != 1.f)) {
          // the max grew: rescale O, which must hold tiles 0..j-1, before this
          // tile's P*V is issued
          const int tl = tw - 1;
          if (!__all_sync(0xffffffffu, mbar_wait(OD + 8 * (tl % PB), (uint32_t)((tl / PB) & 1), ab)))
            break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD; c += 16) {
            float o[16];
            tmem_ld16(tOw + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              const float2 r2 = fmul2(make_float2(o[i], o[i + 1]), splat(corr));
              o[i] = r2.x;
              o[i + 1] = r2.y;
            }
            tmem_st16(tOw + c, o);
          }
          tmem_wait_st();
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(PF + 8 * pb);
        ++tw;
      }
      // item epilogue: wait for the last P*V, read O, release it, normalise and store
      // (the item's sample, head and split are looked up again here rather than
      // kept in registers through the tile loop)
      const Item xe = item_of(it);
      const size_t mrow = (size_t)xe.s * R + rloc;
      const int tl = tw - 1;
      const bool ok = __all_sync(
          0xffffffffu, (j == x.nt) && mbar_wait(OD + 8 * (tl % PB), (uint32_t)((tl / PB) & 1), ab));
      tc_fence_after();
      const float lt = l2.x + l2.y;
      const bool valid = ok && rloc >= 0 && rloc < R;
      const float inv = 1.f / lt;
      // hd 64, one split: a warp whose 32 rows all lie in the sample stages them
      // (bf16, 32-byte swizzle, 16 columns per 1 KB) in its quarter of a free P
      // tile and writes them with TMA bulk stores; other rows are stored directly
      const int q0 = x.q_begin + quarter * 32;
      const bool tma_out = HD == 64 && nsplit == 1 && ok && q0 >= 0 && q0 + 31 < R;   // warp-uniform
      const int sb = (tw + 1) % PB;                          // the P tile written last by the next item
      uint8_t* stg = sP + sb * Cfg::P_BYTES + q * 4096;
      if (tma_out && stg_buf >= 0) {
        // at most one staging in flight: the previous item's stores have read theirs
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        stg_buf = -1;
      }
      // 32 columns at a time; O is released after the last TMEM read
#pragma unroll
      for (int h0 = 0; h0 < HD; h0 += 32) {
        float o[32];
        if (wvalid && ok) {
          tmem_ld16(tOw + h0, o);
          tmem_ld16(tOw + h0 + 16, o + 16);
          tmem_wait_ld();
        }
        if (h0 + 32 == HD) {
          tc_fence_before();
          mbar_arrive(OR);                           // O may be overwritten by the group's next item
        }
        if (tma_out) {
#pragma unroll
          for (int c = 0; c < 32; c += 16) {
            uint8_t* rp = stg + ((h0 + c) >> 4) * 1024 + lane * 32;
            const int swz = (lane >> 2) & 1;
            *reinterpret_cast<uint4*>(rp + (swz << 4)) =
                make_uint4(pack_bf16(o[c] * inv, o[c + 1] * inv), pack_bf16(o[c + 2] * inv, o[c + 3] * inv),
                           pack_bf16(o[c + 4] * inv, o[c + 5] * inv), pack_bf16(o[c + 6] * inv, o[c + 7] * inv));
            *reinterpret_cast<uint4*>(rp + ((1 ^ swz) << 4)) =
                make_uint4(pack_bf16(o[c + 8] * inv, o[c + 9] * inv), pack_bf16(o[c + 10] * inv, o[c + 11] * inv),
                           pack_bf16(o[c + 12] * inv, o[c + 13] * inv), pack_bf16(o[c + 14] * inv, o[c + 15] * inv));
          }
          continue;
        }
        if (!valid) continue;
        if (nsplit == 1) {
          uint4* dst = reinterpret_cast<uint4*>(g.o + mrow * g.d + xe.hh * HD + h0);
#pragma unroll
          for (int c = 0; c < 32; c += 8)
            dst[c >> 3] = make_uint4(pack_bf16(o[c] * inv, o[c + 1] * inv), pack_bf16(o[c + 2] * inv, o[c + 3] * inv),
                                     pack_bf16(o[c + 4] * inv, o[c + 5] * inv), pack_bf16(o[c + 6] * inv, o[c + 7] * inv));
        } else {
          float4* dst =
              reinterpret_cast<float4*>(g.opart + ((size_t)xe.split * g.m_max + mrow) * g.d + xe.hh * HD + h0);
#pragma unroll
          for (int c = 0; c < 32; c += 4) dst[c >> 2] = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        }
      }
      if (tma_out) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          if (g.l2_keep) {
            const uint64_t pol = policy_evict_last();
            for (int ch = 0; ch < HD / 16; ++ch)
              tma_store_2d_hint(&tmO, smem_u32(stg + ch * 1024), xe.hh * HD + ch * 16, xe.s * R + q0, pol);
          } else {
            for (int ch = 0; ch < HD / 16; ++ch)
              tma_store_2d(&tmO, smem_u32(stg + ch * 1024), xe.hh * HD + ch * 16, xe.s * R + q0);
          }
          bulk_commit();
        }
        stg_buf = sb;
      }
      if (valid && nsplit > 1) {
        float* ml = g.mlpart + (((size_t)xe.split * g.m_max + mrow) * g.heads + xe.hh) * 2;
        ml[0] = m_use;
        ml[1] = lt;
      }
      alive = ok;
    }
    if (lane == 0) bulk_wait_all();                           // the output stores are complete before exit
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(err, ERR_ATTN_WAIT);
}

// Merge the splits' partials: o = sum_i 2^(m_i - m) o_i / sum_i 2^(m_i - m) l_i.
template <int HD>
__global__ void __launch_bounds__(256) k_attn_combine(AttnArgs g) {
  pdl_trigger();
  pdl_wait();
  const int wg = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int M = g.ctl->M;
  const int nsplit = split_plan(g.ctl->R, g.ctl->p0, g.heads, g.batch, g.nsplit_max, g.sms, AttnCfg<HD>::BKV, g.km).nsplit;
  if (nsplit == 1 || wg >= M * g.heads) return;      // one split: the attention kernel wrote o itself
  const int row = wg / g.heads, hh = wg - row * g.heads;
  // lane i holds split i's (max, sum) (nsplit <= kMaxSplits = 32), so the
  // partials' statistics arrive in one round trip; the outputs of all splits
  // are then summed in split order with weights 2^(m_i - max).
  const size_t mstride = (size_t)g.m_max * g.heads * 2;
  const float* mlb = g.mlpart + ((size_t)row * g.heads + hh) * 2;
  float mi = -INFINITY, li = 0.f;
  if (lane < nsplit) {
    const float2 v = *reinterpret_cast<const float2*>(mlb + lane * mstride);
    mi = v.x;
    li = v.y;
  }
  float mx = mi;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float wi = mi == -INFINITY ? 0.f : exp2f(mi - mx);
  float lsum = wi * li;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  constexpr int PER = HD / 32;
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  const float* ob = g.opart + (size_t)row * g.d + hh * HD + lane;
  const size_t ostride = (size_t)g.m_max * g.d;
  for (int i0 = 0; i0 < nsplit; i0 += 4) {
    // four splits' loads in flight before their sums
    float v[4][PER];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int k = 0; k < PER; ++k) v[u][k] = i0 + u < nsplit ? ob[(i0 + u) * ostride + 32 * k] : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float w = __shfl_sync(0xffffffffu, wi, (i0 + u) & 31);
      if (i0 + u < nsplit && w != 0.f) {
#pragma unroll
        for (int k = 0; k < PER; ++k) acc[k] = fmaf(w, v[u][k], acc[k]);
      }
    }
  }
  const float inv = 1.f / lsum;
#pragma unroll
  for (int k = 0; k < PER; ++k) g.o[(size_t)row * g.d + hh * HD + lane + 32 * k] = __float2bfloat16_rn(acc[k] * inv);
}

template <int HD>
bool launch_hd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
               const AttnArgs& g, int batch, int r_max, int* err, cudaStream_t st) {
  using Cfg = AttnCfg<HD>;
  // the shared-memory opt-in is a per-device setting of the function
  static bool attr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (!attr[dev]) {
    if (cudaFuncSetAttribute(k_attn_tc<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM) != cudaSuccess)
      return false;
    attr[dev] = true;
  }
  // an upper bound of the items of any pass with at most r_max rows per sample
  const long long items = (long long)((r_max + BQ - 1) / BQ) * g.heads * batch * g.nsplit_max;
  const int grid = (int)(items < g.sms ? items : g.sms);
  launch_k(k_attn_tc<HD>, dim3(grid), dim3(kAttnThreads), Cfg::SMEM, st, tq, tk, tv, to, g, err);
  if (g.nsplit_max > 1) {
    const long long warps = (long long)g.m_max * g.heads;
    launch_k(k_attn_combine<HD>, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0, st, g);
  }
  return true;
}

}  // namespace

int attn_tc_splits(int batch, int heads, int r_max, int Lc, int num_sms) {
  (void)r_max;
  const int bkv = 64;
  const int base_min = heads * batch;                       // a pass with a single query tile
  if (base_min >= num_sms) return 1;
  const int want = (num_sms + base_min - 1) / base_min;
  const int key_tiles = (Lc + bkv - 1) / bkv;
  const int by_len = (key_tiles + kMinSplitTiles - 1) / kMinSplitTiles;
  int n = want < by_len ? want : by_len;
  if (n > kMaxSplits) n = kMaxSplits;
  return n < 1 ? 1 : n;
}

bool launch_attn_tc2(const Ctl* ctl, const bf16* q, const bf16* kc, const bf16* vc, bf16* o, float* opart,
                     float* mlpart, int nsplit_max, int batch, int Lc, int d, int heads, int r_max, int m_max,
                     int num_sms, uint64_t wait_ns, int mask_frame, int mask_ahead, int l2_keep, int* err,
                     cudaStream_t st) {
  const int hd = d / heads;
  const int bkv = hd == 64 ? AttnCfg<64>::BKV : AttnCfg<128>::BKV;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, m_max, d, 32) || !make_tmap_bf16(&tk, kc, batch * Lc, d, bkv) ||
      !make_tmap_bf16(&tv, vc, batch * Lc, d, bkv) || !make_tmap_out(&to, o, false, m_max, d))
    return false;
  AttnArgs g;
  g.ctl = ctl;
  g.o = o;
  g.opart = opart;
  g.mlpart = mlpart;
  g.Lc = Lc;
  g.d = d;
  g.heads = heads;
  g.nsplit_max = nsplit_max;
  g.m_max = m_max;
  g.batch = batch;
  g.sms = num_sms;
  g.wait_ns = wait_ns;
  g.km.F = mask_frame;
  g.km.ahead = mask_ahead;
  g.km.Lc = Lc;
  g.l2_keep = l2_keep;
  return hd == 64 ? launch_hd<64>(tq, tk, tv, to, g, batch, r_max, err, st)
                  : launch_hd<128>(tq, tk, tv, to, g, batch, r_max, err, st);
}

}  // namespace af
