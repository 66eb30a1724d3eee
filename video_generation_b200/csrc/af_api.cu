// af_api.cu -- the C ABI of libaf (declared in include/af.h): model packing,
// workspace layout, the pass of one AF block, the forward and block-Jacobi
// graphs, and the stacks of alternating-direction blocks.
//
// The AF block and its inverse follow "STARFlow-V: End-to-End Video Generative
// Modeling with Autoregressive Normalizing Flows" (CVPR 2026 paper notes):
// key design 1 (the affine AF equation, alternating-direction stacks) and key
// design 3 (block-wise Jacobi with KV cache, warm start and the tau test).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <map>
#include <string>
#include <vector>

#include "../../include/af.h"
#include "af_kernels.h"

using namespace af;

namespace af {
thread_local int g_pdl = 1;
}

namespace {

thread_local char g_errbuf[512] = "";

void set_err(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_errbuf, sizeof g_errbuf, fmt, ap);
  va_end(ap);
}

#define CK(call)                                                                     \
  do {                                                                               \
    cudaError_t e_ = (call);                                                         \
    if (e_ != cudaSuccess) {                                                         \
      set_err("%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
      return AF_ERR_CUDA;                                                            \
    }                                                                                \
  } while (0)

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

uint16_t f2bf(float f) {     // float -> bfloat16 bits, round to nearest even
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

struct LayerW {
  void *w_qkv, *w_o, *w_1, *w_2;   // bf16 or fp32 [out, in]
  float *ln1_g, *ln1_b, *b_qkv, *b_o, *ln2_g, *ln2_b, *b_1, *b_2;
};

}  // namespace

struct af_model {
  af_config cfg;
  int fd, hd;
  bool bf;
  void* w_in;
  float *b_in, *pos_space, *pos_time;
  std::vector<LayerW> layers;
  float *lnf_g, *lnf_b;
  void* w_head;       // rows interleaved: 2c -> mu_c, 2c+1 -> s_c
  float* b_head;      // interleaved the same way
  int* d_err;
  int num_sms;
  int device;         // the CUDA device holding the weights
  int pdl;            // launch with programmatic dependent launch (see af_kernels.h)
  uint64_t wait_ns;   // limit of one pipeline wait in the tensor-core kernels
  int kind;           // KIND_FLOW (an AF block) or KIND_DENOISER
  int l2_keep;        // keep the hidden state / residual stream / attention output in L2 (evict_last stores)
  std::vector<void*> allocs;
  // graph cache (keyed by every pointer and scalar baked into the graph)
  std::map<std::string, cudaGraphExec_t> graphs;
  std::vector<std::string> graph_order;
  cudaStream_t cap, cap2;   // private streams used for capture only
  cudaEvent_t ev_frame = nullptr, ev_done = nullptr;   // pipelined decoding (created on first use)
};

namespace {

// What an af_model computes: an affine AF block (input shifted by one token,
// token-causal attention, head of interleaved (mu, s) pairs) or the
// flow-score-matching denoiser (input unshifted, attention by frames with one
// frame of look-ahead in the first layer, head of C plain outputs).
enum { KIND_FLOW = 0, KIND_DENOISER = 1 };

// ------------------------------------------------------------------ workspace

struct Bufs {
  Ctl* ctl;
  int* active;
  float* part;
  float* h;
  void* xin;
  void* a;
  void* q;
  void* u;
  void* kv;
  size_t kv_bytes;
  float* tmp;
  int* btab;      // Jacobi block table (af_common.cuh)
  float* opart;   // split-attention partials (bf16 path)
  float* mlpart;
  int nsplit;
  float* kpart;   // split-K partials of the residual GEMMs [ksplit][kpart_rows][d] (bf16 path, few tiles)
  int* ks_out;    // the splits the last residual GEMM used
  int ksplit;     // 1: the residual GEMMs reduce-add into h directly
  int kpart_rows;
  size_t total;
};

// Rows per sample a pass may carry: a Jacobi update of a block of at most B
// tokens, plus the previous block's tokens on the update that commits them.
int rows_per_sample(int L, int B) { return B >= L ? L : (2 * B < L ? 2 * B : L); }

Bufs carve(const af_model* m, void* ws, int batch, int L, int B) {
  const af_config& c = m->cfg;
  const size_t es = m->bf ? 2 : 4;
  const size_t mmax = (size_t)batch * rows_per_sample(L, B);
  const int G = (2 * c.C) / 16;
  Bufs b{};
  size_t off = 0;
  char* base = static_cast<char*>(ws);
  auto take = [&](size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  b.ctl = (Ctl*)take(sizeof(Ctl));
  b.active = (int*)take(sizeof(int) * batch);
  b.part = (float*)take(sizeof(float) * mmax * G * 2);
  b.h = (float*)take(sizeof(float) * mmax * c.d);
  b.xin = take(es * mmax * c.C);
  b.a = take(es * mmax * c.d);
  b.q = take(es * mmax * c.d);
  b.u = take(es * mmax * m->fd);
  b.kv_bytes = es * (size_t)c.layers * 2 * batch * L * c.d;
  b.kv = take(b.kv_bytes);
  b.tmp = (float*)take(sizeof(float) * (size_t)batch * L * c.C);
  b.btab = (int*)take(sizeof(int) * btab_ints(L));
  b.nsplit = m->bf ? attn_tc_splits(batch, c.heads, rows_per_sample(L, B), L, m->num_sms) : 1;
  if (b.nsplit > 1) {
    b.opart = (float*)take(sizeof(float) * (size_t)b.nsplit * mmax * c.d);
    b.mlpart = (float*)take(sizeof(float) * (size_t)b.nsplit * mmax * c.heads * 2);
  }
  b.ksplit = 1;
  if (m->bf) {
    // The residual GEMMs (N = d) split K when the tiles of the fewest rows a
    // pass of this workspace has (half its rows, on a Jacobi workspace whose
    // passes carry one block except on a commit) leave half the SM pairs idle.
    const int pick = gemm_tc_pick(c.d, (int)mmax, m->num_sms, 0, 256);
    const int fewest = B < L ? (int)(mmax / 2) : (int)mmax;
    const int tiles = gemm_tc_tiles(pick, c.d, fewest);
    const int units = pick ? m->num_sms / (pick % 10) : 0;
    if (tiles > 0 && 2 * tiles <= units) {
      b.ksplit = units / tiles < 4 ? units / tiles : 4;
      b.kpart_rows = (int)((mmax + 255) / 256 * 256);
      b.kpart = (float*)take(sizeof(float) * (size_t)b.ksplit * b.kpart_rows * c.d);
      b.ks_out = (int*)take(sizeof(int));
    }
  }
  b.total = off;
  return b;
}

// ------------------------------------------------------------------ one pass

struct HeadIO {
  int mode;             // 0 forward, 1 Jacobi update, 2 denoise
  const float* xin_f;   // forward: x   inverse: z   denoise: x_noisy
  float* xout_f;        // forward: z   inverse: x   denoise: x
  float sigma;          // denoise: the noise level
};

// One pass of the AF block over the rows described by ctl (see af_common.cuh):
// shifted gather, input projection + positions, `layers` pre-LN Transformer
// blocks writing K/V into the cache, final LayerNorm and the fused head.
af_status enqueue_pass(const af_model* m, const Bufs& b, int batch, int L, int dir, int m_max, int r_max,
                       const float* xsrc, const HeadIO& hio, cudaStream_t st) {
  const af_config& c = m->cfg;
  const int d = c.d, C = c.C, fd = m->fd;
  const int G = (2 * C) / 16;
  EpiArgs e{};
  e.ctl = b.ctl;
  e.h = b.h;
  e.d = d;
  e.wait_ns = m->wait_ns;
  e.l2_keep = m->l2_keep;
  e.Lc = L;
  e.pos_space = m->pos_space;
  e.pos_time = m->pos_time;
  e.frame_len = c.frame_len;
  const size_t es = m->bf ? 2 : 4;
  const size_t kv_layer = (size_t)batch * L * d * es;

  EpiArgs eh = e;
  eh.bias = m->b_head;
  eh.head_mode = hio.mode;
  eh.sigma = hio.sigma;
  // the AF block's self-exclusive mask is a one-token input shift with
  // token-causal attention; the denoiser reads its input unshifted and
  // attends by frames, one frame ahead in its first layer only
  const bool den = m->kind == KIND_DENOISER;
  const int shift = den ? 0 : 1;
  const int head_n = den ? C : 2 * C;
  auto mask_frame = [&](int l) { return den ? c.frame_len : 0; };
  auto mask_ahead = [&](int l) { return den && l == 0 ? 1 : 0; };
  eh.L = L;
  eh.C = C;
  eh.dir = dir;
  eh.xin_f = hio.xin_f;
  eh.xout_f = hio.xout_f;
  eh.active = b.active;
  eh.part = b.part;

  if (!m->bf) {
    float* xin = (float*)b.xin;
    float* a = (float*)b.a;
    float* q = (float*)b.q;
    float* u = (float*)b.u;
    launch_gather<float>(b.ctl, xsrc, L, C, dir, shift, xin, m_max, st);
    e.bias = m->b_in;
    launch_gemm_simt(EPI_INPROJ, xin, (const float*)m->w_in, d, C, m_max, e, st);
    for (int l = 0; l < c.layers; ++l) {
      const LayerW& w = m->layers[l];
      char* kvl = (char*)b.kv + 2 * l * kv_layer;
      launch_layernorm<float>(b.ctl, b.h, w.ln1_g, w.ln1_b, a, d, m_max, st);
      EpiArgs eq = e;
      eq.bias = w.b_qkv;
      eq.out = q;
      eq.kc = kvl;
      eq.vc = kvl + kv_layer;
      launch_gemm_simt(EPI_QKV, a, (const float*)w.w_qkv, 3 * d, d, m_max, eq, st);
      launch_attn_simt(b.ctl, q, (const float*)kvl, (const float*)(kvl + kv_layer), a, batch, L, d, c.heads, m_max,
                       mask_frame(l), mask_ahead(l), st);
      EpiArgs eo = e;
      eo.bias = w.b_o;
      launch_gemm_simt(EPI_RESID, a, (const float*)w.w_o, d, d, m_max, eo, st);
      launch_layernorm<float>(b.ctl, b.h, w.ln2_g, w.ln2_b, a, d, m_max, st);
      EpiArgs eu = e;
      eu.bias = w.b_1;
      eu.out = u;
      eu.ldo = fd;
      launch_gemm_simt(EPI_GELU, a, (const float*)w.w_1, fd, d, m_max, eu, st);
      EpiArgs ed = e;
      ed.bias = w.b_2;
      launch_gemm_simt(EPI_RESID, u, (const float*)w.w_2, d, fd, m_max, ed, st);
    }
    launch_layernorm<float>(b.ctl, b.h, m->lnf_g, m->lnf_b, a, d, m_max, st);
    launch_head_simt(a, (const float*)m->w_head, head_n, d, m_max, eh, st);
  } else {
    bf16* xin = (bf16*)b.xin;
    bf16* a = (bf16*)b.a;
    bf16* q = (bf16*)b.q;
    bf16* u = (bf16*)b.u;
    const int ns = m->num_sms;
    CUtensorMap tA_x, tA_a, tA_u, tB, tC_h, tC_u, tC_q, tC_k, tC_v;
    bool ok = make_tmap_bf16(&tA_x, xin, m_max, C, 128) && make_tmap_bf16(&tA_a, a, m_max, d, 128) &&
              make_tmap_bf16(&tA_u, u, m_max, fd, 128) && make_tmap_out(&tC_h, b.h, true, m_max, d) &&
              make_tmap_out(&tC_u, u, false, m_max, fd) && make_tmap_out(&tC_q, q, false, m_max, d);
    if (!ok) { set_err("cuTensorMapEncodeTiled failed for an activation"); return AF_ERR_CUDA; }
    CUtensorMap tC_p;
    if (b.ksplit > 1 && !make_tmap_out(&tC_p, b.kpart, true, b.ksplit * b.kpart_rows, d)) {
      set_err("cuTensorMapEncodeTiled failed for the split-K partials");
      return AF_ERR_CUDA;
    }
    auto gemm = [&](int epi, const CUtensorMap& tA, const void* W, int N, int K, const EpiArgs& ea) -> bool {
      // the position-add epilogue keeps two row sets in flight and stays at
      // <= 192 columns (a QKV tile may span q, K and V: its epilogue places
      // each 16-column chunk)
      const int pick = gemm_tc_pick(N, m_max, ns, 0, epi == EPI_INPROJ ? 192 : 256);
      if (!pick || !make_tmap_bf16(&tB, W, N, K, (pick / 10) / (pick % 10))) return false;
      if (epi == EPI_RESID && b.ksplit > 1) {
        // split K: the partials by TMA store, then one fixed-order sum into h
        EpiArgs ep = ea;
        ep.ksplit = b.ksplit;
        ep.kpart_rows = b.kpart_rows;
        ep.ks_out = b.ks_out;
        launch_gemm_tc(EPI_PART, tA, tB, &tC_p, &tC_h, nullptr, pick, N, K, m_max, ep, m->d_err, ns, st);
        launch_split_sum(b.ctl, b.kpart, b.kpart_rows, N, b.ks_out, ea.bias, b.h, m_max, st);
        return true;
      }
      const CUtensorMap* tC = epi == EPI_RESID ? &tC_h : (epi == EPI_GELU ? &tC_u : (epi == EPI_QKV ? &tC_q : nullptr));
      launch_gemm_tc(epi, tA, tB, tC, epi == EPI_QKV ? &tC_k : nullptr, epi == EPI_QKV ? &tC_v : nullptr, pick, N, K,
                     m_max, ea, m->d_err, ns, st);
      return true;
    };
    launch_gather<bf16>(b.ctl, xsrc, L, C, dir, shift, xin, m_max, st);
    e.bias = m->b_in;
    if (!gemm(EPI_INPROJ, tA_x, m->w_in, d, C, e)) { set_err("GEMM plan failed (in-proj)"); return AF_ERR_CUDA; }
    for (int l = 0; l < c.layers; ++l) {
      const LayerW& w = m->layers[l];
      char* kvl = (char*)b.kv + 2 * l * kv_layer;
      launch_layernorm<bf16>(b.ctl, b.h, w.ln1_g, w.ln1_b, a, d, m_max, st);
      EpiArgs eq = e;
      eq.bias = w.b_qkv;
      eq.out = q;
      eq.kc = kvl;
      eq.vc = kvl + kv_layer;
      if (!make_tmap_out(&tC_k, kvl, false, batch * L, d) || !make_tmap_out(&tC_v, kvl + kv_layer, false, batch * L, d)) {
        set_err("cuTensorMapEncodeTiled failed for the KV cache");
        return AF_ERR_CUDA;
      }
      if (!gemm(EPI_QKV, tA_a, w.w_qkv, 3 * d, d, eq)) { set_err("GEMM plan failed (qkv)"); return AF_ERR_CUDA; }
      if (!launch_attn_tc2(b.ctl, q, (const bf16*)kvl, (const bf16*)(kvl + kv_layer), a, b.opart, b.mlpart, b.nsplit,
                           batch, L, d, c.heads, r_max, m_max, m->num_sms, m->wait_ns, mask_frame(l), mask_ahead(l),
                           m->l2_keep, m->d_err, st)) {
        set_err("attention plan failed");
        return AF_ERR_CUDA;
      }
      EpiArgs eo = e;
      eo.bias = w.b_o;
      if (!gemm(EPI_RESID, tA_a, w.w_o, d, d, eo)) { set_err("GEMM plan failed (out)"); return AF_ERR_CUDA; }
      launch_layernorm<bf16>(b.ctl, b.h, w.ln2_g, w.ln2_b, a, d, m_max, st);
      EpiArgs eu = e;
      eu.bias = w.b_1;
      eu.out = u;
      eu.ldo = fd;
      if (!gemm(EPI_GELU, tA_a, w.w_1, fd, d, eu)) { set_err("GEMM plan failed (mlp up)"); return AF_ERR_CUDA; }
      EpiArgs ed = e;
      ed.bias = w.b_2;
      if (!gemm(EPI_RESID, tA_u, w.w_2, d, fd, ed)) { set_err("GEMM plan failed (mlp down)"); return AF_ERR_CUDA; }
    }
    launch_layernorm<bf16>(b.ctl, b.h, m->lnf_g, m->lnf_b, a, d, m_max, st);
    if (!gemm(den ? EPI_DENOISE : EPI_HEAD, tA_a, m->w_head, head_n, d, eh)) {
      set_err("GEMM plan failed (head)");
      return AF_ERR_CUDA;
    }
  }
  (void)G;
  CK(cudaGetLastError());
  return AF_OK;
}

// ------------------------------------------------------------------ graphs

af_status add_while(cudaStream_t cs, cudaGraphConditionalHandle* h, unsigned dflt, unsigned flags,
                    cudaGraph_t* body) {
  cudaStreamCaptureStatus stat;
  cudaGraph_t g;
  const cudaGraphNode_t* deps = nullptr;
  size_t nd = 0;
  CK(cudaStreamGetCaptureInfo(cs, &stat, nullptr, &g, &deps, &nd));
  if (stat != cudaStreamCaptureStatusActive) { set_err("stream not capturing"); return AF_ERR_CUDA; }
  CK(cudaGraphConditionalHandleCreate(h, g, dflt, flags));
  alignas(cudaGraphNodeParams) unsigned char pbuf[sizeof(cudaGraphNodeParams)] = {};
  cudaGraphNodeParams& p = *reinterpret_cast<cudaGraphNodeParams*>(pbuf);
  p.type = cudaGraphNodeTypeConditional;
  p.conditional.handle = *h;
  p.conditional.type = cudaGraphCondTypeWhile;
  p.conditional.size = 1;
  cudaGraphNode_t node;
  CK(cudaGraphAddNode(&node, g, deps, nd, &p));
  *body = p.conditional.phGraph_out[0];
  CK(cudaStreamUpdateCaptureDependencies(cs, &node, 1, cudaStreamSetCaptureDependencies));
  return AF_OK;
}

struct JacobiJob {
  const af_model* m;
  const float* z;
  float* x;
  int dir;
  int32_t* iters;
  bool reset_nonconv;
};

// Block schedule of a Jacobi call, as held on the host before it is written
// to the workspace's block table.
struct Schedule {
  std::vector<int> starts;   // nb + 1 start positions, the last = L
  int b_begin, b_end;
  int B_max;                 // the largest block
  bool uniform;              // every block the same size
};

Schedule uniform_schedule(int L, int B) {
  Schedule sc;
  for (int p = 0; p <= L; p += B) sc.starts.push_back(p);
  sc.b_begin = 0;
  sc.b_end = L / B;
  sc.B_max = B;
  sc.uniform = true;
  return sc;
}

// Capture the block-Jacobi inverse of one AF block into the stream `cs`,
// which is capturing: [call init] WHILE(blocks) { [block init]
// WHILE(updates) { pass; [jacobi step] } [block advance] }.
// The block sizes, the number of blocks and the range of blocks come from the
// workspace's block table at run time; B_max (the largest block) sizes the
// passes, so one graph serves every schedule and range with that bound.
af_status capture_jacobi(const JacobiJob& jb, const Bufs& b, int batch, int L, int B_max, float tau, int max_iter,
                         int warm, cudaStream_t cs) {
  const af_model* m = jb.m;
  const int G = (2 * m->cfg.C) / 16;
  const int r_max = rows_per_sample(L, B_max);
  const int m_max = batch * r_max;
  launch_call_init(b.ctl, b.btab, jb.reset_nonconv ? 1 : 0, cs);
  cudaGraphConditionalHandle h_outer, h_inner;
  cudaGraph_t body_outer, body_inner;
  af_status s = add_while(cs, &h_outer, 1, cudaGraphCondAssignDefault, &body_outer);
  if (s) return s;
  // The outer body and the inner body are captured with a second private stream.
  cudaStream_t cs2 = m->cap2;
  af_status rc = AF_OK;
  do {
    if (cudaStreamBeginCaptureToGraph(cs2, body_outer, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
      set_err("capture of the block loop failed"); rc = AF_ERR_CUDA; break;
    }
    // the inner handle lives in the outer body; block init sets it to 1
    cudaStreamCaptureStatus stat;
    cudaGraph_t gcap;
    if (cudaStreamGetCaptureInfo(cs2, &stat, nullptr, &gcap, nullptr, nullptr) != cudaSuccess ||
        cudaGraphConditionalHandleCreate(&h_inner, gcap, 0, 0) != cudaSuccess) {
      set_err("conditional handle creation failed"); rc = AF_ERR_CUDA;
    }
    if (!rc) {
      // bf16: V rows of layer l at kv + (2l + 1) * (batch * L * d) elements
      const size_t kv_layer = (size_t)batch * L * m->cfg.d * 2;
      bf16* vtail = m->bf ? (bf16*)((char*)b.kv + kv_layer) : nullptr;
      launch_block_init(b.ctl, b.btab, b.active, jb.z, jb.x, batch, L, m->cfg.C, B_max, m->cfg.frame_len, jb.dir, warm,
                        vtail, 2 * kv_layer, m->cfg.layers, m->cfg.d, h_inner, cs2);
      cudaStreamCaptureStatus st2;
      cudaGraph_t g2;
      const cudaGraphNode_t* deps = nullptr;
      size_t nd = 0;
      alignas(cudaGraphNodeParams) unsigned char pbuf[sizeof(cudaGraphNodeParams)] = {};
      cudaGraphNodeParams& p = *reinterpret_cast<cudaGraphNodeParams*>(pbuf);
      cudaGraphNode_t node;
      if (cudaStreamGetCaptureInfo(cs2, &st2, nullptr, &g2, &deps, &nd) != cudaSuccess) { rc = AF_ERR_CUDA; }
      else {
        p.type = cudaGraphNodeTypeConditional;
        p.conditional.handle = h_inner;
        p.conditional.type = cudaGraphCondTypeWhile;
        p.conditional.size = 1;
        if (cudaGraphAddNode(&node, g2, deps, nd, &p) != cudaSuccess ||
            cudaStreamUpdateCaptureDependencies(cs2, &node, 1, cudaStreamSetCaptureDependencies) != cudaSuccess) {
          set_err("adding the update loop failed"); rc = AF_ERR_CUDA;
        } else {
          body_inner = p.conditional.phGraph_out[0];
        }
      }
      if (!rc) launch_block_advance(b.ctl, b.btab, h_outer, cs2);
    }
    cudaGraph_t dummy;
    if (cudaStreamEndCapture(cs2, &dummy) != cudaSuccess && !rc) { set_err("end of block-loop capture failed"); rc = AF_ERR_CUDA; }
    if (rc) break;
    // the update body
    if (cudaStreamBeginCaptureToGraph(cs2, body_inner, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
      set_err("capture of the update loop failed"); rc = AF_ERR_CUDA; break;
    }
    HeadIO hio{1, jb.z, jb.x, 0.f};
    rc = enqueue_pass(m, b, batch, L, jb.dir, m_max, r_max, jb.x, hio, cs2);
    if (!rc) launch_jacobi_step(b.ctl, b.btab, b.active, b.part, batch, G, tau, max_iter, jb.iters, h_inner, cs2);
    if (cudaStreamEndCapture(cs2, &dummy) != cudaSuccess && !rc) { set_err("end of update capture failed"); rc = AF_ERR_CUDA; }
  } while (0);
  return rc;
}

af_status graph_run(const af_model* mc, const std::string& key, cudaStream_t st,
                    af_status (*build)(void*, cudaStream_t), void* ctx) {
  af_model* m = const_cast<af_model*>(mc);
  auto it = m->graphs.find(key);
  if (it == m->graphs.end()) {
    cudaGraphExec_t ex;
    g_pdl = m->pdl;
    for (int attempt = 0;; ++attempt) {
      cudaGraph_t g;
      CK(cudaGraphCreate(&g, 0));
      CK(cudaStreamBeginCaptureToGraph(m->cap, g, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed));
      af_status s = build(ctx, m->cap);
      cudaGraph_t g2;
      cudaError_t ee = cudaStreamEndCapture(m->cap, &g2);
      cudaError_t ie = cudaErrorUnknown;
      if (!s && ee == cudaSuccess) ie = cudaGraphInstantiate(&ex, g, 0);
      cudaGraphDestroy(g);
      if (!s && ee == cudaSuccess && ie == cudaSuccess) break;
      cudaGetLastError();
      if (attempt == 0 && g_pdl) {   // programmatic edges refused here: plain edges instead
        g_pdl = 0;
        m->pdl = 0;
        continue;
      }
      if (s) return s;
      set_err("graph capture/instantiation failed: %s", cudaGetErrorString(ee != cudaSuccess ? ee : ie));
      return AF_ERR_CUDA;
    }
    if (m->graph_order.size() >= 16) {
      cudaGraphExecDestroy(m->graphs[m->graph_order.front()]);
      m->graphs.erase(m->graph_order.front());
      m->graph_order.erase(m->graph_order.begin());
    }
    it = m->graphs.emplace(key, ex).first;
    m->graph_order.push_back(key);
  }
  CK(cudaGraphLaunch(it->second, st));
  return AF_OK;
}

std::string keyf(const char* tag, std::initializer_list<long long> v) {
  std::string s(tag);
  char buf[32];
  for (long long x : v) { snprintf(buf, sizeof buf, ":%llx", x); s += buf; }
  return s;
}

// ------------------------------------------------------------------ argument checks

af_status check_model(const af_model* m) {
  if (!m) { set_err("null model"); return AF_ERR_ARG; }
  return AF_OK;
}

af_status check_ws(const af_model* m, void* ws, size_t ws_bytes, int batch, int L, int B) {
  const size_t need = af_workspace_bytes(m, batch, L, B);
  if (!need) { set_err("bad batch/L/B for this model"); return AF_ERR_ARG; }
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < need) {
    set_err("workspace: need %zu bytes, 256-aligned; got %zu at %p", need, ws_bytes, ws);
    return AF_ERR_WORKSPACE;
  }
  return AF_OK;
}

bool same_cfg(const af_config& a, const af_config& b) {
  return a.C == b.C && a.d == b.d && a.heads == b.heads && a.layers == b.layers && a.mlp_ratio == b.mlp_ratio &&
         a.frame_len == b.frame_len && a.max_frames == b.max_frames && a.dtype == b.dtype;
}

// ------------------------------------------------------------------ forward / stacks

struct FwdCtx {
  const af_model* const* blocks;
  const af_dir* dirs;
  int T, batch, L;
  const float* x;
  float* z;
  float* logdet;
  Bufs b;
};

af_status build_forward(void* vctx, cudaStream_t cs) {
  FwdCtx* c = static_cast<FwdCtx*>(vctx);
  const int G = (2 * c->blocks[0]->cfg.C) / 16;
  const int m_max = c->batch * c->L;
  // No cache clearing: a forward pass writes K / V of every position before
  // its attention reads them; the key tile past a sample's last position
  // holds the next sample's rows (written by the same pass) or lies past the
  // cache, where the TMA load fills zeros.
  for (int t = 0; t < c->T; ++t) {
    // block t writes z when T-1-t is even, else tmp; block t reads what t-1 wrote
    const float* in = t == 0 ? c->x : (((c->T - t) % 2 == 0) ? c->z : c->b.tmp);
    float* out = ((c->T - 1 - t) % 2 == 0) ? c->z : c->b.tmp;
    launch_ctl_forward(c->b.ctl, c->batch, c->L, cs);
    HeadIO hio{0, in, out, 0.f};
    af_status s = enqueue_pass(c->blocks[t], c->b, c->batch, c->L, c->dirs[t], m_max, c->L, in, hio, cs);
    if (s) return s;
    launch_logdet_finalize(c->b.part, c->batch, c->L, G, c->logdet, t > 0, cs);
  }
  CK(cudaGetLastError());
  return AF_OK;
}

struct InvCtx {
  const af_model* const* blocks;
  const af_dir* dirs;
  int T, batch, L, B_max, nb, max_iter, warm;
  float tau;
  const float* z;
  float* x;
  int32_t* iters;
  Bufs b;
};

af_status build_inverse(void* vctx, cudaStream_t cs) {
  InvCtx* c = static_cast<InvCtx*>(vctx);
  // the masked V rows each block's attention reads are zeroed by its block init
  for (int t = c->T - 1; t >= 0; --t) {
    float* out = (t % 2 == 0) ? c->x : c->b.tmp;
    const float* in = (t == c->T - 1) ? c->z : ((((t + 1) % 2) == 0) ? c->x : c->b.tmp);
    JacobiJob jb{c->blocks[t], in, out, c->dirs[t], c->iters + (size_t)t * c->batch * c->nb, t == c->T - 1};
    af_status s = capture_jacobi(jb, c->b, c->batch, c->L, c->B_max, c->tau, c->max_iter, c->warm, cs);
    if (s) return s;
  }
  CK(cudaGetLastError());
  return AF_OK;
}

// Writes the schedule into the workspace's block table on `st`, then runs
// (capturing on first use) the Jacobi graph of the stack.  The graph depends
// on B_max, not on the schedule or range, which are data.
af_status run_inverse(const af_model* const* blocks, const af_dir* dirs, int T, const float* z, int batch, int L,
                      const Schedule& sc, float tau, int max_iter, int warm, float* x, int32_t* iters, void* ws,
                      cudaStream_t st, bool write_table = true) {
  const int nb = (int)sc.starts.size() - 1;
  InvCtx c{blocks, dirs, T, batch, L, sc.B_max, nb, max_iter, warm ? 1 : 0, tau, z, x, iters,
           carve(blocks[0], ws, batch, L, sc.B_max)};
  g_pdl = blocks[0]->pdl;
  if (write_table) launch_table_write(c.b.btab, sc.starts.data(), nb, sc.b_begin, sc.b_end, st);
  CK(cudaGetLastError());
  uint32_t taubits;
  memcpy(&taubits, &tau, 4);
  std::string key = keyf("inv", {(long long)z, (long long)x, (long long)iters, (long long)ws, batch, L, sc.B_max, nb,
                                 (long long)taubits, max_iter, c.warm, T, (long long)blocks[0]->wait_ns});
  for (int t = 0; t < T; ++t) key += keyf("", {(long long)blocks[t], dirs[t]});
  return graph_run(blocks[0], key, st, build_inverse, &c);
}

// The work of a call runs on the current device; every model's weights must
// live there, and so must the stream (when it is not the default stream).
af_status device_checks(const af_model* m, cudaStream_t st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); set_err("no current CUDA device"); return AF_ERR_CUDA; }
  if (dev != m->device) {
    set_err("the model's weights are on device %d but device %d is current", m->device, dev);
    return AF_ERR_ARG;
  }
  if (st) {
    int sdev = -1;
    if (cudaStreamGetDevice(st, &sdev) != cudaSuccess) {
      cudaGetLastError();
      set_err("the stream is not a valid CUDA stream");
      return AF_ERR_ARG;
    }
    if (sdev != dev) { set_err("the stream belongs to device %d, the model to device %d", sdev, dev); return AF_ERR_ARG; }
  }
  return AF_OK;
}

struct EncCtx {
  const af_model* m;
  const float* x;
  int batch, L, B, n_tokens, dir;
  Bufs b;
};

// Flow-encode of observed tokens 0 .. n_tokens-1 into the KV cache: passes of
// at most rows_per_sample(L, B) positions, in order, each attending the cache
// of the passes before it; no head output.
af_status build_encode(void* vctx, cudaStream_t cs) {
  EncCtx* c = static_cast<EncCtx*>(vctx);
  const af_model* m = c->m;
  const int r_max = rows_per_sample(c->L, c->B);
  const int m_max = c->batch * r_max;
  const size_t kv_layer = (size_t)c->batch * c->L * m->cfg.d * 2;
  bf16* vtail = m->bf ? (bf16*)((char*)c->b.kv + kv_layer) : nullptr;
  for (int p0 = 0; p0 < c->n_tokens; p0 += r_max) {
    const int R = (c->n_tokens - p0) < r_max ? (c->n_tokens - p0) : r_max;
    launch_set_pass(c->b.ctl, p0, R, c->batch, vtail, 2 * kv_layer, m->cfg.layers, c->L, m->cfg.d, cs);
    HeadIO hio{1, c->x, c->b.tmp, 0.f};            // no row reaches the head's output
    af_status s = enqueue_pass(m, c->b, c->batch, c->L, c->dir, m_max, r_max, c->x, hio, cs);
    if (s) return s;
  }
  CK(cudaGetLastError());
  return AF_OK;
}

struct DenCtx {
  const af_model* m;
  const float* xn;
  float* x;
  int batch, L;
  float sigma;
  Bufs b;
};

// The denoiser's forward pass over all positions of every sequence.
af_status build_denoise(void* vctx, cudaStream_t cs) {
  DenCtx* c = static_cast<DenCtx*>(vctx);
  launch_ctl_forward(c->b.ctl, c->batch, c->L, cs);
  HeadIO hio{2, c->xn, c->x, c->sigma};
  af_status s = enqueue_pass(c->m, c->b, c->batch, c->L, AF_L2R, c->batch * c->L, c->L, c->xn, hio, cs);
  if (s) return s;
  CK(cudaGetLastError());
  return AF_OK;
}

af_status stack_checks(const af_model* const* blocks, const af_dir* dirs, int T, cudaStream_t st) {
  if (!blocks || !dirs || T < 1) { set_err("blocks/dirs/T"); return AF_ERR_ARG; }
  for (int t = 0; t < T; ++t) {
    if (!blocks[t]) { set_err("null block %d", t); return AF_ERR_ARG; }
    if (blocks[t]->kind != KIND_FLOW) { set_err("block %d is a denoiser, not an AF block", t); return AF_ERR_ARG; }
    if (!same_cfg(blocks[t]->cfg, blocks[0]->cfg)) { set_err("blocks must share one config"); return AF_ERR_ARG; }
    if (dirs[t] != AF_L2R && dirs[t] != AF_R2L) { set_err("bad direction"); return AF_ERR_ARG; }
    if (blocks[t]->device != blocks[0]->device) { set_err("blocks must live on one device"); return AF_ERR_ARG; }
  }
  return device_checks(blocks[0], st);
}

}  // namespace

// ------------------------------------------------------------------ direct launch (no graph)

namespace af {

void set_error_text(const char* msg) { set_err("%s", msg); }

// AF_OK when `m` lives on the current device and `st` (if not the default
// stream) belongs to it; used by entry points outside this file.
af_status check_call_device(const af_model* m, cudaStream_t st) {
  if (!m) { set_err("null model"); return AF_ERR_ARG; }
  return device_checks(m, st);
}

// The forward pass of one block launched kernel by kernel on `st`, with the
// workspace at `ws`; used by af_forward_noalloc.
af_status forward_direct(const af_model* m, const float* x, int batch, int L, af_dir dir, float* z, float* logdet,
                         void* ws, size_t ws_bytes, cudaStream_t st) {
  const af_model* blocks[1] = {m};
  af_dir dirs[1] = {dir};
  if (af_status s = stack_checks(blocks, dirs, 1, st)) return s;
  if (af_status s = check_ws(m, ws, ws_bytes, batch, L, L)) return s;
  FwdCtx c{blocks, dirs, 1, batch, L, x, z, logdet, carve(m, ws, batch, L, L)};
  g_pdl = m->pdl;
  return build_forward(&c, st);
}

}  // namespace af

// ============================================================================ C ABI

extern "C" {

int af_num_tensors(const af_config* cfg) { return cfg ? 4 + 12 * cfg->layers + 4 : 0; }

}  // extern "C"

namespace {

af_status create_model(const af_config* cfg, const float* const* tensors, int n_tensors, af_model** out, int kind) {
  if (!cfg || !tensors || !out) { set_err("null argument"); return AF_ERR_ARG; }
  const af_config c = *cfg;
  if (c.C <= 0 || c.d <= 0 || c.heads <= 0 || c.layers <= 0 || c.mlp_ratio <= 0 || c.frame_len <= 0 ||
      c.max_frames <= 0 || c.d % c.heads || c.C % 8 || c.d % 4) {
    set_err("invalid config");
    return AF_ERR_ARG;
  }
  const int hd = c.d / c.heads;
  if (c.dtype == AF_FP32) {
    if (hd != 16 && hd != 32 && hd != 64 && hd != 128) { set_err("fp32 path: head dim must be 16/32/64/128"); return AF_ERR_ARG; }
  } else if (c.dtype == AF_BF16) {
    if (c.C % 64 || c.d % 128 || (hd != 64 && hd != 128) || (c.mlp_ratio * c.d) % 128) {
      set_err("bf16 path: needs C%%64==0, d%%128==0, head dim 64 or 128");
      return AF_ERR_ARG;
    }
  } else {
    set_err("bad dtype");
    return AF_ERR_ARG;
  }
  if (kind == KIND_DENOISER && c.dtype == AF_BF16 && c.C % 128 && c.C % 192) {
    set_err("bf16 denoiser: the head's C outputs need C %% 128 == 0 or C %% 192 == 0 (tensor-core tile widths)");
    return AF_ERR_ARG;
  }
  if (n_tensors != af_num_tensors(cfg)) { set_err("expected %d tensors, got %d", af_num_tensors(cfg), n_tensors); return AF_ERR_ARG; }
  for (int i = 0; i < n_tensors; ++i)
    if (!tensors[i]) { set_err("null tensor %d", i); return AF_ERR_ARG; }

  af_model* m = new af_model();
  m->kind = kind;
  m->pdl = 1;
  m->wait_ns = 2000000000ull;
  m->l2_keep = 1;
  if (const char* v = getenv("AF_L2_KEEP")) m->l2_keep = atoi(v) != 0;
  if (const char* v = getenv("AF_PDL")) m->pdl = atoi(v) != 0;
  m->cfg = c;
  m->fd = c.mlp_ratio * c.d;
  m->hd = hd;
  m->bf = c.dtype == AF_BF16;
  int dev = 0;
  cudaGetDevice(&dev);
  m->device = dev;
  if (cudaDeviceGetAttribute(&m->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    set_err("no CUDA device");
    delete m;
    return AF_ERR_CUDA;
  }
  bool fail = false;
  auto upload_f32 = [&](const float* src, size_t n) -> float* {
    void* p = nullptr;
    if (cudaMalloc(&p, n * 4) != cudaSuccess || cudaMemcpy(p, src, n * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
      fail = true;
      return nullptr;
    }
    m->allocs.push_back(p);
    return (float*)p;
  };
  auto upload_w = [&](const float* src, size_t n) -> void* {   // matrices: bf16 or fp32
    if (!m->bf) return upload_f32(src, n);
    std::vector<uint16_t> tmp(n);
    for (size_t i = 0; i < n; ++i) tmp[i] = f2bf(src[i]);
    void* p = nullptr;
    if (cudaMalloc(&p, n * 2) != cudaSuccess || cudaMemcpy(p, tmp.data(), n * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
      fail = true;
      return nullptr;
    }
    m->allocs.push_back(p);
    return p;
  };
  // vectors: bf16 models use bf16-rounded values held in fp32
  auto upload_v = [&](const float* src, size_t n) -> float* {
    if (!m->bf) return upload_f32(src, n);
    std::vector<float> tmp(n);
    for (size_t i = 0; i < n; ++i) {
      const uint32_t u = (uint32_t)f2bf(src[i]) << 16;
      memcpy(&tmp[i], &u, 4);
    }
    return upload_f32(tmp.data(), n);
  };
  const size_t d = c.d, C = c.C, fd = m->fd;
  int k = 0;
  m->w_in = upload_w(tensors[k++], d * C);
  m->b_in = upload_v(tensors[k++], d);
  m->pos_space = upload_v(tensors[k++], (size_t)c.frame_len * d);
  m->pos_time = upload_v(tensors[k++], (size_t)c.max_frames * d);
  for (int l = 0; l < c.layers; ++l) {
    LayerW w;
    w.ln1_g = upload_v(tensors[k++], d);
    w.ln1_b = upload_v(tensors[k++], d);
    w.w_qkv = upload_w(tensors[k++], 3 * d * d);
    w.b_qkv = upload_v(tensors[k++], 3 * d);
    w.w_o = upload_w(tensors[k++], d * d);
    w.b_o = upload_v(tensors[k++], d);
    w.ln2_g = upload_v(tensors[k++], d);
    w.ln2_b = upload_v(tensors[k++], d);
    w.w_1 = upload_w(tensors[k++], fd * d);
    w.b_1 = upload_v(tensors[k++], fd);
    w.w_2 = upload_w(tensors[k++], d * fd);
    w.b_2 = upload_v(tensors[k++], d);
    m->layers.push_back(w);
  }
  m->lnf_g = upload_v(tensors[k++], d);
  m->lnf_b = upload_v(tensors[k++], d);
  if (kind == KIND_DENOISER) {                  // head [C, d], b [C] as given
    m->w_head = upload_w(tensors[k], C * d);
    m->b_head = upload_v(tensors[k + 1], C);
    k += 2;
  } else {
    const float* wh = tensors[k++];
    const float* bh = tensors[k++];
    std::vector<float> wi(2 * C * d), bi(2 * C);
    for (size_t ch = 0; ch < C; ++ch) {
      memcpy(&wi[(2 * ch) * d], wh + ch * d, d * 4);
      memcpy(&wi[(2 * ch + 1) * d], wh + (C + ch) * d, d * 4);
      bi[2 * ch] = bh[ch];
      bi[2 * ch + 1] = bh[C + ch];
    }
    m->w_head = upload_w(wi.data(), 2 * C * d);
    m->b_head = upload_v(bi.data(), 2 * C);
  }
  void* e = nullptr;
  if (cudaMalloc(&e, 256) != cudaSuccess || cudaMemset(e, 0, 256) != cudaSuccess) fail = true;
  else m->allocs.push_back(e);
  m->d_err = (int*)e;
  if (!fail && (cudaStreamCreateWithFlags(&m->cap, cudaStreamNonBlocking) != cudaSuccess ||
                cudaStreamCreateWithFlags(&m->cap2, cudaStreamNonBlocking) != cudaSuccess))
    fail = true;
  if (fail) {
    set_err("device allocation/copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    for (void* p : m->allocs) cudaFree(p);
    delete m;
    return AF_ERR_CUDA;
  }
  *out = m;
  return AF_OK;
}

}  // namespace

extern "C" {

af_status af_model_create(const af_config* cfg, const float* const* tensors, int n_tensors, af_model** out) {
  return create_model(cfg, tensors, n_tensors, out, KIND_FLOW);
}

int af_denoiser_num_tensors(const af_config* cfg) { return af_num_tensors(cfg); }

af_status af_denoiser_create(const af_config* cfg, const float* const* tensors, int n_tensors, af_model** out) {
  return create_model(cfg, tensors, n_tensors, out, KIND_DENOISER);
}

af_status af_model_destroy(af_model* m) {
  if (!m) return AF_ERR_ARG;
  cudaDeviceSynchronize();
  for (auto& kv : m->graphs) cudaGraphExecDestroy(kv.second);
  for (void* p : m->allocs) cudaFree(p);
  cudaStreamDestroy(m->cap);
  cudaStreamDestroy(m->cap2);
  if (m->ev_frame) cudaEventDestroy(m->ev_frame);
  if (m->ev_done) cudaEventDestroy(m->ev_done);
  delete m;
  return AF_OK;
}

size_t af_workspace_bytes(const af_model* m, int batch, int L, int B) {
  if (!m || batch < 1 || L < 1 || B < 1 || L > m->cfg.frame_len * m->cfg.max_frames) return 0;
  return carve(m, nullptr, batch, L, B < L ? B : L).total;
}

af_status af_forward(const af_model* m, const float* x, int batch, int L, af_dir dir, float* z, float* logdet,
                     void* ws, size_t ws_bytes, void* stream) {
  af_dir dirs[1] = {dir};
  const af_model* blocks[1] = {m};
  if (af_status s = check_model(m)) return s;
  return flow_stack_forward(blocks, dirs, 1, x, batch, L, z, logdet, ws, ws_bytes, stream);
}

af_status flow_stack_forward(const af_model* const* blocks, const af_dir* dirs, int T, const float* x, int batch,
                             int L, float* z, float* logdet, void* ws, size_t ws_bytes, void* stream) {
  if (af_status s = stack_checks(blocks, dirs, T, (cudaStream_t)stream)) return s;
  if (!x || !z || !logdet || x == z) { set_err("x/z/logdet (x and z must not alias)"); return AF_ERR_ARG; }
  if (af_status s = check_ws(blocks[0], ws, ws_bytes, batch, L, L)) return s;
  FwdCtx c{blocks, dirs, T, batch, L, x, z, logdet, carve(blocks[0], ws, batch, L, L)};
  std::vector<long long> kv = {(long long)x, (long long)z, (long long)logdet, (long long)ws, batch, L, T,
                               (long long)blocks[0]->wait_ns};
  std::string key = keyf("fwd", {});
  for (int t = 0; t < T; ++t) key += keyf("", {(long long)blocks[t], dirs[t]});
  for (long long v : kv) key += keyf("", {v});
  return graph_run(blocks[0], key, (cudaStream_t)stream, build_forward, &c);
}

af_status af_inverse_jacobi(const af_model* m, const float* z, int batch, int L, af_dir dir, int B, float tau,
                            int max_iter, int warm_start, float* x, int32_t* iters, void* ws, size_t ws_bytes,
                            void* stream) {
  af_dir dirs[1] = {dir};
  const af_model* blocks[1] = {m};
  if (af_status s = check_model(m)) return s;
  return flow_stack_inverse(blocks, dirs, 1, z, batch, L, B, tau, max_iter, warm_start, x, iters, ws, ws_bytes,
                            stream);
}

af_status flow_stack_inverse(const af_model* const* blocks, const af_dir* dirs, int T, const float* z, int batch,
                             int L, int B, float tau, int max_iter, int warm_start, float* x, int32_t* iters,
                             void* ws, size_t ws_bytes, void* stream) {
  if (af_status s = stack_checks(blocks, dirs, T, (cudaStream_t)stream)) return s;
  if (!z || !x || !iters || x == z) { set_err("z/x/iters (x and z must not alias)"); return AF_ERR_ARG; }
  if (B < 1 || L % B || max_iter < 1 || !(tau >= 0.f) || tau == INFINITY) {
    set_err("need L %% B == 0, max_iter >= 1, finite tau >= 0");
    return AF_ERR_ARG;
  }
  if (af_status s = check_ws(blocks[0], ws, ws_bytes, batch, L, B)) return s;
  return run_inverse(blocks, dirs, T, z, batch, L, uniform_schedule(L, B), tau, max_iter, warm_start, x, iters, ws,
                     (cudaStream_t)stream);
}

af_status af_inverse_jacobi_schedule(const af_model* m, const float* z, int batch, int L, af_dir dir,
                                     const int* block_sizes, int n_blocks, int b_begin, int b_end, float tau,
                                     int max_iter, int warm_start, float* x, int32_t* iters, void* ws,
                                     size_t ws_bytes, void* stream) {
  af_dir dirs[1] = {dir};
  const af_model* blocks[1] = {m};
  if (af_status s = stack_checks(blocks, dirs, 1, (cudaStream_t)stream)) return s;
  if (!z || !x || !iters || x == z) { set_err("z/x/iters (x and z must not alias)"); return AF_ERR_ARG; }
  if (!block_sizes || n_blocks < 1 || n_blocks > L || b_begin < 0 || b_end > n_blocks || b_begin >= b_end) {
    set_err("need 1 <= n_blocks <= L and 0 <= b_begin < b_end <= n_blocks");
    return AF_ERR_ARG;
  }
  if (max_iter < 1 || !(tau >= 0.f) || tau == INFINITY) { set_err("need max_iter >= 1, finite tau >= 0"); return AF_ERR_ARG; }
  Schedule sc;
  sc.starts.push_back(0);
  sc.B_max = 0;
  sc.uniform = true;
  for (int i = 0; i < n_blocks; ++i) {
    const int bs = block_sizes[i];
    if (bs < 1 || sc.starts.back() > L - bs) { set_err("block %d: sizes must be >= 1 and sum to L", i); return AF_ERR_ARG; }
    sc.starts.push_back(sc.starts.back() + bs);
    if (bs > sc.B_max) sc.B_max = bs;
    if (bs != block_sizes[0]) sc.uniform = false;
  }
  if (sc.starts.back() != L) { set_err("block sizes sum to %d, not L = %d", sc.starts.back(), L); return AF_ERR_ARG; }
  sc.b_begin = b_begin;
  sc.b_end = b_end;
  if (af_status s = check_ws(m, ws, ws_bytes, batch, L, sc.B_max)) return s;
  return run_inverse(blocks, dirs, 1, z, batch, L, sc, tau, max_iter, warm_start, x, iters, ws, (cudaStream_t)stream);
}

af_status af_prefix_encode(const af_model* m, const float* x, int batch, int L, af_dir dir, int B, int n_tokens,
                           void* ws, size_t ws_bytes, void* stream) {
  af_dir dirs[1] = {dir};
  const af_model* blocks[1] = {m};
  if (af_status s = stack_checks(blocks, dirs, 1, (cudaStream_t)stream)) return s;
  if (!x || n_tokens < 1 || n_tokens > L || B < 1) { set_err("need x, 1 <= n_tokens <= L, B >= 1"); return AF_ERR_ARG; }
  if (af_status s = check_ws(m, ws, ws_bytes, batch, L, B)) return s;
  const int Bc = B < L ? B : L;
  EncCtx c{m, x, batch, L, Bc, n_tokens, dir, carve(m, ws, batch, L, Bc)};
  g_pdl = m->pdl;
  std::string key = keyf("enc", {(long long)x, (long long)ws, batch, L, Bc, n_tokens, dir, (long long)m->wait_ns});
  return graph_run(m, key, (cudaStream_t)stream, build_encode, &c);
}

size_t flow_pipeline_workspace_bytes(const af_model* shallow, int T, int batch, int frame_len, int group) {
  if (!shallow || T < 1 || batch < 1 || group < 1) return 0;
  const int nb = batch * group;                    // a shallow call's samples: group frames of every video
  const size_t stack = af_workspace_bytes(shallow, nb, frame_len, frame_len);
  if (!stack) return 0;
  const size_t frames = align256((size_t)nb * frame_len * shallow->cfg.C * sizeof(float));
  return stack + 2 * frames + align256((size_t)T * nb * sizeof(int32_t));
}

af_status flow_pipeline_inverse(const af_model* deep, const af_model* const* shallow, const af_dir* shallow_dirs, int T,
                                const float* z, int batch, int L, int B, float tau, int max_iter_deep,
                                int max_iter_shallow, int warm_start, int group, float* x, int32_t* iters_deep,
                                int32_t* iters_shallow, void* ws_deep, size_t ws_deep_bytes, void* ws_shallow,
                                size_t ws_shallow_bytes, void* stream_deep, void* stream_shallow) {
  cudaStream_t sd = (cudaStream_t)stream_deep, ss = (cudaStream_t)stream_shallow;
  af_dir ddir[1] = {AF_L2R};
  const af_model* dblk[1] = {deep};
  if (af_status s = stack_checks(dblk, ddir, 1, sd)) return s;
  if (af_status s = stack_checks(shallow, shallow_dirs, T, ss)) return s;
  if (shallow[0]->device != deep->device) { set_err("deep and shallow models on different devices"); return AF_ERR_ARG; }
  const int F = deep->cfg.frame_len;
  const int C = deep->cfg.C;
  if (shallow[0]->cfg.C != C || shallow[0]->cfg.frame_len * shallow[0]->cfg.max_frames < F) {
    set_err("the shallow blocks must take frames of %d tokens of %d channels", F, C);
    return AF_ERR_ARG;
  }
  if (!z || !x || !iters_deep || !iters_shallow || x == z) { set_err("z/x/iters (x and z must not alias)"); return AF_ERR_ARG; }
  if (B < 1 || L % F || F % B || max_iter_deep < 1 || max_iter_shallow < 1 || !(tau >= 0.f) || tau == INFINITY) {
    set_err("need L %% frame_len == 0, frame_len %% B == 0, max_iter >= 1, finite tau >= 0");
    return AF_ERR_ARG;
  }
  const int nf = L / F;
  if (group < 1 || group > nf) { set_err("need 1 <= group <= L / frame_len (%d), got %d", nf, group); return AF_ERR_ARG; }
  if (af_status s = check_ws(deep, ws_deep, ws_deep_bytes, batch, L, B)) return s;
  const size_t need_s = flow_pipeline_workspace_bytes(shallow[0], T, batch, F, group);
  if (!ws_shallow || (reinterpret_cast<uintptr_t>(ws_shallow) & 255u) || ws_shallow_bytes < need_s) {
    set_err("shallow workspace: need %zu bytes, 256-aligned; got %zu", need_s, ws_shallow_bytes);
    return AF_ERR_WORKSPACE;
  }
  af_model* dm = const_cast<af_model*>(deep);
  if (!dm->ev_frame) {
    CK(cudaEventCreateWithFlags(&dm->ev_frame, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&dm->ev_done, cudaEventDisableTiming));
  }
  // the shallow side's workspace: the stack's own (for batch * group samples),
  // then the staged frames in / out and the counts
  const int nbmax = batch * group;
  const size_t stack_bytes = af_workspace_bytes(shallow[0], nbmax, F, F);
  const size_t frames = align256((size_t)nbmax * F * C * sizeof(float));
  char* wsS = static_cast<char*>(ws_shallow);
  float* stage_in = (float*)(wsS + stack_bytes);
  float* stage_out = (float*)(wsS + stack_bytes + frames);
  int32_t* stage_it = (int32_t*)(wsS + stack_bytes + 2 * frames);
  // the deep flow's output u (the shallow stack's input) stays in its workspace
  float* u = carve(deep, ws_deep, batch, L, B).tmp;
  const int bpf = F / B;
  Schedule sc = uniform_schedule(L, B);
  const size_t frame_bytes = (size_t)F * C * sizeof(float);
  const size_t video_pitch = (size_t)L * C * sizeof(float);
  for (int f = 0; f < nf; ++f) {
    // f_D^{-1}: the blocks of frame f (the table once, then only the range)
    sc.b_begin = f * bpf;
    sc.b_end = (f + 1) * bpf;
    if (f > 0) launch_set_range(carve(deep, ws_deep, batch, L, B).btab, sc.b_begin, sc.b_end, sd);
    if (af_status s = run_inverse(dblk, ddir, 1, z, batch, L, sc, tau, max_iter_deep, warm_start, u, iters_deep,
                                  ws_deep, sd, f == 0))
      return s;
    const int f0 = (f / group) * group;           // first frame of f's group
    const int g = (f0 + group <= nf ? group : nf - f0);
    if (f != f0 + g - 1) continue;                // the group is not complete yet
    CK(cudaEventRecord(dm->ev_frame, sd));
    // f_S^{-1} of frames f0 .. f on the second stream, while f_D goes on:
    // every video's g frames, each frame a sample of its own ([batch * g, F, C])
    CK(cudaStreamWaitEvent(ss, dm->ev_frame, 0));
    const size_t run = (size_t)g * frame_bytes;
    CK(cudaMemcpy2DAsync(stage_in, run, u + (size_t)f0 * F * C, video_pitch, run, batch, cudaMemcpyDeviceToDevice, ss));
    if (af_status s = flow_stack_inverse(shallow, shallow_dirs, T, stage_in, batch * g, F, F, tau, max_iter_shallow, 0,
                                         stage_out, stage_it, ws_shallow, stack_bytes, ss))
      return s;
    CK(cudaMemcpy2DAsync(x + (size_t)f0 * F * C, video_pitch, stage_out, run, run, batch, cudaMemcpyDeviceToDevice, ss));
    // counts [T, batch * g] -> iters_shallow[T, batch, f0 .. f0 + g)
    CK(cudaMemcpy2DAsync(iters_shallow + f0, (size_t)nf * sizeof(int32_t), stage_it, (size_t)g * sizeof(int32_t),
                         (size_t)g * sizeof(int32_t), (size_t)T * batch, cudaMemcpyDeviceToDevice, ss));
  }
  CK(cudaEventRecord(dm->ev_done, ss));
  CK(cudaStreamWaitEvent(sd, dm->ev_done, 0));
  return AF_OK;
}

size_t af_stream_workspace_bytes(const af_model* m, int batch, int window) {
  if (!m || batch < 1 || window < 1) return 0;
  const int F = m->cfg.frame_len;
  const int Lw = window * F;
  const size_t base = af_workspace_bytes(m, batch, Lw, F);
  if (!base) return 0;
  const size_t frames = align256((size_t)batch * Lw * m->cfg.C * sizeof(float));
  return base + 2 * frames + align256((size_t)batch * window * sizeof(int32_t));
}

af_status af_inverse_jacobi_stream(const af_model* m, const float* z, int batch, int n_frames, int window, int overlap,
                                   float tau, int max_iter, int warm_start, float* x, int32_t* iters, void* ws,
                                   size_t ws_bytes, void* stream) {
  af_dir dirs[1] = {AF_L2R};
  const af_model* blocks[1] = {m};
  cudaStream_t st = (cudaStream_t)stream;
  if (af_status s = stack_checks(blocks, dirs, 1, st)) return s;
  if (!z || !x || !iters || x == z) { set_err("z/x/iters (x and z must not alias)"); return AF_ERR_ARG; }
  const int F = m->cfg.frame_len, C = m->cfg.C;
  if (n_frames < 1 || window < 1 || window > m->cfg.max_frames || overlap < 0 || overlap >= window ||
      max_iter < 1 || !(tau >= 0.f) || tau == INFINITY) {
    set_err("need n_frames >= 1, 1 <= window <= max_frames, 0 <= overlap < window, max_iter >= 1, finite tau >= 0");
    return AF_ERR_ARG;
  }
  const size_t need = af_stream_workspace_bytes(m, batch, window);
  if (!need || !ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < need) {
    set_err("stream workspace: need %zu bytes, 256-aligned; got %zu", need, ws_bytes);
    return AF_ERR_WORKSPACE;
  }
  // the window's own workspace, then the staged window of x and z and its counts
  const size_t win_bytes = af_workspace_bytes(m, batch, window * F, F);
  const size_t frames = align256((size_t)batch * window * F * C * sizeof(float));
  char* base = static_cast<char*>(ws);
  float* xw = (float*)(base + win_bytes);
  float* zw = (float*)(base + win_bytes + frames);
  int32_t* itw = (int32_t*)(base + win_bytes + 2 * frames);
  const size_t rowL = (size_t)n_frames * F * C * sizeof(float);     // pitch of z and x
  for (int s0 = 0, i = 0;; s0 += window - overlap, ++i) {
    const int nf = (n_frames - s0) < window ? (n_frames - s0) : window;
    const int Lw = nf * F;
    const int n_obs = i > 0 ? overlap : 0;
    const size_t rowW = (size_t)Lw * C * sizeof(float);
    const size_t off = (size_t)s0 * F * C;
    CK(cudaMemcpy2DAsync(zw, rowW, z + off, rowL, rowW, batch, cudaMemcpyDeviceToDevice, st));
    std::vector<int> sizes(nf, F);
    if (n_obs) {
      // the previous window's last frames, observed: flow-encoded into the cache
      const size_t rowO = (size_t)n_obs * F * C * sizeof(float);
      CK(cudaMemcpy2DAsync(xw, rowW, x + off, rowL, rowO, batch, cudaMemcpyDeviceToDevice, st));
      if (af_status s = af_prefix_encode(m, xw, batch, Lw, AF_L2R, F, n_obs * F, ws, win_bytes, stream)) return s;
    }
    if (af_status s = af_inverse_jacobi_schedule(m, zw, batch, Lw, AF_L2R, sizes.data(), nf, n_obs, nf, tau, max_iter,
                                                 warm_start, xw, itw, ws, win_bytes, stream))
      return s;
    const size_t skip = (size_t)n_obs * F * C;
    CK(cudaMemcpy2DAsync(x + off + skip, rowL, xw + skip, rowW, rowW - skip * sizeof(float), batch,
                         cudaMemcpyDeviceToDevice, st));
    CK(cudaMemcpy2DAsync(iters + s0 + n_obs, (size_t)n_frames * sizeof(int32_t), itw + n_obs,
                         (size_t)nf * sizeof(int32_t), (size_t)(nf - n_obs) * sizeof(int32_t), batch,
                         cudaMemcpyDeviceToDevice, st));
    if (s0 + window >= n_frames) break;
  }
  return AF_OK;
}

af_status af_last_convergence(void* ws, int* n_unconverged, void* stream) {
  if (!ws || !n_unconverged) { set_err("null argument"); return AF_ERR_ARG; }
  CK(cudaStreamSynchronize((cudaStream_t)stream));
  Ctl c;
  CK(cudaMemcpy(&c, ws, sizeof c, cudaMemcpyDeviceToHost));
  *n_unconverged = c.nonconv;
  return c.nonconv ? AF_NOT_CONVERGED : AF_OK;
}

af_status af_denoise(const af_model* m, const float* x_noisy, int batch, int L, float sigma, float* x, void* ws,
                     size_t ws_bytes, void* stream) {
  if (!m || m->kind != KIND_DENOISER) { set_err("af_denoise needs a model from af_denoiser_create"); return AF_ERR_ARG; }
  if (af_status s = device_checks(m, (cudaStream_t)stream)) return s;
  if (!x_noisy || !x || x == x_noisy) { set_err("x_noisy/x (they must not alias)"); return AF_ERR_ARG; }
  if (!(sigma == sigma) || sigma == INFINITY || sigma == -INFINITY) { set_err("sigma must be finite"); return AF_ERR_ARG; }
  if (af_status s = check_ws(m, ws, ws_bytes, batch, L, L)) return s;
  DenCtx c{m, x_noisy, x, batch, L, sigma, carve(m, ws, batch, L, L)};
  g_pdl = m->pdl;
  uint32_t sb;
  memcpy(&sb, &sigma, 4);
  std::string key = keyf("den", {(long long)x_noisy, (long long)x, (long long)ws, batch, L, (long long)sb,
                                 (long long)m->wait_ns});
  return graph_run(m, key, (cudaStream_t)stream, build_denoise, &c);
}

af_status af_set_wait_limit(af_model* m, double seconds) {
  if (!m || !(seconds > 0.0) || seconds > 60.0) { set_err("need a model and 0 < seconds <= 60"); return AF_ERR_ARG; }
  m->wait_ns = (uint64_t)(seconds * 1e9);
  if (m->wait_ns < 1) m->wait_ns = 1;
  return AF_OK;
}

af_status af_device_error(const af_model* m, int* code) {
  if (!m) { set_err("null model"); return AF_ERR_ARG; }
  CK(cudaDeviceSynchronize());
  int v = 0;
  CK(cudaMemcpy(&v, m->d_err, sizeof v, cudaMemcpyDeviceToHost));
  if (code) *code = v;
  if (v) {
    CK(cudaMemset(m->d_err, 0, sizeof v));
    set_err("device error code %d", v);
    return AF_ERR_DEVICE;
  }
  return AF_OK;
}

const char* af_status_string(af_status s) {
  switch (s) {
    case AF_OK: return "AF_OK";
    case AF_ERR_ARG: return "AF_ERR_ARG: bad argument";
    case AF_ERR_CUDA: return "AF_ERR_CUDA: a CUDA call failed";
    case AF_ERR_WORKSPACE: return "AF_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case AF_NOT_CONVERGED: return "AF_NOT_CONVERGED: a block stopped at max_iter";
    case AF_ERR_DEVICE: return "AF_ERR_DEVICE: a kernel gave up a bounded wait";
  }
  return "unknown af_status";
}

const char* af_last_error_string(void) { return g_errbuf; }

}  // extern "C"
