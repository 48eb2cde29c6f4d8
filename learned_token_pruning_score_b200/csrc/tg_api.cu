// tg_api.cu -- the C ABI of libtokengate (declared in include/tokengate.h).
//
// Host-side argument validation, workspace planning and the orchestration of
// the gated prefill. Every call validates on the host, then only enqueues
// kernels on the caller's stream: no allocation, no host synchronisation.
//
// The gated forward runs in three stages (Tencent Cloud article
// "TokenGate：端到端可训练的 Token 剪枝机制，让大模型 Prefill 提速 11.3 倍", section
// "TokenGate 提前筛选 Token"; farwalk.ai item on TokenGate, section "论文的方法";
// ai.866data.com article "让大模型学会"略读"…", section "可学习剪枝的机制设计"):
// layers below the gate over all N tokens; at the gate layer, attention over
// all N tokens, then the scorer on the post-attention residual, the top-K
// selector and compaction; the gate layer's FFN and all layers above over
// the K kept rows, with token-gated attention, writing K-row KV only.
#include <cuda_bf16.h>

#include <cmath>
#include <map>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "../../include/tokengate.h"
#include "tg_internal.h"

__device__ unsigned int g_tg_error_word;

namespace tg {

namespace {
thread_local int t_last_cuda_error = 0;
constexpr int kMaxDevices = 64;

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}
}  // namespace

int num_sms() {
  static int cache[kMaxDevices] = {0};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

unsigned int* device_error_word() {
  static unsigned int* cache[kMaxDevices] = {nullptr};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  if (cache[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_tg_error_word) == cudaSuccess)
      cache[dev] = static_cast<unsigned int*>(ptr);
  }
  return cache[dev];
}

cudaError_t set_smem_attr_once(const void* fn, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({fn, dev})) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert({fn, dev});
  return e;
}

namespace {

// ------------------------------------------------------------------ tracing
struct Tracer {
  bool on = false;
  int cap = 0;
  int layer = -1;
  std::vector<cudaEvent_t> ev;  // 2 per record
  std::vector<tg_trace_record> recs;
};
thread_local Tracer t_trace;

// Runs `launch` (which enqueues one kernel, or one fixed group of kernels)
// and, while tracing is on, brackets it with a pair of events.
template <class F>
cudaError_t traced(tg_kernel kernel, int64_t rows, double flops, double bytes, cudaStream_t st,
                   F&& launch) {
  Tracer& T = t_trace;
  if (!T.on || static_cast<int>(T.recs.size()) >= T.cap) return launch();
  const size_t i = T.recs.size();
  cudaEventRecord(T.ev[2 * i], st);
  const cudaError_t e = launch();
  cudaEventRecord(T.ev[2 * i + 1], st);
  T.recs.push_back(tg_trace_record{static_cast<int32_t>(kernel), T.layer, rows, 0.f, flops, bytes});
  return e;
}

tg_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TG_OK;
  t_last_cuda_error = static_cast<int>(e);
  return TG_ERR_CUDA;
}

#define TG_TRY(expr)                                  \
  do {                                                \
    const cudaError_t tg_e_ = (expr);                 \
    if (tg_e_ != cudaSuccess) return cuda_status(tg_e_); \
  } while (0)

#define TG_CHECK(cond, code) \
  do {                       \
    if (!(cond)) return (code); \
  } while (0)

size_t elem_size(tg_dtype dt) { return dt == TG_BF16 ? 2 : 4; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ plans
// Each plan carves its buffers from an Arena; with a null base it only
// measures, so sizing and use can never disagree.

struct ScorePlan {
  void* y = nullptr;     // [n, d] normed rows (dtype)
  float* hpre = nullptr; // fp32 path: [n, f] pre-activation
  size_t bytes = 0;
  ScorePlan(void* ws, int64_t n, int d, int f, tg_dtype dt) {
    Arena a(ws);
    y = a.carve(size_t(n) * d * elem_size(dt));
    if (dt == TG_F32) hpre = static_cast<float*>(a.carve(size_t(n) * f * 4));
    bytes = a.used;
  }
};

struct AttnPlan {
  void* q_rot = nullptr;  // [k, hq, dh]
  void* k_rot = nullptr;  // [k, hkv, dh]
  void* vT = nullptr;     // bf16: [hkv, dh, t_pad]
  float* lsig = nullptr;  // [k]
  void* kaug = nullptr;   // bf16 [k, 16] gate-bias rows (tensor-core path)
  void* split = nullptr;  // scratch for split query tiles of short sequences
  size_t split_bytes = 0;
  int64_t t_pad = 0;
  size_t bytes = 0;
  // split_rows: the shortest sequence this plan's attention will run (its
  // split scratch is sized for it; 0: none)
  AttnPlan(void* ws, int64_t k, int hq, int hkv, int dh, tg_dtype dt, bool need_k,
           int64_t split_rows = 0) {
    Arena a(ws);
    const size_t e = elem_size(dt);
    t_pad = static_cast<int64_t>(align_up(static_cast<size_t>(k), 64));
    q_rot = a.carve(size_t(k) * hq * dh * e);
    if (need_k) k_rot = a.carve(size_t(k) * hkv * dh * e);
    if (dt == TG_BF16) vT = a.carve(size_t(hkv) * dh * t_pad * e);
    lsig = static_cast<float*>(a.carve(size_t(k) * 4 + 16));
    if (dt == TG_BF16) kaug = a.carve(size_t(k) * 32);
    if (dt == TG_BF16 && dh == 128 && split_rows > 0) {
      split_bytes = attn_split_bytes(split_rows, hq, hkv);
      if (split_bytes > 0) split = a.carve(split_bytes);
    }
    bytes = a.used;
  }
};

// Backward of the standalone gated attention in fp32 (head_dim 64 or 128).
struct GdnPlan {
  GdnArgs a{};
  size_t bytes = 0;
  GdnPlan(void* ws, int64_t T, int hk, int hv, int dk, int dv) {
    Arena ar(ws);
    const int64_t tp = (T + kGdnChunk - 1) / kGdnChunk * kGdnChunk;
    a.t_pad = tp;
    a.qn = static_cast<float*>(ar.carve(size_t(hk) * tp * dk * 4));
    a.kn = static_cast<float*>(ar.carve(size_t(hk) * tp * dk * 4));
    a.vb = static_cast<float*>(ar.carve(size_t(hv) * tp * dv * 4));
    a.gl = static_cast<float*>(ar.carve(size_t(hv) * tp * 4));
    a.be = static_cast<float*>(ar.carve(size_t(hv) * tp * 4));
    a.eg = static_cast<float*>(ar.carve(size_t(hv) * tp * 4));
    a.tt = static_cast<float*>(ar.carve(size_t(hv) * tp * kGdnLd * 4));
    a.mm = static_cast<float*>(ar.carve(size_t(hv) * tp * kGdnLd * 4));
    a.o = static_cast<float*>(ar.carve(size_t(T) * hv * dv * 4));
    bytes = ar.used;
  }
};

// The four launches of the Gated DeltaNet mixer over g.T tokens (prep with
// the carried conv rows, per-chunk matrices, the recurrence, the gated norm).
cudaError_t gdn_run(const GdnArgs& g, bool bf, cudaStream_t st);
int64_t gdn_channels(const tg_gdn_layer& G);
int64_t gdn_proj_width(const tg_gdn_layer& G);

struct AttnBwdF32Plan {
  float* q_rot = nullptr;   // [n, hq, dh]
  float* k_rot = nullptr;   // [n, hkv, dh]
  float* lsig = nullptr;    // [n]
  float2* cs = nullptr;     // [dh/2, n]
  float* colsum = nullptr;  // [2, hq, n]
  float* qdq = nullptr;     // [hq, n]
  size_t bytes = 0;
  AttnBwdF32Plan(void* ws, int64_t n, int hq, int hkv, int dh) {
    Arena a(ws);
    q_rot = static_cast<float*>(a.carve(size_t(n) * hq * dh * 4));
    k_rot = static_cast<float*>(a.carve(size_t(n) * hkv * dh * 4));
    lsig = static_cast<float*>(a.carve(size_t(n) * 4 + 16));
    cs = static_cast<float2*>(a.carve(size_t(dh / 2) * n * 8));
    colsum = static_cast<float*>(a.carve(size_t(2) * hq * n * 4));
    qdq = static_cast<float*>(a.carve(size_t(hq) * n * 4));
    bytes = a.used;
  }
};

// Backward of the standalone gated attention (bf16, head_dim 128).
struct AttnBwdPlan {
  void* q_rot = nullptr;   // [n, hq, dh] rotated as in the forward
  void* k_rot = nullptr;   // [n, hkv, dh]
  float2* cs = nullptr;    // [dh/2, n] RoPE table
  void* qT = nullptr;      // [hq, dh, t_pad]
  void* doT = nullptr;     // [hq, dh, t_pad]
  float* lse2 = nullptr;   // [hq, t_pad]
  float* dd = nullptr;     // [hq, t_pad]
  float* colsum = nullptr; // [2, hq, t_pad]
  float* qdq = nullptr;    // [hq, t_pad / 128, 8]
  float* bias = nullptr;   // [t_pad] logsigmoid(s), zero-padded
  int64_t t_pad = 0;
  size_t bytes = 0;
  AttnBwdPlan(void* ws, int64_t n, int hq, int hkv, int dh) {
    Arena a(ws);
    t_pad = static_cast<int64_t>(attn_bwd_t_pad(n));
    const size_t tp = static_cast<size_t>(t_pad);
    q_rot = a.carve(size_t(n) * hq * dh * 2);
    k_rot = a.carve(size_t(n) * hkv * dh * 2);
    cs = static_cast<float2*>(a.carve(size_t(dh / 2) * n * 8));
    qT = a.carve(size_t(hq) * dh * tp * 2);
    doT = a.carve(size_t(hq) * dh * tp * 2);
    lse2 = static_cast<float*>(a.carve(size_t(hq) * tp * 4));
    dd = static_cast<float*>(a.carve(size_t(hq) * tp * 4));
    colsum = static_cast<float*>(a.carve(size_t(2) * hq * tp * 4));
    qdq = static_cast<float*>(a.carve(size_t(hq) * (tp / 128) * 32));
    bias = static_cast<float*>(a.carve(tp * 4));
    bytes = a.used;
  }
};

// Rows per block of the FFN sub-layer (its intermediate [rows, I] buffer).
constexpr int64_t kFfnRows = 16384;

struct PrefillPlan {
  void* h = nullptr;       // [n, d] residual stream (all-token stage)
  void* hk = nullptr;      // [k, d] residual stream (kept rows)
  void* y = nullptr;       // [n, d] normed rows
  void* qkv = nullptr;     // [n, (hq + 2 hkv) dh]
  void* attn_o = nullptr;  // [n, hq dh]
  void* mlp = nullptr;     // [n, I] (fp32: + [n, 2I] gate/up product)
  void* gu = nullptr;
  float* scores = nullptr; // [n]
  float* hpre = nullptr;   // fp32 scorer pre-activation [n, F]
  // Folded RMSNorm (bf16): per residual stream (h, hk) the row sums of
  // squares its last residual GEMM left, [ss_parts][ld] (one per
  // 256-column block), and how many leading rows they describe (-1: none).
  // Anything other than a residual GEMM that writes a stream resets it.
  float* ss = nullptr;    // rows of h: [ss_parts][n]
  float* ss_k = nullptr;  // rows of hk: [ss_parts][k]
  int64_t ss_ld = 0, ss_ld_k = 0;
  int ss_parts = 0;
  mutable int64_t ss_rows_h = -1, ss_rows_hk = -1;
  int32_t* pos_k = nullptr;
  float* s_k = nullptr;
  float* lsig_k = nullptr;
  void* kaug_k = nullptr;  // bf16 [k, 16] gate-bias rows of the kept tokens
  void* sel_ws = nullptr;
  float2* cs_n = nullptr;  // [dh/2][n] cos/sin of positions 0..n-1 (dense stage)
  float2* cs_k = nullptr;  // [dh/2][k] cos/sin of the kept positions
  AttnPlan attn;           // sized for n rows, reused by every layer
  // hybrid stacks (Gated DeltaNet layers): projections, mixer output, mixer
  // workspace, sized for n rows and the widest such layer
  void* gdn_proj = nullptr;
  void* gdn_y = nullptr;
  void* gdn_ws = nullptr;
  size_t bytes = 0;
  // (the attention's split scratch serves any gated layer of up to 8192 rows)
  PrefillPlan(void* ws, const tg_model& m, int64_t n, int64_t k)
      : attn(nullptr, n, m.n_heads_q, m.n_heads_kv, m.head_dim, m.dtype, true, 1) {
    Arena a(ws);
    const size_t e = elem_size(m.dtype);
    const int d = m.d_model, hq = m.n_heads_q, hkv = m.n_heads_kv, dh = m.head_dim;
    h = a.carve(size_t(n) * d * e);
    hk = a.carve(size_t(k) * d * e);
    y = a.carve(size_t(n) * d * e);
    // the un-fused projection path only: bf16 attention with head_dim 128 and
    // paired query heads projects straight into q / k / V^T (QKV epilogue)
    if (!(m.dtype == TG_BF16 && dh == 128 && hq % 2 == 0))
      qkv = a.carve(size_t(n) * (hq + 2 * hkv) * dh * e);
    attn_o = a.carve(size_t(n) * hq * dh * e);
    if (m.d_ffn > 0) {  // the FFN runs in row blocks of at most kFfnRows
      const size_t fr = static_cast<size_t>(std::min<int64_t>(n, kFfnRows));
      mlp = a.carve(fr * m.d_ffn * e);
      if (m.dtype == TG_F32) gu = a.carve(fr * 2 * m.d_ffn * 4);
    }
    scores = static_cast<float*>(a.carve(size_t(n) * 4));
    if (m.dtype == TG_BF16) {
      ss_parts = ss_parts_of(d);
      ss_ld = n;
      ss_ld_k = k;
      ss = static_cast<float*>(a.carve(size_t(ss_parts) * n * 4));
      ss_k = static_cast<float*>(a.carve(size_t(ss_parts) * k * 4));
    }
    if (m.dtype == TG_F32) hpre = static_cast<float*>(a.carve(size_t(n) * m.d_score * 4));
    pos_k = static_cast<int32_t*>(a.carve(size_t(k) * 4));
    s_k = static_cast<float*>(a.carve(size_t(k) * 4));
    lsig_k = static_cast<float*>(a.carve(size_t(k) * 4));
    if (m.dtype == TG_BF16) kaug_k = a.carve(size_t(k) * 32);
    sel_ws = a.carve(select_ws_bytes(n));
    cs_n = static_cast<float2*>(a.carve(size_t(n) * (dh / 2) * sizeof(float2)));
    cs_k = static_cast<float2*>(a.carve(size_t(k) * (dh / 2) * sizeof(float2)));
    void* attn_base = a.carve(attn.bytes);
    attn = AttnPlan(attn_base, n, hq, hkv, dh, m.dtype, true, 1);
    size_t proj_w = 0, y_w = 0, gws = 0;
    for (int l = 0; l < m.n_layers; ++l) {
      const tg_gdn_layer* G = m.layers[l].gdn;
      if (G == nullptr) continue;
      proj_w = std::max(proj_w, static_cast<size_t>(gdn_proj_width(*G)));
      y_w = std::max(y_w, static_cast<size_t>(G->n_heads_v) * G->head_dim_v);
      gws = std::max(gws, GdnPlan(nullptr, n, G->n_heads_k, G->n_heads_v, G->head_dim_k,
                                  G->head_dim_v).bytes);
    }
    if (proj_w > 0) {
      gdn_proj = a.carve(size_t(n) * proj_w * e);
      gdn_y = a.carve(size_t(n) * y_w * e);
      gdn_ws = a.carve(gws);
    }
    bytes = a.used;
  }
};

// ------------------------------------------------------------------ pieces

cudaError_t gemm(const GemmArgs& g, tg_dtype dt, cudaStream_t st) {
  const double e = static_cast<double>(elem_size(dt));
  const double flops = 2.0 * double(g.M) * g.N * g.K;
  double out_bytes = 0.0;
  tg_kernel kid = TG_K_GEMM_F32;
  switch (g.epi) {
    case EPI_STORE: out_bytes = double(g.M) * g.N * e; kid = TG_K_GEMM_STORE; break;
    case EPI_RESIDUAL: out_bytes = 2.0 * double(g.M) * g.N * e; kid = TG_K_GEMM_RESIDUAL; break;
    case EPI_SWIGLU: out_bytes = double(g.M) * g.inter * e; kid = TG_K_GEMM_SWIGLU; break;
    case EPI_SCORE: out_bytes = double(g.M) * 4.0; kid = TG_K_GEMM_SCORE; break;
    case EPI_QKV: out_bytes = double(g.M) * g.N * e + (g.v_out ? double(g.M) * g.hkv * 128 * e : 0.0);
      kid = TG_K_GEMM_QKV; break;
  }
  const double bytes = (double(g.M) + g.N) * g.K * e + out_bytes;
  if (dt == TG_BF16) {
    if (!gemm_tc_supported(g)) return cudaErrorInvalidValue;
    return traced(kid, g.M, flops, bytes, st, [&] { return launch_gemm_tc(g, st); });
  }
  return traced(TG_K_GEMM_F32, g.M, flops, bytes, st, [&] { return launch_gemm_simt_f32(g, st); });
}

cudaError_t rmsnorm(const void* x, const float* gamma, float eps, int64_t rows, int d, tg_dtype dt,
                    void* y, cudaStream_t st) {
  const double bytes = 2.0 * double(rows) * d * elem_size(dt) + 4.0 * d;
  return traced(TG_K_RMSNORM, rows, 0.0, bytes, st,
                [&] { return launch_rmsnorm(x, gamma, eps, rows, d, dt == TG_BF16, y, st); });
}

cudaError_t copy_rows(void* dst, const void* src, size_t bytes, int64_t rows, cudaStream_t st) {
  return traced(TG_K_COPY, rows, 0.0, 2.0 * double(bytes), st, [&] {
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st);
  });
}

cudaError_t select_topk(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                        int32_t* kept, void* ws, cudaStream_t st) {
  const double bytes = 4.0 * n + (protect ? double(n) : 0.0) + 4.0 * k;
  return traced(TG_K_SELECT, n, 0.0, bytes, st,
                [&] { return launch_topk_select(scores, protect, n, k, kept, ws, st); });
}

cudaError_t compact(const void* x, const int32_t* pos_in, const float* scores, const int32_t* idx,
                    int64_t n, int64_t k, int row_bytes, void* x_out, int32_t* pos_out,
                    float* s_out, float* lsig_out, cudaStream_t st, const SsGather& ss = {}) {
  const double bytes = 2.0 * double(k) * row_bytes + 4.0 * k /*idx*/ + 4.0 * k /*pos*/ +
                       (scores ? 4.0 * k : 0.0) + (s_out ? 4.0 * k : 0.0) +
                       (lsig_out ? 4.0 * k : 0.0);
  return traced(TG_K_COMPACT, k, 0.0, bytes, st, [&] {
    return launch_compact(x, pos_in, scores, idx, n, k, row_bytes, x_out, pos_out, s_out,
                          lsig_out, ss, st);
  });
}

GemmArgs gemm_args(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc,
                   int64_t M, int N, int K, EpiKind epi) {
  GemmArgs g{};
  g.A = A; g.lda = lda; g.B = B; g.ldb = ldb; g.C = C; g.ldc = ldc;
  g.M = M; g.N = N; g.K = K; g.epi = epi;
  return g;
}

// Folded RMSNorm: rows [0, rows) of the stream h carry the row sums of
// squares their last residual GEMM left in P.ss.
bool ss_ready(const PrefillPlan& P, const void* h, int64_t rows) {
  if (P.ss == nullptr) return false;
  if (h == P.h) return P.ss_rows_h == rows;
  return h == P.hk && P.ss_rows_hk == rows;
}
// The row sums of the stream h (the all-token buffer or the kept-row one).
float* ss_of(const PrefillPlan& P, const void* h) { return h == P.hk ? P.ss_k : P.ss; }
int64_t ss_ld_of(const PrefillPlan& P, const void* h) { return h == P.hk ? P.ss_ld_k : P.ss_ld; }
// The projection of rows [row0, row0 + M) of h scales its accumulator rows by 1 / rms.
void ss_consume(GemmArgs& g, const PrefillPlan& P, const void* h, float eps, int d, int64_t row0) {
  g.ss_in = ss_of(P, h) + row0;
  g.ss_ld = ss_ld_of(P, h);
  g.ss_parts = P.ss_parts;
  g.ss_inv_n = 1.0f / static_cast<float>(d);
  g.ss_eps = eps;
}
// The residual GEMM of rows [row0, row0 + M) of h leaves their sums of squares.
void ss_produce(GemmArgs& g, const PrefillPlan& P, const void* h, int64_t row0) {
  if (P.ss == nullptr) return;
  g.ss_out = ss_of(P, h) + row0;
  g.ss_ld = ss_ld_of(P, h);
}
void ss_mark(const PrefillPlan& P, const void* h, int64_t rows) {
  if (P.ss == nullptr) return;
  if (h == P.h) P.ss_rows_h = rows;
  if (h == P.hk) P.ss_rows_hk = rows;
}

// Scorer over `rows` rows of x (dtype dt) into scores[rows]. With a plan
// whose row sums describe x and the folded w1_g, no RMSNorm kernel runs.
cudaError_t run_score(const void* x, int64_t rows, int d, int f, const float* norm_w, float eps,
                      const void* w1, const float* b1, const float* w2, const float* b2,
                      tg_dtype dt, float* scores, void* y, float* hpre, cudaStream_t st,
                      const PrefillPlan* P = nullptr, const void* w1_g = nullptr) {
  const bool fold = P != nullptr && w1_g != nullptr && ss_ready(*P, x, rows);
  cudaError_t e = cudaSuccess;
  if (!fold) {
    e = rmsnorm(x, norm_w, eps, rows, d, dt, y, st);
    if (e != cudaSuccess) return e;
  }
  if (dt == TG_BF16) {
    GemmArgs g = gemm_args(fold ? x : y, d, fold ? w1_g : w1, d, nullptr, 0, rows, f, d, EPI_SCORE);
    g.b1 = b1; g.w2 = w2; g.b2 = b2; g.scores = scores;
    if (fold) ss_consume(g, *P, x, eps, d, 0);
    return gemm(g, dt, st);
  }
  GemmArgs g = gemm_args(y, d, w1, d, hpre, f, rows, f, d, EPI_STORE);
  e = gemm(g, dt, st);
  if (e != cudaSuccess) return e;
  return traced(TG_K_F32_HELPER, rows, 0.0, double(rows) * f * 4.0, st, [&] {
    return launch_score_dot_f32(hpre, rows, f, b1, w2, b2, scores, st);
  });
}

// Attention over prepared (rotated) q/k and prepared V (bf16: V^T [hkv, dh, t_pad]).
cudaError_t attn_core(const AttnPlan& plan, const void* k_rot, const void* v, int64_t v_stride,
                      const float* lsig, const void* kaug, const float* gain, const float* tau,
                      int64_t rows, int hq, int hkv, int dh, tg_dtype dt, void* out,
                      cudaStream_t st, float* lse = nullptr, float* out_f32 = nullptr,
                      bool split_cnt_zeroed = false, int64_t q_lo = 0, bool whole_tiles = false) {
  const size_t es = elem_size(dt);
  // causal work of query rows [q_lo, rows) over keys [0, rows)
  const double attn_flops = 4.0 * dh * hq *
                            (double(rows) * double(rows + 1) - double(q_lo) * double(q_lo + 1)) / 2.0;
  const double attn_bytes = double(rows - q_lo) * 2 * hq * dh * es + double(rows) * 2 * hkv * dh * es;
  AttnArgs a{};
  a.q = plan.q_rot;
  a.k = k_rot;
  a.lsig = lsig;
  a.kaug = kaug;
  a.gain = gain; a.tau = tau;
  a.T = rows; a.hq = hq; a.hkv = hkv; a.dh = dh;
  a.out = out;
  a.lse = lse;
  a.out_f32 = out_f32;
  // whole_tiles: one CTA per query tile (no split tiles), as in a launch over
  // more rows than the split schedule covers
  a.split_ws = whole_tiles ? nullptr : plan.split;
  a.split_ws_bytes = whole_tiles ? 0 : plan.split_bytes;
  a.split_cnt_zeroed = split_cnt_zeroed;
  a.q_lo = q_lo;
  if (dt == TG_BF16) {
    a.v = plan.vT;
    a.t_pad = plan.t_pad;
    if (!attn_tc_supported(a)) return cudaErrorInvalidValue;
    return traced(TG_K_ATTENTION, rows, attn_flops, attn_bytes, st,
                  [&] { return launch_attn_tc(a, st); });
  }
  a.v = v;
  a.t_pad = v_stride;
  return traced(TG_K_ATTENTION_F32, rows, attn_flops, attn_bytes, st,
                [&] { return launch_attn_simt_f32(a, st); });
}

// RoPE/qk-norm prep + attention, q/k/v taken from rows with the given strides.
cudaError_t run_attention(const void* q, int64_t q_stride, const void* kk, int64_t k_stride,
                          const void* v, int64_t v_stride, const int32_t* pos, const float* s,
                          const float* lsig_ready, const float* gain, const float* tau,
                          const float* q_norm, const float* k_norm, float eps, int64_t rows,
                          int hq, int hkv, int dh, float rope_base, tg_dtype dt,
                          const AttnPlan& plan, void* k_out, void* v_out, void* out,
                          cudaStream_t st, float* lse = nullptr, float* out_f32 = nullptr) {
  RopePrepArgs r{};
  r.q_src = q; r.k_src = kk; r.v_src = v;
  r.q_stride = q_stride; r.k_stride = k_stride; r.v_stride = v_stride;
  r.pos = pos; r.q_norm = q_norm; r.k_norm = k_norm; r.eps = eps;
  r.T = rows; r.hq = hq; r.hkv = hkv; r.dh = dh; r.rope_base = rope_base;
  r.bf16 = dt == TG_BF16;
  r.q_out = plan.q_rot;
  r.k_out = k_out ? k_out : plan.k_rot;
  r.vT_out = dt == TG_BF16 ? plan.vT : nullptr;
  r.t_pad = plan.t_pad;
  r.kv_v_out = v_out;
  r.s = lsig_ready ? nullptr : s;
  r.lsig_out = plan.lsig;
  const size_t es = elem_size(dt);
  const double prep_bytes = double(rows) * (hq + hkv) * dh * es * 2.0 +
                            (dt == TG_BF16 ? double(rows) * hkv * dh * es * 2.0 : 0.0) +
                            (v_out ? double(rows) * hkv * dh * es : 0.0) + (r.s ? 8.0 * rows : 0.0);
  cudaError_t e = traced(TG_K_ROPE_PREP, rows, 0.0, prep_bytes, st,
                         [&] { return launch_rope_prep(r, st); });
  if (e != cudaSuccess) return e;
  const float* lsig = (s || lsig_ready) ? (lsig_ready ? lsig_ready : plan.lsig) : nullptr;
  if (lsig && dt == TG_BF16) {
    e = traced(TG_K_ROPE_PREP, rows, 0.0, 36.0 * rows, st,
               [&] { return launch_bias_aug(lsig, rows, plan.kaug, st); });
    if (e != cudaSuccess) return e;
  }
  return attn_core(plan, r.k_out, v, v_stride, lsig, dt == TG_BF16 ? plan.kaug : nullptr, gain,
                   tau, rows, hq, hkv, dh, dt, out, st, lse, out_f32);
}

// ---- the decoder-layer pieces used by tg_prefill

struct Dims {
  int d, hq, hkv, dh, inter, qkv;
};

// Attention of several packed requests, one launch per request over its own
// rows (see SegRows: request b's rows start at segs.off[b], a multiple of
// 128, so every slice of q, k, V^T and the bias rows stays 16-byte aligned).
cudaError_t attn_segments(const AttnPlan& plan, const void* k_rot, const float* lsig,
                          const void* kaug, const float* gain, const float* tau,
                          const SegRows& segs, int hq, int hkv, int dh, void* out,
                          cudaStream_t st) {
  const size_t e = 2;
  for (int b = 0; b < segs.count; ++b) {
    const int64_t off = segs.off[b], rows = segs.len[b];
    AttnArgs a{};
    a.q = static_cast<const char*>(plan.q_rot) + size_t(off) * hq * dh * e;
    a.k = static_cast<const char*>(k_rot) + size_t(off) * hkv * dh * e;
    a.v = static_cast<const char*>(plan.vT) + size_t(off) * e;  // column offset in V^T rows
    a.t_pad = plan.t_pad;
    a.lsig = lsig ? lsig + off : nullptr;
    a.kaug = kaug ? static_cast<const char*>(kaug) + size_t(off) * 32 : nullptr;
    a.gain = gain;
    a.tau = tau;
    a.T = rows; a.hq = hq; a.hkv = hkv; a.dh = dh;
    a.out = static_cast<char*>(out) + size_t(off) * hq * dh * e;
    a.split_ws = plan.split;
    a.split_ws_bytes = plan.split_bytes;
    a.split_cnt_zeroed = true;
    if (!attn_tc_supported(a)) return cudaErrorInvalidValue;
    const double fl = 4.0 * dh * hq * double(rows) * double(rows + 1) / 2.0;
    const double by = double(rows) * (2 * hq + 2 * hkv) * dh * e;
    const cudaError_t err =
        traced(TG_K_ATTENTION, rows, fl, by, st, [&] { return launch_attn_tc(a, st); });
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

cudaError_t attention_sublayer(const tg_model& m, const tg_layer& lw, const Dims& D,
                               const PrefillPlan& P, void* h, int64_t rows, const int32_t* pos,
                               const float2* cs, const float* lsig, const void* kaug,
                               const float* gain, const float* tau, const tg_kv* kv,
                               cudaStream_t st, const SegRows* segs = nullptr,
                               const tg_layer_taps* taps = nullptr,
                               const void* h_in = nullptr) {
  const tg_dtype dt = m.dtype;
  const size_t e = elem_size(dt);
  // h_in: the sub-layer's input rows when they are not in h yet (the
  // stack's input, read in place); the output rows h = h_in + attention go to h
  const void* hsrc = h_in ? h_in : h;
  // folded RMSNorm (h's rows fresh from a residual GEMM), else the norm kernel
  const bool fold = lw.wqkv_g != nullptr && h_in == nullptr && ss_ready(P, h, rows);
  cudaError_t err = cudaSuccess;
  if (!fold) {
    err = rmsnorm(hsrc, lw.attn_norm, m.norm_eps, rows, D.d, dt, P.y, st);
    if (err != cudaSuccess) return err;
  }
  const void* xin = fold ? h : P.y;
  const void* wqkv = fold ? lw.wqkv_g : lw.wqkv;
  void* k_dst = (kv && kv->k) ? kv->k : P.attn.k_rot;
  GemmArgs gq = gemm_args(xin, D.d, wqkv, D.d, nullptr, 0, rows, D.qkv, D.d, EPI_QKV);
  if (fold) ss_consume(gq, P, h, m.norm_eps, D.d, 0);
  gq.hq = D.hq; gq.hkv = D.hkv; gq.rope_cs = cs; gq.q_norm = lw.q_norm; gq.k_norm = lw.k_norm;
  gq.eps = m.norm_eps; gq.q_out = P.attn.q_rot; gq.k_out = k_dst; gq.vT_out = P.attn.vT;
  gq.t_pad = P.attn.t_pad; gq.v_out = kv ? kv->v : nullptr;
  if (dt == TG_BF16 && D.dh == 128 && cs != nullptr && gemm_tc_supported(gq)) {
    // fused: projection + qk-norm + RoPE + V^T in the GEMM epilogue
    err = gemm(gq, dt, st);
    if (err != cudaSuccess) return err;
    if (segs != nullptr)
      err = attn_segments(P.attn, k_dst, lsig, kaug, gain, tau, *segs, D.hq, D.hkv, D.dh,
                          P.attn_o, st);
    else
      err = attn_core(P.attn, k_dst, nullptr, 0, lsig, kaug, gain, tau, rows, D.hq, D.hkv, D.dh,
                      dt, P.attn_o, st, nullptr, nullptr, true);
  } else if (segs != nullptr || P.qkv == nullptr) {
    return cudaErrorInvalidValue;  // packed requests need the fused bf16 path
  } else {
    GemmArgs gs = gemm_args(xin, D.d, wqkv, D.d, P.qkv, D.qkv, rows, D.qkv, D.d, EPI_STORE);
    if (fold) ss_consume(gs, P, h, m.norm_eps, D.d, 0);
    err = gemm(gs, dt, st);
    if (err != cudaSuccess) return err;
    const char* qkv = static_cast<const char*>(P.qkv);
    err = run_attention(qkv, D.qkv, qkv + size_t(D.hq) * D.dh * e, D.qkv,
                        qkv + size_t(D.hq + D.hkv) * D.dh * e, D.qkv, pos, nullptr, lsig, gain,
                        tau, lw.q_norm, lw.k_norm, m.norm_eps, rows, D.hq, D.hkv, D.dh,
                        m.rope_base, dt, P.attn, kv ? kv->k : nullptr, kv ? kv->v : nullptr,
                        P.attn_o, st);
  }
  if (err != cudaSuccess) return err;
  if (taps && taps->attn_out) {
    err = copy_rows(taps->attn_out, P.attn_o, size_t(rows) * D.hq * D.dh * e, rows, st);
    if (err != cudaSuccess) return err;
  }
  GemmArgs g = gemm_args(P.attn_o, int64_t(D.hq) * D.dh, lw.wo, int64_t(D.hq) * D.dh, h, D.d, rows,
                         D.d, D.hq * D.dh, EPI_RESIDUAL);
  g.R = hsrc;
  g.ldr = D.d;
  ss_produce(g, P, h, 0);
  err = gemm(g, dt, st);
  if (err != cudaSuccess) return err;
  ss_mark(P, h, rows);
  if (!taps || !taps->resid) return err;
  return copy_rows(taps->resid, h, size_t(rows) * D.d * e, rows, st);
}

cudaError_t ffn_sublayer(const tg_model& m, const tg_layer& lw, const Dims& D,
                         const PrefillPlan& P, void* h, int64_t rows, cudaStream_t st) {
  if (lw.w_gate_up == nullptr) return cudaSuccess;
  const tg_dtype dt = m.dtype;
  const size_t e = elem_size(dt);
  // folded RMSNorm (h's rows fresh from a residual GEMM), else the norm kernel
  const bool fold = lw.w_gate_up_g != nullptr && ss_ready(P, h, rows);
  cudaError_t err = cudaSuccess;
  if (!fold) {
    err = rmsnorm(h, lw.ffn_norm, m.norm_eps, rows, D.d, dt, P.y, st);
    if (err != cudaSuccess) return err;
  }
  // row blocks of at most kFfnRows share the intermediate buffer
  for (int64_t r0 = 0; r0 < rows; r0 += kFfnRows) {
    const int64_t rb = std::min<int64_t>(kFfnRows, rows - r0);
    const char* yb = static_cast<const char*>(fold ? h : P.y) + size_t(r0) * D.d * e;
    void* hb = static_cast<char*>(h) + size_t(r0) * D.d * e;
    if (dt == TG_BF16) {
      GemmArgs g = gemm_args(yb, D.d, fold ? lw.w_gate_up_g : lw.w_gate_up, D.d, P.mlp, D.inter, rb,
                             2 * D.inter, D.d, EPI_SWIGLU);
      g.inter = D.inter;
      if (fold) ss_consume(g, P, h, m.norm_eps, D.d, r0);
      err = gemm(g, dt, st);
    } else {
      err = gemm(gemm_args(yb, D.d, lw.w_gate_up, D.d, P.gu, 2 * D.inter, rb, 2 * D.inter, D.d,
                           EPI_STORE), dt, st);
      if (err == cudaSuccess)
        err = traced(TG_K_F32_HELPER, rb, 0.0, double(rb) * D.inter * 12.0, st, [&] {
          return launch_swiglu_f32(static_cast<const float*>(P.gu), rb, D.inter,
                                   static_cast<float*>(P.mlp), st);
        });
    }
    if (err != cudaSuccess) return err;
    GemmArgs g = gemm_args(P.mlp, D.inter, lw.w_down, D.inter, hb, D.d, rb, D.d, D.inter,
                           EPI_RESIDUAL);
    g.R = hb;
    g.ldr = D.d;
    ss_produce(g, P, h, r0);
    err = gemm(g, dt, st);
    if (err != cudaSuccess) return err;
  }
  ss_mark(P, h, rows);
  return cudaSuccess;
}

cudaError_t gdn_run(const GdnArgs& g, bool bf, cudaStream_t st) {
  const int64_t T = g.T;
  const double C = double(2 * g.hk * g.dk + g.hv * g.dv);
  const double e = bf ? 2.0 : 4.0, tt = double(T);
  const double prep_bytes = tt * (C * e + 2.0 * g.hv * e) + tt * 4.0 * (C + g.hv * 2.0);
  const double chunk_flops = tt * g.hv * 2.0 * kGdnChunk * g.dk;  // the two Gram products
  const double recur_flops = tt * g.hv * 6.0 * g.dv * g.dk;
  const double out_bytes = tt * g.hv * g.dv * (4.0 + 2.0 * e);
  cudaError_t err =
      traced(TG_K_GDN_PREP, T, 0.0, prep_bytes, st, [&] { return launch_gdn(g, bf, 0, st); });
  if (err == cudaSuccess)
    err = traced(TG_K_GDN_CHUNK, T, chunk_flops, 0.0, st, [&] { return launch_gdn(g, bf, 1, st); });
  if (err == cudaSuccess)
    err = traced(TG_K_GDN_RECUR, T, recur_flops, 0.0, st, [&] { return launch_gdn(g, bf, 2, st); });
  if (err == cudaSuccess)
    err = traced(TG_K_GDN_OUT, T, 0.0, out_bytes, st, [&] { return launch_gdn(g, bf, 3, st); });
  return err;
}

// A hybrid model's Gated DeltaNet layer (token mixer part) over `rows` rows
// of h: h += W_out . mixer(W_in . RMSNorm(h)), the mixer running over each
// sequence (one, or each packed request of `segs`) in row order. kv, when
// given, receives the last conv rows (k) and the final state (v).
cudaError_t gdn_sublayer(const tg_model& m, const tg_layer& lw, const Dims& D,
                         const PrefillPlan& P, void* h, int64_t rows, const tg_kv* kv,
                         cudaStream_t st, const SegRows* segs, const tg_layer_taps* taps) {
  const tg_gdn_layer& G = *lw.gdn;
  const tg_dtype dt = m.dtype;
  const size_t e = elem_size(dt);
  const int64_t C = gdn_channels(G), Nt = gdn_proj_width(G);
  const int hv = G.n_heads_v, vd = G.n_heads_v * G.head_dim_v;
  cudaError_t err = rmsnorm(h, lw.attn_norm, m.norm_eps, rows, D.d, dt, P.y, st);
  if (err != cudaSuccess) return err;
  err = gemm(gemm_args(P.y, D.d, lw.w_in, D.d, P.gdn_proj, Nt, rows, static_cast<int>(Nt), D.d,
                       EPI_STORE), dt, st);
  if (err != cudaSuccess) return err;
  if (taps && taps->mixer_in) {
    err = copy_rows(taps->mixer_in, P.gdn_proj, size_t(rows) * Nt * e, rows, st);
    if (err != cudaSuccess) return err;
  }
  const int n_seq = segs ? segs->count : 1;
  for (int b = 0; b < n_seq; ++b) {
    const int64_t off = segs ? segs->off[b] : 0, len = segs ? segs->len[b] : rows;
    GdnArgs g = GdnPlan(P.gdn_ws, len, G.n_heads_k, hv, G.head_dim_k, G.head_dim_v).a;
    const char* pr = static_cast<const char*>(P.gdn_proj) + size_t(off) * Nt * e;
    g.qkv = pr;
    g.z = pr + size_t(C) * e;
    g.a = pr + size_t(C + vd) * e;
    g.b = pr + size_t(C + vd + hv) * e;
    g.ld_qkv = g.ld_z = g.ld_ab = Nt;
    g.T = len;
    g.hk = G.n_heads_k;
    g.hv = hv;
    g.dk = G.head_dim_k;
    g.dv = G.head_dim_v;
    g.W = G.conv_width;
    g.conv_w = G.conv_w;
    g.A_log = G.A_log;
    g.dt_bias = G.dt_bias;
    g.norm_w = G.norm_w;
    g.eps = G.norm_eps;
    g.conv_in = nullptr;
    g.state_in = nullptr;
    g.conv_out = (kv && !segs) ? kv->k : nullptr;
    g.state_out = (kv && !segs) ? static_cast<float*>(kv->v) : nullptr;
    g.y = static_cast<char*>(P.gdn_y) + size_t(off) * vd * e;
    g.err = device_error_word();
    err = gdn_run(g, dt == TG_BF16, st);
    if (err != cudaSuccess) return err;
  }
  if (taps && taps->attn_out) {
    err = copy_rows(taps->attn_out, P.gdn_y, size_t(rows) * vd * e, rows, st);
    if (err != cudaSuccess) return err;
  }
  GemmArgs g = gemm_args(P.gdn_y, vd, lw.w_out, vd, h, D.d, rows, D.d, vd, EPI_RESIDUAL);
  g.R = h;
  g.ldr = D.d;
  ss_produce(g, P, h, 0);
  err = gemm(g, dt, st);
  if (err != cudaSuccess) return err;
  ss_mark(P, h, rows);
  if (!taps || !taps->resid) return err;
  return copy_rows(taps->resid, h, size_t(rows) * D.d * e, rows, st);
}

// The token-mixer sub-layer of layer lw: attention, or the Gated DeltaNet
// mixer of a hybrid model's linear-attention layer.
cudaError_t mixer_sublayer(const tg_model& m, const tg_layer& lw, const Dims& D,
                           const PrefillPlan& P, void* h, int64_t rows, const int32_t* pos,
                           const float2* cs, const float* lsig, const void* kaug,
                           const float* gain, const float* tau, const tg_kv* kv, cudaStream_t st,
                           const SegRows* segs = nullptr, const tg_layer_taps* taps = nullptr) {
  if (lw.gdn != nullptr) return gdn_sublayer(m, lw, D, P, h, rows, kv, st, segs, taps);
  return attention_sublayer(m, lw, D, P, h, rows, pos, cs, lsig, kaug, gain, tau, kv, st, segs,
                            taps);
}

// Workspace of one decode step (batch 1, bf16).
struct DecodePlan {
  __nv_bfloat16* h = nullptr;    // [d] the token's residual stream
  __nv_bfloat16* qkv = nullptr;  // [(hq + 2 hkv) dh] projected q | k | v
  __nv_bfloat16* o = nullptr;    // [hq dh] attention output
  __nv_bfloat16* act = nullptr;  // [I] SwiGLU product
  float* lsig = nullptr;         // [k_kept] logsigmoid of the kept prompt scores
  float* part = nullptr;         // split softmax states of the attention
  unsigned int* cnt = nullptr;   // [hkv] split counters, then [2] grid-barrier words
  size_t cnt_bytes = 0;
  size_t bytes = 0;
  DecodePlan(void* base, const tg_model& m, int64_t k_kept) {
    Arena a(base);
    const int64_t dh = m.head_dim, hq = m.n_heads_q, hkv = m.n_heads_kv;
    h = static_cast<__nv_bfloat16*>(a.carve(size_t(m.d_model) * 2));
    qkv = static_cast<__nv_bfloat16*>(a.carve(size_t(hq + 2 * hkv) * dh * 2));
    o = static_cast<__nv_bfloat16*>(a.carve(size_t(hq) * dh * 2));
    act = static_cast<__nv_bfloat16*>(a.carve(size_t(m.d_ffn > 0 ? m.d_ffn : 1) * 2));
    lsig = static_cast<float*>(a.carve(size_t(k_kept > 0 ? k_kept : 1) * 4));
    part = static_cast<float*>(
        a.carve(size_t(hkv) * kDecodeMaxSplits * size_t(hq / (hkv > 0 ? hkv : 1)) * (dh + 2) * 4));
    cnt_bytes = size_t(hkv + 2) * 4;
    cnt = static_cast<unsigned int*>(a.carve(cnt_bytes));
    bytes = a.used;
  }
};

tg_status validate_decode(const tg_model* m, const void* x, int64_t pos, int gate_layer,
                          const tg_kv* kv, const int64_t* lens, const float* scores, int64_t n,
                          const int32_t* kept_idx, int64_t k_kept, const void* out) {
  TG_CHECK(m != nullptr && m->layers != nullptr && x && out && kv && lens, TG_ERR_INVALID_ARG);
  TG_CHECK(m->dtype == TG_BF16 || m->dtype == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(m->dtype == TG_BF16 && m->head_dim == 128, TG_ERR_UNSUPPORTED);
  TG_CHECK(m->n_layers >= 1 && m->d_model > 0 && m->n_heads_q > 0 && m->n_heads_kv > 0,
           TG_ERR_INVALID_ARG);
  TG_CHECK(m->n_layers <= kDecodeMaxLayers, TG_ERR_UNSUPPORTED);
  TG_CHECK(m->n_heads_q % m->n_heads_kv == 0, TG_ERR_INVALID_ARG);
  const int group = m->n_heads_q / m->n_heads_kv;
  TG_CHECK(group == 1 || group == 2 || group == 4 || group == 8, TG_ERR_UNSUPPORTED);
  TG_CHECK(m->d_model % 8 == 0 && (m->d_ffn <= 0 || m->d_ffn % 8 == 0), TG_ERR_UNSUPPORTED);
  // a stage's input vector is staged in registers, 4 x 16 bytes per thread
  TG_CHECK(m->d_model <= 8192 && m->d_ffn <= 8192 && m->n_heads_q * 128 <= 8192,
           TG_ERR_UNSUPPORTED);
  TG_CHECK(gate_layer >= -1 && gate_layer < m->n_layers, TG_ERR_INVALID_ARG);
  TG_CHECK(pos >= 0 && pos < (int64_t(1) << 31), TG_ERR_INVALID_ARG);
  TG_CHECK(std::isfinite(m->norm_eps) && m->norm_eps >= 0.f && m->rope_base > 1.f,
           TG_ERR_INVALID_ARG);
  TG_CHECK(aligned16(x) && aligned16(out), TG_ERR_INVALID_ARG);
  if (scores != nullptr) {
    TG_CHECK(kept_idx != nullptr && n >= 1, TG_ERR_INVALID_ARG);
    TG_CHECK(k_kept >= 1 && k_kept <= n, TG_ERR_BUDGET);
  }
  for (int l = 0; l < m->n_layers; ++l) {
    const tg_layer& L = m->layers[l];
    TG_CHECK(L.gdn == nullptr, TG_ERR_UNSUPPORTED);  // attention layers only
    TG_CHECK(L.attn_norm && L.wqkv && L.wo, TG_ERR_INVALID_ARG);
    TG_CHECK((L.q_norm == nullptr) == (L.k_norm == nullptr), TG_ERR_INVALID_ARG);
    if (L.w_gate_up) TG_CHECK(L.w_down && L.ffn_norm && m->d_ffn > 0, TG_ERR_INVALID_ARG);
    TG_CHECK(aligned16(L.wqkv) && aligned16(L.wo) && aligned16(L.attn_norm), TG_ERR_INVALID_ARG);
    if (L.w_gate_up)
      TG_CHECK(aligned16(L.w_gate_up) && aligned16(L.w_down) && aligned16(L.ffn_norm),
               TG_ERR_INVALID_ARG);
    TG_CHECK(kv[l].k != nullptr && kv[l].v != nullptr, TG_ERR_INVALID_ARG);
    TG_CHECK(aligned16(kv[l].k) && aligned16(kv[l].v), TG_ERR_INVALID_ARG);
    TG_CHECK(lens[l] >= 0 && lens[l] < (int64_t(1) << 31) - 1, TG_ERR_INVALID_ARG);
    // above the gate the kept prompt tokens are the first k_kept cache rows
    if (l > gate_layer && scores != nullptr) TG_CHECK(lens[l] >= k_kept, TG_ERR_INVALID_ARG);
  }
  return TG_OK;
}

// Columns of a Gated DeltaNet layer's input projection: qkv (C channels),
// z (hv dv), a and b (hv each).
int64_t gdn_channels(const tg_gdn_layer& G) {
  return 2 * int64_t(G.n_heads_k) * G.head_dim_k + int64_t(G.n_heads_v) * G.head_dim_v;
}
int64_t gdn_proj_width(const tg_gdn_layer& G) {
  return gdn_channels(G) + int64_t(G.n_heads_v) * G.head_dim_v + 2 * int64_t(G.n_heads_v);
}

tg_status validate_gdn_layer(const tg_gdn_layer* L) {
  TG_CHECK(L != nullptr, TG_ERR_INVALID_ARG);
  TG_CHECK(L->n_heads_k >= 1 && L->n_heads_v >= 1 && L->n_heads_v % L->n_heads_k == 0 &&
               L->n_heads_v <= 4096,
           TG_ERR_INVALID_ARG);
  TG_CHECK(L->conv_width >= 1 && L->conv_width <= 4, TG_ERR_INVALID_ARG);
  TG_CHECK(L->conv_w && L->A_log && L->dt_bias && L->norm_w, TG_ERR_INVALID_ARG);
  TG_CHECK(std::isfinite(L->norm_eps) && L->norm_eps >= 0.f, TG_ERR_INVALID_ARG);
  TG_CHECK(L->head_dim_k == 64 || L->head_dim_k == 128, TG_ERR_UNSUPPORTED);
  TG_CHECK(L->head_dim_v >= 32 && L->head_dim_v <= 256 && L->head_dim_v % 32 == 0,
           TG_ERR_UNSUPPORTED);
  return TG_OK;
}

tg_status validate_model(const tg_model* m, int64_t n, int64_t k, int gate_layer) {
  TG_CHECK(m != nullptr && m->layers != nullptr, TG_ERR_INVALID_ARG);
  TG_CHECK(m->dtype == TG_BF16 || m->dtype == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(m->n_layers >= 1 && m->d_model > 0 && m->n_heads_q > 0 && m->n_heads_kv > 0,
           TG_ERR_INVALID_ARG);
  TG_CHECK(m->n_heads_q % m->n_heads_kv == 0, TG_ERR_INVALID_ARG);
  TG_CHECK(gate_layer >= -1 && gate_layer < m->n_layers, TG_ERR_INVALID_ARG);
  TG_CHECK(n >= 1 && n < (int64_t(1) << 31) - 256, TG_ERR_INVALID_ARG);
  TG_CHECK(k >= 1 && k <= n, TG_ERR_BUDGET);
  TG_CHECK(m->score_norm && m->score_w1 && m->score_w2 && m->d_score >= 1, TG_ERR_INVALID_ARG);
  TG_CHECK(std::isfinite(m->norm_eps) && m->norm_eps >= 0.f && m->rope_base > 1.f,
           TG_ERR_INVALID_ARG);
  const int d = m->d_model, dh = m->head_dim, qkv = (m->n_heads_q + 2 * m->n_heads_kv) * dh;
  for (int l = 0; l < m->n_layers; ++l) {
    const tg_layer& L = m->layers[l];
    if (L.gdn != nullptr) {  // a hybrid model's Gated DeltaNet layer
      const tg_status gs = validate_gdn_layer(L.gdn);
      if (gs != TG_OK) return gs;
      TG_CHECK(L.attn_norm && L.w_in && L.w_out, TG_ERR_INVALID_ARG);
      TG_CHECK(m->dtype == TG_BF16, TG_ERR_UNSUPPORTED);
      TG_CHECK(gdn_proj_width(*L.gdn) % 32 == 0, TG_ERR_UNSUPPORTED);
      TG_CHECK(aligned16(L.w_in) && aligned16(L.w_out), TG_ERR_INVALID_ARG);
    } else {
      TG_CHECK(L.attn_norm && L.wqkv && L.wo, TG_ERR_INVALID_ARG);
      TG_CHECK((L.q_norm == nullptr) == (L.k_norm == nullptr), TG_ERR_INVALID_ARG);
    }
    if (L.w_gate_up) TG_CHECK(L.w_down && L.ffn_norm && m->d_ffn > 0, TG_ERR_INVALID_ARG);
    // folded-norm weights: bf16 only, TMA-aligned, beside the weights they fold
    const void* wqkv_g = L.gdn == nullptr ? L.wqkv_g : nullptr;  // unused by a mixer layer
    if (wqkv_g || L.w_gate_up_g) TG_CHECK(m->dtype == TG_BF16, TG_ERR_UNSUPPORTED);
    if (wqkv_g) TG_CHECK(aligned16(wqkv_g), TG_ERR_INVALID_ARG);
    if (L.w_gate_up_g) TG_CHECK(L.w_gate_up && aligned16(L.w_gate_up_g), TG_ERR_INVALID_ARG);
  }
  if (m->score_w1_g) {
    TG_CHECK(m->dtype == TG_BF16, TG_ERR_UNSUPPORTED);
    TG_CHECK(aligned16(m->score_w1_g), TG_ERR_INVALID_ARG);
  }
  bool any_ffn = false;
  for (int l = 0; l < m->n_layers; ++l) any_ffn |= m->layers[l].w_gate_up != nullptr;
  if (m->dtype == TG_BF16) {
    TG_CHECK(dh == 128, TG_ERR_UNSUPPORTED);
    TG_CHECK(d % 32 == 0 && qkv % 32 == 0, TG_ERR_UNSUPPORTED);
    TG_CHECK(m->d_score <= 256, TG_ERR_UNSUPPORTED);
    if (any_ffn) TG_CHECK(m->d_ffn % 128 == 0, TG_ERR_UNSUPPORTED);
  } else {
    TG_CHECK(dh == 64 || dh == 128, TG_ERR_UNSUPPORTED);
  }
  return TG_OK;
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" {

size_t tg_workspace_size(tg_op op, const tg_shape* s) {
  if (s == nullptr) return 0;
  switch (op) {
    case TG_OP_SCORE:
      return ScorePlan(nullptr, s->n, s->d_model, s->d_score, s->dtype).bytes;
    case TG_OP_TOPK_SELECT:
      return select_ws_bytes(s->n);
    case TG_OP_COMPACT:
      return 0;
    case TG_OP_GATED_ATTN:
      return AttnPlan(nullptr, s->k, s->n_heads_q, s->n_heads_kv, s->head_dim, s->dtype, true,
                      s->k).bytes;
    case TG_OP_GATED_ATTN_BWD:
      if (s->dtype == TG_F32)
        return AttnBwdF32Plan(nullptr, s->k, s->n_heads_q, s->n_heads_kv, s->head_dim).bytes;
      return AttnBwdPlan(nullptr, s->k, s->n_heads_q, s->n_heads_kv, s->head_dim).bytes;
    case TG_OP_PREFILL: {
      tg_model m{};
      m.dtype = s->dtype;
      m.d_model = s->d_model;
      m.n_heads_q = s->n_heads_q;
      m.n_heads_kv = s->n_heads_kv;
      m.head_dim = s->head_dim;
      m.d_ffn = s->d_ffn;
      m.d_score = s->d_score;
      return PrefillPlan(nullptr, m, s->n, s->k).bytes;
    }
    case TG_OP_DECODE: {
      tg_model m{};
      m.dtype = s->dtype;
      m.d_model = s->d_model;
      m.n_heads_q = s->n_heads_q;
      m.n_heads_kv = s->n_heads_kv;
      m.head_dim = s->head_dim;
      m.d_ffn = s->d_ffn;
      return DecodePlan(nullptr, m, s->k).bytes;
    }
  }
  return 0;
}

tg_status tg_score(const void* x, int64_t n, int32_t d, int32_t f, const float* norm_w, float eps,
                   const void* w1, const float* b1, const float* w2, const float* b2, tg_dtype dt,
                   float* scores, void* ws, size_t ws_bytes, tg_stream stream) {
  TG_CHECK(dt == TG_BF16 || dt == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(x && norm_w && w1 && w2 && scores && n >= 1 && d >= 1 && f >= 1, TG_ERR_INVALID_ARG);
  if (dt == TG_BF16) {
    TG_CHECK(f <= 256 && d % 8 == 0, TG_ERR_UNSUPPORTED);
    TG_CHECK(aligned16(x) && aligned16(w1), TG_ERR_INVALID_ARG);
  } else {
    TG_CHECK(f <= 1024, TG_ERR_UNSUPPORTED);
  }
  ScorePlan plan(nullptr, n, d, f, dt);
  TG_CHECK(ws != nullptr && ws_bytes >= plan.bytes, TG_ERR_WORKSPACE);
  plan = ScorePlan(ws, n, d, f, dt);
  return cuda_status(run_score(x, n, d, f, norm_w, eps, w1, b1, w2, b2, dt, scores, plan.y,
                               plan.hpre, reinterpret_cast<cudaStream_t>(stream)));
}

tg_status tg_topk_select(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                         int32_t* kept_idx, void* ws, size_t ws_bytes, tg_stream stream) {
  TG_CHECK(scores && kept_idx && n >= 1 && n < (int64_t(1) << 31) - 4096, TG_ERR_INVALID_ARG);
  TG_CHECK(k >= 1 && k <= n, TG_ERR_BUDGET);
  TG_CHECK(ws != nullptr && ws_bytes >= select_ws_bytes(n), TG_ERR_WORKSPACE);
  TG_CHECK((reinterpret_cast<uintptr_t>(ws) & 15u) == 0, TG_ERR_INVALID_ARG);
  return cuda_status(select_topk(scores, protect, n, k, kept_idx, ws,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

tg_status tg_linear(const void* x, const void* w, const void* residual, int64_t m, int32_t n,
                    int32_t k, tg_dtype dt, void* y, tg_stream stream) {
  TG_CHECK(dt == TG_BF16 || dt == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(x && w && y && m >= 1 && n >= 1 && k >= 1, TG_ERR_INVALID_ARG);
  GemmArgs g = gemm_args(x, k, w, k, y, n, m, n, k, residual ? EPI_RESIDUAL : EPI_STORE);
  g.R = residual;
  g.ldr = n;
  if (dt == TG_BF16) {
    TG_CHECK(n % 32 == 0 && k % 8 == 0, TG_ERR_UNSUPPORTED);
    TG_CHECK(gemm_tc_supported(g), TG_ERR_INVALID_ARG);
  }
  return cuda_status(gemm(g, dt, reinterpret_cast<cudaStream_t>(stream)));
}

tg_status tg_fold_norm_weight(const void* w, const float* g, int64_t rows, int64_t cols, void* out,
                              tg_stream stream) {
  TG_CHECK(w && g && out && rows >= 1 && cols >= 1, TG_ERR_INVALID_ARG);
  TG_CHECK(rows <= (int64_t(1) << 40) / cols, TG_ERR_INVALID_ARG);
  const uintptr_t wa = reinterpret_cast<uintptr_t>(w), oa = reinterpret_cast<uintptr_t>(out);
  const uintptr_t nb = static_cast<uintptr_t>(rows * cols * 2);
  TG_CHECK(oa + nb <= wa || wa + nb <= oa, TG_ERR_INVALID_ARG);  // no overlap
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(traced(TG_K_FOLD_NORM, rows, 0.0, 4.0 * rows * cols + 4.0 * cols, st, [&] {
    return launch_fold_norm_weight(w, g, rows, cols, out, st);
  }));
}

tg_status tg_topk_select_noalloc(const float* scores, const uint8_t* protect, int64_t n,
                                 int64_t k, int32_t* kept_idx, tg_stream stream) {
  TG_CHECK(scores && kept_idx && n >= 1, TG_ERR_INVALID_ARG);
  TG_CHECK(n <= select_noalloc_max_n(), TG_ERR_UNSUPPORTED);
  TG_CHECK(k >= 1 && k <= n, TG_ERR_BUDGET);
  const double bytes = 4.0 * n + (protect ? double(n) : 0.0) + 4.0 * k;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return cuda_status(traced(TG_K_SELECT, n, 0.0, bytes, st, [&] {
    return launch_topk_select_noalloc(scores, protect, n, k, kept_idx, st);
  }));
}

tg_status tg_compact(const void* x, const int32_t* pos_in, const float* scores,
                     const int32_t* kept_idx, int64_t n, int64_t k, int32_t d, tg_dtype dt,
                     void* x_out, int32_t* pos_out, float* scores_out, tg_stream stream) {
  TG_CHECK(dt == TG_BF16 || dt == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(x && kept_idx && x_out && pos_out && n >= 1 && d >= 1, TG_ERR_INVALID_ARG);
  TG_CHECK(k >= 1 && k <= n, TG_ERR_BUDGET);
  TG_CHECK(scores_out == nullptr || scores != nullptr, TG_ERR_INVALID_ARG);
  const int64_t row_bytes = int64_t(d) * int64_t(elem_size(dt));
  TG_CHECK(row_bytes % 16 == 0 && row_bytes < (int64_t(1) << 30), TG_ERR_UNSUPPORTED);
  TG_CHECK(aligned16(x) && aligned16(x_out), TG_ERR_INVALID_ARG);
  return cuda_status(compact(x, pos_in, scores, kept_idx, n, k, static_cast<int>(row_bytes), x_out,
                             pos_out, scores_out, nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {
tg_status gated_attn(const void* q, const void* kk, const void* v, const int32_t* pos,
                     const float* s, const float* gain, const float* tau, int64_t k, int32_t hq,
                     int32_t hkv, int32_t dh, float rope_base, tg_dtype dt, void* out, float* lse,
                     float* out_f32, void* ws, size_t ws_bytes, tg_stream stream) {
  TG_CHECK(dt == TG_BF16 || dt == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(q && kk && v && pos && out && k >= 1 && hq >= 1 && hkv >= 1, TG_ERR_INVALID_ARG);
  TG_CHECK(k < (int64_t(1) << 31) - 256, TG_ERR_INVALID_ARG);
  TG_CHECK(hq % hkv == 0 && rope_base > 1.f, TG_ERR_INVALID_ARG);
  if (dt == TG_BF16) {
    TG_CHECK(dh == 128, TG_ERR_UNSUPPORTED);
    TG_CHECK(aligned16(q) && aligned16(kk) && aligned16(v) && aligned16(out), TG_ERR_INVALID_ARG);
  } else {
    TG_CHECK(dh == 64 || dh == 128, TG_ERR_UNSUPPORTED);
  }
  AttnPlan plan(nullptr, k, hq, hkv, dh, dt, true, k);
  TG_CHECK(ws != nullptr && ws_bytes >= plan.bytes, TG_ERR_WORKSPACE);
  plan = AttnPlan(ws, k, hq, hkv, dh, dt, true, k);
  return cuda_status(run_attention(q, int64_t(hq) * dh, kk, int64_t(hkv) * dh, v,
                                   int64_t(hkv) * dh, pos, s, nullptr, gain, tau, nullptr, nullptr,
                                   0.f, k, hq, hkv, dh, rope_base, dt, plan, nullptr, nullptr, out,
                                   reinterpret_cast<cudaStream_t>(stream), lse, out_f32));
}
}  // namespace

extern "C" {

tg_status tg_gated_attn_prefill(const void* q, const void* kk, const void* v, const int32_t* pos,
                                const float* s, const float* gain, const float* tau, int64_t k,
                                int32_t hq, int32_t hkv, int32_t dh, float rope_base,
                                tg_dtype dt, void* out, void* ws, size_t ws_bytes,
                                tg_stream stream) {
  return gated_attn(q, kk, v, pos, s, gain, tau, k, hq, hkv, dh, rope_base, dt, out, nullptr,
                    nullptr, ws, ws_bytes, stream);
}

tg_status tg_gated_attn_forward(const void* q, const void* kk, const void* v, const int32_t* pos,
                                const float* s, const float* gain, const float* tau, int64_t k,
                                int32_t hq, int32_t hkv, int32_t dh, float rope_base,
                                tg_dtype dt, void* out, float* lse, float* out_f32, void* ws,
                                size_t ws_bytes, tg_stream stream) {
  TG_CHECK(dt == TG_BF16 || dt == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(lse != nullptr && aligned16(out_f32), TG_ERR_INVALID_ARG);
  TG_CHECK(dt == TG_BF16 || out_f32 == nullptr, TG_ERR_INVALID_ARG);  // fp32: out is the fp32 output
  return gated_attn(q, kk, v, pos, s, gain, tau, k, hq, hkv, dh, rope_base, dt, out, lse, out_f32,
                    ws, ws_bytes, stream);
}

tg_status tg_gated_attn_backward(const void* q, const void* kk, const void* v, const int32_t* pos,
                                 const float* s, const float* gain, const float* tau, int64_t k,
                                 int32_t hq, int32_t hkv, int32_t dh, float rope_base, tg_dtype dt,
                                 const void* out, const float* out_f32, const float* lse,
                                 const void* dout, void* dq,
                                 void* dk, void* dv, float* ds, float* dgain, float* dtau,
                                 void* ws, size_t ws_bytes, tg_stream stream) {
  TG_CHECK(dt == TG_BF16 || dt == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(dt == TG_BF16 ? dh == 128 : (dh == 64 || dh == 128), TG_ERR_UNSUPPORTED);
  TG_CHECK(q && kk && v && pos && out && lse && dout && dq && dk && dv, TG_ERR_INVALID_ARG);
  if (dt == TG_F32) {
    TG_CHECK(k >= 1 && hq >= 1 && hkv >= 1 && k < (int64_t(1) << 31) - 256, TG_ERR_INVALID_ARG);
    TG_CHECK(hq % hkv == 0 && rope_base > 1.f, TG_ERR_INVALID_ARG);
    TG_CHECK(ds == nullptr || s != nullptr, TG_ERR_INVALID_ARG);
    TG_CHECK(out_f32 == nullptr && aligned16(ws), TG_ERR_INVALID_ARG);
    AttnBwdF32Plan fp(nullptr, k, hq, hkv, dh);
    TG_CHECK(ws != nullptr && ws_bytes >= fp.bytes, TG_ERR_WORKSPACE);
    fp = AttnBwdF32Plan(ws, k, hq, hkv, dh);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    RopePrepArgs r{};
    r.q_src = q; r.k_src = kk; r.v_src = v;
    r.q_stride = int64_t(hq) * dh; r.k_stride = int64_t(hkv) * dh; r.v_stride = int64_t(hkv) * dh;
    r.pos = pos;
    r.T = k; r.hq = hq; r.hkv = hkv; r.dh = dh; r.rope_base = rope_base;
    r.bf16 = false;
    r.q_out = fp.q_rot;
    r.k_out = fp.k_rot;
    r.s = s;
    r.lsig_out = fp.lsig;
    const double rows = double(k);
    TG_TRY(traced(TG_K_ROPE_PREP, k, 0.0, rows * (hq + hkv) * dh * 8.0, st,
                  [&] { return launch_rope_prep(r, st); }));
    TG_TRY(traced(TG_K_ROPE_TABLE, k, 0.0, 8.0 * (dh / 2) * rows, st,
                  [&] { return launch_rope_table(pos, k, dh, rope_base, fp.cs, st); }));
    AttnBwdF32Args b{};
    b.q_rot = fp.q_rot; b.k_rot = fp.k_rot;
    b.v = static_cast<const float*>(v);
    b.out = static_cast<const float*>(out);
    b.dout = static_cast<const float*>(dout);
    b.lse = lse;
    b.lsig = s ? fp.lsig : nullptr;
    b.gain = gain; b.tau = tau; b.cs = fp.cs;
    b.T = k; b.t_pad = k; b.hq = hq; b.hkv = hkv; b.dh = dh;
    b.colsum = s ? fp.colsum : nullptr;
    b.qdq = fp.qdq;
    b.dq = static_cast<float*>(dq); b.dk = static_cast<float*>(dk); b.dv = static_cast<float*>(dv);
    const double prod = 2.0 * dh * hq * rows * (rows + 1) / 2.0;
    TG_TRY(traced(TG_K_ATTENTION_F32, k, 4.0 * prod, 0.0, st,
                  [&] { return launch_attn_bwd_f32(b, st); }));
    if (ds || dgain || dtau) {
      AttnBwdArgs f{};
      f.s = s; f.bias = fp.lsig; f.gain = gain; f.tau = tau;
      f.colsum = fp.colsum; f.qdq = fp.qdq; f.qdq_per_head = k;
      f.T = k; f.t_pad = k; f.hq = hq; f.hkv = hkv;
      f.ds = ds; f.dgain = dgain; f.dtau = dtau;
      TG_TRY(traced(TG_K_ATTN_BWD_FINAL, k, 0.0, rows * hq * 4.0, st,
                    [&] { return launch_attn_bwd(f, st, 3); }));
    }
    return TG_OK;
  }
  TG_CHECK(k >= 1 && hq >= 1 && hkv >= 1 && k < (int64_t(1) << 31) - 256, TG_ERR_INVALID_ARG);
  TG_CHECK(hq % hkv == 0 && rope_base > 1.f, TG_ERR_INVALID_ARG);
  TG_CHECK(ds == nullptr || s != nullptr, TG_ERR_INVALID_ARG);
  TG_CHECK(aligned16(q) && aligned16(kk) && aligned16(v) && aligned16(out) && aligned16(dout) &&
               aligned16(dq) && aligned16(dk) && aligned16(dv) && aligned16(ws) &&
               aligned16(out_f32),
           TG_ERR_INVALID_ARG);
  AttnBwdPlan plan(nullptr, k, hq, hkv, dh);
  TG_CHECK(ws != nullptr && ws_bytes >= plan.bytes, TG_ERR_WORKSPACE);
  plan = AttnBwdPlan(ws, k, hq, hkv, dh);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const double rows = double(k);
  AttnBwdArgs a{};
  a.q = q; a.k = kk; a.pos = pos; a.rope_base = rope_base;
  a.v = v; a.out = out; a.dout = dout; a.out_f32 = out_f32;
  a.lse = lse; a.s = s; a.gain = gain; a.tau = tau;
  a.T = k; a.t_pad = plan.t_pad; a.hq = hq; a.hkv = hkv;
  a.q_rot = plan.q_rot; a.k_rot = plan.k_rot; a.cs = plan.cs;
  a.qT = plan.qT; a.doT = plan.doT;
  a.lse2 = plan.lse2; a.dd = plan.dd; a.colsum = plan.colsum; a.qdq = plan.qdq;
  a.bias = plan.bias;
  a.dq = dq; a.dk = dk; a.dv = dv; a.ds = ds; a.dgain = dgain; a.dtau = dtau;
  // one [T x T x dh] causal product of all query heads (half of the forward's FLOPs)
  const double prod = 2.0 * dh * hq * rows * (rows + 1) / 2.0;
  // reads q, k, dO and o; writes q, k rotated and q, dO transposed
  const double prep_bytes = rows * dh * 2.0 * (2.0 * (hq + hkv) + 3.0 * hq) +
                            rows * hq * dh * (out_f32 ? 4.0 : 2.0);
  TG_TRY(traced(TG_K_ATTN_BWD_PREP, k, 0.0, prep_bytes, st,
                [&] { return launch_attn_bwd(a, st, 0); }));
  TG_TRY(traced(TG_K_ATTN_BWD_DKDV, k, 4.0 * prod, 0.0, st,
                [&] { return launch_attn_bwd(a, st, 1); }));
  TG_TRY(traced(TG_K_ATTN_BWD_DQ, k, 3.0 * prod, 0.0, st,
                [&] { return launch_attn_bwd(a, st, 2); }));
  if (ds || dgain || dtau)
    TG_TRY(traced(TG_K_ATTN_BWD_FINAL, k, 0.0, rows * hq * 4.0, st,
                  [&] { return launch_attn_bwd(a, st, 3); }));
  return TG_OK;
}

}  // extern "C"

namespace {

struct LayerTag {  // annotates traced launches with their decoder layer
  explicit LayerTag(int l) { t_trace.layer = l; }
  ~LayerTag() { t_trace.layer = -1; }
};

Dims model_dims(const tg_model& m) {
  return Dims{m.d_model, m.n_heads_q, m.n_heads_kv, m.head_dim, m.d_ffn,
              (m.n_heads_q + 2 * m.n_heads_kv) * m.head_dim};
}

// Rows per chunk of a prefill whose input arrives from host memory (small
// chunks expose less of the first copy; every later copy hides behind the
// growing attention work of the chunk before it).
constexpr int64_t kHostChunkRows = 4096;

// Whether tg_prefill_host can overlap the input copy with layer 0: the
// paired-head tensor-core attention, layer 0 an attention layer at or below
// the gate, and n above the 8192 rows up to which the one-shot attention may
// split query tiles (the chunks run whole tiles, so the results stay equal).
bool host_chunks_apply(const tg_model& m, const Dims& D, int64_t n, int gate_layer) {
  return m.dtype == TG_BF16 && D.dh == 128 && (D.hq / D.hkv) % 2 == 0 && gate_layer >= 0 &&
         m.layers[0].gdn == nullptr && n > 8192;
}

// Layer 0's attention sub-layer while its input rows arrive from host
// memory: the rows are copied into P.h in chunks on `copy_st`; as each chunk
// lands, its RMSNorm, its fused QKV projection and the attention of its
// query rows (over every key up to the chunk's end) run on `st`, so that the
// copies of the later chunks overlap the work of the earlier ones. Then the
// output projection over all n rows. Each query tile and each GEMM tile is
// computed exactly as by the one-shot launches (chunk bounds are multiples of
// the 256-row GEMM tile).
tg_status attn_layer0_from_host(const tg_model& m, const Dims& D, const PrefillPlan& P,
                                const void* x_host, int64_t n, const tg_kv* kv,
                                cudaStream_t st, cudaStream_t copy_st) {
  const tg_layer& lw = m.layers[0];
  const size_t e = elem_size(m.dtype), row = size_t(D.d) * e;
  const int64_t n_chunks = (n + kHostChunkRows - 1) / kHostChunkRows;
  std::vector<cudaEvent_t> landed(static_cast<size_t>(n_chunks), nullptr);
  cudaEvent_t start = nullptr;
  auto release = [&] {
    for (cudaEvent_t ev : landed)
      if (ev) cudaEventDestroy(ev);
    if (start) cudaEventDestroy(start);
  };
  cudaError_t err = cudaEventCreateWithFlags(&start, cudaEventDisableTiming);
  for (int64_t c = 0; c < n_chunks && err == cudaSuccess; ++c)
    err = cudaEventCreateWithFlags(&landed[size_t(c)], cudaEventDisableTiming);
  // the copies start after the work already queued on st (it may still read P.h)
  if (err == cudaSuccess) err = cudaEventRecord(start, st);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(copy_st, start, 0);
  for (int64_t c = 0; c < n_chunks && err == cudaSuccess; ++c) {
    const int64_t r0 = c * kHostChunkRows, rc = std::min(kHostChunkRows, n - r0);
    err = traced(TG_K_COPY, rc, 0.0, double(rc) * row, copy_st, [&] {
      return cudaMemcpyAsync(static_cast<char*>(P.h) + size_t(r0) * row,
                             static_cast<const char*>(x_host) + size_t(r0) * row,
                             size_t(rc) * row, cudaMemcpyHostToDevice, copy_st);
    });
    if (err == cudaSuccess) err = cudaEventRecord(landed[size_t(c)], copy_st);
  }
  void* k_dst = (kv && kv->k) ? kv->k : P.attn.k_rot;
  for (int64_t c = 0; c < n_chunks && err == cudaSuccess; ++c) {
    const int64_t r0 = c * kHostChunkRows, r1 = std::min(n, r0 + kHostChunkRows), rc = r1 - r0;
    err = cudaStreamWaitEvent(st, landed[size_t(c)], 0);
    if (err != cudaSuccess) break;
    char* yc = static_cast<char*>(P.y) + size_t(r0) * row;
    err = rmsnorm(static_cast<char*>(P.h) + size_t(r0) * row, lw.attn_norm, m.norm_eps, rc, D.d,
                  m.dtype, yc, st);
    if (err != cudaSuccess) break;
    GemmArgs gq = gemm_args(yc, D.d, lw.wqkv, D.d, nullptr, 0, rc, D.qkv, D.d, EPI_QKV);
    gq.hq = D.hq; gq.hkv = D.hkv; gq.q_norm = lw.q_norm; gq.k_norm = lw.k_norm;
    gq.eps = m.norm_eps;
    gq.rope_cs = P.cs_n + r0;
    gq.rope_ld = n;
    gq.q_out = static_cast<char*>(P.attn.q_rot) + size_t(r0) * D.hq * D.dh * e;
    gq.k_out = static_cast<char*>(k_dst) + size_t(r0) * D.hkv * D.dh * e;
    gq.vT_out = static_cast<__nv_bfloat16*>(P.attn.vT) + r0;
    gq.t_pad = P.attn.t_pad;
    gq.v_out = (kv && kv->v) ? static_cast<char*>(kv->v) + size_t(r0) * D.hkv * D.dh * e : nullptr;
    if (!gemm_tc_supported(gq)) {
      err = cudaErrorInvalidValue;
      break;
    }
    err = gemm(gq, m.dtype, st);
    if (err != cudaSuccess) break;
    // whole query tiles, as the one-shot launch over n > 8192 rows runs them
    err = attn_core(P.attn, k_dst, nullptr, 0, nullptr, nullptr, nullptr, nullptr, r1, D.hq,
                    D.hkv, D.dh, m.dtype, P.attn_o, st, nullptr, nullptr, true, r0, true);
  }
  release();  // events may still be pending; their resources go when they complete
  if (err != cudaSuccess) return cuda_status(err);
  GemmArgs g = gemm_args(P.attn_o, int64_t(D.hq) * D.dh, lw.wo, int64_t(D.hq) * D.dh, P.h, D.d, n,
                         D.d, D.hq * D.dh, EPI_RESIDUAL);
  g.R = P.h;
  g.ldr = D.d;
  ss_produce(g, P, P.h, 0);
  TG_TRY(gemm(g, m.dtype, st));
  ss_mark(P, P.h, n);
  return TG_OK;
}

// Stage 1 of the gated forward: the layers below the gate and the gate
// layer's attention over all n rows (in P.h), then the scores of every row.
// x_in_h: the input rows are already in P.h. With copy_st, x is a host
// pointer and layer 0's attention overlaps its copy (attn_layer0_from_host).
tg_status prefill_below_gate(const tg_model& m, const Dims& D, const PrefillPlan& P, const void* x,
                             int64_t n, int gate_layer, const tg_kv* kv,
                             const tg_layer_taps* taps, float* sc, cudaStream_t st,
                             bool x_in_h = false, cudaStream_t copy_st = nullptr) {
  const size_t e = elem_size(m.dtype);
  const bool x_host = copy_st != nullptr;
  // Device input and an attention layer 0 below or at the gate: layer 0
  // reads x in place and writes its residual output into P.h, so x is never
  // copied. (Scores of the input itself, gate_layer < 0, need x in P.h.)
  const bool x_direct = !x_in_h && !x_host && gate_layer >= 0 && m.layers[0].gdn == nullptr;
  if (!x_in_h && !x_host && !x_direct) TG_TRY(copy_rows(P.h, x, size_t(n) * D.d * e, n, st));
  P.ss_rows_h = -1;  // the input rows carry no row sums
  // every attention launch of the call then finds its split counters zero
  TG_TRY(attn_split_clear(P.attn.split, P.attn.split_bytes, D.hq, st));
  const bool tables = m.dtype == TG_BF16 && D.dh == 128;
  const double cs_bytes = 8.0 * (D.dh / 2);
  if (tables && gate_layer >= 0)
    TG_TRY(traced(TG_K_ROPE_TABLE, n, 0.0, cs_bytes * n, st, [&] {
      return launch_rope_table(nullptr, n, D.dh, m.rope_base, P.cs_n, st);
    }));
  auto mixer = [&](int l) -> tg_status {
    LayerTag tag(l);
    if (l == 0 && x_host) return attn_layer0_from_host(m, D, P, x, n, kv ? &kv[0] : nullptr, st,
                                                       copy_st);
    if (l == 0 && x_direct)
      return cuda_status(attention_sublayer(m, m.layers[0], D, P, P.h, n, nullptr, P.cs_n, nullptr,
                                            nullptr, nullptr, nullptr, kv ? &kv[0] : nullptr, st,
                                            nullptr, taps ? &taps[0] : nullptr, x));
    return cuda_status(mixer_sublayer(m, m.layers[l], D, P, P.h, n, nullptr, P.cs_n, nullptr,
                                      nullptr, nullptr, nullptr, kv ? &kv[l] : nullptr, st,
                                      nullptr, taps ? &taps[l] : nullptr));
  };
  for (int l = 0; l < gate_layer; ++l) {
    const tg_status ms = mixer(l);
    if (ms != TG_OK) return ms;
    LayerTag tag(l);
    TG_TRY(ffn_sublayer(m, m.layers[l], D, P, P.h, n, st));
    if (taps && taps[l].hidden)
      TG_TRY(copy_rows(taps[l].hidden, P.h, size_t(n) * D.d * e, n, st));
  }
  if (gate_layer >= 0) {
    const tg_status ms = mixer(gate_layer);
    if (ms != TG_OK) return ms;
  }
  // score the post-attention residual
  TG_TRY(run_score(P.h, n, D.d, m.d_score, m.score_norm, m.norm_eps, m.score_w1, m.score_b1,
                   m.score_w2, m.score_b2, m.dtype, sc, P.y, P.hpre, st, &P, m.score_w1_g));
  return TG_OK;
}

// Stages 2-3 for one budget k: select, compact, the gate layer's FFN and
// the layers above over the k kept rows (in P.hk; P.h is only read), final
// norm into out.
tg_status prefill_above_gate(const tg_model& m, const Dims& D, const PrefillPlan& P,
                             const uint8_t* protect, int64_t n, int64_t k, int gate_layer,
                             const float* sc, void* out, int32_t* kept_idx, const tg_kv* kv,
                             const tg_layer_taps* taps, cudaStream_t st) {
  const size_t e = elem_size(m.dtype);
  const bool tables = m.dtype == TG_BF16 && D.dh == 128;
  const double cs_bytes = 8.0 * (D.dh / 2);
  TG_TRY(select_topk(sc, protect, n, k, kept_idx, P.sel_ws, st));
  // the kept rows take their row sums along when h's are current
  SsGather sg;
  const bool carry = ss_ready(P, P.h, n) && P.ss_parts <= 32;
  if (carry) sg = SsGather{P.ss, P.ss_ld, P.ss_k, P.ss_ld_k, P.ss_parts};
  TG_TRY(compact(P.h, nullptr, sc, kept_idx, n, k, static_cast<int>(D.d * e), P.hk, P.pos_k, P.s_k,
                 P.lsig_k, st, sg));
  P.ss_rows_hk = carry ? k : -1;
  if (tables) {
    TG_TRY(traced(TG_K_ROPE_TABLE, k, 0.0, cs_bytes * k + 4.0 * k, st, [&] {
      return launch_rope_table(P.pos_k, k, D.dh, m.rope_base, P.cs_k, st);
    }));
    // gate-bias rows of the kept tokens, shared by every gated layer
    TG_TRY(traced(TG_K_ROPE_TABLE, k, 0.0, 36.0 * k, st,
                  [&] { return launch_bias_aug(P.lsig_k, k, P.kaug_k, st); }));
  }
  if (gate_layer >= 0) {
    LayerTag tag(gate_layer);
    TG_TRY(ffn_sublayer(m, m.layers[gate_layer], D, P, P.hk, k, st));
    if (taps && taps[gate_layer].hidden)
      TG_TRY(copy_rows(taps[gate_layer].hidden, P.hk, size_t(k) * D.d * e, k, st));
  }
  for (int l = gate_layer + 1; l < m.n_layers; ++l) {
    LayerTag tag(l);
    const tg_layer& L = m.layers[l];
    TG_TRY(mixer_sublayer(m, L, D, P, P.hk, k, P.pos_k, P.cs_k, P.lsig_k, P.kaug_k, L.gain,
                              L.tau, kv ? &kv[l] : nullptr, st, nullptr,
                              taps ? &taps[l] : nullptr));
    TG_TRY(ffn_sublayer(m, L, D, P, P.hk, k, st));
    if (taps && taps[l].hidden)
      TG_TRY(copy_rows(taps[l].hidden, P.hk, size_t(k) * D.d * e, k, st));
  }
  if (m.final_norm)
    TG_TRY(rmsnorm(P.hk, m.final_norm, m.norm_eps, k, D.d, m.dtype, out, st));
  else
    TG_TRY(copy_rows(out, P.hk, size_t(k) * D.d * e, k, st));
  return TG_OK;
}

// Workspace of a batch of packed requests: the prefill plan over the padded
// row counts, plus the positions of the padded all-token rows.
struct BatchPlan {
  PrefillPlan P;
  int32_t* pos_n = nullptr;
  size_t bytes = 0;
  BatchPlan(void* ws, const tg_model& m, int64_t n_pad, int64_t k_pad)
      : P(ws, m, n_pad, k_pad) {
    Arena a(ws);
    a.used = P.bytes;
    pos_n = static_cast<int32_t*>(a.carve(size_t(n_pad) * 4));
    bytes = a.used;
  }
};

constexpr int64_t kSegAlign = 128;

// Validates a batch and lays it out: request b's rows at segs_n.off[b], its
// kept rows at segs_k.off[b] (each padded to 128 rows).
// (validate = false: sizes only, for the workspace query.)
tg_status batch_layout(const tg_model* model, const int64_t* cu_n, const int64_t* ks,
                       int32_t batch, int32_t gate_layer, bool validate, SegRows* segs_n,
                       SegRows* segs_k, int64_t* n_pad, int64_t* k_pad) {
  TG_CHECK(model && cu_n && ks, TG_ERR_INVALID_ARG);
  TG_CHECK(batch >= 1 && batch <= TG_MAX_BATCH && batch <= kMaxSegs, TG_ERR_INVALID_ARG);
  TG_CHECK(cu_n[0] == 0, TG_ERR_INVALID_ARG);
  TG_CHECK(model->dtype == TG_BF16 || model->dtype == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(model->dtype == TG_BF16 && model->head_dim == 128, TG_ERR_UNSUPPORTED);
  segs_n->count = segs_k->count = batch;
  int64_t on = 0, ok = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = cu_n[b + 1] - cu_n[b];
    TG_CHECK(n >= 1, TG_ERR_INVALID_ARG);
    TG_CHECK(ks[b] >= 1 && ks[b] <= n, TG_ERR_BUDGET);
    if (validate) {
      const tg_status vs = validate_model(model, n, ks[b], gate_layer);
      if (vs != TG_OK) return vs;
    }
    segs_n->off[b] = on;
    segs_n->len[b] = n;
    segs_k->off[b] = ok;
    segs_k->len[b] = ks[b];
    on += static_cast<int64_t>(align_up(static_cast<size_t>(n), kSegAlign));
    ok += static_cast<int64_t>(align_up(static_cast<size_t>(ks[b]), kSegAlign));
  }
  TG_CHECK(on < (int64_t(1) << 31) - 4096, TG_ERR_INVALID_ARG);
  *n_pad = on;
  *k_pad = ok;
  return TG_OK;
}

}  // namespace

extern "C" {

size_t tg_prefill_workspace_size(const tg_model* model, int64_t n, int64_t k) {
  if (model == nullptr || model->layers == nullptr || n < 1 || k < 1 || k > n) return 0;
  return PrefillPlan(nullptr, *model, n, k).bytes;
}

tg_status tg_prefill(const tg_model* model, const void* x, const uint8_t* protect, int64_t n,
                     int64_t k, int32_t gate_layer, void* out, int32_t* kept_idx, float* scores,
                     const tg_kv* kv, const tg_layer_taps* taps, void* ws, size_t ws_bytes,
                     tg_stream stream) {
  const tg_status vs = validate_model(model, n, k, gate_layer);
  if (vs != TG_OK) return vs;
  TG_CHECK(x && out && kept_idx, TG_ERR_INVALID_ARG);
  const tg_model& m = *model;
  if (m.dtype == TG_BF16) TG_CHECK(aligned16(x) && aligned16(out), TG_ERR_INVALID_ARG);
  if (m.dtype == TG_BF16 && kv != nullptr)  // written by the QKV GEMM's epilogue
    for (int l = 0; l < m.n_layers; ++l)
      TG_CHECK(aligned16(kv[l].k) && aligned16(kv[l].v), TG_ERR_INVALID_ARG);
  PrefillPlan P(nullptr, m, n, k);
  TG_CHECK(ws != nullptr && ws_bytes >= P.bytes, TG_ERR_WORKSPACE);
  P = PrefillPlan(ws, m, n, k);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Dims D = model_dims(m);
  float* sc = scores ? scores : P.scores;
  const tg_status s1 = prefill_below_gate(m, D, P, x, n, gate_layer, kv, taps, sc, st);
  if (s1 != TG_OK) return s1;
  return prefill_above_gate(m, D, P, protect, n, k, gate_layer, sc, out, kept_idx, kv, taps, st);
}

// A non-blocking stream per device for the host-input copies of
// tg_prefill_host (created on first use, kept for the process).
static cudaStream_t host_copy_stream(cudaError_t* err) {
  static std::mutex mu;
  static std::map<int, cudaStream_t> streams;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  auto it = streams.find(dev);
  if (it != streams.end()) return it->second;
  cudaStream_t s = nullptr;
  *err = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (*err != cudaSuccess) return nullptr;
  streams[dev] = s;
  return s;
}

tg_status tg_prefill_host(const tg_model* model, const void* x_host, const uint8_t* protect,
                          int64_t n, int64_t k, int32_t gate_layer, void* out, int32_t* kept_idx,
                          float* scores, const tg_kv* kv, void* ws, size_t ws_bytes,
                          tg_stream stream) {
  const tg_status vs = validate_model(model, n, k, gate_layer);
  if (vs != TG_OK) return vs;
  TG_CHECK(x_host && out && kept_idx, TG_ERR_INVALID_ARG);
  const tg_model& m = *model;
  if (m.dtype == TG_BF16) TG_CHECK(aligned16(out), TG_ERR_INVALID_ARG);
  if (m.dtype == TG_BF16 && kv != nullptr)
    for (int l = 0; l < m.n_layers; ++l)
      TG_CHECK(aligned16(kv[l].k) && aligned16(kv[l].v), TG_ERR_INVALID_ARG);
  PrefillPlan P(nullptr, m, n, k);
  TG_CHECK(ws != nullptr && ws_bytes >= P.bytes, TG_ERR_WORKSPACE);
  P = PrefillPlan(ws, m, n, k);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Dims D = model_dims(m);
  float* sc = scores ? scores : P.scores;
  tg_status s1 = TG_OK;
  if (host_chunks_apply(m, D, n, gate_layer)) {
    cudaError_t e = cudaSuccess;
    cudaStream_t cs = host_copy_stream(&e);
    if (e != cudaSuccess) return cuda_status(e);
    s1 = prefill_below_gate(m, D, P, x_host, n, gate_layer, kv, nullptr, sc, st, false, cs);
  } else {
    const size_t bytes = size_t(n) * D.d * elem_size(m.dtype);
    TG_TRY(traced(TG_K_COPY, n, 0.0, double(bytes), st, [&] {
      return cudaMemcpyAsync(P.h, x_host, bytes, cudaMemcpyHostToDevice, st);
    }));
    s1 = prefill_below_gate(m, D, P, P.h, n, gate_layer, kv, nullptr, sc, st, true);
  }
  if (s1 != TG_OK) return s1;
  return prefill_above_gate(m, D, P, protect, n, k, gate_layer, sc, out, kept_idx, kv, nullptr, st);
}

tg_status tg_prefill_multi(const tg_model* model, const void* x, const uint8_t* protect,
                           int64_t n, const int64_t* ks, int32_t n_budgets, int32_t gate_layer,
                           void* const* outs, int32_t* const* kept_idx, float* scores, void* ws,
                           size_t ws_bytes, tg_stream stream) {
  TG_CHECK(ks != nullptr && outs != nullptr && kept_idx != nullptr, TG_ERR_INVALID_ARG);
  TG_CHECK(n_budgets >= 1 && n_budgets <= TG_MAX_BUDGETS, TG_ERR_INVALID_ARG);
  int64_t k_max = 0;
  for (int b = 0; b < n_budgets; ++b) {
    const tg_status vs = validate_model(model, n, ks[b], gate_layer);
    if (vs != TG_OK) return vs;
    TG_CHECK(outs[b] && kept_idx[b], TG_ERR_INVALID_ARG);
    if (model->dtype == TG_BF16) TG_CHECK(aligned16(outs[b]), TG_ERR_INVALID_ARG);
    k_max = ks[b] > k_max ? ks[b] : k_max;
  }
  TG_CHECK(x != nullptr, TG_ERR_INVALID_ARG);
  const tg_model& m = *model;
  if (m.dtype == TG_BF16) TG_CHECK(aligned16(x), TG_ERR_INVALID_ARG);
  PrefillPlan P(nullptr, m, n, k_max);
  TG_CHECK(ws != nullptr && ws_bytes >= P.bytes, TG_ERR_WORKSPACE);
  P = PrefillPlan(ws, m, n, k_max);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Dims D = model_dims(m);
  float* sc = scores ? scores : P.scores;
  const tg_status s1 = prefill_below_gate(m, D, P, x, n, gate_layer, nullptr, nullptr, sc, st);
  if (s1 != TG_OK) return s1;
  for (int b = 0; b < n_budgets; ++b) {
    const tg_status sb = prefill_above_gate(m, D, P, protect, n, ks[b], gate_layer, sc, outs[b],
                                            kept_idx[b], nullptr, nullptr, st);
    if (sb != TG_OK) return sb;
  }
  return TG_OK;
}

size_t tg_prefill_batch_workspace_size(const tg_model* model, const int64_t* cu_n,
                                       const int64_t* ks, int32_t batch) {
  SegRows sn{}, sk{};
  int64_t n_pad = 0, k_pad = 0;
  if (batch_layout(model, cu_n, ks, batch, 0, false, &sn, &sk, &n_pad, &k_pad) != TG_OK)
    return 0;
  return BatchPlan(nullptr, *model, n_pad, k_pad).bytes;
}

tg_status tg_prefill_batch(const tg_model* model, const void* x, const uint8_t* protect,
                           const int64_t* cu_n, const int64_t* ks, int32_t batch,
                           int32_t gate_layer, void* out, int32_t* kept_idx, float* scores,
                           void* ws, size_t ws_bytes, tg_stream stream) {
  SegRows sn{}, sk{};
  int64_t n_pad = 0, k_pad = 0;
  const tg_status vs =
      batch_layout(model, cu_n, ks, batch, gate_layer, true, &sn, &sk, &n_pad, &k_pad);
  if (vs != TG_OK) return vs;
  TG_CHECK(x && out && kept_idx, TG_ERR_INVALID_ARG);
  TG_CHECK(aligned16(x) && aligned16(out), TG_ERR_INVALID_ARG);
  const tg_model& m = *model;
  BatchPlan B(nullptr, m, n_pad, k_pad);
  TG_CHECK(ws != nullptr && ws_bytes >= B.bytes, TG_ERR_WORKSPACE);
  B = BatchPlan(ws, m, n_pad, k_pad);
  const PrefillPlan& P = B.P;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Dims D = model_dims(m);
  const size_t e = elem_size(m.dtype);
  const size_t row = size_t(D.d) * e;
  char* h = static_cast<char*>(P.h);
  char* hk = static_cast<char*>(P.hk);
  TG_TRY(attn_split_clear(P.attn.split, P.attn.split_bytes, D.hq, st));
  // packed rows in, padding rows zero
  for (int b = 0; b < batch; ++b) {
    const int64_t n = sn.len[b], pad = static_cast<int64_t>(align_up(size_t(n), kSegAlign)) - n;
    TG_TRY(copy_rows(h + sn.off[b] * row, static_cast<const char*>(x) + cu_n[b] * row, n * row, n,
                     st));
    if (pad > 0) TG_TRY(cudaMemsetAsync(h + (sn.off[b] + n) * row, 0, pad * row, st));
  }
  TG_TRY(launch_segment_positions(sn, n_pad, B.pos_n, st));
  const double cs_bytes = 8.0 * (D.dh / 2);
  TG_TRY(traced(TG_K_ROPE_TABLE, n_pad, 0.0, cs_bytes * n_pad, st, [&] {
    return launch_rope_table(B.pos_n, n_pad, D.dh, m.rope_base, P.cs_n, st);
  }));
  // below the gate: projections over every request's rows, attention per request
  for (int l = 0; l < gate_layer; ++l) {
    LayerTag tag(l);
    TG_TRY(mixer_sublayer(m, m.layers[l], D, P, P.h, n_pad, nullptr, P.cs_n, nullptr, nullptr,
                              nullptr, nullptr, nullptr, st, &sn));
    TG_TRY(ffn_sublayer(m, m.layers[l], D, P, P.h, n_pad, st));
  }
  if (gate_layer >= 0) {
    LayerTag tag(gate_layer);
    TG_TRY(mixer_sublayer(m, m.layers[gate_layer], D, P, P.h, n_pad, nullptr, P.cs_n, nullptr,
                              nullptr, nullptr, nullptr, nullptr, st, &sn));
  }
  float* sc = P.scores;
  TG_TRY(run_score(P.h, n_pad, D.d, m.d_score, m.score_norm, m.norm_eps, m.score_w1, m.score_b1,
                   m.score_w2, m.score_b2, m.dtype, sc, P.y, P.hpre, st, &P, m.score_w1_g));
  // per request: select, compact into its padded block of kept rows (with
  // the rows' sums of squares when h's are current; padding rows get 0)
  TG_TRY(cudaMemsetAsync(P.pos_k, 0, size_t(k_pad) * 4, st));
  const bool carry = ss_ready(P, P.h, n_pad) && P.ss_parts <= 32;
  if (carry) TG_TRY(cudaMemsetAsync(P.ss_k, 0, size_t(P.ss_parts) * P.ss_ld_k * 4, st));
  int64_t ck = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = sn.len[b], k = sk.len[b];
    if (scores) TG_TRY(cudaMemcpyAsync(scores + cu_n[b], sc + sn.off[b], size_t(n) * 4,
                                       cudaMemcpyDeviceToDevice, st));
    TG_TRY(select_topk(sc + sn.off[b], protect ? protect + cu_n[b] : nullptr, n, k, kept_idx + ck,
                       P.sel_ws, st));
    SsGather sg;
    if (carry)
      sg = SsGather{P.ss + sn.off[b], P.ss_ld, P.ss_k + sk.off[b], P.ss_ld_k, P.ss_parts};
    TG_TRY(compact(h + sn.off[b] * row, nullptr, sc + sn.off[b], kept_idx + ck, n, k,
                   static_cast<int>(row), hk + sk.off[b] * row, P.pos_k + sk.off[b],
                   P.s_k + sk.off[b], P.lsig_k + sk.off[b], st, sg));
    const int64_t pad = static_cast<int64_t>(align_up(size_t(k), kSegAlign)) - k;
    if (pad > 0) TG_TRY(cudaMemsetAsync(hk + (sk.off[b] + k) * row, 0, pad * row, st));
    ck += k;
  }
  P.ss_rows_hk = carry ? k_pad : -1;
  TG_TRY(traced(TG_K_ROPE_TABLE, k_pad, 0.0, cs_bytes * k_pad + 4.0 * k_pad, st, [&] {
    return launch_rope_table(P.pos_k, k_pad, D.dh, m.rope_base, P.cs_k, st);
  }));
  TG_TRY(traced(TG_K_ROPE_TABLE, k_pad, 0.0, 36.0 * k_pad, st,
                [&] { return launch_bias_aug(P.lsig_k, k_pad, P.kaug_k, st); }));
  // the gate layer's FFN and the layers above over every request's kept rows
  if (gate_layer >= 0) {
    LayerTag tag(gate_layer);
    TG_TRY(ffn_sublayer(m, m.layers[gate_layer], D, P, P.hk, k_pad, st));
  }
  for (int l = gate_layer + 1; l < m.n_layers; ++l) {
    LayerTag tag(l);
    const tg_layer& L = m.layers[l];
    TG_TRY(mixer_sublayer(m, L, D, P, P.hk, k_pad, P.pos_k, P.cs_k, P.lsig_k, P.kaug_k, L.gain,
                              L.tau, nullptr, st, &sk));
    TG_TRY(ffn_sublayer(m, L, D, P, P.hk, k_pad, st));
  }
  ck = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t k = sk.len[b];
    char* ob = static_cast<char*>(out) + ck * row;
    if (m.final_norm)
      TG_TRY(rmsnorm(hk + sk.off[b] * row, m.final_norm, m.norm_eps, k, D.d, m.dtype, ob, st));
    else
      TG_TRY(copy_rows(ob, hk + sk.off[b] * row, k * row, k, st));
    ck += k;
  }
  return TG_OK;
}

const char* tg_status_string(tg_status s) {
  switch (s) {
    case TG_OK: return "ok";
    case TG_ERR_INVALID_ARG: return "invalid argument";
    case TG_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case TG_ERR_BUDGET: return "invalid budget (k < 1, k > n, or more protected tokens than k)";
    case TG_ERR_WORKSPACE: return "workspace too small";
    case TG_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int tg_last_cuda_error(void) { return t_last_cuda_error; }

tg_status tg_device_error(uint32_t* word, int clear) {
  TG_CHECK(word != nullptr, TG_ERR_INVALID_ARG);
  unsigned int v = 0;
  TG_TRY(cudaMemcpyFromSymbol(&v, g_tg_error_word, sizeof(v)));
  *word = v;
  if (clear) {
    const unsigned int z = 0;
    TG_TRY(cudaMemcpyToSymbol(g_tg_error_word, &z, sizeof(z)));
  }
  return TG_OK;
}

tg_status tg_selftest_wait_timeout(int32_t mode, int64_t limit_ns, int32_t* result, void* ws,
                                   size_t ws_bytes, tg_stream stream) {
  TG_CHECK(mode >= 0 && mode <= 2 && result != nullptr, TG_ERR_INVALID_ARG);
  TG_CHECK(limit_ns >= 1000 && limit_ns <= 1000000000, TG_ERR_INVALID_ARG);
  TG_CHECK(aligned16(result), TG_ERR_INVALID_ARG);
  if (mode == 2) TG_CHECK(ws != nullptr && ws_bytes >= 16 && aligned16(ws), TG_ERR_WORKSPACE);
  unsigned int* err = device_error_word();
  TG_CHECK(err != nullptr, TG_ERR_CUDA);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const auto lim = static_cast<unsigned long long>(limit_ns);
  if (mode == 2) {
    TG_TRY(cudaMemsetAsync(ws, 0, 16, st));
    TG_TRY(launch_selftest_gridbar(static_cast<unsigned*>(ws), err, lim, result, st));
    return TG_OK;
  }
  TG_TRY(launch_selftest_mbar(err, lim, mode == 1 ? 1 : 0, result, st));
  return TG_OK;
}

const char* tg_version(void) { return "tokengate-b200 0.1.0 (sm_100a)"; }

tg_status tg_trace_start(int32_t capacity) {
  TG_CHECK(capacity >= 1 && capacity <= (1 << 20), TG_ERR_INVALID_ARG);
  Tracer& T = t_trace;
  while (T.ev.size() < size_t(2) * capacity) {
    cudaEvent_t ev;
    TG_TRY(cudaEventCreate(&ev));
    T.ev.push_back(ev);
  }
  T.cap = capacity;
  T.recs.clear();
  T.layer = -1;
  T.on = true;
  return TG_OK;
}

int32_t tg_trace_stop(tg_trace_record* out, int32_t cap) {
  Tracer& T = t_trace;
  T.on = false;
  const int n = static_cast<int>(T.recs.size());
  if (n == 0) return 0;
  cudaError_t e = cudaEventSynchronize(T.ev[2 * (n - 1) + 1]);
  if (e != cudaSuccess) return -static_cast<int32_t>(cuda_status(e));
  int count = 0;
  for (int i = 0; i < n && i < cap; ++i) {
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, T.ev[2 * i], T.ev[2 * i + 1]);
    if (e != cudaSuccess) return -static_cast<int32_t>(cuda_status(e));
    T.recs[i].ms = ms;
    if (out) out[i] = T.recs[i];
    ++count;
  }
  T.recs.clear();
  return count;
}

tg_status tg_decode_step(const tg_model* model, const void* x, int64_t pos, int32_t gate_layer,
                         const tg_kv* kv, const int64_t* lens, const float* scores, int64_t n,
                         const int32_t* kept_idx, int64_t k_kept, void* out, void* ws,
                         size_t ws_bytes, tg_stream stream) {
  const tg_status vs =
      validate_decode(model, x, pos, gate_layer, kv, lens, scores, n, kept_idx, k_kept, out);
  if (vs != TG_OK) return vs;
  const tg_model& m = *model;
  DecodePlan P(nullptr, m, scores ? k_kept : 0);
  TG_CHECK(ws != nullptr && ws_bytes >= P.bytes, TG_ERR_WORKSPACE);
  P = DecodePlan(ws, m, scores ? k_kept : 0);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int hkv = m.n_heads_kv;

  DecStepParams p{};
  for (int l = 0; l < m.n_layers; ++l) {
    const tg_layer& L = m.layers[l];
    DecLayerPtrs& q = p.layer[l];
    q.wqkv = static_cast<const __nv_bfloat16*>(L.wqkv);
    q.wo = static_cast<const __nv_bfloat16*>(L.wo);
    q.w_gate_up = static_cast<const __nv_bfloat16*>(L.w_gate_up);
    q.w_down = static_cast<const __nv_bfloat16*>(L.w_down);
    q.attn_norm = L.attn_norm;
    q.ffn_norm = L.ffn_norm;
    q.q_norm = L.q_norm;
    q.k_norm = L.k_norm;
    q.gain = L.gain;
    q.tau = L.tau;
    q.k_cache = static_cast<__nv_bfloat16*>(kv[l].k);
    q.v_cache = static_cast<__nv_bfloat16*>(kv[l].v);
    q.len = lens[l];
  }
  p.n_layers = m.n_layers;
  p.d = m.d_model;
  p.hq = m.n_heads_q;
  p.hkv = hkv;
  p.dffn = m.d_ffn;
  p.gate_layer = gate_layer;
  p.eps = m.norm_eps;
  p.rope_base = m.rope_base;
  p.final_norm = m.final_norm;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.pos = pos;
  p.scores = scores;
  p.n_scores = n;
  p.kept_idx = kept_idx;
  p.k_kept = scores ? k_kept : 0;
  p.h = P.h;
  p.qkv = P.qkv;
  p.o = P.o;
  p.act = P.act;
  p.lsig = P.lsig;
  p.part = P.part;
  p.merge_cnt = P.cnt;
  p.bar = P.cnt + hkv;
  p.grid = decode_grid();
  p.n_split = decode_splits(hkv);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = device_error_word();
  // algorithmic bytes: every weight once, every cached k/v row once, the new rows written
  double bytes = 0.0;
  const double qkvw = double(m.n_heads_q + 2 * hkv) * m.head_dim * m.d_model;
  for (int l = 0; l < m.n_layers; ++l) {
    bytes += 2.0 * (qkvw + double(m.d_model) * m.n_heads_q * m.head_dim);
    if (m.layers[l].w_gate_up) bytes += 2.0 * 3.0 * double(m.d_ffn) * m.d_model;
    bytes += (2.0 * lens[l] + 2.0) * hkv * m.head_dim * 2.0;
  }
  TG_TRY(cudaMemsetAsync(P.cnt, 0, P.cnt_bytes, st));
  TG_TRY(traced(TG_K_DECODE_STEP, 1, 0.0, bytes, st, [&] { return launch_decode_step(p, st); }));
  return TG_OK;
}

// ---- Gated DeltaNet mixer
namespace {
bool overlaps(const void* p, size_t pn, const void* q, size_t qn) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
  return a < b + qn && b < a + pn;
}
}  // namespace

size_t tg_gated_deltanet_workspace_size(const tg_gdn_layer* L, int64_t T) {
  if (validate_gdn_layer(L) != TG_OK || T < 0) return 0;
  return GdnPlan(nullptr, T, L->n_heads_k, L->n_heads_v, L->head_dim_k, L->head_dim_v).bytes;
}

tg_status tg_gated_deltanet(const tg_gdn_layer* L, const void* qkv, const void* z, const void* a,
                            const void* b, int64_t T, tg_dtype dtype, const void* conv_in,
                            void* conv_out, const float* state_in, float* state_out, void* y,
                            void* ws, size_t ws_bytes, tg_stream stream) {
  const tg_status vs = validate_gdn_layer(L);
  if (vs != TG_OK) return vs;
  TG_CHECK(dtype == TG_BF16 || dtype == TG_F32, TG_ERR_UNSUPPORTED);
  TG_CHECK(T >= 0 && T < (int64_t(1) << 31) - 64, TG_ERR_INVALID_ARG);
  if (T > 0) TG_CHECK(qkv && z && a && b && y, TG_ERR_INVALID_ARG);
  const int hk = L->n_heads_k, hv = L->n_heads_v, dk = L->head_dim_k, dv = L->head_dim_v;
  const int W = L->conv_width;
  const size_t C = size_t(2) * hk * dk + size_t(hv) * dv;
  const size_t conv_bytes = size_t(W - 1) * C * elem_size(dtype);
  const size_t state_bytes = size_t(hv) * dv * dk * 4;
  if (conv_in && conv_out && W > 1)
    TG_CHECK(!overlaps(conv_in, conv_bytes, conv_out, conv_bytes), TG_ERR_INVALID_ARG);
  if (state_in && state_out && state_in != state_out)
    TG_CHECK(!overlaps(state_in, state_bytes, state_out, state_bytes), TG_ERR_INVALID_ARG);
  GdnPlan plan(nullptr, T, hk, hv, dk, dv);
  TG_CHECK(ws != nullptr || plan.bytes == 0, TG_ERR_WORKSPACE);
  TG_CHECK(ws_bytes >= plan.bytes, TG_ERR_WORKSPACE);
  TG_CHECK(aligned16(ws), TG_ERR_INVALID_ARG);
  plan = GdnPlan(ws, T, hk, hv, dk, dv);
  GdnArgs g = plan.a;
  g.qkv = qkv;
  g.z = z;
  g.a = a;
  g.b = b;
  g.ld_qkv = static_cast<int64_t>(C);
  g.ld_z = int64_t(hv) * dv;
  g.ld_ab = hv;
  g.T = T;
  g.hk = hk;
  g.hv = hv;
  g.dk = dk;
  g.dv = dv;
  g.W = W;
  g.conv_w = L->conv_w;
  g.A_log = L->A_log;
  g.dt_bias = L->dt_bias;
  g.norm_w = L->norm_w;
  g.eps = L->norm_eps;
  g.conv_in = conv_in;
  g.conv_out = conv_out;
  g.state_in = state_in;
  g.state_out = state_out;
  g.y = y;
  g.err = device_error_word();
  TG_TRY(gdn_run(g, dtype == TG_BF16, reinterpret_cast<cudaStream_t>(stream)));
  return TG_OK;
}

const char* tg_kernel_name(int32_t kernel) {
  static const char* names[TG_K_COUNT] = {
      "copy", "rmsnorm", "gemm_tc_store", "gemm_tc_residual", "gemm_tc_swiglu", "gemm_tc_score",
      "rope_prep", "attention_tc", "select", "compact", "gemm_f32", "attention_f32", "f32_helper",
      "gemm_tc_qkv", "rope_table", "decode_step", "attn_bwd_prep", "attn_bwd_dkdv",
      "attn_bwd_dq", "attn_bwd_final", "gdn_prep", "gdn_chunk", "gdn_recur", "gdn_out",
      "fold_norm"};
  return (kernel >= 0 && kernel < TG_K_COUNT) ? names[kernel] : "unknown";
}

}  // extern "C"
