// k_gdn.cu -- the Gated DeltaNet token mixer over a token sequence (in the
// gated prefill of a hybrid model: the kept tokens, in order).
//
// In hybrid models most layers are Gated DeltaNet layers. The scorer reads
// hidden states, so the gate may sit at such a layer. The gate's logit bias
// exists only in the full-attention layers; a Gated DeltaNet layer above the
// gate has no logits and simply runs on the kept tokens (Tencent Cloud
// article "TokenGate：端到端可训练的 Token 剪枝机制，让大模型 Prefill 提速 11.3 倍",
// section "门控位置影响剪枝效果", figure 5). The layer itself is the published
// gated delta rule (Yang, Kautz and Hatamizadeh, "Gated Delta Networks:
// Improving Mamba2 with Delta Rule", ICLR 2025) in the Qwen3-Next layer shape:
//   c_t   = SiLU(causal depthwise conv of width W over the qkv channels)
//   q_t   = l2norm(c_q) / sqrt(dk),  k_t = l2norm(c_k),  v_t = c_v
//   alpha = exp(-exp(A_log) softplus(a_t + dt_bias)),  beta = sigmoid(b_t)
//   S_t   = alpha S_{t-1} (I - beta k k^T) + beta v k^T      (S: dv x dk)
//   o_t   = S_t q_t,   y_t = RMSNorm(o_t) * w * SiLU(z_t)   (per value head)
//
// Kernels, in launch order:
//   gdn_prep   one warp per (16 tokens, q or k of a key head, or 128
//              channels of a value head): the sliding convolution, SiLU, the L2 norms, the log
//              decay g and beta; fp32 operands in the layouts the later
//              kernels stream, zero rows past the last token.
//   gdn_chunk  one CTA per (value head, 32-token chunk): the chunk's Gram
//              entries k_i.k_j and q_i.k_j, and from them the two triangular
//              matrices that solve the chunk's recurrence for any incoming
//              state row (the WY / UT form of the delta rule).
//   gdn_recur  the state. Rows of S evolve independently, so a CTA owns 16
//              rows of one value head, each held in registers by dk/8 lanes
//              (8 columns each), and walks the chunks in order: the row's
//              dot products with the chunk's 32 keys and queries, one
//              cross-lane reduction, two triangular matrix-vector products
//              (outputs, corrections), and the rank-32 update of the row. No
//              step waits on the previous token; a producer warp streams each
//              chunk's operands into a 3-stage ring with bulk copies.
//   gdn_out    one warp per (token, value head): the gated RMSNorm.
// plus gdn_conv_state, which writes the carried convolution rows.
#include <algorithm>

#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kCh = kGdnChunk;  // tokens per chunk
constexpr int kStages = 3;      // chunks in flight in the recurrence's ring
constexpr int kRows = 16;       // state rows (value dims) per recurrence CTA
constexpr int kLd = kGdnLd;     // row stride (floats) of the chunk matrices
constexpr int kTb = 16;      // tokens per prep warp
constexpr int kMaxW = 4;     // widest convolution
constexpr float kL2Eps = 1e-6f;

template <typename T>
__device__ __forceinline__ float ld_act(const T* p);
template <>
__device__ __forceinline__ float ld_act<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_act<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}
template <typename T>
__device__ __forceinline__ T st_act(float v);
template <>
__device__ __forceinline__ float st_act<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 st_act<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Packed fp32 pair product (Blackwell f32x2 instruction).
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}

// The input row r of the convolution: token r of qkv for r >= 0, else the
// carried row W-1+r (zeros when none is carried).
template <typename T>
__device__ __forceinline__ float conv_src(const GdnArgs& a, int64_t r, int64_t c, int C) {
  if (r >= 0) return ld_act(static_cast<const T*>(a.qkv) + r * a.ld_qkv + c);
  if (a.conv_in == nullptr) return 0.f;
  return ld_act(static_cast<const T*>(a.conv_in) + (r + a.W - 1) * C + c);
}

// ------------------------------------------------------------------ prep
// One warp per (16-token block, key head) or (16-token block, value head).
// Lane l owns channels l + 32 j of its slot, so every load and store of a
// token row is coalesced. The convolution slides: each channel's W weights
// and its last W-1 inputs stay in registers across the block's tokens.
// Tokens in [T, t_pad) get zeros, so padded rows add nothing downstream.
// x * sigmoid(x) from the hardware exponential and reciprocal (relative
// error ~1e-6, far inside the fp32 path's 1e-4 parity bound); for x below
// about -88 the exponential overflows and the reciprocal of inf gives -0.
__device__ __forceinline__ float silu_fast(float x) {
  return __fdividef(x, 1.f + __expf(-x));
}

template <typename T, int kPer>
struct ConvWindow {
  float w[kPer][kMaxW];         // w[j][0]: weight of the current row; w[j][1+m]: of row t-1-m
  float hist[kPer][kMaxW - 1];  // hist[j][m]: input row t-1-m
  float next[kPer];             // the next token's inputs, loaded one step ahead

  __device__ __forceinline__ void load(const GdnArgs& a, const int (&ch)[kPer],
                                       const bool (&on)[kPer], int64_t t, int C) {
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      next[j] = (on[j] && t < a.T) ? ld_act(static_cast<const T*>(a.qkv) + t * a.ld_qkv + ch[j])
                                   : 0.f;
  }

  __device__ __forceinline__ void init(const GdnArgs& a, const int (&ch)[kPer], bool (&on)[kPer],
                                       int64_t t0, int C) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
#pragma unroll
      for (int i = 0; i < kMaxW; ++i) w[j][i] = 0.f;
#pragma unroll
      for (int m = 0; m < kMaxW - 1; ++m) hist[j][m] = 0.f;
      if (!on[j]) continue;
      const float* cw = a.conv_w + static_cast<int64_t>(ch[j]) * a.W;
      w[j][0] = __ldg(cw + a.W - 1);
#pragma unroll
      for (int m = 0; m < kMaxW - 1; ++m)
        if (m < a.W - 1) {
          w[j][1 + m] = __ldg(cw + a.W - 2 - m);
          // a block wholly past the last token only writes zeros: no row >= T is read
          const int64_t r = t0 - 1 - m;
          hist[j][m] = r < a.T ? conv_src<T>(a, r, ch[j], C) : 0.f;
        }
    }
    load(a, ch, on, t0, C);
  }

  // SiLU(conv) of token t (whose inputs load() fetched), then slides the
  // window and fetches token t + 1.
  __device__ __forceinline__ void step(const GdnArgs& a, const int (&ch)[kPer],
                                       const bool (&on)[kPer], int64_t t, int C,
                                       float (&out)[kPer]) {
    float x[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) x[j] = next[j];
    load(a, ch, on, t + 1, C);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      float acc = w[j][0] * x[j];
#pragma unroll
      for (int m = 0; m < kMaxW - 1; ++m) acc = fmaf(w[j][1 + m], hist[j][m], acc);
#pragma unroll
      for (int m = kMaxW - 2; m > 0; --m) hist[j][m] = hist[j][m - 1];
      hist[j][0] = x[j];
      out[j] = silu_fast(acc);
    }
  }
};

// q (which = 0) or k (which = 1) of key head h: L2-normalised, q also
// scaled by dk^-1/2.
template <typename T, int kDk>
__device__ __forceinline__ void prep_qk(const GdnArgs& a, int h, int which, int64_t t0, int lane,
                                        int C) {
  constexpr int kPer = kDk / 32;
  int ch[kPer];
  bool on[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    ch[j] = which * a.hk * kDk + h * kDk + lane + 32 * j;
    on[j] = true;
  }
  ConvWindow<T, kPer> cw;
  cw.init(a, ch, on, t0, C);
  const int64_t tp = a.t_pad;
  const float scale = which == 0 ? 1.f / sqrtf(static_cast<float>(kDk)) : 1.f;
  float* dst = (which == 0 ? a.qn : a.kn) + h * tp * kDk + lane;
  for (int tt = 0; tt < kTb; ++tt) {
    const int64_t t = t0 + tt;
    float* row = dst + t * kDk;
    if (t >= a.T) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) row[32 * j] = 0.f;
      continue;
    }
    float c[kPer];
    cw.step(a, ch, on, t, C, c);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kPer; ++j) ss = fmaf(c[j], c[j], ss);
    ss = warp_sum(ss);
    const float r = scale / sqrtf(ss + kL2Eps);
#pragma unroll
    for (int j = 0; j < kPer; ++j) row[32 * j] = c[j] * r;
  }
}

// Channels [128 part, 128 part + 128) of value head h (4 per lane, those
// past dv predicated off); part 0 also writes g and beta.
template <typename T>
__device__ __forceinline__ void prep_v(const GdnArgs& a, int h, int part, int64_t t0, int lane,
                                       int C) {
  constexpr int kPer = 4;
  int ch[kPer];
  bool on[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int cl = 128 * part + lane + 32 * j;
    ch[j] = 2 * a.hk * a.dk + h * a.dv + cl;
    on[j] = cl < a.dv;
  }
  ConvWindow<T, kPer> cw;
  cw.init(a, ch, on, t0, C);
  const int64_t tp = a.t_pad;
  const int rblocks = a.dv / kRows;
  const float A = expf(__ldg(a.A_log + h));
  const float dtb = __ldg(a.dt_bias + h);
  for (int tt = 0; tt < kTb; ++tt) {
    const int64_t t = t0 + tt;
    const bool live = t < a.T;
    float c[kPer];
    if (live) cw.step(a, ch, on, t, C, c);
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      if (on[j]) {
        const int cl = 128 * part + lane + 32 * j;  // channel within the head
        a.vb[((static_cast<int64_t>(h) * rblocks + cl / kRows) * tp + t) * kRows + cl % kRows] =
            live ? c[j] : 0.f;
      }
    if (lane == 0 && part == 0) {
      float g = 0.f, beta = 0.f;
      if (live) {
        const float av = ld_act(static_cast<const T*>(a.a) + t * a.ld_ab + h);
        const float bv = ld_act(static_cast<const T*>(a.b) + t * a.ld_ab + h);
        g = -A * softplus_f(av + dtb);
        beta = 1.f / (1.f + expf(-bv));
      }
      a.gl[h * tp + t] = g;
      a.be[h * tp + t] = beta;
    }
  }
}

constexpr int prep_v_parts(int dv) { return (dv + 127) / 128; }

template <typename T, int kDk>
__global__ void __launch_bounds__(256) gdn_prep(GdnArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int vparts = prep_v_parts(a.dv);
  const int slots = 2 * a.hk + a.hv * vparts;  // q heads, k heads, value-head parts
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (gw >= (a.t_pad / kTb) * slots) return;
  const int64_t t0 = (gw / slots) * kTb;
  const int slot = static_cast<int>(gw % slots);
  const int C = 2 * a.hk * kDk + a.hv * a.dv;
  if (slot < 2 * a.hk) {
    prep_qk<T, kDk>(a, slot % a.hk, slot / a.hk, t0, lane, C);
  } else {
    const int v = slot - 2 * a.hk;
    prep_v<T>(a, v / vparts, v % vparts, t0, lane, C);
  }
}

// The last W-1 rows of [carried rows; qkv], the next call's carried rows.
template <typename T>
__global__ void __launch_bounds__(256) gdn_conv_state(GdnArgs a) {
  pdl_trigger();
  pdl_wait();
  const int C = 2 * a.hk * a.dk + a.hv * a.dv;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(a.W - 1) * C) return;
  const int64_t r = idx / C, c = idx % C;
  const int64_t src = a.T + r - (a.W - 1);  // row of qkv, or (negative) of the carried rows
  const float v = conv_src<T>(a, src, c, C);
  static_cast<T*>(a.conv_out)[idx] = st_act<T>(v);
}

// ------------------------------------------------------------------ chunk matrices
// The recurrence over one 32-token chunk, solved in closed form. With gamma
// the running sum of g inside the chunk, a state row s entering the chunk,
// Pk_i = s.k_i, Pq_i = s.q_i and r_i = beta_i (v_i - e^gamma_i Pk_i), the
// per-token corrections u_i = beta_i (v_i - alpha_i s_{i-1}.k_i) satisfy
//   (I + A) u = r,  A_ij = beta_i e^(gamma_i - gamma_j) (k_i.k_j)   (j < i),
// the outputs are o_i = e^gamma_i Pq_i + sum_{j<=i} e^(gamma_i - gamma_j) (q_i.k_j) u_j
// and the row leaving the chunk is e^gamma_31 s + sum_i e^(gamma_31 - gamma_i) u_i k_i.
// This kernel forms, once per (value head, chunk), the two matrices that
// map r to what the rows need:
//   Tt = diag(e^(gamma_31 - gamma)) (I + A)^-1     (u decayed to the chunk end)
//   M  = Wqk (I + A)^-1,  Wqk_ij = e^(gamma_i - gamma_j) (q_i.k_j)  (j <= i)
// and e^gamma. Both are lower triangular; rows are stored kLd floats apart
// (zeros above the diagonal and in the padding columns).
template <int kDk>
__global__ void __launch_bounds__(256) gdn_chunk(GdnArgs a) {
  __shared__ __align__(16) float ks[kCh][kDk + 4];
  __shared__ __align__(16) float qs[kCh][kDk + 4];
  __shared__ float Am[kCh][kCh + 1];
  __shared__ float Wq[kCh][kCh + 1];
  __shared__ float Tm[kCh][kCh + 1];
  __shared__ float gam[kCh], bes[kCh], dec[kCh];
  pdl_trigger();
  pdl_wait();
  const int c = blockIdx.x, h = blockIdx.y;
  const int hkey = h / (a.hv / a.hk);
  const int64_t tp = a.t_pad, t0 = static_cast<int64_t>(c) * kCh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int idx = tid; idx < kCh * kDk / 4; idx += 256) {
    const int i = idx / (kDk / 4), d = (idx % (kDk / 4)) * 4;
    *reinterpret_cast<float4*>(&ks[i][d]) =
        *reinterpret_cast<const float4*>(a.kn + (hkey * tp + t0 + i) * kDk + d);
    *reinterpret_cast<float4*>(&qs[i][d]) =
        *reinterpret_cast<const float4*>(a.qn + (hkey * tp + t0 + i) * kDk + d);
  }
  if (warp == 0) {
    float x = a.gl[h * tp + t0 + lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    const float last = __shfl_sync(0xFFFFFFFFu, x, 31);
    gam[lane] = x;
    dec[lane] = expf(last - x);
    bes[lane] = a.be[h * tp + t0 + lane];
    a.eg[h * tp + t0 + lane] = expf(x);
  }
  __syncthreads();
  // Gram entries: lane = column j, rows i = warp + 8 r
  {
    float gk[4] = {0.f, 0.f, 0.f, 0.f}, gq[4] = {0.f, 0.f, 0.f, 0.f};
    for (int d = 0; d < kDk; d += 4) {
      const float4 kj = *reinterpret_cast<const float4*>(&ks[lane][d]);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 ki = *reinterpret_cast<const float4*>(&ks[warp + 8 * r][d]);
        const float4 qi = *reinterpret_cast<const float4*>(&qs[warp + 8 * r][d]);
        gk[r] = fmaf(ki.x, kj.x, fmaf(ki.y, kj.y, fmaf(ki.z, kj.z, fmaf(ki.w, kj.w, gk[r]))));
        gq[r] = fmaf(qi.x, kj.x, fmaf(qi.y, kj.y, fmaf(qi.z, kj.z, fmaf(qi.w, kj.w, gq[r]))));
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = warp + 8 * r, j = lane;
      const float e = j <= i ? expf(gam[i] - gam[j]) : 0.f;
      Am[i][j] = j < i ? bes[i] * e * gk[r] : 0.f;
      Wq[i][j] = e * gq[r];
    }
  }
  __syncthreads();
  // (I + A)^-1 by forward substitution, one column per lane of warp 0
  if (warp == 0) {
    float col[kCh];
#pragma unroll
    for (int i = 0; i < kCh; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) acc = fmaf(Am[i][m], col[m], acc);
      col[i] = i < lane ? 0.f : (i == lane ? 1.f : -acc);
    }
#pragma unroll
    for (int i = 0; i < kCh; ++i) Tm[i][lane] = col[i];
  }
  __syncthreads();
  const int64_t base = (static_cast<int64_t>(h) * (tp / kCh) + c) * kCh * kLd;
  for (int p = tid; p < kCh * kLd; p += 256) {
    const int i = p / kLd, j = p % kLd;
    float tv = 0.f, mv = 0.f;
    if (j <= i) {
      tv = dec[i] * Tm[i][j];
      for (int m = j; m <= i; ++m) mv = fmaf(Wq[i][m], Tm[m][j], mv);
    }
    a.tt[base + p] = tv;
    a.mm[base + p] = mv;
  }
}

// ------------------------------------------------------------------ recurrence
template <int kDk>
struct RecurSmem {
  float q[kStages][kCh][kDk];
  float k[kStages][kCh][kDk];
  float v[kStages][kCh][kRows];
  float be[kStages][kCh];
  float eg[kStages][kCh];
  float tt[kStages][kCh][kLd];
  float mm[kStages][kCh][kLd];
  float prow[kRows][2 * kCh];  // per row: Pk (32) then Pq (32), reduced
  float urow[kRows][kCh];      // per row: the decayed corrections Tt r
  uint64_t full[kStages];
  uint64_t empty[kStages];
};

template <int kDk>
constexpr int recur_lanes() { return kDk / 8; }  // lanes per state row, 8 columns each
template <int kDk>
constexpr int recur_consumers() { return kRows * recur_lanes<kDk>(); }

// One level of the cross-lane transpose-reduce: the lanes whose bit `o` is
// set keep the upper half of their N values, the others the lower half, and
// each adds its partner's copy of the half it keeps.
template <int N, int O>
__device__ __forceinline__ void reduce_rows(float (&P)[2 * kCh], int j) {
  const bool up = (j & O) != 0;
#pragma unroll
  for (int v = 0; v < N / 2; ++v) {
    const float send = up ? P[v] : P[v + N / 2];
    const float keep = up ? P[v + N / 2] : P[v];
    P[v] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, O);
  }
  if constexpr (O > 1) reduce_rows<N / 2, O / 2>(P, j);
}

template <int kDk>
__global__ void __launch_bounds__(recur_consumers<kDk>() + 32) gdn_recur(GdnArgs a) {
  constexpr int kLpr = recur_lanes<kDk>();
  constexpr int kVec = 8 / 4;  // float4 column groups per lane
  constexpr int kCons = recur_consumers<kDk>();
  constexpr int kConsWarps = kCons / 32;
  constexpr int kHeld = 2 * kCh / kLpr;  // reduced values a lane holds
  constexpr uint32_t kStageBytes =
      2u * kCh * kDk * 4u + kCh * kRows * 4u + 2u * kCh * 4u + 2u * kCh * kLd * 4u;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  RecurSmem<kDk>& sm = *reinterpret_cast<RecurSmem<kDk>*>(smem_raw);
  unsigned int* err = a.err;

  const int rblocks = a.dv / kRows;
  const int h = blockIdx.x / rblocks;
  const int rb = blockIdx.x % rblocks;
  const int hkey = h / (a.hv / a.hk);
  const int64_t tp = a.t_pad;
  const int n_chunks = static_cast<int>(tp / kCh);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();

  if (threadIdx.x >= kCons) {
    // ---- producer warp
    if (threadIdx.x != kCons) return;
    int issued = 0;
    for (int c = 0; c < n_chunks; ++c) {
      const int s = c % kStages;
      if (c >= kStages && !mbar_wait(&sm.empty[s], ((c / kStages) - 1) & 1, err)) break;
      mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
      const int64_t t0 = static_cast<int64_t>(c) * kCh;
      const int64_t mat = (static_cast<int64_t>(h) * n_chunks + c) * kCh * kLd;
      bulk_load(&sm.q[s][0][0], a.qn + (hkey * tp + t0) * kDk, kCh * kDk * 4, &sm.full[s]);
      bulk_load(&sm.k[s][0][0], a.kn + (hkey * tp + t0) * kDk, kCh * kDk * 4, &sm.full[s]);
      bulk_load(&sm.v[s][0][0], a.vb + ((static_cast<int64_t>(h) * rblocks + rb) * tp + t0) * kRows,
                kCh * kRows * 4, &sm.full[s]);
      bulk_load(&sm.be[s][0], a.be + h * tp + t0, kCh * 4, &sm.full[s]);
      bulk_load(&sm.eg[s][0], a.eg + h * tp + t0, kCh * 4, &sm.full[s]);
      bulk_load(&sm.tt[s][0][0], a.tt + mat, kCh * kLd * 4, &sm.full[s]);
      bulk_load(&sm.mm[s][0][0], a.mm + mat, kCh * kLd * 4, &sm.full[s]);
      issued = c + 1;
    }
    // Let every copy this thread issued land before the CTA can exit.
    for (int c = std::max(0, issued - kStages); c < issued; ++c)
      mbar_wait(&sm.full[c % kStages], (c / kStages) & 1, err);
    return;
  }

  // ---- consumers: thread = (row g of the CTA, lane j of the row)
  const int g = threadIdx.x / kLpr;
  const int j = threadIdx.x % kLpr;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(h) * a.dv + rb * kRows + g;
  // columns j*4 + 4*kLpr*m + e: for each m the kLpr lanes of a row read one
  // contiguous 16*kLpr-byte run of q/k (every row reads the same: broadcast)
  float2 s[2 * kVec];
#pragma unroll
  for (int m = 0; m < kVec; ++m)
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const int col = j * 4 + 4 * kLpr * m + e;
      s[m * 2 + e / 2] = a.state_in ? make_float2(a.state_in[row * kDk + col],
                                                  a.state_in[row * kDk + col + 1])
                                    : make_float2(0.f, 0.f);
    }
  float* out = a.o + static_cast<int64_t>(h) * a.dv + rb * kRows + g;
  const int64_t out_stride = static_cast<int64_t>(a.hv) * a.dv;

  for (int c = 0; c < n_chunks; ++c) {
    const int st = c % kStages;
    if (!mbar_wait_warp(&sm.full[st], (c / kStages) & 1, err)) break;
    const int64_t t0 = static_cast<int64_t>(c) * kCh;
    // (1) partial dot products of this lane's 16 columns with every k_i, q_i
    float P[2 * kCh];
#pragma unroll
    for (int i = 0; i < kCh; ++i) {
      const float4* kr = reinterpret_cast<const float4*>(&sm.k[st][i][j * 4]);
      const float4* qr = reinterpret_cast<const float4*>(&sm.q[st][i][j * 4]);
      float2 ak = make_float2(0.f, 0.f), aq = ak;
#pragma unroll
      for (int m = 0; m < kVec; ++m) {
        const float4 k4 = kr[m * kLpr];
        const float4 q4 = qr[m * kLpr];
        ak = ffma2(s[2 * m], make_float2(k4.x, k4.y), ak);
        ak = ffma2(s[2 * m + 1], make_float2(k4.z, k4.w), ak);
        aq = ffma2(s[2 * m], make_float2(q4.x, q4.y), aq);
        aq = ffma2(s[2 * m + 1], make_float2(q4.z, q4.w), aq);
      }
      P[i] = ak.x + ak.y;
      P[kCh + i] = aq.x + aq.y;
    }
    // (2) sum over the row's lanes; lane j ends with values [j kHeld, (j+1) kHeld)
    reduce_rows<2 * kCh, kLpr / 2>(P, j);
#pragma unroll
    for (int v = 0; v < kHeld; v += 4)
      *reinterpret_cast<float4*>(&sm.prow[g][j * kHeld + v]) =
          make_float4(P[v], P[v + 1], P[v + 2], P[v + 3]);
    __syncwarp();
    // (3) r, then this lane's outputs i = j + kLpr m: Tt r and M r
    float r[kCh];
#pragma unroll
    for (int i = 0; i < kCh; i += 4) {
      const float4 b4 = *reinterpret_cast<const float4*>(&sm.be[st][i]);
      const float4 e4 = *reinterpret_cast<const float4*>(&sm.eg[st][i]);
      const float4 p4 = *reinterpret_cast<const float4*>(&sm.prow[g][i]);
      r[i] = b4.x * (sm.v[st][i][g] - e4.x * p4.x);
      r[i + 1] = b4.y * (sm.v[st][i + 1][g] - e4.y * p4.y);
      r[i + 2] = b4.z * (sm.v[st][i + 2][g] - e4.z * p4.z);
      r[i + 3] = b4.w * (sm.v[st][i + 3][g] - e4.w * p4.w);
    }
#pragma unroll
    for (int m = 0; m < kCh / kLpr; ++m) {
      const int i = j + kLpr * m;
      const float4* trow = reinterpret_cast<const float4*>(&sm.tt[st][i][0]);
      const float4* mrow = reinterpret_cast<const float4*>(&sm.mm[st][i][0]);
      float ut = 0.f, oo = sm.eg[st][i] * sm.prow[g][kCh + i];
#pragma unroll
      for (int b = 0; b < kLpr * (m + 1) / 4; ++b) {  // entries past i are zero
        const float4 t4 = trow[b];
        const float4 m4 = mrow[b];
        ut = fmaf(t4.x, r[4 * b], fmaf(t4.y, r[4 * b + 1],
                  fmaf(t4.z, r[4 * b + 2], fmaf(t4.w, r[4 * b + 3], ut))));
        oo = fmaf(m4.x, r[4 * b], fmaf(m4.y, r[4 * b + 1],
                  fmaf(m4.z, r[4 * b + 2], fmaf(m4.w, r[4 * b + 3], oo))));
      }
      sm.urow[g][i] = ut;
      if (t0 + i < a.T) out[(t0 + i) * out_stride] = oo;
    }
    __syncwarp();
    // (4) the row leaving the chunk: e^gamma_31 s + sum_i (Tt r)_i k_i
    const float e31 = sm.eg[st][kCh - 1];
    const float2 e2 = make_float2(e31, e31);
#pragma unroll
    for (int m = 0; m < 2 * kVec; ++m) s[m] = fmul2(e2, s[m]);
#pragma unroll
    for (int i = 0; i < kCh; i += 4) {
      const float4 u4 = *reinterpret_cast<const float4*>(&sm.urow[g][i]);
      const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
      for (int d = 0; d < 4; ++d) {
        const float4* kr = reinterpret_cast<const float4*>(&sm.k[st][i + d][j * 4]);
        const float2 u2 = make_float2(uu[d], uu[d]);
#pragma unroll
        for (int m = 0; m < kVec; ++m) {
          const float4 k4 = kr[m * kLpr];
          s[2 * m] = ffma2(u2, make_float2(k4.x, k4.y), s[2 * m]);
          s[2 * m + 1] = ffma2(u2, make_float2(k4.z, k4.w), s[2 * m + 1]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);
  }
  if (a.state_out) {
#pragma unroll
    for (int m = 0; m < kVec; ++m)
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int col = j * 4 + 4 * kLpr * m + e;
        a.state_out[row * kDk + col] = s[m * 2 + e / 2].x;
        a.state_out[row * kDk + col + 1] = s[m * 2 + e / 2].y;
      }
  }
}

// ------------------------------------------------------------------ output
template <typename T>
__global__ void __launch_bounds__(256) gdn_out(GdnArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (gw >= a.T * a.hv) return;
  const int per = a.dv / 32;  // at most 8
  const float* o = a.o + gw * a.dv + lane * per;
  const T* z = static_cast<const T*>(a.z) + (gw / a.hv) * a.ld_z + (gw % a.hv) * a.dv + lane * per;
  T* y = static_cast<T*>(a.y) + gw * a.dv + lane * per;
  float v[8];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per) {
      v[j] = o[j];
      ss = fmaf(v[j], v[j], ss);
    }
  ss = warp_sum(ss);
  const float r = 1.f / sqrtf(ss / static_cast<float>(a.dv) + a.eps);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < per)
      y[j] = st_act<T>(v[j] * r * __ldg(a.norm_w + lane * per + j) * silu_f(ld_act(z + j)));
}

template <typename T>
cudaError_t launch_gdn_t(const GdnArgs& a, int stage, cudaStream_t st) {
  const int n_chunks = static_cast<int>(a.t_pad / kCh);
  if (stage == 0) {
    if (a.T > 0) {
      const int64_t warps = (a.t_pad / kTb) * (2 * a.hk + a.hv * prep_v_parts(a.dv));
      const dim3 grid(static_cast<unsigned>((warps + 7) / 8));
      if (a.dk == 128) {
        TG_CUDA_TRY(launch_pdl(gdn_prep<T, 128>, grid, dim3(256), 0, st, a));
      } else {
        TG_CUDA_TRY(launch_pdl(gdn_prep<T, 64>, grid, dim3(256), 0, st, a));
      }
    }
    if (a.conv_out != nullptr && a.W > 1) {
      const int64_t n = static_cast<int64_t>(a.W - 1) * (2 * a.hk * a.dk + a.hv * a.dv);
      TG_CUDA_TRY(launch_pdl(gdn_conv_state<T>, dim3(static_cast<unsigned>((n + 255) / 256)),
                             dim3(256), 0, st, a));
    }
    return cudaGetLastError();
  }
  if (stage == 1) {
    if (n_chunks > 0) {
      const dim3 grid(static_cast<unsigned>(n_chunks), static_cast<unsigned>(a.hv));
      if (a.dk == 128) {
        TG_CUDA_TRY(launch_pdl(gdn_chunk<128>, grid, dim3(256), 0, st, a));
      } else {
        TG_CUDA_TRY(launch_pdl(gdn_chunk<64>, grid, dim3(256), 0, st, a));
      }
    }
    return cudaGetLastError();
  }
  if (stage == 2) {
    const dim3 grid(static_cast<unsigned>(a.hv * (a.dv / kRows)));
    if (a.dk == 128) {
      const size_t smem = sizeof(RecurSmem<128>);
      TG_CUDA_TRY(cudaFuncSetAttribute(gdn_recur<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
      TG_CUDA_TRY(launch_pdl(gdn_recur<128>, grid, dim3(recur_consumers<128>() + 32), smem, st, a));
    } else {
      const size_t smem = sizeof(RecurSmem<64>);
      TG_CUDA_TRY(cudaFuncSetAttribute(gdn_recur<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem)));
      TG_CUDA_TRY(launch_pdl(gdn_recur<64>, grid, dim3(recur_consumers<64>() + 32), smem, st, a));
    }
    return cudaGetLastError();
  }
  if (a.T > 0) {
    const int64_t warps = a.T * a.hv;
    TG_CUDA_TRY(launch_pdl(gdn_out<T>, dim3(static_cast<unsigned>((warps + 7) / 8)), dim3(256), 0,
                           st, a));
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gdn(const GdnArgs& a, bool bf16, int stage, cudaStream_t st) {
  return bf16 ? launch_gdn_t<__nv_bfloat16>(a, stage, st) : launch_gdn_t<float>(a, stage, st);
}

}  // namespace tg
