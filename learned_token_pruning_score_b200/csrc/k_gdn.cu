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
// Three kernels:
//   gdn_prep   one warp per (token, key head) or (token, value head): the
//              convolution, SiLU, the L2 norms, k.q, alpha and beta; writes
//              fp32 operands in the layouts the recurrence streams.
//   gdn_recur  the recurrence. Row i of S evolves on its own:
//                s_i <- alpha s_i + u_i k,  u_i = beta (v_i - alpha s_i.k)
//                o_i  = alpha s_i.q + u_i (k.q)          (s_i the old row)
//              so a CTA owns 16 rows of one value head, each row held in
//              registers by dk/16 lanes (16 columns each); per token the
//              lanes of a row form the two dot products s.k and s.q with a
//              few shuffles, then update. A producer warp streams 32-token
//              chunks of q, k, v, alpha, beta, k.q into a 4-stage shared
//              memory ring with bulk copies. The state stays fp32 in
//              registers for the whole sequence.
//   gdn_out    one warp per (token, value head): the gated RMSNorm.
// plus gdn_conv_state, which writes the carried convolution rows.
#include <algorithm>

#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kCh = 32;      // tokens per staged chunk
constexpr int kStages = 4;   // chunks in flight
constexpr int kRows = 16;    // state rows (value dims) per CTA
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
  if (r >= 0) return ld_act(static_cast<const T*>(a.qkv) + r * C + c);
  if (a.conv_in == nullptr) return 0.f;
  return ld_act(static_cast<const T*>(a.conv_in) + (r + a.W - 1) * C + c);
}

template <typename T>
__device__ __forceinline__ float conv_silu(const GdnArgs& a, int64_t t, int64_t c, int C) {
  float acc = 0.f;
  for (int i = 0; i < a.W; ++i)
    acc = fmaf(__ldg(a.conv_w + c * a.W + i), conv_src<T>(a, t - (a.W - 1) + i, c, C), acc);
  return silu_f(acc);
}

// ------------------------------------------------------------------ prep
template <typename T, int kDk>
__global__ void __launch_bounds__(256) gdn_prep(GdnArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int kPer = kDk / 32;
  const int lane = threadIdx.x & 31;
  const int tasks = a.hk + a.hv;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (gw >= a.T * tasks) return;
  const int64_t t = gw / tasks;
  const int task = static_cast<int>(gw % tasks);
  const int C = 2 * a.hk * kDk + a.hv * a.dv;
  const int64_t tp = a.t_pad;
  if (task < a.hk) {
    const int h = task;
    float q[kPer], k[kPer];
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int c = h * kDk + lane * kPer + j;
      q[j] = conv_silu<T>(a, t, c, C);
      k[j] = conv_silu<T>(a, t, a.hk * kDk + c, C);
      sq = fmaf(q[j], q[j], sq);
      sk = fmaf(k[j], k[j], sk);
    }
    sq = warp_sum(sq);
    sk = warp_sum(sk);
    const float rq = 1.f / (sqrtf(sq + kL2Eps) * sqrtf(static_cast<float>(kDk)));
    const float rk = 1.f / sqrtf(sk + kL2Eps);
    float kq = 0.f;
    float* qn = a.qn + (h * tp + t) * kDk + lane * kPer;
    float* kn = a.kn + (h * tp + t) * kDk + lane * kPer;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      q[j] *= rq;
      k[j] *= rk;
      kq = fmaf(q[j], k[j], kq);
      qn[j] = q[j];
      kn[j] = k[j];
    }
    kq = warp_sum(kq);
    if (lane == 0) a.kq[h * tp + t] = kq;
  } else {
    const int h = task - a.hk;
    const int per = a.dv / 32;
    for (int j = 0; j < per; ++j) {
      const int cl = lane * per + j;  // channel within the head
      const float v = conv_silu<T>(a, t, 2 * a.hk * kDk + h * a.dv + cl, C);
      a.vb[((static_cast<int64_t>(h) * (a.dv / kRows) + cl / kRows) * tp + t) * kRows +
           cl % kRows] = v;
    }
    if (lane == 0) {
      const float av = ld_act(static_cast<const T*>(a.a) + t * a.hv + h);
      const float bv = ld_act(static_cast<const T*>(a.b) + t * a.hv + h);
      const float g = -expf(__ldg(a.A_log + h)) * softplus_f(av + __ldg(a.dt_bias + h));
      a.al[h * tp + t] = expf(g);
      a.be[h * tp + t] = 1.f / (1.f + expf(-bv));
    }
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

// ------------------------------------------------------------------ recurrence
template <int kDk>
struct RecurSmem {
  float q[kStages][kCh][kDk];
  float k[kStages][kCh][kDk];
  float v[kStages][kCh][kRows];
  float al[kStages][kCh];
  float be[kStages][kCh];
  float kq[kStages][kCh];
  uint64_t full[kStages];
  uint64_t empty[kStages];
};

template <int kDk>
constexpr int recur_consumers() { return kRows * (kDk / 16); }

template <int kDk>
__global__ void __launch_bounds__(recur_consumers<kDk>() + 32) gdn_recur(GdnArgs a) {
  constexpr int kLpr = kDk / 16;  // lanes per state row
  constexpr int kCons = recur_consumers<kDk>();
  constexpr int kConsWarps = kCons / 32;
  constexpr uint32_t kStageBytes = 2u * kCh * kDk * 4u + kCh * kRows * 4u + 3u * kCh * 4u;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  RecurSmem<kDk>& sm = *reinterpret_cast<RecurSmem<kDk>*>(smem_raw);
  unsigned int* err = a.err;

  const int rblocks = a.dv / kRows;
  const int h = blockIdx.x / rblocks;
  const int rb = blockIdx.x % rblocks;
  const int hkey = h / (a.hv / a.hk);
  const int64_t tp = a.t_pad;
  const int n_chunks = static_cast<int>((a.T + kCh - 1) / kCh);

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
      bulk_load(&sm.q[s][0][0], a.qn + (hkey * tp + t0) * kDk, kCh * kDk * 4, &sm.full[s]);
      bulk_load(&sm.k[s][0][0], a.kn + (hkey * tp + t0) * kDk, kCh * kDk * 4, &sm.full[s]);
      bulk_load(&sm.v[s][0][0], a.vb + ((static_cast<int64_t>(h) * rblocks + rb) * tp + t0) * kRows,
                kCh * kRows * 4, &sm.full[s]);
      bulk_load(&sm.al[s][0], a.al + h * tp + t0, kCh * 4, &sm.full[s]);
      bulk_load(&sm.be[s][0], a.be + h * tp + t0, kCh * 4, &sm.full[s]);
      bulk_load(&sm.kq[s][0], a.kq + hkey * tp + t0, kCh * 4, &sm.full[s]);
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
  float2 s[8];
#pragma unroll
  for (int m = 0; m < 4; ++m)
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
    const int n_tok = static_cast<int>(std::min<int64_t>(kCh, a.T - static_cast<int64_t>(c) * kCh));
    for (int tt = 0; tt < n_tok; ++tt) {
      const float4* kr = reinterpret_cast<const float4*>(&sm.k[st][tt][j * 4]);
      const float4* qr = reinterpret_cast<const float4*>(&sm.q[st][tt][j * 4]);
      float2 kk[8], qq[8];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 k4 = kr[m * kLpr];
        const float4 q4 = qr[m * kLpr];
        kk[2 * m] = make_float2(k4.x, k4.y);
        kk[2 * m + 1] = make_float2(k4.z, k4.w);
        qq[2 * m] = make_float2(q4.x, q4.y);
        qq[2 * m + 1] = make_float2(q4.z, q4.w);
      }
      float2 dk0 = make_float2(0.f, 0.f), dk1 = dk0, dq0 = dk0, dq1 = dk0;
#pragma unroll
      for (int m = 0; m < 8; m += 2) {
        dk0 = ffma2(s[m], kk[m], dk0);
        dk1 = ffma2(s[m + 1], kk[m + 1], dk1);
        dq0 = ffma2(s[m], qq[m], dq0);
        dq1 = ffma2(s[m + 1], qq[m + 1], dq1);
      }
      float sk = (dk0.x + dk0.y) + (dk1.x + dk1.y);
      float sq = (dq0.x + dq0.y) + (dq1.x + dq1.y);
#pragma unroll
      for (int o = 1; o < kLpr; o <<= 1) {
        sk += __shfl_xor_sync(0xFFFFFFFFu, sk, o);
        sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
      }
      const float al = sm.al[st][tt];
      const float u = sm.be[st][tt] * (sm.v[st][tt][g] - al * sk);
      const float2 al2 = make_float2(al, al), u2 = make_float2(u, u);
#pragma unroll
      for (int m = 0; m < 8; ++m) s[m] = ffma2(al2, s[m], fmul2(u2, kk[m]));
      if (j == 0) out[(static_cast<int64_t>(c) * kCh + tt) * out_stride] = fmaf(al, sq, u * sm.kq[st][tt]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);
  }
  if (a.state_out) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
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
  const T* z = static_cast<const T*>(a.z) + gw * a.dv + lane * per;
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
  if (stage == 0) {
    if (a.T > 0) {
      const int64_t warps = a.T * (a.hk + a.hv);
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
