// k_simt_f32.cu -- fp32 kernels on the CUDA cores (no tensor cores).
//
// The tensor cores have no fp32-input kind (only TF32, ~1e-3 relative), so
// the fp32 configuration of the path (checked to 1e-4) runs here: a tiled
// SIMT GEMM with a store / residual epilogue, and a token-gated causal GQA
// attention with an online softmax.
//
// The gated attention computes, for the kept rows in compacted order,
//   l_ij = (q_i . k_j) / (sqrt(dh) * tau_h) + gain_h * logsigmoid(s_j), j <= i,
// the kept tokens' scores entering the logits as a bias with per-head gain
// and temperature (Tencent Cloud article "TokenGate：端到端可训练的 Token 剪枝机制，
// 让大模型 Prefill 提速 11.3 倍", section "门控机制为评分网络建立梯度路径";
// ai.866data.com article "让大模型学会"略读"…", section "可学习剪枝的机制设计").
// Positions ascend with the row index, so "causal by original position" is
// "causal by row".
#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16;

__global__ void __launch_bounds__(256) gemm_f32(GemmArgs g) {
  pdl_trigger();
  pdl_wait();
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  const float* A = static_cast<const float*>(g.A);
  const float* B = static_cast<const float*>(g.B);
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
  const int n0 = blockIdx.x * kBN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += kBK) {
    for (int i = threadIdx.x; i < kBM * kBK; i += 256) {
      const int r = i / kBK, c = i % kBK;
      const int64_t gm = m0 + r;
      const int gk = k0 + c;
      As[c][r] = (gm < g.M && gk < g.K) ? A[gm * g.lda + gk] : 0.f;
      const int gn = n0 + r;
      Bs[c][r] = (gn < g.N && gk < g.K) ? B[static_cast<int64_t>(gn) * g.ldb + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* C = static_cast<float*>(g.C);
  const float* R = static_cast<const float*>(g.R);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = m0 + ty * 4 + i;
    if (gm >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= g.N) continue;
      float v = acc[i][j];
      if (g.epi == EPI_RESIDUAL) v += R[gm * g.ldr + gn];
      C[gm * g.ldc + gn] = v;
    }
  }
}

// One warp per (query row, query head). Lanes split the head dimension;
// keys are visited in order with an online (running max) softmax.
template <int kDh>
__global__ void __launch_bounds__(256) attn_f32(AttnArgs a, int64_t v_stride) {
  pdl_trigger();
  pdl_wait();
  constexpr int kPer = kDh / 32;
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= a.T * a.hq) return;
  const int64_t i = item / a.hq;
  const int h = static_cast<int>(item % a.hq);
  const int g = h / (a.hq / a.hkv);
  const float* q = static_cast<const float*>(a.q) + (i * a.hq + h) * kDh;
  const float* kb = static_cast<const float*>(a.k);
  const float* vb = static_cast<const float*>(a.v);
  const float tau = a.tau ? __ldg(a.tau + h) : 1.0f;
  const float gain = a.gain ? __ldg(a.gain + h) : 0.0f;
  const float scale = 1.0f / (sqrtf(static_cast<float>(kDh)) * tau);
  float qr[kPer], o[kPer];
#pragma unroll
  for (int p = 0; p < kPer; ++p) {
    qr[p] = __ldg(q + lane + 32 * p);
    o[p] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int64_t j = 0; j <= i; ++j) {
    const float* kr = kb + (j * a.hkv + g) * kDh;
    float d = 0.f;
#pragma unroll
    for (int p = 0; p < kPer; ++p) d = fmaf(qr[p], __ldg(kr + lane + 32 * p), d);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xFFFFFFFFu, d, off);
    const float logit = d * scale + (a.lsig ? gain * __ldg(a.lsig + j) : 0.f);
    const float m_new = fmaxf(m, logit);
    const float corr = expf(m - m_new);
    const float p_j = expf(logit - m_new);
    l = l * corr + p_j;
    const float* vr = vb + j * v_stride + g * kDh;
#pragma unroll
    for (int p = 0; p < kPer; ++p) o[p] = o[p] * corr + p_j * __ldg(vr + lane + 32 * p);
    m = m_new;
  }
  float* out = static_cast<float*>(a.out) + (i * a.hq + h) * kDh;
  const float inv = 1.0f / l;
  if (a.lse && lane == 0) a.lse[static_cast<int64_t>(h) * a.T + i] = m + logf(l);
#pragma unroll
  for (int p = 0; p < kPer; ++p) out[lane + 32 * p] = o[p] * inv;
}

}  // namespace

cudaError_t launch_gemm_simt_f32(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((g.N + kBN - 1) / kBN),
                  static_cast<unsigned>((g.M + kBM - 1) / kBM));
  TG_CUDA_TRY(launch_pdl(gemm_f32, dim3(grid), dim3(256), 0, st, g));
  return cudaGetLastError();
}

cudaError_t launch_attn_simt_f32(const AttnArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const int64_t items = a.T * a.hq;
  const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
  // fp32 v is [T, hkv, dh] unless the caller passes a wider row in t_pad
  const int64_t v_stride = a.t_pad > 0 ? a.t_pad : static_cast<int64_t>(a.hkv) * a.dh;
  if (a.dh == 128) TG_CUDA_TRY(launch_pdl(attn_f32<128>, dim3(blocks), dim3(256), 0, st, a, v_stride));
  else TG_CUDA_TRY(launch_pdl(attn_f32<64>, dim3(blocks), dim3(256), 0, st, a, v_stride));
  return cudaGetLastError();
}

}  // namespace tg
