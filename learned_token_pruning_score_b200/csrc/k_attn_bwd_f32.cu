// k_attn_bwd_f32.cu -- backward of the token-gated causal GQA attention in
// fp32 on the CUDA cores (the fp32 path of the library: head_dim 64 or 128).
// The same gradients as the tensor-core backward (k_attn_bwd.cu):
//   P_ij = exp(l_ij - lse_i), dl_ij = P_ij (dout_i . v_j - dout_i . o_i)
//   dq_i = sum_j dl_ij k_j / (sqrt(dh) tau_h), dk_j = sum_h sum_i dl_ij q_i / (sqrt(dh) tau_h)
//   dv_j = sum_h sum_i P_ij dout_i, C_hj = sum_i dl_ij
// with q and k rotated by RoPE before the logits and their gradients rotated
// back. One warp per (query row, query head) for dq and q . dq, one warp per
// (key row, KV head) for dk, dv and C; lanes split the head dimension, and
// every sum runs in a fixed order (deterministic).
#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

template <int kDh>
__device__ __forceinline__ float warp_dot(const float (&a)[kDh / 32], const float* b, int lane) {
  float d = 0.f;
#pragma unroll
  for (int p = 0; p < kDh / 32; ++p) d = fmaf(a[p], __ldg(b + lane + 32 * p), d);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xFFFFFFFFu, d, off);
  return d;
}

// Rotates a gradient row (lanes own elements lane + 32 p) back through RoPE:
// pairs (e, e + dh/2) sit in the same lane at p and p + kPer/2.
template <int kDh>
__device__ __forceinline__ void rope_back_lanes(float (&x)[kDh / 32], const float2* cs, int64_t T,
                                                int64_t row, int lane) {
  constexpr int kHalf = kDh / 64;
#pragma unroll
  for (int p = 0; p < kHalf; ++p) {
    const float2 c = __ldg(cs + static_cast<int64_t>(lane + 32 * p) * T + row);
    const float a = x[p], b = x[p + kHalf];
    x[p] = a * c.x + b * c.y;
    x[p + kHalf] = b * c.x - a * c.y;
  }
}

template <int kDh>
__global__ void __launch_bounds__(256) attn_bwd_q_f32(AttnBwdF32Args a) {
  pdl_trigger();
  pdl_wait();
  constexpr int kPer = kDh / 32;
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= a.T * a.hq) return;
  const int64_t i = item / a.hq;
  const int h = static_cast<int>(item % a.hq);
  const int g = h / (a.hq / a.hkv);
  const float tau = a.tau ? __ldg(a.tau + h) : 1.0f;
  const float gain = a.gain ? __ldg(a.gain + h) : 0.0f;
  const float c = 1.0f / (sqrtf(static_cast<float>(kDh)) * tau);
  const float lse = __ldg(a.lse + static_cast<int64_t>(h) * a.T + i);
  float q[kPer], go[kPer], dq[kPer];
  float di = 0.f;
#pragma unroll
  for (int p = 0; p < kPer; ++p) {
    q[p] = __ldg(a.q_rot + (i * a.hq + h) * kDh + lane + 32 * p);
    go[p] = __ldg(a.dout + (i * a.hq + h) * kDh + lane + 32 * p);
    di = fmaf(go[p], __ldg(a.out + (i * a.hq + h) * kDh + lane + 32 * p), di);
    dq[p] = 0.f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) di += __shfl_xor_sync(0xFFFFFFFFu, di, off);
  for (int64_t j = 0; j <= i; ++j) {
    const float* kr = a.k_rot + (j * a.hkv + g) * kDh;
    const float s = warp_dot<kDh>(q, kr, lane);
    const float pr = expf(s * c + (a.lsig ? gain * __ldg(a.lsig + j) : 0.f) - lse);
    const float dp = warp_dot<kDh>(go, a.v + (j * a.hkv + g) * kDh, lane);
    const float dl = pr * (dp - di);
#pragma unroll
    for (int p = 0; p < kPer; ++p) dq[p] = fmaf(dl, __ldg(kr + lane + 32 * p), dq[p]);
  }
  float qd = 0.f;
#pragma unroll
  for (int p = 0; p < kPer; ++p) {
    dq[p] *= c;
    qd = fmaf(q[p], dq[p], qd);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) qd += __shfl_xor_sync(0xFFFFFFFFu, qd, off);
  if (lane == 0) a.qdq[static_cast<int64_t>(h) * a.T + i] = qd;
  rope_back_lanes<kDh>(dq, a.cs, a.T, i, lane);
#pragma unroll
  for (int p = 0; p < kPer; ++p) a.dq[(i * a.hq + h) * kDh + lane + 32 * p] = dq[p];
}

template <int kDh>
__global__ void __launch_bounds__(256) attn_bwd_kv_f32(AttnBwdF32Args a) {
  pdl_trigger();
  pdl_wait();
  constexpr int kPer = kDh / 32;
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= a.T * a.hkv) return;
  const int64_t j = item / a.hkv;
  const int g = static_cast<int>(item % a.hkv);
  const int group = a.hq / a.hkv;
  float k[kPer], v[kPer], dk[kPer], dv[kPer];
#pragma unroll
  for (int p = 0; p < kPer; ++p) {
    k[p] = __ldg(a.k_rot + (j * a.hkv + g) * kDh + lane + 32 * p);
    v[p] = __ldg(a.v + (j * a.hkv + g) * kDh + lane + 32 * p);
    dk[p] = 0.f;
    dv[p] = 0.f;
  }
  const float bj = a.lsig ? __ldg(a.lsig + j) : 0.f;
  for (int hh = 0; hh < group; ++hh) {
    const int h = g * group + hh;
    const float tau = a.tau ? __ldg(a.tau + h) : 1.0f;
    const float gain = a.gain ? __ldg(a.gain + h) : 0.0f;
    const float c = 1.0f / (sqrtf(static_cast<float>(kDh)) * tau);
    float csum = 0.f;
    for (int64_t i = j; i < a.T; ++i) {
      const float* qr = a.q_rot + (i * a.hq + h) * kDh;
      const float* gr = a.dout + (i * a.hq + h) * kDh;
      const float s = warp_dot<kDh>(k, qr, lane);
      const float pr = expf(s * c + gain * bj - __ldg(a.lse + static_cast<int64_t>(h) * a.T + i));
      const float dp = warp_dot<kDh>(v, gr, lane);
      // D_i = dout_i . o_i
      float di = 0.f;
#pragma unroll
      for (int p = 0; p < kPer; ++p)
        di = fmaf(__ldg(gr + lane + 32 * p), __ldg(a.out + (i * a.hq + h) * kDh + lane + 32 * p),
                  di);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) di += __shfl_xor_sync(0xFFFFFFFFu, di, off);
      const float dl = pr * (dp - di);
      csum += dl;
#pragma unroll
      for (int p = 0; p < kPer; ++p) {
        dk[p] = fmaf(c * dl, __ldg(qr + lane + 32 * p), dk[p]);
        dv[p] = fmaf(pr, __ldg(gr + lane + 32 * p), dv[p]);
      }
    }
    if (a.colsum && lane == 0) {
      a.colsum[static_cast<int64_t>(h) * a.t_pad + j] = csum;
      a.colsum[static_cast<int64_t>(a.hq + h) * a.t_pad + j] = 0.f;
    }
  }
  rope_back_lanes<kDh>(dk, a.cs, a.T, j, lane);
#pragma unroll
  for (int p = 0; p < kPer; ++p) {
    a.dk[(j * a.hkv + g) * kDh + lane + 32 * p] = dk[p];
    a.dv[(j * a.hkv + g) * kDh + lane + 32 * p] = dv[p];
  }
}

}  // namespace

cudaError_t launch_attn_bwd_f32(const AttnBwdF32Args& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const unsigned bq = static_cast<unsigned>((a.T * a.hq + 7) / 8);
  const unsigned bk = static_cast<unsigned>((a.T * a.hkv + 7) / 8);
  if (a.dh == 128) {
    TG_CUDA_TRY(launch_pdl(attn_bwd_q_f32<128>, dim3(bq), dim3(256), 0, st, a));
    TG_CUDA_TRY(launch_pdl(attn_bwd_kv_f32<128>, dim3(bk), dim3(256), 0, st, a));
  } else {
    TG_CUDA_TRY(launch_pdl(attn_bwd_q_f32<64>, dim3(bq), dim3(256), 0, st, a));
    TG_CUDA_TRY(launch_pdl(attn_bwd_kv_f32<64>, dim3(bk), dim3(256), 0, st, a));
  }
  return cudaGetLastError();
}

}  // namespace tg
