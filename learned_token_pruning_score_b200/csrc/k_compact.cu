// k_compact.cu -- gather of the kept rows, their original positions and scores.
//
// Only the kept tokens continue into the layers above the gate, and they
// keep their original positions (Tencent Cloud article "TokenGate：端到端可训练的
// Token 剪枝机制，让大模型 Prefill 提速 11.3 倍", section "TokenGate 提前筛选
// Token"; farwalk.ai item on TokenGate, section "论文的方法").
//
// HBM-bound copy: one warp per kept row, 16-byte vector loads/stores with
// several independent transactions in flight per lane; streaming cache hints
// (the source rows are read once, the output is consumed by the next kernel).
// With a folded RMSNorm the rows' sums of squares travel with them.
#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kWarps * 32) compact_rows(
    const uint4* __restrict__ x, const int32_t* __restrict__ pos_in,
    const float* __restrict__ scores, const int32_t* __restrict__ idx, int64_t n, int64_t k,
    int vec_per_row, uint4* __restrict__ x_out, int32_t* __restrict__ pos_out,
    float* __restrict__ s_out, float* __restrict__ lsig_out, SsGather ss, unsigned int* err) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (row >= k) return;
  const int32_t src = __ldg(idx + row);
  const bool ok = src >= 0 && src < n;
  if (!ok && lane == 0) report_error(err, kErrIndexRange);
  const uint4* s = x + static_cast<int64_t>(ok ? src : 0) * vec_per_row;
  uint4* d = x_out + row * vec_per_row;
  int c = lane;
  for (; c + 32 * (kUnroll - 1) < vec_per_row; c += 32 * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = ok ? __ldcs(s + c + 32 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) __stcg(d + c + 32 * u, v[u]);
  }
  for (; c < vec_per_row; c += 32) __stcg(d + c, ok ? __ldcs(s + c) : make_uint4(0, 0, 0, 0));
  if (lane == 0) {
    pos_out[row] = ok ? (pos_in ? __ldg(pos_in + src) : src) : 0;
    if (scores) {
      const float sv = ok ? __ldg(scores + src) : 0.0f;
      if (s_out) s_out[row] = sv;
      if (lsig_out) lsig_out[row] = logsigmoid_f(sv);
    }
  }
  if (ss.out != nullptr && lane < ss.parts)
    ss.out[lane * ss.ld_out + row] = ok ? __ldg(ss.in + lane * ss.ld_in + src) : 0.0f;
}

}  // namespace

cudaError_t launch_compact(const void* x, const int32_t* pos_in, const float* scores,
                           const int32_t* kept_idx, int64_t n, int64_t k, int row_bytes,
                           void* x_out, int32_t* pos_out, float* scores_out, float* lsig_out,
                           const SsGather& ss, cudaStream_t st) {
  if (k <= 0) return cudaSuccess;
  if (ss.out != nullptr && (ss.in == nullptr || ss.parts < 1 || ss.parts > 32))
    return cudaErrorInvalidValue;
  const int64_t blocks = (k + kWarps - 1) / kWarps;
  TG_CUDA_TRY(launch_pdl(compact_rows, dim3(static_cast<unsigned>(blocks)), dim3(kWarps * 32), 0, st, static_cast<const uint4*>(x), pos_in, scores, kept_idx, n, k, row_bytes / 16, static_cast<uint4*>(x_out), pos_out, scores_out, lsig_out, ss, device_error_word()));
  return cudaGetLastError();
}

}  // namespace tg
