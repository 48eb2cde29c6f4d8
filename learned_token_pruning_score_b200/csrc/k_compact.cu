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
#include <algorithm>

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
    float* __restrict__ s_out, float* __restrict__ lsig_out, unsigned int* err) {
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
}

// Bulk-copy form for rows of at most kBulkMaxRow bytes. One thread per CTA
// streams the CTA's rows (r = blockIdx.x + i * gridDim.x) through a ring of
// kSlots shared-memory slots: the row is loaded by cp.async.bulk (completion
// counted on the slot's mbarrier), then stored by a bulk copy kLead rows
// later; a slot is reused once its previous store has read it. A row whose
// index is out of range is stored as zeros (and reported). The other
// threads write the rows' positions, scores and logsigmoids.
constexpr int kSlots = 8;
constexpr int kLead = 4;
constexpr int kBulkMaxRow = 8192;
constexpr int kBulkThreads = 128;

__global__ void __launch_bounds__(kBulkThreads) compact_rows_bulk(
    const uint8_t* __restrict__ x, const int32_t* __restrict__ pos_in,
    const float* __restrict__ scores, const int32_t* __restrict__ idx, int64_t n, int64_t k,
    int row_bytes, uint8_t* __restrict__ x_out, int32_t* __restrict__ pos_out,
    float* __restrict__ s_out, float* __restrict__ lsig_out, unsigned int* err) {
  extern __shared__ __align__(128) uint8_t slots[];  // kSlots x row_bytes
  __shared__ __align__(8) uint64_t full[kSlots];
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  const int64_t first = blockIdx.x, step = gridDim.x;
  const int64_t mine = first < k ? (k - first + step - 1) / step : 0;
  if (threadIdx.x == 0) {
    auto store_row = [&](int64_t i) {
      const int s = static_cast<int>(i % kSlots);
      if (!mbar_wait(&full[s], static_cast<uint32_t>((i / kSlots) & 1), err)) return false;
      bulk_store(x_out + (first + i * step) * static_cast<int64_t>(row_bytes),
                 slots + static_cast<size_t>(s) * row_bytes, static_cast<uint32_t>(row_bytes));
      bulk_commit();
      return true;
    };
    bool ok = true;
    for (int64_t i = 0; i < mine && ok; ++i) {
      const int s = static_cast<int>(i % kSlots);
      // slot s last held row i - kSlots, stored at step i - kSlots + kLead;
      // since then kSlots - kLead - 1 more stores were committed
      if (i >= kSlots) bulk_wait_read<kSlots - kLead - 1>();
      const int32_t src = __ldg(idx + first + i * step);
      uint8_t* slot = slots + static_cast<size_t>(s) * row_bytes;
      if (src >= 0 && src < n) {
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(row_bytes));
        bulk_load(slot, x + static_cast<int64_t>(src) * row_bytes, static_cast<uint32_t>(row_bytes),
                  &full[s]);
      } else {
        report_error(err, kErrIndexRange);
        for (int b = 0; b < row_bytes; b += 16)
          *reinterpret_cast<uint4*>(slot + b) = make_uint4(0u, 0u, 0u, 0u);
        fence_async_smem();
        mbar_arrive(&full[s]);
      }
      if (i >= kLead) ok = store_row(i - kLead);
    }
    for (int64_t i = mine > kLead ? mine - kLead : 0; i < mine && ok; ++i) ok = store_row(i);
    bulk_wait_read<0>();  // the slots stay valid until every store has read them
  } else {
    for (int64_t i = threadIdx.x - 1; i < mine; i += kBulkThreads - 1) {
      const int64_t row = first + i * step;
      const int32_t src = __ldg(idx + row);
      const bool ok = src >= 0 && src < n;
      pos_out[row] = ok ? (pos_in ? __ldg(pos_in + src) : src) : 0;
      if (scores) {
        const float sv = ok ? __ldg(scores + src) : 0.0f;
        if (s_out) s_out[row] = sv;
        if (lsig_out) lsig_out[row] = logsigmoid_f(sv);
      }
    }
  }
}

}  // namespace

cudaError_t launch_compact(const void* x, const int32_t* pos_in, const float* scores,
                           const int32_t* kept_idx, int64_t n, int64_t k, int row_bytes,
                           void* x_out, int32_t* pos_out, float* scores_out, float* lsig_out,
                           cudaStream_t st) {
  if (k <= 0) return cudaSuccess;
  if (row_bytes <= kBulkMaxRow && row_bytes % 16 == 0) {
    const size_t smem = static_cast<size_t>(kSlots) * row_bytes;
    TG_CUDA_TRY(set_smem_attr_once(reinterpret_cast<const void*>(compact_rows_bulk),
                                   static_cast<int>(smem)));
    const int64_t blocks = std::min<int64_t>(k, int64_t(num_sms()) * 4);
    TG_CUDA_TRY(launch_pdl(compact_rows_bulk, dim3(static_cast<unsigned>(blocks)),
                           dim3(kBulkThreads), smem, st, static_cast<const uint8_t*>(x), pos_in,
                           scores, kept_idx, n, k, row_bytes, static_cast<uint8_t*>(x_out),
                           pos_out, scores_out, lsig_out, device_error_word()));
    return cudaGetLastError();
  }
  const int64_t blocks = (k + kWarps - 1) / kWarps;
  TG_CUDA_TRY(launch_pdl(compact_rows, dim3(static_cast<unsigned>(blocks)), dim3(kWarps * 32), 0, st, static_cast<const uint4*>(x), pos_in, scores, kept_idx, n, k, row_bytes / 16, static_cast<uint4*>(x_out), pos_out, scores_out, lsig_out, device_error_word()));
  return cudaGetLastError();
}

}  // namespace tg
