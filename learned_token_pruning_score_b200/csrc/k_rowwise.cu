// k_rowwise.cu -- row-wise kernels around the GEMMs and the attention:
// RMSNorm, RoPE (with optional per-head qk-norm) at original positions, the
// V-tile transpose feeding the tensor-core attention, the per-key gate bias
// logsigmoid(s_j), and two fp32 helpers of the SIMT path.
//
// RoPE at the kept tokens' original positions keeps the relative geometry of
// the pruned context (the pages state that kept tokens continue with their
// positions: Tencent Cloud article "TokenGate：端到端可训练的 Token 剪枝机制，
// 让大模型 Prefill 提速 11.3 倍", section "TokenGate 提前筛选 Token"). The
// rotate-half pairing and theta_i = base^(-2i/dh) follow the Qwen3 backbone
// the pages evaluate. The angle pos * theta_i is formed and reduced modulo
// 2*pi in double precision before the fp32 sine/cosine: at pos ~1.3e5 an
// fp32 angle would be off by ~1e-2 rad.
#include <algorithm>

#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}
template <typename T>
__device__ __forceinline__ T to_t(float v);
template <>
__device__ __forceinline__ float to_t<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 to_t<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// ---------------------------------------------------------------- RMSNorm
// One warp per row: y = x * rsqrt(mean(x^2) + eps) * gamma.
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_rows(const T* __restrict__ x,
                                                    const float* __restrict__ g, float eps,
                                                    int64_t rows, int d, T* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const T* xr = x + row * d;
  T* yr = y + row * d;
  constexpr int kVec = 16 / sizeof(T);
  float ss = 0.f;
  const bool vec = (d % kVec) == 0;
  if (vec) {
    for (int c = lane * kVec; c < d; c += 32 * kVec) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + c));
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int j = 0; j < kVec; ++j) {
        const float f = to_float(e[j]);
        ss += f * f;
      }
    }
  } else {
    for (int c = lane; c < d; c += 32) {
      const float f = ld_f(xr + c);
      ss += f * f;
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / static_cast<float>(d) + eps);
  if (vec) {
    for (int c = lane * kVec; c < d; c += 32 * kVec) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + c));
      const T* e = reinterpret_cast<const T*>(&u);
      uint4 o;
      T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
      for (int j = 0; j < kVec; ++j) oe[j] = to_t<T>(to_float(e[j]) * r * __ldg(g + c + j));
      *reinterpret_cast<uint4*>(yr + c) = o;
    }
  } else {
    for (int c = lane; c < d; c += 32) yr[c] = to_t<T>(ld_f(xr + c) * r * __ldg(g + c));
  }
}

// bf16 rows of width kVPL * 256: one warp per row, the row held in registers
// (kVPL 16-byte vectors per lane), so it is read from HBM once and all loads
// of a lane are independent.
template <int kVPL>
__global__ void __launch_bounds__(256) rmsnorm_rows_bf16_reg(const __nv_bfloat16* __restrict__ x,
                                                            const float* __restrict__ g, float eps,
                                                            int64_t rows,
                                                            __nv_bfloat16* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  constexpr int kD = kVPL * 256;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * kD);
  uint4 v[kVPL];
#pragma unroll
  for (int i = 0; i < kVPL; ++i) v[i] = __ldcs(xr + lane + 32 * i);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kVPL; ++i) {
    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(e[j]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / static_cast<float>(kD) + eps);
  uint4* yr = reinterpret_cast<uint4*>(y + row * kD);
#pragma unroll
  for (int i = 0; i < kVPL; ++i) {
    const int c = (lane + 32 * i) * 8;  // first element of this vector
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(g + c));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(g + c) + 1);
    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
    const float2 f0 = __bfloat1622float2(e[0]), f1 = __bfloat1622float2(e[1]);
    const float2 f2 = __bfloat1622float2(e[2]), f3 = __bfloat1622float2(e[3]);
    uint4 o;
    o.x = pack_bf16x2(f0.x * r * g0.x, f0.y * r * g0.y);
    o.y = pack_bf16x2(f1.x * r * g0.z, f1.y * r * g0.w);
    o.z = pack_bf16x2(f2.x * r * g1.x, f2.y * r * g1.y);
    o.w = pack_bf16x2(f3.x * r * g1.z, f3.y * r * g1.w);
    yr[lane + 32 * i] = o;
  }
}

// ---------------------------------------------------------------- RoPE + qk-norm
// One CTA (4 warps) per token; cos/sin of this token's position in shared
// memory, then each warp rotates whole heads. Thread 0 also writes the
// token's gate bias logsigmoid(s_t).
template <typename T, int kDh>
__global__ void __launch_bounds__(128) rope_qk(RopePrepArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int kHalf = kDh / 2;
  constexpr int kPairs = kHalf / 32;  // pairs per lane
  __shared__ float s_cos[kHalf], s_sin[kHalf];
  const int64_t t = blockIdx.x;
  const int pos = a.pos ? __ldg(a.pos + t) : static_cast<int>(t);
  if (threadIdx.x < kHalf) {
    const int i = threadIdx.x;
    const float2 cs = rope_cos_sin(pos, i, kDh, a.rope_base);
    s_cos[i] = cs.x;
    s_sin[i] = cs.y;
  }
  if (threadIdx.x == 0 && a.s != nullptr) a.lsig_out[t] = logsigmoid_f(__ldg(a.s + t));
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int heads = a.hq + a.hkv;
  for (int h = warp; h < heads; h += 4) {
    const bool is_q = h < a.hq;
    const int hh = is_q ? h : h - a.hq;
    const T* src = static_cast<const T*>(is_q ? a.q_src : a.k_src) +
                   t * (is_q ? a.q_stride : a.k_stride) + hh * kDh;
    T* dst = static_cast<T*>(is_q ? a.q_out : a.k_out) +
             (t * (is_q ? a.hq : a.hkv) + hh) * kDh;
    const float* nw = is_q ? a.q_norm : a.k_norm;
    float lo[kPairs], hi[kPairs];
    float ss = 0.f;
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
      lo[p] = ld_f(src + lane + 32 * p);
      hi[p] = ld_f(src + lane + 32 * p + kHalf);
      ss += lo[p] * lo[p] + hi[p] * hi[p];
    }
    if (nw != nullptr) {
      const float r = rsqrtf(warp_sum(ss) / static_cast<float>(kDh) + a.eps);
#pragma unroll
      for (int p = 0; p < kPairs; ++p) {
        lo[p] = lo[p] * r * __ldg(nw + lane + 32 * p);
        hi[p] = hi[p] * r * __ldg(nw + lane + 32 * p + kHalf);
      }
    }
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
      const int i = lane + 32 * p;
      const float c = s_cos[i], s = s_sin[i];
      dst[i] = to_t<T>(lo[p] * c - hi[p] * s);
      dst[i + kHalf] = to_t<T>(hi[p] * c + lo[p] * s);
    }
  }
}

// cos/sin of every (position, frequency) pair, built once per set of
// positions and read by the QKV GEMM epilogue of every layer. Frequency-major
// ([half][T]): the epilogue's threads hold consecutive rows, so a warp reads
// 32 consecutive entries of one frequency.
__global__ void rope_table_kernel(const int32_t* __restrict__ pos, int64_t T, int half, int dh,
                                  float rope_base, float2* __restrict__ cs) {
  pdl_trigger();
  pdl_wait();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= T * half) return;
  const int i = static_cast<int>(idx / T);
  const int64_t t = idx % T;
  const int p = pos ? __ldg(pos + t) : static_cast<int>(t);
  cs[idx] = rope_cos_sin(p, i, dh, rope_base);
}

// Gate-bias rows for the attention's extra K-step (see launch_bias_aug).
__global__ void bias_aug_kernel(const float* __restrict__ lsig, int64_t T, uint4* __restrict__ kaug) {
  pdl_trigger();
  pdl_wait();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const float b = __ldg(lsig + t);
  const __nv_bfloat16 hi = __float2bfloat16_rn(b);
  const __nv_bfloat16 lo = __float2bfloat16_rn(b - __bfloat162float(hi));
  __nv_bfloat162 hl;
  hl.x = hi;
  hl.y = lo;
  const uint32_t w = *reinterpret_cast<uint32_t*>(&hl);
  kaug[2 * t] = make_uint4(w, w, 0u, 0u);
  kaug[2 * t + 1] = make_uint4(0u, 0u, 0u, 0u);
}

// ---------------------------------------------------------------- V transpose
// One CTA per (64-token tile, KV head): vT[g][e][t] = v[t][g][e] (zero for
// t >= T), so that the attention's P.V product reads V K-major. Also copies
// v into a [T, hkv, dh] KV-cache buffer when asked.
template <int kDh>
__global__ void __launch_bounds__(256) v_transpose(RopePrepArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int kTile = 64;
  constexpr int kLd = kDh + 8;  // padded row (bf16 elements)
  __shared__ __align__(16) __nv_bfloat16 tile[kTile * kLd];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int g = blockIdx.y;
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(a.v_src);
  __nv_bfloat16* kvv = static_cast<__nv_bfloat16*>(a.kv_v_out);
  constexpr int kVecRow = kDh / 8;  // uint4 per row
  for (int i = threadIdx.x; i < kTile * kVecRow; i += 256) {
    const int r = i / kVecRow, c = i % kVecRow;
    const int64_t t = t0 + r;
    uint4 u = make_uint4(0, 0, 0, 0);
    if (t < a.T) {
      u = __ldg(reinterpret_cast<const uint4*>(v + t * a.v_stride + g * kDh) + c);
      if (kvv) reinterpret_cast<uint4*>(kvv + (t * a.hkv + g) * kDh)[c] = u;
    }
    *reinterpret_cast<uint4*>(&tile[r * kLd + c * 8]) = u;
  }
  __syncthreads();
  __nv_bfloat16* vt = static_cast<__nv_bfloat16*>(a.vT_out) + static_cast<int64_t>(g) * kDh * a.t_pad;
  for (int i = threadIdx.x; i < kDh * (kTile / 8); i += 256) {
    const int e = i / (kTile / 8), c = i % (kTile / 8);
    uint4 o;
    __nv_bfloat16* oe = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
    for (int j = 0; j < 8; ++j) oe[j] = tile[(c * 8 + j) * kLd + e];
    *reinterpret_cast<uint4*>(vt + static_cast<int64_t>(e) * a.t_pad + t0 + c * 8) = o;
  }
}

// fp32 path: plain copy of v into a KV-cache buffer.
__global__ void copy_v_f32(RopePrepArgs a) {
  pdl_trigger();
  pdl_wait();
  const int64_t t = blockIdx.x;
  const float* v = static_cast<const float*>(a.v_src) + t * a.v_stride;
  float* o = static_cast<float*>(a.kv_v_out) + t * a.hkv * a.dh;
  for (int i = threadIdx.x; i < a.hkv * a.dh; i += blockDim.x) o[i] = __ldg(v + i);
}

// ---------------------------------------------------------------- fp32 helpers
__global__ void swiglu_f32(const float* __restrict__ gu, int64_t rows, int inter,
                           float* __restrict__ h) {
  pdl_trigger();
  pdl_wait();
  const int64_t total = rows * inter;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / inter;
    const int j = static_cast<int>(i % inter);
    const float g = gu[r * 2 * inter + j], u = gu[r * 2 * inter + inter + j];
    h[i] = silu_f(g) * u;
  }
}

__global__ void score_dot_f32(const float* __restrict__ hpre, int64_t rows, int f,
                              const float* __restrict__ b1, const float* __restrict__ w2,
                              const float* __restrict__ b2, float* __restrict__ scores) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  float acc = 0.f;
  for (int j = lane; j < f; j += 32) {
    const float h = hpre[row * f + j] + (b1 ? __ldg(b1 + j) : 0.f);
    acc += __ldg(w2 + j) * silu_f(h);
  }
  acc = warp_sum(acc);
  if (lane == 0) scores[row] = acc + (b2 ? __ldg(b2) : 0.f);
}

}  // namespace

// W_g[j, i] = bf16(W[j, i] * g[i]), eight elements per thread (cols % 8 == 0,
// 16-byte aligned) or one.
template <int kVec>
__global__ void __launch_bounds__(256) fold_norm_weight(const __nv_bfloat16* __restrict__ w,
                                                        const float* __restrict__ g, int64_t rows,
                                                        int64_t cols, __nv_bfloat16* __restrict__ out) {
  const int64_t n = rows * cols / kVec;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t c = (i * kVec) % cols;
    if constexpr (kVec == 8) {
      const uint4 u = __ldcs(reinterpret_cast<const uint4*>(w) + i);
      const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&u);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(e[j]);
        ow[j] = pack_bf16x2(f.x * __ldg(g + c + 2 * j), f.y * __ldg(g + c + 2 * j + 1));
      }
      __stcs(reinterpret_cast<uint4*>(out) + i, o);
    } else {
      out[i] = __float2bfloat16_rn(__bfloat162float(w[i]) * __ldg(g + c));
    }
  }
}

cudaError_t launch_fold_norm_weight(const void* w, const float* g, int64_t rows, int64_t cols,
                                    void* out, cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  const bool vec = cols % 8 == 0 &&
                   ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(out)) & 15u) == 0;
  const int64_t work = rows * cols / (vec ? 8 : 1);
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((work + 255) / 256, 148 * 16));
  const auto* wb = static_cast<const __nv_bfloat16*>(w);
  auto* ob = static_cast<__nv_bfloat16*>(out);
  if (vec)
    fold_norm_weight<8><<<blocks, 256, 0, st>>>(wb, g, rows, cols, ob);
  else
    fold_norm_weight<1><<<blocks, 256, 0, st>>>(wb, g, rows, cols, ob);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const void* x, const float* gamma, float eps, int64_t rows, int d,
                           bool bf16, void* y, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  const bool g_al = (reinterpret_cast<uintptr_t>(gamma) & 15u) == 0;
  const bool xy_al = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15u) == 0;
  if (bf16 && g_al && xy_al && d % 256 == 0 && d <= 16 * 256) {
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    auto* yb = static_cast<__nv_bfloat16*>(y);
    switch (d / 256) {
      case 1: TG_CUDA_TRY(launch_pdl(rmsnorm_rows_bf16_reg<1>, dim3(blocks), dim3(256), 0, st, xb, gamma, eps, rows, yb)); break;
      case 2: TG_CUDA_TRY(launch_pdl(rmsnorm_rows_bf16_reg<2>, dim3(blocks), dim3(256), 0, st, xb, gamma, eps, rows, yb)); break;
      case 4: TG_CUDA_TRY(launch_pdl(rmsnorm_rows_bf16_reg<4>, dim3(blocks), dim3(256), 0, st, xb, gamma, eps, rows, yb)); break;
      case 8: TG_CUDA_TRY(launch_pdl(rmsnorm_rows_bf16_reg<8>, dim3(blocks), dim3(256), 0, st, xb, gamma, eps, rows, yb)); break;
      case 16: TG_CUDA_TRY(launch_pdl(rmsnorm_rows_bf16_reg<16>, dim3(blocks), dim3(256), 0, st, xb, gamma, eps, rows, yb)); break;
      default:
        TG_CUDA_TRY(launch_pdl(rmsnorm_rows<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, xb, gamma, eps, rows, d, yb));
    }
    return cudaGetLastError();
  }
  if (bf16)
    TG_CUDA_TRY(launch_pdl(rmsnorm_rows<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x), gamma, eps, rows, d, static_cast<__nv_bfloat16*>(y)));
  else
    TG_CUDA_TRY(launch_pdl(rmsnorm_rows<float>, dim3(blocks), dim3(256), 0, st, static_cast<const float*>(x), gamma, eps, rows, d, static_cast<float*>(y)));
  return cudaGetLastError();
}

cudaError_t launch_rope_prep(const RopePrepArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(a.T);
  if (a.bf16) {
    if (a.dh == 128) TG_CUDA_TRY(launch_pdl(rope_qk<__nv_bfloat16, 128>, dim3(grid), dim3(128), 0, st, a));
    else TG_CUDA_TRY(launch_pdl(rope_qk<__nv_bfloat16, 64>, dim3(grid), dim3(128), 0, st, a));
    if (a.vT_out) {
      const dim3 g2(static_cast<unsigned>(a.t_pad / 64), static_cast<unsigned>(a.hkv));
      if (a.dh == 128) TG_CUDA_TRY(launch_pdl(v_transpose<128>, dim3(g2), dim3(256), 0, st, a));
      else TG_CUDA_TRY(launch_pdl(v_transpose<64>, dim3(g2), dim3(256), 0, st, a));
    }
  } else {
    if (a.dh == 128) TG_CUDA_TRY(launch_pdl(rope_qk<float, 128>, dim3(grid), dim3(128), 0, st, a));
    else TG_CUDA_TRY(launch_pdl(rope_qk<float, 64>, dim3(grid), dim3(128), 0, st, a));
    if (a.kv_v_out) TG_CUDA_TRY(launch_pdl(copy_v_f32, dim3(grid), dim3(128), 0, st, a));
  }
  return cudaGetLastError();
}

cudaError_t launch_rope_table(const int32_t* pos, int64_t T, int dh, float rope_base, float2* cs,
                              cudaStream_t st) {
  const int half = dh / 2;
  const int64_t total = T * half;
  if (total <= 0) return cudaSuccess;
  TG_CUDA_TRY(launch_pdl(rope_table_kernel, dim3(static_cast<unsigned>((total + 255) / 256)), dim3(256), 0, st, pos, T, half, dh, rope_base, cs));
  return cudaGetLastError();
}

// Positions of packed requests (see launch_segment_positions): each thread
// finds its request by a scan of the (at most 64) offsets.
__global__ void segment_positions_kernel(SegRows s, int64_t total, int32_t* __restrict__ pos) {
  pdl_trigger();
  pdl_wait();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  int32_t p = 0;
  for (int b = 0; b < s.count; ++b) {
    const int64_t i = t - s.off[b];
    if (i >= 0 && i < s.len[b]) p = static_cast<int32_t>(i);
  }
  pos[t] = p;
}

cudaError_t launch_segment_positions(const SegRows& s, int64_t total, int32_t* pos,
                                     cudaStream_t st) {
  if (total <= 0) return cudaSuccess;
  TG_CUDA_TRY(launch_pdl(segment_positions_kernel, dim3(static_cast<unsigned>((total + 255) / 256)),
                         dim3(256), 0, st, s, total, pos));
  return cudaGetLastError();
}

cudaError_t launch_bias_aug(const float* lsig, int64_t T, void* kaug, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  TG_CUDA_TRY(launch_pdl(bias_aug_kernel, dim3(static_cast<unsigned>((T + 255) / 256)), dim3(256), 0, st, lsig, T, static_cast<uint4*>(kaug)));
  return cudaGetLastError();
}

cudaError_t launch_swiglu_f32(const float* gu, int64_t rows, int inter, float* h, cudaStream_t st) {
  const int64_t total = rows * inter;
  if (total <= 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, 148 * 16));
  TG_CUDA_TRY(launch_pdl(swiglu_f32, dim3(blocks), dim3(256), 0, st, gu, rows, inter, h));
  return cudaGetLastError();
}

cudaError_t launch_score_dot_f32(const float* hpre, int64_t rows, int f, const float* b1,
                                 const float* w2, const float* b2, float* scores, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  TG_CUDA_TRY(launch_pdl(score_dot_f32, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, st, hpre, rows, f, b1, w2, b2, scores));
  return cudaGetLastError();
}

}  // namespace tg
