// k_decode.cu -- one generated token through the stack (batch 1).
//
// After a gated prefill a generated token runs every layer (generated tokens
// are never pruned) and attends over each layer's cache: the whole prompt at
// and below the gate, the kept tokens above it, plus the tokens generated so
// far. At batch 1 every weight matrix and every cached k/v row is read once
// per token and used for one row of arithmetic, so the step is bound by HBM
// bandwidth and there is nothing for the tensor cores to reuse: these kernels
// stream with 16-byte loads spread over every SM, on the CUDA cores.
//
//   dec_gemv   y = W x, W [n, k] bf16 row-major, fp32 accumulate; one warp per
//              output (two W rows for SwiGLU), x staged in shared memory and
//              optionally RMSNorm'd first (each CTA normalises the short vector
//              itself, which costs less than a launch); epilogues: store,
//              residual add in place, SwiGLU.
//   dec_attn   one query token; a CTA per (key split, KV head) handles the
//              query heads of that KV head's group. Every CTA forms the new
//              token's q and k itself (qk-norm, RoPE at its position); split 0
//              appends k and v to the cache; the last CTA of a KV head to
//              finish merges the splits' softmax states (no inter-CTA waits).
#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kDh = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// 8 bf16 (one 16-byte vector) to fp32.
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(e[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ float dot8(const uint4& w, const uint4& x) {
  float a[8], b[8];
  unpack8(w, a);
  unpack8(x, b);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s = fmaf(a[i], b[i], s);
  return s;
}

// Streaming 16-byte load (read once per step; evict first from L2).
__device__ __forceinline__ uint4 ld_stream(const uint4* p) { return __ldcs(p); }

// ---------------------------------------------------------------- GEMV
constexpr int kGemvWarps = 8;

template <int kEpi, bool kNorm>
__global__ void __launch_bounds__(kGemvWarps * 32) dec_gemv(DecGemvArgs a) {
  extern __shared__ __align__(16) uint8_t dyn_smem[];
  uint4* xs = reinterpret_cast<uint4*>(dyn_smem);  // x (normalised if kNorm), bf16 [k]
  __shared__ float red[kGemvWarps];
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nv = a.k / 8;  // 16-byte vectors per row
  const uint4* xg = reinterpret_cast<const uint4*>(a.x);
  if (kNorm) {
    float ss = 0.f;
    for (int v = tid; v < nv; v += kGemvWarps * 32) {
      float f[8];
      unpack8(xg[v], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
    }
    ss = warp_sum32(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) tot += red[w];
    const float r = rsqrtf(tot / static_cast<float>(a.k) + a.eps);
    for (int v = tid; v < nv; v += kGemvWarps * 32) {
      float f[8];
      unpack8(xg[v], f);
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma) + 2 * v);
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma) + 2 * v + 1);
      uint4 o;
      o.x = pack_bf16x2(f[0] * r * g0.x, f[1] * r * g0.y);
      o.y = pack_bf16x2(f[2] * r * g0.z, f[3] * r * g0.w);
      o.z = pack_bf16x2(f[4] * r * g1.x, f[5] * r * g1.y);
      o.w = pack_bf16x2(f[6] * r * g1.z, f[7] * r * g1.w);
      xs[v] = o;
    }
  } else {
    for (int v = tid; v < nv; v += kGemvWarps * 32) xs[v] = xg[v];
  }
  __syncthreads();
  const int row = blockIdx.x * kGemvWarps + warp;
  if (row >= a.n_out) return;
  const uint4* w0 = reinterpret_cast<const uint4*>(a.w) + static_cast<int64_t>(row) * nv;
  const uint4* w1 = kEpi == DEC_EPI_SWIGLU
                        ? reinterpret_cast<const uint4*>(a.w) + static_cast<int64_t>(a.inter + row) * nv
                        : w0;
  float acc0 = 0.f, acc1 = 0.f;
  int v = lane;
  // eight vectors per lane in flight per pass
  for (; v + 32 * 7 < nv; v += 32 * 8) {
    uint4 wa[8], wb[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      wa[u] = ld_stream(w0 + v + 32 * u);
      if (kEpi == DEC_EPI_SWIGLU) wb[u] = ld_stream(w1 + v + 32 * u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint4 xv = xs[v + 32 * u];
      acc0 += dot8(wa[u], xv);
      if (kEpi == DEC_EPI_SWIGLU) acc1 += dot8(wb[u], xv);
    }
  }
  for (; v < nv; v += 32) {
    const uint4 xv = xs[v];
    acc0 += dot8(ld_stream(w0 + v), xv);
    if (kEpi == DEC_EPI_SWIGLU) acc1 += dot8(ld_stream(w1 + v), xv);
  }
  acc0 = warp_sum32(acc0);
  if (kEpi == DEC_EPI_SWIGLU) acc1 = warp_sum32(acc1);
  if (lane == 0) {
    if (kEpi == DEC_EPI_STORE) {
      a.y[row] = __float2bfloat16_rn(acc0);
    } else if (kEpi == DEC_EPI_RESIDUAL) {
      a.y[row] = __float2bfloat16_rn(__bfloat162float(a.y[row]) + acc0);
    } else {
      a.y[row] = __float2bfloat16_rn(silu_f(acc0) * acc1);
    }
  }
}

// ---------------------------------------------------------------- attention
constexpr int kAttnThreads = 128;      // 4 warps = 8 half-warps, one key per half-warp
constexpr int kHalfWarps = kAttnThreads / 16;
static_assert(kAttnThreads == kDh, "one thread per head-dim element in the merges");
constexpr int kKeysInFlight = 4;       // keys loaded ahead per half-warp

template <int kGroup>
__global__ void __launch_bounds__(kAttnThreads) dec_attn(DecAttnArgs a) {
  __shared__ float qs[kGroup][kDh];                    // rotated q (bf16-rounded values)
  __shared__ __align__(16) __nv_bfloat16 kv_new[2][kDh];  // the new token's k (rotated), v
  __shared__ float red_m[kHalfWarps][kGroup], red_l[kHalfWarps][kGroup];
  __shared__ float red_o[kHalfWarps][kGroup][kDh];
  __shared__ float cta_m[kGroup], cta_l[kGroup];
  __shared__ int is_last;
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = blockIdx.y, split = blockIdx.x, n_split = gridDim.x;
  const int head0 = g * kGroup;

  // 1. The new token's q (the group's heads) and k: qk-norm, RoPE at pos,
  //    rounded as the prefill stores them; v as projected.
  for (int r = warp; r <= kGroup; r += kAttnThreads / 32) {
    const bool is_q = r < kGroup;
    const __nv_bfloat16* src = a.qkv + (is_q ? (head0 + r) : (a.hq + g)) * kDh;
    const float* nw = is_q ? a.q_norm : a.k_norm;
    float lo[2], hi[2], ss = 0.f;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      lo[p] = __bfloat162float(src[lane + 32 * p]);
      hi[p] = __bfloat162float(src[lane + 32 * p + kDh / 2]);
      ss += lo[p] * lo[p] + hi[p] * hi[p];
    }
    if (nw != nullptr) {
      const float rs = rsqrtf(warp_sum32(ss) / static_cast<float>(kDh) + a.eps);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        lo[p] = lo[p] * rs * __ldg(nw + lane + 32 * p);
        hi[p] = hi[p] * rs * __ldg(nw + lane + 32 * p + kDh / 2);
      }
    }
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int i = lane + 32 * p;
      const float2 cs = rope_cos_sin(a.pos, i, kDh, a.rope_base);
      const __nv_bfloat16 olo = __float2bfloat16_rn(lo[p] * cs.x - hi[p] * cs.y);
      const __nv_bfloat16 ohi = __float2bfloat16_rn(hi[p] * cs.x + lo[p] * cs.y);
      if (is_q) {
        qs[r][i] = __bfloat162float(olo);
        qs[r][i + kDh / 2] = __bfloat162float(ohi);
      } else {
        kv_new[0][i] = olo;
        kv_new[0][i + kDh / 2] = ohi;
      }
    }
  }
  kv_new[1][tid] = a.qkv[(a.hq + a.hkv + g) * kDh + tid];
  __syncthreads();

  // 2. Split 0 appends the new row to the cache (no CTA reads that row from
  //    memory in this launch: the split holding it takes it from shared).
  const int64_t len = a.len;
  if (split == 0) {
    a.k_cache[(len * a.hkv + g) * kDh + tid] = kv_new[0][tid];
    a.v_cache[(len * a.hkv + g) * kDh + tid] = kv_new[1][tid];
  }

  // 3. This split's keys: rows [c0, c1) of the cache rows 0..len (row len is
  //    the new token). One half-warp per key, 8 elements per lane.
  const int64_t total = len + 1;
  const int64_t per = (total + n_split - 1) / n_split;
  const int64_t c0 = static_cast<int64_t>(split) * per;
  const int64_t c1 = c0 + per < total ? c0 + per : total;
  const int hw = tid >> 4, sub = lane & 15;
  // the two half-warps of a warp run different keys (and trip counts)
  const unsigned half_mask = 0xFFFFu << (lane & 16);
  float qr[kGroup][8], sc[kGroup], bc[kGroup], m[kGroup], l[kGroup], o[kGroup][8];
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
#pragma unroll
    for (int e = 0; e < 8; ++e) qr[h][e] = qs[h][sub * 8 + e];
    const float tau = a.tau ? __ldg(a.tau + head0 + h) : 1.0f;
    sc[h] = kLog2e / (sqrtf(static_cast<float>(kDh)) * tau);
    bc[h] = a.gain ? __ldg(a.gain + head0 + h) * kLog2e : 0.f;
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
  }
  const uint4* knew4 = reinterpret_cast<const uint4*>(kv_new[0]);
  const uint4* vnew4 = reinterpret_cast<const uint4*>(kv_new[1]);
  for (int64_t jb = c0 + hw; jb < c1; jb += kHalfWarps * kKeysInFlight) {
    uint4 kk[kKeysInFlight], vv[kKeysInFlight];
    float bias[kKeysInFlight];
#pragma unroll
    for (int u = 0; u < kKeysInFlight; ++u) {
      const int64_t j = jb + static_cast<int64_t>(u) * kHalfWarps;
      bias[u] = 0.f;
      if (j < len) {
        const int64_t off = ((j * a.hkv + g) * kDh) / 8 + sub;
        kk[u] = ld_stream(reinterpret_cast<const uint4*>(a.k_cache) + off);
        vv[u] = ld_stream(reinterpret_cast<const uint4*>(a.v_cache) + off);
        if (a.lsig != nullptr && j < a.k_kept) bias[u] = __ldg(a.lsig + j);
      } else {
        kk[u] = knew4[sub];
        vv[u] = vnew4[sub];
      }
    }
#pragma unroll
    for (int u = 0; u < kKeysInFlight; ++u) {
      const int64_t j = jb + static_cast<int64_t>(u) * kHalfWarps;
      if (j >= c1) continue;  // uniform within the half-warp
      float kf[8], vf[8];
      unpack8(kk[u], kf);
      unpack8(vv[u], vf);
#pragma unroll
      for (int h = 0; h < kGroup; ++h) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) d = fmaf(qr[h][e], kf[e], d);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) d += __shfl_xor_sync(half_mask, d, off);
        const float s = d * sc[h] + bc[h] * bias[u];  // log2 domain
        const float mn = fmaxf(m[h], s);
        const float base = mn == -INFINITY ? 0.f : mn;
        const float al = ex2_approx(m[h] - base);
        const float p = ex2_approx(s - base);
        l[h] = l[h] * al + p;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = fmaf(o[h][e], al, p * vf[e]);
        m[h] = mn;
      }
    }
  }

  // 4. Merge the 8 half-warps.
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
    if (sub == 0) {
      red_m[hw][h] = m[h];
      red_l[hw][h] = l[h];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red_o[hw][h][sub * 8 + e] = o[h][e];
  }
  __syncthreads();
  if (tid < kGroup) {
    float mx = -INFINITY;
    for (int w = 0; w < kHalfWarps; ++w) mx = fmaxf(mx, red_m[w][tid]);
    const float base = mx == -INFINITY ? 0.f : mx;
    float ls = 0.f;
    for (int w = 0; w < kHalfWarps; ++w) ls += red_l[w][tid] * ex2_approx(red_m[w][tid] - base);
    cta_m[tid] = mx;
    cta_l[tid] = ls;
  }
  __syncthreads();
  float* part = a.part + (static_cast<int64_t>(g) * a.max_split + split) * kGroup * (kDh + 2);
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
    const float mx = cta_m[h];
    const float base = mx == -INFINITY ? 0.f : mx;
    float acc = 0.f;
    for (int w = 0; w < kHalfWarps; ++w) acc += red_o[w][h][tid] * ex2_approx(red_m[w][h] - base);
    part[h * (kDh + 2) + 2 + tid] = acc;
    if (tid == 0) {
      part[h * (kDh + 2)] = mx;
      part[h * (kDh + 2) + 1] = cta_l[h];
    }
  }

  // 5. The last split of this KV head merges every split's state.
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(a.counters + g, 1u) == static_cast<unsigned>(n_split - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const float* base_part = a.part + static_cast<int64_t>(g) * a.max_split * kGroup * (kDh + 2);
#pragma unroll 1
  for (int h = 0; h < kGroup; ++h) {
    float mx = -INFINITY;
    for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, __ldcg(base_part + (s * kGroup + h) * (kDh + 2)));
    const float base = mx == -INFINITY ? 0.f : mx;
    float ls = 0.f, acc = 0.f;
    for (int s = 0; s < n_split; ++s) {
      const float* ps = base_part + (s * kGroup + h) * (kDh + 2);
      const float w = ex2_approx(__ldcg(ps) - base);
      ls += __ldcg(ps + 1) * w;
      acc += __ldcg(ps + 2 + tid) * w;
    }
    a.out[(head0 + h) * kDh + tid] = __float2bfloat16_rn(acc / ls);
  }
  if (tid == 0) a.counters[g] = 0u;  // ready for the next layer's launch
}

// logsigmoid of the kept prompt tokens' scores (the decode bias inputs).
// An index outside [0, n) gets no bias and sets bit 2 of the error word.
__global__ void dec_lsig(const float* __restrict__ scores, int64_t n,
                         const int32_t* __restrict__ kept_idx, int64_t k, float* __restrict__ lsig,
                         unsigned int* err) {
  pdl_trigger();
  pdl_wait();
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= k) return;
  const int32_t i = __ldg(kept_idx + j);
  if (i < 0 || i >= n) {
    report_error(err, kErrIndexRange);
    lsig[j] = 0.f;
    return;
  }
  lsig[j] = logsigmoid_f(__ldg(scores + i));
}

}  // namespace

int decode_splits(int64_t rows, int hkv) {
  const int64_t want = (2 * int64_t(num_sms()) + hkv - 1) / hkv;
  const int64_t by_len = (rows + 63) / 64;  // at least ~64 keys per CTA
  int64_t s = want < by_len ? want : by_len;
  if (s < 1) s = 1;
  if (s > kDecodeMaxSplits) s = kDecodeMaxSplits;
  return static_cast<int>(s);
}

cudaError_t launch_decode_gemv(const DecGemvArgs& a, int epi, bool norm, cudaStream_t st) {
  if (a.n_out <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((a.n_out + kGemvWarps - 1) / kGemvWarps));
  const dim3 block(kGemvWarps * 32);
  const size_t smem = static_cast<size_t>(a.k) * 2;
  if (epi == DEC_EPI_STORE)
    return norm ? launch_pdl(dec_gemv<DEC_EPI_STORE, true>, grid, block, smem, st, a)
                : launch_pdl(dec_gemv<DEC_EPI_STORE, false>, grid, block, smem, st, a);
  if (epi == DEC_EPI_RESIDUAL)
    return norm ? launch_pdl(dec_gemv<DEC_EPI_RESIDUAL, true>, grid, block, smem, st, a)
                : launch_pdl(dec_gemv<DEC_EPI_RESIDUAL, false>, grid, block, smem, st, a);
  return norm ? launch_pdl(dec_gemv<DEC_EPI_SWIGLU, true>, grid, block, smem, st, a)
              : launch_pdl(dec_gemv<DEC_EPI_SWIGLU, false>, grid, block, smem, st, a);
}

cudaError_t launch_decode_attn(const DecAttnArgs& a, int n_split, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(n_split), static_cast<unsigned>(a.hkv));
  const dim3 block(kAttnThreads);
  switch (a.hq / a.hkv) {
    case 1: return launch_pdl(dec_attn<1>, grid, block, 0, st, a);
    case 2: return launch_pdl(dec_attn<2>, grid, block, 0, st, a);
    case 4: return launch_pdl(dec_attn<4>, grid, block, 0, st, a);
    case 8: return launch_pdl(dec_attn<8>, grid, block, 0, st, a);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_lsig(const float* scores, int64_t n, const int32_t* kept_idx, int64_t k,
                               float* lsig, cudaStream_t st) {
  if (k <= 0) return cudaSuccess;
  return launch_pdl(dec_lsig, dim3(static_cast<unsigned>((k + 255) / 256)), dim3(256), 0, st,
                    scores, n, kept_idx, k, lsig, device_error_word());
}

}  // namespace tg
