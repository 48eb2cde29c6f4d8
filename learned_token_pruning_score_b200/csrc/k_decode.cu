// k_decode.cu -- one generated token through the stack (batch 1).
//
// After a gated prefill a generated token runs every layer (generated tokens
// are never pruned) and attends over each layer's cache: the whole prompt at
// and below the gate, the kept tokens above it, plus the tokens generated so
// far. At batch 1 every weight matrix and every cached k/v row is read once
// per token and used for one row of arithmetic, so the step is bound by HBM
// bandwidth and there is nothing for the tensor cores to reuse: the work is
// streamed with 16-byte loads spread over every SM, on the CUDA cores.
//
// One cooperative, persistent kernel runs the whole step (one CTA per SM).
// Per layer it walks five stages separated by grid barriers:
//   QKV        y = W_qkv RMSNorm(h)          (matrix-vector, rows over all warps)
//   attention  one query token; a CTA per (KV head, key split) handles the
//              query heads of that KV head; every CTA forms the token's q and
//              k itself (qk-norm, RoPE at its position); split 0 appends k, v
//              to the cache; the last split of a KV head merges the splits'
//              softmax states
//   O          h += W_o o
//   gate/up    a = SiLU(W_g y) * (W_u y), y = RMSNorm(h)
//   down       h += W_d a
// Between arriving at a barrier and waiting on it, every warp already loads
// its first weight chunk of the next stage (weights never change), so the
// weight stream overlaps the barrier. Separate launches cost ~9 us each at
// this size (launch, ramp-up, tail), more than most stages' own traffic.
// Every barrier wait is bounded; a timeout sets the error word and an abort
// flag that makes every CTA leave at its next barrier.
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

// ---------------------------------------------------------------- barrier
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid barrier over a monotonic counter: arrival adds 1; the n-th barrier of
// the launch completes when the counter reaches n * gridDim.x.
struct GridBar {
  unsigned* count;
  unsigned* abort;
  unsigned* err;
  unsigned target;
};

__device__ __forceinline__ void bar_arrive(GridBar& b) {
  __syncthreads();  // the CTA's writes of this stage are done
  b.target += gridDim.x;
  if (threadIdx.x == 0) {
    __threadfence();
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(b.count) : "memory");
  }
}

// false: the launch is aborting (a wait somewhere ran out); leave the kernel.
__device__ __forceinline__ bool bar_wait(GridBar& b, int* s_ok) {
  if (threadIdx.x == 0) {
    int ok = 1;
    if (ld_acquire_u32(b.count) < b.target) {
      const unsigned long long t0 = global_ns();
      for (unsigned i = 1;; ++i) {
        if (ld_acquire_u32(b.count) >= b.target) break;
        if ((i & 63u) == 0) {
          if (ld_relaxed_u32(b.abort) != 0u) { ok = 0; break; }
          if (global_ns() - t0 > kWaitLimitNs) {
            report_error(b.err, kErrWaitTimeout);
            atomicExch(b.abort, 1u);
            ok = 0;
            break;
          }
        }
      }
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

// ---------------------------------------------------------------- stages
constexpr int kStepThreads = 256;
constexpr int kStepWarps = kStepThreads / 32;

// x [k] (written by the previous stage; read past L1) into shared memory as
// bf16, RMSNorm'd with gamma when gamma is set (rounded like the prefill's
// normed GEMM operand).
__device__ void stage_x(const __nv_bfloat16* x, int k, const float* gamma, float eps, uint4* xs,
                        float* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nv = k / 8;
  const uint4* xg = reinterpret_cast<const uint4*>(x);
  if (gamma != nullptr) {
    float ss = 0.f;
    for (int v = tid; v < nv; v += kStepThreads) {
      float f[8];
      unpack8(__ldcg(xg + v), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
    }
    ss = warp_sum32(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kStepWarps; ++w) tot += red[w];
    const float r = rsqrtf(tot / static_cast<float>(k) + eps);
    for (int v = tid; v < nv; v += kStepThreads) {
      float f[8];
      unpack8(__ldcg(xg + v), f);
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma) + 2 * v);
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma) + 2 * v + 1);
      uint4 o;
      o.x = pack_bf16x2(f[0] * r * g0.x, f[1] * r * g0.y);
      o.y = pack_bf16x2(f[2] * r * g0.z, f[3] * r * g0.w);
      o.z = pack_bf16x2(f[4] * r * g1.x, f[5] * r * g1.y);
      o.w = pack_bf16x2(f[6] * r * g1.z, f[7] * r * g1.w);
      xs[v] = o;
    }
  } else {
    for (int v = tid; v < nv; v += kStepThreads) xs[v] = __ldcg(xg + v);
  }
  __syncthreads();
}

// A matrix-vector stage: item i (0 <= i < n_items) is W row i (and, for
// SwiGLU, row inter + i); rows are nv 16-byte vectors, read in chunks of kV
// vectors per lane. Items go to warps round-robin across CTAs. A warp's
// (item, chunk) sequence streams through a ring of kDepth chunks held in
// registers: the first kDepth are loaded before the barrier that precedes
// the stage (weights never change), and each consumed slot is refilled with
// the chunk kDepth places ahead.
struct GemvJob {
  const uint4* w;
  int nv, n_items, inter;
};

template <int kV, bool kTwo>
struct Chunk {
  uint4 a[kV];
  uint4 b[kTwo ? kV : 1];
};

template <int kV, bool kTwo, int kDepth>
struct GemvStream {
  Chunk<kV, kTwo> ring[kDepth];
};

// Loads sequence element q of warp wg (nothing past the warp's last item).
template <int kV, bool kTwo>
__device__ __forceinline__ void gemv_load(const GemvJob& j, int wg, int tw, int n_chunks, int q,
                                          Chunk<kV, kTwo>& ch) {
  const int lane = threadIdx.x & 31;
  const int item = wg + (q / n_chunks) * tw, c = q % n_chunks;
  const bool live = item < j.n_items;
  const uint4* r0 = j.w + static_cast<int64_t>(live ? item : 0) * j.nv;
  const uint4* r1 = kTwo ? j.w + static_cast<int64_t>(j.inter + (live ? item : 0)) * j.nv : r0;
#pragma unroll
  for (int u = 0; u < kV; ++u) {
    const int v = c * 32 * kV + lane + 32 * u;
    const bool in = live && v < j.nv;
    ch.a[u] = in ? ld_stream(r0 + v) : make_uint4(0u, 0u, 0u, 0u);
    if (kTwo) ch.b[u] = in ? ld_stream(r1 + v) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int kV, bool kTwo, int kDepth>
__device__ __forceinline__ void gemv_prefetch(const GemvJob& j, int wg, int tw,
                                              GemvStream<kV, kTwo, kDepth>& st) {
  const int n_chunks = (j.nv + 32 * kV - 1) / (32 * kV);
#pragma unroll
  for (int r = 0; r < kDepth; ++r) gemv_load<kV, kTwo>(j, wg, tw, n_chunks, r, st.ring[r]);
}

template <int kV, bool kTwo, int kDepth, class Epi>
__device__ __forceinline__ void gemv_run(const GemvJob& j, const uint4* xs, int wg, int tw,
                                         GemvStream<kV, kTwo, kDepth>& st, Epi epi) {
  const int lane = threadIdx.x & 31;
  const int n_chunks = (j.nv + 32 * kV - 1) / (32 * kV);
  const int my_items = wg < j.n_items ? (j.n_items - wg + tw - 1) / tw : 0;
  const int total = my_items * n_chunks;
  float acc0 = 0.f, acc1 = 0.f;
  for (int q0 = 0; q0 < total; q0 += kDepth) {
#pragma unroll
    for (int r = 0; r < kDepth; ++r) {
      const int q = q0 + r;
      if (q < total) {
        const int c = q % n_chunks;
#pragma unroll
        for (int u = 0; u < kV; ++u) {
          const int v = c * 32 * kV + lane + 32 * u;
          if (v < j.nv) {
            const uint4 xv = xs[v];
            acc0 += dot8(st.ring[r].a[u], xv);
            if (kTwo) acc1 += dot8(st.ring[r].b[u], xv);
          }
        }
        if (q + kDepth < total) gemv_load<kV, kTwo>(j, wg, tw, n_chunks, q + kDepth, st.ring[r]);
        if (c == n_chunks - 1) {
          acc0 = warp_sum32(acc0);
          if (kTwo) acc1 = warp_sum32(acc1);
          if (lane == 0) epi(wg + (q / n_chunks) * tw, acc0, acc1);
          acc0 = 0.f;
          acc1 = 0.f;
        }
      }
    }
  }
}

// ---------------------------------------------------------------- attention
constexpr int kHalfWarps = kStepThreads / 16;  // one key per 16-lane group
constexpr int kKeys = 4;                       // keys in flight per group

template <int kGroup>
struct AttnSmem {
  float qs[kGroup][kDh];
  __nv_bfloat16 kv_new[2][kDh];
  float red_m[kHalfWarps][kGroup], red_l[kHalfWarps][kGroup];
  float red_o[kHalfWarps][kGroup][kDh];
  float cta_m[kGroup], cta_l[kGroup];
  int is_last;
};

// One (KV head g, key split) unit of a layer's attention.
template <int kGroup>
__device__ void attn_unit(const DecStepParams& p, const DecLayerPtrs& L, bool upper, int g,
                          int split, int n_split, AttnSmem<kGroup>& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int head0 = g * kGroup;
  const __nv_bfloat16* qkv = p.qkv;
  // 1. The token's q (this group's heads) and k: qk-norm, RoPE at pos,
  //    rounded as the prefill stores them; v as projected.
  for (int r = warp; r <= kGroup; r += kStepWarps) {
    const bool is_q = r < kGroup;
    const __nv_bfloat16* src = qkv + (is_q ? (head0 + r) : (p.hq + g)) * kDh;
    const float* nw = is_q ? L.q_norm : L.k_norm;
    float lo[2], hi[2], ss = 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      lo[q] = __bfloat162float(__ldcg(src + lane + 32 * q));
      hi[q] = __bfloat162float(__ldcg(src + lane + 32 * q + kDh / 2));
      ss += lo[q] * lo[q] + hi[q] * hi[q];
    }
    if (nw != nullptr) {
      const float rs = rsqrtf(warp_sum32(ss) / static_cast<float>(kDh) + p.eps);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        lo[q] = lo[q] * rs * __ldg(nw + lane + 32 * q);
        hi[q] = hi[q] * rs * __ldg(nw + lane + 32 * q + kDh / 2);
      }
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int i = lane + 32 * q;
      const float2 cs = rope_cos_sin(p.pos, i, kDh, p.rope_base);
      const __nv_bfloat16 olo = __float2bfloat16_rn(lo[q] * cs.x - hi[q] * cs.y);
      const __nv_bfloat16 ohi = __float2bfloat16_rn(hi[q] * cs.x + lo[q] * cs.y);
      if (is_q) {
        sm.qs[r][i] = __bfloat162float(olo);
        sm.qs[r][i + kDh / 2] = __bfloat162float(ohi);
      } else {
        sm.kv_new[0][i] = olo;
        sm.kv_new[0][i + kDh / 2] = ohi;
      }
    }
  }
  if (tid < kDh) sm.kv_new[1][tid] = __ldcg(qkv + (p.hq + p.hkv + g) * kDh + tid);
  __syncthreads();

  // 2. Split 0 appends the new row (no unit reads that row from memory in
  //    this step: the split holding it takes it from shared memory).
  const int64_t len = L.len;
  if (split == 0 && tid < kDh) {
    L.k_cache[(len * p.hkv + g) * kDh + tid] = sm.kv_new[0][tid];
    L.v_cache[(len * p.hkv + g) * kDh + tid] = sm.kv_new[1][tid];
  }

  // 3. This split's keys: rows [c0, c1) of rows 0..len (row len is the new
  //    token); one 16-lane group per key, 8 head-dim elements per lane.
  const int64_t total = len + 1;
  const int64_t per = (total + n_split - 1) / n_split;
  const int64_t c0 = static_cast<int64_t>(split) * per;
  const int64_t c1 = c0 + per < total ? c0 + per : total;
  const int hw = tid >> 4, sub = lane & 15;
  const unsigned half_mask = 0xFFFFu << (lane & 16);
  const float* gain = upper ? L.gain : nullptr;
  const float* tau = upper ? L.tau : nullptr;
  const float* lsig = (upper && p.scores != nullptr) ? p.lsig : nullptr;
  float qr[kGroup][8], sc[kGroup], bc[kGroup], m[kGroup], l[kGroup], o[kGroup][8];
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
#pragma unroll
    for (int e = 0; e < 8; ++e) qr[h][e] = sm.qs[h][sub * 8 + e];
    const float t = tau ? __ldg(tau + head0 + h) : 1.0f;
    sc[h] = kLog2e / (sqrtf(static_cast<float>(kDh)) * t);
    bc[h] = gain ? __ldg(gain + head0 + h) * kLog2e : 0.f;
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
  }
  const uint4* knew4 = reinterpret_cast<const uint4*>(sm.kv_new[0]);
  const uint4* vnew4 = reinterpret_cast<const uint4*>(sm.kv_new[1]);
  const uint4* kc4 = reinterpret_cast<const uint4*>(L.k_cache);
  const uint4* vc4 = reinterpret_cast<const uint4*>(L.v_cache);
  for (int64_t jb = c0 + hw; jb < c1; jb += kHalfWarps * kKeys) {
    uint4 kk[kKeys], vv[kKeys];
    float bias[kKeys];
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {
      const int64_t j = jb + static_cast<int64_t>(u) * kHalfWarps;
      bias[u] = 0.f;
      if (j < len) {
        const int64_t off = ((j * p.hkv + g) * kDh) / 8 + sub;
        kk[u] = ld_stream(kc4 + off);
        vv[u] = ld_stream(vc4 + off);
        if (lsig != nullptr && j < p.k_kept) bias[u] = __ldcg(lsig + j);
      } else {
        kk[u] = knew4[sub];
        vv[u] = vnew4[sub];
      }
    }
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {
      const int64_t j = jb + static_cast<int64_t>(u) * kHalfWarps;
      if (j >= c1) continue;  // uniform within the 16-lane group
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
        const float pj = ex2_approx(s - base);
        l[h] = l[h] * al + pj;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = fmaf(o[h][e], al, pj * vf[e]);
        m[h] = mn;
      }
    }
  }

  // 4. Merge the 16-lane groups.
#pragma unroll
  for (int h = 0; h < kGroup; ++h) {
    if (sub == 0) {
      sm.red_m[hw][h] = m[h];
      sm.red_l[hw][h] = l[h];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sm.red_o[hw][h][sub * 8 + e] = o[h][e];
  }
  __syncthreads();
  if (tid < kGroup) {
    float mx = -INFINITY;
    for (int w = 0; w < kHalfWarps; ++w) mx = fmaxf(mx, sm.red_m[w][tid]);
    const float base = mx == -INFINITY ? 0.f : mx;
    float ls = 0.f;
    for (int w = 0; w < kHalfWarps; ++w) ls += sm.red_l[w][tid] * ex2_approx(sm.red_m[w][tid] - base);
    sm.cta_m[tid] = mx;
    sm.cta_l[tid] = ls;
  }
  __syncthreads();
  float* part = p.part + (static_cast<int64_t>(g) * kDecodeMaxSplits + split) * kGroup * (kDh + 2);
  if (tid < kDh) {
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
      const float mx = sm.cta_m[h];
      const float base = mx == -INFINITY ? 0.f : mx;
      float acc = 0.f;
      for (int w = 0; w < kHalfWarps; ++w)
        acc += sm.red_o[w][h][tid] * ex2_approx(sm.red_m[w][h] - base);
      part[h * (kDh + 2) + 2 + tid] = acc;
      if (tid == 0) {
        part[h * (kDh + 2)] = mx;
        part[h * (kDh + 2) + 1] = sm.cta_l[h];
      }
    }
  }

  // 5. The last split of this KV head merges every split's state.
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.is_last = atomicAdd(p.merge_cnt + g, 1u) == static_cast<unsigned>(n_split - 1);
  __syncthreads();
  if (!sm.is_last) return;
  __threadfence();
  if (tid < kDh) {
    const float* bp = p.part + static_cast<int64_t>(g) * kDecodeMaxSplits * kGroup * (kDh + 2);
#pragma unroll 1
    for (int h = 0; h < kGroup; ++h) {
      float mx = -INFINITY;
#pragma unroll 8
      for (int s = 0; s < n_split; ++s) mx = fmaxf(mx, __ldcg(bp + (s * kGroup + h) * (kDh + 2)));
      const float base = mx == -INFINITY ? 0.f : mx;
      float ls = 0.f, acc = 0.f;
#pragma unroll 8
      for (int s = 0; s < n_split; ++s) {
        const float* ps = bp + (s * kGroup + h) * (kDh + 2);
        const float w = ex2_approx(__ldcg(ps) - base);
        ls += __ldcg(ps + 1) * w;
        acc += __ldcg(ps + 2 + tid) * w;
      }
      p.o[(head0 + h) * kDh + tid] = __float2bfloat16_rn(acc / ls);
    }
  }
  if (tid == 0) p.merge_cnt[g] = 0u;  // ready for the next layer
}

// ---------------------------------------------------------------- the step
template <int kGroup>
__global__ void __launch_bounds__(kStepThreads, 1) dec_step(const __grid_constant__ DecStepParams p) {
  extern __shared__ __align__(16) uint8_t dyn_smem[];
  uint4* xs = reinterpret_cast<uint4*>(dyn_smem);  // a stage's input vector (bf16)
  AttnSmem<kGroup>& asm_ = *reinterpret_cast<AttnSmem<kGroup>*>(dyn_smem);
  __shared__ float red[kStepWarps];
  __shared__ int s_ok;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int wg = warp * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);  // spread over SMs
  const int tw = static_cast<int>(gridDim.x) * kStepWarps;
  const int d = p.d, qd = p.hq * kDh, nqkv = (p.hq + 2 * p.hkv) * kDh;
  GridBar bar{p.bar, p.bar + 1, p.err, 0u};

  // Stage 0: the residual stream starts as x; the kept tokens' bias inputs.
  if (blockIdx.x == 0) {
    const uint4* x4 = reinterpret_cast<const uint4*>(p.x);
    uint4* h4 = reinterpret_cast<uint4*>(p.h);
    for (int v = tid; v < d / 8; v += kStepThreads) h4[v] = x4[v];
  }
  if (p.scores != nullptr) {
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * kStepThreads + tid; j < p.k_kept;
         j += static_cast<int64_t>(gridDim.x) * kStepThreads) {
      const int32_t i = __ldg(p.kept_idx + j);
      float b = 0.f;
      if (i < 0 || i >= p.n_scores) report_error(p.err, kErrIndexRange);
      else b = logsigmoid_f(__ldg(p.scores + i));
      p.lsig[j] = b;
    }
  }
  const int n_units = p.hkv * p.n_split;
  auto store_qkv = [&](int i, float a0, float) { p.qkv[i] = __float2bfloat16_rn(a0); };
  auto add_h = [&](int i, float a0, float) {
    p.h[i] = __float2bfloat16_rn(__bfloat162float(__ldcg(p.h + i)) + a0);
  };
  auto swiglu = [&](int i, float a0, float a1) { p.act[i] = __float2bfloat16_rn(silu_f(a0) * a1); };
  // Each block: arrive (the previous stage's writes are done), load the next
  // stage's first weight chunk, wait, run the stage.
  for (int li = 0; li < p.n_layers; ++li) {
    const DecLayerPtrs& L = p.layer[li];
    const bool upper = li > p.gate_layer;
    {  // QKV
      const GemvJob j{reinterpret_cast<const uint4*>(L.wqkv), d / 8, nqkv, 0};
      GemvStream<8, false, 4> c;
      bar_arrive(bar);
      gemv_prefetch(j, wg, tw, c);
      if (!bar_wait(bar, &s_ok)) return;
      stage_x(p.h, d, L.attn_norm, p.eps, xs, red);
      gemv_run(j, xs, wg, tw, c, store_qkv);
    }
    {  // attention
      bar_arrive(bar);
      if (!bar_wait(bar, &s_ok)) return;
      if (static_cast<int>(blockIdx.x) < n_units)
        attn_unit<kGroup>(p, L, upper, static_cast<int>(blockIdx.x) % p.hkv,
                          static_cast<int>(blockIdx.x) / p.hkv, p.n_split, asm_);
    }
    {  // O projection + residual
      const GemvJob j{reinterpret_cast<const uint4*>(L.wo), qd / 8, d, 0};
      GemvStream<8, false, 4> c;
      bar_arrive(bar);
      gemv_prefetch(j, wg, tw, c);
      if (!bar_wait(bar, &s_ok)) return;
      stage_x(p.o, qd, nullptr, p.eps, xs, red);
      gemv_run(j, xs, wg, tw, c, add_h);
    }
    if (L.w_gate_up != nullptr) {
      {  // gate/up + SwiGLU
        const GemvJob j{reinterpret_cast<const uint4*>(L.w_gate_up), d / 8, p.dffn, p.dffn};
        GemvStream<4, true, 4> c;
        bar_arrive(bar);
        gemv_prefetch(j, wg, tw, c);
        if (!bar_wait(bar, &s_ok)) return;
        stage_x(p.h, d, L.ffn_norm, p.eps, xs, red);
        gemv_run(j, xs, wg, tw, c, swiglu);
      }
      {  // down + residual
        const GemvJob j{reinterpret_cast<const uint4*>(L.w_down), p.dffn / 8, d, 0};
        GemvStream<8, false, 4> c;
        bar_arrive(bar);
        gemv_prefetch(j, wg, tw, c);
        if (!bar_wait(bar, &s_ok)) return;
        stage_x(p.act, p.dffn, nullptr, p.eps, xs, red);
        gemv_run(j, xs, wg, tw, c, add_h);
      }
    }
  }
  bar_arrive(bar);
  if (!bar_wait(bar, &s_ok)) return;
  // Final RMSNorm of the token's hidden state.
  if (blockIdx.x == 0) {
    if (p.final_norm != nullptr) {
      stage_x(p.h, d, p.final_norm, p.eps, xs, red);
      uint4* out4 = reinterpret_cast<uint4*>(p.out);
      for (int v = tid; v < d / 8; v += kStepThreads) out4[v] = xs[v];
    } else {
      for (int v = tid; v < d / 8; v += kStepThreads)
        reinterpret_cast<uint4*>(p.out)[v] = __ldcg(reinterpret_cast<const uint4*>(p.h) + v);
    }
  }
}

template <int kGroup>
size_t step_smem(const DecStepParams& p) {
  const int kmax = p.d > p.dffn ? p.d : p.dffn;
  const int qd = p.hq * kDh;
  const size_t xs = static_cast<size_t>(kmax > qd ? kmax : qd) * 2;
  const size_t at = sizeof(AttnSmem<kGroup>);
  return xs > at ? xs : at;
}

template <int kGroup>
cudaError_t launch_step(const DecStepParams& p, cudaStream_t st) {
  auto kern = dec_step<kGroup>;
  const size_t smem = step_smem<kGroup>(p);
  cudaError_t e = set_smem_attr_once(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kStepThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.grid));
  cfg.blockDim = dim3(kStepThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barriers can complete
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int decode_grid() { return num_sms(); }

int decode_splits(int hkv) {
  int s = num_sms() / hkv;
  if (s < 1) s = 1;
  if (s > kDecodeMaxSplits) s = kDecodeMaxSplits;
  return s;
}

cudaError_t launch_decode_step(const DecStepParams& p, cudaStream_t st) {
  switch (p.hq / p.hkv) {
    case 1: return launch_step<1>(p, st);
    case 2: return launch_step<2>(p, st);
    case 4: return launch_step<4>(p, st);
    case 8: return launch_step<8>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tg
