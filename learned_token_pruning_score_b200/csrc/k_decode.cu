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
// Weights never change, so they do not wait for the barriers: a producer
// warp in every CTA streams the CTA's share of every weight matrix of the
// step (its contiguous rows of each layer's QKV, O, gate/up and down, in that
// order) with bulk copies into a ring of 32 KB shared-memory slots, running
// ahead of the eleven consumer warps by up to the ring's size. A single
// stream across stages keeps HBM busy through the barriers and avoids the
// per-stage ramp (separate launches cost ~9 us each at this size, more than
// most stages' own traffic). Every wait is bounded; a timed-out grid barrier
// sets the error word and an abort flag that makes every CTA leave at its
// next barrier.
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

// ---------------------------------------------------------------- roles
constexpr int kConsumers = 352;               // 11 consumer warps (12 in all: 168 registers)
constexpr int kConsumerWarps = kConsumers / 32;
constexpr int kStepThreads = kConsumers + 32;  // + the producer warp
constexpr int kSlotBytes = 32768;             // one ring slot
constexpr int kMaxSlots = 6;

// Consumer-only CTA barrier (the producer warp never joins).
__device__ __forceinline__ void cons_sync() { named_bar_sync(1, kConsumers); }

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

// Grid barrier over a monotonic counter among the consumer warps of every
// CTA: arrival adds 1; the n-th barrier of the launch completes when the
// counter reaches n * gridDim.x.
struct GridBar {
  unsigned* count;
  unsigned* abort;
  unsigned* err;
  unsigned target;
  unsigned long long limit_ns = kWaitLimitNs;  // other values: the self-test only
};

__device__ __forceinline__ void bar_arrive(GridBar& b) {
  cons_sync();  // the CTA's writes of this stage are done
  b.target += gridDim.x;
  if (threadIdx.x == 0)  // release: the CTA's writes (ordered by the bar.sync above) go first
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(b.count) : "memory");
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
          if (global_ns() - t0 > b.limit_ns) {
            report_error(b.err, kErrWaitTimeout);
            atomicExch(b.abort, 1u);
            ok = 0;
            break;
          }
        }
      }
    }
    *s_ok = ok;
  }
  cons_sync();
  return *s_ok != 0;
}

// ---------------------------------------------------------------- x staging
// x [k] (written by the previous stage; read past L1) into shared memory as
// bf16, RMSNorm'd with gamma when gamma is set (rounded like the prefill's
// normed GEMM operand). Consumers only.
__device__ void stage_x(const __nv_bfloat16* x, int k, const float* gamma, float eps, uint4* xs,
                        float* red) {
  constexpr int kMaxVec = 5;  // 16-byte vectors per thread: k <= 8 * 5 * kConsumers
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nv = k / 8;
  const uint4* xg = reinterpret_cast<const uint4*>(x);
  uint4 v[kMaxVec];
#pragma unroll
  for (int i = 0; i < kMaxVec; ++i) {
    const int idx = tid + i * kConsumers;
    v[i] = idx < nv ? __ldcg(xg + idx) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (gamma != nullptr) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
      float f[8];
      unpack8(v[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
    }
    ss = warp_sum32(ss);
    if (lane == 0) red[warp] = ss;
    cons_sync();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += red[w];
    const float r = rsqrtf(tot / static_cast<float>(k) + eps);
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
      const int idx = tid + i * kConsumers;
      if (idx < nv) {
        float f[8];
        unpack8(v[i], f);
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma) + 2 * idx);
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma) + 2 * idx + 1);
        uint4 o;
        o.x = pack_bf16x2(f[0] * r * g0.x, f[1] * r * g0.y);
        o.y = pack_bf16x2(f[2] * r * g0.z, f[3] * r * g0.w);
        o.z = pack_bf16x2(f[4] * r * g1.x, f[5] * r * g1.y);
        o.w = pack_bf16x2(f[6] * r * g1.z, f[7] * r * g1.w);
        xs[idx] = o;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
      const int idx = tid + i * kConsumers;
      if (idx < nv) xs[idx] = v[i];
    }
  }
  cons_sync();
}

// ---------------------------------------------------------------- weight stream
// A matrix-vector block: this CTA's items [i0, i1) of a stage. Item i is W
// row i (SwiGLU: rows i and inter + i). A chunk (one ring slot) holds `per`
// consecutive items: `per` rows, or for SwiGLU `per` gate rows followed by
// the matching `per` up rows.
struct Block {
  const uint8_t* w;
  int row_bytes, i0, i1, inter, per;
  bool two;
  __device__ int n_chunks() const { return (i1 - i0 + per - 1) / per; }
};

__device__ __forceinline__ Block make_block(const void* w, int k, int n_items, bool two, int inter,
                                            int cta, int n_cta) {
  Block b;
  b.w = static_cast<const uint8_t*>(w);
  b.row_bytes = k * 2;
  b.i0 = static_cast<int>((static_cast<int64_t>(n_items) * cta) / n_cta);
  b.i1 = static_cast<int>((static_cast<int64_t>(n_items) * (cta + 1)) / n_cta);
  b.inter = inter;
  b.two = two;
  const int rows_per_slot = kSlotBytes / b.row_bytes;  // >= 1: k <= 8192
  b.per = two ? (rows_per_slot / 2 > 0 ? rows_per_slot / 2 : 1) : rows_per_slot;
  if (b.per > kConsumerWarps) b.per = kConsumerWarps;
  return b;
}

// The blocks of layer li for this CTA, in stream order (a layer without an
// FFN has two).
__device__ __forceinline__ int layer_blocks(const DecStepParams& p, int li, int cta, int n_cta,
                                            Block (&b)[4]) {
  const DecLayerPtrs& L = p.layer[li];
  const int nqkv = (p.hq + 2 * p.hkv) * kDh, qd = p.hq * kDh;
  b[0] = make_block(L.wqkv, p.d, nqkv, false, 0, cta, n_cta);
  b[1] = make_block(L.wo, qd, p.d, false, 0, cta, n_cta);
  if (L.w_gate_up == nullptr) return 2;
  b[2] = make_block(L.w_gate_up, p.d, p.dffn, true, p.dffn, cta, n_cta);
  b[3] = make_block(L.w_down, p.dffn, p.d, false, 0, cta, n_cta);
  return 4;
}

struct Ring {
  uint8_t* slots;
  uint64_t* full;
  uint64_t* empty;
  int n_slots;
};

// Producer: every chunk of the step, in order. Returns when all are issued
// (or a wait runs out) after the last copies have landed.
__device__ void produce(const DecStepParams& p, const Ring& r, unsigned* abort) {
  const int lane = threadIdx.x & 31;
  uint32_t seq = 0;
  bool ok = true;
  for (int li = 0; li < p.n_layers && ok; ++li) {
    Block b[4];
    const int nb = layer_blocks(p, li, blockIdx.x, gridDim.x, b);
    for (int bi = 0; bi < nb && ok; ++bi) {
      const int nc = b[bi].n_chunks();
      for (int c = 0; c < nc; ++c, ++seq) {
        const int s = static_cast<int>(seq % r.n_slots);
        const uint32_t ph = (seq / r.n_slots) & 1u;
        if (lane == 0) ok = mbar_wait(&r.empty[s], ph ^ 1u, p.err);
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (!ok || ld_relaxed_u32(abort) != 0u) { ok = false; break; }
        if (lane == 0) {
          const Block& B = b[bi];
          const int first = B.i0 + c * B.per;
          const int cnt = (B.i1 - first) < B.per ? (B.i1 - first) : B.per;
          const uint32_t part = static_cast<uint32_t>(cnt * B.row_bytes);
          uint8_t* dst = r.slots + static_cast<size_t>(s) * kSlotBytes;
          mbar_arrive_expect_tx(&r.full[s], B.two ? 2 * part : part);
          bulk_load(dst, B.w + static_cast<int64_t>(first) * B.row_bytes, part, &r.full[s]);
          if (B.two)
            bulk_load(dst + part, B.w + static_cast<int64_t>(B.inter + first) * B.row_bytes, part,
                      &r.full[s]);
        }
      }
    }
  }
  // Drain: the last copies land before the CTA may exit.
  if (lane == 0) {
    const uint32_t n = seq < static_cast<uint32_t>(r.n_slots) ? seq : static_cast<uint32_t>(r.n_slots);
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t q = seq - 1 - i;
      if (!mbar_wait(&r.full[q % r.n_slots], (q / r.n_slots) & 1u, p.err)) break;
    }
  }
}

// Consumers: one block. Item j (local) goes to warp j % 11; its chunk is
// waited on, the row(s) dotted with x from shared memory, and the chunk's
// empty barrier gets this warp's share of the 11 arrivals a chunk releases
// (the warp of the chunk's first item also arrives for the warps that have
// no item in it).
template <class Epi>
__device__ void consume(const Block& B, const Ring& r, uint32_t seq0, const uint4* xs, unsigned* err,
                        unsigned* abort, Epi epi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_items = B.i1 - B.i0;
  const int nv = B.row_bytes / 16;
  for (int j = warp; j < n_items; j += kConsumerWarps) {
    const int c = j / B.per, jj = j % B.per;
    const uint32_t q = seq0 + static_cast<uint32_t>(c);
    const int s = static_cast<int>(q % r.n_slots);
    const int first = c * B.per;
    const int cnt = (n_items - first) < B.per ? (n_items - first) : B.per;
    if (!mbar_wait_warp(&r.full[s], (q / r.n_slots) & 1u, err)) {
      if (lane == 0) atomicExch(abort, 1u);  // every CTA leaves at its next grid barrier
      return;
    }
    const uint4* row = reinterpret_cast<const uint4*>(r.slots + static_cast<size_t>(s) * kSlotBytes +
                                                      static_cast<size_t>(jj) * B.row_bytes);
    const uint4* row2 = row + static_cast<size_t>(cnt) * nv;  // SwiGLU: the matching up row
    float a0 = 0.f, a1 = 0.f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 xv = xs[v];
      a0 += dot8(row[v], xv);
      if (B.two) a1 += dot8(row2[v], xv);
    }
    a0 = warp_sum32(a0);
    if (B.two) a1 = warp_sum32(a1);
    __syncwarp();
    if (lane == 0) {
      epi(B.i0 + j, a0, a1);
      mbar_arrive_n(&r.empty[s], jj == 0 ? static_cast<uint32_t>(kConsumerWarps - cnt + 1) : 1u);
    }
  }
}

// ---------------------------------------------------------------- attention
constexpr int kHalfWarps = kConsumers / 16;  // one key per 16-lane group
constexpr int kKeys = 6;                       // keys in flight per group

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
                          int split, int n_split, const float2 (&rcs)[2], AttnSmem<kGroup>& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int head0 = g * kGroup;
  const __nv_bfloat16* qkv = p.qkv;
  // 1. The token's q (this group's heads) and k: qk-norm, RoPE at pos,
  //    rounded as the prefill stores them; v as projected.
  for (int r = warp; r <= kGroup; r += kConsumerWarps) {
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
      const float2 cs = rcs[q];
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
  cons_sync();

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
  cons_sync();
  if (tid < kGroup) {
    float mx = -INFINITY;
    for (int w = 0; w < kHalfWarps; ++w) mx = fmaxf(mx, sm.red_m[w][tid]);
    const float base = mx == -INFINITY ? 0.f : mx;
    float ls = 0.f;
    for (int w = 0; w < kHalfWarps; ++w) ls += sm.red_l[w][tid] * ex2_approx(sm.red_m[w][tid] - base);
    sm.cta_m[tid] = mx;
    sm.cta_l[tid] = ls;
  }
  cons_sync();
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
  cons_sync();
  if (tid == 0) sm.is_last = atomicAdd(p.merge_cnt + g, 1u) == static_cast<unsigned>(n_split - 1);
  cons_sync();
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
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  __shared__ __align__(8) uint64_t full[kMaxSlots], empty[kMaxSlots];
  __shared__ float red[kConsumerWarps];
  __shared__ int s_ok;
  Ring ring{dyn_smem, full, empty, p.n_slots};
  uint8_t* scratch = dyn_smem + static_cast<size_t>(p.n_slots) * kSlotBytes;  // xs | attention
  uint4* xs = reinterpret_cast<uint4*>(scratch);
  AttnSmem<kGroup>& asm_ = *reinterpret_cast<AttnSmem<kGroup>*>(scratch);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < p.n_slots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == kConsumerWarps) {  // ------------------------------ producer warp
    produce(p, ring, p.bar + 1);
    return;
  }
  // ------------------------------------------------------------ consumers
  const int d = p.d, qd = p.hq * kDh;
  GridBar bar{p.bar, p.bar + 1, p.err, 0u};
  // (cos, sin) of the token's position for head-dim pairs lane and lane + 32:
  // the same in every layer
  float2 rcs[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) rcs[q] = rope_cos_sin(p.pos, (tid & 31) + 32 * q, kDh, p.rope_base);

  // Stage 0: the residual stream starts as x; the kept tokens' bias inputs.
  if (blockIdx.x == 0) {
    const uint4* x4 = reinterpret_cast<const uint4*>(p.x);
    uint4* h4 = reinterpret_cast<uint4*>(p.h);
    for (int v = tid; v < d / 8; v += kConsumers) h4[v] = x4[v];
  }
  if (p.scores != nullptr) {
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * kConsumers + tid; j < p.k_kept;
         j += static_cast<int64_t>(gridDim.x) * kConsumers) {
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
  uint32_t seq = 0;  // chunks of the stream consumed before the current block
  for (int li = 0; li < p.n_layers; ++li) {
    const DecLayerPtrs& L = p.layer[li];
    const bool upper = li > p.gate_layer;
    Block b[4];
    const int nb = layer_blocks(p, li, blockIdx.x, gridDim.x, b);
    // QKV
    bar_arrive(bar);
    if (!bar_wait(bar, &s_ok)) return;
    stage_x(p.h, d, L.attn_norm, p.eps, xs, red);
    consume(b[0], ring, seq, xs, p.err, p.bar + 1, store_qkv);
    seq += static_cast<uint32_t>(b[0].n_chunks());
    // attention
    bar_arrive(bar);
    if (!bar_wait(bar, &s_ok)) return;
    if (static_cast<int>(blockIdx.x) < n_units)
      attn_unit<kGroup>(p, L, upper, static_cast<int>(blockIdx.x) % p.hkv,
                        static_cast<int>(blockIdx.x) / p.hkv, p.n_split, rcs, asm_);
    // O projection + residual
    bar_arrive(bar);
    if (!bar_wait(bar, &s_ok)) return;
    stage_x(p.o, qd, nullptr, p.eps, xs, red);
    consume(b[1], ring, seq, xs, p.err, p.bar + 1, add_h);
    seq += static_cast<uint32_t>(b[1].n_chunks());
    if (nb == 4) {
      bar_arrive(bar);
      if (!bar_wait(bar, &s_ok)) return;
      stage_x(p.h, d, L.ffn_norm, p.eps, xs, red);
      consume(b[2], ring, seq, xs, p.err, p.bar + 1, swiglu);
      seq += static_cast<uint32_t>(b[2].n_chunks());
      bar_arrive(bar);
      if (!bar_wait(bar, &s_ok)) return;
      stage_x(p.act, p.dffn, nullptr, p.eps, xs, red);
      consume(b[3], ring, seq, xs, p.err, p.bar + 1, add_h);
      seq += static_cast<uint32_t>(b[3].n_chunks());
    }
  }
  bar_arrive(bar);
  if (!bar_wait(bar, &s_ok)) return;
  // Final RMSNorm of the token's hidden state.
  if (blockIdx.x == 0) {
    if (p.final_norm != nullptr) {
      stage_x(p.h, d, p.final_norm, p.eps, xs, red);
      uint4* out4 = reinterpret_cast<uint4*>(p.out);
      for (int v = tid; v < d / 8; v += kConsumers) out4[v] = xs[v];
    } else {
      for (int v = tid; v < d / 8; v += kConsumers)
        reinterpret_cast<uint4*>(p.out)[v] = __ldcg(reinterpret_cast<const uint4*>(p.h) + v);
    }
  }
}

template <int kGroup>
size_t step_scratch(const DecStepParams& p) {
  const int kmax = p.d > p.dffn ? p.d : p.dffn;
  const int qd = p.hq * kDh;
  const size_t xs = static_cast<size_t>(kmax > qd ? kmax : qd) * 2;
  const size_t at = sizeof(AttnSmem<kGroup>);
  return ((xs > at ? xs : at) + 127) & ~size_t(127);
}

template <int kGroup>
cudaError_t launch_step(DecStepParams p, cudaStream_t st) {
  auto kern = dec_step<kGroup>;
  const size_t scratch = step_scratch<kGroup>(p);
  const size_t limit = 227 * 1024 - 1024;  // dynamic shared memory per CTA, minus static
  int slots = static_cast<int>((limit - scratch) / kSlotBytes);
  if (slots > kMaxSlots) slots = kMaxSlots;
  if (slots < 2) return cudaErrorInvalidConfiguration;
  p.n_slots = slots;
  const size_t smem = static_cast<size_t>(slots) * kSlotBytes + scratch;
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

// Self-test of the grid barrier's bounded wait: one CTA of consumers waits
// for a barrier that no CTA arrives at (words[0] = 0 < target 1). After
// limit_ns the wait gives up, records the timeout in err and sets the abort
// word (words[1]); result[0] = 1 if the wait completed, 0 if it gave up (as
// it must here).
__global__ void __launch_bounds__(kConsumers, 1)
    dec_selftest_gridbar(unsigned* words, unsigned* err, unsigned long long limit_ns,
                         int* result) {
  __shared__ int s_ok;
  GridBar bar{words, words + 1, err, 1u};
  bar.limit_ns = limit_ns;
  const bool ok = bar_wait(bar, &s_ok);
  if (threadIdx.x == 0) result[0] = ok ? 1 : 0;
}

}  // namespace

cudaError_t launch_selftest_gridbar(unsigned* words, unsigned* err, unsigned long long limit_ns,
                                    int* result, cudaStream_t st) {
  dec_selftest_gridbar<<<1, kConsumers, 0, st>>>(words, err, limit_ns, result);
  return cudaGetLastError();
}

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
