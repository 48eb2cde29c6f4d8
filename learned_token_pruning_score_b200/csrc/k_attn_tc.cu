// k_attn_tc.cu -- token-gated causal GQA attention on the 5th-generation
// tensor cores (sm_100a), bf16 operands, fp32 accumulation and softmax.
//
// For the kept rows i, j (compacted order; positions ascend with the row):
//   l_ij = (q_i . k_j) / (sqrt(dh) * tau_h) + gain_h * logsigmoid(s_j),  j <= i
//   o_i  = sum_j softmax_j(l_ij) v_j
// The kept tokens' gate scores enter the logits of the upper layers' attention
// as a bias, with a learnable per-head gain and a per-head temperature that
// compensates the sharper softmax over fewer keys (Tencent Cloud article
// "TokenGate：端到端可训练的 Token 剪枝机制，让大模型 Prefill 提速 11.3 倍", section
// "门控机制为评分网络建立梯度路径"; ai.866data.com article "让大模型学会"略读"…",
// section "可学习剪枝的机制设计"). The pages' own kernel was a FlashAttention-2
// variant with a per-key bias (section "TokenGate 的工程验证仍有限"); this is a
// new design for sm_100a. With gain = 0 and tau = 1 it is plain causal
// attention (the dense layers below the gate use it that way).
//
// One CTA per (128-row query tile, query head); heavy (late) tiles first.
//   warp 0     TMA: Q tile once; K and V^T tiles (128 keys) into a 2-deep ring.
//   warp 1     MMA: S_j = Q K_j^T into one of two TMEM S buffers (issued one
//              tile ahead), then O += P_j V_j into a TMEM O accumulator.
//   warps 4-7  softmax, one thread per query row: tcgen05.ld of its S row,
//              scale + gate bias (log2 domain), causal mask, running max with
//              lazy rescaling (O and l are rescaled only when the max grows
//              by more than 2^8), P = exp2(...) written bf16 to shared memory
//              in the 128-byte-swizzled K-major layout the MMA reads.
//   end        O / l read from TMEM, written bf16.
// TMEM: S0 = cols [0,128), S1 = [128,256), O = [256,384) of 512.
#include <algorithm>
#include <atomic>
#include <functional>
#include <map>
#include <memory>
#include <mutex>
#include <queue>
#include <type_traits>
#include <vector>

#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kBlk = 128;         // query rows per tile = keys per KV tile
constexpr int kDh = 128;
constexpr int kThreads = 256;
constexpr int kSub = 128 * 128;   // bytes of one [128 rows x 64 bf16] swizzled sub-tile
constexpr int kTile = 2 * kSub;   // [128 x 128] bf16 tile
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;          // 2 stages
constexpr int kOffV = kOffK + 2 * kTile;      // 2 stages
constexpr int kOffP = kOffV + 2 * kTile;      // 2 buffers
constexpr int kOffBar = kOffP + 2 * kTile;
constexpr size_t kSmem = 1024 + kOffBar + 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThresh = 8.0f;  // log2 units

struct Params {
  int64_t T;
  int hq, hkv;
  int n_qtiles;
  const float* lsig;
  const float* gain;
  const float* tau;
  __nv_bfloat16* out;
  float* lse;      // [hq, T] or null
  float* out_f32;  // [T, hq, dh] or null: the output before rounding
  unsigned int* err;
};


__global__ void __launch_bounds__(kThreads, 1)
    attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* p_full = bars + 7;    // [2]
  uint64_t* pv_done = bars + 9;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x / p.hq);  // heavy first
  const int head = static_cast<int>(blockIdx.x % p.hq);
  const int g = head / (p.hq / p.hkv);
  const int q0 = qt * kBlk;
  const int n_kv = qt + 1;  // causal: KV tiles 0..qt

  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 2) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // q, k, V^T and the bias rows come from the previous kernels

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    mbar_arrive_expect_tx(q_full, kTile);
    tma_load_3d(&tmQ, q_full, smem + kOffQ, 0, head, q0);
    tma_load_3d(&tmQ, q_full, smem + kOffQ + kSub, 64, head, q0);
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!mbar_wait(&kv_empty[s], ((j >> 1) & 1) ^ 1, p.err)) break;
      mbar_arrive_expect_tx(&kv_full[s], 2 * kTile);
      uint8_t* kd = smem + kOffK + s * kTile;
      uint8_t* vd = smem + kOffV + s * kTile;
      tma_load_3d(&tmK, &kv_full[s], kd, 0, g, j * kBlk);
      tma_load_3d(&tmK, &kv_full[s], kd + kSub, 64, g, j * kBlk);
      tma_load_3d(&tmV, &kv_full[s], vd, j * kBlk, 0, g);
      tma_load_3d(&tmV, &kv_full[s], vd + kSub, j * kBlk + 64, 0, g);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
    const uint32_t q_addr = smem_addr(smem + kOffQ);
    auto issue_qk = [&](int j) {
      const int s = j & 1;
      const uint32_t k_addr = smem_addr(smem + kOffK + s * kTile);
      const uint32_t d = tmem + static_cast<uint32_t>(s * 128);
#pragma unroll
      for (int kk = 0; kk < kDh / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
        umma_f16_ss(d, sdesc_kmajor_sw128(q_addr + off), sdesc_kmajor_sw128(k_addr + off), idesc,
                    kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[s]);
    };
    bool ok = mbar_wait(q_full, 0, p.err) && mbar_wait(&kv_full[0], 0, p.err);
    if (ok) {
      tc_fence_after();
      issue_qk(0);
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      if (j + 1 < n_kv) {
        if (!mbar_wait(&kv_full[(j + 1) & 1], ((j + 1) >> 1) & 1, p.err)) break;
        tc_fence_after();
        issue_qk(j + 1);
      }
      const int b = j & 1;
      if (!mbar_wait(&p_full[b], (j >> 1) & 1, p.err)) break;
      tc_fence_after();
      const uint32_t p_addr = smem_addr(smem + kOffP + b * kTile);
      const uint32_t v_addr = smem_addr(smem + kOffV + b * kTile);
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
        umma_f16_ss(tmem + 256, sdesc_kmajor_sw128(p_addr + off),
                    sdesc_kmajor_sw128(v_addr + off), idesc, (j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&kv_empty[b]);
      umma_commit(&pv_done[b]);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- softmax
    const int r = threadIdx.x - 128;  // row within the tile = TMEM lane
    const int64_t q_row = static_cast<int64_t>(q0) + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float tau = p.tau ? __ldg(p.tau + head) : 1.0f;
    const float scale2 = kLog2e / (sqrtf(static_cast<float>(kDh)) * tau);
    const float gb2 = (p.gain && p.lsig) ? __ldg(p.gain + head) * kLog2e : 0.0f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      const int b = j & 1;
      if (!mbar_wait_warp(&s_full[b], (j >> 1) & 1, p.err)) { ok = false; break; }
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float t[32];
        tmem_ld32_wait(tmem + lane_off + static_cast<uint32_t>(b * 128 + c * 32), t);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[c * 32 + i] = t[i];
      }
      const int kv0 = j * kBlk;
      float rmax = -INFINITY;
      const bool diag = (j == n_kv - 1);
      if (gb2 != 0.0f) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const int col = kv0 + i;
          const float bias = col < p.T ? __ldg(p.lsig + col) : 0.0f;
          x[i] = fmaf(x[i], scale2, gb2 * bias);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] *= scale2;
      }
      if (diag) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (kv0 + i > q_row) x[i] = -INFINITY;
      }
#pragma unroll
      for (int i = 0; i < 128; ++i) rmax = fmaxf(rmax, x[i]);
      float alpha = 1.0f;
      if (rmax > m + kRescaleThresh || m == -INFINITY) {
        alpha = ex2_approx(m - rmax);  // 0 on the first tile
        l *= alpha;
        m = rmax;
      }
      // TMEM loads/stores are warp-collective: the warp rescales its 32 O
      // rows together (alpha = 1 for rows whose max did not move).
      const bool rescale_o = j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f);
      float rsum = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        x[i] = ex2_approx(x[i] - m);
        rsum += x[i];
      }
      l += rsum;
      // P buffer b is free once PV_{j-2} has completed; when O must be
      // rescaled, PV_{j-1} must have completed too (it implies PV_{j-2}).
      if (rescale_o) {
        if (!mbar_wait_warp(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err)) { ok = false; break; }
      } else if (j >= 2) {
        if (!mbar_wait_warp(&pv_done[b], ((j - 2) >> 1) & 1, p.err)) { ok = false; break; }
      }
      tc_fence_after();
      uint8_t* pb = smem + kOffP + b * kTile;
#pragma unroll
      for (int cidx = 0; cidx < 16; ++cidx) {
        const int hs = cidx >> 3, c = cidx & 7;
        uint4 u;
        u.x = pack_bf16x2(x[cidx * 8 + 0], x[cidx * 8 + 1]);
        u.y = pack_bf16x2(x[cidx * 8 + 2], x[cidx * 8 + 3]);
        u.z = pack_bf16x2(x[cidx * 8 + 4], x[cidx * 8 + 5]);
        u.w = pack_bf16x2(x[cidx * 8 + 6], x[cidx * 8 + 7]);
        *reinterpret_cast<uint4*>(pb + hs * kSub + r * 128 + ((c ^ (r & 7)) << 4)) = u;
      }
      if (rescale_o) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          const uint32_t ta = tmem + lane_off + 256u + static_cast<uint32_t>(c * 32);
          tmem_ld32_wait(ta, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32_wait(ta, o);
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && mbar_wait_warp(&pv_done[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, p.err)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      // log-sum-exp of the row's logits: m and l are in log2 units
      if (p.lse && q_row < p.T) p.lse[head * p.T + q_row] = (m + log2f(l)) * kLn2;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32_wait(tmem + lane_off + 256u + static_cast<uint32_t>(c * 32), o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= inv;
        if (q_row < p.T) {
          if (p.out_f32) {
            float4* d32 = reinterpret_cast<float4*>(p.out_f32 + (q_row * p.hq + head) * kDh + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              d32[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.out + (q_row * p.hq + head) * kDh + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = pack_bf16x2(o[8 * v + 0], o[8 * v + 1]);
            u.y = pack_bf16x2(o[8 * v + 2], o[8 * v + 3]);
            u.z = pack_bf16x2(o[8 * v + 4], o[8 * v + 5]);
            u.w = pack_bf16x2(o[8 * v + 6], o[8 * v + 7]);
            dst[v] = u;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}


// ============================================================================
// Paired-head design: one CTA per (128-row query tile, pair of query heads
// sharing one KV head). The K/V tiles are loaded once for both heads.
//   warp 0      TMA: both Q tiles once; K and V^T tiles in 2-deep rings.
//   warp 1      MMA (one thread), per KV tile j:
//                 O_A += P_A V_j  (P_A read from TMEM), S_A = Q_A K_{j+1}^T,
//                 O_B += P_B V_j,                      S_B = Q_B K_{j+1}^T
//               so while one softmax warpgroup works, the tensor pipe serves
//               the other head (ping-pong).
//   warps 4-7   softmax of head A, warps 8-11 softmax of head B; one thread
//               per query row. S is read from TMEM, P is written back to TMEM
//               as packed bf16 over the first half of S's columns.
// The gate bias is added by the tensor core: S = Q K^T gets one more 16-wide
// K-step whose A row is (g_hi, g_hi, g_lo, g_lo, 0...) for the head and
// whose B row is (b_hi, b_lo, b_hi, b_lo, 0...) for the key, where
// g = gain_h * sqrt(dh) * tau_h and b = logsigmoid(s_j), each split into two
// bf16 parts; the step adds (g_hi + g_lo)(b_hi + b_lo) = g b to relative
// 2^-17 (so (S + g b) / (sqrt(dh) tau_h) carries gain_h * logsigmoid(s_j)).
// The softmax then needs no per-key loads.
// TMEM columns: S_A [0,128) (P_A [0,64)), S_B [128,256) (P_B [128,192)),
//               O_A [256,384), O_B [384,512).
// Ordering: the commit that signals S_h(j+1) is issued after O_h += P_h(j) V_j,
// so when a softmax thread sees S_h(j+1) the previous P.V of its head has
// finished: O_h may be rescaled and P_h overwritten without another wait.
// ============================================================================
namespace pair {

constexpr int kThreads = 384;
// Register split (setmaxnreg): the kernel launches with kRegsLaunch per
// thread (the most that 384 threads may hold); warpgroup 0 drops to
// kRegsLow and the softmax warpgroups rise to kRegsHigh. The split must use
// exactly the registers the CTA launched with, or setmaxnreg.inc would wait
// for registers that never come: the launcher checks the compiled count.
constexpr uint32_t kRegsLaunch = 168, kRegsLow = 72, kRegsHigh = 216;
static_assert(kRegsLow * 128 + kRegsHigh * 256 == kRegsLaunch * kThreads, "register split");
// Shared-memory layout. With the gate bias, its 32-byte-swizzled tiles come
// first (an addressing slip there cannot reach past the allocation), then
// the 128-byte-swizzled operand tiles.
constexpr int kAugTile = 128 * 32;  // [128 rows x 16 bf16]
template <bool kBias>
struct Layout {
  static constexpr int kAug = kBias ? kAugTile : 0;
  static constexpr int kOffQAugA = 0;
  static constexpr int kOffQAugB = kOffQAugA + kAug;
  static constexpr int kOffKAug = kOffQAugB + kAug;      // 2 stages
  static constexpr int kOffQA = kOffKAug + 2 * kAug;     // 0 or 16 KB: 1024-aligned
  static constexpr int kOffQB = kOffQA + kTile;
  static constexpr int kOffK = kOffQB + kTile;           // 2 stages
  static constexpr int kOffV = kOffK + 2 * kTile;        // 2 stages
  static constexpr int kOffBar = kOffV + 2 * kTile;
  static constexpr size_t kSmem = 1024 + kOffBar + 256;
};

// Work-item table of a short sequence (see Schedule below): entry i gives
// one part of one query tile, and the grid runs n_pairs CTAs per entry.
//   x = qt | kv_lo << 10 | kv_hi << 20        (KV tiles kv_lo..kv_hi)
//   y = part | (n_parts - 1) << 4 | split << 8 | slot0 << 20
// A query tile split into n_parts parts has one counter (`split`) and
// n_parts partial-result slots slot0 .. slot0 + n_parts - 1.
constexpr int kMaxItems = 256;
constexpr int kMaxSlots = 32;  // partial-result slots per head pair
constexpr int kMaxParts = 4;

struct Params {
  int64_t T;
  int hq, hkv;
  int n_qtiles;
  int qt_lo;     // first query tile of the launch (tiles qt_lo .. n_qtiles - 1)
  int kv_major;  // 1: CTAs ordered KV-head-major (large T), 0: heaviest tiles first
  const float* gain;
  const float* tau;
  __nv_bfloat16* out;
  float* lse;      // [hq, T] or null
  float* out_f32;  // [T, hq, dh] or null: the output before rounding
  unsigned int* err;
  // Split query tiles (n_items > 0): each part writes its unnormalised
  // output rows and (m, l) to a slot; the part that finishes last (per-tile
  // counter) merges every slot in slot order and writes the result.
  int n_items;      // 0: closed-form order, no splits
  float* part_o;    // [slots][n_pairs][2 heads][128 / 4 column quads][128 rows] float4
  float* part_ml;   // [slots][n_pairs][2][128][2] fp32 (m in log2 units, l)
  unsigned* cnt;    // [splits][n_pairs], zero between launches
  uint2 items[kMaxItems];
};

// bar.red.and over the `count` threads of named barrier `id`.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

template <bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKAug,
                 const __grid_constant__ CUtensorMap tmO, const __grid_constant__ Params p) {
  using Lay = Layout<kBias>;
  constexpr int kOffQAugA = Lay::kOffQAugA, kOffQAugB = Lay::kOffQAugB, kOffKAug = Lay::kOffKAug;
  constexpr int kOffQA = Lay::kOffQA, kOffQB = Lay::kOffQB, kOffK = Lay::kOffK, kOffV = Lay::kOffV;
  constexpr int kOffBar = Lay::kOffBar;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2 heads]
  uint64_t* p_full = bars + 11;   // [2 heads]
  uint64_t* o_full = bars + 13;   // head A; head B's is bars + 16
  uint64_t* qaug_full = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA order. When all K/V fits in L2 easily, the heaviest (latest) query
  // tiles of every head go first (longest-first list scheduling). Otherwise
  // KV-head-major, so that the CTAs running together share one KV head's
  // K/V in L2, heaviest first within each KV head.
  const int pairs_per_kv = (p.hq / p.hkv) / 2;
  const int n_pairs = p.hq / 2;
  int qt, head0;
  int kv_lo = 0;
  if (p.n_items > 0) {
    const uint32_t x = p.items[blockIdx.x / n_pairs].x;
    head0 = 2 * (static_cast<int>(blockIdx.x) % n_pairs);
    qt = static_cast<int>(x & 1023u);
    kv_lo = static_cast<int>((x >> 10) & 1023u);
  } else if (p.kv_major) {
    const int per_kv = (p.n_qtiles - p.qt_lo) * pairs_per_kv;
    const int g0 = static_cast<int>(blockIdx.x) / per_kv;
    const int rem = static_cast<int>(blockIdx.x) % per_kv;
    qt = p.n_qtiles - 1 - rem / pairs_per_kv;
    head0 = g0 * (p.hq / p.hkv) + 2 * (rem % pairs_per_kv);
  } else {
    qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / n_pairs;
    head0 = 2 * (static_cast<int>(blockIdx.x) % n_pairs);
  }
  const int g = head0 / (p.hq / p.hkv);
  const int q0 = qt * kBlk;
  // KV tiles kv_lo .. kv_hi of this item (the diagonal tile is qt)
  const int kv_hi = p.n_items > 0 ? static_cast<int>((p.items[blockIdx.x / n_pairs].x >> 20) & 1023u)
                                  : qt;
  const int n_kv = kv_hi - kv_lo + 1;
  constexpr uint32_t kKBytes = kTile + (kBias ? kAugTile : 0);
  __shared__ int s_last;

  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(o_full, 1);
    mbar_init(bars + 16, 1);
    mbar_init(qaug_full, 256);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (kBias) tma_prefetch_desc(&tmKAug);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 2) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // q, k, V^T and the bias rows come from the previous kernels

  if (warp < 4) {
    // Warpgroup 0 (TMA, MMA, TMEM allocation) needs few registers: it hands
    // them to the two softmax warpgroups.
    setmaxnreg_dec<kRegsLow>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      mbar_arrive_expect_tx(q_full, 2 * kTile);
      tma_load_3d(&tmQ, q_full, smem + kOffQA, 0, head0, q0);
      tma_load_3d(&tmQ, q_full, smem + kOffQA + kSub, 64, head0, q0);
      tma_load_3d(&tmQ, q_full, smem + kOffQB, 0, head0 + 1, q0);
      tma_load_3d(&tmQ, q_full, smem + kOffQB + kSub, 64, head0 + 1, q0);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j & 1;
        const uint32_t ph = ((j >> 1) & 1) ^ 1;
        if (!mbar_wait(&k_empty[s], ph, p.err)) break;
        uint8_t* kd = smem + kOffK + s * kTile;
        mbar_arrive_expect_tx(&k_full[s], kKBytes);
        const int key0 = (kv_lo + j) * kBlk;
        tma_load_3d(&tmK, &k_full[s], kd, 0, g, key0);
        tma_load_3d(&tmK, &k_full[s], kd + kSub, 64, g, key0);
        if (kBias) tma_load_2d(&tmKAug, &k_full[s], smem + kOffKAug + s * kAugTile, 0, key0);
        if (!mbar_wait(&v_empty[s], ph, p.err)) break;
        uint8_t* vd = smem + kOffV + s * kTile;
        mbar_arrive_expect_tx(&v_full[s], kTile);
        tma_load_3d(&tmV, &v_full[s], vd, key0, 0, g);
        tma_load_3d(&tmV, &v_full[s], vd + kSub, key0 + 64, 0, g);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
      auto issue_qk = [&](int h, int j) {
        const uint32_t q_addr = smem_addr(smem + (h ? kOffQB : kOffQA));
        const uint32_t k_addr = smem_addr(smem + kOffK + (j & 1) * kTile);
        const uint32_t d = tmem + static_cast<uint32_t>(h * 128);
  #pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          umma_f16_ss(d, sdesc_kmajor_sw128(q_addr + off), sdesc_kmajor_sw128(k_addr + off), idesc,
                      kk > 0 ? 1u : 0u);
        }
        if (kBias) {  // the gate-bias K-step
          umma_f16_ss(d, sdesc_kmajor_sw32(smem_addr(smem + (h ? kOffQAugB : kOffQAugA))),
                      sdesc_kmajor_sw32(smem_addr(smem + kOffKAug + (j & 1) * kAugTile)), idesc, 1u);
        }
        umma_commit(&s_full[h]);
      };
      auto issue_pv = [&](int h, int j) {
        const uint32_t v_addr = smem_addr(smem + kOffV + (j & 1) * kTile);
        const uint32_t a = tmem + static_cast<uint32_t>(h * 128);        // P_h
        const uint32_t d = tmem + 256u + static_cast<uint32_t>(h * 128);  // O_h
  #pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          umma_f16_ts(d, a + static_cast<uint32_t>(kk * 8), sdesc_kmajor_sw128(v_addr + off), idesc,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, p.err) && mbar_wait(&k_full[0], 0, p.err);
      if (kBias) ok = ok && mbar_wait(qaug_full, 0, p.err);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const bool more = j + 1 < n_kv;
        if (!mbar_wait(&v_full[s], ph, p.err)) break;
        if (!mbar_wait(&p_full[0], j & 1, p.err)) break;
        tc_fence_after();
        issue_pv(0, j);
        if (!more) umma_commit(o_full);  // head A's output is final
        if (more) {
          if (!mbar_wait(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, p.err)) break;
          tc_fence_after();
          issue_qk(0, j + 1);
        }
        if (!mbar_wait(&p_full[1], j & 1, p.err)) break;
        tc_fence_after();
        issue_pv(1, j);
        if (!more) umma_commit(bars + 16);  // head B's output is final
        umma_commit(&v_empty[s]);
        if (more) {
          issue_qk(1, j + 1);
          umma_commit(&k_empty[(j + 1) & 1]);
        }
      }
    }
  } else {
    setmaxnreg_inc<kRegsHigh>();
    // ---------------------------------------------------------- softmax
    const int h = (warp - 4) >> 2;  // 0: head A (warps 4-7), 1: head B (warps 8-11)
    const int head = head0 + h;
    const int r = (threadIdx.x - 128) & 127;  // row within the tile = TMEM lane
    const int64_t q_row = static_cast<int64_t>(q0) + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = static_cast<uint32_t>(h * 128);
    const uint32_t o_col = 256u + static_cast<uint32_t>(h * 128);
    const float tau = p.tau ? __ldg(p.tau + head) : 1.0f;
    const float scale2 = kLog2e / (sqrtf(static_cast<float>(kDh)) * tau);
    if (kBias) {
      // this row of the head's gate-bias A tile: (g_hi, g_hi, g_lo, g_lo, 0 ...)
      const float gs = __ldg(p.gain + head) * sqrtf(static_cast<float>(kDh)) * tau;
      const __nv_bfloat16 ghi = __float2bfloat16_rn(gs);
      const __nv_bfloat16 glo = __float2bfloat16_rn(gs - __bfloat162float(ghi));
      __nv_bfloat162 hh, ll;
      hh.x = ghi;
      hh.y = ghi;
      ll.x = glo;
      ll.y = glo;
      uint8_t* row = smem + (h ? kOffQAugB : kOffQAugA) + r * 32;
      const int sw = (r >> 2) & 1;  // 32-byte swizzle: 16-byte chunk c sits at c ^ sw
      *reinterpret_cast<uint4*>(row + ((0 ^ sw) << 4)) =
          make_uint4(*reinterpret_cast<uint32_t*>(&hh), *reinterpret_cast<uint32_t*>(&ll), 0u, 0u);
      *reinterpret_cast<uint4*>(row + ((1 ^ sw) << 4)) = make_uint4(0u, 0u, 0u, 0u);
      fence_async_smem();
      mbar_arrive(qaug_full);
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      const int kv0 = (kv_lo + j) * kBlk;
      if (!mbar_wait_warp(&s_full[h], j & 1, p.err)) { ok = false; break; }
      tc_fence_after();
      // S row: four TMEM loads in flight, one wait.
      float x[128];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        const uint32_t sa = tmem + lane_off + s_col;
        tmem_ld32(sa, r0);
        tmem_ld32(sa + 32, r1);
        tmem_ld32(sa + 64, r2);
        tmem_ld32(sa + 96, r3);
        tmem_wait_ld_dep(r3);
        tmem_ld_fence(r0);
        tmem_ld_fence(r1);
        tmem_ld_fence(r2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = __uint_as_float(r0[i]);
          x[32 + i] = __uint_as_float(r1[i]);
          x[64 + i] = __uint_as_float(r2[i]);
          x[96 + i] = __uint_as_float(r3[i]);
        }
      }
      const bool diag = kv_lo + j == qt;
      if (diag) {  // diagonal tile: causal mask
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (kv0 + i > q_row) x[i] = -INFINITY;
      }
      // Row max: eight independent chains of 3-input max (a single running
      // max would be a 128-long dependent chain).
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmax3f(x[k], x[8 + k], x[16 + k]);
#pragma unroll
      for (int i = 24; i < 120; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmax3f(mx8[k], x[i + k], x[i + 8 + k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], x[120 + k]);
      const float mx = fmax3f(fmax3f(mx8[0], mx8[1], mx8[2]), fmax3f(mx8[3], mx8[4], mx8[5]),
                              fmaxf(mx8[6], mx8[7])) *
                       scale2;
      float alpha = 1.0f;
      if (mx > m + kRescaleThresh || m == -INFINITY) {
        alpha = ex2_approx(m - mx);  // 0 on the first tile
        l *= alpha;
        m = mx;
      }
      const bool rescale_o = j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f);
      // P = 2^(S * scale2 - m) in packed pairs; the row sum in four packed
      // partial sums. Off the diagonal tile (no masked logits) one pair in
      // four goes through the FMA-pipe polynomial, which unloads the MUFU
      // unit, the bottleneck of this loop.
      float2 sp[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
      const float2 sc2 = make_float2(scale2, scale2), nm2 = make_float2(-m, -m);
      auto exp_tile = [&](auto poly) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 y =
                ffma2(make_float2(x[64 * half + 2 * i], x[64 * half + 2 * i + 1]), sc2, nm2);
            float2 a;
            if (decltype(poly)::value && (i & 3) == 3) {
              a = exp2_poly3_x2(y);
            } else {
              a.x = ex2_approx(y.x);
              a.y = ex2_approx(y.y);
            }
            sp[i & 3] = fadd2(sp[i & 3], a);
            pk[i] = pack_bf16x2(a.x, a.y);
          }
          tmem_st32(tmem + lane_off + s_col + static_cast<uint32_t>(32 * half), pk);
          tmem_wait_st();
        }
      };
      if (diag) exp_tile(std::false_type());
      else exp_tile(std::true_type());
      const float2 s2 = fadd2(fadd2(sp[0], sp[1]), fadd2(sp[2], sp[3]));
      l += s2.x + s2.y;
      if (rescale_o) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          const uint32_t ta = tmem + lane_off + o_col + static_cast<uint32_t>(c * 32);
          tmem_ld32_wait(ta, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32_wait(ta, o);
        }
      }
      tc_fence_before();
      mbar_arrive(&p_full[h]);
    }
    ok = ok && mbar_wait_warp(h ? bars + 16 : o_full, 0, p.err);
    if (ok) tc_fence_after();
    // the item's split fields (decoded here, not kept live through the loop)
    const uint32_t iy = p.n_items > 0 ? p.items[blockIdx.x / n_pairs].y : 0u;
    const int part = static_cast<int>(iy & 15u);
    const int n_parts = static_cast<int>((iy >> 4) & 15u) + 1;
    const int split = static_cast<int>((iy >> 8) & 4095u);
    const int slot0 = static_cast<int>(iy >> 20);
    // Output of a split query tile: this part's rows go to its slot; the
    // part that finishes last merges every slot (slot order, so the result
    // does not depend on which part finishes last) with weights 2^(m_s - M).
    float wts[kMaxParts];
    int n_merge = 1;
    const size_t pair_idx = static_cast<size_t>(head0 / 2);
    auto slot_row = [&](int slot) {
      return ((static_cast<size_t>(slot) * n_pairs + pair_idx) * 2 + h) * kBlk + r;
    };
    // a slot's partial output: [kDh / 4][kBlk rows] float4, so that the
    // rows of a warp are adjacent (coalesced) for every 4 columns
    auto slot_o = [&](int slot) {
      return reinterpret_cast<float4*>(
                 p.part_o + ((static_cast<size_t>(slot) * n_pairs + pair_idx) * 2 + h) * kBlk * kDh) +
             r;
    };
    if (n_parts > 1) {
      if (ok) {
        const size_t ri = slot_row(slot0 + part);
        float4* po = slot_o(slot0 + part);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32_wait(tmem + lane_off + o_col + static_cast<uint32_t>(c * 32), o);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            po[(c * 8 + v) * kBlk] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
        *reinterpret_cast<float2*>(p.part_ml + ri * 2) = make_float2(m, l);
        __threadfence();
      }
      // every softmax thread of the CTA reaches both barriers, whatever ok is
      const bool all_ok = named_bar_and(1, 256, ok);
      if (threadIdx.x == 128) {
        int last = 0;
        if (all_ok) {
          unsigned* c = p.cnt + static_cast<size_t>(split) * n_pairs + pair_idx;
          const unsigned old = atomicAdd(c, 1u);
          __threadfence();
          last = old == static_cast<unsigned>(n_parts - 1);
          if (last) *c = 0u;  // zero again for the next launch
        }
        s_last = last;
      }
      named_bar_sync(1, 256);
      ok = s_last != 0;
      if (ok) {
        float ms[kMaxParts], ls[kMaxParts];
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < kMaxParts; ++s2) {
          if (s2 < n_parts) {
            if (s2 == part) {
              ms[s2] = m;
              ls[s2] = l;
            } else {
              const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml) +
                                       slot_row(slot0 + s2));
              ms[s2] = ml.x;
              ls[s2] = ml.y;
            }
            M = fmaxf(M, ms[s2]);
          }
        }
        float L = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kMaxParts; ++s2) {
          wts[s2] = s2 < n_parts ? ex2_approx(ms[s2] - M) : 0.f;
          if (s2 < n_parts) L = fmaf(ls[s2], wts[s2], L);
        }
        m = M;
        l = L;
        n_merge = n_parts;
      }
    }
    if (ok) {
      const float inv = 1.0f / l;
      // log-sum-exp of the row's logits: m and l are in log2 units
      if (p.lse && q_row < p.T) p.lse[head * p.T + q_row] = (m + log2f(l)) * kLn2;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32_wait(tmem + lane_off + o_col + static_cast<uint32_t>(c * 32), o);
        if (n_merge > 1) {
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
          for (int s2 = 0; s2 < kMaxParts; ++s2) {
            if (s2 >= n_merge) break;
            if (s2 == part) {
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[i] = fmaf(o[i], wts[s2], acc[i]);
            } else {
              const float4* src = slot_o(slot0 + s2) + c * 8 * kBlk;
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                const float4 t = __ldcg(src + v * kBlk);
                acc[4 * v] = fmaf(t.x, wts[s2], acc[4 * v]);
                acc[4 * v + 1] = fmaf(t.y, wts[s2], acc[4 * v + 1]);
                acc[4 * v + 2] = fmaf(t.z, wts[s2], acc[4 * v + 2]);
                acc[4 * v + 3] = fmaf(t.w, wts[s2], acc[4 * v + 3]);
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = acc[i];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= inv;
        if (p.out_f32 && q_row < p.T) {
          float4* d32 = reinterpret_cast<float4*>(p.out_f32 + (q_row * p.hq + head) * kDh + c * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            d32[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
        // the bf16 row into the head's (now idle) Q buffer, in the 128-byte
        // swizzled layout of the output's TMA boxes: columns 32c .. 32c + 31
        // are 16-byte units 4 (c & 1) .. + 3 of box c >> 1
        uint8_t* rowp = smem + (h ? kOffQB : kOffQA) + (c >> 1) * kSub + r * 128;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 u;
          u.x = pack_bf16x2(o[8 * v + 0], o[8 * v + 1]);
          u.y = pack_bf16x2(o[8 * v + 2], o[8 * v + 3]);
          u.z = pack_bf16x2(o[8 * v + 4], o[8 * v + 5]);
          u.w = pack_bf16x2(o[8 * v + 6], o[8 * v + 7]);
          const int unit = 4 * (c & 1) + v;
          *reinterpret_cast<uint4*>(rowp + ((unit ^ (r & 7)) << 4)) = u;
        }
      }
      fence_async_smem();
    }
    // The head's 128 rows leave in two TMA stores (rows past T are not
    // written). Every thread of the warpgroup reaches the barrier.
    const bool head_ok = named_bar_and(2 + h, 128, ok);
    if (head_ok && r == 0) {
      const uint8_t* ob = smem + (h ? kOffQB : kOffQA);
      tma_store_3d(&tmO, ob, 0, head, q0);
      tma_store_3d(&tmO, ob + kSub, 64, head, q0);
      bulk_commit();
      bulk_wait_read_all();  // the buffer is read before the CTA may exit
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Schedule of a short sequence. With few query tiles, one CTA per (tile, head
// pair) leaves SMs idle while the last (longest, causal) tiles finish. The
// table instead lists query-tile parts, longest first, so that the block
// scheduler (which starts CTAs in index order as SMs free up) runs a
// longest-first list schedule, and splits long tiles' KV ranges into up to
// kMaxParts parts, with the part length that gives the shortest simulated
// makespan on the B200's 148 SMs. The schedule depends only on (T, heads), never on the device, so
// the workspace it needs is known on the host.
constexpr int kMaxTableQ = 64;   // query tiles (T <= 8192) eligible for a table
constexpr int kSchedSMs = 148;
// Costs in KV-tile units (one KV tile of a head pair: ~2.2 us on B200).
// Measured per CTA: setup 0.7 us + first S tile 2.1 us + output 3.5 us;
// a split part's partial write and the merge add ~4 us.
constexpr double kItemOverhead = 2.9;  // per-CTA prologue + epilogue
constexpr double kMergeCost = 1.8;     // writing / merging a partial

struct Schedule {
  int n_items = 0, n_split = 0, n_slots = 0;
  uint2 items[kMaxItems];
};

double list_makespan(const std::vector<double>& jobs) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> q;
  for (int i = 0; i < kSchedSMs; ++i) q.push(0.0);
  double mk = 0.0;
  for (double c : jobs) {
    double t = q.top();
    q.pop();
    t += c;
    mk = std::max(mk, t);
    q.push(t);
  }
  return mk;
}

// Fills *out and returns true when a table schedule applies (n_q query tiles
// of n_pairs head pairs); false: the closed-form order, no splits.
bool make_schedule(int n_q, int n_pairs, Schedule* out) {
  if (n_q < 1 || n_q > kMaxTableQ || n_pairs < 1) return false;
  struct Part {
    int qt, lo, hi, part, np;
    double cost;
  };
  double best = 1e300;
  std::vector<Part> best_parts;
  // cap: the most KV tiles one part takes; longer tiles split into
  // ceil(tiles / cap) near-equal parts
  for (int cap = n_q; cap >= (n_q + kMaxParts - 1) / kMaxParts; --cap) {
    std::vector<Part> parts;
    int slots = 0;
    for (int qt = n_q - 1; qt >= 0; --qt) {
      const int c = qt + 1, np = (c + cap - 1) / cap;
      for (int i = 0; i < np; ++i) {
        const int lo = i * c / np, hi = (i + 1) * c / np - 1;
        parts.push_back(Part{qt, lo, hi, i, np,
                             double(hi - lo + 1) + kItemOverhead + (np > 1 ? kMergeCost : 0.0)});
      }
      if (np > 1) slots += np;
    }
    if (static_cast<int>(parts.size()) > kMaxItems || slots > kMaxSlots) continue;
    std::stable_sort(parts.begin(), parts.end(),
                     [](const Part& a, const Part& b) { return a.cost > b.cost; });
    std::vector<double> jobs;
    for (const Part& pt : parts)
      for (int k = 0; k < n_pairs; ++k) jobs.push_back(pt.cost);
    const double mk = list_makespan(jobs);
    if (mk < best - 1e-9) {
      best = mk;
      best_parts = parts;
    }
  }
  if (best_parts.empty()) return false;
  // counters and slots of the split tiles, in query-tile order
  std::vector<int> split_of(n_q, -1), slot_of(n_q, 0);
  int n_split = 0, n_slots = 0;
  for (int qt = 0; qt < n_q; ++qt)
    for (const Part& pt : best_parts)
      if (pt.qt == qt && pt.part == 0 && pt.np > 1) {
        split_of[qt] = n_split++;
        slot_of[qt] = n_slots;
        n_slots += pt.np;
      }
  out->n_items = static_cast<int>(best_parts.size());
  out->n_split = n_split;
  out->n_slots = n_slots;
  for (int i = 0; i < out->n_items; ++i) {
    const Part& pt = best_parts[i];
    const unsigned sp = pt.np > 1 ? static_cast<unsigned>(split_of[pt.qt]) : 0u;
    const unsigned sl = pt.np > 1 ? static_cast<unsigned>(slot_of[pt.qt]) : 0u;
    out->items[i] = make_uint2(static_cast<unsigned>(pt.qt) | static_cast<unsigned>(pt.lo) << 10 |
                                   static_cast<unsigned>(pt.hi) << 20,
                               static_cast<unsigned>(pt.part) |
                                   static_cast<unsigned>(pt.np - 1) << 4 | sp << 8 | sl << 20);
  }
  return true;
}

// make_schedule is a host simulation (about a millisecond); its result
// depends only on (n_q, n_pairs), so it is computed once per shape.
const Schedule* cached_schedule(int n_q, int n_pairs) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, std::unique_ptr<Schedule>> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({n_q, n_pairs});
  if (it == cache.end()) {
    auto sch = std::make_unique<Schedule>();
    if (!make_schedule(n_q, n_pairs, sch.get())) sch.reset();
    it = cache.emplace(std::make_pair(n_q, n_pairs), std::move(sch)).first;
  }
  return it->second.get();
}

}  // namespace pair


}  // namespace

// Byte offset of the split counters inside the split scratch.
static size_t split_cnt_offset(int hq) {
  const size_t rows = size_t(pair::kMaxSlots) * size_t(hq / 2) * 2 * kBlk;
  return align_up(rows * kDh * 4, 256) + align_up(rows * 2 * 4, 256);
}

cudaError_t attn_split_clear(void* split_ws, size_t split_ws_bytes, int hq, cudaStream_t st) {
  if (split_ws == nullptr || split_ws_bytes == 0) return cudaSuccess;
  return cudaMemsetAsync(static_cast<char*>(split_ws) + split_cnt_offset(hq), 0,
                         size_t(pair::kMaxSlots) * size_t(hq / 2) * 4, st);
}

size_t attn_split_bytes(int64_t T, int hq, int hkv) {
  if (T < 1 || hkv < 1 || hq % hkv != 0 || (hq / hkv) % 2 != 0) return 0;
  const int64_t n_q = (T + kBlk - 1) / kBlk;
  if (n_q > pair::kMaxTableQ) return 0;
  const size_t n_pairs = static_cast<size_t>(hq / 2);
  const size_t rows = size_t(pair::kMaxSlots) * n_pairs * 2 * kBlk;
  return align_up(rows * kDh * 4, 256) + align_up(rows * 2 * 4, 256) +
         align_up(size_t(pair::kMaxSlots) * n_pairs * 4, 256);
}

bool attn_tc_supported(const AttnArgs& a) {
  auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  return a.dh == kDh && a.hq % a.hkv == 0 && a.t_pad % 64 == 0 && a.t_pad >= a.T && al16(a.q) &&
         al16(a.k) && al16(a.v) && al16(a.out) && a.T < (int64_t(1) << 31) - kBlk &&
         a.q_lo >= 0 && a.q_lo % kBlk == 0 && a.q_lo < a.T &&
         (a.q_lo == 0 || (a.hq / a.hkv) % 2 == 0);
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const int64_t e = 2;
  if (!make_tmap_3d_bf16(&tq, a.q, kDh, a.hq, a.T, kDh * e, int64_t(a.hq) * kDh * e, 1, kBlk))
    return cudaErrorInvalidValue;
  if (!make_tmap_3d_bf16(&tk, a.k, kDh, a.hkv, a.T, kDh * e, int64_t(a.hkv) * kDh * e, 1, kBlk))
    return cudaErrorInvalidValue;
  // V^T: the inner extent is T (not the padded row length), so key columns
  // past T read as zeros whatever the padding holds.
  if (!make_tmap_3d_bf16(&tv, a.v, a.T, kDh, a.hkv, a.t_pad * e, a.t_pad * kDh * e, kDh, 1))
    return cudaErrorInvalidValue;
  Params p;
  p.T = a.T;
  p.hq = a.hq;
  p.hkv = a.hkv;
  p.n_qtiles = static_cast<int>((a.T + kBlk - 1) / kBlk);
  p.lsig = a.lsig;
  p.gain = a.gain;
  p.tau = a.tau;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.out_f32 = a.out_f32;
  p.err = device_error_word();
  if ((a.hq / a.hkv) % 2 == 0) {
    // paired-head kernel (the two query heads of a pair share a KV head)
    pair::Params pp;
    pp.T = p.T;
    pp.hq = p.hq;
    pp.hkv = p.hkv;
    pp.n_qtiles = p.n_qtiles;
    pp.qt_lo = static_cast<int>(a.q_lo / kBlk);
    // K and V of all KV heads: above ~48 MB the working set would not stay
    // in the 126 MB L2 across a wave of CTAs spread over every head.
    pp.kv_major = (double(a.T) * a.hkv * kDh * 4.0 > 48.0e6) ? 1 : 0;
    pp.gain = p.gain;
    pp.tau = p.tau;
    pp.out = p.out;
    pp.lse = p.lse;
    pp.out_f32 = p.out_f32;
    pp.err = p.err;
    const bool bias = a.lsig != nullptr && a.gain != nullptr;
    CUtensorMap tka, to;
    // the output [T, hq, dh], stored by TMA in the same boxes as q is read
    if (!make_tmap_3d_bf16(&to, a.out, kDh, a.hq, a.T, kDh * e, int64_t(a.hq) * kDh * e, 1, kBlk))
      return cudaErrorInvalidValue;
    if (bias) {
      if (a.kaug == nullptr || !make_tmap_2d_bf16_sw32(&tka, a.kaug, a.T, 16, kBlk))
        return cudaErrorInvalidValue;
    } else {
      tka = tk;  // not read
    }
    pp.n_items = 0;
    pp.part_o = pp.part_ml = nullptr;
    pp.cnt = nullptr;
    unsigned grid = static_cast<unsigned>(p.n_qtiles - pp.qt_lo) * static_cast<unsigned>(a.hq / 2);
    if (pp.qt_lo == 0 && a.split_ws != nullptr &&
        a.split_ws_bytes >= attn_split_bytes(a.T, a.hq, a.hkv)) {
      const pair::Schedule* schp = pair::cached_schedule(p.n_qtiles, a.hq / 2);
      if (schp != nullptr) {
        const pair::Schedule& sch = *schp;
        const size_t n_pairs = static_cast<size_t>(a.hq / 2);
        const size_t rows = size_t(pair::kMaxSlots) * n_pairs * 2 * kBlk;
        char* base = static_cast<char*>(a.split_ws);
        pp.part_o = reinterpret_cast<float*>(base);
        pp.part_ml = reinterpret_cast<float*>(base + align_up(rows * kDh * 4, 256));
        pp.cnt = reinterpret_cast<unsigned*>(base + split_cnt_offset(a.hq));
        pp.n_items = sch.n_items;
        for (int i = 0; i < sch.n_items; ++i) pp.items[i] = sch.items[i];
        grid = static_cast<unsigned>(sch.n_items) * static_cast<unsigned>(n_pairs);
        if (sch.n_split > 0 && !a.split_cnt_zeroed) {
          const cudaError_t e0 =
              cudaMemsetAsync(pp.cnt, 0, size_t(sch.n_split) * n_pairs * 4, st);
          if (e0 != cudaSuccess) return e0;
        }
      }
    }
    auto kern = bias ? pair::attn_tc_pair<true> : pair::attn_tc_pair<false>;
    const size_t smem = bias ? pair::Layout<true>::kSmem : pair::Layout<false>::kSmem;
    cudaError_t err = set_smem_attr_once(reinterpret_cast<const void*>(kern), int(smem));
    if (err != cudaSuccess) return err;
    // The register split inside the kernel assumes the compiled per-thread
    // count; with any other count setmaxnreg.inc could block, so refuse.
    static std::atomic<int> regs_ok[2];
    std::atomic<int>& ok = regs_ok[bias ? 1 : 0];
    if (ok.load() == 0) {
      cudaFuncAttributes fa;
      err = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern));
      if (err != cudaSuccess) return err;
      ok.store(fa.numRegs == int(pair::kRegsLaunch) ? 1 : -1);
    }
    if (ok.load() < 0) return cudaErrorInvalidConfiguration;
    return launch_pdl(kern, dim3(grid), dim3(pair::kThreads), smem, st, tq, tk, tv, tka, to, pp);
  }
  cudaError_t err = set_smem_attr_once(reinterpret_cast<const void*>(attn_tc), int(kSmem));
  if (err != cudaSuccess) return err;
  const unsigned grid = static_cast<unsigned>(p.n_qtiles) * static_cast<unsigned>(a.hq);
  return launch_pdl(attn_tc, dim3(grid), dim3(kThreads), kSmem, st, tq, tk, tv, p);
}

}  // namespace tg
