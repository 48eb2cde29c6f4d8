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
#include <atomic>
#include <type_traits>

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

struct Params {
  int64_t T;
  int hq, hkv;
  int n_qtiles;
  int kv_major;  // 1: CTAs ordered KV-head-major (large T), 0: heaviest tiles first
  const float* gain;
  const float* tau;
  __nv_bfloat16* out;
  float* lse;      // [hq, T] or null
  float* out_f32;  // [T, hq, dh] or null: the output before rounding
  unsigned int* err;
};

template <bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_pair(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKAug,
                 Params p) {
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
  uint64_t* o_full = bars + 13;
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
  if (p.kv_major) {
    const int per_kv = p.n_qtiles * pairs_per_kv;
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
  const int n_kv = qt + 1;
  constexpr uint32_t kKBytes = kTile + (kBias ? kAugTile : 0);

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
    mbar_init(qaug_full, 256);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (kBias) tma_prefetch_desc(&tmKAug);
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
        tma_load_3d(&tmK, &k_full[s], kd, 0, g, j * kBlk);
        tma_load_3d(&tmK, &k_full[s], kd + kSub, 64, g, j * kBlk);
        if (kBias) tma_load_2d(&tmKAug, &k_full[s], smem + kOffKAug + s * kAugTile, 0, j * kBlk);
        if (!mbar_wait(&v_empty[s], ph, p.err)) break;
        uint8_t* vd = smem + kOffV + s * kTile;
        mbar_arrive_expect_tx(&v_full[s], kTile);
        tma_load_3d(&tmV, &v_full[s], vd, j * kBlk, 0, g);
        tma_load_3d(&tmV, &v_full[s], vd + kSub, j * kBlk + 64, 0, g);
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
        if (more) {
          if (!mbar_wait(&k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, p.err)) break;
          tc_fence_after();
          issue_qk(0, j + 1);
        }
        if (!mbar_wait(&p_full[1], j & 1, p.err)) break;
        tc_fence_after();
        issue_pv(1, j);
        umma_commit(&v_empty[s]);
        if (more) {
          issue_qk(1, j + 1);
          umma_commit(&k_empty[(j + 1) & 1]);
        }
      }
      if (ok) umma_commit(o_full);
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
      const int kv0 = j * kBlk;
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
      const bool diag = j == n_kv - 1;
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
    if (ok && mbar_wait_warp(o_full, 0, p.err)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      // log-sum-exp of the row's logits: m and l are in log2 units
      if (p.lse && q_row < p.T) p.lse[head * p.T + q_row] = (m + log2f(l)) * kLn2;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32_wait(tmem + lane_off + o_col + static_cast<uint32_t>(c * 32), o);
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

}  // namespace pair


}  // namespace

bool attn_tc_supported(const AttnArgs& a) {
  auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  return a.dh == kDh && a.hq % a.hkv == 0 && a.t_pad % 64 == 0 && a.t_pad >= a.T && al16(a.q) &&
         al16(a.k) && al16(a.v) && al16(a.out) && a.T < (int64_t(1) << 31) - kBlk;
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
    CUtensorMap tka;
    if (bias) {
      if (a.kaug == nullptr || !make_tmap_2d_bf16_sw32(&tka, a.kaug, a.T, 16, kBlk))
        return cudaErrorInvalidValue;
    } else {
      tka = tk;  // not read
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
    const unsigned grid = static_cast<unsigned>(p.n_qtiles) * static_cast<unsigned>(a.hq / 2);
    return launch_pdl(kern, dim3(grid), dim3(pair::kThreads), smem, st, tq, tk, tv, tka, pp);
  }
  cudaError_t err = set_smem_attr_once(reinterpret_cast<const void*>(attn_tc), int(kSmem));
  if (err != cudaSuccess) return err;
  const unsigned grid = static_cast<unsigned>(p.n_qtiles) * static_cast<unsigned>(a.hq);
  return launch_pdl(attn_tc, dim3(grid), dim3(kThreads), kSmem, st, tq, tk, tv, p);
}

}  // namespace tg
