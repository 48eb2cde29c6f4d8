// k_attn_bwd.cu -- backward of the token-gated causal GQA attention on the
// 5th-generation tensor cores (sm_100a): bf16 operands, fp32 accumulation.
//
// Forward (kept rows i, j in compacted order; positions ascend with the row):
//   l_ij = a_ij + gain_h b_j,  a_ij = (q_i . k_j) / (sqrt(dh) tau_h),  b_j = logsigmoid(s_j)
//   P = softmax_j(l_ij) over j <= i,  o_i = sum_j P_ij v_j
// Backward for the upstream gradient dO, with lse_i = log sum_j exp(l_ij)
// saved by the forward and D_i = dO_i . o_i:
//   P_ij = exp(l_ij - lse_i),  dP_ij = dO_i . v_j,  dl_ij = P_ij (dP_ij - D_i)
//   dq_i = sum_j dl_ij k_j / (sqrt(dh) tau_h)
//   dk_j = sum_{h in group} sum_i dl_ij q_i / (sqrt(dh) tau_h),  dv_j = sum_{h in group} sum_i P_ij dO_i
//   C_hj = sum_i dl_ij:  ds_j = sigmoid(-s_j) sum_h gain_h C_hj,  dgain_h = sum_j b_j C_hj
//   dtau_h = -(1 / tau_h) sum_i q_i . dq_i
// The top-K choice is discrete, but the kept tokens' scores stay in the
// differentiable graph through this bias, which is how the task loss reaches
// the scorer; the per-head gain and temperature are learned along with it
// (Tencent Cloud article "TokenGate：端到端可训练的 Token 剪枝机制，让大模型
// Prefill 提速 11.3 倍", section "门控机制为评分网络建立梯度路径";
// ai.866data.com article "让大模型学会"略读"…", section "可学习剪枝的机制设计").
// q and k are rotated (RoPE at the original positions) before the logits;
// their gradients are rotated back with the transposed rotation.
//
// Kernels, in stream order:
//   bwd_prep   q and k rotated (RoPE at the original positions), q and dO
//              transposed to [head, dh, t_pad] (the K-major B operands of
//              dK and dV), the RoPE table, lse in log2 units,
//              D (from the forward's fp32 output when given: the bf16 output
//              carries a rounding of 2^-9 that D would pass on to every
//              dl_ij of the row), and the zero-padded bias row logsigmoid(s).
//   bwd_dkdv   one CTA per (128-key tile, KV head). For each query head of
//              the group and each query tile at or after the key tile:
//                S^T = K Q^T and dP^T = V dO^T into TMEM (128 columns each);
//                one thread per key row forms P^T and dS^T (dS^T scaled by
//                1 / (sqrt(dh) tau_h)) and writes them back as packed bf16
//                over S^T and dP^T; dV += P^T dO and dK += dS^T Q with A read
//                from TMEM, in two 64-query halves so that the first half
//                overlaps the row math of the second. C_hj is a
//                thread-local sum. (Reading Q and dO MN-major instead of
//                their transposed copies halves this kernel's operand
//                traffic but measured 13-27% slower; keeping K and V in TMEM
//                to double-buffer S^T and dP^T leaves room only for 32-query
//                products, also slower.)
//   bwd_dq     one CTA per (128-query tile, query head); Q and dO in TMEM.
//              Keys up to the diagonal stream through a 4-stage ring (64 per
//              stage): S = Q K^T and dP = dO V^T into one of two TMEM
//              buffers, dS written back over S, dQ += dS K with the same K
//              tile read MN-major (dh contiguous; no transposed copy). Then
//              dq (scaled, rotated back) and per-warp partial sums of
//              q_i . dq_i.
//   bwd_final  ds, dgain, dtau from C and the partial sums, in a fixed
//              order (deterministic: no atomics anywhere).
// Roles in both tensor-core kernels (384 threads): warp 0 TMA producer,
// warp 1 MMA issuer, warp 2 TMEM allocation, warps 4-7 and 8-11 two
// row-math warpgroups (one thread per row each, on half of the columns).
// Every wait is bounded (an expired wait sets the device error word and the
// kernel drains and returns).
#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kBlk = 128;        // rows per tile (queries or keys)
constexpr int kDh = 128;
constexpr int kThreads2 = 384;   // dK/dV and dQ: roles + two row-math warpgroups
constexpr int kSub = 128 * 128;  // bytes of one [128 rows x 64 bf16] 128-byte-swizzled sub-tile
constexpr int kTile = 2 * kSub;  // [128 x 128] bf16 tile
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  int64_t T, t_pad;
  int hq, hkv, n_tiles;
  const float* bias;     // [t_pad] logsigmoid(s_j), zero past T (all zero without scores)
  const float* gain;     // [hq], null: gain 0
  const float* tau;      // [hq], null: tau 1
  const float* lse2;     // [hq, t_pad] lse * log2(e), +inf past T
  const float* dd;       // [hq, t_pad] D_i, 0 past T
  const float2* cs;      // [dh/2, T] RoPE (cos, sin) at each row's position
  __nv_bfloat16* dq;     // [T, hq, dh]
  __nv_bfloat16* dk;     // [T, hkv, dh]
  __nv_bfloat16* dv;     // [T, hkv, dh]
  float* colsum;         // [2, hq, t_pad] C_hj over query halves 0-63 / 64-127, or null
  float* qdq;            // [hq, n_tiles, 8] per-warp partial sums of q_i . dq_i
  unsigned int* err;
};

// Stores 32 fp32 values as bf16 (four 16-byte vectors).
__device__ __forceinline__ void store32_bf16(__nv_bfloat16* dst, const float* x) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 u;
    u.x = pack_bf16x2(x[8 * v + 0], x[8 * v + 1]);
    u.y = pack_bf16x2(x[8 * v + 2], x[8 * v + 3]);
    u.z = pack_bf16x2(x[8 * v + 4], x[8 * v + 5]);
    u.w = pack_bf16x2(x[8 * v + 6], x[8 * v + 7]);
    d[v] = u;
  }
}

// Two TMEM loads of 32 columns (one wait).
__device__ __forceinline__ void tmem_ld2x32(uint32_t ta, uint32_t tb, float (&a)[32],
                                            float (&b)[32]) {
  uint32_t ra[32], rb[32];
  tmem_ld32(ta, ra);
  tmem_ld32(tb, rb);
  tmem_wait_ld_dep(rb);
  tmem_ld_fence(ra);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    a[i] = __uint_as_float(ra[i]);
    b[i] = __uint_as_float(rb[i]);
  }
}

// Rotates the pairs (lo[i], hi[i]) = (x[i0 + i], x[i0 + 64 + i]) of a
// rotated-frame gradient row back through RoPE (frequencies i0 .. i0+31).
__device__ __forceinline__ void rope_back32(float (&lo)[32], float (&hi)[32], const float2* cs,
                                            int64_t T, int64_t row, int i0) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 c = __ldg(cs + static_cast<int64_t>(i0 + i) * T + row);
    const float a = lo[i], b = hi[i];
    lo[i] = a * c.x + b * c.y;
    hi[i] = b * c.x - a * c.y;
  }
}

// Instruction descriptor (bf16 in, fp32 accumulate, M x N) with B read
// MN-major (bit 16).
constexpr uint32_t idesc_bf16_f32_bmn(int m, int n) { return idesc_bf16_f32(m, n) | (1u << 16); }

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzled
// layout: each 128-byte row holds 64 consecutive MN elements of one K index,
// 8-row groups (8 K indices, one swizzle atom) are 1024 bytes apart (stride
// byte offset), and 64-element MN blocks are `lbo` bytes apart (leading byte
// offset). The row-major tiles TMA writes for the K-major products (rows =
// tokens, 128 bytes of dh each) are exactly this layout with tokens as K and
// dh as MN, so one copy serves both products.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);          // start address
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;     // leading byte offset: MN blocks
  d |= static_cast<uint64_t>(1024u >> 4) << 32;               // stride byte offset: 8-row groups
  d |= static_cast<uint64_t>(1u) << 46;                       // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                       // layout: 128-byte swizzle
  return d;
}

// Copies this thread's row r of a [128 x 128] bf16 tile (two 128-byte-
// swizzled [128 x 64] sub-tiles in shared memory) into 64 TMEM columns of
// its lane, two bf16 per column: the A operand of a TS product.
__device__ __forceinline__ void tile_row_to_tmem(const uint8_t* tile, int r, uint32_t taddr) {
#pragma unroll
  for (int hs = 0; hs < 2; ++hs) {
    uint32_t v[32];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 u = *reinterpret_cast<const uint4*>(tile + hs * kSub + r * 128 + ((ch ^ (r & 7)) << 4));
      v[4 * ch + 0] = u.x;
      v[4 * ch + 1] = u.y;
      v[4 * ch + 2] = u.z;
      v[4 * ch + 3] = u.w;
    }
    tmem_st32(taddr + static_cast<uint32_t>(32 * hs), v);
  }
}

// ============================================================================
// dK, dV and C: one CTA per (key tile jt, KV head g), 128 key rows.
// TMEM columns: S^T [0,128), dP^T [128,256), dV [256,384), dK [384,512).
// P^T and dS^T are packed over the first 32 columns of each 64-query half of
// S^T and dP^T (the half's own warpgroup has read them). All 512 columns are in
// use, so the products of one query tile wait for the rows of the previous
// one; the query side is loaded in two halves (stage a: Q, dO for S^T and
// dP^T; stage b: Q^T, dO^T, lse2, D for the rows and dV, dK) so that the
// loads of tile n+1 overlap the work on tile n.
namespace dkdv {
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kTile;
constexpr int kOffQ = kOffV + kTile;     // stage a: Q_i, dO_i
constexpr int kOffDO = kOffQ + kTile;
constexpr int kOffQT = kOffDO + kTile;   // stage b: Q_i^T, dO_i^T, lse2 and D of tile i
constexpr int kOffDOT = kOffQT + kTile;
constexpr int kOffVec = kOffDOT + kTile;
constexpr int kOffBar = kOffVec + 1024;
constexpr size_t kSmem = 1024 + kOffBar + 256;
}  // namespace dkdv

// [128 x 128] x [128 x 128]^T over dh with both operands K-major in shared
// memory (two 64-column swizzled sub-tiles each).
__device__ __forceinline__ void mma_ss_128(uint32_t d, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
#pragma unroll
  for (int kk = 0; kk < kDh / 16; ++kk) {
    const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
    umma_f16_ss(d, sdesc_kmajor_sw128(a_addr + off), sdesc_kmajor_sw128(b_addr + off), idesc,
                kk > 0 ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(kThreads2, 1)
    attn_bwd_dkdv(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmQT,
                  const __grid_constant__ CUtensorMap tmDOT, BwdParams p) {
  using namespace dkdv;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* a_full = bars + 1;
  uint64_t* a_empty = bars + 2;
  uint64_t* b_full = bars + 3;
  uint64_t* b_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_half = bars + 6;  // [2]: P^T, dS^T of queries 0-63 / 64-127 written
  uint64_t* acc_full = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jt = static_cast<int>(blockIdx.x) / p.hkv;  // key tile 0 (the longest) first
  const int g = static_cast<int>(blockIdx.x) % p.hkv;
  const int group = p.hq / p.hkv;
  const int j0 = jt * kBlk;
  const int n_q = p.n_tiles - jt;  // query tiles jt .. n_tiles-1 see this key tile
  const int n_it = group * n_q;

  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    mbar_init(b_full, 1);
    mbar_init(b_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(&p_half[0], 128);
    mbar_init(&p_half[1], 128);
    mbar_init(acc_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmQT);
    tma_prefetch_desc(&tmDOT);
  }
  if (warp == 2) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    mbar_arrive_expect_tx(kv_full, 2 * kTile);
    tma_load_3d(&tmK, kv_full, smem + kOffK, 0, g, j0);
    tma_load_3d(&tmK, kv_full, smem + kOffK + kSub, 64, g, j0);
    tma_load_3d(&tmV, kv_full, smem + kOffV, 0, g, j0);
    tma_load_3d(&tmV, kv_full, smem + kOffV + kSub, 64, g, j0);
    for (int n = 0; n < n_it; ++n) {
      const int h = g * group + n / n_q;
      const int i0 = (jt + n % n_q) * kBlk;
      const uint32_t ph = (n & 1) ^ 1;
      if (!mbar_wait(a_empty, ph, p.err)) break;
      mbar_arrive_expect_tx(a_full, 2 * kTile);
      tma_load_3d(&tmQ, a_full, smem + kOffQ, 0, h, i0);
      tma_load_3d(&tmQ, a_full, smem + kOffQ + kSub, 64, h, i0);
      tma_load_3d(&tmDO, a_full, smem + kOffDO, 0, h, i0);
      tma_load_3d(&tmDO, a_full, smem + kOffDO + kSub, 64, h, i0);
      if (!mbar_wait(b_empty, ph, p.err)) break;
      mbar_arrive_expect_tx(b_full, 2 * kTile + 1024);
      tma_load_3d(&tmQT, b_full, smem + kOffQT, i0, 0, h);
      tma_load_3d(&tmQT, b_full, smem + kOffQT + kSub, i0 + 64, 0, h);
      tma_load_3d(&tmDOT, b_full, smem + kOffDOT, i0, 0, h);
      tma_load_3d(&tmDOT, b_full, smem + kOffDOT + kSub, i0 + 64, 0, h);
      bulk_load(smem + kOffVec, p.lse2 + static_cast<int64_t>(h) * p.t_pad + i0, 512, b_full);
      bulk_load(smem + kOffVec + 512, p.dd + static_cast<int64_t>(h) * p.t_pad + i0, 512, b_full);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    // dV += P^T dO and dK += dS^T Q go in two halves of 64 queries each: the
    // first half runs while the rows of the second are still being formed.
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
    auto grad_half = [&](int half, bool accumulate) {
      const uint32_t dot_addr = smem_addr(smem + kOffDOT) + half * kSub;
      const uint32_t qt_addr = smem_addr(smem + kOffQT) + half * kSub;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // P^T / dS^T of queries 64 half .. + 63: 32 packed columns
        const uint32_t col = static_cast<uint32_t>(half * 64 + kk * 8);
        umma_f16_ts(tmem + 256, tmem + col, sdesc_kmajor_sw128(dot_addr + kk * 32), idesc,
                    (accumulate || kk > 0) ? 1u : 0u);
        umma_f16_ts(tmem + 384, tmem + 128 + col, sdesc_kmajor_sw128(qt_addr + kk * 32), idesc,
                    (accumulate || kk > 0) ? 1u : 0u);
      }
    };
    bool ok = mbar_wait(kv_full, 0, p.err);
    for (int n = 0; n < n_it && ok; ++n) {
      const uint32_t ph = n & 1;
      if (!mbar_wait(a_full, ph, p.err)) break;
      tc_fence_after();
      mma_ss_128(tmem + 0, smem_addr(smem + kOffK), smem_addr(smem + kOffQ));     // S^T
      mma_ss_128(tmem + 128, smem_addr(smem + kOffV), smem_addr(smem + kOffDO));  // dP^T
      umma_commit(s_full);
      umma_commit(a_empty);
      if (!mbar_wait(&p_half[0], ph, p.err) || !mbar_wait(b_full, ph, p.err)) break;
      tc_fence_after();
      grad_half(0, n > 0);
      if (!mbar_wait(&p_half[1], ph, p.err)) break;
      tc_fence_after();
      grad_half(1, true);
      umma_commit(b_empty);
    }
    if (ok) umma_commit(acc_full);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ row math
    // Warpgroup wg (warps 4-7: 0, warps 8-11: 1) forms queries 64 wg .. 64 wg
    // + 63 of every key row (one thread per key row, TMEM lane = row).
    const int wg = (warp - 4) >> 2;
    const int r = (threadIdx.x - 128) & 127;
    const int64_t j = static_cast<int64_t>(j0) + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float* vec_l = reinterpret_cast<const float*>(smem + kOffVec);
    const float* vec_d = vec_l + 128;
    const float bj = __ldg(p.bias + j);  // zero past T
    float csum = 0.f;
    bool ok = true;
    for (int n = 0; n < n_it; ++n) {
      const int h = g * group + n / n_q;
      const int it = jt + n % n_q;
      const uint32_t ph = n & 1;
      const float tau = p.tau ? __ldg(p.tau + h) : 1.0f;
      const float inv_st = 1.0f / (sqrtf(static_cast<float>(kDh)) * tau);
      const float scale2 = kLog2e * inv_st;
      const float b2 = (p.gain ? __ldg(p.gain + h) : 0.0f) * kLog2e * bj;
      if (!mbar_wait_warp(s_full, ph, p.err) || !mbar_wait_warp(b_full, ph, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = it == jt;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * wg + cc;
        uint32_t rs[32], rp[32];
        tmem_ld32(tmem + lane_off + static_cast<uint32_t>(32 * c), rs);
        tmem_ld32(tmem + lane_off + 128u + static_cast<uint32_t>(32 * c), rp);
        tmem_wait_ld_dep(rp);
        tmem_ld_fence(rs);
        uint32_t pk[16], dk16[16];
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const int il = 32 * c + t;
          float p0 = ex2_approx(fmaf(__uint_as_float(rs[t]), scale2, b2) - vec_l[il]);
          float p1 = ex2_approx(fmaf(__uint_as_float(rs[t + 1]), scale2, b2) - vec_l[il + 1]);
          if (diag) {  // query i0 + il sees key j0 + r only when il >= r
            if (il < r) p0 = 0.f;
            if (il + 1 < r) p1 = 0.f;
          }
          const float d0 = p0 * (__uint_as_float(rp[t]) - vec_d[il]);
          const float d1 = p1 * (__uint_as_float(rp[t + 1]) - vec_d[il + 1]);
          csum += d0 + d1;
          pk[t >> 1] = pack_bf16x2(p0, p1);
          dk16[t >> 1] = pack_bf16x2(d0 * inv_st, d1 * inv_st);
        }
        // packed into this warpgroup's own (already read) columns: queries
        // 64 wg + 32 cc .. + 31 at columns 64 wg + 16 cc (P^T) and 128 + the same (dS^T)
        const uint32_t pc = static_cast<uint32_t>(64 * wg + 16 * cc);
        tmem_st16(tmem + lane_off + pc, pk);
        tmem_st16(tmem + lane_off + 128u + pc, dk16);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_half[wg]);
      if (n % n_q == n_q - 1) {  // last query tile of head h: this half's C_hj is complete
        if (p.colsum && j < p.T)
          p.colsum[(static_cast<int64_t>(wg) * p.hq + h) * p.t_pad + j] = csum;
        csum = 0.f;
      }
    }
    if (ok && mbar_wait_warp(acc_full, 0, p.err)) {
      tc_fence_after();
      if (wg == 0) {  // dV
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          float a[32], b[32];
          tmem_ld2x32(tmem + lane_off + 256u + 32u * c, tmem + lane_off + 288u + 32u * c, a, b);
          if (j < p.T) {
            store32_bf16(p.dv + (j * p.hkv + g) * kDh + 32 * c, a);
            store32_bf16(p.dv + (j * p.hkv + g) * kDh + 32 * c + 32, b);
          }
        }
      } else {  // dK, rotated back pair by pair
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float lo[32], hi[32];
          tmem_ld2x32(tmem + lane_off + 384u + 32u * c, tmem + lane_off + 448u + 32u * c, lo, hi);
          if (j < p.T) {
            rope_back32(lo, hi, p.cs, p.T, j, 32 * c);
            store32_bf16(p.dk + (j * p.hkv + g) * kDh + 32 * c, lo);
            store32_bf16(p.dk + (j * p.hkv + g) * kDh + 64 + 32 * c, hi);
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
// dQ: one CTA per (query tile it, query head h), 128 query rows.
// Q and dO sit in TMEM as the A operands; the key side streams through a
// 4-stage ring of 64-key stages, with S and dP double-buffered in TMEM. The
// K tile serves both as the K-major B operand of S and as the MN-major B
// operand of dQ.
// TMEM columns: Q [0,64), dO [64,128) (packed bf16), dQ [128,256), buffer b:
// S [256+128b, +64), dP [320+128b, +64); dS (packed) over columns 0-15
// (keys 0-31) and 32-47 (keys 32-63) of S, each written by the warpgroup
// that read them.
namespace dqk {
constexpr int kHalf64 = 64 * 128;
constexpr int kOffQ = 0;
constexpr int kOffDO = kOffQ + kTile;
constexpr int kOffStage = kOffDO + kTile;
// stage: K [64 x 128], V [64 x 128] (two dh halves each), bias[64]
constexpr int kStK = 0;
constexpr int kStV = kStK + 2 * kHalf64;
constexpr int kStBias = kStV + 2 * kHalf64;
constexpr int kStageBytes = kStBias + 1024;
constexpr uint32_t kStageTx = 2 * 16384 + 256;
constexpr int kStages = 4;
constexpr int kOffBar = kOffStage + kStages * kStageBytes;
constexpr size_t kSmem = 1024 + kOffBar + 256;
constexpr uint32_t kTmQ = 0, kTmDO = 64, kTmDQ = 128, kTmBuf = 256;
}  // namespace dqk

__global__ void __launch_bounds__(kThreads2, 1)
    attn_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                BwdParams p) {
  using namespace dqk;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_ready = bars + 1;     // Q and dO copied into TMEM (256 arrivals)
  uint64_t* st_full = bars + 2;     // [kStages]
  uint64_t* st_empty = bars + 2 + kStages;
  uint64_t* s_full = bars + 2 + 2 * kStages;   // [2]
  uint64_t* p_full = bars + 4 + 2 * kStages;   // [2] (256 arrivals)
  uint64_t* acc_full = bars + 6 + 2 * kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7 + 2 * kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it = p.n_tiles - 1 - static_cast<int>(blockIdx.x) / p.hq;  // longest first
  const int h = static_cast<int>(blockIdx.x) % p.hq;
  const int g = h / (p.hq / p.hkv);
  const int i0 = it * kBlk;
  const int n_sub = 2 * (it + 1);  // 64-key stages up to the diagonal

  pdl_trigger();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_ready, 256);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  if (warp == 2) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    mbar_arrive_expect_tx(q_full, 2 * kTile);
    tma_load_3d(&tmQ, q_full, smem + kOffQ, 0, h, i0);
    tma_load_3d(&tmQ, q_full, smem + kOffQ + kSub, 64, h, i0);
    tma_load_3d(&tmDO, q_full, smem + kOffDO, 0, h, i0);
    tma_load_3d(&tmDO, q_full, smem + kOffDO + kSub, 64, h, i0);
    for (int m = 0; m < n_sub; ++m) {
      const int st = m % kStages;
      const int j0 = 64 * m;
      if (!mbar_wait(&st_empty[st], ((m / kStages) & 1) ^ 1, p.err)) break;
      uint8_t* sb = smem + kOffStage + st * kStageBytes;
      mbar_arrive_expect_tx(&st_full[st], kStageTx);
      tma_load_3d(&tmK, &st_full[st], sb + kStK, 0, g, j0);
      tma_load_3d(&tmK, &st_full[st], sb + kStK + kHalf64, 64, g, j0);
      tma_load_3d(&tmV, &st_full[st], sb + kStV, 0, g, j0);
      tma_load_3d(&tmV, &st_full[st], sb + kStV + kHalf64, 64, g, j0);
      bulk_load(sb + kStBias, p.bias + j0, 256, &st_full[st]);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_n64 = idesc_bf16_f32(128, 64);
    constexpr uint32_t idesc_n128_mn = idesc_bf16_f32_bmn(128, 128);
    auto sp_products = [&](int m) {  // S_b = Q K_m^T, dP_b = dO V_m^T
      const int b = m & 1;
      const uint8_t* sb = smem + kOffStage + (m % kStages) * kStageBytes;
      const uint32_t k_addr = smem_addr(sb + kStK), v_addr = smem_addr(sb + kStV);
      const uint32_t d = tmem + kTmBuf + 128u * b;
#pragma unroll
      for (int kk = 0; kk < kDh / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf64 + (kk & 3) * 32;
        umma_f16_ts(d, tmem + kTmQ + kk * 8, sdesc_kmajor_sw128(k_addr + off), idesc_n64,
                    kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kDh / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf64 + (kk & 3) * 32;
        umma_f16_ts(d + 64u, tmem + kTmDO + kk * 8, sdesc_kmajor_sw128(v_addr + off), idesc_n64,
                    kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[b]);
    };
    auto dq_product = [&](int m) {  // dQ += dS_b K_m, K read MN-major (dh contiguous)
      const int b = m & 1, st = m % kStages;
      const uint32_t k_addr = smem_addr(smem + kOffStage + st * kStageBytes + kStK);
      const uint32_t a = tmem + kTmBuf + 128u * b;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // 16 keys per K-step: 16 rows of 128 bytes
        // dS of keys 0-31 is packed at columns 0-15, of keys 32-63 at 32-47
        const uint32_t col = static_cast<uint32_t>((kk >> 1) * 32 + (kk & 1) * 8);
        umma_f16_ts(tmem + kTmDQ, a + col, sdesc_mnmajor_sw128(k_addr + kk * 2048, kHalf64),
                    idesc_n128_mn, (m > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&st_empty[st]);
    };
    bool ok = mbar_wait(q_ready, 0, p.err);
    for (int m = 0; m < n_sub && ok; ++m) {
      if (!mbar_wait(&st_full[m % kStages], (m / kStages) & 1, p.err)) break;
      tc_fence_after();
      sp_products(m);
      if (m > 0) {
        if (!mbar_wait(&p_full[(m - 1) & 1], ((m - 1) >> 1) & 1, p.err)) break;
        tc_fence_after();
        dq_product(m - 1);
      }
      if (m == n_sub - 1) {
        if (!mbar_wait(&p_full[m & 1], (m >> 1) & 1, p.err)) break;
        tc_fence_after();
        dq_product(m);
        umma_commit(acc_full);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ row math
    // Warpgroup wg (warps 4-7: 0, warps 8-11: 1) forms keys 32 wg .. 32 wg + 31
    // of each 64-key stage for every query row (one thread per row).
    const int wg = (warp - 4) >> 2;
    const int r = (threadIdx.x - 128) & 127;
    const int64_t i = static_cast<int64_t>(i0) + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float tau = p.tau ? __ldg(p.tau + h) : 1.0f;
    const float inv_st = 1.0f / (sqrtf(static_cast<float>(kDh)) * tau);
    const float scale2 = kLog2e * inv_st;
    const float gb2 = p.gain ? __ldg(p.gain + h) * kLog2e : 0.0f;
    const float lse2 = __ldg(p.lse2 + static_cast<int64_t>(h) * p.t_pad + i);
    const float di = __ldg(p.dd + static_cast<int64_t>(h) * p.t_pad + i);
    bool ok = mbar_wait_warp(q_full, 0, p.err);
    if (ok) {  // Q (warpgroup 0) and dO (warpgroup 1) into TMEM
      tile_row_to_tmem(smem + (wg ? kOffDO : kOffQ), r, tmem + lane_off + (wg ? kTmDO : kTmQ));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_ready);
    }
    for (int m = 0; m < n_sub && ok; ++m) {
      const int b = m & 1, st = m % kStages;
      if (!mbar_wait_warp(&s_full[b], (m >> 1) & 1, p.err) ||
          !mbar_wait_warp(&st_full[st], (m / kStages) & 1, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* bias = reinterpret_cast<const float*>(smem + kOffStage + st * kStageBytes +
                                                         kStBias);
      const int lim = static_cast<int>(i - 64 * m);  // key 64m + t is visible when t <= lim
      const uint32_t ta = tmem + lane_off + kTmBuf + 128u * b;
      const int c = wg;
      uint32_t rs[32], rp[32];
      tmem_ld32(ta + 32u * c, rs);
      tmem_ld32(ta + 64u + 32u * c, rp);
      tmem_wait_ld_dep(rp);
      tmem_ld_fence(rs);
      uint32_t dk16[16];
#pragma unroll
      for (int t = 0; t < 32; t += 2) {
        const int jl = 32 * c + t;
        float p0 = ex2_approx(fmaf(__uint_as_float(rs[t]), scale2, gb2 * bias[jl]) - lse2);
        float p1 = ex2_approx(fmaf(__uint_as_float(rs[t + 1]), scale2, gb2 * bias[jl + 1]) - lse2);
        if (jl > lim) p0 = 0.f;
        if (jl + 1 > lim) p1 = 0.f;
        dk16[t >> 1] = pack_bf16x2(p0 * (__uint_as_float(rp[t]) - di),
                                   p1 * (__uint_as_float(rp[t + 1]) - di));
      }
      tmem_st16(ta + 32u * c, dk16);  // into this warpgroup's own (already read) columns
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && mbar_wait_warp(acc_full, 0, p.err)) {
      tc_fence_after();
      // this warpgroup's columns: [32 wg, 32 wg + 32) and [64 + 32 wg, 96 + 32 wg)
      float lo[32], hi[32];
      tmem_ld2x32(tmem + lane_off + kTmDQ + 32u * wg, tmem + lane_off + kTmDQ + 64u + 32u * wg,
                  lo, hi);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        lo[e] *= inv_st;
        hi[e] *= inv_st;
      }
      // q_i . dq_i in the rotated frame (rows past T contribute nothing)
      float dot = 0.f;
      if (i < p.T) {
        const uint8_t* qrow = smem + kOffQ + r * 128;
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int ch = 4 * wg + k4;
            const uint4 u =
                *reinterpret_cast<const uint4*>(qrow + hs * kSub + ((ch ^ (r & 7)) << 4));
            const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const float2 f = __bfloat1622float2(e2[q2]);
              const int d = k4 * 8 + 2 * q2;  // within this warpgroup's 32 columns
              dot = hs ? fmaf(f.x, hi[d], fmaf(f.y, hi[d + 1], dot))
                       : fmaf(f.x, lo[d], fmaf(f.y, lo[d + 1], dot));
            }
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
      if (lane == 0)
        p.qdq[(static_cast<int64_t>(h) * p.n_tiles + it) * 8 + wg * 4 + (warp & 3)] = dot;
      if (i < p.T) {
        rope_back32(lo, hi, p.cs, p.T, i, 32 * wg);
        store32_bf16(p.dq + (i * p.hq + h) * kDh + 32 * wg, lo);
        store32_bf16(p.dq + (i * p.hq + h) * kDh + 64 + 32 * wg, hi);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// ============================================================================
// Prep, one CTA per (64 rows, head slot); the slots are the hq query heads,
// the hkv key heads and the hq heads of dO. Query and key rows are rotated
// by RoPE at their positions (the arithmetic of rope_cos_sin with theta_i
// computed once per CTA) and written row-major for the 128-row operand
// tiles; every slot is also written transposed, [head, dh, t_pad], for the
// K-major operands of the products that contract over rows. The CTAs of
// query head 0 write the (cos, sin) table that rotates the gradients back;
// those of key head 0 the zero-padded bias row logsigmoid(s); those of dO
// lse * log2(e) and D = dO . o per row.
// The [64 x 128] tile sits in shared memory as 32-bit words (two bf16),
// word w of row r at r * 64 + (w ^ (r >> 1)): the row-wise fill and the
// column-wise reads of the transpose (two rows per lane) are both free of
// bank conflicts.
struct PrepArgs {
  const __nv_bfloat16* src[3];  // q, k (un-rotated), dO: [T, H, 128]
  int heads[3];
  __nv_bfloat16* rot[2];        // q_rot, k_rot [T, H, 128]
  __nv_bfloat16* dst[3];        // [H, 128, t_pad]
  const int32_t* pos;
  float rope_base;
  const __nv_bfloat16* out;     // forward output [T, hq, dh]
  const float* out_f32;         // the same before rounding, or null
  const float* lse;             // [hq, T]
  const float* s;               // [T] or null
  float* lse2;                  // [hq, t_pad]
  float* dd;                    // [hq, t_pad]
  float* bias;                  // [t_pad]: logsigmoid(s), zero past T (all zero without s)
  float2* cs;                   // [64, T]
  int64_t T, t_pad;
};

__device__ __forceinline__ float2 rope_cs_theta(int64_t pos, double theta) {
  const double ang = static_cast<double>(pos) * theta;
  const double two_pi = 6.283185307179586476925286766559;
  const double red = ang - two_pi * rint(ang * (1.0 / two_pi));
  float sv, cv;
  sincosf(static_cast<float>(red), &sv, &cv);
  return make_float2(cv, sv);
}

__global__ void __launch_bounds__(256) attn_bwd_prep(PrepArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int kRows = 64;
  __shared__ uint32_t tile[kRows * 64];
  __shared__ double theta[64];
  int slot = blockIdx.y, which = 0;
  while (which < 2 && slot >= a.heads[which]) slot -= a.heads[which++];
  const int h = slot;
  const int H = which == 1 ? a.heads[1] : a.heads[0];
  const __nv_bfloat16* src = which == 0 ? a.src[0] : (which == 1 ? a.src[1] : a.src[2]);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRows;
  if (which < 2 && threadIdx.x < 64)
    theta[threadIdx.x] = exp2(-(2.0 * threadIdx.x / kDh) * log2(static_cast<double>(a.rope_base)));
  __syncthreads();
  __nv_bfloat16* rot = which == 0 ? a.rot[0] : a.rot[1];
  for (int e = threadIdx.x; e < kRows * 32; e += 256) {
    const int r = e >> 5, w = e & 31;  // words w and w + 32: elements (2w, 2w+1) and (2w+64, 2w+65)
    const int64_t t = t0 + r;
    uint32_t lo = 0u, hi = 0u;
    if (t < a.T) {
      const uint32_t* row = reinterpret_cast<const uint32_t*>(src + (t * H + h) * kDh);
      lo = __ldg(row + w);
      hi = __ldg(row + w + 32);
      if (which < 2) {
        const int64_t p = a.pos ? __ldg(a.pos + t) : t;
        const float2 c0 = rope_cs_theta(p, theta[2 * w]);
        const float2 c1 = rope_cs_theta(p, theta[2 * w + 1]);
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lo));
        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
        lo = pack_bf16x2(x.x * c0.x - y.x * c0.y, x.y * c1.x - y.y * c1.y);
        hi = pack_bf16x2(y.x * c0.x + x.x * c0.y, y.y * c1.x + x.y * c1.y);
        uint32_t* rrow = reinterpret_cast<uint32_t*>(rot + (t * H + h) * kDh);
        rrow[w] = lo;
        rrow[w + 32] = hi;
        if (which == 0 && h == 0) {
          a.cs[static_cast<int64_t>(2 * w) * a.T + t] = c0;
          a.cs[static_cast<int64_t>(2 * w + 1) * a.T + t] = c1;
        }
      }
    }
    tile[r * 64 + (w ^ (r >> 1))] = lo;
    tile[r * 64 + ((w + 32) ^ (r >> 1))] = hi;
  }
  if (which == 1 && h == 0 && threadIdx.x < kRows) {
    const int64_t t = t0 + threadIdx.x;
    a.bias[t] = (a.s && t < a.T) ? logsigmoid_f(__ldg(a.s + t)) : 0.0f;
  }
  __syncthreads();
  __nv_bfloat16* dst = a.dst[which] ? a.dst[which] + static_cast<int64_t>(h) * kDh * a.t_pad
                                    : nullptr;
  for (int e = threadIdx.x; dst != nullptr && e < kDh * 32; e += 256) {
    const int d = e >> 5, l = e & 31;  // output row d, rows 2l and 2l + 1 of the tile
    const int w = d >> 1, sh = (d & 1) * 16;
    const uint32_t w0 = tile[(2 * l) * 64 + (w ^ l)];
    const uint32_t w1 = tile[(2 * l + 1) * 64 + (w ^ l)];
    const uint32_t v = ((w0 >> sh) & 0xFFFFu) | (((w1 >> sh) & 0xFFFFu) << 16);
    *reinterpret_cast<uint32_t*>(dst + static_cast<int64_t>(d) * a.t_pad + t0 + 2 * l) = v;
  }
  if (which == 2) {
    // four threads per row, 16 words (32 elements) each
    const int rr = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int64_t t = t0 + rr;
    float acc = 0.f;
    if (t < a.T) {
      const int64_t base = (t * H + h) * kDh;
#pragma unroll 4
      for (int k = 0; k < 16; ++k) {
        const int w = part * 16 + k;
        const uint32_t u = tile[rr * 64 + (w ^ (rr >> 1))];
        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        float2 o;
        if (a.out_f32) {
          o = __ldg(reinterpret_cast<const float2*>(a.out_f32 + base) + w);
        } else {
          const uint32_t ob = __ldg(reinterpret_cast<const uint32_t*>(a.out + base) + w);
          o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ob));
        }
        acc = fmaf(g.x, o.x, fmaf(g.y, o.y, acc));
      }
    }
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 2);
    if (part == 0) {
      const int64_t k = static_cast<int64_t>(h) * a.t_pad + t;
      a.dd[k] = t < a.T ? acc : 0.0f;
      a.lse2[k] = t < a.T ? __ldg(a.lse + static_cast<int64_t>(h) * a.T + t) * kLog2e : INFINITY;
    }
  }
}

// ============================================================================
// ds, dgain, dtau. Blocks [0, hq): one head each (dgain_h, dtau_h); the rest:
// 256 keys each (ds_j). Fixed summation order throughout.
struct FinalArgs {
  const float* s;       // [T] scores (null: no scores)
  const float* bias;    // [t_pad] logsigmoid(s)
  const float* gain;    // [hq] or null
  const float* tau;     // [hq] or null
  const float* colsum;  // [2, hq, t_pad] (two partial sums per entry)
  const float* qdq;     // [hq, per_head] partial sums of q . dq
  int64_t T, t_pad, per_head;
  int hq;
  float* ds;            // [T] or null
  float* dgain;         // [hq] or null
  float* dtau;          // [hq] or null
};

__device__ __forceinline__ float block_sum_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0)
    for (int w = 0; w < 8; ++w) s += red[w];
  __syncthreads();
  return s;  // valid in thread 0
}

__global__ void __launch_bounds__(256) attn_bwd_final(FinalArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  if (static_cast<int>(blockIdx.x) < a.hq) {
    const int h = blockIdx.x;
    float acc = 0.f;
    if (a.s)
      for (int64_t j = threadIdx.x; j < a.T; j += 256)
        acc = fmaf(__ldg(a.bias + j),
                   __ldg(a.colsum + static_cast<int64_t>(h) * a.t_pad + j) +
                       __ldg(a.colsum + static_cast<int64_t>(a.hq + h) * a.t_pad + j),
                   acc);
    const float dg = block_sum_256(acc, red);
    float acc2 = 0.f;
    for (int64_t e = threadIdx.x; e < a.per_head; e += 256)
      acc2 += __ldg(a.qdq + static_cast<int64_t>(h) * a.per_head + e);
    const float qd = block_sum_256(acc2, red);
    if (threadIdx.x == 0) {
      if (a.dgain) a.dgain[h] = dg;
      if (a.dtau) a.dtau[h] = -qd / (a.tau ? __ldg(a.tau + h) : 1.0f);
    }
    return;
  }
  const int64_t j = static_cast<int64_t>(blockIdx.x - a.hq) * 256 + threadIdx.x;
  if (!a.ds || j >= a.T) return;
  float sum = 0.f;
  if (a.gain)
    for (int h = 0; h < a.hq; ++h)
      sum = fmaf(__ldg(a.gain + h),
                 __ldg(a.colsum + static_cast<int64_t>(h) * a.t_pad + j) +
                     __ldg(a.colsum + static_cast<int64_t>(a.hq + h) * a.t_pad + j),
                 sum);
  a.ds[j] = sum / (1.0f + expf(__ldg(a.s + j)));  // sigmoid(-s_j) = 1 / (1 + e^s_j)
}

}  // namespace

size_t attn_bwd_t_pad(int64_t T) { return align_up(static_cast<size_t>(T), kBlk); }

cudaError_t launch_attn_bwd(const AttnBwdArgs& a, cudaStream_t st, int stage) {
  if (a.T <= 0) return cudaSuccess;
  const int64_t e = 2;
  const int n_tiles = static_cast<int>((a.T + kBlk - 1) / kBlk);
  if (stage == 0) {
    PrepArgs pa{};
    pa.src[0] = static_cast<const __nv_bfloat16*>(a.q);
    pa.src[1] = static_cast<const __nv_bfloat16*>(a.k);
    pa.src[2] = static_cast<const __nv_bfloat16*>(a.dout);
    pa.heads[0] = a.hq;
    pa.heads[1] = a.hkv;
    pa.heads[2] = a.hq;
    pa.rot[0] = static_cast<__nv_bfloat16*>(a.q_rot);
    pa.rot[1] = static_cast<__nv_bfloat16*>(a.k_rot);
    pa.dst[0] = static_cast<__nv_bfloat16*>(a.qT);
    pa.dst[1] = nullptr;  // K is read MN-major by dQ: no transposed copy
    pa.dst[2] = static_cast<__nv_bfloat16*>(a.doT);
    pa.pos = a.pos;
    pa.rope_base = a.rope_base;
    pa.out = static_cast<const __nv_bfloat16*>(a.out);
    pa.out_f32 = a.out_f32;
    pa.lse = a.lse;
    pa.s = a.s;
    pa.lse2 = a.lse2;
    pa.dd = a.dd;
    pa.bias = a.bias;
    pa.cs = a.cs;
    pa.T = a.T;
    pa.t_pad = a.t_pad;
    const dim3 grid(static_cast<unsigned>(a.t_pad / 64), static_cast<unsigned>(2 * a.hq + a.hkv));
    TG_CUDA_TRY(launch_pdl(attn_bwd_prep, grid, dim3(256), 0, st, pa));
    return cudaGetLastError();
  }
  BwdParams p{};
  p.T = a.T;
  p.t_pad = a.t_pad;
  p.hq = a.hq;
  p.hkv = a.hkv;
  p.n_tiles = n_tiles;
  p.bias = a.bias;
  p.gain = a.gain;
  p.tau = a.tau;
  p.lse2 = a.lse2;
  p.dd = a.dd;
  p.cs = a.cs;
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.colsum = a.s ? a.colsum : nullptr;
  p.qdq = a.qdq;
  p.err = device_error_word();
  if (stage == 3) {
    FinalArgs f{};
    f.s = a.s;
    f.bias = a.bias;
    f.gain = a.gain;
    f.tau = a.tau;
    f.colsum = a.colsum;
    f.qdq = a.qdq;
    f.T = a.T;
    f.t_pad = a.t_pad;
    f.hq = a.hq;
    f.per_head = a.qdq_per_head > 0 ? a.qdq_per_head : int64_t(n_tiles) * 8;
    f.ds = a.s ? a.ds : nullptr;
    f.dgain = a.dgain;
    f.dtau = a.dtau;
    const unsigned blocks = static_cast<unsigned>(a.hq + (a.ds && a.s ? (a.T + 255) / 256 : 0));
    TG_CUDA_TRY(launch_pdl(attn_bwd_final, dim3(blocks), dim3(256), 0, st, f));
    return cudaGetLastError();
  }
  // row-major [T, H, dh] operands (rows past T read as zeros), as 128-row
  // tiles (the CTA's own rows) and 64-row stages (the streamed side)
  auto rows_map = [&](CUtensorMap* m, const void* base, int heads, int box_rows) {
    return make_tmap_3d_bf16(m, base, kDh, heads, a.T, kDh * e, int64_t(heads) * kDh * e, 1,
                             box_rows);
  };
  // transposed [H, dh, t_pad] operands, loaded as [128 dh x 64 rows] boxes;
  // the inner extent is T, so rows past T read as zeros
  auto cols_map = [&](CUtensorMap* m, const void* base, int heads) {
    return make_tmap_3d_bf16(m, base, a.T, kDh, heads, a.t_pad * e, a.t_pad * kDh * e, kDh, 1);
  };
  if (stage == 1) {
    CUtensorMap tq, tk, tv, tdo, tqT, tdoT;
    if (!rows_map(&tq, a.q_rot, a.hq, kBlk) || !rows_map(&tdo, a.dout, a.hq, kBlk) ||
        !rows_map(&tk, a.k_rot, a.hkv, kBlk) || !rows_map(&tv, a.v, a.hkv, kBlk) ||
        !cols_map(&tqT, a.qT, a.hq) || !cols_map(&tdoT, a.doT, a.hq))
      return cudaErrorInvalidValue;
    cudaError_t err = set_smem_attr_once(reinterpret_cast<const void*>(attn_bwd_dkdv),
                                         int(dkdv::kSmem));
    if (err != cudaSuccess) return err;
    const unsigned grid = static_cast<unsigned>(n_tiles) * static_cast<unsigned>(a.hkv);
    return launch_pdl(attn_bwd_dkdv, dim3(grid), dim3(kThreads2), dkdv::kSmem, st, tq, tk, tv,
                      tdo, tqT, tdoT, p);
  }
  CUtensorMap tq, tk, tv, tdo;
  if (!rows_map(&tq, a.q_rot, a.hq, kBlk) || !rows_map(&tdo, a.dout, a.hq, kBlk) ||
      !rows_map(&tk, a.k_rot, a.hkv, 64) || !rows_map(&tv, a.v, a.hkv, 64))
    return cudaErrorInvalidValue;
  cudaError_t err = set_smem_attr_once(reinterpret_cast<const void*>(attn_bwd_dq), int(dqk::kSmem));
  if (err != cudaSuccess) return err;
  const unsigned grid = static_cast<unsigned>(n_tiles) * static_cast<unsigned>(a.hq);
  return launch_pdl(attn_bwd_dq, dim3(grid), dim3(kThreads2), dqk::kSmem, st, tq, tk, tv, tdo,
                    p);
}

}  // namespace tg
