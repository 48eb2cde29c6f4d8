// k_gemm_tc.cu -- bf16 GEMM on the 5th-generation tensor cores (sm_100a).
//
//   C[M, N] = A[M, K] . B[N, K]^T   (both operands K-major, fp32 accumulate)
//
// Used for every dense contraction of the path: the scorer's first layer,
// QKV, the output projection, SwiGLU gate/up and down. Epilogues fused into
// the TMEM read-out: plain store, residual add (x + W.o), SwiGLU
// (SiLU(gate) * up, with gate and up tiles side by side in one 256-wide
// accumulator), the scorer's tail s = w2 . SiLU(h + b1) + b2 (all F <= 256
// hidden units of a row sit in one accumulator row, so the dot is
// thread-local), and QKV (qk-norm, RoPE, V transposed).
//
// Structure: persistent clusters of two CTAs on two SMs (a CTA pair), 8
// warps each. The pair computes 256 x 256 output tiles with one
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16) per K-step: each CTA stages
// its 128 rows of A and its 128 rows of B, so per SM a K-step reads 32 KB of
// operands from shared memory (a one-SM 128 x 256 tile reads 48 KB) and the
// L2 traffic per FLOP is two thirds of the one-SM kernel's.
//   warp 0    (both)   TMA producer, 6-stage ring of 32 KB stages, 128-byte
//                      swizzle; the bytes of both CTAs count on rank 0's
//                      full barrier.
//   warp 1    (rank 0) MMA issuer: 4 MMAs per stage into a TMEM accumulator,
//                      then commits that free the stage in both CTAs.
//   warp 2    (both)   TMEM allocation: 2 x 256 columns (double-buffered
//                      accumulator, cta_group::2).
//   warps 4-7 (both)   epilogue: tcgen05.ld of their 32-lane quarter of the
//                      CTA's 128 rows, fused op, store; then arrive on rank
//                      0's accumulator-empty barrier.
// The epilogue of tile t overlaps the MMAs of tile t+1.
#include <atomic>

#include "tg_device.cuh"
#include "tg_internal.h"

namespace tg {
namespace {

constexpr int kBK = 64;
constexpr int kThreads = 256;

struct EpiParams {
  int64_t M;
  int N, K, inter;
  void* C;
  int64_t ldc;
  const void* R;
  int64_t ldr;
  const float* b1;
  const float* w2;
  const float* b2;
  float* scores;
  int tiles_m, tiles_n;
  unsigned int* err;
  // EPI_QKV
  int hq, hkv;
  const float2* rope_cs;
  const float* q_norm;
  const float* k_norm;
  float eps;
  __nv_bfloat16* q_out;
  __nv_bfloat16* k_out;
  __nv_bfloat16* vT_out;
  int64_t t_pad;
  __nv_bfloat16* v_out;
  int64_t rope_ld;
  // folded RMSNorm: row sums of squares out (RESIDUAL) / in (the others)
  float* ss_out;
  const float* ss_in;
  int64_t ss_ld;
  int ss_parts;
  float ss_inv_n, ss_eps;
};

__device__ __forceinline__ float round_bf16_f(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ void store32_bf16(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = u;
  }
}

__device__ __forceinline__ void add32_bf16(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = s[q];
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[8 * q + j] += __bfloat162float(e[j]);
  }
}

// The fused epilogue of one accumulator tile, run by one epilogue warp for
// its 32 rows: this thread owns accumulator row `row` (global index), whose
// kBN fp32 columns start at TMEM address `t_row`; `nb` is the tile's column
// block; `stage` (QKV only): the warp's 8 KB of shared memory (1024-byte
// aligned) through which its 32 rows of a q/k head leave in two TMA stores
// (tm_q / tm_k: q_out [M, hq, 128] and k_out [M, hkv, 128], boxes of 64 x 1 x 32).
template <int kBN, int kEpi>
__device__ __forceinline__ void epilogue_tile(const EpiParams& p, int64_t row, uint32_t t_row,
                                              int nb, uint8_t* stage, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k) {
  const bool row_ok = row < p.M;
  // Folded RMSNorm of the input row: B holds W . diag(g), and the row's
  // accumulator is scaled by rs = 1 / sqrt(mean(x^2) + eps), the mean from the
  // producing residual GEMM's per-column-block sums (added in block order).
  float rs = 1.0f;
  if (kEpi != EPI_RESIDUAL && p.ss_in != nullptr && row_ok) {
    float ss = 0.f;
    for (int q = 0; q < p.ss_parts; ++q) ss += __ldcg(p.ss_in + q * p.ss_ld + row);
    rs = rsqrtf(ss * p.ss_inv_n + p.ss_eps);
  }
  if constexpr (kEpi == EPI_STORE || kEpi == EPI_RESIDUAL) {
    float ss = 0.f;  // RESIDUAL: sum of squares of the stored values
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      float v[32];
      tmem_ld32_wait(t_row + c * 32, v);
      const int col = nb * kBN + c * 32;
      if (row_ok && col < p.N) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.C) + row * p.ldc + col;
        if (kEpi == EPI_RESIDUAL) {
          add32_bf16(static_cast<const __nv_bfloat16*>(p.R) + row * p.ldr + col, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float f = round_bf16_f(v[j]);
            ss = fmaf(f, f, ss);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= rs;
        }
        store32_bf16(dst, v);
      }
    }
    if (kEpi == EPI_RESIDUAL && p.ss_out != nullptr && row_ok) p.ss_out[nb * p.ss_ld + row] = ss;
  } else if constexpr (kEpi == EPI_SWIGLU) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float g[32], u[32];
      tmem_ld32_wait(t_row + c * 32, g);
      tmem_ld32_wait(t_row + 128 + c * 32, u);
#pragma unroll
      for (int j = 0; j < 32; ++j) g[j] = silu_f(g[j] * rs) * (u[j] * rs);
      if (row_ok)
        store32_bf16(static_cast<__nv_bfloat16*>(p.C) + row * p.ldc + nb * 128 + c * 32, g);
    }
  } else if constexpr (kEpi == EPI_QKV) {
    // Two whole heads per tile (head dim 128). The accumulator is rounded
    // to bf16 first (the stored-q/k/v value), then q/k get the optional
    // per-head RMSNorm and RoPE; v is written transposed (and as cache).
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      const int hg = nb * 2 + hh;  // head index across the q | k | v columns
      const uint32_t t_head = t_row + static_cast<uint32_t>(hh * 128);
      if (hg < p.hq + p.hkv) {
        const bool is_q = hg < p.hq;
        const float* nw = is_q ? p.q_norm : p.k_norm;
        float rstd = 1.0f;
        if (nw != nullptr) {
          float ss = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tmem_ld32_wait(t_head + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float f = round_bf16_f(v[i] * rs);
              ss = fmaf(f, f, ss);
            }
          }
          rstd = rsqrtf(ss * (1.0f / 128.0f) + p.eps);
        }
        const float2* cs = p.rope_cs + row;  // frequency-major: entry i at cs[i * rope_ld]
        const int lane = static_cast<int>(threadIdx.x & 31);
        // The stage is free once this warp's previous stores have read it.
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        // this thread's row in the stage: two 64-column boxes of 32 rows x 128
        // bytes, 128-byte swizzle (16-byte unit u of row r at u ^ (r & 7))
        uint8_t* srow = stage + lane * 128;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          float lo[32], hi[32];
          tmem_ld32_wait(t_head + c * 32, lo);
          tmem_ld32_wait(t_head + 64 + c * 32, hi);
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int pi = c * 32 + i;
              float a = round_bf16_f(lo[i] * rs) * rstd;
              float b = round_bf16_f(hi[i] * rs) * rstd;
              if (nw != nullptr) {
                a *= __ldg(nw + pi);
                b *= __ldg(nw + pi + 64);
              }
              const float2 t = __ldg(cs + static_cast<int64_t>(pi) * p.rope_ld);
              lo[i] = a * t.x - b * t.y;
              hi[i] = b * t.x + a * t.y;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 ul, uh;
              ul.x = pack_bf16x2(lo[8 * q + 0], lo[8 * q + 1]);
              ul.y = pack_bf16x2(lo[8 * q + 2], lo[8 * q + 3]);
              ul.z = pack_bf16x2(lo[8 * q + 4], lo[8 * q + 5]);
              ul.w = pack_bf16x2(lo[8 * q + 6], lo[8 * q + 7]);
              uh.x = pack_bf16x2(hi[8 * q + 0], hi[8 * q + 1]);
              uh.y = pack_bf16x2(hi[8 * q + 2], hi[8 * q + 3]);
              uh.z = pack_bf16x2(hi[8 * q + 4], hi[8 * q + 5]);
              uh.w = pack_bf16x2(hi[8 * q + 6], hi[8 * q + 7]);
              // dims 32c + 8q (box 0) and 64 + 32c + 8q (box 1): unit 4c + q
              const int u = (4 * c + q) ^ (lane & 7);
              *reinterpret_cast<uint4*>(srow + (u << 4)) = ul;
              *reinterpret_cast<uint4*>(srow + 4096 + (u << 4)) = uh;
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {  // rows past M are not written
          const int64_t row0 = row - lane;
          const CUtensorMap* tm = is_q ? tm_q : tm_k;
          const int head = is_q ? hg : hg - p.hq;
          tma_store_3d(tm, stage, 0, head, static_cast<int>(row0));
          tma_store_3d(tm, stage + 4096, 64, head, static_cast<int>(row0));
          bulk_commit();
        }
      } else {
        const int g = hg - p.hq - p.hkv;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32_wait(t_head + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= rs;
          if (row_ok) {
            if (p.v_out) store32_bf16(p.v_out + (row * p.hkv + g) * 128 + c * 32, v);
            __nv_bfloat16* vt = p.vT_out + (static_cast<int64_t>(g) * 128 + c * 32) * p.t_pad + row;
#pragma unroll
            for (int i = 0; i < 32; ++i) vt[static_cast<int64_t>(i) * p.t_pad] = __float2bfloat16_rn(v[i]);
          }
        }
      }
    }
  } else {  // EPI_SCORE
    float acc = 0.f;
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      float v[32];
      tmem_ld32_wait(t_row + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int f = c * 32 + j;
        if (f < p.N) {
          const float h = v[j] * rs + (p.b1 ? __ldg(p.b1 + f) : 0.f);
          acc = fmaf(__ldg(p.w2 + f), silu_f(h), acc);
        }
      }
    }
    if (row_ok) p.scores[row] = acc + (p.b2 ? __ldg(p.b2) : 0.f);
  }
}

// ------------------------------------------------------------------ kernel
// SWIGLU: rank 0 stages the 128 gate rows of B, rank 1 the matching 128 up
// rows, so accumulator columns [0, 128) hold gate and [128, 256) hold up.
struct PairCfg {
  static constexpr int kHalfBytes = 128 * kBK * 2;       // 128 rows x 64 bf16
  static constexpr int kStageBytes = 2 * kHalfBytes;     // A half + B half
  static constexpr int kStages = 6;
  static constexpr int kTmemCols = 512;                  // 2 x 256 fp32 accumulators
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + 256;
  // QKV: 8 KB per epilogue warp (after the barriers, 1024-aligned) through
  // which its q/k rows leave by TMA
  static constexpr size_t kStageQkv = 1024 - 256 + 4 * 8192;
};
template <int kEpi>
constexpr size_t gemm_smem() {
  return PairCfg::kSmem + (kEpi == EPI_QKV ? PairCfg::kStageQkv : 0);
}

template <int kEpi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmQo, const __grid_constant__ CUtensorMap tmKo,
            EpiParams p) {
  using C = PairCfg;
  constexpr int kBN = 256;
  static_assert(kBN == kSsBlockCols, "row sums of squares are per 256-column block");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled tiles; the offset is the same in
  // both CTAs (same kernel, same static layout).
  const uint32_t raw_addr = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  uint8_t* tiles = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(C::kStages) * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);   // rank 0: its producer's arrive + both CTAs' bytes
      mbar_init(&empty[s], 1);  // one commit from rank 0's MMA thread
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);  // rank 0: 4 epilogue warps x 2 CTAs
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 2) tmem_alloc_pair(tmem_slot, C::kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the previous kernel's outputs (A, the residual) are complete

  const int num_tiles = p.tiles_m * p.tiles_n;
  const int num_kb = (p.K + kBK - 1) / kBK;
  const int pair = static_cast<int>(blockIdx.x >> 1), n_pairs = static_cast<int>(gridDim.x >> 1);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producers
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += n_pairs) {
      const int mb = tile / p.tiles_n, nb = tile % p.tiles_n;
      const int a_row = mb * 256 + static_cast<int>(rank) * 128;
      const int b_row = kEpi == EPI_SWIGLU ? (rank ? p.inter : 0) + nb * 128
                                           : nb * 256 + static_cast<int>(rank) * 128;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err)) { ok = false; break; }
        uint8_t* a_dst = tiles + size_t(s) * C::kStageBytes;
        uint8_t* b_dst = a_dst + C::kHalfBytes;
        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::kStageBytes);
        const uint32_t bar = mapa_shared(smem_addr(&full[s]), 0);
        tma_load_2d_pair(&tmA, bar, a_dst, kb * kBK, a_row);
        tma_load_2d_pair(&tmB, bar, b_dst, kb * kBK, b_row);
        if (++s == C::kStages) { s = 0; ph ^= 1u; }
      }
    }
    // Drain: every stage this CTA filled is released (by a commit that
    // writes into this CTA's shared memory) before the CTA may exit.
    for (int i = 0; i < C::kStages && ok; ++i) {
      if (!mbar_wait(&empty[s], ph ^ 1u, p.err)) break;
      if (++s == C::kStages) { s = 0; ph ^= 1u; }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(256, kBN);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    int it = 0;
    for (int tile = pair; tile < num_tiles && ok; tile += n_pairs, ++it) {
      const int a = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      if (!mbar_wait(&acc_empty[a], (use & 1u) ^ 1u, p.err)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * kBN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[s], ph, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_addr(tiles + size_t(s) * C::kStageBytes);
        const uint32_t b_addr = a_addr + C::kHalfBytes;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          umma_f16_ss_pair(d_tmem, sdesc_kmajor_sw128(a_addr + k * 32),
                           sdesc_kmajor_sw128(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
        }
        const uint32_t e = smem_addr(&empty[s]);
        umma_commit_pair(e);
        umma_commit_pair(mapa_shared(e, 1));
        if (++s == C::kStages) { s = 0; ph ^= 1u; }
      }
      if (ok) {
        const uint32_t f = smem_addr(&acc_full[a]);
        umma_commit_pair(f);
        umma_commit_pair(mapa_shared(f, 1));
      }
    }
    // Drain: both accumulators released by both CTAs' epilogues (their
    // arrivals write into this CTA's shared memory) before exit.
    for (int i = 0; i < 2 && ok; ++i, ++it) {
      const int a = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      if (!mbar_wait(&acc_empty[a], (use & 1u) ^ 1u, p.err)) break;
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += n_pairs, ++it) {
      const int mb = tile / p.tiles_n, nb = tile % p.tiles_n;
      const int a = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      if (!mbar_wait_warp(&acc_full[a], use & 1u, p.err)) break;
      tc_fence_after();
      const int64_t row =
          static_cast<int64_t>(mb) * 256 + static_cast<int64_t>(rank) * 128 + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(a * kBN);
      uint8_t* stage = kEpi == EPI_QKV
                           ? tiles + size_t(C::kStages) * C::kStageBytes + 1024 + quarter * 8192
                           : nullptr;
      epilogue_tile<kBN, kEpi>(p, row, t_row, nb, stage, &tmQo, &tmKo);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&acc_empty[a]), 0));
    }
    // the last TMA stores have read this warp's stage before the CTA exits
    if (kEpi == EPI_QKV && lane == 0) bulk_wait_read_all();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  __syncwarp();
  if (warp == 2) tmem_dealloc_pair(tmem_base, C::kTmemCols);
}

template <int kEpi>
cudaError_t run(const GemmArgs& g, cudaStream_t st) {
  using C = PairCfg;
  CUtensorMap ta, tb, tqo, tko;
  if (!make_tmap_2d_bf16(&ta, g.A, g.M, g.K, g.lda, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, g.B, g.N, g.K, g.ldb, 128)) return cudaErrorInvalidValue;
  if (kEpi == EPI_QKV) {  // q_out [M, hq, 128] and k_out [M, hkv, 128], 32-row boxes
    if (!make_tmap_3d_bf16(&tqo, g.q_out, 128, g.hq, g.M, 256, int64_t(g.hq) * 256, 1, 32) ||
        !make_tmap_3d_bf16(&tko, g.k_out, 128, g.hkv, g.M, 256, int64_t(g.hkv) * 256, 1, 32))
      return cudaErrorInvalidValue;
  } else {
    tqo = ta;  // not read
    tko = ta;
  }
  EpiParams p;
  p.M = g.M;
  p.N = kEpi == EPI_SWIGLU ? g.inter : g.N;
  p.K = g.K;
  p.inter = g.inter;
  p.C = g.C;
  p.ldc = g.ldc;
  p.R = g.R;
  p.ldr = g.ldr;
  p.b1 = g.b1;
  p.w2 = g.w2;
  p.b2 = g.b2;
  p.scores = g.scores;
  p.hq = g.hq;
  p.hkv = g.hkv;
  p.rope_cs = g.rope_cs;
  p.q_norm = g.q_norm;
  p.k_norm = g.k_norm;
  p.eps = g.eps;
  p.q_out = static_cast<__nv_bfloat16*>(g.q_out);
  p.k_out = static_cast<__nv_bfloat16*>(g.k_out);
  p.vT_out = static_cast<__nv_bfloat16*>(g.vT_out);
  p.t_pad = g.t_pad;
  p.v_out = static_cast<__nv_bfloat16*>(g.v_out);
  p.rope_ld = g.rope_ld > 0 ? g.rope_ld : g.M;
  p.ss_out = g.ss_out;
  p.ss_in = g.ss_in;
  p.ss_ld = g.ss_ld;
  p.ss_parts = g.ss_parts;
  p.ss_inv_n = g.ss_inv_n;
  p.ss_eps = g.ss_eps;
  p.tiles_m = static_cast<int>((g.M + 255) / 256);
  p.tiles_n = kEpi == EPI_SWIGLU ? g.inter / 128 : (g.N + 255) / 256;
  p.err = device_error_word();
  const int tiles = p.tiles_m * p.tiles_n;
  if (tiles == 0) return cudaSuccess;
  auto kern = gemm_tc<kEpi>;
  constexpr size_t kSmemBytes = gemm_smem<kEpi>();
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  cudaError_t e = set_smem_attr_once(reinterpret_cast<const void*>(kern), static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  // Persistent grid: as many pairs as can be resident at once (the SMs of a
  // pair must share a TPC, so this can be below num_sms() / 2).
  constexpr int kMaxDevices = 64;
  static std::atomic<int> resident[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  int max_pairs = (dev >= 0 && dev < kMaxDevices) ? resident[dev].load() : 0;
  if (max_pairs <= 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    if (cudaOccupancyMaxActiveClusters(&max_pairs, kern, &cfg) != cudaSuccess || max_pairs <= 0) {
      cudaGetLastError();
      max_pairs = num_sms() / 2;
    }
    if (dev >= 0 && dev < kMaxDevices) resident[dev].store(max_pairs);
  }
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  return launch_pdl(kern, dim3(2 * pairs), dim3(kThreads), kSmemBytes, st, ta, tb, tqo, tko, p);
}

}  // namespace

bool gemm_tc_supported(const GemmArgs& g) {
  // TMA: 16-byte aligned bases and row strides.
  auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (!al16(g.A) || !al16(g.B) || (g.lda % 8) || (g.ldb % 8) || g.K % 8 || g.K <= 0) return false;
  switch (g.epi) {
    case EPI_STORE:
    case EPI_RESIDUAL:
      return g.N % 32 == 0 && al16(g.C) && g.ldc % 8 == 0 &&
             (g.epi == EPI_STORE || (al16(g.R) && g.ldr % 8 == 0));
    case EPI_SWIGLU:
      return g.inter % 128 == 0 && g.N == 2 * g.inter && al16(g.C) && g.ldc % 8 == 0;
    case EPI_SCORE:
      return g.N >= 1 && g.N <= 256 && g.scores != nullptr && g.w2 != nullptr;
    case EPI_QKV:
      return g.hq > 0 && g.hkv > 0 && g.hq % 2 == 0 && g.N == (g.hq + 2 * g.hkv) * 128 &&
             g.rope_cs != nullptr && al16(g.q_out) && al16(g.k_out) && g.vT_out != nullptr &&
             g.t_pad >= g.M && (g.v_out == nullptr || al16(g.v_out));
  }
  return false;
}

cudaError_t launch_gemm_tc(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0) return cudaSuccess;
  switch (g.epi) {
    case EPI_STORE: return run<EPI_STORE>(g, st);
    case EPI_RESIDUAL: return run<EPI_RESIDUAL>(g, st);
    case EPI_SWIGLU: return run<EPI_SWIGLU>(g, st);
    case EPI_SCORE: return run<EPI_SCORE>(g, st);
    case EPI_QKV: return run<EPI_QKV>(g, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tg
