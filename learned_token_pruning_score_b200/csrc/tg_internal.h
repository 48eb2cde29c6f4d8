// tg_internal.h -- launchers shared between the kernel files and the C ABI.
// Host code only. Each launcher enqueues work on `st` and returns the launch
// status (cudaSuccess or the CUDA error); argument checks are the caller's.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace tg {

// Rounds `x` up to a multiple of `a` (a power of two).
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) & ~(a - 1); }

// Bump allocator over a caller-provided workspace. carve() returns nullptr
// in size-only mode (base == nullptr) so the same code computes sizes.
struct Arena {
  char* base;
  size_t used;
  explicit Arena(void* b) : base(static_cast<char*>(b)), used(0) {}
  void* carve(size_t bytes) {
    used = align_up(used, 256);
    void* p = base ? base + used : nullptr;
    used += bytes;
    return p;
  }
};

// Enqueues `kernel<<<grid, block, smem, st>>>(args...)` with programmatic
// stream serialization allowed (see pdl_trigger / pdl_wait in
// tg_device.cuh): the kernel may be scheduled, and run its prologue, while
// the previous kernel of the stream drains. Every kernel launched this way
// calls pdl_wait() before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Returns the CUDA error of `expr` from the enclosing launcher, if any.
#define TG_CUDA_TRY(expr)                           \
  do {                                              \
    const cudaError_t tg_e_ = (expr);               \
    if (tg_e_ != cudaSuccess) return tg_e_;         \
  } while (0)

int num_sms();
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device).
cudaError_t set_smem_attr_once(const void* fn, int bytes);
unsigned int* device_error_word();  // device address of the sticky error word

// ---- selection (k_select.cu)
size_t select_ws_bytes(int64_t n);
cudaError_t launch_topk_select(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                               int32_t* kept_idx, void* ws, cudaStream_t st);
// Same selection with its scratch in a static device array (no workspace).
int64_t select_noalloc_max_n();
cudaError_t launch_topk_select_noalloc(const float* scores, const uint8_t* protect, int64_t n,
                                       int64_t k, int32_t* kept_idx, cudaStream_t st);

// ---- compaction (k_compact.cu). Optional lsig_out[r] = logsigmoid(scores[idx[r]]).
// Optional row sums of squares (folded RMSNorm): ss_out[p * ss_ld_out + r] =
// ss_in[p * ss_ld_in + idx[r]] for p < ss_parts.
struct SsGather {
  const float* in = nullptr;
  int64_t ld_in = 0;
  float* out = nullptr;
  int64_t ld_out = 0;
  int parts = 0;
};
cudaError_t launch_compact(const void* x, const int32_t* pos_in, const float* scores,
                           const int32_t* kept_idx, int64_t n, int64_t k, int row_bytes,
                           void* x_out, int32_t* pos_out, float* scores_out, float* lsig_out,
                           const SsGather& ss, cudaStream_t st);

// ---- row-wise kernels (k_rowwise.cu)
// W_g = bf16(W . diag(g)) for bf16 W [rows, cols] (tg_fold_norm_weight)
cudaError_t launch_fold_norm_weight(const void* w, const float* g, int64_t rows, int64_t cols,
                                    void* out, cudaStream_t st);
cudaError_t launch_rmsnorm(const void* x, const float* gamma, float eps, int64_t rows, int d,
                           bool bf16, void* y, cudaStream_t st);

// RoPE/qk-norm preparation of one attention call.
//  src rows: q at q_src + t*q_stride, k at k_src + t*k_stride, v at v_src + t*v_stride
//  (element strides, dtype elements). Writes:
//   q_out [T, hq, dh], k_out [T, hkv, dh] (rotated, optional qk-norm),
//   bf16 only: vT_out [hkv, dh, t_pad] (zero in columns >= T)
//   fp32 only: v_out [T, hkv, dh] (plain copy) when v_out != nullptr
//   kv_v_out [T, hkv, dh] (copy of v) when non-null
//   lsig_out [T] = logsigmoid(s) when s != nullptr
struct RopePrepArgs {
  const void* q_src; const void* k_src; const void* v_src;
  int64_t q_stride, k_stride, v_stride;
  const int32_t* pos;  // nullptr: position = row index
  const float* q_norm; const float* k_norm; float eps;
  int64_t T; int hq, hkv, dh; float rope_base; bool bf16;
  void* q_out; void* k_out; void* vT_out; int64_t t_pad; void* v_out; void* kv_v_out;
  const float* s; float* lsig_out;
};
cudaError_t launch_rope_prep(const RopePrepArgs& a, cudaStream_t st);
// cs[i][t] = (cos, sin)(pos[t] * base^(-2i/dh)), i < dh/2 (frequency-major);
// pos null = row index.
cudaError_t launch_rope_table(const int32_t* pos, int64_t T, int dh, float rope_base, float2* cs,
                              cudaStream_t st);

// Rows of up to kMaxSegs requests packed back to back, each starting at
// off[b] (a multiple of 128) and len[b] rows long: pos[off[b] + i] = i for
// i < len[b], 0 in the padding after each request, for `total` rows.
constexpr int kMaxSegs = 64;
struct SegRows {
  int count;
  int64_t off[kMaxSegs];
  int64_t len[kMaxSegs];
};
cudaError_t launch_segment_positions(const SegRows& s, int64_t total, int32_t* pos,
                                     cudaStream_t st);

// Gate-bias rows for the attention's extra K-step: kaug[t] = (b_hi, b_lo,
// b_hi, b_lo, 0 x 12) in bf16 with b = lsig[t], b_hi = bf16(b),
// b_lo = bf16(b - b_hi).
cudaError_t launch_bias_aug(const float* lsig, int64_t T, void* kaug, cudaStream_t st);

// fp32 helpers used by the SIMT path
cudaError_t launch_swiglu_f32(const float* gu, int64_t rows, int inter, float* h, cudaStream_t st);
cudaError_t launch_score_dot_f32(const float* hpre, int64_t rows, int f, const float* b1,
                                 const float* w2, const float* b2, float* scores, cudaStream_t st);

// ---- GEMMs. C[M,N] = A[M,K] . B[N,K]^T with an epilogue.
enum EpiKind { EPI_STORE = 0, EPI_RESIDUAL = 1, EPI_SWIGLU = 2, EPI_SCORE = 3, EPI_QKV = 4 };
struct GemmArgs {
  const void* A; int64_t lda;      // [M, K] elements, row stride lda
  const void* B; int64_t ldb;      // [N, K]
  void* C; int64_t ldc;            // [M, N] (SWIGLU: [M, N/2]); unused for SCORE
  const void* R; int64_t ldr;      // residual [M, N] (EPI_RESIDUAL), may equal C
  int64_t M; int N; int K;
  EpiKind epi;
  int inter;                       // SWIGLU: I (B rows [0,I) gate, [I,2I) up), N = 2I
  const float* b1; const float* w2; const float* b2; float* scores;  // SCORE
  // QKV (head dim 128): columns [0, hq*128) are q heads, then hkv k heads,
  // then hkv v heads. Writes q_out [M, hq, 128] and k_out [M, hkv, 128]
  // (optional per-head RMSNorm, then RoPE from rope_cs [64][M] (cos, sin)),
  // vT_out [hkv, 128, t_pad] and, if set, v_out [M, hkv, 128].
  int hq, hkv;
  const float2* rope_cs; const float* q_norm; const float* k_norm; float eps;
  void* q_out; void* k_out; void* vT_out; int64_t t_pad; void* v_out;
  int64_t rope_ld = 0;  // stride of rope_cs between frequencies (0: M)
  // Folded RMSNorm (tensor-core path only). RESIDUAL: ss_out[nb * ss_ld + m]
  // = sum of squares of the stored bf16 row m over the tile column block nb
  // (256 columns; ceil(N / 256) blocks). STORE / SWIGLU / SCORE / QKV: when
  // ss_in is set, row m of the accumulator is scaled by
  // 1 / sqrt(ss_inv_n * sum_{p < ss_parts} ss_in[p * ss_ld + m] + ss_eps)
  // before the epilogue's own math (B holding W . diag(g)).
  float* ss_out = nullptr;
  const float* ss_in = nullptr;
  int64_t ss_ld = 0;
  int ss_parts = 0;
  float ss_inv_n = 0.f, ss_eps = 0.f;
};
// tile column blocks of a residual GEMM's row sums of squares
constexpr int kSsBlockCols = 256;
inline int ss_parts_of(int n) { return (n + kSsBlockCols - 1) / kSsBlockCols; }
// bf16 on the 5th-generation tensor cores (k_gemm_tc.cu)
bool gemm_tc_supported(const GemmArgs& g);
cudaError_t launch_gemm_tc(const GemmArgs& g, cudaStream_t st);
// fp32 SIMT (k_gemm_simt.cu); SWIGLU and SCORE are not handled here (the
// caller stores the product and runs the fp32 helpers above).
cudaError_t launch_gemm_simt_f32(const GemmArgs& g, cudaStream_t st);

// ---- attention. q [T,hq,dh] rotated, k [T,hkv,dh] rotated, lsig [T] or null.
struct AttnArgs {
  const void* q; const void* k; const void* v;  // v: bf16 -> vT [hkv, dh, t_pad]; fp32 -> [T,hkv,dh]
  int64_t t_pad;  // bf16: padded token count of vT; fp32: row stride of v in elements (0 = hkv*dh)
  const float* lsig; const float* gain; const float* tau;
  const void* kaug;  // bf16 [T, 16] gate-bias rows (launch_bias_aug of lsig), needed with lsig
  int64_t T; int hq, hkv, dh;
  void* out;                                    // [T, hq, dh]
  float* lse;      // optional [hq, T]: log sum_j exp(l_ij) per row (tensor-core path only)
  float* out_f32;  // optional [T, hq, dh]: the output before rounding (tensor-core path only)
  // optional scratch for split query tiles of short sequences
  // (attn_split_bytes); split_cnt_zeroed: its counters are already zero (the
  // kernel leaves them zero after every launch)
  void* split_ws = nullptr;
  size_t split_ws_bytes = 0;
  bool split_cnt_zeroed = false;
  // First query row of this launch (a multiple of 128; paired-head bf16
  // kernel only): rows [q_lo, T) attend to keys [0, T). Rows below q_lo are
  // neither read as queries nor written.
  int64_t q_lo = 0;
};
// Scratch the tensor-core attention over T rows can use to split long query
// tiles across CTAs (0 when T is too long to need it).
size_t attn_split_bytes(int64_t T, int hq, int hkv);
// Zeroes the split counters of such scratch (before the first launch that
// passes split_cnt_zeroed = true).
cudaError_t attn_split_clear(void* split_ws, size_t split_ws_bytes, int hq, cudaStream_t st);
bool attn_tc_supported(const AttnArgs& a);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st);      // bf16, tcgen05
cudaError_t launch_attn_simt_f32(const AttnArgs& a, cudaStream_t st); // fp32 SIMT

// ---- gated-attention backward (k_attn_bwd.cu): bf16, head_dim 128.
struct AttnBwdArgs {
  const void* q; const void* k;          // [T, hq|hkv, dh] as given to the forward (un-rotated)
  const int32_t* pos; float rope_base;
  const void* v; const void* out; const void* dout;  // [T, hkv|hq, dh]
  const float* out_f32;                  // [T, hq, dh] or null (then D comes from out)
  const float* lse;                      // [hq, T]
  const float* s;                        // [T] scores, or null
  const float* gain; const float* tau;   // [hq] or null
  int64_t T, t_pad; int hq, hkv;
  void* q_rot; void* k_rot;              // workspace [T, hq|hkv, dh], rotated as in the forward
  float2* cs;                            // workspace [dh/2, T] RoPE (cos, sin) table
  void* qT; void* doT;                   // workspace [hq, dh, t_pad] (transposed q, dO)
  float* lse2; float* dd;                // workspace [hq, t_pad]
  float* colsum;                         // workspace [2, hq, t_pad]
  float* qdq;                            // workspace [hq, n_tiles, 8]
  float* bias;                           // workspace [t_pad] logsigmoid(s), zero-padded
  void* dq; void* dk; void* dv;          // outputs [T, H, dh]
  float* ds; float* dgain; float* dtau;  // outputs, each optional
  int64_t qdq_per_head;                  // entries of qdq per head (0: n_tiles * 8)
};
size_t attn_bwd_t_pad(int64_t T);
// stage 0: prep (RoPE, transposes of q and dO, table, lse2, D, bias); 1: dK/dV/C;
// 2: dQ; 3: ds/dgain/dtau.
cudaError_t launch_attn_bwd(const AttnBwdArgs& a, cudaStream_t st, int stage);

// fp32 backward on the CUDA cores (k_attn_bwd_f32.cu), head_dim 64 or 128:
// dq, dk, dv, the per-key sums C (colsum [2, hq, t_pad], second half zero)
// and the per-row q . dq (qdq [hq, T]); ds/dgain/dtau then come from
// launch_attn_bwd stage 3 with qdq_per_head = T.
struct AttnBwdF32Args {
  const float* q_rot; const float* k_rot;  // [T, hq|hkv, dh] rotated
  const float* v; const float* out; const float* dout;
  const float* lse;                        // [hq, T]
  const float* lsig;                       // [T] or null
  const float* gain; const float* tau;
  const float2* cs;                        // [dh/2, T]
  int64_t T, t_pad; int hq, hkv, dh;
  float* colsum; float* qdq;
  float* dq; float* dk; float* dv;
};
cudaError_t launch_attn_bwd_f32(const AttnBwdF32Args& a, cudaStream_t st);

// ---- decode (k_decode.cu): one generated token, batch 1, bf16, head_dim 128.
// One cooperative launch per step runs every layer (see k_decode.cu).
constexpr int kDecodeMaxLayers = 64;
constexpr int kDecodeMaxSplits = 128;
struct DecLayerPtrs {
  const __nv_bfloat16* wqkv;       // [(hq + 2 hkv) 128, d]
  const __nv_bfloat16* wo;         // [d, hq 128]
  const __nv_bfloat16* w_gate_up;  // [2 I, d] or null (no FFN)
  const __nv_bfloat16* w_down;     // [d, I]
  const float* attn_norm;
  const float* ffn_norm;
  const float* q_norm;             // [128] or null
  const float* k_norm;
  const float* gain;               // [hq] or null; used above the gate
  const float* tau;
  __nv_bfloat16* k_cache;          // [>= len + 1, hkv, 128] post-RoPE keys; row len is written
  __nv_bfloat16* v_cache;
  int64_t len;                     // cached rows before this token
};
struct DecStepParams {
  DecLayerPtrs layer[kDecodeMaxLayers];
  int n_layers, d, hq, hkv, dffn, gate_layer;
  float eps, rope_base;
  const float* final_norm;         // [d] or null
  const __nv_bfloat16* x;          // [d] the token's input hidden state
  int64_t pos;                     // its position
  const float* scores;             // [n_scores] prefill gate scores, or null (no bias)
  int64_t n_scores;
  const int32_t* kept_idx;         // [k_kept]: upper-cache row j < k_kept is prompt token kept_idx[j]
  int64_t k_kept;
  __nv_bfloat16* h;                // [d] residual stream
  __nv_bfloat16* qkv;              // [(hq + 2 hkv) 128]
  __nv_bfloat16* o;                // [hq 128] attention output
  __nv_bfloat16* act;              // [I] SwiGLU product
  float* lsig;                     // [k_kept] logsigmoid of the kept prompt tokens' scores
  float* part;                     // [hkv][kDecodeMaxSplits][hq / hkv][130] split softmax states
  unsigned int* merge_cnt;         // [hkv] split counters, zero at launch
  unsigned int* bar;               // [2] grid-barrier counter and abort flag, zero at launch
  int grid, n_split;               // CTAs (one per SM) and key splits per KV head
  int n_slots;                     // weight-stream ring slots (set by the launcher)
  __nv_bfloat16* out;              // [d]
  unsigned int* err;
};
int decode_grid();
int decode_splits(int hkv);
cudaError_t launch_decode_step(const DecStepParams& p, cudaStream_t st);

// Self-tests of the bounded waits (tg_selftest_wait_timeout).
cudaError_t launch_selftest_mbar(unsigned* err, unsigned long long limit_ns, int arrive,
                                 int* result, cudaStream_t st);
cudaError_t launch_selftest_gridbar(unsigned* words, unsigned* err, unsigned long long limit_ns,
                                    int* result, cudaStream_t st);

// ---- Gated DeltaNet mixer (k_gdn.cu)
// One token sequence (the kept tokens of a hybrid model's gated prefill).
// Workspace buffers are fp32, laid out for the recurrence's bulk copies; the
// padded token count t_pad is a multiple of kGdnChunk.
constexpr int kGdnChunk = 32;  // tokens per chunk of the recurrence
constexpr int kGdnLd = 36;     // row stride (floats) of the per-chunk matrices
struct GdnArgs {
  const void* qkv;        // [T, 2 hk dk + hv dv] before the convolution
  const void* z;          // [T, hv dv] output gate
  const void* a;          // [T, hv] decay input
  const void* b;          // [T, hv] write-strength input
  int64_t ld_qkv, ld_z, ld_ab;  // row strides (elements) of qkv, z and a / b
  int64_t T;
  int64_t t_pad;
  int hk, hv, dk, dv, W;
  const float* conv_w;    // [C, W]
  const float* A_log;     // [hv]
  const float* dt_bias;   // [hv]
  const float* norm_w;    // [dv]
  float eps;
  const void* conv_in;    // [W-1, C] or null (zeros)
  void* conv_out;         // [W-1, C] or null
  const float* state_in;  // [hv, dv, dk] or null (zeros)
  float* state_out;       // [hv, dv, dk] or null; may equal state_in
  void* y;                // [T, hv dv]
  float* qn;              // [hk, t_pad, dk]  l2norm(q) / sqrt(dk)
  float* kn;              // [hk, t_pad, dk]  l2norm(k)
  float* vb;              // [hv, dv / 16, t_pad, 16]
  float* gl;              // [hv, t_pad] log decay g
  float* be;              // [hv, t_pad] beta
  float* eg;              // [hv, t_pad] exp of g summed from the chunk start
  float* tt;              // [hv, t_pad / kGdnChunk, kGdnChunk, kGdnLd] per-chunk solve matrix
  float* mm;              // [hv, t_pad / kGdnChunk, kGdnChunk, kGdnLd] per-chunk output matrix
  float* o;               // [T, hv, dv] S_t q_t
  unsigned int* err;
};
// stage 0: prep (+ carried conv rows); 1: chunk matrices; 2: recurrence;
// 3: gated output norm.
cudaError_t launch_gdn(const GdnArgs& a, bool bf16, int stage, cudaStream_t st);

// ---- tensor maps (tg_tmap.cu)
// 2-D bf16 tensor map, row-major [rows, cols] with row stride ld (elements),
// box [box_rows, 64 cols], 128-byte swizzle. Returns false on failure.
bool make_tmap_2d_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                       int box_rows);
// 2-D bf16 tensor map of 16-column rows (row stride ld elements), box
// [box_rows, 16], 32-byte swizzle: one MMA K-step per row.
bool make_tmap_2d_bf16_sw32(CUtensorMap* m, const void* base, int64_t rows, int64_t ld,
                            int box_rows);
// 3-D bf16 tensor map over dims (x fastest): sizes {d0, d1, d2}, byte strides
// {s1, s2} of dims 1 and 2, box {64, b1, b2}, 128-byte swizzle.
bool make_tmap_3d_bf16(CUtensorMap* m, const void* base, int64_t d0, int64_t d1, int64_t d2,
                       int64_t s1_bytes, int64_t s2_bytes, int b1, int b2);

}  // namespace tg
