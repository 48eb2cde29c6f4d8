// k_select.cu -- deterministic top-K selection with protected tokens.
//
// The top-K selector keeps the K best-scoring tokens and never drops the
// protected (question) span (Tencent Cloud article "TokenGate：端到端可训练的
// Token 剪枝机制，让大模型 Prefill 提速 11.3 倍", section "TokenGate 提前筛选
// Token"; ai.866data.com article "让大模型学会"略读"…", section
// "可学习剪枝的机制设计"). Ranking is (score descending, index ascending),
// with -0.0 == +0.0 and NaN lowest.
//
// Method: radix select over the 32-bit order-preserving key of each fp32
// score. Up to 131072 tokens (sel_cluster): one launch of one CTA or one
// thread-block cluster, keys in registers, four 8-bit digits with one
// cluster barrier each. Above that (sel_hist0 ... sel_write): five kernels
// over the key stream in three digits (11, 11, 10 bits). Each pass
// histograms the next digit of the keys that still match the prefix found
// so far; every CTA finds the threshold bin from the finished histogram of
// the previous pass (identical work, identical result), so no CTA waits on
// another. The last step counts, per chunk, the tokens kept for sure and the
// tokens tied at the threshold key, then writes the kept indices in index
// order: the tied tokens taken are the lowest-index ones. Integer atomics
// only, so the result is bit-reproducible.
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "tg_device.cuh"
#include "tg_internal.h"
#include "tokengate.h"

namespace tg {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kChunk = kThreads * kPerThread;  // tokens per CTA

// Workspace layout (32-bit words).
struct SelState {
  int32_t status;    // 0 = ok, 3 = more protected tokens than k
  uint32_t n_prot;   // protected count (atomic sum)
  uint32_t prefix;   // key bits found so far
  uint32_t need;     // unprotected tokens still to take at/below prefix
  uint32_t thresh;   // final threshold key
  uint32_t ties;     // tokens with key == thresh to take (lowest indices)
  uint32_t pad[2];
};
constexpr int kHist0 = 2048, kHist1 = 2048, kHist2 = 1024;
constexpr size_t kOffHist0 = sizeof(SelState);
constexpr size_t kOffHist1 = kOffHist0 + kHist0 * 4;
constexpr size_t kOffHist2 = kOffHist1 + kHist1 * 4;
constexpr size_t kOffCounts = kOffHist2 + kHist2 * 4;  // then 2 x C words
constexpr size_t kZeroBytes = kOffCounts;

struct Ws {
  SelState* st;
  uint32_t* h0;
  uint32_t* h1;
  uint32_t* h2;
  uint32_t* n_def;  // [C] tokens kept for sure in chunk c
  uint32_t* n_tie;  // [C] unprotected tokens with key == thresh in chunk c
};

__host__ __device__ inline Ws ws_view(void* base, int64_t chunks) {
  char* b = static_cast<char*>(base);
  Ws w;
  w.st = reinterpret_cast<SelState*>(b);
  w.h0 = reinterpret_cast<uint32_t*>(b + kOffHist0);
  w.h1 = reinterpret_cast<uint32_t*>(b + kOffHist1);
  w.h2 = reinterpret_cast<uint32_t*>(b + kOffHist2);
  w.n_def = reinterpret_cast<uint32_t*>(b + kOffCounts);
  w.n_tie = w.n_def + chunks;
  return w;
}

// Loads this thread's 8 tokens: keys (protected tokens flagged separately).
template <bool kVec>
__device__ __forceinline__ int load_tokens(const float* __restrict__ scores,
                                           const uint8_t* __restrict__ protect, int64_t n,
                                           int64_t first, uint32_t (&key)[kPerThread],
                                           bool (&prot)[kPerThread]) {
  int valid = 0;
  if (kVec && first + kPerThread <= n) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(scores + first));
    const float4 b = __ldg(reinterpret_cast<const float4*>(scores + first) + 1);
    const float s[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint2 pm = make_uint2(0u, 0u);
    if (protect) pm = __ldg(reinterpret_cast<const uint2*>(protect + first));
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      key[j] = score_key(s[j]);
      const uint32_t word = j < 4 ? pm.x : pm.y;
      prot[j] = ((word >> (8 * (j & 3))) & 0xFFu) != 0u;
    }
    valid = kPerThread;
  } else {
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      const int64_t i = first + j;
      if (i < n) {
        key[j] = score_key(__ldg(scores + i));
        prot[j] = protect ? (__ldg(protect + i) != 0) : false;
        ++valid;
      } else {
        key[j] = 0u;
        prot[j] = false;
      }
    }
  }
  return valid;
}

// Exclusive prefix sum over the CTA (thread order). Returns this thread's
// exclusive prefix; *total receives the CTA sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* total) {
  __shared__ uint32_t warp_sums[kThreads / 32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < kThreads / 32 ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kThreads / 32) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const uint32_t before_warp = wid ? warp_sums[wid - 1] : 0u;
  if (total) *total = warp_sums[kThreads / 32 - 1];
  const uint32_t r = before_warp + x - v;
  __syncthreads();
  return r;
}

// Finds, scanning bins from the highest, the bin b* where the running count
// of higher bins is < need and reaches need inside b*. Returns b* and the
// rank left inside it (need - count above). Every thread gets the result.
template <int kBins>
__device__ __forceinline__ void find_bin(const uint32_t* __restrict__ hist, uint32_t need,
                                         uint32_t* bin_out, uint32_t* need_out) {
  constexpr int kPer = kBins / kThreads;
  __shared__ uint32_t s_bin, s_need;
  uint32_t h[kPer];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    h[j] = hist[kBins - 1 - (threadIdx.x * kPer + j)];  // descending bins
    local += h[j];
  }
  if (threadIdx.x == 0) {
    s_bin = 0u;
    s_need = need;
  }
  uint32_t total;
  const uint32_t before = block_excl_scan(local, &total);
  if (before < need && need <= before + local) {
    uint32_t run = before;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (run + h[j] >= need) {
        s_bin = static_cast<uint32_t>(kBins - 1 - (threadIdx.x * kPer + j));
        s_need = need - run;
        break;
      }
      run += h[j];
    }
  }
  __syncthreads();
  *bin_out = s_bin;
  *need_out = s_need;
}

// Pass 0: protected count and the top-digit histogram.
template <bool kVec>
__global__ void __launch_bounds__(kThreads) sel_hist0(const float* __restrict__ scores,
                                                      const uint8_t* __restrict__ protect,
                                                      int64_t n, Ws w) {
  pdl_trigger();
  pdl_wait();
  __shared__ uint32_t hist[kHist0];
  for (int i = threadIdx.x; i < kHist0; i += kThreads) hist[i] = 0u;
  __syncthreads();
  uint32_t key[kPerThread];
  bool prot[kPerThread];
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kChunk + threadIdx.x * kPerThread;
  const int valid = load_tokens<kVec>(scores, protect, n, first, key, prot);
  uint32_t np = 0;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    if (j < valid) {
      if (prot[j]) ++np;
      else atomicAdd(&hist[key[j] >> 21], 1u);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) np += __shfl_xor_sync(0xFFFFFFFFu, np, o);
  if ((threadIdx.x & 31) == 0 && np) atomicAdd(&w.st->n_prot, np);
  __syncthreads();
  for (int i = threadIdx.x; i < kHist0; i += kThreads)
    if (hist[i]) atomicAdd(&w.h0[i], hist[i]);
}

// Pass 1 / 2: find the previous digit, histogram the next one.
template <bool kVec, int kPass>
__global__ void __launch_bounds__(kThreads) sel_hist_next(const float* __restrict__ scores,
                                                          const uint8_t* __restrict__ protect,
                                                          int64_t n, int64_t k, Ws w) {
  pdl_trigger();
  pdl_wait();
  constexpr int kBinsPrev = kPass == 1 ? kHist0 : kHist1;
  constexpr int kBinsNext = kPass == 1 ? kHist1 : kHist2;
  __shared__ uint32_t hist[kBinsNext];
  uint32_t need, prefix;
  if (kPass == 1) {
    const int64_t np = w.st->n_prot;
    if (np > k) {
      if (blockIdx.x == 0 && threadIdx.x == 0) w.st->status = 3;
      return;
    }
    need = static_cast<uint32_t>(k - np);
    prefix = 0u;
  } else {
    if (w.st->status != 0) return;
    need = w.st->need;
    prefix = w.st->prefix;
  }
  if (need == 0u) return;  // nothing unprotected to keep
  uint32_t bin, rest;
  find_bin<kBinsPrev>(kPass == 1 ? w.h0 : w.h1, need, &bin, &rest);
  const uint32_t new_prefix = kPass == 1 ? bin : ((prefix << 11) | bin);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    w.st->prefix = new_prefix;
    w.st->need = rest;
  }
  for (int i = threadIdx.x; i < kBinsNext; i += kThreads) hist[i] = 0u;
  __syncthreads();
  uint32_t key[kPerThread];
  bool prot[kPerThread];
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kChunk + threadIdx.x * kPerThread;
  const int valid = load_tokens<kVec>(scores, protect, n, first, key, prot);
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    if (j < valid && !prot[j]) {
      if (kPass == 1) {
        if ((key[j] >> 21) == new_prefix) atomicAdd(&hist[(key[j] >> 10) & 0x7FFu], 1u);
      } else {
        if ((key[j] >> 10) == new_prefix) atomicAdd(&hist[key[j] & 0x3FFu], 1u);
      }
    }
  }
  __syncthreads();
  uint32_t* gh = kPass == 1 ? w.h1 : w.h2;
  for (int i = threadIdx.x; i < kBinsNext; i += kThreads)
    if (hist[i]) atomicAdd(&gh[i], hist[i]);
}

// Final digit, then per-chunk counts of sure keeps and threshold ties.
template <bool kVec>
__global__ void __launch_bounds__(kThreads) sel_count(const float* __restrict__ scores,
                                                      const uint8_t* __restrict__ protect,
                                                      int64_t n, int64_t k, Ws w) {
  pdl_trigger();
  pdl_wait();
  if (w.st->status != 0) return;
  const int64_t np = w.st->n_prot;
  uint32_t thresh, ties;
  if (static_cast<int64_t>(np) == k) {
    thresh = 0xFFFFFFFFu;  // no unprotected token is kept
    ties = 0u;
  } else {
    uint32_t bin, rest;
    find_bin<kHist2>(w.h2, w.st->need, &bin, &rest);
    thresh = (w.st->prefix << 10) | bin;
    ties = rest;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    w.st->thresh = thresh;
    w.st->ties = ties;
  }
  uint32_t key[kPerThread];
  bool prot[kPerThread];
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kChunk + threadIdx.x * kPerThread;
  const int valid = load_tokens<kVec>(scores, protect, n, first, key, prot);
  uint32_t nd = 0, nt = 0;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    if (j < valid) {
      if (prot[j] || key[j] > thresh) ++nd;
      else if (key[j] == thresh) ++nt;
    }
  }
  uint32_t td, tt;
  block_excl_scan(nd, &td);
  block_excl_scan(nt, &tt);
  if (threadIdx.x == 0) {
    w.n_def[blockIdx.x] = td;
    w.n_tie[blockIdx.x] = tt;
  }
}

// Writes the kept indices of this chunk, in index order, at their global rank.
template <bool kVec>
__global__ void __launch_bounds__(kThreads) sel_write(const float* __restrict__ scores,
                                                      const uint8_t* __restrict__ protect,
                                                      int64_t n, int64_t k,
                                                      int32_t* __restrict__ kept_idx, Ws w) {
  pdl_trigger();
  pdl_wait();
  if (w.st->status != 0) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < k;
         i += static_cast<int64_t>(gridDim.x) * kThreads)
      kept_idx[i] = -1;
    return;
  }
  const uint32_t thresh = w.st->thresh, ties = w.st->ties;
  // Bases from the chunks before this one: ties seen before this chunk, and
  // kept tokens before it, where chunk c keeps n_def[c] plus
  // clamp(ties - ties_before(c), 0, n_tie[c]) of its tied tokens.
  uint32_t tie_base = 0, out_base = 0;
  for (uint32_t g = 0; g < blockIdx.x; g += kThreads) {
    const uint32_t c = g + threadIdx.x;
    const bool in = c < blockIdx.x;
    const uint32_t nt = in ? w.n_tie[c] : 0u;
    uint32_t group_ties, group_out;
    const uint32_t before = tie_base + block_excl_scan(nt, &group_ties);
    uint32_t take = 0;
    if (in && before < ties) take = min(nt, ties - before);
    const uint32_t contrib = in ? w.n_def[c] + take : 0u;
    block_excl_scan(contrib, &group_out);
    tie_base += group_ties;
    out_base += group_out;
  }
  uint32_t key[kPerThread];
  bool prot[kPerThread];
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kChunk + threadIdx.x * kPerThread;
  const int valid = load_tokens<kVec>(scores, protect, n, first, key, prot);
  uint32_t lt = 0;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j)
    if (j < valid && !prot[j] && key[j] == thresh) ++lt;
  uint32_t dummy;
  const uint32_t tie_before = tie_base + block_excl_scan(lt, &dummy);
  bool keep[kPerThread];
  uint32_t lk = 0, run = tie_before;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    bool kp = false;
    if (j < valid) {
      if (prot[j] || key[j] > thresh) {
        kp = true;
      } else if (key[j] == thresh) {
        kp = run < ties;
        ++run;
      }
    }
    keep[j] = kp;
    lk += kp ? 1u : 0u;
  }
  uint32_t pos = out_base + block_excl_scan(lk, &dummy);
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    if (keep[j]) {
      if (pos < static_cast<uint64_t>(k)) kept_idx[pos] = static_cast<int32_t>(first + j);
      ++pos;
    }
  }
}

// ---------------------------------------------------------------------------
// One-launch selection for n <= kClusterMaxN: one thread-block cluster of C
// CTAs (C = 1, 2, 4, 8 or 16; 8192 tokens per CTA, 8 per thread) holds every
// key in registers, so the scores are read once. Each radix pass builds a
// per-CTA shared-memory histogram of the next digit; CTA c then sums slice c
// of the bins over the cluster's CTAs (distributed shared memory), every CTA
// finds the slice and then the bin where the count from the top reaches the
// rank still needed, and the next pass refines that prefix. After the three
// digits (11, 11, 10 bits) the threshold key and the number of tied tokens
// to take are known; the CTAs exchange their counts of sure keeps and ties
// and write the kept indices in index order. No global scratch besides the
// status word; cluster barriers (hardware, all CTAs co-resident) separate
// the steps.
constexpr int kCThreads = 1024;
constexpr int kCChunk = kCThreads * kPerThread;  // tokens per CTA
constexpr int kCMaxCtas = 16;
constexpr int64_t kClusterMaxN = int64_t(kCMaxCtas) * kCChunk;  // 131072

// Exclusive prefix over the 1024 threads of a CTA (thread order); *total
// receives the CTA sum. Uses the caller's 32-word scratch.
__device__ __forceinline__ uint32_t cta_excl_scan_1024(uint32_t v, uint32_t* total,
                                                       uint32_t* warp_sums) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const uint32_t before_warp = wid ? warp_sums[wid - 1] : 0u;
  if (total) *total = warp_sums[31];
  const uint32_t r = before_warp + x - v;
  __syncthreads();
  return r;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// kOne: a single CTA (no cluster), whose barriers are plain __syncthreads
// and whose "remote" shared memory is its own.
template <bool kOne>
__device__ __forceinline__ void sel_sync() {
  if (kOne) __syncthreads();
  else cluster_sync();
}
template <bool kOne>
__device__ __forceinline__ uint32_t ld_rank(const uint32_t* p, uint32_t rank) {
  if (kOne) return *reinterpret_cast<const volatile uint32_t*>(p);
  return ld_cluster_u32(mapa_shared(smem_addr(p), rank));
}

// One launch, four 8-bit digits, most significant first. Pass p histograms
// digit p of the unprotected keys that match the digits found so far into
// hist[p & 1] (pass 0 also counts the CTA's protected tokens, in bin 256).
// One barrier over the cluster per pass; then every CTA sums the cluster's
// counts itself and its warp 0 scans the 256 bins from the top for the bin
// where the count reaches `need`, so no second exchange is needed. A buffer
// is zeroed again in the pass after its use, once every CTA has passed that
// pass's barrier and so has finished reading it. kPer tokens per thread (a
// multiple of 8).
constexpr int kRBins = 260;  // 256 digit bins + the protected count, padded
template <bool kVec, int kPer, bool kOne>
__global__ void __launch_bounds__(kCThreads, 1)
    sel_cluster(const float* __restrict__ scores, const uint8_t* __restrict__ protect, int64_t n,
                int64_t k, int32_t* __restrict__ kept_idx, int32_t* __restrict__ status) {
  __shared__ uint32_t hist[2 * kRBins];  // this CTA's counts, even / odd passes
  __shared__ uint32_t red[kRBins];       // the cluster's counts of the current pass
  __shared__ uint32_t cta_val[2];        // [1]: the CTA's sure keeps | ties (16 + 16 bits)
  __shared__ uint32_t tot[kCMaxCtas];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_bin, s_need, s_stop;
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t C = gridDim.x;  // the grid is one cluster
  const uint32_t rank = kOne ? 0u : cluster_ctarank();
  for (int i = tid; i < 2 * kRBins; i += kCThreads) hist[i] = 0u;
  __syncthreads();
  pdl_wait();
  static_assert(kPer % kPerThread == 0 && kPer <= 16, "tokens per thread");
  uint32_t key[kPer];
  uint32_t pmask = 0u;  // bit j: token j of this thread is protected
  const int64_t first = static_cast<int64_t>(rank) * kCThreads * kPer + static_cast<int64_t>(tid) * kPer;
  int valid = 0;  // tokens of this thread that exist (a prefix of its kPer)
#pragma unroll
  for (int q = 0; q < kPer / kPerThread; ++q) {
    uint32_t kq[kPerThread];
    bool pq[kPerThread];
    valid += load_tokens<kVec>(scores, protect, n, first + q * kPerThread, kq, pq);
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      key[q * kPerThread + j] = kq[j];
      if (pq[j]) pmask |= 1u << (q * kPerThread + j);
    }
  }
  uint32_t np_w = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if (j < valid && ((pmask >> j) & 1u)) ++np_w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) np_w += __shfl_xor_sync(0xFFFFFFFFu, np_w, o);
  bool over = false;
  uint32_t prefix = 0u, need = 0u;
  uint32_t thresh = 0xFFFFFFFFu, ties = 0u;  // no unprotected token kept
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    uint32_t* h = hist + (pass & 1) * kRBins;
    const int shift = 24 - 8 * pass;
    if (pass == 0 && lane == 0 && np_w) atomicAdd(&h[256], np_w);
    // A warp whose keys are all active and in one bin (a run of tied
    // scores) adds once, a warp with no active key skips the pass; otherwise
    // one shared-memory atomic per active key. One vote per warp and pass.
    uint32_t bin[kPer];
    bool same = true;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const bool act = j < valid && !((pmask >> j) & 1u) &&
                       (pass == 0 || (key[j] >> (32 - 8 * pass)) == prefix);
      bin[j] = act ? (key[j] >> shift) & 0xFFu : 0xFFFFFFFFu;
      same = same && bin[j] == bin[0];
    }
    const uint32_t wbin = __shfl_sync(0xFFFFFFFFu, bin[0], 0);
    if (__all_sync(0xFFFFFFFFu, same && bin[0] == wbin)) {
      if (lane == 0 && wbin != 0xFFFFFFFFu) atomicAdd(&h[wbin], 32u * kPer);
    } else {
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        if (bin[j] != 0xFFFFFFFFu) atomicAdd(&h[bin[j]], 1u);
    }
    sel_sync<kOne>();  // every CTA's counts of this pass are complete
    if (tid <= 256) {
      uint32_t sum = 0u;
      for (uint32_t r = 0; r < C; ++r) sum += ld_rank<kOne>(&h[tid], r);
      red[tid] = sum;
    } else if (tid >= 512 && tid < 512 + kRBins) {
      hist[((pass + 1) & 1) * kRBins + (tid - 512)] = 0u;  // read last in the pass before
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t nd = need, stop = 0u;
      if (pass == 0) {
        const uint32_t np = red[256];
        if (static_cast<int64_t>(np) > k) stop = 2u;
        else nd = static_cast<uint32_t>(k - static_cast<int64_t>(np));
        if (nd == 0u && stop == 0u) stop = 1u;
      }
      if (stop == 0u) {
        // lane l holds bins 255 - 8l ... 248 - 8l (descending)
        uint32_t c[8], sum = 0u;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          c[q] = red[255 - 8 * lane - q];
          sum += c[q];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t run = incl - sum;
        if (run < nd && nd <= incl) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (run + c[q] >= nd) {
              s_bin = static_cast<uint32_t>(255 - 8 * lane - q);
              s_need = nd - run;
              break;
            }
            run += c[q];
          }
        }
      }
      if (lane == 0) s_stop = stop;
    }
    __syncthreads();
    const uint32_t stop = s_stop;
    if (stop != 0u) {
      over = stop == 2u;
      break;
    }
    prefix = (prefix << 8) | s_bin;
    need = s_need;
    if (pass == 3) {
      thresh = prefix;
      ties = need;
    }
  }
  if (over) {
    if (rank == 0 && tid == 0) *status = 3;
    for (int64_t i = static_cast<int64_t>(rank) * kCThreads + tid; i < k;
         i += static_cast<int64_t>(C) * kCThreads)
      kept_idx[i] = -1;
    sel_sync<kOne>();  // no CTA leaves while another may still read its shared memory
    return;
  }
  // sure keeps and ties of this thread, CTA and the CTAs before it, as one
  // packed count (sure << 16 | ties; at most 8192 of each per CTA)
  uint32_t nd = 0u, nt = 0u;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (j < valid) {
      if (((pmask >> j) & 1u) || key[j] > thresh) ++nd;
      else if (key[j] == thresh) ++nt;
    }
  }
  uint32_t packed_cta;
  const uint32_t packed = cta_excl_scan_1024((nd << 16) | nt, &packed_cta, warp_sums);
  if (tid == 0) cta_val[1] = packed_cta;
  sel_sync<kOne>();
  uint32_t sb = packed >> 16, tb = packed & 0xFFFFu;
  if constexpr (!kOne) {  // the counts of the CTAs before this one
    if (tid < static_cast<int>(rank)) tot[tid] = ld_rank<kOne>(&cta_val[1], tid);
    __syncthreads();
    for (uint32_t r = 0; r < rank; ++r) {
      sb += tot[r] >> 16;
      tb += tot[r] & 0xFFFFu;
    }
  }
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (j < valid) {
      const bool sure = ((pmask >> j) & 1u) || key[j] > thresh;
      const bool tie = !sure && key[j] == thresh;
      if (sure) {
        const uint32_t pos = sb + min(tb, ties);
        if (pos < static_cast<uint64_t>(k)) kept_idx[pos] = static_cast<int32_t>(first + j);
        ++sb;
      } else if (tie) {
        if (tb < ties) {
          const uint32_t pos = sb + tb;
          if (pos < static_cast<uint64_t>(k)) kept_idx[pos] = static_cast<int32_t>(first + j);
        }
        ++tb;
      }
    }
  }
  if (rank == 0 && tid == 0) *status = 0;
  sel_sync<kOne>();  // no CTA leaves while another may still read its shared memory
}

// Cluster size for n tokens (0: n is past the one-launch path).
int cluster_ctas(int64_t n) {
  static int max_ctas = 0;  // 16 where the device can co-schedule it, else 8
  static std::once_flag once;
  std::call_once(once, [] {
    max_ctas = 8;
    auto kern = sel_cluster<true, kPerThread, false>;
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(kern),
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(reinterpret_cast<const void*>(sel_cluster<false, kPerThread, false>),
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16);
      cfg.blockDim = dim3(kCThreads);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters >= 1)
        max_ctas = 16;
    }
    cudaGetLastError();  // a refused attribute is not an error of a later call
  });
  if (n > kClusterMaxN) return 0;
  int c = 1;
  while (int64_t(c) * kCChunk < n) c *= 2;
  return c <= max_ctas ? c : 0;
}

// One CTA (n <= 8192, no cluster barriers), else one cluster of `ctas`
// CTAs; 8 tokens per thread. (One CTA with 16 tokens per thread at
// n <= 16384 measured as slow as a 4-CTA cluster at 32768.)
template <bool kVec>
cudaError_t run_select_cluster(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                               int32_t* kept_idx, void* ws, int ctas, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kCThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  int32_t* status = static_cast<int32_t*>(ws);
  if (n <= kCChunk) {
    cfg.gridDim = dim3(1);
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sel_cluster<kVec, kPerThread, true>, scores, protect, n, k,
                              kept_idx, status);
  }
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(ctas);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, sel_cluster<kVec, kPerThread, false>, scores, protect, n, k,
                            kept_idx, status);
}

template <bool kVec>
cudaError_t run_select(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                       int32_t* kept_idx, void* ws, cudaStream_t st) {
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  Ws w = ws_view(ws, chunks);
  cudaError_t e = cudaMemsetAsync(ws, 0, kZeroBytes, st);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(chunks));
  TG_CUDA_TRY(launch_pdl(sel_hist0<kVec>, dim3(grid), dim3(kThreads), 0, st, scores, protect, n, w));
  TG_CUDA_TRY(launch_pdl(sel_hist_next<kVec, 1>, dim3(grid), dim3(kThreads), 0, st, scores, protect, n, k, w));
  TG_CUDA_TRY(launch_pdl(sel_hist_next<kVec, 2>, dim3(grid), dim3(kThreads), 0, st, scores, protect, n, k, w));
  TG_CUDA_TRY(launch_pdl(sel_count<kVec>, dim3(grid), dim3(kThreads), 0, st, scores, protect, n, k, w));
  TG_CUDA_TRY(launch_pdl(sel_write<kVec>, dim3(grid), dim3(kThreads), 0, st, scores, protect, n, k, kept_idx, w));
  return cudaGetLastError();
}

// Scratch of the allocation-free variant: one array per device, sized for
// the largest n it accepts, shared by every call on that device.
constexpr int64_t kNoAllocMaxN = int64_t(1) << 20;
static_assert(kNoAllocMaxN == TG_SELECT_NOALLOC_MAX_N, "the documented limit is the built one");
constexpr size_t kNoAllocBytes = kOffCounts + size_t(kNoAllocMaxN / kChunk) * 2 * 4;
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocBytes];

// The array's device address, cached per CUDA context. A context is keyed by
// its unique id (cuCtxGetId), which changes when cudaDeviceReset recreates a
// device's primary context or when a caller makes another context current
// through the driver API; either case makes a fresh lookup.
struct ScratchAddr {
  int dev;
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_scratch_mu;
std::vector<ScratchAddr> g_scratch_addr;
constexpr size_t kMaxScratchAddr = 256;

// Id of the current context, or 0 when none is current yet or the driver's
// entry points cannot be fetched (then every call looks the address up).
unsigned long long current_ctx_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace

int64_t select_noalloc_max_n() { return kNoAllocMaxN; }

// Host code cannot use g_select_scratch's name as a device address: the
// symbol's device address is looked up (cudaGetSymbolAddress, with the
// caller's device current) on the first call in each context and cached;
// kernels then get that pointer.
cudaError_t launch_topk_select_noalloc(const float* scores, const uint8_t* protect, int64_t n,
                                       int64_t k, int32_t* kept_idx, cudaStream_t st) {
  if (n > kNoAllocMaxN) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const unsigned long long id = current_ctx_id();
    if (id != 0)
      for (const ScratchAddr& a : g_scratch_addr)
        if (a.dev == dev && a.ctx_id == id) scratch = a.ptr;
    if (scratch == nullptr) {
      e = cudaGetSymbolAddress(&scratch, g_select_scratch);
      if (e != cudaSuccess) return e;
      // the lookup makes the device's primary context current if none was
      const unsigned long long id_now = current_ctx_id();
      if (id_now != 0) {
        if (g_scratch_addr.size() >= kMaxScratchAddr) g_scratch_addr.clear();
        g_scratch_addr.push_back(ScratchAddr{dev, id_now, scratch});
      }
    }
  }
  return launch_topk_select(scores, protect, n, k, kept_idx, scratch, st);
}

size_t select_ws_bytes(int64_t n) {
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  return kOffCounts + static_cast<size_t>(chunks) * 2 * 4;
}

cudaError_t launch_topk_select(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                               int32_t* kept_idx, void* ws, cudaStream_t st) {
  const bool vec = (reinterpret_cast<uintptr_t>(scores) % 16 == 0) &&
                   (protect == nullptr || reinterpret_cast<uintptr_t>(protect) % 8 == 0);
  const int ctas = cluster_ctas(n);
  if (ctas > 0)
    return vec ? run_select_cluster<true>(scores, protect, n, k, kept_idx, ws, ctas, st)
               : run_select_cluster<false>(scores, protect, n, k, kept_idx, ws, ctas, st);
  return vec ? run_select<true>(scores, protect, n, k, kept_idx, ws, st)
             : run_select<false>(scores, protect, n, k, kept_idx, ws, st);
}

}  // namespace tg
