// topk.cu -- per-query top-k selection on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": each query keeps its k best-scoring entries;
// "DeepSeek-V3.2" atlas entry, "Design overview": token-level selection):
// for each query row with n = p+1 candidate scores, the positions of the
// min(k, n) largest, ties to the lower position, -0.0 == +0.0, written in
// ascending position order and padded with -1.
//
// How: one CTA per row.  Scores map to order-preserving 32-bit keys
// (larger float -> larger unsigned key; -0 folded into +0).  Three radix
// passes (11 + 11 + 10 bits, most significant first) over the row find the
// exact k-th key T and how many keys equal to T must be kept (krem); each
// pass builds a shared-memory histogram with warp-aggregated atomics and
// picks the digit by a block-wide suffix scan.  A final pass walks the row in
// position order and keeps every key > T plus the first krem keys == T, with
// block-wide ballot scans giving each kept position its output slot -- which
// yields ascending order and the lowest-position tie-break by construction.
// The row is read from global memory each pass: the first read comes from
// HBM, the later ones from L2 (a 128 KB row per CTA stays resident).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  uint32_t hist[2048];
  uint32_t warp_a[kWarps];
  uint32_t warp_b[kWarps];
  uint32_t sel_digit;
  uint32_t cnt_above;
  uint32_t out_pos;
  uint32_t eq_seen;
};

// Block-wide exclusive scan of one value per thread (all kThreads threads).
// Returns the exclusive prefix; *total receives the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_buf, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_buf[lane];
    uint32_t s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_buf[lane] = s - w;  // exclusive prefix of warp sums
    if (lane == 31) warp_buf[32 + 0] = s;
  }
  __syncthreads();
  const uint32_t res = warp_buf[warp] + x - v;
  *total = warp_buf[32];
  __syncthreads();
  return res;
}

// One radix pass over the candidates (keys matching `prefix` on `mask`):
// histogram of bits [shift, shift+BITS), then the digit that holds the
// krem-th largest candidate.  Updates prefix/mask/krem.
template <int BITS>
__device__ __forceinline__ void radix_pass(const float* __restrict__ row, int n, int shift,
                                           uint32_t& prefix, uint32_t& mask, uint32_t& krem,
                                           Shared& sh, uint32_t* scan_buf) {
  constexpr int NB = 1 << BITS;
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NB; i += kThreads) sh.hist[i] = 0;
  __syncthreads();
  for (int base = (threadIdx.x & ~31); base < n; base += kThreads) {
    const int j = base + lane;
    bool in = j < n;
    uint32_t u = in ? order_key(__ldg(row + j)) : 0u;
    in = in && ((u & mask) == prefix);
    const uint32_t digit = (u >> shift) & (NB - 1);
    const uint32_t grp = __match_any_sync(0xffffffffu, in ? digit : (0x10000u | lane));
    if (in && lane == __ffs(grp) - 1) atomicAdd(&sh.hist[digit], __popc(grp));
  }
  __syncthreads();
  // Suffix counts in descending digit order: thread t owns digits
  // NB-1-t*per .. NB-per-t*per (per = NB / kThreads bins, at least 1).
  constexpr int PER = NB >= kThreads ? NB / kThreads : 1;
  uint32_t local = 0;
  const int t = threadIdx.x;
  const bool owns = t * PER < NB;
  if (owns) {
#pragma unroll
    for (int q = 0; q < PER; ++q) local += sh.hist[NB - 1 - (t * PER + q)];
  }
  uint32_t tot;
  const uint32_t above = block_excl_scan(owns ? local : 0u, scan_buf, &tot);
  if (owns && above < krem && above + local >= krem) {
    uint32_t c = above;
    for (int q = 0; q < PER; ++q) {
      const int d = NB - 1 - (t * PER + q);
      const uint32_t h = sh.hist[d];
      if (c + h >= krem) {
        sh.sel_digit = static_cast<uint32_t>(d);
        sh.cnt_above = c;
        break;
      }
      c += h;
    }
  }
  __syncthreads();
  prefix |= sh.sel_digit << shift;
  mask |= static_cast<uint32_t>(NB - 1) << shift;
  krem -= sh.cnt_above;
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ cu_q,
                const int32_t* __restrict__ cu_k, int B, int k, int32_t* __restrict__ idx,
                float* __restrict__ val) {
  __shared__ Shared sh;
  __shared__ uint32_t scan_buf[64];
  const int64_t r = blockIdx.x;
  // sequence of this row
  int lo = 0, hi = B;  // cu_q[lo] <= r < cu_q[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu_q + mid) <= r) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int len_q = __ldg(cu_q + b + 1) - __ldg(cu_q + b);
  const int len_k = __ldg(cu_k + b + 1) - __ldg(cu_k + b);
  const int i = static_cast<int>(r - __ldg(cu_q + b));
  const int n = len_k - len_q + i + 1;  // candidates 0..p
  const float* row = logits + r * ld;
  int32_t* out = idx + r * k;
  float* vout = val ? val + r * k : nullptr;

  if (n <= k) {
    for (int j = threadIdx.x; j < k; j += kThreads) {
      const bool v = j < n;
      out[j] = v ? j : -1;
      if (vout) vout[j] = v ? row[j] : __int_as_float(0x7fc00000);
    }
    return;
  }

  uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k);
  radix_pass<11>(row, n, 21, prefix, mask, krem, sh, scan_buf);
  radix_pass<11>(row, n, 10, prefix, mask, krem, sh, scan_buf);
  radix_pass<10>(row, n, 0, prefix, mask, krem, sh, scan_buf);
  const uint32_t T = prefix;

  if (threadIdx.x == 0) {
    sh.out_pos = 0;
    sh.eq_seen = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < n; base += kThreads) {
    const int j = base + threadIdx.x;
    const bool in = j < n;
    const float f = in ? __ldg(row + j) : 0.f;
    const uint32_t u = in ? order_key(f) : 0u;
    const bool gt = in && u > T;
    const bool eq = in && u == T;
    const uint32_t eq_seen = sh.eq_seen;
    const uint32_t pos_base = sh.out_pos;
    uint32_t eq_tot;
    const uint32_t eq_rank = block_excl_scan(eq ? 1u : 0u, scan_buf, &eq_tot);
    const bool take = gt || (eq && eq_seen + eq_rank < krem);
    uint32_t take_tot;
    const uint32_t pos = block_excl_scan(take ? 1u : 0u, scan_buf, &take_tot);
    if (take) {
      out[pos_base + pos] = j;
      if (vout) vout[pos_base + pos] = f;
    }
    if (threadIdx.x == 0) {
      sh.out_pos = pos_base + take_tot;
      sh.eq_seen = eq_seen + eq_tot;
    }
    __syncthreads();
    (void)lt_mask;
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, DevErr err, cudaStream_t s) {
  (void)err;
  if (a.total_q == 0) return cudaSuccess;
  topk_kernel<<<static_cast<unsigned>(a.total_q), kThreads, 0, s>>>(a.logits, a.ld, a.cu_q, a.cu_k,
                                                                     a.B, a.k, a.idx, a.val);
  return cudaGetLastError();
}

}  // namespace dsa
