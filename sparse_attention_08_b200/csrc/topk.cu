// topk.cu -- per-query top-k selection on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": each query keeps its k best-scoring entries;
// "DeepSeek-V3.2" atlas entry, "Design overview": token-level selection):
// for each query row with n = p+1 candidate scores, the positions of the
// min(k, n) largest, ties to the lower position, -0.0 == +0.0, written in
// ascending position order and padded with -1.
//
// How: one CTA of 512 threads per row; scores map to order-preserving 32-bit
// keys (larger float -> larger unsigned key, -0 folded into +0).
//  1. Threshold estimate.  1024 evenly spaced samples of the row give, by an
//     exact radix select among them, a key t0 that with a wide safety margin
//     lies below the row's k-th largest key.  (Rows with n <= 8192 skip this
//     and take t0 = 0, i.e. every element.)
//  2. Filter.  One vectorised streaming pass appends every (position, key)
//     with key >= t0 to a shared-memory candidate buffer.
//  3. Exact select among the candidates: three radix passes (11/11/10 bits)
//     over shared memory give the exact k-th key T and how many keys equal
//     to T must be kept (krem).
//  4. Ordered output.  Kept positions are marked in a shared bitmap of the
//     row (keys > T, then the first krem keys == T in position order, found
//     by a scan over a second bitmap of the ties); a block scan over the
//     bitmap words writes them in ascending order.
// If the estimate fails (fewer than k candidates, or more than the buffer
// holds, e.g. rows of massive ties) or the row is longer than the bitmap,
// the row falls back to exact radix passes over the whole row in global
// memory followed by an ordered ballot-scan compaction.  Both routes give the
// same, unique answer.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kCap = 8192;        // candidate buffer entries
constexpr int kSamples = 1024;
constexpr int kMaxBitmapN = 262144;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  uint32_t hist[2048];
  uint32_t scan_buf[kWarps + 1];
  uint32_t sel_digit;
  uint32_t cnt_above;
  uint32_t count;
  uint32_t overflow;
  uint32_t out_pos;
  uint32_t eq_seen;
  uint32_t cand_key[kCap];
  int32_t cand_pos[kCap];
  // followed in dynamic shared memory by two bitmaps of `words` words each
};

// Block-wide exclusive scan of one value per thread; *total gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* buf, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) buf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < kWarps ? buf[lane] : 0u;
    uint32_t s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) buf[lane] = s - w;
    if (lane == kWarps - 1) buf[kWarps] = s;
  }
  __syncthreads();
  const uint32_t res = buf[warp] + x - v;
  *total = buf[kWarps];
  __syncthreads();
  return res;
}

// Key source: either a shared-memory key array or a global score row.
struct SmemKeys {
  const uint32_t* k;
  __device__ __forceinline__ uint32_t operator()(int j) const { return k[j]; }
};
struct RowKeys {
  const float* row;
  __device__ __forceinline__ uint32_t operator()(int j) const { return order_key(__ldg(row + j)); }
};

// One radix pass over the m keys matching `prefix` on `mask`: histogram of
// bits [shift, shift+BITS) with warp-aggregated shared atomics, then the digit
// holding the krem-th largest candidate (block suffix scan).
template <int BITS, class Keys>
__device__ __forceinline__ void radix_pass(const Keys& keys, int m, int shift, uint32_t& prefix,
                                           uint32_t& mask, uint32_t& krem, Shared& sh) {
  constexpr int NB = 1 << BITS;
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NB; i += kThreads) sh.hist[i] = 0;
  __syncthreads();
  for (int base = (threadIdx.x & ~31); base < m; base += kThreads) {
    const int j = base + lane;
    bool in = j < m;
    const uint32_t u = in ? keys(j) : 0u;
    in = in && ((u & mask) == prefix);
    const uint32_t digit = (u >> shift) & (NB - 1);
    const uint32_t grp = __match_any_sync(0xffffffffu, in ? digit : (0x10000u | lane));
    if (in && lane == __ffs(grp) - 1) atomicAdd(&sh.hist[digit], __popc(grp));
  }
  __syncthreads();
  constexpr int PER = NB / kThreads > 0 ? NB / kThreads : 1;
  const int t = threadIdx.x;
  const bool owns = t * PER < NB;
  uint32_t local = 0;
  if (owns) {
#pragma unroll
    for (int q = 0; q < PER; ++q) local += sh.hist[NB - 1 - (t * PER + q)];
  }
  uint32_t tot;
  const uint32_t above = block_excl_scan(owns ? local : 0u, sh.scan_buf, &tot);
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

// Exact kk-th largest key among m keys; krem returns how many keys equal to
// it belong to the kk largest.
template <class Keys>
__device__ __forceinline__ uint32_t select_kth(const Keys& keys, int m, uint32_t kk, uint32_t& krem,
                                               Shared& sh) {
  uint32_t prefix = 0, mask = 0;
  krem = kk;
  radix_pass<11>(keys, m, 21, prefix, mask, krem, sh);
  radix_pass<11>(keys, m, 10, prefix, mask, krem, sh);
  radix_pass<10>(keys, m, 0, prefix, mask, krem, sh);
  return prefix;
}

// Fallback: exact select over the whole row in global memory, then an
// ordered ballot-scan compaction.
__device__ void topk_row_global(const float* __restrict__ row, int n, int k, int32_t* out,
                                float* vout, Shared& sh) {
  uint32_t krem;
  const uint32_t T = select_kth(RowKeys{row}, n, static_cast<uint32_t>(k), krem, sh);
  if (threadIdx.x == 0) {
    sh.out_pos = 0;
    sh.eq_seen = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += kThreads) {
    const int j = base + threadIdx.x;
    const bool in = j < n;
    const float f = in ? __ldg(row + j) : 0.f;
    const uint32_t u = in ? order_key(f) : 0u;
    const bool gt = in && u > T;
    const bool eq = in && u == T;
    const uint32_t eq_seen = sh.eq_seen;
    const uint32_t pos_base = sh.out_pos;
    uint32_t eq_tot, take_tot;
    const uint32_t eq_rank = block_excl_scan(eq ? 1u : 0u, sh.scan_buf, &eq_tot);
    const bool take = gt || (eq && eq_seen + eq_rank < krem);
    const uint32_t pos = block_excl_scan(take ? 1u : 0u, sh.scan_buf, &take_tot);
    if (take) {
      out[pos_base + pos] = j;
      if (vout) vout[pos_base + pos] = f;
    }
    if (threadIdx.x == 0) {
      sh.out_pos = pos_base + take_tot;
      sh.eq_seen = eq_seen + eq_tot;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads, 2)
    topk_kernel(const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ cu_q,
                const int32_t* __restrict__ cu_k, int B, int k, int bitmap_n,
                int32_t* __restrict__ idx, float* __restrict__ val) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Shared& sh = *reinterpret_cast<Shared*>(smem_raw);
  const int words_cap = (bitmap_n + 31) / 32;
  uint32_t* keep_bm = reinterpret_cast<uint32_t*>(smem_raw + sizeof(Shared));
  uint32_t* tie_bm = keep_bm + words_cap;

  const int64_t r = blockIdx.x;
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
  if (n > bitmap_n) {
    topk_row_global(row, n, k, out, vout, sh);
    return;
  }

  // ---- 1. threshold estimate from evenly spaced samples
  uint32_t t0 = 0u;
  if (n > kCap) {
    for (int s = threadIdx.x; s < kSamples; s += kThreads) {
      const int j = static_cast<int>((static_cast<int64_t>(2 * s + 1) * n) / (2 * kSamples));
      sh.cand_key[s] = order_key(__ldg(row + j));
    }
    __syncthreads();
    const float expect = static_cast<float>(kSamples) * k / n;
    int r0 = static_cast<int>(ceilf(expect + 4.f * sqrtf(expect) + 8.f));
    if (r0 < kSamples) {
      uint32_t unused;
      t0 = select_kth(SmemKeys{sh.cand_key}, kSamples, static_cast<uint32_t>(r0), unused, sh);
    }
  }

  // ---- 2. filter: append every (position, key) with key >= t0
  if (threadIdx.x == 0) {
    sh.count = 0;
    sh.overflow = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int n4 = n >> 2;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  for (int base = (threadIdx.x & ~31); base < n4; base += kThreads) {
    const int j4 = base + lane;
    uint32_t u[4] = {0u, 0u, 0u, 0u};
    int c = 0;
    if (j4 < n4) {
      const float4 f = __ldg(row4 + j4);
      u[0] = order_key(f.x);
      u[1] = order_key(f.y);
      u[2] = order_key(f.z);
      u[3] = order_key(f.w);
#pragma unroll
      for (int e = 0; e < 4; ++e) c += u[e] >= t0 ? 1 : 0;
    }
    uint32_t incl = static_cast<uint32_t>(c);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t wbase = 0;
    if (lane == 31) wbase = atomicAdd(&sh.count, incl);
    wbase = __shfl_sync(0xffffffffu, wbase, 31);
    uint32_t pos = wbase + incl - static_cast<uint32_t>(c);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (j4 < n4 && u[e] >= t0) {
        if (pos < kCap) {
          sh.cand_key[pos] = u[e];
          sh.cand_pos[pos] = 4 * j4 + e;
        }
        ++pos;
      }
    }
  }
  for (int j = 4 * n4 + threadIdx.x; j < n; j += kThreads) {  // ragged tail
    const uint32_t u = order_key(__ldg(row + j));
    if (u >= t0) {
      const uint32_t pos = atomicAdd(&sh.count, 1u);
      if (pos < kCap) {
        sh.cand_key[pos] = u;
        sh.cand_pos[pos] = j;
      }
    }
  }
  __syncthreads();
  const uint32_t m = sh.count;
  if (m > kCap || m < static_cast<uint32_t>(k)) {
    topk_row_global(row, n, k, out, vout, sh);
    return;
  }

  // ---- 3. exact k-th key among the candidates
  uint32_t krem;
  const uint32_t T = select_kth(SmemKeys{sh.cand_key}, static_cast<int>(m),
                                static_cast<uint32_t>(k), krem, sh);

  // ---- 4. mark kept positions, resolve ties in position order, emit in order
  const int words = (n + 31) / 32;
  for (int w = threadIdx.x; w < words; w += kThreads) {
    keep_bm[w] = 0u;
    tie_bm[w] = 0u;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < static_cast<int>(m); c += kThreads) {
    const uint32_t u = sh.cand_key[c];
    const int j = sh.cand_pos[c];
    if (u > T) atomicOr(&keep_bm[j >> 5], 1u << (j & 31));
    else if (u == T) atomicOr(&tie_bm[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  const int wpt = (words + kThreads - 1) / kThreads;   // words per thread, in order
  const int w0 = threadIdx.x * wpt;
  {
    uint32_t local = 0;
    for (int w = w0; w < min(w0 + wpt, words); ++w) local += __popc(tie_bm[w]);
    uint32_t tot;
    uint32_t rank = block_excl_scan(local, sh.scan_buf, &tot);
    for (int w = w0; w < min(w0 + wpt, words); ++w) {
      uint32_t bits = tie_bm[w];
      uint32_t keep = 0;
      while (bits) {
        const uint32_t lsb = bits & (0u - bits);
        if (rank < krem) keep |= lsb;
        ++rank;
        bits ^= lsb;
      }
      keep_bm[w] |= keep;
    }
  }
  __syncthreads();
  {
    uint32_t local = 0;
    for (int w = w0; w < min(w0 + wpt, words); ++w) local += __popc(keep_bm[w]);
    uint32_t tot;
    uint32_t pos = block_excl_scan(local, sh.scan_buf, &tot);
    for (int w = w0; w < min(w0 + wpt, words); ++w) {
      uint32_t bits = keep_bm[w];
      while (bits) {
        const int bit = __ffs(bits) - 1;
        const int j = w * 32 + bit;
        out[pos] = j;
        if (vout) vout[pos] = row[j];
        ++pos;
        bits &= bits - 1;
      }
    }
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, DevErr err, cudaStream_t s) {
  (void)err;
  if (a.total_q == 0) return cudaSuccess;
  const int bitmap_n = a.max_len_k < kMaxBitmapN ? a.max_len_k : kMaxBitmapN;
  const size_t smem = sizeof(Shared) + 2 * sizeof(uint32_t) * ((bitmap_n + 31) / 32);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<static_cast<unsigned>(a.total_q), kThreads, smem, s>>>(
      a.logits, a.ld, a.cu_q, a.cu_k, a.B, a.k, bitmap_n, a.idx, a.val);
  return cudaGetLastError();
}

}  // namespace dsa
