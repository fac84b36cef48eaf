// topk.cu -- per-query top-k selection on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": each query keeps its k best-scoring entries;
// "DeepSeek-V3.2" atlas entry, "Design overview": token-level selection):
// for each query row with n = p+1 candidate scores, the positions of the
// min(k, n) largest, ties to the lower position, -0.0 == +0.0, written in
// ascending position order and padded with -1.
//
// How: one CTA of 256 threads (8 warps) per row, three CTAs per SM; scores
// map to order-preserving 32-bit keys (larger float -> larger unsigned key,
// -0 folded into +0).  Warp w owns the w-th contiguous eighth of the row and
// the w-th eighth of a shared candidate buffer, so candidates stay in
// position order without any sorting.
//  1. Threshold estimate (rows longer than the candidate buffer).  1024
//     evenly spaced samples give, by an exact radix select among them, a key
//     t0 that with a wide safety margin lies below the row's k-th largest.
//  2. Filter.  Each warp streams its segment once from memory (16-byte
//     loads, eight in flight per lane) and appends every (position, key)
//     with key >= t0 to its region, in position order (ballot + prefix).
//  3. Exact select among the candidates: radix passes of 8 bits, starting
//     below the bits that all candidates share, give the exact k-th key T
//     and how many keys equal to T are kept (krem).
//  4. Ordered output.  Warps walk their regions in order; a key is kept if
//     it is > T or it is one of the first krem keys == T (tie ranks from a
//     prefix over the regions); output slots come from a second prefix.
// If the estimate fails (fewer than k candidates, or a region overflows,
// e.g. rows of massive ties), the row falls back to exact radix passes over
// the whole row in global memory followed by an ordered ballot-scan
// compaction.  Both routes give the same, unique answer.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCap = 8192;                 // candidate buffer entries
constexpr int kRegion = kCap / kWarps;     // per warp
constexpr int kSamples = 1024;
constexpr int kUnroll = 8;                 // 16-byte loads in flight per lane

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  uint32_t hist[256];
  uint32_t wsum[kWarps];
  uint32_t wsum2[kWarps];
  uint32_t wcnt[kWarps];       // candidates per region
  uint32_t red_min, red_max;
  uint32_t sel_digit;
  uint32_t cnt_above;
  uint32_t overflow;
  uint32_t out_pos;
  uint32_t eq_seen;
  uint32_t cand_key[kCap];
  int32_t cand_pos[kCap];
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
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t s = buf[w];
    before += w < warp ? s : 0u;
    tot += s;
  }
  *total = tot;
  __syncthreads();
  return before + x - v;
}

// Key source of a radix select: either the candidate regions in shared
// memory (warp w scans region w) or a whole score row in global memory
// (block-strided).
struct RegionKeys {
  const Shared* sh;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t cnt = sh->wcnt[warp];
    const uint32_t* keys = sh->cand_key + warp * kRegion;
    for (uint32_t i = lane; i < cnt; i += 32) f(keys[i]);
  }
};
struct RowKeys {
  const float* row;
  int n;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    for (int j = threadIdx.x; j < n; j += kThreads) f(order_key(__ldg(row + j)));
  }
};

// Exact kk-th largest key (kk >= 1, at most the number of keys); krem
// returns how many keys equal to it belong to the kk largest.  The bits that
// all keys share are found first (block min / max); radix passes of 8 bits
// then resolve the rest from the highest differing bit down.  All threads
// return the same values.
template <class Keys>
__device__ uint32_t select_kth(const Keys& keys, uint32_t kk, uint32_t& krem, Shared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t mn = 0xffffffffu, mx = 0u;
  keys.for_each([&](uint32_t u) {
    mn = min(mn, u);
    mx = max(mx, u);
  });
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (threadIdx.x == 0) {
    sh.red_min = 0xffffffffu;
    sh.red_max = 0u;
  }
  __syncthreads();
  if (lane == 0) {
    atomicMin(&sh.red_min, mn);
    atomicMax(&sh.red_max, mx);
  }
  __syncthreads();
  const uint32_t diff = sh.red_min ^ sh.red_max;
  krem = kk;
  if (diff == 0u) return sh.red_max;               // every key is equal
  const int top = 31 - __clz(diff);                 // highest differing bit
  uint32_t mask = top == 31 ? 0u : ~((2u << top) - 1u);
  uint32_t prefix = sh.red_max & mask;
  for (int hi = top; hi >= 0; hi -= 8) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dmask = (2u << (hi - lo)) - 1u;
    sh.hist[threadIdx.x] = 0u;                      // 256 threads, 256 bins
    __syncthreads();
    keys.for_each([&](uint32_t u) {
      if ((u & mask) == prefix) atomicAdd(&sh.hist[(u >> lo) & dmask], 1u);
    });
    __syncthreads();
    // thread t owns bin 255 - t: an inclusive scan from the top bin down
    const uint32_t h = sh.hist[255 - threadIdx.x];
    uint32_t x = h;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh.wsum[warp] = x;
    __syncthreads();
    uint32_t before = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) before += w < warp ? sh.wsum[w] : 0u;
    const uint32_t incl = before + x, excl = incl - h;
    if (excl < krem && incl >= krem) {
      sh.sel_digit = 255u - threadIdx.x;
      sh.cnt_above = excl;
    }
    __syncthreads();
    prefix |= sh.sel_digit << lo;
    mask |= dmask << lo;
    krem -= sh.cnt_above;
  }
  return prefix;
}

// Fallback: exact select over the whole row in global memory, then an
// ordered ballot-scan compaction.
__device__ void topk_row_global(const float* __restrict__ row, int n, int k, int32_t* out,
                                float* vout, Shared& sh) {
  uint32_t krem;
  const uint32_t T = select_kth(RowKeys{row, n}, static_cast<uint32_t>(k), krem, sh);
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
    const uint32_t eq_rank = block_excl_scan(eq ? 1u : 0u, sh.wsum, &eq_tot);
    const bool take = gt || (eq && eq_seen + eq_rank < krem);
    const uint32_t pos = block_excl_scan(take ? 1u : 0u, sh.wsum, &take_tot);
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

// Appends, in lane order, the flagged keys of this lane (flags bit e for
// key[e], position pos0 + e) to the warp's region; returns the new count.
__device__ __forceinline__ uint32_t region_append(uint32_t* rk, int32_t* rp, uint32_t cnt,
                                                  const uint32_t (&key)[4], uint32_t flags,
                                                  int pos0) {
  const int lane = threadIdx.x & 31;
  const uint32_t c = __popc(flags);
  const uint32_t lt = (1u << lane) - 1u;
  const uint32_t b0 = __ballot_sync(0xffffffffu, c & 1u);
  const uint32_t b1 = __ballot_sync(0xffffffffu, c & 2u);
  const uint32_t b2 = __ballot_sync(0xffffffffu, c & 4u);
  uint32_t pos = cnt + __popc(b0 & lt) + 2u * __popc(b1 & lt) + 4u * __popc(b2 & lt);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if ((flags >> e) & 1u) {
      if (pos < kRegion) {
        rk[pos] = key[e];
        rp[pos] = pos0 + e;
      }
      ++pos;
    }
  }
  return cnt + __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
}

__global__ void __launch_bounds__(kThreads, 3)
    topk_kernel(const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ cu_q,
                const int32_t* __restrict__ cu_k, int B, int k, int32_t* __restrict__ idx,
                float* __restrict__ val) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Shared& sh = *reinterpret_cast<Shared*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

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

  // ---- 1. threshold estimate from evenly spaced samples
  uint32_t t0 = 0u;
  if (n > kCap) {
#pragma unroll
    for (int q = 0; q < kSamples / kThreads; ++q) {
      const int s = threadIdx.x + q * kThreads;
      const int j = static_cast<int>((static_cast<int64_t>(2 * s + 1) * n) / (2 * kSamples));
      sh.cand_key[(s / (kSamples / kWarps)) * kRegion + s % (kSamples / kWarps)] =
          order_key(__ldg(row + j));
    }
    if (lane == 0) sh.wcnt[warp] = kSamples / kWarps;
    __syncthreads();
    const float expect = static_cast<float>(kSamples) * k / n;
    const int r0 = static_cast<int>(ceilf(expect + 4.f * sqrtf(expect) + 8.f));
    if (r0 < kSamples) {
      uint32_t unused;
      t0 = select_kth(RegionKeys{&sh}, static_cast<uint32_t>(r0), unused, sh);
    }
    __syncthreads();   // the samples are overwritten below
  }

  // ---- 2. filter: warp w appends the keys >= t0 of its eighth of the row
  {
    const int n4 = n >> 2;
    const int seg = (n4 + kWarps - 1) / kWarps;
    const int f0 = min(warp * seg, n4), f1 = min(f0 + seg, n4);
    uint32_t* rk = sh.cand_key + warp * kRegion;
    int32_t* rp = sh.cand_pos + warp * kRegion;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    uint32_t cnt = 0;
    for (int base = f0; base < f1; base += 32 * kUnroll) {
      float4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j4 = base + u * 32 + lane;
        v[u] = j4 < f1 ? __ldg(row4 + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j4 = base + u * 32 + lane;
        const uint32_t key[4] = {order_key(v[u].x), order_key(v[u].y), order_key(v[u].z),
                                 order_key(v[u].w)};
        uint32_t flags = 0;
        if (j4 < f1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) flags |= (key[e] >= t0 ? 1u : 0u) << e;
        }
        cnt = region_append(rk, rp, cnt, key, flags, 4 * j4);
      }
    }
    if (warp == kWarps - 1) {           // ragged tail: the last warp's region comes last
      const int j = 4 * n4 + lane;
      uint32_t key[4] = {0u, 0u, 0u, 0u};
      uint32_t flags = 0;
      if (lane < 4 && j < n) {
        key[0] = order_key(__ldg(row + j));
        flags = key[0] >= t0 ? 1u : 0u;
      }
      // one key per lane: positions j = 4*n4 + lane
      cnt = region_append(rk, rp, cnt, key, flags, j);
    }
    if (lane == 0) sh.wcnt[warp] = cnt;
  }
  __syncthreads();
  uint32_t m = 0;
  bool overflow = false;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    m += sh.wcnt[w];
    overflow |= sh.wcnt[w] > static_cast<uint32_t>(kRegion);
  }
  if (overflow || m < static_cast<uint32_t>(k)) {
    topk_row_global(row, n, k, out, vout, sh);
    return;
  }

  // ---- 3. exact k-th key among the candidates
  uint32_t krem;
  const uint32_t T = select_kth(RegionKeys{&sh}, static_cast<uint32_t>(k), krem, sh);

  // ---- 4. ordered output: keys > T, and the first krem keys == T
  {
    const uint32_t cnt = sh.wcnt[warp];
    const uint32_t* rk = sh.cand_key + warp * kRegion;
    const int32_t* rp = sh.cand_pos + warp * kRegion;
    uint32_t gt = 0, eq = 0;
    for (uint32_t c = lane; c < cnt; c += 32) {
      const uint32_t u = rk[c];
      gt += u > T ? 1u : 0u;
      eq += u == T ? 1u : 0u;
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if (lane == 0) {
      sh.wsum[warp] = eq;
      sh.wsum2[warp] = gt;
    }
    __syncthreads();
    uint32_t tie_before = 0, out_before = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) {
        const uint32_t room = krem > tie_before ? krem - tie_before : 0u;
        out_before += sh.wsum2[w] + min(sh.wsum[w], room);
        tie_before += sh.wsum[w];
      }
    }
    const uint32_t lt = (1u << lane) - 1u;
    for (uint32_t c0 = 0; c0 < cnt; c0 += 32) {
      const uint32_t c = c0 + lane;
      const uint32_t u = c < cnt ? rk[c] : 0u;
      const bool is_gt = c < cnt && u > T;
      const bool is_eq = c < cnt && u == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, is_eq);
      const bool take = is_gt || (is_eq && tie_before + __popc(eqb & lt) < krem);
      const uint32_t tb = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int j = rp[c];
        const uint32_t slot = out_before + __popc(tb & lt);
        out[slot] = j;
        if (vout) vout[slot] = row[j];
      }
      out_before += __popc(tb);
      tie_before += __popc(eqb);
    }
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, DevErr err, cudaStream_t s) {
  (void)err;
  if (a.total_q == 0) return cudaSuccess;
  const size_t smem = sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<static_cast<unsigned>(a.total_q), kThreads, smem, s>>>(
      a.logits, a.ld, a.cu_q, a.cu_k, a.B, a.k, a.idx, a.val);
  return cudaGetLastError();
}

}  // namespace dsa
