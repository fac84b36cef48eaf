// fused.cu -- the first pass of the fused indexer + top-k: sampled keys and
// per-row score thresholds.
//
// What it serves ("DeepSeek V3.2 and the lightning indexer", section "What we
// would test": at long context the indexer's quadratic term is the cost that
// remains, and its L x L score matrix is what a fused indexer + top-k keeps
// out of HBM).  The selection is unchanged: each row keeps its k best causal
// scores.  The fused path finds them in two passes over the keys:
//  1. the indexer scores every query against a 1/32 sample of its sequence's
//     keys (positions 0, 32, 64, ...: this file gathers them), and each row
//     takes as its threshold the r0-th largest score among the samples it may
//     see (positions <= p), r0 = E + 4 sqrt(E) + 8 for E = S k / n the
//     expected number of its S samples above the row's k-th best score (n =
//     p + 1 scores); rows of at most 4096 scores keep every score;
//  2. the indexer scores every causal pair again and appends only the scores
//     at or above the row's threshold to the row's candidate list, and top-k
//     selects from that list (topk.cu).  A row whose list holds fewer than k
//     or more entries than it can keep goes through the unfused path.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "keys.cuh"

namespace dsa {
namespace {

// cu_k_s[b] = sum over the sequences before b of ceil(len_k / kSampleStride).
__global__ void __launch_bounds__(1024) sample_offsets_kernel(const int32_t* __restrict__ cu_k,
                                                              int B, int32_t* __restrict__ cu_k_s) {
  __shared__ int32_t wsum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t carry = 0;
  for (int b0 = 0; b0 < B; b0 += 1024) {
    const int b = b0 + threadIdx.x;
    const int32_t c =
        b < B ? (__ldg(cu_k + b + 1) - __ldg(cu_k + b) + kSampleStride - 1) / kSampleStride : 0;
    int32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int32_t before = 0, tot = 0;
    for (int w = 0; w < 32; ++w) {
      before += w < warp ? wsum[w] : 0;
      tot += wsum[w];
    }
    if (b < B) cu_k_s[b] = carry + before + x - c;
    carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) cu_k_s[B] = carry;
}

// One thread per sampled key: its d_I FP8 bytes and its scale.
__global__ void __launch_bounds__(256) sample_gather_kernel(FusedSampleArgs a) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= a.max_samples || g >= __ldg(a.cu_k_s + a.B)) return;
  int lo = 0, hi = a.B;   // cu_k_s[lo] <= g < cu_k_s[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a.cu_k_s + mid) <= g) lo = mid; else hi = mid;
  }
  const int64_t m = g - __ldg(a.cu_k_s + lo);
  const int64_t src = __ldg(a.cu_k + lo) + m * kSampleStride;
  const uint4* s = reinterpret_cast<const uint4*>(a.k8 + src * a.d_I);
  uint4* d = reinterpret_cast<uint4*>(a.k8_s + g * a.d_I);
  for (int i = 0; i < a.d_I / 16; ++i) d[i] = __ldg(s + i);
  a.k_scale_s[g] = __ldg(a.k_scale + src);
}

// One warp per row: the r0-th largest sampled score by four 8-bit radix
// passes over the row's visible samples (a 256-bin histogram per warp).
constexpr int kThrWarps = 8;

__global__ void __launch_bounds__(kThrWarps * 32) threshold_kernel(FusedThresholdArgs a) {
  __shared__ uint32_t hist_all[kThrWarps][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kThrWarps + warp;
  if (r >= a.total_q) return;
  uint32_t* hist = hist_all[warp];
  int lo = 0, hi = a.B;   // cu_q[lo] <= r < cu_q[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a.cu_q + mid) <= r) lo = mid; else hi = mid;
  }
  const int len_q = __ldg(a.cu_q + lo + 1) - __ldg(a.cu_q + lo);
  const int len_k = __ldg(a.cu_k + lo + 1) - __ldg(a.cu_k + lo);
  const int p = len_k - len_q + static_cast<int>(r - __ldg(a.cu_q + lo));
  const int n = p + 1;
  float t = -INFINITY;
  if (n > kFusedAllPass) {
    const int len_s = __ldg(a.cu_k_s + lo + 1) - __ldg(a.cu_k_s + lo);
    const int S = min(len_s, p / kSampleStride + 1);
    const float expect = static_cast<float>(S) * a.k / n;
    const int r0 = static_cast<int>(ceilf(expect + 4.f * sqrtf(expect) + 8.f));
    if (r0 < S) {
      const float* row = a.logits_s + r * a.ld_s;
      uint32_t prefix = 0u, mask = 0u, krem = static_cast<uint32_t>(r0);
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int j = lane; j < 256; j += 32) hist[j] = 0u;
        __syncwarp();
        for (int j = lane; j < S; j += 32) {
          const uint32_t u = order_key(row[j]);
          if ((u & mask) == prefix) atomicAdd(hist + ((u >> shift) & 255u), 1u);
        }
        __syncwarp();
        // lane l owns bins 255 - 8l .. 248 - 8l, counted from the top down
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist[255 - 8 * lane - e];
          sum += c[e];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t cum = incl - sum, digit = 0u, above = 0u;
        const bool mine = cum < krem && incl >= krem;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (mine && cum < krem && cum + c[e] >= krem) {
            digit = static_cast<uint32_t>(255 - 8 * lane - e);
            above = cum;
          }
          cum += c[e];
        }
        const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        prefix |= digit << shift;
        mask |= 255u << shift;
        krem -= above;
        __syncwarp();
      }
      t = key_float(prefix);
    }
  }
  if (lane == 0) a.thr[r] = t;
}

}  // namespace

cudaError_t launch_fused_sample(const FusedSampleArgs& a, cudaStream_t s) {
  if (a.B == 0 || a.max_samples == 0) return cudaSuccess;
  if (a.d_I % 16 != 0) return cudaErrorInvalidValue;
  sample_offsets_kernel<<<1, 1024, 0, s>>>(a.cu_k, a.B, a.cu_k_s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t blocks = (a.max_samples + 255) / 256;
  sample_gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fused_threshold(const FusedThresholdArgs& a, cudaStream_t s) {
  if (a.total_q == 0) return cudaSuccess;
  const int64_t blocks = (a.total_q + kThrWarps - 1) / kThrWarps;
  threshold_kernel<<<static_cast<unsigned>(blocks), kThrWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
