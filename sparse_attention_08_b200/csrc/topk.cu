// topk.cu -- per-query top-k selection on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": each query keeps its k best-scoring entries;
// "DeepSeek-V3.2" atlas entry, "Design overview": token-level selection):
// for each query row with n = p+1 candidate scores, the positions of the
// min(k, n) largest, ties to the lower position, -0.0 == +0.0, written in
// ascending position order and padded with -1.
//
// How: scores map to order-preserving 32-bit keys (larger float -> larger
// unsigned key, -0 folded into +0).  When the batch has enough rows to fill
// the GPU, a persistent grid of four 256-thread CTAs per SM walks the rows,
// one CTA per row, and pulls its next row into L2 while it works on the
// current one.  A few long rows (a decode batch) are split over a cluster of
// kSplitC CTAs that filter a quarter of the row each and hand their
// candidates to cluster rank 0, which finishes the row.  The row's 16-byte
// groups are cut into 8C contiguous segments in position order; warp w of
// rank c owns segment 8c + w and one region of its CTA's candidate buffer, so
// candidates stay in position order without any sorting.
//  1. Threshold.  Rows longer than about 2k (or than the candidate buffers)
//     draw S evenly spaced samples (S = 1024, or 4096 past 32768 scores).
//     Two levels of 2048-bin histograms of their keys (over [min, max], then
//     inside the bin holding the r0-th largest sample) give a key t0, the
//     lower edge of the fine bin holding that sample, with at least r0
//     samples at or above it; r0 = E + 4 sqrt(E) + 8 for E = S k / n
//     expected samples above the row's k-th largest, so t0 lies below that
//     score with a wide margin.  Every CTA of a cluster computes the same t0.
//  2. Filter.  Each warp streams its segment once (16-byte loads), compares
//     the raw floats with t0 as a float, and appends the (key, position) of
//     every score that passes to its region in position order (ballot
//     prefix), tracking the candidates' key range.  In a cluster every CTA
//     then stores its regions into rank 0's merge buffer after those of the
//     lower ranks, which gives one list in position order.
//  3. Exact k-th key.  Two levels of 2048-bin histograms of the candidates
//     (over their key range, then inside the bin that holds the k-th largest)
//     find a fine bin holding the k-th largest and how many keys lie above
//     it; the few keys of that bin are ranked against each other, which gives
//     the k-th key T and how many keys equal to T are kept (krem).
//  4. Ordered output.  A key is kept if it is > T or one of the first krem
//     keys == T in position order (tie ranks from a prefix over the warps'
//     contiguous shares of the list); output slots come from a second prefix.
// If the threshold fails (fewer than k candidates, or a region overflows,
// e.g. rows of massive ties) or the fine bin holds too many keys, one CTA
// falls back to exact radix passes over the whole row in global memory and an
// ordered ballot-scan compaction.  Both routes give the same, unique answer.
// Every decision that changes how many cluster barriers a CTA passes is taken
// from values that all CTAs of the cluster read alike.
//
// The fused indexer + top-k (fused.cu) hands this file candidate lists
// instead of score rows: topk_cand_kernel puts a row's candidates in position
// order through a bitmap of their positions and runs steps 3 and 4 on them;
// a row it cannot settle is flagged, and topk_kernel then runs on the flagged
// rows only (row_on).
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "keys.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;                 // 16-byte loads in flight per lane
constexpr int kSplitC = 4;                 // CTAs per row for few long rows
constexpr int kBins = 2048;                // histogram bins (11 bits)
constexpr int kBinBits = 11;
constexpr int kBinsPerThread = kBins / kThreads;
constexpr int kList = 512;                 // keys of the fine bin ranked directly

// Bin shift that maps keys in [lo, hi] onto at most kBins bins.
__device__ __forceinline__ int bin_shift(uint32_t lo, uint32_t hi) {
  const uint32_t span = hi - lo;
  const int bits = span == 0u ? 0 : 32 - __clz(span);
  return bits > kBinBits ? bits - kBinBits : 0;
}

// Values a CTA shares with the other CTAs of its cluster.
enum { kXCand = 0, kXOverflow, kXCount };

template <int CAP>
struct Shared {
  uint32_t hist[kBins];
  uint32_t wsum[kWarps];
  uint32_t wsum2[kWarps];
  uint32_t wcnt[kWarps];       // candidates per region
  uint32_t red_min, red_max;
  uint32_t sel_digit;
  uint32_t cnt_above;
  uint32_t out_pos;
  uint32_t eq_seen;
  uint32_t list_n;
  uint32_t res_key, res_rem;
  uint32_t xch[kXCount];
  uint32_t xall[kSplitC][kXCount];   // every CTA's xch, gathered once (clusters)
  uint32_t list_key[kList];
  uint32_t cand_key[CAP];
  int32_t cand_pos[CAP];
  // (clusters: a merge buffer of CAP keys and CAP positions follows)
};

// Cluster of C CTAs working on one row; with C == 1 a plain CTA.
template <int C>
struct Cluster {
  __device__ __forceinline__ static unsigned rank() {
    if constexpr (C == 1) return 0;
    else return cg::this_cluster().block_rank();
  }
  __device__ __forceinline__ static void sync() {
    if constexpr (C == 1) __syncthreads();
    else cg::this_cluster().sync();
  }
  // Address of `p` (a location in this CTA's shared memory) in CTA r.
  template <class T>
  __device__ __forceinline__ static T* at(T* p, unsigned r) {
    if constexpr (C == 1) return p;
    else return cg::this_cluster().map_shared_rank(p, r);
  }
};

// Block-wide exclusive scan of one value per thread; *total gets the sum.
template <int CAP>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, Shared<CAP>& sh,
                                                    uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.wsum[warp] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t s = sh.wsum[w];
    before += w < warp ? s : 0u;
    tot += s;
  }
  *total = tot;
  __syncthreads();
  return before + x - v;
}

// A warp's candidates: cnt (key, position) pairs in position order.
struct Seg {
  const uint32_t* key;
  const int32_t* pos;
  uint32_t cnt;
};

// Key sources.  for_each(f) calls f(key) on every key.
struct SegKeys {                 // each warp its own segment
  Seg seg;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    for (uint32_t i = threadIdx.x & 31; i < seg.cnt; i += 32) f(seg.key[i]);
  }
};
struct RowKeys {                 // a whole score row in global memory
  const float* row;
  int n;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    for (int j = threadIdx.x; j < n; j += kThreads) f(order_key(__ldg(row + j)));
  }
};

// The keys of `base` that fall into one bin of (key - lo) >> shift.
template <class Keys>
struct BinKeys {
  Keys base;
  uint32_t lo;
  int shift;
  uint32_t bin;
  template <class F>
  __device__ __forceinline__ void for_each(F f) const {
    const uint32_t l = lo, b = bin;
    const int sh = shift;
    base.for_each([&](uint32_t u) {
      if (((u - l) >> sh) == b) f(u);
    });
  }
};

// The CTA-wide min and max of per-thread key ranges, in sh.red_min / red_max.
template <int CAP>
__device__ void block_minmax(uint32_t mn, uint32_t mx, Shared<CAP>& sh) {
  const int lane = threadIdx.x & 31;
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
}

// Histogram cut: bins of (key - lo) >> shift over one CTA's keys; finds the
// bin holding the kk-th largest key (sh.sel_digit) and how many keys lie in
// higher bins (sh.cnt_above).  kk >= 1 and at most the number of keys.
template <int CAP, class Keys>
__device__ void hist_cut(const Keys& keys, uint32_t kk, uint32_t lo, int shift, Shared<CAP>& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < kBinsPerThread; ++i) sh.hist[threadIdx.x + i * kThreads] = 0u;
  __syncthreads();
  keys.for_each([&](uint32_t u) { atomicAdd(&sh.hist[(u - lo) >> shift], 1u); });
  __syncthreads();
  // thread t owns bins kBins-1-8t .. kBins-8-8t, counted from the top down
  uint32_t h[kBinsPerThread];
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kBinsPerThread; ++i) {
    h[i] = sh.hist[kBins - 1 - kBinsPerThread * threadIdx.x - i];
    s += h[i];
  }
  uint32_t x = s;
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
  uint32_t c = before + x - s;                  // keys in the bins above this thread's
  if (c < kk && c + s >= kk) {
#pragma unroll
    for (int i = 0; i < kBinsPerThread; ++i) {
      if (c < kk && c + h[i] >= kk) {
        sh.sel_digit = static_cast<uint32_t>(kBins - 1 - kBinsPerThread * threadIdx.x - i);
        sh.cnt_above = c;
      }
      c += h[i];
    }
  }
  __syncthreads();
}

// Exact kk-th largest key by radix passes (kk >= 1, at most the number of
// keys) over one CTA's keys; krem returns how many keys equal to it belong to
// the kk largest.  Used on the fallback path only.
template <int CAP, class Keys>
__device__ uint32_t radix_select(const Keys& keys, uint32_t kk, uint32_t& krem, Shared<CAP>& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t mn = 0xffffffffu, mx = 0u;
  keys.for_each([&](uint32_t u) {
    mn = min(mn, u);
    mx = max(mx, u);
  });
  block_minmax(mn, mx, sh);
  const uint32_t diff = sh.red_min ^ sh.red_max;
  krem = kk;
  if (diff == 0u) return sh.red_max;              // every key is equal
  const int top = 31 - __clz(diff);
  uint32_t mask = top == 31 ? 0u : ~((2u << top) - 1u);
  uint32_t prefix = sh.red_max & mask;
  for (int hi = top; hi >= 0; hi -= 8) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dmask = (2u << (hi - lo)) - 1u;
    sh.hist[threadIdx.x] = 0u;
    __syncthreads();
    keys.for_each([&](uint32_t u) {
      if ((u & mask) == prefix) atomicAdd(&sh.hist[(u >> lo) & dmask], 1u);
    });
    __syncthreads();
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
// ordered ballot-scan compaction (one CTA).
template <int CAP>
__device__ void topk_row_global(const float* __restrict__ row, int n, int k, int32_t* out,
                                float* vout, Shared<CAP>& sh) {
  uint32_t krem;
  const uint32_t T = radix_select(RowKeys{row, n}, static_cast<uint32_t>(k), krem, sh);
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
    const uint32_t eq_rank = block_excl_scan(eq ? 1u : 0u, sh, &eq_tot);
    const bool take = gt || (eq && eq_seen + eq_rank < krem);
    const uint32_t pos = block_excl_scan(take ? 1u : 0u, sh, &take_tot);
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

// Appends, in lane order, the flagged entries of this lane (flags bit e for
// v[e], position pos0 + e) to the warp's region and widens the lane's key
// range; returns the new count.
template <int CAP>
__device__ __forceinline__ uint32_t region_append(uint32_t* rk, int32_t* rp, uint32_t cnt,
                                                  const float (&v)[4], uint32_t flags, int pos0,
                                                  uint32_t& mn, uint32_t& mx) {
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
      const uint32_t u = order_key(v[e]);
      mn = min(mn, u);
      mx = max(mx, u);
      if (pos < static_cast<uint32_t>(CAP / kWarps)) {
        rk[pos] = u;
        rp[pos] = pos0 + e;
      }
      ++pos;
    }
  }
  return cnt + __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
}

// Steps 3 and 4 on one CTA: each warp holds `seg`, its contiguous share of
// the row's m >= k candidates (the warps' shares in warp order give every
// candidate once, in position order); (cmn, cmx) is this thread's part of the
// candidates' key range.  Writes the k kept positions (and scores) to out and
// returns true, or returns false without writing when too many keys share
// the cut bin (massive ties), for the caller's exact fallback.
template <int CAP>
__device__ bool select_and_output(const float* __restrict__ row, int n, int k,
                                  int32_t* __restrict__ out, float* __restrict__ vout,
                                  Shared<CAP>& sh, const Seg seg, uint32_t cmn, uint32_t cmx) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const SegKeys keys{seg};

  // ---- 3. exact k-th key: two histogram cuts, then the fine bin's keys ranked
  block_minmax(cmn, cmx, sh);
  uint32_t lo = sh.red_min;
  int shift = bin_shift(lo, sh.red_max);
  hist_cut(keys, static_cast<uint32_t>(k), lo, shift, sh);
  uint32_t bsel = sh.sel_digit;
  uint32_t kk = static_cast<uint32_t>(k) - sh.cnt_above;   // rank inside the cut bin
  if (shift > 0) {
    // the candidates can span many binades (a row whose k-th score is
    // negative spans the sign), so the first cut can be coarse: cut again
    // inside its bin
    const uint32_t lo2 = lo + (bsel << shift);
    const int shift2 = shift > kBinBits ? shift - kBinBits : 0;
    hist_cut(BinKeys<SegKeys>{keys, lo, shift, bsel}, kk, lo2, shift2, sh);
    bsel = sh.sel_digit;
    kk -= sh.cnt_above;
    lo = lo2;
    shift = shift2;
  }
  uint32_t T, krem;
  if (shift == 0) {
    // every key of the bin is the same key
    T = lo + bsel;
    krem = kk;
  } else {
    if (threadIdx.x == 0) sh.list_n = 0;
    __syncthreads();
    keys.for_each([&](uint32_t u) {
      if (((u - lo) >> shift) == bsel) {
        const uint32_t i = atomicAdd(&sh.list_n, 1u);
        if (i < static_cast<uint32_t>(kList)) sh.list_key[i] = u;
      }
    });
    __syncthreads();
    const uint32_t total = sh.list_n;
    if (total > static_cast<uint32_t>(kList)) return false;   // (uniform: sh.list_n)
    // rank every key of the bin against all of them: the kk-th largest is the
    // key with fewer than kk keys above it and at least kk at or above it
    if (threadIdx.x == 0) sh.res_key = 0u;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < total; i += kThreads) {
      const uint32_t own = sh.list_key[i];
      uint32_t gt = 0, ge = 0;
      for (uint32_t j = 0; j < total; ++j) {
        const uint32_t v = sh.list_key[j];
        gt += v > own ? 1u : 0u;
        ge += v >= own ? 1u : 0u;
      }
      if (gt < kk && ge >= kk) {
        sh.res_key = own;
        sh.res_rem = kk - gt;
      }
    }
    __syncthreads();
    T = sh.res_key;
    krem = sh.res_rem;
  }

  // ---- 4. ordered output: keys > T, and the first krem keys == T
  uint32_t gt = 0, eq = 0;
  for (uint32_t c = lane; c < seg.cnt; c += 32) {
    const uint32_t u = seg.key[c];
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
  for (uint32_t c0 = 0; c0 < seg.cnt; c0 += 32) {
    const uint32_t c = c0 + lane;
    const uint32_t u = c < seg.cnt ? seg.key[c] : 0u;
    const bool is_gt = c < seg.cnt && u > T;
    const bool is_eq = c < seg.cnt && u == T;
    const uint32_t eqb = __ballot_sync(0xffffffffu, is_eq);
    const bool take = is_gt || (is_eq && tie_before + __popc(eqb & lt) < krem);
    const uint32_t tb = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int j = seg.pos[c];
      const uint32_t slot = out_before + __popc(tb & lt);
      out[slot] = j;
      if (vout) vout[slot] = row[j];
    }
    out_before += __popc(tb);
    tie_before += __popc(eqb);
  }
  __syncthreads();   // the next row may reuse shared memory
  return true;
}

// One row, by every thread of every CTA of the cluster (C > 1: the merged
// candidates are finished by rank 0 alone, in the CAP keys and CAP positions
// that follow its Shared block).
template <int C, int CAP>
__device__ void topk_row(const float* __restrict__ row, int n, int k, int32_t* __restrict__ out,
                         float* __restrict__ vout, Shared<CAP>& sh) {
  constexpr int kRegion = CAP / kWarps;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned crank = Cluster<C>::rank();

  // (the whole cluster takes this branch alike: it depends on the row only)
  if (n <= k) {
    if (crank == 0) {
      for (int j = threadIdx.x; j < k; j += kThreads) {
        const bool v = j < n;
        out[j] = v ? j : -1;
        if (vout) vout[j] = v ? row[j] : __int_as_float(0x7fc00000);
      }
    }
    return;
  }

  // ---- 1. threshold from evenly spaced samples (identical in every CTA)
  float fth = -INFINITY;
  {
    const int S = n > 32768 ? 4096 : 1024;
    // below this no region, and no cluster's merged list, can overflow
    const int all_fit = C == 1 ? CAP - 64 : CAP;
    const int need = max(S, min(2 * k + 64, all_fit));
    if (n > need) {
      const int per = S / kWarps;                 // samples per region (<= kRegion)
      uint32_t mn = 0xffffffffu, mx = 0u;
      for (int s = threadIdx.x; s < S; s += kThreads) {
        const int j = static_cast<int>((static_cast<int64_t>(2 * s + 1) * n) / (2 * S));
        const uint32_t u = order_key(__ldg(row + j));
        sh.cand_key[(s / per) * kRegion + s % per] = u;
        mn = min(mn, u);
        mx = max(mx, u);
      }
      block_minmax(mn, mx, sh);                   // (its barriers publish the samples)
      const float expect = static_cast<float>(S) * k / n;
      const int r0 = static_cast<int>(ceilf(expect + 4.f * sqrtf(expect) + 8.f));
      if (r0 < S) {
        // two histogram levels: the bin of the r0-th largest sample, then
        // the same inside that bin, so the edge lies within 2^(shift-11)
        // keys of the sample itself (a coarse edge would let many more
        // scores through than the margin allows)
        const SegKeys samples{Seg{sh.cand_key + warp * kRegion, nullptr,
                                  static_cast<uint32_t>(per)}};
        const uint32_t lo = sh.red_min;
        const int shift = bin_shift(lo, sh.red_max);
        hist_cut(samples, static_cast<uint32_t>(r0), lo, shift, sh);
        const uint32_t b1 = sh.sel_digit;
        uint32_t t0 = lo + (b1 << shift);
        if (shift > 0) {
          const uint32_t r1 = static_cast<uint32_t>(r0) - sh.cnt_above;
          const int shift2 = shift > kBinBits ? shift - kBinBits : 0;
          hist_cut(BinKeys<SegKeys>{samples, lo, shift, b1}, r1, t0, shift2, sh);
          t0 += sh.sel_digit << shift2;
        }
        fth = key_float(t0);
      }
      __syncthreads();   // the samples are overwritten below
    }
  }

  // ---- 2. filter: warp w of rank c appends the passing scores of segment 8c + w
  uint32_t cmn = 0xffffffffu, cmx = 0u;
  uint32_t* rk = sh.cand_key + warp * kRegion;
  int32_t* rp = sh.cand_pos + warp * kRegion;
  {
    const int n4 = n >> 2;
    const int gw = static_cast<int>(crank) * kWarps + warp;
    const int seg = (n4 + C * kWarps - 1) / (C * kWarps);
    const int f0 = min(gw * seg, n4), f1 = min(f0 + seg, n4);
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
        const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t flags = 0;
        if (j4 < f1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) flags |= (x[e] >= fth ? 1u : 0u) << e;
        }
        if (__any_sync(0xffffffffu, flags != 0))
          cnt = region_append<CAP>(rk, rp, cnt, x, flags, 4 * j4, cmn, cmx);
      }
    }
    if (gw == C * kWarps - 1) {         // ragged tail: the last segment's region comes last
      const int j = 4 * n4 + lane;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t flags = 0;
      if (lane < 4 && j < n) {
        x[0] = __ldg(row + j);
        flags = x[0] >= fth ? 1u : 0u;
      }
      cnt = region_append<CAP>(rk, rp, cnt, x, flags, j, cmn, cmx);
    }
    if (lane == 0) sh.wcnt[warp] = cnt;
  }
  __syncthreads();
  uint32_t m = 0, overflow = 0, before = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t c = sh.wcnt[w];
    before += w < warp ? c : 0u;
    m += c;
    overflow |= c > static_cast<uint32_t>(kRegion) ? 1u : 0u;
  }

  if constexpr (C == 1) {
    if (overflow || m < static_cast<uint32_t>(k)) {
      topk_row_global(row, n, k, out, vout, sh);
      return;
    }
    if (!select_and_output<CAP>(row, n, k, out, vout, sh, Seg{rk, rp, sh.wcnt[warp]}, cmn, cmx))
      topk_row_global(row, n, k, out, vout, sh);
  } else {
    // merge: every CTA stores its regions, in warp order, into rank 0's merge
    // buffer after those of the lower ranks
    if (threadIdx.x == 0) {
      sh.xch[kXCand] = m;
      sh.xch[kXOverflow] = overflow;
    }
    Cluster<C>::sync();
    if (threadIdx.x < C * kXCount) {
      const unsigned q = threadIdx.x / kXCount, f = threadIdx.x % kXCount;
      sh.xall[q][f] = Cluster<C>::at(&sh.xch[f], q)[0];
    }
    __syncthreads();
    uint32_t total = 0;
    overflow = 0;
    for (unsigned q = 0; q < C; ++q) {
      before += q < crank ? sh.xall[q][kXCand] : 0u;
      total += sh.xall[q][kXCand];
      overflow |= sh.xall[q][kXOverflow];
    }
    const bool fits = !overflow && total >= static_cast<uint32_t>(k) &&
                      total <= static_cast<uint32_t>(CAP);
    uint32_t* mk = reinterpret_cast<uint32_t*>(&sh + 1);
    int32_t* mp = reinterpret_cast<int32_t*>(mk + CAP);
    if (fits) {
      uint32_t* dk = Cluster<C>::at(mk, 0u) + before;
      int32_t* dp = Cluster<C>::at(mp, 0u) + before;
      for (uint32_t c = lane; c < sh.wcnt[warp]; c += 32) {
        dk[c] = rk[c];
        dp[c] = rp[c];
      }
    }
    Cluster<C>::sync();   // the merged list is complete; no CTA reads another's memory after
    if (crank != 0) return;
    if (!fits) {
      topk_row_global(row, n, k, out, vout, sh);
      return;
    }
    const uint32_t share = (total + kWarps - 1) / kWarps;
    const uint32_t s0 = min(warp * share, total), s1 = min(s0 + share, total);
    cmn = 0xffffffffu;
    cmx = 0u;
    for (uint32_t c = s0 + lane; c < s1; c += 32) {
      cmn = min(cmn, mk[c]);
      cmx = max(cmx, mk[c]);
    }
    if (!select_and_output<CAP>(row, n, k, out, vout, sh, Seg{mk + s0, mp + s0, s1 - s0}, cmn,
                                cmx))
      topk_row_global(row, n, k, out, vout, sh);
  }
}

struct RowInfo {
  const float* row;
  int n;
};

__device__ __forceinline__ RowInfo row_info(int64_t r, const float* logits, int64_t ld,
                                            const int32_t* cu_q, const int32_t* cu_k, int B) {
  int lo = 0, hi = B;  // cu_q[lo] <= r < cu_q[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu_q + mid) <= r) lo = mid; else hi = mid;
  }
  const int len_q = __ldg(cu_q + lo + 1) - __ldg(cu_q + lo);
  const int len_k = __ldg(cu_k + lo + 1) - __ldg(cu_k + lo);
  const int i = static_cast<int>(r - __ldg(cu_q + lo));
  RowInfo ri;
  ri.row = logits + r * ld;
  ri.n = len_k - len_q + i + 1;  // candidates 0..p
  return ri;
}

// Pulls a score row towards L2 (16-byte granules; the tail below 16 bytes is
// read normally).
__device__ __forceinline__ void prefetch_row(const float* row, int n) {
  const uint32_t bytes = static_cast<uint32_t>(n) * 4u & ~15u;
  for (uint32_t off = 0; off < bytes; off += 32768u)
    prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(row) + off, min(32768u, bytes - off));
}

// C == 1: a persistent grid; CTA b takes rows b, b + grid, ... and pulls its
// next row into L2 at the start of each row.  C > 1: one row per cluster.
template <int C, int CAP>
__global__ void __launch_bounds__(kThreads, C == 1 ? (CAP <= 5120 ? 4 : 2) : 2)
    topk_kernel(const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ cu_q,
                const int32_t* __restrict__ cu_k, int B, int64_t total_q, int k,
                int32_t* __restrict__ idx, float* __restrict__ val,
                const uint32_t* __restrict__ row_on, const uint32_t* __restrict__ any_on) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Shared<CAP>& sh = *reinterpret_cast<Shared<CAP>*>(smem_raw);
  // a launch on a row subset with no row set does nothing
  if (any_on && *any_on == 0u) return;
  auto on = [&](int64_t r) { return row_on == nullptr || row_on[r] != 0u; };
  if constexpr (C == 1) {
    int64_t r = blockIdx.x;
    while (r < total_q && !on(r)) r += gridDim.x;
    if (r >= total_q) return;
    RowInfo cur = row_info(r, logits, ld, cu_q, cu_k, B);
    if (threadIdx.x == 0) prefetch_row(cur.row, cur.n);
    while (r < total_q) {
      int64_t rn = r + gridDim.x;
      while (rn < total_q && !on(rn)) rn += gridDim.x;
      RowInfo nxt = cur;
      if (rn < total_q) {
        nxt = row_info(rn, logits, ld, cu_q, cu_k, B);
        if (threadIdx.x == 0) prefetch_row(nxt.row, nxt.n);
      }
      topk_row<1, CAP>(cur.row, cur.n, k, idx + r * k, val ? val + r * k : nullptr, sh);
      cur = nxt;
      r = rn;
    }
  } else {
    const int64_t r = blockIdx.x / C;
    if (!on(r)) return;   // (the whole cluster alike)
    const RowInfo ri = row_info(r, logits, ld, cu_q, cu_k, B);
    topk_row<C, CAP>(ri.row, ri.n, k, idx + r * k, val ? val + r * k : nullptr, sh);
  }
}

template <int C, int CAP>
cudaError_t launch_t(const TopkArgs& a, cudaStream_t s) {
  // clusters: rank 0 also holds the merge buffer (CAP keys, CAP positions)
  const size_t smem = sizeof(Shared<CAP>) + (C > 1 ? 2 * CAP * sizeof(uint32_t) : 0);
  auto kern = topk_kernel<C, CAP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int64_t grid = a.total_q * C;
  if (C == 1) {
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) !=
            cudaSuccess || per_sm < 1)
      per_sm = 1;
    const int64_t cap = static_cast<int64_t>(sms) * per_sm;
    if (grid > cap) grid = cap;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = C > 1 ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a.logits, a.ld, a.cu_q, a.cu_k, a.B, a.total_q, a.k, a.idx,
                         a.val, a.row_on, a.any_on);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Top-k of rows whose candidates an indexer launch in compact mode listed
// (every causal score at or above the row's threshold, in no particular
// order).  With m >= k candidates the row's k best scores are all among them,
// ties included, so the selection equals the one over the whole row.  The
// candidates are put in position order through a bitmap of their positions
// (a prefix over its words ranks each one), then selected as above.  A row
// with fewer than k candidates, more than the list holds, or too many keys in
// the cut bin is marked in row_on (and any_on set) for the unfused path.
template <int CAP>
__global__ void __launch_bounds__(kThreads, 2)
    topk_cand_kernel(const uint32_t* __restrict__ cand_key, const int32_t* __restrict__ cand_pos,
                     const uint32_t* __restrict__ cnt, int cap, const int32_t* __restrict__ cu_q,
                     const int32_t* __restrict__ cu_k, int B, int64_t total_q, int k,
                     int32_t* __restrict__ idx, uint32_t* __restrict__ row_on,
                     uint32_t* __restrict__ any_on, int max_words) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Shared<CAP>& sh = *reinterpret_cast<Shared<CAP>*>(smem_raw);
  uint32_t* bm = reinterpret_cast<uint32_t*>(&sh + 1);        // position bitmap
  uint16_t* wpre = reinterpret_cast<uint16_t*>(bm + max_words);  // candidates before each word
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t r = blockIdx.x; r < total_q; r += gridDim.x) {
    const int n = row_info(r, nullptr, 0, cu_q, cu_k, B).n;
    int32_t* out = idx + r * k;
    if (n <= k) {
      for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
      continue;
    }
    const uint32_t m = cnt[r];
    if (m < static_cast<uint32_t>(k) || m > static_cast<uint32_t>(CAP) ||
        m > static_cast<uint32_t>(cap)) {
      if (threadIdx.x == 0) {
        row_on[r] = 1u;
        *any_on = 1u;
      }
      continue;
    }
    const uint32_t* ck = cand_key + r * cap;
    const int32_t* cp = cand_pos + r * cap;
    const int words = (n + 31) >> 5;
    for (int w = threadIdx.x; w < words; w += kThreads) bm[w] = 0u;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < m; i += kThreads) {
      const int pos = cp[i];
      atomicOr(bm + (pos >> 5), 1u << (pos & 31));
    }
    __syncthreads();
    const int wpt = (words + kThreads - 1) / kThreads;
    const int w0 = min(static_cast<int>(threadIdx.x) * wpt, words), w1 = min(w0 + wpt, words);
    uint32_t run = 0;
    for (int w = w0; w < w1; ++w) run += __popc(bm[w]);
    uint32_t tot;
    run = block_excl_scan(run, sh, &tot);
    for (int w = w0; w < w1; ++w) {
      wpre[w] = static_cast<uint16_t>(run);
      run += __popc(bm[w]);
    }
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < m; i += kThreads) {
      const int pos = cp[i];
      const uint32_t rank = wpre[pos >> 5] + __popc(bm[pos >> 5] & ((1u << (pos & 31)) - 1u));
      sh.cand_key[rank] = ck[i];
      sh.cand_pos[rank] = pos;
    }
    __syncthreads();
    const uint32_t share = (m + kWarps - 1) / kWarps;
    const uint32_t s0 = min(warp * share, m), s1 = min(s0 + share, m);
    uint32_t cmn = 0xffffffffu, cmx = 0u;
    for (uint32_t c = s0 + lane; c < s1; c += 32) {
      cmn = min(cmn, sh.cand_key[c]);
      cmx = max(cmx, sh.cand_key[c]);
    }
    if (!select_and_output<CAP>(nullptr, n, k, out, nullptr, sh,
                                Seg{sh.cand_key + s0, sh.cand_pos + s0, s1 - s0}, cmn, cmx)) {
      if (threadIdx.x == 0) {
        row_on[r] = 1u;
        *any_on = 1u;
      }
      __syncthreads();
    }
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, DevErr err, cudaStream_t s) {
  (void)err;
  if (a.total_q == 0) return cudaSuccess;
  // A row per CTA fills the GPU when there are enough rows; a few long rows
  // (a decode batch) are each split over a cluster of CTAs.
  const bool split = a.total_q < 148 && a.max_len_k > 16384 && a.k <= 2048;
  if (split) return launch_t<kSplitC, 5120>(a, s);
  if (a.k <= 2048) return launch_t<1, 5120>(a, s);
  return launch_t<1, 8192>(a, s);
}

cudaError_t launch_topk_candidates(const TopkCandArgs& a, DevErr err, cudaStream_t s) {
  (void)err;
  if (a.total_q == 0) return cudaSuccess;
  if (a.k > 2048 || a.max_len_k > kFusedMaxLenK || a.cap > kFusedCap) return cudaErrorInvalidValue;
  constexpr int CAP = kFusedCap;
  const int max_words = (a.max_len_k + 31) / 32;
  const size_t smem = sizeof(Shared<CAP>) + static_cast<size_t>(max_words) * 4 +
                      (static_cast<size_t>(max_words) * 2 + 15) / 16 * 16;
  auto kern = topk_cand_kernel<CAP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) !=
          cudaSuccess || per_sm < 1)
    per_sm = 1;
  int64_t grid = a.total_q;
  if (grid > static_cast<int64_t>(sms) * per_sm) grid = static_cast<int64_t>(sms) * per_sm;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(
      a.cand_key, a.cand_pos, a.cnt, a.cap, a.cu_q, a.cu_k, a.B, a.total_q, a.k, a.idx, a.row_on,
      a.any_on, max_words);
  return cudaGetLastError();
}

}  // namespace dsa
