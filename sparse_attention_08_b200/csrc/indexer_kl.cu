// indexer_kl.cu -- the indexer's training signal on sm_100a: the KL
// divergence between the main attention's distribution (summed over heads)
// and the softmax of the indexer scores, over each query's selected entries,
// and its gradient with respect to those scores.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section
// "Teaching a dense model to be sparse": the indexer's scores are fitted to
// the main attention's distribution by minimising a KL divergence;
// "DeepSeek-V3.2" atlas entry, "Design overview": the target is the head-wise
// attention distribution summed over heads).  For query t with valid
// selected entries S (index-row entries 0 <= s <= p):
//
//   p[t,s]  = (1/H) sum_h exp(scale * q[t,h,:] . c[s,:] - lse[t,h])
//   q[t,s]  = softmax_{s in S} I[t,s]
//   kl[t]   = sum_{s in S} p[t,s] (log p[t,s] - log q[t,s])
//   grad    = dkl / dI[t,s] = q[t,s] - p[t,s]
//
// lse is the attention's log-sum-exp over S per head (what
// dsa_sparse_mla_fwd writes), so each head's distribution sums to one.
//
// Two kernels.  attn_target_kernel: a persistent grid of one CTA per SM; a
// work item is (query, group of 128 heads).  Without an output accumulator
// the 128-head query tile (288 TMEM columns) and three 64-column score
// buffers fit in TMEM, so the score MMAs have M = 128 (all heads of a query,
// the full tensor rate).  Threads:
//  * warps 5..8 gather the 576-d latents of each block of 64 selected entries
//    into a ring of three 72 KB slots (16-byte cp.async, 128-byte swizzle),
//    after two slots of the item's query rows, which they also move into
//    TMEM once the previous item's last score product is done;
//  * warp 4 issues S = Q K^T (36 tcgen05.mma, M=128, N=64, K=16);
//  * warps 0..3 (keys 0..31 of a block) and 9..12 (keys 32..63): the warp on
//    sub-partition sp holds heads 32sp..32sp+31, one per lane (TMEM 32x32b
//    shape); it turns its 32 scores into probabilities with the head's lse,
//    sums them over its 32 heads with a butterfly across the lanes (lane c
//    ends with key c) and writes the 32 partial sums to its own slice of the
//    workspace: plain stores, no atomics, so the result is deterministic.
// kl_kernel: one CTA per query; adds the slices, takes the softmax of the
// indexer scores of the selected entries and writes kl, grad and target.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kHeads = 128;      // heads per work item (MMA M)
constexpr int kBlockN = 64;      // selected entries per block
constexpr int kDqk = 576;
constexpr int kChunks = kDqk / 64;                 // 9 column chunks of 64
constexpr uint32_t kChunkBytes = 64 * 128;         // 64 rows x 128 B
constexpr int kStages = 3;
constexpr uint32_t kKvBytes = kChunks * kChunkBytes;    // 73728
constexpr uint32_t kOffBar = kStages * kKvBytes;        // 221184
enum : uint32_t {
  kBKvFull = 0,    // [3] gather -> MMA              (128 arrivals)
  kBKvEmpty = 3,   // [3] MMA / query copy -> gather  (1)
  kBSFull = 6,     // [3] MMA -> target warps        (commit)
  kBSFree = 9,     // [3] target warps -> MMA        (8)
  kBQReady = 12,   // query tile in TMEM             (1)
  kBSLast = 13,    // last S of an item done         (commit; one phase per item)
  kBDrain = 14,    // every MMA of the CTA done      (commit)
  kNumBars = 16
};
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmem = kOffMisc + 16;
static_assert(kSmem <= 232448, "shared memory budget");

constexpr int kThreads = 32 * 13;            // 416
constexpr int kMmaWarp = 4;
constexpr int kProdWarp0 = 5;                // warps 5..8
constexpr int kProdThreads = 128;
constexpr int kHiWarp0 = 9;                  // warps 9..12: keys 32..63
constexpr uint32_t kBarProducer = 1;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCols = 64;
constexpr uint32_t kNumS = 3;
constexpr uint32_t kQCol = kNumS * kSCols;   // 192: query tile, 288 columns
constexpr uint32_t kIdescS = instr_desc(kFmtBF16, kFmtBF16, 0, 0, kHeads, kBlockN);
static_assert(kQCol + kDqk / 2 <= kTmemCols, "tensor memory budget");

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv;
  const int32_t* idx;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const float* lse;          // [total_q, H], natural log
  int B, H, k, head_groups;
  int64_t total_q;
  int64_t n_items;           // total_q * head_groups
  float scale_log2;          // sm_scale * log2(e)
  float* part;               // [head_groups * 4][total_q][k] partial sums over 32 heads
  int64_t part_stride;       // total_q * k
  DevErr err;
};

// One work item: a query row and a group of 128 heads.
struct Item {
  int64_t q_row;
  int hg;
  int p;            // absolute position of the query
  int n_sel;        // selected entries: min(k, p + 1)
  int nb;           // blocks of 64 entries
  int heads_here;   // heads of the group that exist
  int ck0;          // first key row of the sequence
};

// The longest rows (the last queries of the batch) come first.
__device__ __forceinline__ Item item_at(const Params& P, int64_t w) {
  Item it;
  it.q_row = P.total_q - 1 - w / P.head_groups;
  it.hg = static_cast<int>(w % P.head_groups);
  int lo = 0, hi = P.B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(P.cu_q + mid) <= it.q_row) lo = mid; else hi = mid;
  }
  const int cq0 = __ldg(P.cu_q + lo);
  it.ck0 = __ldg(P.cu_k + lo);
  const int len_q = __ldg(P.cu_q + lo + 1) - cq0;
  const int len_k = __ldg(P.cu_k + lo + 1) - it.ck0;
  it.p = len_k - len_q + static_cast<int>(it.q_row - cq0);
  it.n_sel = min(P.k, it.p + 1);
  it.nb = (it.n_sel + kBlockN - 1) / kBlockN;
  it.heads_here = min(kHeads, P.H - it.hg * kHeads);
  return it;
}

// Gather warps: two slots of query rows per item (heads 0..63, 64..127),
// then one slot per block of 64 selected latents; the query rows go into
// TMEM while the item's first block is in flight.
__device__ __forceinline__ void gather_loop(const Params& P, uint8_t* smem, uint32_t ring,
                                            uint32_t bar0, uint32_t tmem,
                                            volatile int* abort_flag) {
  const int tg = threadIdx.x - 32 * kProdWarp0;        // 0..127
  const int lane = threadIdx.x & 31;
  const int rsub = tg >> 3;                            // rows rsub + 16*pass
  const int l8 = tg & 7;                               // 16-byte piece within 128 B
  const uint32_t full0 = bar0 + 8u * kBKvFull;
  const uint32_t empty0 = bar0 + 8u * kBKvEmpty;
  uint32_t u = 0, ii = 0;
  for (int64_t w = blockIdx.x; w < P.n_items; w += gridDim.x, ++ii) {
    const Item it = item_at(P, w);
    const int32_t* idx_row = P.idx + it.q_row * P.k;
    const __nv_bfloat16* kv_seq = P.kv + static_cast<int64_t>(it.ck0) * kDqk;
    auto load_idx = [&](int j, int r) -> int {
      const int e = j * kBlockN + r;
      int s = -1;
      if (e < it.n_sel) s = __ldg(idx_row + e);
      return (s >= 0 && s <= it.p) ? s : 0;            // invalid entries read row 0 (masked)
    };
    int rows[4];
    const uint32_t uq = u;                             // the item's query slots: uq, uq + 1
    for (int j = -2; j < it.nb; ++j, ++u) {
      const uint32_t st = u % kStages;
      // every gather thread takes the same decision to stop
      const bool failed = tg == 0 && !mbar_wait(empty0 + 8u * st, ((u / kStages) & 1) ^ 1, P.err);
      if (named_bar_or(kBarProducer, kProdThreads, failed || *abort_flag)) {
        if (failed) *abort_flag = 1;
        return;
      }
      const uint32_t stage = ring + st * kKvBytes;
      if (j < 0) {
        if (j == -2 && tg == 0 && w + gridDim.x < P.n_items) {
          // the next item's query rows come from HBM: start them towards L2
          const Item nx = item_at(P, w + gridDim.x);
          prefetch_l2_bulk(P.q + (nx.q_row * P.H + nx.hg * kHeads) * kDqk,
                           static_cast<uint32_t>(nx.heads_here) * kDqk * 2u);
        }
        const __nv_bfloat16* q_grp = P.q + (it.q_row * P.H + it.hg * kHeads) * kDqk;
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int r = rsub + 16 * pass;              // row within the slot
          const int h = r + 64 * (j + 2);              // head
          const uint32_t dst = stage + r * 128 + ((l8 ^ (r & 7)) << 4);
          if (h < it.heads_here) {
            const __nv_bfloat16* src = q_grp + static_cast<int64_t>(h) * kDqk + l8 * 8;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) cp_async16(dst + c * kChunkBytes, src + c * 64);
          } else {
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
              asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst + c * kChunkBytes),
                           "r"(0u)
                           : "memory");
          }
        }
        cp_async_commit();
        if (j == -1) {
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) rows[pass] = load_idx(0, rsub + 16 * pass);
        }
      } else {
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int r = rsub + 16 * pass;
          const __nv_bfloat16* src = kv_seq + static_cast<int64_t>(rows[pass]) * kDqk + l8 * 8;
          const uint32_t dst = stage + r * 128 + ((l8 ^ (r & 7)) << 4);
#pragma unroll
          for (int c = 0; c < kChunks; ++c) cp_async16(dst + c * kChunkBytes, src + c * 64);
        }
        cp_async_commit();
        if (j + 1 < it.nb) {
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) rows[pass] = load_idx(j + 1, rsub + 16 * pass);
        }
        if (j == 0) {
          // Query tile -> TMEM.  Every gather thread has waited for its own
          // query copies and passed the barrier above, so both query slots
          // are complete.  The warp on sub-partition sp moves heads
          // 32sp..32sp+31 (TMEM lanes of the same numbers): thread t takes
          // row 32(sp&1) + t of slot uq + sp/2; column 192 + 32c + i of its
          // lane holds the elements 64c + 2i, +1 of the head's query.
          const bool qfail =
              tg == 0 && ii > 0 && !mbar_wait(bar0 + 8u * kBSLast, (ii - 1) & 1, P.err);
          if (named_bar_or(kBarProducer, kProdThreads, qfail || *abort_flag)) {
            if (qfail) *abort_flag = 1;
            return;
          }
          tc_fence_after();
          const int sp = (threadIdx.x >> 5) & 3;
          const int rs = 32 * (sp & 1) + lane;
          const uint8_t* qs = smem + ((uq + (sp >> 1)) % kStages) * kKvBytes + rs * 128;
          const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
#pragma unroll 1
          for (int c = 0; c < kChunks; ++c) {
            uint32_t r[32];
#pragma unroll
            for (int pc = 0; pc < 8; ++pc) {
              const uint4 v =
                  *reinterpret_cast<const uint4*>(qs + c * kChunkBytes + ((pc ^ (rs & 7)) << 4));
              r[4 * pc + 0] = v.x;
              r[4 * pc + 1] = v.y;
              r[4 * pc + 2] = v.z;
              r[4 * pc + 3] = v.w;
            }
            tmem_st_32x32b_x32(tmem + kQCol + lane_base + 32u * c, r);
          }
          tmem_wait_st();
          tc_fence_before();
          named_bar_sync(kBarProducer, kProdThreads);
          if (tg == 0) {
            mbar_arrive(empty0 + 8u * (uq % kStages));
            mbar_arrive(empty0 + 8u * ((uq + 1) % kStages));
            mbar_arrive(bar0 + 8u * kBQReady);
          }
        }
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(full0 + 8u * st);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) attn_target_kernel(const Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // every tile offset assumes a 1024-byte aligned base (the 128-byte swizzle
  // repeats every 1024 bytes); the allocation has no slack for realignment
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) raise_error(P.err, kErrBounds);
    return;
  }
  const uint32_t bar0 = sbase + kOffBar;
  auto bar = [&](uint32_t i) { return bar0 + 8u * i; };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(kBKvFull + i), kProdThreads);
      mbar_init(bar(kBKvEmpty + i), 1);
      mbar_init(bar(kBSFull + i), 1);
      mbar_init(bar(kBSFree + i), 8);
    }
    mbar_init(bar(kBQReady), 1);
    mbar_init(bar(kBSLast), 1);
    mbar_init(bar(kBDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp >= kProdWarp0 && warp < kProdWarp0 + 4) {
    // ------------------------------------------------------------ gathers
    gather_loop(P, smem, sbase, bar0, tmem, abort_flag);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ S = Q K^T
    const uint64_t dS0 = smem_desc(sbase, 16, 1024, kSwizzle128B);   // K, K-major
    constexpr uint64_t kStageStep = kKvBytes >> 4;
    const uint32_t tmem_q = tmem + kQCol;
    uint32_t u = 2, gb = 0, ii = 0;   // slots 0, 1 hold the first item's query
    for (int64_t w = blockIdx.x; ok && w < P.n_items; w += gridDim.x, ++ii, u += 2) {
      const Item it = item_at(P, w);
      for (int j = 0; j < it.nb; ++j, ++u, ++gb) {
        const uint32_t st = u % kStages;
        const uint32_t sb = gb % kNumS;
        ok = (j != 0 || warp_wait(bar(kBQReady), ii & 1, P.err)) &&
             warp_wait(bar(kBKvFull + st), (u / kStages) & 1, P.err) &&
             warp_wait(bar(kBSFree + sb), ((gb / kNumS) & 1) ^ 1, P.err);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dS = dS0 + st * kStageStep;
        const uint32_t d = tmem + kSCols * sb;
        if (elect_one()) {
#pragma unroll
          for (int cc = 0; cc < kChunks; ++cc) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f16_ts(d, tmem_q + 32u * cc + 8u * kk, dS + ((cc * kChunkBytes + kk * 32) >> 4),
                         kIdescS, (cc | kk) != 0 ? 1u : 0u);
            }
          }
          mma_commit(bar(kBKvEmpty + st));
          mma_commit(bar(kBSFull + sb));
          if (j + 1 == it.nb) mma_commit(bar(kBSLast));
        }
        __syncwarp();
      }
    }
    mma_commit_warp(bar(kBDrain));
    if (lane == 0) {
      mbar_wait_drain(bar(kBDrain), 0, P.err);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ targets
    const bool hi = warp >= kHiWarp0;
    const int sp = warp & 3;
    const int row = 32 * sp + lane;            // this lane's head in the group
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    const int c0 = hi ? 32 : 0;                // first key of the block this warp takes
    uint32_t gb = 0;
    auto entry_ok = [&](const Item& x, int e) -> bool {
      if (e >= x.n_sel) return false;
      const int s = __ldg(P.idx + x.q_row * P.k + e);
      return s >= 0 && s <= x.p;
    };
    for (int64_t w = blockIdx.x; ok && w < P.n_items; w += gridDim.x) {
      const Item it = item_at(P, w);
      // the head's lse in log2 units; rows past the last head contribute 0
      const float lse2 =
          row < it.heads_here ? __ldg(P.lse + it.q_row * P.H + it.hg * kHeads + row) *
                                    1.4426950408889634f
                              : INFINITY;
      float* out_row = P.part + static_cast<int64_t>(it.hg * 4 + sp) * P.part_stride +
                       it.q_row * P.k;
      for (int j = 0; j < it.nb; ++j, ++gb) {
        const uint32_t sb = gb % kNumS;
        const uint32_t vmask =
            __ballot_sync(0xffffffffu, entry_ok(it, j * kBlockN + c0 + lane));  // bit c: key c0+c
        if (!warp_wait(bar(kBSFull + sb), (gb / kNumS) & 1, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + kSCols * sb + c0, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBSFree + sb));
        // probabilities of this head (one per lane) for the warp's 32 keys
        float a[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float x = ((vmask >> c) & 1u) ? __uint_as_float(v[c]) : -INFINITY;
          a[c] = fast_exp2(fmaf(x, P.scale_log2, -lse2));
        }
        // sum over the warp's 32 heads: at width 16, 8, 4, 2, 1 every lane
        // keeps half of its remaining columns (the half its lane bit names)
        // and adds the partner's copy of them; lane c ends with key c
#pragma unroll
        for (int wdt = 16; wdt >= 1; wdt >>= 1) {
          const bool upper = (lane & wdt) != 0;
#pragma unroll
          for (int i = 0; i < wdt; ++i) {
            const float send = upper ? a[i] : a[i + wdt];
            const float keep = upper ? a[i + wdt] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, wdt);
          }
        }
        const int e = j * kBlockN + c0 + lane;
        if (e < P.k) out_row[e] = a[0];
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One CTA per query row: the target from the slices, the softmax of the
// indexer scores over the valid selected entries, the loss and its gradient.
constexpr int kKlThreads = 256;
constexpr int kKlPer = 4096 / kKlThreads;    // entries per thread at the largest k

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, y) : v + y;
  }
  __syncthreads();
  if (lane == 0) buf[warp] = v;
  __syncthreads();
  float r = buf[0];
#pragma unroll
  for (int w = 1; w < kKlThreads / 32; ++w) r = is_max ? fmaxf(r, buf[w]) : r + buf[w];
  return r;
}

__global__ void __launch_bounds__(kKlThreads)
    kl_kernel(const float* __restrict__ part, int64_t part_stride, int nparts, float inv_h,
              const int32_t* __restrict__ idx, const float* __restrict__ logits, int64_t ld,
              const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int B, int k,
              float* __restrict__ kl, float* __restrict__ grad, float* __restrict__ target) {
  __shared__ float red[kKlThreads / 32];
  const int64_t t = blockIdx.x;
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid;
  }
  const int len_q = __ldg(cu_q + lo + 1) - __ldg(cu_q + lo);
  const int len_k = __ldg(cu_k + lo + 1) - __ldg(cu_k + lo);
  const int p = len_k - len_q + static_cast<int>(t - __ldg(cu_q + lo));
  const int n_sel = min(k, p + 1);
  const int32_t* irow = idx + t * k;
  const float* lrow = logits + t * ld;
  float sc[kKlPer], pt[kKlPer];
  float m = -INFINITY;
#pragma unroll
  for (int u = 0; u < kKlPer; ++u) {
    const int j = threadIdx.x + u * kKlThreads;
    sc[u] = -INFINITY;
    pt[u] = 0.f;
    if (j < n_sel) {
      const int s = __ldg(irow + j);
      if (s >= 0 && s <= p) {
        sc[u] = __ldg(lrow + s);
        float acc = 0.f;
        for (int g = 0; g < nparts; ++g) acc += __ldg(part + g * part_stride + t * k + j);
        pt[u] = acc * inv_h;
        m = fmaxf(m, sc[u]);
      }
    }
  }
  m = block_reduce(m, true, red);
  float z = 0.f;
#pragma unroll
  for (int u = 0; u < kKlPer; ++u) z += sc[u] == -INFINITY ? 0.f : expf(sc[u] - m);
  z = block_reduce(z, false, red);
  const float log_z = m == -INFINITY ? 0.f : logf(z);
  float loss = 0.f;
#pragma unroll
  for (int u = 0; u < kKlPer; ++u) {
    const int j = threadIdx.x + u * kKlThreads;
    if (j >= k) break;
    const bool valid = sc[u] != -INFINITY;
    const float log_q = valid ? sc[u] - m - log_z : 0.f;
    if (valid && pt[u] > 0.f) loss += pt[u] * (logf(pt[u]) - log_q);
    if (grad) grad[t * k + j] = valid ? expf(log_q) - pt[u] : 0.f;
    if (target) target[t * k + j] = valid ? pt[u] : 0.f;
  }
  loss = block_reduce(loss, false, red);
  if (threadIdx.x == 0) kl[t] = loss;
}

}  // namespace

cudaError_t launch_indexer_kl(const KlArgs& a, DevErr err, cudaStream_t s) {
  if (a.total_q == 0) return cudaSuccess;
  Params P;
  P.q = static_cast<const __nv_bfloat16*>(a.q);
  P.kv = static_cast<const __nv_bfloat16*>(a.kv);
  P.idx = a.idx;
  P.cu_q = a.cu_q;
  P.cu_k = a.cu_k;
  P.lse = a.lse;
  P.B = a.B;
  P.H = a.H;
  P.k = a.k;
  P.head_groups = (a.H + kHeads - 1) / kHeads;
  P.total_q = a.total_q;
  P.n_items = a.total_q * P.head_groups;
  P.scale_log2 = a.sm_scale * 1.4426950408889634f;
  P.part = a.part;
  P.part_stride = a.total_q * a.k;
  P.err = err;
  cudaError_t e = cudaFuncSetAttribute(attn_target_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  const int64_t grid = P.n_items < a.num_sms ? P.n_items : a.num_sms;
  attn_target_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, s>>>(P);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // slices past a short row's last block are never written; the KL kernel
  // reads only entries j < min(k, p+1), which the target kernel wrote
  kl_kernel<<<static_cast<unsigned>(a.total_q), kKlThreads, 0, s>>>(
      a.part, P.part_stride, P.head_groups * 4, 1.0f / static_cast<float>(a.H), a.idx,
      a.logits, a.ld, a.cu_q, a.cu_k, a.B, a.k, a.kl, a.grad, a.target);
  return cudaGetLastError();
}

size_t indexer_kl_workspace_bytes(int64_t total_q, int H, int k) {
  const int64_t groups = (H + kHeads - 1) / kHeads;
  return static_cast<size_t>(groups * 4 * total_q * k * 4);
}

}  // namespace dsa
