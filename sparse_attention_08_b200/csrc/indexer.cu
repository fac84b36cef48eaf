// indexer.cu -- lightning-indexer scores on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": per query and earlier token, a handful of FP8
// indexer heads each give a ReLU-clipped dot product, combined with per-head
// weights into one score):
//
//   logits[t, s] = k_scale[s] * sum_j (w[t,j] * q_scale[t,j]) * ReLU(q8[t,j,:] . k8[s,:])
//
// for all causal pairs s <= p(t).
//
// How: the dot products form one dense FP8 contraction per tile,
//   D[s, (t,j)] = sum_d k8[s,d] * q8[t,j,d],     M = 128 keys, N = 256 = QPT*H_I,
// issued as tcgen05.mma kind::f8f6f4 (e4m3 x e4m3 -> f32) from TMA-fed,
// 128/64-byte-swizzled shared-memory tiles into a double-buffered TMEM
// accumulator.  Epilogue threads own one key (TMEM lane) each and fold
// ReLU, the (w * q_scale) head weights, the k_scale multiply and the causal
// mask into the read-out, so no per-head score ever leaves the SM.
//
// Work items: (sequence, group of QPT queries, chunk of KB_PER_ITEM key
// blocks) on a persistent grid of one CTA per SM, strided over a virtual item
// space; items outside the causal triangle are skipped by every role alike.
// The number of virtual key chunks is padded to be coprime with the grid, so
// that every CTA's stride visits every chunk index alike: chunks far from
// the diagonal are skipped more often, and a CTA that only ever saw them
// would finish early.
//
// Warp roles (576 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..17 = four epilogue warpgroups.  Warpgroup g reads
// accumulator buffer g/2 and the column half g%2 (half of the tile's
// queries); warp w reads TMEM lanes 32*(w%4)...  The ReLU / weighted-sum
// read-out costs about as many issue slots as the MMA takes cycles, so it
// is spread over four warps per sub-partition to hide TMEM and FMA latency.
//
// Read-out modes (the fused indexer + top-k, fused.cu): kIdxRect stores the
// score of every key of the sequence (no causal mask; for the sampled keys),
// and kIdxCompact (a separate instantiation, 64 heads) stores no scores but
// appends the (order key, position) of each causal score at or above its
// row's threshold to the row's candidate list: one ballot per warp and
// query, one atomic on the row's count to reserve the slots.  A launch may be
// limited to the query groups that hold a flagged row (row_on), and does
// nothing while no row is flagged (any_on).
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "keys.cuh"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kBlockK = 128;      // keys per tile (MMA M)
constexpr int kKbPerItem = 16;    // key blocks per work item
constexpr int kDenseKb = 8;       // key blocks per work item of a one-query batch
constexpr int kMaxDenseB = 2048;  // sequences a one-query batch may have for the dense list
constexpr int kStages = 6;        // key-tile pipeline depth
constexpr int kEpiThreads = 128;   // one epilogue warpgroup

struct Params {
  const float* q_scale;
  const float* w;
  const float* k_scale;
  const int32_t* cu_q;
  const int32_t* cu_k;
  float* logits;
  int64_t ld;
  int B;
  int n_qg;   // query groups per sequence (virtual)
  int n_kc;   // key chunks per sequence (virtual)
  int64_t n_items;
  int dense;  // 1: one query per sequence; items are the real (sequence, key chunk) pairs
  int mode;   // kIdxCausal, kIdxRect or kIdxCompact
  const float* thr;
  uint32_t* cand_key;
  int32_t* cand_pos;
  uint32_t* cnt;
  int cap;
  const uint32_t* row_on;
  const uint32_t* any_on;
  DevErr err;
};

struct Item {
  int q_row0;   // global query row of the group's first query
  int k_row0;   // global key row of the sequence's first key
  int len_q, len_k;
  int q0;       // local index of the group's first query
  int nq;       // queries in the group (<= QPT)
  int kb0;      // first key block (sequence-local, units of kBlockK)
  int nkb;      // key blocks in the item
};

// The item of sequence b, query group qg, key chunk kc of kb key blocks.
template <int QPT>
__device__ __forceinline__ bool fill_item(int b, int qg, int kc, int kb, const Params& P, Item& it) {
  const int cq0 = __ldg(P.cu_q + b), cq1 = __ldg(P.cu_q + b + 1);
  const int ck0 = __ldg(P.cu_k + b), ck1 = __ldg(P.cu_k + b + 1);
  it.len_q = cq1 - cq0;
  it.len_k = ck1 - ck0;
  it.q0 = qg * QPT;
  if (it.q0 >= it.len_q) return false;
  if (P.mode != kIdxRect && it.len_q > it.len_k) return false;
  it.nq = min(QPT, it.len_q - it.q0);
  // the last key any query of the group reads (every key without the mask)
  const int p_max =
      P.mode == kIdxRect ? it.len_k - 1 : it.len_k - it.len_q + it.q0 + it.nq - 1;
  const int kbeg = kc * kb * kBlockK;
  const int kend = min(kbeg + kb * kBlockK, p_max + 1);
  if (kbeg >= kend) return false;
  it.kb0 = kbeg / kBlockK;
  it.nkb = (kend - kbeg + kBlockK - 1) / kBlockK;
  it.q_row0 = cq0 + it.q0;
  it.k_row0 = ck0;
  if (P.row_on) {
    // only groups holding a row to compute (every role reads the same flags)
    bool any = false;
    for (int i = 0; i < it.nq; ++i) any |= P.row_on[it.q_row0 + i] != 0u;
    if (!any) return false;
  }
  return true;
}

// Item number -> item.  Prefill and chunk batches use a virtual item space
// (sequence, query group, key chunk) in which items outside the causal
// triangle are skipped.  One-query batches (decode) list only their real
// (sequence, key chunk) pairs: pre[b] counts the chunks of the sequences
// before b, so the persistent grid's stride deals out equal shares of work
// whatever the mix of cache lengths.
template <int QPT>
__device__ __forceinline__ bool decode_item(int64_t item, const Params& P, const int* pre,
                                            Item& it) {
  if (QPT == 1 && P.dense) {
    int lo = 0, hi = P.B;   // pre[lo] <= item < pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= item) lo = mid; else hi = mid;
    }
    return fill_item<QPT>(lo, 0, static_cast<int>(item - pre[lo]), kDenseKb, P, it);
  }
  const int kc = static_cast<int>(item % P.n_kc);
  const int64_t rest = item / P.n_kc;
  const int qg = static_cast<int>(rest % P.n_qg);
  const int b = static_cast<int>(rest / P.n_qg);
  if (b >= P.B) return false;
  return fill_item<QPT>(b, qg, kc, kKbPerItem, P, it);
}

// NT = MMA N = queries per tile * H_I: 256 (four queries of 64 heads) for
// prefill; 64 (one query of 64 heads) when every sequence has one query
// (decode), so a tile does not carry three empty queries.
template <int H_I, int D_I, int NT>
struct Layout {
  static constexpr int kN = NT;
  static constexpr int QPT = NT / H_I;
  // epilogue warpgroups per accumulator buffer: two column halves when a
  // tile holds two or more queries, else one warpgroup reads all columns
  static constexpr int kHalves = QPT >= 2 ? 2 : 1;
  // accumulator buffers in TMEM: two of 256 columns fill it; 64-column tiles
  // keep four in flight, which hides more of a tile's hand-over latency
  static constexpr int kBufs = (NT <= 64 && kHalves == 1) ? 4 : 2;
  static constexpr int kEpiGroups = kBufs * kHalves;
  static constexpr int kThreads = 64 + kEpiGroups * kEpiThreads;   // producer, MMA, epilogue
  static constexpr uint32_t kTmemCols =
      kBufs * NT >= 512 ? 512 : (kBufs * NT >= 256 ? 256 : (kBufs * NT >= 128 ? 128 : 64));
  static constexpr uint32_t kQBytes = NT * D_I;          // one query group tile
  static constexpr uint32_t kKBytes = kBlockK * D_I;     // one key tile
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;
  static constexpr uint32_t kOffWq = kOffK + kStages * kKBytes;
  static constexpr uint32_t kOffBar = kOffWq + kEpiGroups * (kN / kHalves) * 4;  // wq per warpgroup
  // barriers: q_full[2], q_empty[2], k_full[S], k_empty[S], acc_full[B], acc_empty[B], drain
  static constexpr uint32_t kNumBars = 2 + 2 + kStages + kStages + 2 * kBufs + 1;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kOffPre = kOffMisc + 16;     // int32 [kMaxDenseB + 1]
  static constexpr uint32_t kBytes = kOffPre + (kMaxDenseB + 1) * 4;
  static constexpr uint32_t kSmem = kBytes + 1024;      // + alignment slack
  static constexpr uint32_t kSwizzle = D_I == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t kSbo = 8 * D_I;              // 8 rows of one swizzle width
  static constexpr uint32_t kIdesc = instr_desc(kFmtE4M3, kFmtE4M3, 0, 0, kBlockK, kN);
};

// CMP: the read-out appends candidates (kIdxCompact) instead of storing scores.
template <int H_I, int D_I, int NT, bool CMP>
__global__ void __launch_bounds__(Layout<H_I, D_I, NT>::kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k, const Params P) {
  using L = Layout<H_I, D_I, NT>;
  constexpr int kN = L::kN;
  constexpr int QPT = L::QPT;
  // a launch on a row subset with no row set does nothing (the same word
  // for every thread, read before any barrier or TMEM allocation)
  if (P.any_on && *P.any_on == 0u) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  float* wq_s = reinterpret_cast<float*>(smem + L::kOffWq);
  const uint32_t bar0 = sbase + L::kOffBar;
  auto q_full = [&](int i) { return bar0 + 8u * i; };
  auto q_empty = [&](int i) { return bar0 + 8u * (2 + i); };
  auto k_full = [&](int i) { return bar0 + 8u * (4 + i); };
  auto k_empty = [&](int i) { return bar0 + 8u * (4 + kStages + i); };
  constexpr int kBufs = L::kBufs;
  auto acc_full = [&](int i) { return bar0 + 8u * (4 + 2 * kStages + i); };
  auto acc_empty = [&](int i) { return bar0 + 8u * (4 + 2 * kStages + kBufs + i); };
  const uint32_t drain_bar = bar0 + 8u * (4 + 2 * kStages + 2 * kBufs);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);
  int* pre = reinterpret_cast<int*>(smem + L::kOffPre);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // one-query batches: chunk counts of the sequences, prefix-summed by warp 0
  // (made visible to every role by the barrier after the TMEM allocation)
  int64_t n_items = P.n_items;
  if (QPT == 1 && P.dense) {
    if (warp == 0) {
      int carry = 0;
      for (int b0 = 0; b0 < P.B; b0 += 32) {
        const int b = b0 + lane;
        int c = 0;
        if (b < P.B && __ldg(P.cu_q + b + 1) > __ldg(P.cu_q + b)) {
          const int len_k = __ldg(P.cu_k + b + 1) - __ldg(P.cu_k + b);
          c = (len_k + kDenseKb * kBlockK - 1) / (kDenseKb * kBlockK);
        }
        int x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (b < P.B) pre[b] = carry + x - c;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) pre[P.B] = carry;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
    }
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 4 * L::kHalves);   // every warp that reads the buffer
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (QPT == 1 && P.dense) n_items = pre[P.B];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int64_t qc = 0, kc = 0;
      int st = 0;            // key stage of tile kc and its fill parity
      uint32_t kpar = 0u;
      bool ok = true;
      const bool dropped = (P.err.inject & kInjectDropFirstKeyLoad) != 0;
      // the key tiles are read by every query group: keep them in L2 while
      // the score rows stream through it
      const uint64_t keep = l2_policy_evict_last();
      for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        Item it;
        if (!decode_item<QPT>(item, P, pre, it)) continue;
        const int qb = static_cast<int>(qc & 1);
        if (!(ok = mbar_wait(q_empty(qb), static_cast<uint32_t>(((qc >> 1) & 1) ^ 1), P.err))) break;
        mbar_arrive_expect_tx(q_full(qb), L::kQBytes);
        tma_load_2d(sbase + L::kOffQ + qb * L::kQBytes, &tmap_q, 0, it.q_row0 * H_I, q_full(qb));
        ++qc;
        for (int j = 0; j < it.nkb; ++j) {
          if (!(ok = mbar_wait(k_empty(st), kpar ^ 1u, P.err))) break;
          // test hook: the first key tile is never loaded, so the MMA
          // issuer's bounded wait for it runs out
          if (kc != 0 || !dropped) {
            mbar_arrive_expect_tx(k_full(st), L::kKBytes);
            tma_load_2d_hint(sbase + L::kOffK + st * L::kKBytes, &tmap_k, 0,
                             it.k_row0 + (it.kb0 + j) * kBlockK, k_full(st), keep);
          }
          ++kc;
          if (++st == kStages) {
            st = 0;
            kpar ^= 1u;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      // Let this CTA's own loads in flight land before leaving.  On the
      // normal path the MMA issuer has consumed every one of them and these
      // waits return at once; after a failure elsewhere (the MMA issuer or
      // an epilogue warp gave up) some may still be landing.
      for (int64_t u = (kc > kStages ? kc - kStages : 0); u < kc; ++u) {
        if (u == 0 && dropped) continue;
        mbar_wait_drain(k_full(static_cast<int>(u % kStages)),
                        static_cast<uint32_t>((u / kStages) & 1), P.err);
      }
      for (int64_t u = (qc > 2 ? qc - 2 : 0); u < qc; ++u)
        mbar_wait_drain(q_full(static_cast<int>(u & 1)), static_cast<uint32_t>((u >> 1) & 1),
                        P.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Lane 0 alone walks the items, waits and issues a tile's MMAs: the warp
    // shares its scheduler with the read-out warps, so every instruction per
    // tile counts (no broadcast of wait verdicts, no elect, no warp sync).
    // The descriptors are built once (a stage or query buffer adds a multiple
    // of its size, in 16-byte units, to the start-address field) and the ring
    // positions are running counters: key stage st and its fill parity,
    // accumulator buffer ab and its phase.
    bool ok = true;
    if (lane == 0) {
      int64_t qc = 0;
      int st = 0, ab = 0;
      uint32_t kpar = 0u, apar = 0u;
      const uint64_t a0 = smem_desc(sbase + L::kOffK, 16, L::kSbo, L::kSwizzle);
      const uint64_t b0 = smem_desc(sbase + L::kOffQ, 16, L::kSbo, L::kSwizzle);
      for (int64_t item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        Item it;
        if (!decode_item<QPT>(item, P, pre, it)) continue;
        const int qb = static_cast<int>(qc & 1);
        if (!(ok = mbar_wait(q_full(qb), static_cast<uint32_t>((qc >> 1) & 1), P.err))) break;
        const uint64_t bq = b0 + ((static_cast<uint32_t>(qb) * L::kQBytes) >> 4);
        for (int j = 0; j < it.nkb; ++j) {
          ok = mbar_wait(k_full(st), kpar, P.err) && mbar_wait(acc_empty(ab), apar ^ 1u, P.err);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ak = a0 + ((static_cast<uint32_t>(st) * L::kKBytes) >> 4);
          const uint32_t d = tmem + static_cast<uint32_t>(ab) * kN;
#pragma unroll
          for (int kk = 0; kk < D_I / 32; ++kk)
            mma_f8(d, ak + (kk * 32 >> 4), bq + (kk * 32 >> 4), L::kIdesc, kk > 0 ? 1u : 0u);
          mma_commit(k_empty(st));
          mma_commit(acc_full(ab));
          if (++st == kStages) {
            st = 0;
            kpar ^= 1u;
          }
          if (++ab == kBufs) {
            ab = 0;
            apar ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(q_empty(qb));
        ++qc;
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    // every MMA issued by this warp completes before TMEM is released
    mma_commit_warp(drain_bar);
    if (lane == 0) {
      mbar_wait_drain(drain_bar, 0, P.err);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Warpgroup eg reads accumulator buffer eg / kHalves (every kBufs-th
    // tile) and the column half eg % kHalves.  Warp w reads TMEM lanes
    // 32*(w%4)..; a thread owns one key of the tile.
    const int eg = (warp - 2) >> 2;            // warpgroup 0..3
    const int ab_mine = eg / L::kHalves;
    const int hf = eg % L::kHalves;
    const int et = threadIdx.x - 64 - eg * kEpiThreads;   // 0..127 within the group
    const uint32_t bar_id = 1 + eg;
    const int sp = warp & 3;                  // TMEM sub-partition of this warp
    const int row = sp * 32 + lane;           // TMEM lane = key within the tile
    const uint32_t lane_addr = static_cast<uint32_t>(sp * 32) << 16;
    constexpr int kHalf = kN / L::kHalves;    // columns per warpgroup
    constexpr int QH = QPT / L::kHalves;      // queries per warpgroup
    // independent FMA chains per query (latency hiding)
    constexpr int NCH = H_I >= 16 ? 4 : (H_I >= 8 ? 2 : 1);
    // chunks of 32 columns loaded per tcgen05.wait (register budget)
    constexpr int kChunksPerWait = 1;
    float* wq = wq_s + eg * kHalf;
    int64_t ac = 0;
    bool ok = true;
    // compact mode: per query of this warpgroup, the last key it may append
    // (its position or the sequence's last key) and its threshold
    constexpr int QP = CMP ? QH : 1;
    int lim_q[QP];
    float thr_q[QP];
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
      Item it;
      if (!decode_item<QPT>(item, P, pre, it)) continue;
      // the warpgroup stops together once a wait of one of its warps gave up
      if (named_bar_or(bar_id, kEpiThreads, !ok)) break;
      // head weights of this half of the query group: w * q_scale
      for (int n = et; n < kHalf; n += kEpiThreads) {
        const int col = hf * kHalf + n;
        const int qi = col / H_I;
        float v = 0.f;
        if (qi < it.nq) {
          const int64_t o = static_cast<int64_t>(it.q_row0 + qi) * H_I + (col % H_I);
          v = __ldg(P.w + o) * __ldg(P.q_scale + o);
        }
        wq[n] = v;
      }
      if constexpr (CMP) {
#pragma unroll
        for (int ql = 0; ql < QP; ++ql) {
          const int qi = hf * QH + ql;
          thr_q[ql] = qi < it.nq ? __ldg(P.thr + it.q_row0 + qi) : 0.f;
          lim_q[ql] = qi < it.nq ? min(it.len_k - it.len_q + it.q0 + qi, it.len_k - 1) : -1;
        }
      }
      named_bar_sync(bar_id, kEpiThreads);
      for (int j = 0; j < it.nkb; ++j, ++ac) {
        const int ab = static_cast<int>(ac % kBufs);
        if (ab != ab_mine) continue;
        // the key's scale is fetched before the accumulator is waited for,
        // so its latency hides behind the MMA
        const int s_local = (it.kb0 + j) * kBlockK + row;
        const float ks = s_local < it.len_k ? __ldg(P.k_scale + it.k_row0 + s_local) : 0.f;
        // each warp waits and releases on its own: no warpgroup barrier per tile
        if (!warp_wait(acc_full(ab), static_cast<uint32_t>((ac / kBufs) & 1), P.err)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        float2 acc[QH][NCH];
#pragma unroll
        for (int qi = 0; qi < QH; ++qi) {
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) acc[qi][ch] = make_float2(0.f, 0.f);
        }
        const uint32_t dcol = tmem + lane_addr + static_cast<uint32_t>(ab) * kN + hf * kHalf;
#pragma unroll
        // Columns of queries past the group's last one (a sequence's last
        // group) carry weight 0 and add exactly nothing; their scores are not
        // stored, so every tile is read out alike, without branches.
        for (int cg = 0; cg < kHalf / 32; cg += kChunksPerWait) {
          uint32_t v[kChunksPerWait][32];
#pragma unroll
          for (int u = 0; u < kChunksPerWait; ++u) tmem_ld_32x32b_x32(dcol + (cg + u) * 32, v[u]);
          tmem_wait_ld();
          if (cg + kChunksPerWait >= kHalf / 32) {
            // the last columns are in registers: hand the buffer back before
            // they are folded, so the next MMA into it can start earlier
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(ab));
          }
#pragma unroll
          for (int u = 0; u < kChunksPerWait; ++u) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const int n = (cg + u) * 32 + c;          // column within the half
              const int ql = n / H_I;                   // query within the half
              const int ch = ((n % H_I) / 4) % NCH;
              const float4 w4 = *reinterpret_cast<const float4*>(wq + n);
              const float2 x01 = make_float2(fmaxf(__uint_as_float(v[u][c]), 0.f),
                                             fmaxf(__uint_as_float(v[u][c + 1]), 0.f));
              const float2 x23 = make_float2(fmaxf(__uint_as_float(v[u][c + 2]), 0.f),
                                             fmaxf(__uint_as_float(v[u][c + 3]), 0.f));
              acc[ql][ch] = __ffma2_rn(make_float2(w4.x, w4.y), x01, acc[ql][ch]);
              acc[ql][ch] = __ffma2_rn(make_float2(w4.z, w4.w), x23, acc[ql][ch]);
            }
          }
        }
        const int p0 = it.len_k - it.len_q + it.q0;
        if constexpr (CMP) {
          // candidates: the causal scores at or above the row's threshold;
          // one atomic per warp and query reserves their slots, lane order
          // fills them
#pragma unroll
          for (int ql = 0; ql < QH; ++ql) {
            float sum = 0.f;
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) sum += acc[ql][ch].x + acc[ql][ch].y;
            const float sc = sum * ks;
            const bool pass = s_local <= lim_q[ql] && sc >= thr_q[ql];
            const uint32_t bal = __ballot_sync(0xffffffffu, pass);
            if (bal != 0u) {
              const int64_t r = it.q_row0 + hf * QH + ql;
              uint32_t base = 0u;
              if (lane == 0) base = atomicAdd(P.cnt + r, static_cast<uint32_t>(__popc(bal)));
              base = __shfl_sync(0xffffffffu, base, 0);
              const uint32_t slot = base + __popc(bal & ((1u << lane) - 1u));
              if (pass && slot < static_cast<uint32_t>(P.cap)) {
                const int64_t o = r * P.cap + slot;
                P.cand_key[o] = order_key(sc);
                P.cand_pos[o] = s_local;
              }
            }
          }
        } else if (s_local < it.len_k) {
#pragma unroll
          for (int ql = 0; ql < QH; ++ql) {
            const int qi = hf * QH + ql;
            float sum = 0.f;
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) sum += acc[ql][ch].x + acc[ql][ch].y;
            if (qi < it.nq && (P.mode == kIdxRect || s_local <= p0 + qi))
              st_global_stream(P.logits + static_cast<int64_t>(it.q_row0 + qi) * P.ld + s_local,
                               sum * ks);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int H_I, int D_I, int NT, bool CMP>
cudaError_t launch_t(const CUtensorMap& tq, const CUtensorMap& tk, const IndexerArgs& a,
                     int num_sms, DevErr err, cudaStream_t s) {
  using L = Layout<H_I, D_I, NT>;
  Params P;
  P.q_scale = a.q_scale;
  P.w = a.w;
  P.k_scale = a.k_scale;
  P.cu_q = a.cu_q;
  P.cu_k = a.cu_k;
  P.logits = a.logits;
  P.ld = a.ld;
  P.B = a.B;
  P.dense = (L::QPT == 1 && a.max_len_q <= 1 && a.B <= kMaxDenseB) ? 1 : 0;
  P.mode = a.mode;
  P.thr = a.thr;
  P.cand_key = a.cand_key;
  P.cand_pos = a.cand_pos;
  P.cnt = a.cnt;
  P.cap = a.cap;
  P.row_on = a.row_on;
  P.any_on = a.any_on;
  P.n_qg = (a.max_len_q + L::QPT - 1) / L::QPT;
  P.n_kc = (a.max_len_k + kKbPerItem * kBlockK - 1) / (kKbPerItem * kBlockK);
  P.n_items = static_cast<int64_t>(a.B) * P.n_qg * P.n_kc;
  P.err = err;
  if (P.n_items == 0) return cudaSuccess;
  const int64_t grid = P.n_items < num_sms ? P.n_items : num_sms;
  // Virtual key chunks past the last one are skipped like any chunk outside
  // the causal triangle; padding their count to be coprime with the grid
  // makes each CTA's stride cycle through every chunk index.
  auto gcd = [](int64_t x, int64_t y) {
    while (y) {
      const int64_t t = x % y;
      x = y;
      y = t;
    }
    return x;
  };
  while (gcd(P.n_kc, grid) != 1) ++P.n_kc;
  P.n_items = static_cast<int64_t>(a.B) * P.n_qg * P.n_kc;
  auto kern = indexer_kernel<H_I, D_I, NT, CMP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kSmem));
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(grid), L::kThreads, L::kSmem, s>>>(tq, tk, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer(const CUtensorMap& tq, const CUtensorMap& tk, const IndexerArgs& a,
                           int num_sms, DevErr err, cudaStream_t s) {
  // the compact read-out is built for the 64-head indexer only
  if (a.mode == kIdxCompact) {
    if (a.H_I != 64) return cudaErrorInvalidValue;
    if (a.d_I == 128 && a.tile_n == 256) return launch_t<64, 128, 256, true>(tq, tk, a, num_sms, err, s);
    if (a.d_I == 128 && a.tile_n == 64) return launch_t<64, 128, 64, true>(tq, tk, a, num_sms, err, s);
    if (a.d_I == 64 && a.tile_n == 256) return launch_t<64, 64, 256, true>(tq, tk, a, num_sms, err, s);
    if (a.d_I == 64 && a.tile_n == 64) return launch_t<64, 64, 64, true>(tq, tk, a, num_sms, err, s);
    return cudaErrorInvalidValue;
  }
#define DSA_IDX_CASE(h, d)                                                               \
  if (a.H_I == h && a.d_I == d && a.tile_n == 256) return launch_t<h, d, 256, false>(tq, tk, a, num_sms, err, s);
#define DSA_IDX_CASE_DECODE(h, d)                                                        \
  if (a.H_I == h && a.d_I == d && a.tile_n == 64) return launch_t<h, d, 64, false>(tq, tk, a, num_sms, err, s);
  DSA_IDX_CASE(4, 64)
  DSA_IDX_CASE(8, 64)
  DSA_IDX_CASE(16, 64)
  DSA_IDX_CASE(32, 64)
  DSA_IDX_CASE(64, 64)
  DSA_IDX_CASE(128, 64)
  DSA_IDX_CASE(4, 128)
  DSA_IDX_CASE(8, 128)
  DSA_IDX_CASE(16, 128)
  DSA_IDX_CASE(32, 128)
  DSA_IDX_CASE(64, 128)
  DSA_IDX_CASE(128, 128)
  DSA_IDX_CASE_DECODE(16, 64)
  DSA_IDX_CASE_DECODE(32, 64)
  DSA_IDX_CASE_DECODE(64, 64)
  DSA_IDX_CASE_DECODE(16, 128)
  DSA_IDX_CASE_DECODE(32, 128)
  DSA_IDX_CASE_DECODE(64, 128)
#undef DSA_IDX_CASE
#undef DSA_IDX_CASE_DECODE
  return cudaErrorInvalidValue;
}

}  // namespace dsa
