// sparse_mla.cu -- sparse attention in the MQA mode of MLA on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": attention reads nothing but the selected
// entries, and in MQA mode each selected latent is used by every query head; "DeepSeek-V3.2" atlas entry, "Inference efficiency": only the chosen
// latents of the cache are touched):
//
//   out[t,h,:] = sum_{s in S_t} softmax_s(scale * q[t,h,:] . c[s,:]) * c[s,0:512]
//   lse[t,h]   = log sum_{s in S_t} exp(scale * q[t,h,:] . c[s,:])
//
// How: a persistent grid of one CTA per SM.  A work item is (query, group of
// 64 heads); CTA c takes items c, c + grid, ... with the longest rows first.
// Every item is one query tile followed by its blocks of 64 selected keys,
// and all of them flow through one ring of three 72 KB shared-memory slots,
// so consecutive items overlap: the next item's query and first scores are
// in flight while the previous item's last products and output finish.
// 448 threads:
//  * warps 5..8 (gather): fill the ring slot by slot with 16-byte cp.async
//    into 128-byte-swizzled tiles (64 rows x 9 chunks of 64 columns): the
//    query rows of an item, or the 576-d latent rows its indices select.
//    Eight threads cover one 128-byte row segment, so every warp
//    instruction moves four full 128-byte lines.  A gathered tile is shared
//    by all 64 heads of the item (group-shared selection).
//  * warps 4 and 13 (MMA): warp 4 issues S of each block (36 tcgen05.mma,
//    M=64 heads, N=64 keys, K=16, query read from TMEM) and warp 13 O += P V
//    (8 tcgen05.mma, M=64, N=256, K=16) with P from shared memory and V
//    read MN-major from the first 512 columns of the same tile; in each, one
//    elected lane issues a block's run of MMAs.  P of a block is
//    written over that block's RoPE columns (512..575), which S no longer
//    needs, so P lives and dies with its slot.
//  * warps 0..3 (softmax): each owns 16 heads and all 32 lanes work: the
//    16x256b TMEM access shape gives lane t the rows t/4 and 8+t/4 of the
//    warp's 16, two adjacent columns of every group of 8.  Per block they
//    read S, run the online softmax in fp32 (exp2, lazily rescaled maximum),
//    write P (bf16) to shared memory and rescale their own O rows in TMEM
//    when their maximum moves; at the end of an item they hand the row
//    statistics on.
//  * warps 9..12 (output, same lane mapping): move each item's query tile
//    from its ring slot into TMEM (as soon as the previous item's last S
//    is done), and once an item's last product has landed, normalise O and
//    store bf16 out (16-byte stores after a 4 x 4 shuffle transpose) and the
//    lse, handing the accumulator back after its last chunk is loaded.
//
// TMEM (512 columns x 128 lanes): an M=64 accumulator fills lanes 0-15 of
// each 32-lane sub-partition; a second one at lane offset 16 fills lanes
// 16-31.  O (64 heads x 512 fp32) takes columns 0..511 at lane offset 0; the
// two S buffers (64 x 64) take columns 0..63 and 64..127 at lane offset 16,
// and the query tile (64 x 576 bf16, two elements per column) takes columns
// 128..415 at lane offset 16, the same lanes as the S rows it produces.
// Sub-partition w holds S, O and query rows of heads 16w..16w+15, and in
// each of them a lane holds the same two heads.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kHeads = 64;       // heads per item (MMA M)
constexpr int kBlockN = 64;      // keys per block
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kChunks = kDqk / 64;                // 9 column chunks of 64
constexpr uint32_t kChunkBytes = 64 * 128;        // 64 rows x 128 B
constexpr int kStages = 3;                        // ring slots
constexpr uint32_t kKvBytes = kChunks * kChunkBytes;  // 73728
constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffPInStage = 8 * kChunkBytes;    // P (64 x 64 bf16) over the RoPE chunk
constexpr int kStatRing = 4;                      // row statistics of items in flight
constexpr uint32_t kOffBar = kOffKv + kStages * kKvBytes;
// barriers: kv_full[S], kv_empty[S], p_full[S], s_full[2], s_free[2],
// q_ready, o_full, o_free, stats_full[kStatRing], drain[2], s_last
constexpr uint32_t kNumBars = 3 * kStages + 4 + 3 + kStatRing + 2 + 1;
constexpr uint32_t kOffStats = (kOffBar + kNumBars * 8 + 15) & ~15u;   // [kStatRing][64][4] floats
constexpr uint32_t kOffMisc = kOffStats + kStatRing * kHeads * 4 * 4;
constexpr uint32_t kSmem = kOffMisc + 32 + 1024;
constexpr uint32_t kQCol = 128;                 // TMEM column of the query tile

constexpr int kSmWarps = 4;                 // warps 0..3
constexpr int kMmaWarp = 4;                 // warp 4
constexpr int kProdWarp0 = 5;               // warps 5..8
constexpr int kProdThreads = 128;
constexpr int kOutWarp0 = 9;                // warps 9..12
constexpr int kPvWarp = 13;                 // warp 13
constexpr int kThreads = 32 * 14;           // 448
constexpr uint32_t kBarProducer = 1;        // named barrier of the ring filler
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescS = instr_desc(kFmtBF16, kFmtBF16, 0, 0, kHeads, kBlockN);
constexpr uint32_t kIdescPV = instr_desc(kFmtBF16, kFmtBF16, 0, 1, kHeads, 256);
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmem <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv;
  const int32_t* idx;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, H, k, head_groups;
  int64_t total_q;
  int64_t n_items;           // total_q * head_groups
  float scale_log2;          // sm_scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  DevErr err;
};

// One work item: a query row and a group of 64 heads.
struct Item {
  int64_t q_row;
  int hg;
  int p;            // absolute position of the query
  int n_sel;        // selected entries: min(k, p + 1)
  int nb;           // blocks of 64 entries
  int heads_here;   // heads of the group that exist
  int ck0;          // first key row of the sequence
};

// Items are numbered so that the longest rows (the last queries of the
// batch) come first: a CTA that draws short rows at the end fills the tail.
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

// Exchanges four 32-bit values among the four lanes that share a row in the
// 16x256b layout (lanes 4r..4r+3): afterwards lane q holds v[g] = the value
// lane g held in v[q].
__device__ __forceinline__ void transpose4(uint32_t (&v)[4], int q) {
  {
    const bool odd = (q & 1) != 0;
    const uint32_t r0 = __shfl_xor_sync(0xffffffffu, odd ? v[0] : v[1], 1);
    const uint32_t r1 = __shfl_xor_sync(0xffffffffu, odd ? v[2] : v[3], 1);
    if (odd) { v[0] = r0; v[2] = r1; } else { v[1] = r0; v[3] = r1; }
  }
  {
    const bool hi = (q & 2) != 0;
    const uint32_t r0 = __shfl_xor_sync(0xffffffffu, hi ? v[0] : v[2], 2);
    const uint32_t r1 = __shfl_xor_sync(0xffffffffu, hi ? v[1] : v[3], 2);
    if (hi) { v[0] = r0; v[1] = r1; } else { v[2] = r0; v[3] = r1; }
  }
}

// Position in this CTA's block sequence, for the roles that walk it.
struct Cursor {
  int64_t w;       // item
  Item it;
  int j;           // block within the item
  uint32_t u;      // ring slot of the block
  uint32_t gb;     // block count over all items (S buffer = gb & 1)
  uint32_t ii;     // item count
  bool valid;
};

__device__ __forceinline__ void cursor_start(Cursor& c, const Params& P) {
  c.w = blockIdx.x;
  c.j = 0;
  c.u = 1;          // slot 0 holds the first item's query
  c.gb = 0;
  c.ii = 0;
  c.valid = c.w < P.n_items;
  if (c.valid) c.it = item_at(P, c.w);
}

__device__ __forceinline__ void cursor_next(Cursor& c, const Params& P) {
  ++c.j;
  ++c.u;
  ++c.gb;
  if (c.j == c.it.nb) {
    c.j = 0;
    c.w += gridDim.x;
    ++c.ii;
    ++c.u;          // the next item's query slot
    c.valid = c.w < P.n_items;
    if (c.valid) c.it = item_at(P, c.w);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto kv_full = [&](uint32_t i) { return bar0 + 8u * i; };
  auto kv_empty = [&](uint32_t i) { return bar0 + 8u * (kStages + i); };
  auto p_full = [&](uint32_t i) { return bar0 + 8u * (2 * kStages + i); };
  auto s_full = [&](uint32_t i) { return bar0 + 8u * (3 * kStages + i); };
  auto s_free = [&](uint32_t i) { return bar0 + 8u * (3 * kStages + 2 + i); };
  const uint32_t q_ready = bar0 + 8u * (3 * kStages + 4);   // query tile in TMEM
  const uint32_t o_full = bar0 + 8u * (3 * kStages + 5);    // last P V of an item done
  const uint32_t o_free = bar0 + 8u * (3 * kStages + 6);    // O read out
  auto stats_full = [&](uint32_t i) { return bar0 + 8u * (3 * kStages + 7 + i); };
  auto drain_bar = [&](uint32_t i) { return bar0 + 8u * (3 * kStages + 7 + kStatRing + i); };
  // last S of an item done: one phase per item, so a waiter that is an item
  // ahead of the score products can never see a stale phase
  const uint32_t s_last = bar0 + 8u * (3 * kStages + 9 + kStatRing);
  float* stats = reinterpret_cast<float*>(smem + kOffStats);      // [ring][row][m, l, lr, -]
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  uint32_t* q_reads = reinterpret_cast<uint32_t*>(smem + kOffMisc + 8);   // softmax warps done with a query slot

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(kv_full(i), kProdThreads);
      mbar_init(kv_empty(i), 1);
      mbar_init(p_full(i), kSmWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), kSmWarps);
    }
    mbar_init(q_ready, kSmWarps);
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    for (int i = 0; i < kStatRing; ++i) mbar_init(stats_full(i), kSmWarps);
    mbar_init(drain_bar(0), 1);
    mbar_init(drain_bar(1), 1);
    mbar_init(s_last, 1);
    *abort_flag = 0;
    *q_reads = 0u;
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
  const uint32_t tmem_o = tmem;                         // + 256*h
  const uint32_t tmem_s = tmem + (16u << 16);           // + 64*buffer (MMA destination)
  const uint32_t tmem_q = tmem + (16u << 16) + kQCol;   // query tile (MMA A operand)

  if (warp >= kProdWarp0 && warp < kOutWarp0) {
    // ------------------------------------------------------------ ring filler
    const int tg = threadIdx.x - 32 * kProdWarp0;        // 0..127
    const int rsub = tg >> 3;                            // rows rsub + 16*pass, pass 0..3
    const int l8 = tg & 7;                               // 16-byte piece within 128 B
    bool ok = true;
    uint32_t u = 0;
    for (int64_t w = blockIdx.x; ok && w < P.n_items; w += gridDim.x) {
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
      // slot -1 is the query tile, slots 0..nb-1 the blocks
      for (int j = -1; j < it.nb; ++j, ++u) {
        const uint32_t st = u % kStages;
        // every filler thread takes the same decision to stop
        const bool failed =
            tg == 0 && !mbar_wait(kv_empty(st), static_cast<uint32_t>(((u / kStages) & 1) ^ 1), P.err);
        if (named_bar_or(kBarProducer, kProdThreads, failed || *abort_flag)) {
          if (failed) *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t stage = sbase + kOffKv + st * kKvBytes;
        if (j < 0 && tg == 0 && w + gridDim.x < P.n_items) {
          // the next item's query rows come from HBM: start them towards L2 now,
          // an item ahead of their slot
          const Item nx = item_at(P, w + gridDim.x);
          prefetch_l2_bulk(P.q + (nx.q_row * P.H + nx.hg * kHeads) * kDqk,
                           static_cast<uint32_t>(nx.heads_here) * kDqk * 2u);
        }
        if (j < 0) {
          // the query rows of the head group; rows past the last head are zero
          const __nv_bfloat16* q_grp = P.q + (it.q_row * P.H + it.hg * kHeads) * kDqk;
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) {
            const int r = rsub + 16 * pass;
            const uint32_t dst = stage + r * 128 + ((l8 ^ (r & 7)) << 4);
            if (r < it.heads_here) {
              const __nv_bfloat16* src = q_grp + static_cast<int64_t>(r) * kDqk + l8 * 8;
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
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(kv_full(st));
        // the next block's rows, loaded after the arrive: its release
        // semantics would otherwise hold the slot back until they land
        if (j + 1 < it.nb) {
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) rows[pass] = load_idx(j + 1, rsub + 16 * pass);
        }
      }
    }
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // ------------------------------------------------------------ MMA issuers
    // Two warps issue: warp kMmaWarp the score products S = Q K^T, warp
    // kPvWarp the value products O += P V, each walking the block sequence
    // on its own.  Each runs its loop in lockstep and one elected lane issues
    // a block's run of MMAs; every value the MMAs use is warp-uniform.  With
    // two issuers the waits and bookkeeping of one overlap the other's
    // MMAs, so the tensor pipe does not drain between the two products.
    // Descriptors are built once; every MMA only adds a compile-time offset
    // (in 16-byte units) to the start-address field.
    constexpr uint64_t kStageStep = kKvBytes >> 4;
    bool ok = true;
    Cursor c;
    cursor_start(c, P);
    if (warp == kMmaWarp) {
      const uint64_t dS0 = smem_desc(sbase + kOffKv, 16, 1024, kSwizzle128B);  // K, K-major
      while (ok && c.valid) {
        const uint32_t st = c.u % kStages;
        const uint32_t sb = c.gb & 1;              // S buffer
        ok = (c.j != 0 || warp_wait(q_ready, c.ii & 1, P.err)) &&
             warp_wait(kv_full(st), (c.u / kStages) & 1, P.err) &&
             warp_wait(s_free(sb), ((c.gb >> 1) & 1) ^ 1, P.err);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dS = dS0 + st * kStageStep;
        const uint32_t d = tmem_s + 64u * sb;
        if (elect_one()) {
#pragma unroll
          for (int cc = 0; cc < kChunks; ++cc) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f16_ts(d, tmem_q + 32u * cc + 8u * kk, dS + ((cc * kChunkBytes + kk * 32) >> 4),
                         kIdescS, (cc | kk) != 0 ? 1u : 0u);
            }
          }
          mma_commit(s_full(sb));
          if (c.j + 1 == c.it.nb) mma_commit(s_last);
        }
        __syncwarp();
        cursor_next(c, P);
      }
    } else {
      const uint64_t dP0 = smem_desc(sbase + kOffKv + kOffPInStage, 16, 1024, kSwizzle128B);
      const uint64_t dV0 = smem_desc(sbase + kOffKv, kChunkBytes, 1024, kSwizzle128B);  // MN-major
      while (ok && c.valid) {
        const uint32_t st = c.u % kStages;
        // the first product of an item overwrites O: the previous item's
        // output must have been read out
        ok = (c.j != 0 || c.ii == 0 || warp_wait(o_free, (c.ii - 1) & 1, P.err)) &&
             warp_wait(p_full(st), (c.u / kStages) & 1, P.err);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dP = dP0 + st * kStageStep;
        const uint64_t dV = dV0 + st * kStageStep;
        const uint32_t first = c.j > 0 ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f16(tmem_o + 256u * h, dP + (kk * 32 >> 4),
                      dV + ((4 * h * kChunkBytes + kk * 2048) >> 4), kIdescPV,
                      kk > 0 ? 1u : first);
            }
          }
          mma_commit(kv_empty(st));
          if (c.j + 1 == c.it.nb) mma_commit(o_full);
        }
        __syncwarp();
        cursor_next(c, P);
      }
    }
    // every MMA issued by this warp completes before TMEM is released
    const uint32_t drain = drain_bar(warp == kMmaWarp ? 0 : 1);
    mma_commit_warp(drain);
    if (lane == 0) {
      mbar_wait_drain(drain, 0, P.err);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp < kSmWarps) {
    // ------------------------------------------------------------ softmax
    const int w = warp;                       // sub-partition
    const int qd = lane & 3;                  // column pair within each group of 8
    const int ra = 16 * w + (lane >> 2);      // this lane's two heads (rows) in the group
    const int rb = ra + 8;
    const uint32_t lane_base = static_cast<uint32_t>(w * 32) << 16;
    bool ok = true;
    uint32_t u = 0, gb = 0, ii = 0;
    // Validity of block entries: lane l checks entries 2l and 2l+1.
    auto entry_ok = [&](const Item& x, int e) -> bool {
      if (e >= x.n_sel) return false;
      const int s = __ldg(P.idx + x.q_row * P.k + e);
      return s >= 0 && s <= x.p;
    };
    // The next item's bookkeeping (its global loads) is done one item ahead,
    // off the path from the last block of an item to the first of the next.
    Item it = item_at(P, blockIdx.x);
    bool nx0 = entry_ok(it, 2 * lane), nx1 = entry_ok(it, 2 * lane + 1);
    for (int64_t wi = blockIdx.x; ok && wi < P.n_items; wi += gridDim.x, ++ii) {
      ++u;                                      // the item's query slot (output warps)
      float m_a = -INFINITY, m_b = -INFINITY;   // running maxima, log2 units
      float l_a = 0.f, l_b = 0.f;               // partial denominators (fp32 probabilities), lse
      float lr_a = 0.f, lr_b = 0.f;             // partial denominators of the bf16 P, for O
      const int64_t wn = wi + gridDim.x;
      Item nit = it;
      if (wn < P.n_items) nit = item_at(P, wn);
      for (int j = 0; j < it.nb; ++j, ++u, ++gb) {
        const uint32_t sb = gb & 1;            // S buffer
        const uint32_t st = u % kStages;       // slot (P goes over its RoPE chunk)
        if (!warp_wait(s_full(sb), (gb >> 1) & 1, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[32];
        tmem_ld_16x256b_x8(tmem_s + lane_base + 64u * sb, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(sb));
        const uint32_t vmask_lo = __ballot_sync(0xffffffffu, nx0);
        const uint32_t vmask_hi = __ballot_sync(0xffffffffu, nx1);

        // key of register 4i+e (row a) and 4i+2+e (row b): 8i + 2qd + e.
        // Entries outside the selection get the raw score -inf; full blocks
        // (all but the last block of short rows) skip the masking.
        if ((vmask_lo & vmask_hi) != 0xffffffffu) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              if (!((((e ? vmask_hi : vmask_lo) >> (4 * i + qd)) & 1u) != 0)) {
                v[4 * i + e] = 0xff800000u;
                v[4 * i + 2 + e] = 0xff800000u;
              }
            }
          }
        }
        // row maxima on the raw scores (the scale is positive), in log2 units
        float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          mxa = fmaxf(mxa, fmaxf(__uint_as_float(v[4 * i + 0]), __uint_as_float(v[4 * i + 1])));
          mxb = fmaxf(mxb, fmaxf(__uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])));
        }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        mxa *= P.scale_log2;
        mxb *= P.scale_log2;
        float al_a = 1.f, al_b = 1.f;
        bool moved = false;
        if (mxa > m_a + kRescaleThreshold) {
          al_a = fast_exp2(m_a - mxa);   // 0 when m = -inf
          m_a = mxa;
          moved = true;
        }
        if (mxb > m_b + kRescaleThreshold) {
          al_b = fast_exp2(m_b - mxb);
          m_b = mxb;
          moved = true;
        }
        const bool rescale = j > 0 && __any_sync(0xffffffffu, moved);

        // P = exp2(scale * s - m) (bf16) over the slot's RoPE chunk: row r,
        // keys 8i..8i+7 are the 16-byte piece i, stored at piece i ^ (r & 7).
        // A row with no entry yet (m = -inf) has only -inf scores: p = 0.
        const float nma = m_a == -INFINITY ? 0.f : -m_a;
        const float nmb = m_b == -INFINITY ? 0.f : -m_b;
        uint8_t* pst = smem + kOffKv + st * kKvBytes + kOffPInStage;
        // two sums per row, as packed pairs: of the fp32 probabilities (for
        // the lse) and of the bf16-rounded ones the MMA consumes (O is
        // normalised by these, so its weights sum to one exactly)
        float2 s2a = make_float2(0.f, 0.f), s2b = s2a, r2a = s2a, r2b = s2a;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float pa0 = fast_exp2(fmaf(__uint_as_float(v[4 * i + 0]), P.scale_log2, nma));
          const float pa1 = fast_exp2(fmaf(__uint_as_float(v[4 * i + 1]), P.scale_log2, nma));
          const float pb0 = fast_exp2(fmaf(__uint_as_float(v[4 * i + 2]), P.scale_log2, nmb));
          const float pb1 = fast_exp2(fmaf(__uint_as_float(v[4 * i + 3]), P.scale_log2, nmb));
          s2a = __fadd2_rn(s2a, make_float2(pa0, pa1));
          s2b = __fadd2_rn(s2b, make_float2(pb0, pb1));
          const uint32_t ka = pack_bf16x2(pa0, pa1), kb = pack_bf16x2(pb0, pb1);
          r2a = __fadd2_rn(r2a, make_float2(__uint_as_float(ka << 16), __uint_as_float(ka & 0xFFFF0000u)));
          r2b = __fadd2_rn(r2b, make_float2(__uint_as_float(kb << 16), __uint_as_float(kb & 0xFFFF0000u)));
          *reinterpret_cast<uint32_t*>(pst + ra * 128 + ((i ^ (ra & 7)) << 4) + 4 * qd) = ka;
          *reinterpret_cast<uint32_t*>(pst + rb * 128 + ((i ^ (rb & 7)) << 4) + 4 * qd) = kb;
        }
        l_a = l_a * al_a + (s2a.x + s2a.y);
        l_b = l_b * al_b + (s2b.x + s2b.y);
        lr_a = lr_a * al_a + (r2a.x + r2a.y);
        lr_b = lr_b * al_b + (r2b.x + r2b.y);

        // When a maximum moved, this warp's O rows are rescaled before P V of
        // this block may run: after P V of the previous block has completed
        // (its slot is released).
        if (rescale) {
          const uint32_t pu = u - 1;
          if (!warp_wait(kv_empty(pu % kStages), (pu / kStages) & 1, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int k8 = 0; k8 < kDv / 64; ++k8) {
            uint32_t o[32];
            const uint32_t ta = tmem_o + lane_base + 64u * k8;
            tmem_ld_16x256b_x8(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              o[4 * i + 0] = __float_as_uint(__uint_as_float(o[4 * i + 0]) * al_a);
              o[4 * i + 1] = __float_as_uint(__uint_as_float(o[4 * i + 1]) * al_a);
              o[4 * i + 2] = __float_as_uint(__uint_as_float(o[4 * i + 2]) * al_b);
              o[4 * i + 3] = __float_as_uint(__uint_as_float(o[4 * i + 3]) * al_b);
            }
            tmem_st_16x256b_x8(ta, o);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(st));
        // validity of the next block's entries, loaded after the arrive (its
        // release semantics would otherwise wait for them)
        if (j + 1 < it.nb) {
          nx0 = entry_ok(it, (j + 1) * kBlockN + 2 * lane);
          nx1 = entry_ok(it, (j + 1) * kBlockN + 2 * lane + 1);
        } else if (wn < P.n_items) {
          nx0 = entry_ok(nit, 2 * lane);
          nx1 = entry_ok(nit, 2 * lane + 1);
        }
      }
      if (!ok) break;
      // ---- row statistics for the output warps
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      lr_a += __shfl_xor_sync(0xffffffffu, lr_a, 1);
      lr_a += __shfl_xor_sync(0xffffffffu, lr_a, 2);
      lr_b += __shfl_xor_sync(0xffffffffu, lr_b, 1);
      lr_b += __shfl_xor_sync(0xffffffffu, lr_b, 2);
      float* sr = stats + (ii % kStatRing) * kHeads * 4;
      if (qd == 0) {
        *reinterpret_cast<float4*>(sr + 4 * ra) = make_float4(m_a, l_a, lr_a, 0.f);
        *reinterpret_cast<float4*>(sr + 4 * rb) = make_float4(m_b, l_b, lr_b, 0.f);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(stats_full(ii % kStatRing));
      it = nit;
    }
    if (!ok && lane == 0) *abort_flag = 1;
  } else {
    // ------------------------------------------------------------ output
    // Per item: first move the next item's query tile into TMEM (as soon as
    // the item's last S product is complete), then read out O.
    const int sp = warp & 3;                  // sub-partition (warps 9..12 -> 1,2,3,0)
    const int qd = lane & 3;
    const int ra = 16 * sp + (lane >> 2);     // this lane's two heads (rows) in the group
    const int rb = ra + 8;
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    bool ok = true;
    // Query tile: ring slot uq -> TMEM columns kQCol.., lanes 16..31.
    // Column 32c+8i+2qd+e holds elements 64c+16i+4qd+2e, +1 of a row.
    auto copy_query = [&](uint32_t uq) -> bool {
      const uint32_t st = uq % kStages;
      if (!warp_wait(kv_full(st), (uq / kStages) & 1, P.err)) return false;
      const uint8_t* qs = smem + kOffKv + st * kKvBytes;
#pragma unroll 3
      for (int c = 0; c < kChunks; ++c) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pc = 2 * i + (qd >> 1);
          const uint2 va = *reinterpret_cast<const uint2*>(
              qs + c * kChunkBytes + ra * 128 + ((pc ^ (ra & 7)) << 4) + 8 * (qd & 1));
          const uint2 vb = *reinterpret_cast<const uint2*>(
              qs + c * kChunkBytes + rb * 128 + ((pc ^ (rb & 7)) << 4) + 8 * (qd & 1));
          r[4 * i + 0] = va.x;
          r[4 * i + 1] = va.y;
          r[4 * i + 2] = vb.x;
          r[4 * i + 3] = vb.y;
        }
        tmem_st_16x256b_x4(tmem_q + lane_base + 32u * c, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // The fourth warp to finish reading hands the slot back.  This comes
        // before q_ready: once q_ready completes, every warp has counted
        // itself, so the counter is back at zero for the next item.
        if (atomicAdd(q_reads, 1u) == 3u) {
          *q_reads = 0u;
          mbar_arrive(kv_empty(st));
        }
        // every slot completes one phase of each of its barriers, so the
        // phase parities stay a function of the slot number alone
        mbar_arrive(p_full(st));
        mbar_arrive(q_ready);
      }
      return true;
    };
    uint32_t u = 0, ii = 0;
    Item it = item_at(P, blockIdx.x);
    ok = copy_query(0);
    for (int64_t wi = blockIdx.x; ok && wi < P.n_items; wi += gridDim.x, ++ii) {
      u += 1 + it.nb;                          // the next item's query slot
      const int64_t wn = wi + gridDim.x;
      Item nit = it;
      if (wn < P.n_items) {
        nit = item_at(P, wn);
        // the query region of TMEM is free once this item's last S is done
        ok = warp_wait(s_last, ii & 1, P.err) && copy_query(u);
        if (!ok) break;
      }
      if (!warp_wait(stats_full(ii % kStatRing), (ii / kStatRing) & 1, P.err) ||
          !warp_wait(o_full, ii & 1, P.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // O is read two chunks at a time: the load of the next chunk is in
      // flight while the current one is converted and stored, and O is
      // handed back as soon as the last chunk has landed in registers.
      uint32_t oa_[32], ob_[32];
      tmem_ld_16x256b_x8(tmem_o + lane_base, oa_);
      const float* sr = stats + (ii % kStatRing) * kHeads * 4;
      const float4 sa = *reinterpret_cast<const float4*>(sr + 4 * ra);
      const float4 sb = *reinterpret_cast<const float4*>(sr + 4 * rb);
      const float inv_a = sa.z > 0.f ? 1.f / sa.z : 0.f;
      const float inv_b = sb.z > 0.f ? 1.f / sb.z : 0.f;
      const int64_t head0 = it.q_row * P.H + it.hg * kHeads;
      const bool have_a = ra < it.heads_here, have_b = rb < it.heads_here;
      __nv_bfloat16* oa = P.out + (head0 + ra) * kDv;
      __nv_bfloat16* ob = P.out + (head0 + rb) * kDv;
      auto store_chunk = [&](const uint32_t (&o)[32], int k8) {
#pragma unroll
        for (int uu = 0; uu < 2; ++uu) {
          // groups 4uu..4uu+3 (dims 64k8 + 32uu .. +31); after the transpose
          // lane qd holds the 8 dims of group 4uu+qd as one 16-byte piece
          uint32_t pa[4], pb[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int i = 4 * uu + g;
            pa[g] = pack_bf16x2(__uint_as_float(o[4 * i + 0]) * inv_a,
                                __uint_as_float(o[4 * i + 1]) * inv_a);
            pb[g] = pack_bf16x2(__uint_as_float(o[4 * i + 2]) * inv_b,
                                __uint_as_float(o[4 * i + 3]) * inv_b);
          }
          transpose4(pa, qd);
          transpose4(pb, qd);
          const int dim = 64 * k8 + 8 * (4 * uu + qd);
          if (have_a) *reinterpret_cast<uint4*>(oa + dim) = make_uint4(pa[0], pa[1], pa[2], pa[3]);
          if (have_b) *reinterpret_cast<uint4*>(ob + dim) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
        }
      };
#pragma unroll 1
      for (int k2 = 0; k2 < kDv / 128; ++k2) {
        tmem_wait_ld();
        tmem_ld_16x256b_x8(tmem_o + lane_base + 64u * (2 * k2 + 1), ob_);
        store_chunk(oa_, 2 * k2);
        tmem_wait_ld();
        if (k2 + 1 < kDv / 128) {
          tmem_ld_16x256b_x8(tmem_o + lane_base + 64u * (2 * k2 + 2), oa_);
        } else {
          // O has been read: the next item's first P V may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
        store_chunk(ob_, 2 * k2 + 1);
      }
      if (P.lse && qd == 0) {
        if (have_a) P.lse[head0 + ra] = sa.y > 0.f ? (sa.x + log2f(sa.y)) * 0.69314718055994531f : -INFINITY;
        if (have_b) P.lse[head0 + rb] = sb.y > 0.f ? (sb.x + log2f(sb.y)) * 0.69314718055994531f : -INFINITY;
      }
      it = nit;
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

}  // namespace

cudaError_t launch_sparse_mla(const void* q, const void* kv, const MlaArgs& a, DevErr err,
                              cudaStream_t s) {
  Params P;
  P.q = static_cast<const __nv_bfloat16*>(q);
  P.kv = static_cast<const __nv_bfloat16*>(kv);
  P.idx = a.idx;
  P.cu_q = a.cu_q;
  P.cu_k = a.cu_k;
  P.B = a.B;
  P.H = a.H;
  P.k = a.k;
  P.head_groups = (a.H + kHeads - 1) / kHeads;
  P.total_q = a.total_q;
  P.n_items = a.total_q * P.head_groups;
  P.scale_log2 = a.sm_scale * 1.4426950408889634f;
  P.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  P.lse = a.lse;
  P.err = err;
  if (P.n_items == 0) return cudaSuccess;
  const int64_t grid = P.n_items < a.num_sms ? P.n_items : a.num_sms;
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  sparse_mla_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, s>>>(P);
  return cudaGetLastError();
}

}  // namespace dsa
