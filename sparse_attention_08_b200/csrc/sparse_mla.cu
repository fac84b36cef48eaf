// sparse_mla.cu -- sparse attention in the MQA mode of MLA on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section "How
// the lightning indexer works": the main attention runs only over the
// selected entries, and in MQA mode every selected latent serves all query
// heads; "DeepSeek-V3.2" atlas entry, "Inference efficiency": only the chosen
// latents of the cache are touched):
//
//   out[t,h,:] = sum_{s in S_t} softmax_s(scale * q[t,h,:] . c[s,:]) * c[s,0:512]
//   lse[t,h]   = log sum_{s in S_t} exp(scale * q[t,h,:] . c[s,:])
//
// How (one CTA per (query, group of 64 heads), 416 threads):
//  * warps 5..12 (gather): two groups of 128 threads take alternate blocks
//    of 64 selected keys, so two blocks are in flight; each copies the 576-d
//    latent rows with 16-byte cp.async into a 128-byte-swizzled 72 KB tile
//    (three stages).  Eight threads cover one 128-byte row segment, so every
//    warp instruction moves four full 128-byte lines.  The gathered tile is
//    shared by all 64 heads of the CTA (group-shared selection).  Before its
//    first block, group 0 copies the CTA's 64 x 576 query tile the same way
//    into the third stage, which is handed back once the query is in TMEM.
//  * warp 4 (MMA): the whole warp runs the issue loop and one elected lane
//    issues, in a fixed order: S of block j+1 (36 tcgen05.mma, M=64 heads,
//    N=64 keys, K=16, query read from TMEM), then O += P V of block j (8
//    tcgen05.mma, M=64, N=256, K=16) with P from shared memory and V read
//    MN-major from the first 512 columns of the same tile.  P of a block is
//    written over that block's RoPE columns (512..575), which S no longer
//    needs, so P lives and dies with its latent stage.
//  * warps 0..3 (softmax): each owns 16 heads and all 32 lanes work: the
//    16x256b TMEM access shape gives lane t the rows t/4 and 8+t/4 of the
//    warp's 16, two adjacent columns of every group of 8.  They move the
//    query tile into TMEM; then per block read S, run the online softmax in
//    fp32 (exp2, lazily rescaled maximum), write P (bf16) to shared memory
//    and rescale their own O rows in TMEM when their maximum moves; finally
//    they normalise O and store bf16 out (16-byte stores after a 4 x 4
//    shuffle transpose) and the lse.
//
// TMEM (512 columns x 128 lanes): an M=64 accumulator fills lanes 0-15 of
// each 32-lane sub-partition; a second one at lane offset 16 fills lanes
// 16-31.  O (64 heads x 512 fp32) takes columns 0..511 at lane offset 0; the
// two S buffers (64 x 64) take columns 0..63 and 64..127 at lane offset 16,
// and the query tile (64 x 576 bf16, two elements per column) takes columns
// 128..415 at lane offset 16, the same lanes as the S rows it produces.
// Softmax warp w (sub-partition w) thus holds S, O and query rows of heads
// 16w..16w+15, and every lane the same two heads in all three.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kHeads = 64;       // heads per CTA (MMA M)
constexpr int kBlockN = 64;      // keys per block
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kChunks = kDqk / 64;                // 9 column chunks of 64
constexpr uint32_t kChunkBytes = 64 * 128;        // 64 rows x 128 B
constexpr int kStages = 3;
constexpr int kQStage = 2;                        // stage that first holds the query tile
constexpr uint32_t kKvBytes = kChunks * kChunkBytes;  // 73728
constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffPInStage = 8 * kChunkBytes;    // P (64 x 64 bf16) over the RoPE chunk
constexpr uint32_t kOffBar = kOffKv + kStages * kKvBytes;
// barriers: q_full, q_ready, q_free, kv_full[S], kv_empty[S], p_full[S],
// s_full[2], s_free[2], drain
constexpr uint32_t kNumBars = 3 + 3 * kStages + 4 + 1;
constexpr uint32_t kQCol = 128;                 // TMEM column of the query tile
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmem = kOffMisc + 32 + 1024;

constexpr int kSmWarps = 4;                 // warps 0..3
constexpr int kMmaWarp = 4;                 // warp 4
constexpr int kProdWarp0 = 5;               // warps 5..12
constexpr int kProdWarps = 8;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kGroupThreads = kProdThreads / 2;   // one producer group
constexpr int kThreads = 32 * (kSmWarps + 1 + kProdWarps);   // 416
constexpr uint32_t kBarProducer = 2;        // producer groups use named barriers 2 and 3
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
  float scale_log2;  // sm_scale * log2(e)
  __nv_bfloat16* out;
  float* lse;
  DevErr err;
};

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

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  const uint32_t q_full = bar0;          // query tile copied into the stage
  const uint32_t q_ready = bar0 + 8u;    // query tile in TMEM
  const uint32_t q_free = bar0 + 16u;    // the stage that held it is free
  auto kv_full = [&](int i) { return bar0 + 8u * (3 + i); };
  auto kv_empty = [&](int i) { return bar0 + 8u * (3 + kStages + i); };
  auto p_full = [&](int i) { return bar0 + 8u * (3 + 2 * kStages + i); };
  auto s_full = [&](int i) { return bar0 + 8u * (3 + 3 * kStages + i); };
  auto s_free = [&](int i) { return bar0 + 8u * (5 + 3 * kStages + i); };
  const uint32_t drain_bar = bar0 + 8u * (7 + 3 * kStages);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* prod_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- which query / heads
  const int64_t q_row = blockIdx.x / P.head_groups;
  const int hg = static_cast<int>(blockIdx.x % P.head_groups);
  int lo = 0, hi = P.B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(P.cu_q + mid) <= q_row) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int cq0 = __ldg(P.cu_q + b);
  const int ck0 = __ldg(P.cu_k + b);
  const int len_q = __ldg(P.cu_q + b + 1) - cq0;
  const int len_k = __ldg(P.cu_k + b + 1) - ck0;
  const int p = len_k - len_q + static_cast<int>(q_row - cq0);   // absolute position
  const int n_sel = min(P.k, p + 1);
  const int nb = (n_sel + kBlockN - 1) / kBlockN;
  const int heads_here = min(kHeads, P.H - hg * kHeads);
  const int32_t* idx_row = P.idx + q_row * P.k;

  if (threadIdx.x == 0) {
    mbar_init(q_full, kGroupThreads);
    mbar_init(q_ready, kSmWarps);
    mbar_init(q_free, kSmWarps);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(kv_full(i), kGroupThreads);
      mbar_init(kv_empty(i), 1);
      mbar_init(p_full(i), kSmWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), kSmWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *prod_abort = 0;
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

  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ query tile + latent gather
    const int tp = threadIdx.x - 32 * kProdWarp0;        // 0..255
    const int grp = tp / kGroupThreads;                  // takes blocks j with j % 2 == grp
    const int tg = tp % kGroupThreads;                   // 0..127
    const int rsub = tg >> 3;                            // rows rsub + 16*pass, pass 0..3
    const int l8 = tg & 7;                               // 16-byte piece within 128 B
    const uint32_t bar_id = kBarProducer + grp;
    const __nv_bfloat16* kv_seq = P.kv + static_cast<int64_t>(ck0) * kDqk;
    if (grp == 0) {
      // The query rows of this head group, in the layout of a latent tile;
      // rows past the last head are zero.
      const uint32_t stage = sbase + kOffKv + kQStage * kKvBytes;
      const __nv_bfloat16* q_grp = P.q + (q_row * P.H + hg * kHeads) * kDqk;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int r = rsub + 16 * pass;
        const uint32_t dst = stage + r * 128 + ((l8 ^ (r & 7)) << 4);
        if (r < heads_here) {
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
      cp_async_wait_all();
      mbar_arrive(q_full);
    }
    auto load_idx = [&](int j, int r) -> int {
      const int e = j * kBlockN + r;
      int s = -1;
      if (e < n_sel) s = __ldg(idx_row + e);
      return (s >= 0 && s <= p) ? s : 0;                 // invalid entries read row 0 (masked)
    };
    int cur[4], nxt[4];
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) cur[pass] = grp < nb ? load_idx(grp, rsub + 16 * pass) : 0;
    for (int j = grp; j < nb; j += 2) {
      const int st = j % kStages;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass)                           // prefetch this group's next block
        nxt[pass] = j + 2 < nb ? load_idx(j + 2, rsub + 16 * pass) : 0;
      // The first use of the query stage waits for the query to leave it.
      const uint32_t free_bar = j == kQStage ? q_free : kv_empty(st);
      const uint32_t free_par = j == kQStage ? 0u : static_cast<uint32_t>(((j / kStages) & 1) ^ 1);
      if (tg == 0 && !mbar_wait(free_bar, free_par, P.err)) *prod_abort = 1;
      named_bar_sync(bar_id, kGroupThreads);
      if (*prod_abort) break;
      const uint32_t stage = sbase + kOffKv + st * kKvBytes;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int r = rsub + 16 * pass;
        const __nv_bfloat16* src = kv_seq + static_cast<int64_t>(cur[pass]) * kDqk + l8 * 8;
        const uint32_t dst = stage + r * 128 + ((l8 ^ (r & 7)) << 4);
#pragma unroll
        for (int c = 0; c < kChunks; ++c) cp_async16(dst + c * kChunkBytes, src + c * 64);
      }
      cp_async_commit();
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(kv_full(st));
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) cur[pass] = nxt[pass];
    }
    if (*prod_abort && tp == 0) *abort_flag = 1;
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop in lockstep and one elected lane issues
    // each MMA; every value the MMAs use is warp-uniform.  S of block j+1
    // goes to the tensor pipe before P V of block j, so the softmax of block
    // j overlaps P V of block j-1 and S of block j+1.
    // Descriptors are built once; every MMA only adds a compile-time offset
    // (in 16-byte units) to the start-address field.
    const uint64_t dS0 = smem_desc(sbase + kOffKv, 16, 1024, kSwizzle128B);          // K, K-major
    const uint64_t dP0 = smem_desc(sbase + kOffKv + kOffPInStage, 16, 1024, kSwizzle128B);
    const uint64_t dV0 = smem_desc(sbase + kOffKv, kChunkBytes, 1024, kSwizzle128B);  // V, MN-major
    constexpr uint64_t kStageStep = kKvBytes >> 4;
    bool ok = warp_wait(q_ready, 0, P.err);
    auto issue_s = [&](int js) -> bool {
      const int st = js % kStages;
      const int sb = js & 1;                   // S buffer
      if (!warp_wait(kv_full(st), static_cast<uint32_t>((js / kStages) & 1), P.err)) return false;
      if (!warp_wait(s_free(sb), static_cast<uint32_t>(((js >> 1) & 1) ^ 1), P.err)) return false;
      tc_fence_after();
      const uint64_t dS = dS0 + st * kStageStep;
      const uint32_t d = tmem_s + 64u * sb;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_f16_ts_warp(d, tmem_q + 32u * c + 8u * kk, dS + ((c * kChunkBytes + kk * 32) >> 4),
                          kIdescS, (c | kk) != 0 ? 1u : 0u);
        }
      }
      mma_commit_warp(s_full(sb));
      return true;
    };
    auto issue_pv = [&](int jp) -> bool {
      const int st = jp % kStages;
      if (!warp_wait(p_full(st), static_cast<uint32_t>((jp / kStages) & 1), P.err)) return false;
      tc_fence_after();
      const uint64_t dP = dP0 + st * kStageStep;
      const uint64_t dV = dV0 + st * kStageStep;
      const uint32_t first = jp > 0 ? 1u : 0u;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_f16_warp(tmem_o + 256u * h, dP + (kk * 32 >> 4),
                       dV + ((4 * h * kChunkBytes + kk * 2048) >> 4), kIdescPV,
                       kk > 0 ? 1u : first);
        }
      }
      mma_commit_warp(kv_empty(st));
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; ok && j < nb; ++j) {
      if (j + 1 < nb) ok = issue_s(j + 1);
      if (ok) ok = issue_pv(j);
    }
    // every MMA issued by this warp completes before TMEM is released
    mma_commit_warp(drain_bar);
    if (lane == 0) {
      mbar_wait_drain(drain_bar, 0);
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int w = warp;                       // sub-partition
    const int qd = lane & 3;                  // column pair within each group of 8
    const int ra = 16 * w + (lane >> 2);      // this lane's two heads (rows) in the group
    const int rb = ra + 8;
    const uint32_t lane_base = static_cast<uint32_t>(w * 32) << 16;
    float m_a = -INFINITY, m_b = -INFINITY;   // running maxima, log2 units
    float l_a = 0.f, l_b = 0.f;               // partial denominators (fp32 probabilities), lse
    float lr_a = 0.f, lr_b = 0.f;             // partial denominators of the bf16 P, for O
    bool ok = warp_wait(q_full, 0, P.err);
    if (ok) {
      // Query tile: shared memory -> TMEM columns kQCol.., lanes 16..31.
      // Column 32c+8i+2qd+e holds elements 64c+16i+4qd+2e, +1 of a row.
      const uint8_t* qs = smem + kOffKv + kQStage * kKvBytes;
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
        mbar_arrive(q_ready);
        mbar_arrive(q_free);
      }
    }
    // Validity of block entries: lane l checks entries 2l and 2l+1.
    auto entry_ok = [&](int e) -> bool {
      if (e >= n_sel) return false;
      const int s = __ldg(idx_row + e);
      return s >= 0 && s <= p;
    };
    bool nx0 = entry_ok(2 * lane), nx1 = entry_ok(2 * lane + 1);
    for (int j = 0; ok && j < nb; ++j) {
      const int sb = j & 1;                  // S buffer
      const int st = j % kStages;            // latent stage (P goes over its RoPE chunk)
      const uint32_t vmask_lo = __ballot_sync(0xffffffffu, nx0);
      const uint32_t vmask_hi = __ballot_sync(0xffffffffu, nx1);
      if (j + 1 < nb) {
        nx0 = entry_ok((j + 1) * kBlockN + 2 * lane);
        nx1 = entry_ok((j + 1) * kBlockN + 2 * lane + 1);
      }
      if (!warp_wait(s_full(sb), static_cast<uint32_t>((j >> 1) & 1), P.err)) {
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

      // key of register 4i+e (row a) and 4i+2+e (row b): 8i + 2qd + e
      float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool valid = (((e ? vmask_hi : vmask_lo) >> (4 * i + qd)) & 1u) != 0;
          const float xa = valid ? __uint_as_float(v[4 * i + e]) * P.scale_log2 : -INFINITY;
          const float xb = valid ? __uint_as_float(v[4 * i + 2 + e]) * P.scale_log2 : -INFINITY;
          v[4 * i + e] = __float_as_uint(xa);
          v[4 * i + 2 + e] = __float_as_uint(xb);
          mxa = fmaxf(mxa, xa);
          mxb = fmaxf(mxb, xb);
        }
      }
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
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

      // P (bf16) over the stage's RoPE chunk: row r, keys 8i..8i+7 are the
      // 16-byte piece i, stored at piece i ^ (r & 7).
      uint8_t* pst = smem + kOffKv + st * kKvBytes + kOffPInStage;
      float sa = 0.f, sb_ = 0.f, sra = 0.f, srb = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float xa0 = __uint_as_float(v[4 * i + 0]), xa1 = __uint_as_float(v[4 * i + 1]);
        const float xb0 = __uint_as_float(v[4 * i + 2]), xb1 = __uint_as_float(v[4 * i + 3]);
        const float pa0 = xa0 == -INFINITY ? 0.f : fast_exp2(xa0 - m_a);
        const float pa1 = xa1 == -INFINITY ? 0.f : fast_exp2(xa1 - m_a);
        const float pb0 = xb0 == -INFINITY ? 0.f : fast_exp2(xb0 - m_b);
        const float pb1 = xb1 == -INFINITY ? 0.f : fast_exp2(xb1 - m_b);
        sa += pa0 + pa1;
        sb_ += pb0 + pb1;
        const uint32_t ka = pack_bf16x2(pa0, pa1), kb = pack_bf16x2(pb0, pb1);
        // the weights O receives are the rounded ones: normalise by their sum
        sra += __uint_as_float(ka << 16) + __uint_as_float(ka & 0xFFFF0000u);
        srb += __uint_as_float(kb << 16) + __uint_as_float(kb & 0xFFFF0000u);
        *reinterpret_cast<uint32_t*>(pst + ra * 128 + ((i ^ (ra & 7)) << 4) + 4 * qd) = ka;
        *reinterpret_cast<uint32_t*>(pst + rb * 128 + ((i ^ (rb & 7)) << 4) + 4 * qd) = kb;
      }
      l_a = l_a * al_a + sa;
      l_b = l_b * al_b + sb_;
      lr_a = lr_a * al_a + sra;
      lr_b = lr_b * al_b + srb;

      // When a maximum moved, this warp's O rows are rescaled before P V of
      // this block may run: after P V of the previous block has completed
      // (its stage is released).
      if (rescale) {
        const int pj = j - 1;
        if (!warp_wait(kv_empty(pj % kStages), static_cast<uint32_t>((pj / kStages) & 1), P.err)) {
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
    }

    if (ok) {
      // every P V product has completed once the last block's stage is released
      const int pj = nb - 1;
      ok = warp_wait(kv_empty(pj % kStages), static_cast<uint32_t>((pj / kStages) & 1), P.err);
    }
    if (ok) {
      tc_fence_after();
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      lr_a += __shfl_xor_sync(0xffffffffu, lr_a, 1);
      lr_a += __shfl_xor_sync(0xffffffffu, lr_a, 2);
      lr_b += __shfl_xor_sync(0xffffffffu, lr_b, 1);
      lr_b += __shfl_xor_sync(0xffffffffu, lr_b, 2);
      const float inv_a = lr_a > 0.f ? 1.f / lr_a : 0.f;
      const float inv_b = lr_b > 0.f ? 1.f / lr_b : 0.f;
      const int64_t head0 = q_row * P.H + hg * kHeads;
      const bool have_a = ra < heads_here, have_b = rb < heads_here;
      if (P.lse && qd == 0) {
        if (have_a) P.lse[head0 + ra] = l_a > 0.f ? (m_a + log2f(l_a)) * 0.69314718055994531f : -INFINITY;
        if (have_b) P.lse[head0 + rb] = l_b > 0.f ? (m_b + log2f(l_b)) * 0.69314718055994531f : -INFINITY;
      }
      __nv_bfloat16* oa = P.out + (head0 + ra) * kDv;
      __nv_bfloat16* ob = P.out + (head0 + rb) * kDv;
#pragma unroll 1
      for (int k8 = 0; k8 < kDv / 64; ++k8) {
        uint32_t o[32];
        tmem_ld_16x256b_x8(tmem_o + lane_base + 64u * k8, o);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          // groups 4u..4u+3 (dims 64k8 + 32u .. +31); after the transpose lane
          // qd holds the 8 dims of group 4u+qd as one 16-byte piece
          uint32_t pa[4], pb[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int i = 4 * u + g;
            pa[g] = pack_bf16x2(__uint_as_float(o[4 * i + 0]) * inv_a,
                                __uint_as_float(o[4 * i + 1]) * inv_a);
            pb[g] = pack_bf16x2(__uint_as_float(o[4 * i + 2]) * inv_b,
                                __uint_as_float(o[4 * i + 3]) * inv_b);
          }
          transpose4(pa, qd);
          transpose4(pb, qd);
          const int dim = 64 * k8 + 8 * (4 * u + qd);
          if (have_a) *reinterpret_cast<uint4*>(oa + dim) = make_uint4(pa[0], pa[1], pa[2], pa[3]);
          if (have_b) *reinterpret_cast<uint4*>(ob + dim) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
        }
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
  P.scale_log2 = a.sm_scale * 1.4426950408889634f;
  P.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  P.lse = a.lse;
  P.err = err;
  const int64_t grid = a.total_q * P.head_groups;
  if (grid == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  sparse_mla_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, s>>>(P);
  return cudaGetLastError();
}

}  // namespace dsa
