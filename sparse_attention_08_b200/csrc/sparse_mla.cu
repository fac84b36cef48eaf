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
//    warp instruction moves four full 128-byte lines.  The gathered
//    tile is shared by all 64 heads of the CTA (group-shared selection).
//  * warp 4 (MMA): issues, whichever is ready first, S = Q K^T (36
//    tcgen05.mma, M=64 heads, N=64 keys, K=16, with Q read from TMEM) into
//    TMEM, or O += P V (8 tcgen05.mma, M=64, N=256, K=16) with P from shared
//    memory and V read MN-major from the first 512 columns of the same tile.
//    P of a block is written over that block's RoPE columns (512..575),
//    which S no longer needs, so P lives and dies with its latent stage.
//  * warps 0..3 (softmax): first write the 64 x 576 query tile into TMEM;
//    then read S from TMEM, online softmax in fp32 (exp2,
//    lazily rescaled maximum), write P (bf16) to shared memory, rescale O in
//    TMEM when the maximum moves, and finally normalise O and store bf16 out
//    and the lse.
//
// TMEM (512 columns x 128 lanes): an M=64 accumulator fills lanes 0-15 of
// each 32-lane sub-partition; a second one at lane offset 16 fills lanes
// 16-31.  O (64 heads x 512 fp32) takes columns 0..511 at lane offset 0; the
// two S buffers (64 x 64) take columns 0..63 and 64..127 at lane offset 16,
// and the query tile (64 x 576 bf16, two elements per column) takes columns
// 128..415 at lane offset 16, the same lanes as the S rows it produces.
// In softmax warp w (sub-partition w), threads 16..31 own S rows and threads
// 0..15 own the O rows of the same heads.
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
constexpr uint32_t kKvBytes = kChunks * kChunkBytes;  // 73728
constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffPInStage = 8 * kChunkBytes;    // P (64 x 64 bf16) over the RoPE chunk
constexpr uint32_t kOffBar = kOffKv + kStages * kKvBytes;
// barriers: q_ready, kv_full[S], kv_empty[S], p_full[S], s_full[2], s_free[2], drain
constexpr uint32_t kNumBars = 1 + 3 * kStages + 4 + 1;
constexpr uint32_t kQCol = 128;                 // TMEM column of the query tile
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmem = kOffMisc + 32 + 1024;

constexpr int kSmWarps = 4;                 // warps 0..3
constexpr int kMmaWarp = 4;                 // warp 4
constexpr int kProdWarp0 = 5;               // warps 5..12
constexpr int kProdWarps = 8;
constexpr int kSmThreads = 32 * kSmWarps;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kGroupThreads = kProdThreads / 2;   // one producer group
constexpr int kThreads = 32 * (kSmWarps + 1 + kProdWarps);   // 416
constexpr uint32_t kBarSoftmax = 1, kBarProducer = 2;   // producer groups use 2 and 3
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

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  const uint32_t q_ready = bar0;
  auto kv_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto kv_empty = [&](int i) { return bar0 + 8u * (1 + kStages + i); };
  auto p_full = [&](int i) { return bar0 + 8u * (1 + 2 * kStages + i); };
  auto s_full = [&](int i) { return bar0 + 8u * (1 + 3 * kStages + i); };
  auto s_free = [&](int i) { return bar0 + 8u * (3 + 3 * kStages + i); };
  const uint32_t drain_bar = bar0 + 8u * (5 + 3 * kStages);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* prod_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  volatile int* warp_moved = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);  // [4]

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
    mbar_init(q_ready, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(kv_full(i), kGroupThreads);
      mbar_init(kv_empty(i), 1);
      mbar_init(p_full(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), 1);
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
    // ------------------------------------------------------------ latent gather
    const int tp = threadIdx.x - 32 * kProdWarp0;        // 0..255
    const int grp = tp / kGroupThreads;                  // takes blocks j with j % 2 == grp
    const int tg = tp % kGroupThreads;                   // 0..127
    const int rsub = tg >> 3;                            // rows rsub + 16*pass, pass 0..3
    const int l8 = tg & 7;                               // 16-byte piece within 128 B
    const uint32_t bar_id = kBarProducer + grp;
    const __nv_bfloat16* kv_seq = P.kv + static_cast<int64_t>(ck0) * kDqk;
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
      if (tg == 0 &&
          !mbar_wait(kv_empty(st), static_cast<uint32_t>(((j / kStages) & 1) ^ 1), P.err))
        *prod_abort = 1;
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
    if (lane == 0) {
      bool ok = mbar_wait(q_ready, 0, P.err);
      // Descriptors are built once; every MMA only adds a compile-time
      // offset (in 16-byte units) to the start-address field.
      const uint64_t dS0 = smem_desc(sbase + kOffKv, 16, 1024, kSwizzle128B);          // K, K-major
      const uint64_t dP0 = smem_desc(sbase + kOffKv + kOffPInStage, 16, 1024, kSwizzle128B);
      const uint64_t dV0 = smem_desc(sbase + kOffKv, kChunkBytes, 1024, kSwizzle128B);  // V, MN-major
      constexpr uint64_t kStageStep = kKvBytes >> 4;
      int js = 0, jp = 0;          // next block for S, next block for PV
      uint64_t t_idle = 0;
      uint32_t spins = 0;
      while (ok && jp < nb) {
        bool progress = false;
        if (jp < js &&
            mbar_try_wait(p_full(jp % kStages), static_cast<uint32_t>((jp / kStages) & 1))) {
          const int st = jp % kStages;
          tc_fence_after();
          const uint64_t dP = dP0 + st * kStageStep;
          const uint64_t dV = dV0 + st * kStageStep;
          const uint32_t first = jp > 0 ? 1u : 0u;
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
          ++jp;
          progress = true;
        }
        if (js < nb) {
          const int st = js % kStages;
          const int sb = js & 1;                   // S buffer
          if (mbar_try_wait(kv_full(st), static_cast<uint32_t>((js / kStages) & 1)) &&
              mbar_try_wait(s_free(sb), static_cast<uint32_t>(((js >> 1) & 1) ^ 1))) {
            tc_fence_after();
            const uint64_t dS = dS0 + st * kStageStep;
            const uint32_t d = tmem_s + 64u * sb;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                mma_f16_ts(d, tmem_q + 32u * c + 8u * kk, dS + ((c * kChunkBytes + kk * 32) >> 4),
                           kIdescS, (c | kk) != 0 ? 1u : 0u);
              }
            }
            mma_commit(s_full(sb));
            ++js;
            progress = true;
          }
        }
        if (progress) {
          spins = 0;
          t_idle = 0;
        } else if ((++spins & 255u) == 0) {
          if (launch_failed(P.err)) {
            ok = false;
          } else {
            const uint64_t now = globaltimer_ns();
            if (t_idle == 0) {
              t_idle = now;
            } else if (now - t_idle > kWaitLimitNs) {
              raise_error(P.err, kErrTimeout);
              ok = false;
            }
          }
        }
      }
      // every MMA issued by this thread completes before TMEM is released
      mma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int et = threadIdx.x;              // 0..127
    const int sp = warp;                     // sub-partition
    const bool is_s = lane >= 16;
    const int r_s = sp * 16 + (lane - 16);   // S row owned by lanes 16..31
    const int r_o = sp * 16 + lane;          // O row owned by lanes 0..15
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    float m = -INFINITY;   // running maximum, log2 units
    float l = 0.f;         // running denominator (fp32 probabilities), for the lse
    float lr = 0.f;        // running denominator of the bf16 P the MMA consumes, for O
    bool ok = true;
    {
      // The query tile goes into TMEM: S-row threads (lanes 16..31) store
      // their head's 576 bf16 as 288 columns of packed pairs.  A 32x32b store
      // covers the whole sub-partition, so lanes 0..15 also store (zeros)
      // into the O columns, which the first P V product overwrites.
      const int h = hg * kHeads + r_s;
      const bool have = is_s && r_s < heads_here;
      const uint4* qrow = reinterpret_cast<const uint4*>(P.q + (q_row * P.H + h) * kDqk);
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t qv[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 u = have ? __ldg(qrow + c * 8 + e) : make_uint4(0u, 0u, 0u, 0u);
          qv[4 * e + 0] = u.x;
          qv[4 * e + 1] = u.y;
          qv[4 * e + 2] = u.z;
          qv[4 * e + 3] = u.w;
        }
        tmem_st_32x32b_x32(tmem + lane_base + kQCol + 32u * c, qv);
      }
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(kBarSoftmax, kSmThreads);
      if (et == 0) mbar_arrive(q_ready);
    }
    for (int j = 0; j < nb; ++j) {
      const int sb = j & 1;                  // S buffer
      const int st = j % kStages;            // latent stage (P goes over its RoPE chunk)
      // validity of the 64 entries of this block (each lane checks two)
      uint32_t vmask_lo, vmask_hi;
      {
        const int e0 = j * kBlockN + 2 * lane;
        const int s0 = e0 < n_sel ? __ldg(idx_row + e0) : -1;
        const int s1 = e0 + 1 < n_sel ? __ldg(idx_row + e0 + 1) : -1;
        vmask_lo = __ballot_sync(0xffffffffu, s0 >= 0 && s0 <= p);
        vmask_hi = __ballot_sync(0xffffffffu, s1 >= 0 && s1 <= p);
      }
      if (et == 0 && !mbar_wait(s_full(sb), static_cast<uint32_t>((j >> 1) & 1), P.err))
        *abort_flag = 1;
      named_bar_sync(kBarSoftmax, kSmThreads);
      if (*abort_flag) {
        ok = false;
        break;
      }
      tc_fence_after();
      // A 32x32b load covers the warp's whole 32-lane sub-partition, so it
      // starts at the sub-partition base: lanes 16..31 deliver the S rows.
      uint32_t v[64];
      tmem_ld_32x32b_x64(tmem + lane_base + 64u * sb, v);
      tmem_wait_ld();

      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const uint32_t bits = (c & 1) ? vmask_hi : vmask_lo;
        const bool valid = (bits >> (c >> 1)) & 1u;
        const float x = valid ? __uint_as_float(v[c]) * P.scale_log2 : -INFINITY;
        v[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      float alpha = 1.f;
      bool moved = false;
      if (is_s && mx > m + kRescaleThreshold) {
        alpha = fast_exp2(m - mx);   // 0 when m = -inf
        m = mx;
        moved = true;
      }
      const bool warp_moved_any = __any_sync(0xffffffffu, moved);
      if (lane == 0) warp_moved[sp] = warp_moved_any ? 1 : 0;
      tc_fence_before();
      named_bar_sync(kBarSoftmax, kSmThreads);
      if (et == 0) mbar_arrive(s_free(sb));
      const bool group_moved = (warp_moved[0] | warp_moved[1] | warp_moved[2] | warp_moved[3]) != 0;

      // The row's 64 probabilities are split between the S-row thread (keys
      // 0..31) and its partner 16 lanes down, which owns the O row of the
      // same head (keys 32..63): the partner receives its half by shuffle.
      {
        const float m_row = __shfl_xor_sync(0xffffffffu, m, 16);
        const float m_use = is_s ? m : m_row;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t y = __shfl_xor_sync(0xffffffffu, v[32 + i], 16);
          if (!is_s) v[i] = y;
        }
        const int r = sp * 16 + (lane & 15);
        const int c8_base = is_s ? 0 : 4;
        float sum = 0.f, sum_r = 0.f;
        uint8_t* prow = smem + kOffKv + st * kKvBytes + kOffPInStage + r * 128;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = c8 * 8 + 2 * e;
            const float x0 = __uint_as_float(v[c]), x1 = __uint_as_float(v[c + 1]);
            const float p0 = x0 == -INFINITY ? 0.f : fast_exp2(x0 - m_use);
            const float p1 = x1 == -INFINITY ? 0.f : fast_exp2(x1 - m_use);
            sum += p0 + p1;
            packed[e] = pack_bf16x2(p0, p1);
            // the weights O receives are the rounded ones: normalise by their sum
            sum_r += __uint_as_float(packed[e] << 16) + __uint_as_float(packed[e] & 0xFFFF0000u);
          }
          *reinterpret_cast<uint4*>(prow + (((c8_base + c8) ^ (r & 7)) << 4)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 16);
        sum_r += __shfl_xor_sync(0xffffffffu, sum_r, 16);
        if (is_s) {
          l = l * alpha + sum;
          lr = lr * alpha + sum_r;
        }
      }
      // When the maximum moved, O is rescaled before P V of this block may
      // run: wait until P V of the previous block has completed (its stage
      // is released), rescale, and only then publish P.
      if (j >= 1 && group_moved) {
        const int pj = j - 1;
        if (et == 0 && !mbar_wait(kv_empty(pj % kStages),
                                  static_cast<uint32_t>((pj / kStages) & 1), P.err))
          *abort_flag = 1;
        named_bar_sync(kBarSoftmax, kSmThreads);
        if (*abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (warp_moved_any) {
          const float a_lo = __shfl_sync(0xffffffffu, alpha, 16 + (lane >> 2));
          const float a_hi = __shfl_sync(0xffffffffu, alpha, 24 + (lane >> 2));
#pragma unroll 1
          for (int q = 0; q < kDv / 64; ++q) {
            uint32_t o[32];
            const uint32_t ta = tmem_o + lane_base + 64u * q;
            tmem_ld_16x256b_x8(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
              o[4 * rr + 0] = __float_as_uint(__uint_as_float(o[4 * rr + 0]) * a_lo);
              o[4 * rr + 1] = __float_as_uint(__uint_as_float(o[4 * rr + 1]) * a_lo);
              o[4 * rr + 2] = __float_as_uint(__uint_as_float(o[4 * rr + 2]) * a_hi);
              o[4 * rr + 3] = __float_as_uint(__uint_as_float(o[4 * rr + 3]) * a_hi);
            }
            tmem_st_16x256b_x8(ta, o);
          }
          tmem_wait_st();
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarSoftmax, kSmThreads);
      if (et == 0) mbar_arrive(p_full(st));
    }

    if (ok) {
      // every P V product has completed once the last block's stage is released
      const int pj = nb - 1;
      if (et == 0 && !mbar_wait(kv_empty(pj % kStages), static_cast<uint32_t>((pj / kStages) & 1),
                                P.err))
        *abort_flag = 1;
      named_bar_sync(kBarSoftmax, kSmThreads);
      ok = !*abort_flag;
    }
    if (ok) {
      tc_fence_after();
      const float inv_l_s = lr > 0.f ? 1.f / lr : 0.f;
      const float inv_l = __shfl_sync(0xffffffffu, inv_l_s, (lane & 15) + 16);
      if (is_s && r_s < heads_here && P.lse) {
        const int h = hg * kHeads + r_s;
        P.lse[q_row * P.H + h] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
      const int h = hg * kHeads + r_o;
      __nv_bfloat16* orow = P.out + (q_row * P.H + h) * kDv;
      const bool store = !is_s && r_o < heads_here;
#pragma unroll 1
      for (int cc = 0; cc < kDv / 32; ++cc) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tmem_o + lane_base + 32u * cc, o);
        tmem_wait_ld();
        if (store) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                __uint_as_float(o[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    }
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
