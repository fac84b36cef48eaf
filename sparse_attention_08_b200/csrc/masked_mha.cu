// masked_mha.cu -- the masked MHA mode on sm_100a.
//
// What it computes ("DeepSeek-V3.2" atlas entry, "Design overview" and
// "Inference efficiency": for short prompts the prefill runs a masked form of
// MHA as a stand-in for DSA; the pages name the mode without detail, so it is
// read as dense attention in the MHA form of MLA -- every
// head with its own 192-d key (128 + 64 RoPE) and 128-d value -- restricted
// by a mask to each query's selected set S_t):
//
//   out[t,h,:] = sum_{s in S_t} softmax_s(scale * q[t,h,:] . k[s,h,:]) v[s,h,:]
//   lse[t,h]   = log sum_{s in S_t} exp(scale * q[t,h,:] . k[s,h,:])
//
// S_t is the set of entries 0 <= s <= p among the first min(topk, p+1) of
// idx[t, :]; a repeated entry counts once.
//
// How, in two launches:
//  * mask_kernel: one CTA per query row turns the row's index list into a
//    bitmask over its keys (bit s of word s/32), built with shared-memory
//    atomics and written out whole.
//  * masked_mha_kernel: one CTA per (tile of 128 queries of one sequence,
//    head), flash-attention style over the causal key tiles of 128:
//      warp 0  TMA: the query tile once (three 64-column boxes of a 3-D map
//              [token, head, dim]), then key tiles and value tiles into two
//              two-stage rings of their own (a key stage frees when its S is
//              done, a value stage after its P V);
//      warp 1  TMEM owner and MMA issuer: S = Q K^T (12 tcgen05.mma, M = N =
//              128, K = 16, both operands K-major in shared memory) into one
//              of two S buffers, and O += P V (8 tcgen05.mma, P read from
//              TMEM, V MN-major from shared memory);
//      warps 2..9  two warpgroups, one query row per thread (TMEM lane), each
//              warpgroup half of the tile's keys and half of O's columns:
//              masking (causal and the selection bits), online softmax in
//              fp32 with a lazily rescaled maximum agreed between the halves,
//              P written to TMEM as bf16, and at the end O normalised and
//              stored as bf16 together with the lse.
//    TMEM: S buffers at columns 0 and 128, P (128 x 128 bf16) at 256, O
//    (128 x 128 fp32) at 320.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kBM = 128;                 // queries per tile (MMA M)
constexpr int kBN = 128;                 // keys per tile (MMA N of S, K of P V)
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr uint32_t kBox = 128 * 128;     // one 64-column box of 128 rows: 16 KB
constexpr uint32_t kOffQ = 0;                          // 3 boxes
constexpr int kStages = 2;
constexpr uint32_t kOffK = 3 * kBox;                   // key stages: 3 boxes each
constexpr uint32_t kKBytes = 3 * kBox;
constexpr uint32_t kOffV = kOffK + kStages * kKBytes;  // value stages: 2 boxes each
constexpr uint32_t kVBytes = 2 * kBox;
constexpr uint32_t kOffBar = kOffV + kStages * kVBytes;
// barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], s_free[2],
// p_full, pv_done, drain
constexpr uint32_t kNumBars = 1 + 4 * kStages + 4 + 3;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kOffXchg = kOffMisc + 16;           // row maxima and sums of the two halves
constexpr uint32_t kSmem = kOffXchg + 1024 * 4 + 1024;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;            // + 128 * buffer
constexpr uint32_t kColP = 256;
constexpr uint32_t kColO = 320;
constexpr uint32_t kIdescS = instr_desc(kFmtBF16, kFmtBF16, 0, 0, kBM, kBN);
constexpr uint32_t kIdescPV = instr_desc(kFmtBF16, kFmtBF16, 0, 1, kBM, kDv);
constexpr float kRescaleThreshold = 8.0f;   // log2 units

static_assert(kSmem <= 232448, "shared memory budget");
static_assert(kDqk == 3 * 64 && kDv == 2 * 64, "query/key and value tiles are 64-column boxes");

struct Params {
  const int32_t* cu_q;
  const int32_t* cu_k;
  const uint32_t* mask;     // [total_q, words] selection bits
  int64_t words;            // mask words per row
  int H;
  int q_tiles;              // query tiles per sequence slot (max_len_q / 128, rounded up)
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  DevErr err;
};

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, int32_t x, int32_t y,
                                            int32_t z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------- mask build
// Row t of the mask: bit s set when s is a valid selected entry of row t.
// Words past the row's causal limit stay zero.
__global__ void __launch_bounds__(256) mask_kernel(const int32_t* __restrict__ idx, int topk,
                                                   const int32_t* __restrict__ cu_q,
                                                   const int32_t* __restrict__ cu_k, int B,
                                                   uint32_t* __restrict__ mask, int64_t words) {
  extern __shared__ uint32_t bits[];
  const int64_t t = blockIdx.x;
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid;
  }
  const int len_q = __ldg(cu_q + lo + 1) - __ldg(cu_q + lo);
  const int len_k = __ldg(cu_k + lo + 1) - __ldg(cu_k + lo);
  const int p = len_k - len_q + static_cast<int>(t - __ldg(cu_q + lo));
  for (int64_t i = threadIdx.x; i < words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  const int n = min(topk, p + 1);
  const int32_t* row = idx + t * topk;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int s = __ldg(row + e);
    if (s >= 0 && s <= p) atomicOr(bits + (s >> 5), 1u << (s & 31));
  }
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(mask + t * words);
  const uint4* src = reinterpret_cast<const uint4*>(bits);
  for (int64_t i = threadIdx.x; i < words / 4; i += blockDim.x) dst[i] = src[i];
}

// ------------------------------------------------------------------ attention
__global__ void __launch_bounds__(kThreads, 1)
    masked_mha_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  const uint32_t q_full = bar0;
  auto k_full = [&](uint32_t i) { return bar0 + 8u * (1 + i); };
  auto k_empty = [&](uint32_t i) { return bar0 + 8u * (1 + kStages + i); };
  auto v_full = [&](uint32_t i) { return bar0 + 8u * (1 + 2 * kStages + i); };
  auto v_empty = [&](uint32_t i) { return bar0 + 8u * (1 + 3 * kStages + i); };
  auto s_full = [&](uint32_t i) { return bar0 + 8u * (1 + 4 * kStages + i); };
  auto s_free = [&](uint32_t i) { return bar0 + 8u * (3 + 4 * kStages + i); };
  const uint32_t p_full = bar0 + 8u * (5 + 4 * kStages);
  const uint32_t pv_done = bar0 + 8u * (6 + 4 * kStages);
  const uint32_t drain = bar0 + 8u * (7 + 4 * kStages);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // the tile: sequence b, query tile qt (heaviest first), head h
  const int b = blockIdx.x / P.q_tiles;
  const int qt = P.q_tiles - 1 - static_cast<int>(blockIdx.x % P.q_tiles);
  const int h = blockIdx.y;
  const int cq0 = __ldg(P.cu_q + b);
  const int ck0 = __ldg(P.cu_k + b);
  const int len_q = __ldg(P.cu_q + b + 1) - cq0;
  const int len_k = __ldg(P.cu_k + b + 1) - ck0;
  const int q0 = qt * kBM;
  if (q0 >= len_q) return;                                  // uniform over the CTA
  const int rows = min(kBM, len_q - q0);
  const int off = len_k - len_q;                            // position of local query i: off + i
  const int n_tiles = (off + q0 + rows - 1) / kBN + 1;      // causal key tiles

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), 8);
    }
    mbar_init(p_full, 8);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    // Lane 0 loads the query and the key tiles, lane 1 the value tiles: a key
    // stage is free once its S product is done, a value stage only after its
    // P V product, so the two rings run apart.
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      mbar_arrive_expect_tx(q_full, 3 * kBox);
      for (int c = 0; c < 3; ++c)
        tma_load_3d(sbase + kOffQ + c * kBox, &tq, 64 * c, h, cq0 + q0, q_full);
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t st = j & 1;
        if (!mbar_wait(k_empty(st), ((j >> 1) & 1) ^ 1, P.err)) break;
        const uint32_t dst = sbase + kOffK + st * kKBytes;
        mbar_arrive_expect_tx(k_full(st), kKBytes);
        for (int c = 0; c < 3; ++c)
          tma_load_3d(dst + c * kBox, &tk, 64 * c, h, ck0 + j * kBN, k_full(st));
      }
    } else if (lane == 1) {
      tma_prefetch_desc(&tv);
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t st = j & 1;
        if (!mbar_wait(v_empty(st), ((j >> 1) & 1) ^ 1, P.err)) break;
        const uint32_t dst = sbase + kOffV + st * kVBytes;
        mbar_arrive_expect_tx(v_full(st), kVBytes);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(dst + c * kBox, &tv, 64 * c, h, ck0 + j * kBN, v_full(st));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    const uint64_t dQ = smem_desc(sbase + kOffQ, 16, 1024, kSwizzle128B);
    const uint64_t dK0 = smem_desc(sbase + kOffK, 16, 1024, kSwizzle128B);
    const uint64_t dV0 = smem_desc(sbase + kOffV, kBox, 1024, kSwizzle128B);
    bool ok = warp_wait(q_full, 0, P.err);
    auto issue_pv = [&](int j) -> bool {
      if (!warp_wait(p_full, j & 1, P.err) || !warp_wait(v_full(j & 1), (j >> 1) & 1, P.err))
        return false;
      tc_fence_after();
      const uint64_t dV = dV0 + (j & 1) * (kVBytes >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_f16_ts(tmem + kColO, tmem + kColP + 8u * kk, dV + ((kk * 2048) >> 4), kIdescPV,
                     (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(v_empty(j & 1));
        mma_commit(pv_done);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; ok && j < n_tiles; ++j) {
      const uint32_t st = j & 1;
      ok = warp_wait(k_full(st), (j >> 1) & 1, P.err) &&
           warp_wait(s_free(st), ((j >> 1) & 1) ^ 1, P.err);
      if (!ok) break;
      tc_fence_after();
      const uint64_t dK = dK0 + st * (kKBytes >> 4);
      if (elect_one()) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + kColS + 128u * st, dQ + ((c * kBox + kk * 32) >> 4),
                    dK + ((c * kBox + kk * 32) >> 4), kIdescS, (c | kk) != 0 ? 1u : 0u);
        }
        mma_commit(s_full(st));
        mma_commit(k_empty(st));
      }
      __syncwarp();
      if (j > 0) ok = issue_pv(j - 1);
    }
    if (ok) ok = issue_pv(n_tiles - 1);
    mma_commit_warp(drain);
    if (lane == 0) mbar_wait_drain(drain, 0, P.err);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    // Two warpgroups; warpgroup wg takes keys 64wg..64wg+63 of every tile
    // (and the same 64 value dims of O), a thread one query row (TMEM lane).
    // The halves meet once per tile to agree on the row maximum, through
    // shared memory and a named barrier.
    const int wg = (warp - 2) >> 2;                   // 0 or 1
    const int sp = warp & 3;                          // TMEM sub-partition
    const int r = sp * 32 + lane;                     // query row in the tile
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    const uint32_t c0 = 64u * wg;                     // this half's first column
    const bool row_ok = r < rows;
    const int i = q0 + (row_ok ? r : rows - 1);       // local query index
    const uint2* mrow = reinterpret_cast<const uint2*>(P.mask + static_cast<int64_t>(cq0 + i) * P.words);
    float* pmax = reinterpret_cast<float*>(smem + kOffXchg);        // [2][2][128]
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    bool bad = false;                                 // a wait of this warp gave up
    uint2 mw = __ldg(mrow + wg);
    for (int j = 0; j < n_tiles; ++j) {
      const uint32_t st = j & 1;
      uint32_t v[64];
      float mx = -INFINITY;
      if (!bad) bad = !warp_wait(s_full(st), (j >> 1) & 1, P.err);
      if (!bad) {
        tc_fence_after();
        tmem_ld_32x32b_x64(tmem + lane_base + kColS + 128u * st + c0, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(st));
        // mask: a key counts when it is selected (which implies s <= p) and
        // the row exists; a warp whose 64 keys are all selected skips it
        const uint32_t w0 = row_ok ? mw.x : 0u, w1 = row_ok ? mw.y : 0u;
        if (j + 1 < n_tiles) mw = __ldg(mrow + 2 * (j + 1) + wg);
        if (!__all_sync(0xffffffffu, (w0 & w1) == 0xffffffffu)) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!(((c < 32 ? w0 : w1) >> (c & 31)) & 1u)) v[c] = 0xff800000u;
        }
#pragma unroll
        for (int c = 0; c < 64; ++c) mx = fmaxf(mx, __uint_as_float(v[c]));
      }
      // the row maximum over both halves; the reducing barrier also takes
      // both warpgroups out together when a wait of one of them gave up
      float* px = pmax + st * 256;
      px[wg * 128 + r] = mx;
      if (named_bar_or(1, 256, bad)) {
        ok = false;
        break;
      }
      mx = fmaxf(mx, px[(wg ^ 1) * 128 + r]) * P.scale_log2;
      float al = 1.f;
      bool moved = false;
      if (mx > m + kRescaleThreshold) {
        al = fast_exp2(m - mx);                       // 0 when m = -inf
        m = mx;
        moved = true;
      }
      const float nm = m == -INFINITY ? 0.f : -m;
      const float2 sc2 = make_float2(P.scale_log2, P.scale_log2), nm2 = make_float2(nm, nm);
      uint32_t pk[32];
      float2 s2 = make_float2(0.f, 0.f), r2 = s2;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])),
                                    sc2, nm2);
        const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
        s2 = __fadd2_rn(s2, make_float2(p0, p1));
        pk[c] = pack_bf16x2(p0, p1);
        r2 = __fadd2_rn(r2, make_float2(__uint_as_float(pk[c] << 16), __uint_as_float(pk[c] & 0xFFFF0000u)));
      }
      l = l * al + (s2.x + s2.y);
      lr = lr * al + (r2.x + r2.y);
      // P and O are the previous P V's operands: wait until it is complete
      if (j > 0) {
        if (!warp_wait(pv_done, (j - 1) & 1, P.err)) {
          bad = true;                                 // the next barrier stops everyone
          continue;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, moved)) {
#pragma unroll 1
          for (int c = 0; c < 64; c += 32) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tmem + lane_base + kColO + c0 + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * al);
            tmem_st_32x32b_x32(tmem + lane_base + kColO + c0 + c, o);
          }
        }
      }
      tmem_st_32x32b_x32(tmem + lane_base + kColP + 32u * wg, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // the two halves' sums (every thread reaches this exchange: a thread that
    // stopped on a failed wait brings zeros and stores nothing)
    float* px = pmax + 512;                           // [2][2][128]: l and lr per half
    px[wg * 256 + r] = l;
    px[wg * 256 + 128 + r] = lr;
    named_bar_sync(1, 256);
    const float l_all = l + px[(wg ^ 1) * 256 + r];
    const float lr_all = lr + px[(wg ^ 1) * 256 + 128 + r];
    if (ok && !bad && warp_wait(pv_done, (n_tiles - 1) & 1, P.err)) {
      tc_fence_after();
      const float inv = lr_all > 0.f ? 1.f / lr_all : 0.f;
      __nv_bfloat16* orow = P.out + (static_cast<int64_t>(cq0 + i) * P.H + h) * kDv + c0;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tmem + lane_base + kColO + c0 + c, o);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv, __uint_as_float(o[e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c + e) = w;
          }
        }
      }
      if (row_ok && wg == 0 && P.lse)
        P.lse[static_cast<int64_t>(cq0 + i) * P.H + h] =
            l_all > 0.f ? (m + log2f(l_all)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t masked_mha_workspace_bytes(int64_t total_q, int max_len_k) {
  const int64_t words = ((static_cast<int64_t>(max_len_k) + 127) / 128) * 4;
  return static_cast<size_t>(total_q * words * 4);
}

cudaError_t launch_masked_mha(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const MaskedMhaArgs& a, DevErr err, cudaStream_t s) {
  const int64_t words = ((static_cast<int64_t>(a.max_len_k) + 127) / 128) * 4;
  const size_t mask_smem = static_cast<size_t>(words) * 4;
  cudaError_t e = cudaFuncSetAttribute(mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(mask_smem));
  if (e != cudaSuccess) return e;
  mask_kernel<<<static_cast<unsigned>(a.total_q), 256, mask_smem, s>>>(
      a.idx, a.k, a.cu_q, a.cu_k, a.B, a.mask, words);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  Params P;
  P.cu_q = a.cu_q;
  P.cu_k = a.cu_k;
  P.mask = a.mask;
  P.words = words;
  P.H = a.H;
  P.q_tiles = (a.max_len_q + kBM - 1) / kBM;
  P.scale_log2 = a.sm_scale * 1.4426950408889634f;
  P.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  P.lse = a.lse;
  P.err = err;
  e = cudaFuncSetAttribute(masked_mha_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(a.B) * static_cast<unsigned>(P.q_tiles),
                  static_cast<unsigned>(a.H));
  masked_mha_kernel<<<grid, kThreads, kSmem, s>>>(tq, tk, tv, P);
  return cudaGetLastError();
}

}  // namespace dsa
