// indexer_bwd.cu -- the lightning indexer's backward on sm_100a.
//
// What it computes ("DeepSeek V3.2 and the lightning indexer", section
// "Teaching a dense model to be sparse": in the warm-up only the indexer is
// trained, from the KL signal on its scores).  For the scores
//
//   I[t,s] = sum_j w[t,j] * ReLU(qhat[t,j,:] . khat[s,:]),
//   qhat = q8 * q_scale, khat = k8 * k_scale (the FP8 values dequantised),
//
// and an upstream gradient g[t,s] over the causal pairs s <= p(t), the
// gradients with respect to qhat, w and khat (the quantisation is passed
// straight through; the ReLU's derivative is 0 at 0):
//
//   U[t,j,:]  = sum_s g[t,s] [q8.k8 > 0] k_scale[s] k8[s,:]
//   dq[t,j,:] = w[t,j] U[t,j,:]            dw[t,j] = qhat[t,j,:] . U[t,j,:]
//   dk[s,:]   = sum_{t,j} g[t,s] [q8.k8 > 0] w[t,j] q_scale[t,j] q8[t,j,:]
//
// (the sign of q8.k8 is that of qhat.khat, the scales being positive).
//
// How: the gates come from the forward's FP8 contraction, recomputed per tile
// (tcgen05.mma kind::f8f6f4 into TMEM); an epilogue warpgroup turns them into
// the bf16 A operand of a second contraction (kind::f16) whose B operand is
// the FP8 tile converted to bf16, which e4m3 values fit exactly: the scales,
// the gradient and the head weights are folded into A, so each product is
// rounded to bf16 once.  dq/dw: one CTA per (sequence, group of 4 queries)
// walks its key tiles and accumulates U (256 rows of (query, head) x 128 dims)
// in TMEM.  dk: one CTA per (key tile, run of query groups) accumulates the
// run's share of dk (128 keys x 128 dims) in TMEM and adds it into dk, which
// the caller's entry point zeroes first.  Supported: H_I = 64, d_I = 128.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {
namespace {

constexpr int kBK = 128;                  // keys per tile
constexpr int kHI = 64;
constexpr int kQPT = 4;                   // queries per group
constexpr int kN = kQPT * kHI;            // 256 (query, head) rows
constexpr int kD = 128;                   // d_I
constexpr int kGroupsPerItem = 64;        // query groups per dk work item
constexpr int kThreads = 64 + 128;        // producer, MMA, one epilogue warpgroup
constexpr uint32_t kAtom = kBK * 128;     // 128 rows x 128 B (a swizzle atom column)
constexpr uint32_t kIdescD = instr_desc(kFmtE4M3, kFmtE4M3, 0, 0, kBK, kN);

// e4m3 (the "fn" encoding, no infinities) -> float, from the bit fields.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = e == 0 ? static_cast<float>(m) * 0.001953125f                  // m * 2^-9
                   : __uint_as_float(((e + 120u) << 23) | (m << 20));         // 1.m * 2^(e-7)
  return (b & 0x80u) ? -v : v;
}

// Two e4m3 codes (bits 0-7 and 8-15 of two) -> bf16x2 (first in the low
// half), exactly: the hardware widens e4m3 to f16 (which holds every e4m3
// value), and f16 -> f32 -> bf16 loses nothing for these values either.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h2)
      : "r"(two));
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
  return pack_bf16x2(lo, hi);
}

// ---------------------------------------------------------------------------
// dq, dw
// ---------------------------------------------------------------------------
constexpr uint32_t kQOffQ8 = 0;                         // 256 rows x 128 B (FP8 MMA B)
constexpr uint32_t kQOffK8 = kQOffQ8 + kN * kD;         // 2 stages x 128 rows x 128 B
constexpr uint32_t kK8Bytes = kBK * kD;
constexpr uint32_t kQOffA = kQOffK8 + 2 * kK8Bytes;     // A: 4 M-atoms (MN-major)
constexpr uint32_t kQOffKh = kQOffA + 4 * kAtom;        // B: 2 N-atoms (MN-major)
constexpr uint32_t kQOffBar = kQOffKh + 2 * kAtom;
// barriers: q_full, k_full[2], k_empty[2], d_full, d_empty, a_full, u_done, drain
constexpr uint32_t kQOffMisc = kQOffBar + 10 * 8;
constexpr uint32_t kQSmem = kQOffMisc + 16 + 1024;
constexpr uint32_t kIdescU = instr_desc(kFmtBF16, kFmtBF16, 1, 1, 128, kD);
static_assert(kQSmem <= 232448, "shared memory budget");

struct BwdQParams {
  const float* g;
  int64_t ldg;
  const float* w;
  const float* q_scale;
  const float* k_scale;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, n_qg;
  float* dq;
  float* dw;
  DevErr err;
};

__global__ void __launch_bounds__(kThreads, 1)
    indexer_bwd_q_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k, const BwdQParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kQOffBar;
  const uint32_t q_full = bar0;
  auto k_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto k_empty = [&](int i) { return bar0 + 8u * (3 + i); };
  const uint32_t d_full = bar0 + 40, d_empty = bar0 + 48, a_full = bar0 + 56, u_done = bar0 + 64;
  const uint32_t drain = bar0 + 72;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kQOffMisc);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // the item: sequence b, query group qg (the longest groups first)
  const int b = static_cast<int>(blockIdx.x / P.n_qg);
  const int qg = P.n_qg - 1 - static_cast<int>(blockIdx.x % P.n_qg);
  const int cq0 = __ldg(P.cu_q + b), ck0 = __ldg(P.cu_k + b);
  const int len_q = __ldg(P.cu_q + b + 1) - cq0, len_k = __ldg(P.cu_k + b + 1) - ck0;
  const int q0 = qg * kQPT;
  if (q0 >= len_q || len_q > len_k) return;
  const int nq = min(kQPT, len_q - q0);
  const int off = len_k - len_q;
  const int n_tiles = (off + q0 + nq - 1) / kBK + 1;   // tiles up to the group's last position
  const int q_row0 = cq0 + q0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 4);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, 4);
    mbar_init(a_full, 4);
    mbar_init(u_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // D: columns 0..255; U half mh: 256 + 128 mh

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kN * kD);
      tma_load_2d(sbase + kQOffQ8, &tmap_q, 0, q_row0 * kHI, q_full);
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int st = j & 1;
        if (!mbar_wait(k_empty(st), ((j >> 1) & 1) ^ 1, P.err)) break;
        mbar_arrive_expect_tx(k_full(st), kK8Bytes);
        tma_load_2d(sbase + kQOffK8 + st * kK8Bytes, &tmap_k, 0, ck0 + j * kBK, k_full(st));
      }
      // this CTA's own copies land before it leaves
      for (int u = (j > 2 ? j - 2 : 0); u < j; ++u)
        mbar_wait_drain(k_full(u & 1), (u >> 1) & 1, P.err);
      mbar_wait_drain(q_full, 0, P.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = warp_wait(q_full, 0, P.err);
    for (int j = 0; ok && j < n_tiles; ++j) {
      const int st = j & 1;
      ok = warp_wait(k_full(st), (j >> 1) & 1, P.err) && warp_wait(d_empty, (j & 1) ^ 1, P.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t ka = sbase + kQOffK8 + st * kK8Bytes;
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          mma_f8(tmem, smem_desc(ka + kk * 32, 16, 1024, kSwizzle128B),
                 smem_desc(sbase + kQOffQ8 + kk * 32, 16, 1024, kSwizzle128B), kIdescD,
                 kk > 0 ? 1u : 0u);
        mma_commit(d_full);
      }
      __syncwarp();
      if (!(ok = warp_wait(a_full, j & 1, P.err))) break;
      tc_fence_after();
      if (elect_one()) {
        // U[(t,j) half mh, d] += A[(t,j), s] Khat[s, d]: A and Khat MN-major,
        // K = the tile's keys, 16 per instruction
#pragma unroll
        for (int mh = 0; mh < 2; ++mh) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_f16(tmem + 256u + 128u * mh,
                    smem_desc(sbase + kQOffA + 2 * mh * kAtom + kk * 2048, kAtom, 1024,
                              kSwizzle128B),
                    smem_desc(sbase + kQOffKh + kk * 2048, kAtom, 1024, kSwizzle128B), kIdescU,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(u_done);
      }
      __syncwarp();
    }
    mma_commit_warp(drain);
    if (lane == 0) mbar_wait_drain(drain, 0, P.err);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // thread = key s of the tile (TMEM lane), warp w reads sub-partition w % 4
    const int sp = warp & 3;
    const int s = sp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j & 1;
      const int sl = j * kBK + s;                     // sequence-local key
      // g * k_scale of this key for each query of the group (0 past p)
      float gk[kQPT];
      const float ks = sl < len_k ? __ldg(P.k_scale + ck0 + sl) : 0.f;
#pragma unroll
      for (int i = 0; i < kQPT; ++i) {
        const bool v = i < nq && sl < len_k && sl <= off + q0 + i;
        gk[i] = v ? __ldg(P.g + static_cast<int64_t>(q_row0 + i) * P.ldg + sl) * ks : 0.f;
      }
      if (!warp_wait(d_full, j & 1, P.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the previous U products read A and Khat: wait for them
      if (j > 0 && !warp_wait(u_done, (j - 1) & 1, P.err)) {
        ok = false;
        break;
      }
      // A row s (MN-major: column c of the 256 in M-atom c / 64, 16-byte piece
      // (c % 64) / 8 swizzled with s & 7)
      uint8_t* arow = smem + kQOffA + s * 128;
#pragma unroll 1
      for (int cb = 0; cb < kN; cb += 64) {
        uint32_t dv[64];
        tmem_ld_32x32b_x64(tmem + lane_base + cb, dv);
        tmem_wait_ld();
        const float gt = gk[cb / 64];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = __uint_as_float(dv[8 * ch + 2 * e]) > 0.f ? gt : 0.f;
            const float a1 = __uint_as_float(dv[8 * ch + 2 * e + 1]) > 0.f ? gt : 0.f;
            pk[e] = pack_bf16x2(a0, a1);
          }
          *reinterpret_cast<uint4*>(arow + (cb / 64) * kAtom + ((ch ^ (s & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      tc_fence_before();
      // the key tile is read below through the generic proxy: observe its TMA
      // completion (the stage cannot move on before this warp releases it)
      if (!warp_wait(k_full(st), (j >> 1) & 1, P.err)) {
        ok = false;
        break;
      }
      // Khat row s: the key tile's e4m3 row (K-major, 128-byte swizzle) as
      // exact bf16, MN-major (dims 64 a to an atom)
      const uint8_t* krow = smem + kQOffK8 + st * kK8Bytes + s * 128;
      uint8_t* hrow = smem + kQOffKh + s * 128;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        const uint4 raw = *reinterpret_cast<const uint4*>(krow + ((c16 ^ (s & 7)) << 4));
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t wv = wd[2 * hh + (e >> 1)];
            const int sh = 16 * (e & 1);
            pk[e] = e4m3x2_to_bf16x2((wv >> sh) & 0xFFFFu);
          }
          const int d0 = 16 * c16 + 8 * hh;             // first dim of this 8-dim piece
          *reinterpret_cast<uint4*>(hrow + (d0 / 64) * kAtom + ((((d0 % 64) / 8) ^ (s & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(d_empty);
        mbar_arrive(k_empty(st));
        mbar_arrive(a_full);
      }
    }
    // U rows: thread s reads row s of both M halves: (query, head) c = 128 mh + s;
    // the query tile is read through the generic proxy: observe its TMA first
    if (ok && warp_wait(u_done, (n_tiles - 1) & 1, P.err) && warp_wait(q_full, 0, P.err)) {
      tc_fence_after();
#pragma unroll 1
      for (int mh = 0; mh < 2; ++mh) {
        const int c = 128 * mh + s;
        const int t = c / kHI, jh = c % kHI;
        float acc_dw = 0.f;
        const int64_t o = static_cast<int64_t>(q_row0 + t) * kHI + jh;
        const float wv = t < nq ? __ldg(P.w + o) : 0.f;
        const float qs = t < nq ? __ldg(P.q_scale + o) : 0.f;
        const uint8_t* qrow = smem + kQOffQ8 + c * 128;  // K-major, 128-byte swizzle
        float* dqrow = P.dq + o * kD;
#pragma unroll 1
        for (int d0 = 0; d0 < kD; d0 += 32) {
          uint32_t u[32];
          tmem_ld_32x32b_x32(tmem + lane_base + 256u + 128u * mh + d0, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int d = d0 + e;
            const uint32_t qb = qrow[(((d / 16) ^ (c & 7)) << 4) + (d % 16)];
            acc_dw = fmaf(e4m3_value(qb) * qs, __uint_as_float(u[e]), acc_dw);
          }
          if (t < nq) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dqrow + d0 + e) =
                  make_float4(wv * __uint_as_float(u[e]), wv * __uint_as_float(u[e + 1]),
                              wv * __uint_as_float(u[e + 2]), wv * __uint_as_float(u[e + 3]));
          }
        }
        if (t < nq) P.dw[o] = acc_dw;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dk
// ---------------------------------------------------------------------------
constexpr uint32_t kQ8Bytes = kN * kD;                 // 32 KB
constexpr uint32_t kKOffQ8 = 0;                        // 2 stages of query tiles
constexpr uint32_t kKOffK8 = kKOffQ8 + 2 * kQ8Bytes;   // the key tile
constexpr uint32_t kKOffA = kKOffK8 + kK8Bytes;        // A: 4 K-atoms (K-major)
constexpr uint32_t kKOffB = kKOffA + 4 * kAtom;        // B: 2 N-atoms (MN-major)
constexpr uint32_t kBAtom = kN * 128;                  // 256 rows x 128 B
constexpr uint32_t kKOffWq = kKOffB + 2 * kBAtom;      // w * q_scale of the group, 256 floats
constexpr uint32_t kKOffBar = kKOffWq + kN * 4;
// barriers: k_full, q_full[2], q_empty[2], d_full, d_empty, a_full, dk_done, drain
constexpr uint32_t kKOffMisc = kKOffBar + 10 * 8;
constexpr uint32_t kKSmem = kKOffMisc + 16 + 1024;
constexpr uint32_t kIdescDk = instr_desc(kFmtBF16, kFmtBF16, 0, 1, 128, kD);
static_assert(kKSmem <= 232448, "shared memory budget");

struct BwdKParams {
  const float* g;
  int64_t ldg;
  const float* w;
  const float* q_scale;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, n_kt, n_gc;         // key tiles and runs of query groups per sequence slot
  float* dk;
  DevErr err;
};

__global__ void __launch_bounds__(kThreads, 1)
    indexer_bwd_k_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k, const BwdKParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kKOffBar;
  const uint32_t k_full = bar0;
  auto q_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto q_empty = [&](int i) { return bar0 + 8u * (3 + i); };
  const uint32_t d_full = bar0 + 40, d_empty = bar0 + 48, a_full = bar0 + 56, dk_done = bar0 + 64;
  const uint32_t drain = bar0 + 72;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kKOffMisc);
  float* wq = reinterpret_cast<float*>(smem + kKOffWq);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // the item: sequence b, key tile kt, run gc of query groups
  const int gc = static_cast<int>(blockIdx.x % P.n_gc);
  const int rest = static_cast<int>(blockIdx.x / P.n_gc);
  const int kt = rest % P.n_kt;
  const int b = rest / P.n_kt;
  const int cq0 = __ldg(P.cu_q + b), ck0 = __ldg(P.cu_k + b);
  const int len_q = __ldg(P.cu_q + b + 1) - cq0, len_k = __ldg(P.cu_k + b + 1) - ck0;
  const int s0 = kt * kBK;
  if (s0 >= len_k || len_q > len_k) return;
  const int off = len_k - len_q;
  // query groups whose last query can see key s0 (off + i >= s0), this run's share
  const int i_first = max(0, s0 - off);
  const int g_lo = max(i_first / kQPT, gc * kGroupsPerItem);
  const int g_hi = min((len_q + kQPT - 1) / kQPT, (gc + 1) * kGroupsPerItem);
  if (g_lo >= g_hi) return;
  const int n_groups = g_hi - g_lo;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 4);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, 4);
    mbar_init(a_full, 4);
    mbar_init(dk_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;   // D: columns 0..255; dk: 256..383

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(k_full, kK8Bytes);
      tma_load_2d(sbase + kKOffK8, &tmap_k, 0, ck0 + s0, k_full);
      int gi = 0;
      for (; gi < n_groups; ++gi) {
        const int st = gi & 1;
        if (!mbar_wait(q_empty(st), ((gi >> 1) & 1) ^ 1, P.err)) break;
        mbar_arrive_expect_tx(q_full(st), kQ8Bytes);
        tma_load_2d(sbase + kKOffQ8 + st * kQ8Bytes, &tmap_q, 0,
                    (cq0 + (g_lo + gi) * kQPT) * kHI, q_full(st));
      }
      for (int u = (gi > 2 ? gi - 2 : 0); u < gi; ++u)
        mbar_wait_drain(q_full(u & 1), (u >> 1) & 1, P.err);
      mbar_wait_drain(k_full, 0, P.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = warp_wait(k_full, 0, P.err);
    for (int gi = 0; ok && gi < n_groups; ++gi) {
      const int st = gi & 1;
      ok = warp_wait(q_full(st), (gi >> 1) & 1, P.err) && warp_wait(d_empty, (gi & 1) ^ 1, P.err);
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t qa = sbase + kKOffQ8 + st * kQ8Bytes;
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          mma_f8(tmem, smem_desc(sbase + kKOffK8 + kk * 32, 16, 1024, kSwizzle128B),
                 smem_desc(qa + kk * 32, 16, 1024, kSwizzle128B), kIdescD, kk > 0 ? 1u : 0u);
        mma_commit(d_full);
      }
      __syncwarp();
      if (!(ok = warp_wait(a_full, gi & 1, P.err))) break;
      tc_fence_after();
      if (elect_one()) {
        // dk[s, d] += A[s, (t,j)] B[(t,j), d]: A K-major, B MN-major,
        // K = the group's 256 (query, head) rows, 16 per instruction
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk)
          mma_f16(tmem + 256u,
                  smem_desc(sbase + kKOffA + (kk / 4) * kAtom + (kk % 4) * 32, 16, 1024,
                            kSwizzle128B),
                  smem_desc(sbase + kKOffB + kk * 2048, kBAtom, 1024, kSwizzle128B), kIdescDk,
                  (gi > 0 || kk > 0) ? 1u : 0u);
        mma_commit(dk_done);
      }
      __syncwarp();
    }
    mma_commit_warp(drain);
    if (lane == 0) mbar_wait_drain(drain, 0, P.err);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int sp = warp & 3;
    const int et = threadIdx.x - 64;                  // 0..127
    const int s = sp * 32 + lane;                     // key lane in the tile
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    const int sl = s0 + s;                            // sequence-local key
    bool ok = true;
    for (int gi = 0; gi < n_groups; ++gi) {
      const int st = gi & 1;
      const int qi0 = (g_lo + gi) * kQPT;             // local index of the group's first query
      const int nq = min(kQPT, len_q - qi0);
      float gq[kQPT];
#pragma unroll
      for (int i = 0; i < kQPT; ++i) {
        const bool v = i < nq && sl < len_k && sl <= off + qi0 + i;
        gq[i] = v ? __ldg(P.g + static_cast<int64_t>(cq0 + qi0 + i) * P.ldg + sl) : 0.f;
      }
      // every wait of the group comes first: the group's D, the previous dk
      // products (they read A, B and the weights), and the query tile (read
      // below through the generic proxy); the warpgroup then decides together
      // whether to go on, so no warp is left at the barrier below
      bool fail = !warp_wait(d_full, gi & 1, P.err);
      if (!fail && gi > 0) fail = !warp_wait(dk_done, (gi - 1) & 1, P.err);
      if (!fail) fail = !warp_wait(q_full(st), (gi >> 1) & 1, P.err);
      if (named_bar_or(1, 128, fail)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // w * q_scale of the group's 256 (query, head) rows
      for (int c = et; c < kN; c += 128) {
        const int t = c / kHI;
        const int64_t o = static_cast<int64_t>(cq0 + qi0 + t) * kHI + (c % kHI);
        wq[c] = t < nq ? __ldg(P.w + o) * __ldg(P.q_scale + o) : 0.f;
      }
      named_bar_sync(1, 128);
      // A row s: g * gate * w * q_scale over the 256 (query, head) columns, K-major
      uint8_t* arow = smem + kKOffA + s * 128;
#pragma unroll 1
      for (int cb = 0; cb < kN; cb += 64) {
        uint32_t dv[64];
        tmem_ld_32x32b_x64(tmem + lane_base + cb, dv);
        tmem_wait_ld();
        const float gt = gq[cb / 64];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = cb + 8 * ch + 2 * e;
            const float a0 = __uint_as_float(dv[8 * ch + 2 * e]) > 0.f ? gt * wq[c] : 0.f;
            const float a1 = __uint_as_float(dv[8 * ch + 2 * e + 1]) > 0.f ? gt * wq[c + 1] : 0.f;
            pk[e] = pack_bf16x2(a0, a1);
          }
          *reinterpret_cast<uint4*>(arow + (cb / 64) * kAtom + ((ch ^ (s & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      tc_fence_before();
      // B rows c = s and s + 128: the query tile's e4m3 rows as exact bf16, MN-major
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int c = s + 128 * half;
        const uint8_t* src = smem + kKOffQ8 + st * kQ8Bytes + c * 128;
        uint8_t* dst = smem + kKOffB + c * 128;
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
          const uint4 raw = *reinterpret_cast<const uint4*>(src + ((c16 ^ (c & 7)) << 4));
          const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t wv = wd[2 * hh + (e >> 1)];
              const int sh = 16 * (e & 1);
              pk[e] = e4m3x2_to_bf16x2((wv >> sh) & 0xFFFFu);
            }
            const int d0 = 16 * c16 + 8 * hh;
            *reinterpret_cast<uint4*>(dst + (d0 / 64) * kBAtom +
                                      ((((d0 % 64) / 8) ^ (c & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(d_empty);
        mbar_arrive(q_empty(st));
        mbar_arrive(a_full);
      }
    }
    // this run's share of dk[s, :], added into dk
    if (ok && warp_wait(dk_done, (n_groups - 1) & 1, P.err)) {
      tc_fence_after();
      float* dkrow = P.dk + static_cast<int64_t>(ck0 + sl) * kD;
#pragma unroll 1
      for (int d0 = 0; d0 < kD; d0 += 32) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(tmem + lane_base + 256u + d0, u);
        tmem_wait_ld();
        if (sl < len_k) {
#pragma unroll
          for (int e = 0; e < 32; ++e) atomicAdd(dkrow + d0 + e, __uint_as_float(u[e]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_indexer_bwd(const CUtensorMap& tq, const CUtensorMap& tk,
                               const IndexerBwdArgs& a, DevErr err_q, DevErr err_k,
                               cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(a.dk, 0, static_cast<size_t>(a.total_k) * kD * sizeof(float), s);
  if (e != cudaSuccess) return e;
  BwdQParams Q;
  Q.g = a.g;
  Q.ldg = a.ldg;
  Q.w = a.w;
  Q.q_scale = a.q_scale;
  Q.k_scale = a.k_scale;
  Q.cu_q = a.cu_q;
  Q.cu_k = a.cu_k;
  Q.B = a.B;
  Q.n_qg = (a.max_len_q + kQPT - 1) / kQPT;
  Q.dq = a.dq;
  Q.dw = a.dw;
  Q.err = err_q;
  e = cudaFuncSetAttribute(indexer_bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kQSmem));
  if (e != cudaSuccess) return e;
  const int64_t grid_q = static_cast<int64_t>(a.B) * Q.n_qg;
  if (grid_q > 0) {
    indexer_bwd_q_kernel<<<static_cast<unsigned>(grid_q), kThreads, kQSmem, s>>>(tq, tk, Q);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  BwdKParams K;
  K.g = a.g;
  K.ldg = a.ldg;
  K.w = a.w;
  K.q_scale = a.q_scale;
  K.cu_q = a.cu_q;
  K.cu_k = a.cu_k;
  K.B = a.B;
  K.n_kt = (a.max_len_k + kBK - 1) / kBK;
  K.n_gc = ((a.max_len_q + kQPT - 1) / kQPT + kGroupsPerItem - 1) / kGroupsPerItem;
  K.dk = a.dk;
  K.err = err_k;
  e = cudaFuncSetAttribute(indexer_bwd_k_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kKSmem));
  if (e != cudaSuccess) return e;
  const int64_t grid_k = static_cast<int64_t>(a.B) * K.n_kt * K.n_gc;
  if (grid_k > 0) {
    indexer_bwd_k_kernel<<<static_cast<unsigned>(grid_k), kThreads, kKSmem, s>>>(tq, tk, K);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace dsa
