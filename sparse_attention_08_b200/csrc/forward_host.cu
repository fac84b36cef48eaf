// forward_host.cu -- dsa_forward over inputs and outputs in host memory,
// pipelined in chunks of query rows so that the host-device copies of one
// chunk overlap the kernels of another.
//
// The pages' statement of the method ("DeepSeek V3.2 and the lightning
// indexer", section "How the lightning indexer works") makes every query row
// independent once the keys it may see are on the device: its scores, its
// selection and its attention read only its own row and the key-side
// tensors.  So the keys (FP8 indexer keys, their scales, the latents) are
// copied once, and the query rows go through the GPU in chunks: a chunk is a
// run of consecutive rows, cut out of the batch with the chunked-prefill
// convention of the ABI (a sequence's queries in the chunk are the last
// positions of the key prefix they may see), so the chunk's results are
// bitwise those of one dsa_forward over the whole batch.
//
// Chunk c runs on stream c % n_streams: upload of its query rows, the three
// kernels, download of its outputs.  With separate copy engines for the two
// directions, the upload of chunk c+1, the kernels of chunk c and the
// download of chunk c-1 run at the same time.
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "dsa.h"

namespace {

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Byte offsets into the caller's device workspace.
struct HostLayout {
  size_t cu_q, cu_k, k8, k_scale, kv, keys_end;  // shared by every chunk
  size_t q8, q_scale, w, q, out, lse, ccu_q, ccu_k, fws, fws_bytes, per_stream;  // per stream
  size_t total;
};

bool make_layout(int64_t total_k, int max_len_k, int B, int H_I, int d_I, int H, int k,
                 int chunk_q, int n_streams, HostLayout& L) {
  if (total_k < 0 || max_len_k < 0 || B < 0 || H_I < 1 || d_I < 1 || H < 1 || k < 1 ||
      chunk_q < 1 || n_streams < 1)
    return false;
  const size_t c = static_cast<size_t>(chunk_q);
  const size_t tk = static_cast<size_t>(total_k);
  size_t o = 0;
  L.cu_q = o; o += round256(static_cast<size_t>(B + 1) * 4);
  L.cu_k = o; o += round256(static_cast<size_t>(B + 1) * 4);
  L.k8 = o; o += round256(tk * d_I);
  L.k_scale = o; o += round256(tk * 4);
  L.kv = o; o += round256(tk * 576 * 2);
  L.keys_end = o;
  size_t s = 0;
  L.q8 = s; s += round256(c * H_I * d_I);
  L.q_scale = s; s += round256(c * H_I * 4);
  L.w = s; s += round256(c * H_I * 4);
  L.q = s; s += round256(c * H * 576 * 2);
  L.out = s; s += round256(c * H * 512 * 2);
  L.lse = s; s += round256(c * H * 4);
  const size_t nb = static_cast<size_t>(B < chunk_q ? B : chunk_q) + 1;
  L.ccu_q = s; s += round256(nb * 4);
  L.ccu_k = s; s += round256(nb * 4);
  L.fws_bytes = dsa_forward_workspace_size(chunk_q, max_len_k, k);
  if (L.fws_bytes == 0) return false;
  L.fws = s; s += round256(L.fws_bytes);
  L.per_stream = s;
  L.total = o + static_cast<size_t>(n_streams) * s;
  return true;
}

// cu_seqlens of one chunk: sequences b0 .. b0+nb-1 of the batch, restricted
// to the query rows [r0, r1); keys are counted from the first sequence's
// first key.  Only the chunk's last sequence can have queries beyond r1;
// its keys end at the position of its last query in the chunk.
__global__ void chunk_cu_kernel(const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k,
                                int b0, int nb, int64_t r0, int64_t r1, int32_t* ccu_q,
                                int32_t* ccu_k) {
  const int32_t k0 = cu_k[b0];
  for (int i = threadIdx.x; i <= nb; i += blockDim.x) {
    if (i < nb) {
      const int b = b0 + i;
      const int64_t qa = cu_q[b] > r0 ? cu_q[b] : r0;
      ccu_q[i] = static_cast<int32_t>(qa - r0);
      ccu_k[i] = cu_k[b] - k0;
    } else {
      const int b = b0 + nb - 1;
      const int64_t qe = cu_q[b + 1] < r1 ? cu_q[b + 1] : r1;
      const int32_t len_q = cu_q[b + 1] - cu_q[b];
      const int32_t len_k = cu_k[b + 1] - cu_k[b];
      ccu_q[nb] = static_cast<int32_t>(r1 - r0);
      ccu_k[nb] = (cu_k[b] - k0) + (len_k - len_q) + static_cast<int32_t>(qe - cu_q[b]);
    }
  }
}

}  // namespace

extern "C" {

size_t dsa_forward_host_workspace_size(int64_t total_k, int max_len_k, int B, int H_I, int d_I,
                                       int H, int k, int chunk_q, int n_streams) {
  HostLayout L;
  if (!make_layout(total_k, max_len_k, B, H_I, d_I, H, k, chunk_q, n_streams, L)) return 0;
  return L.total;
}

dsa_status_t dsa_forward_host(const void* q_fp8, const float* q_scale, const float* w,
                              const void* k_fp8, const float* k_scale, const void* q,
                              const void* kv, const int32_t* cu_seqlens_q,
                              const int32_t* cu_seqlens_k, int B, int max_len_q, int max_len_k,
                              int64_t total_q, int64_t total_k, int H_I, int d_I, int H, int d_qk,
                              int d_v, int k, float sm_scale, void* out, float* lse, int chunk_q,
                              void* workspace, size_t workspace_bytes, void* const* streams,
                              int n_streams) {
  if (!cu_seqlens_q || !cu_seqlens_k || B < 0 || total_q < 0 || total_k < 0 || max_len_q < 0 ||
      max_len_k < 0 || chunk_q < 1 || n_streams < 1 || !streams)
    return DSA_ERR_INVALID_ARG;
  if (!q_fp8 || !q_scale || !w || !k_fp8 || !k_scale || !q || !kv || !out)
    return DSA_ERR_INVALID_ARG;
  if (d_qk != 576 || d_v != 512) return DSA_ERR_UNSUPPORTED;
  for (int i = 0; i < n_streams; ++i)
    if (i > 0 && !streams[i]) return DSA_ERR_INVALID_ARG;   // stream 0 may be the legacy stream
  // the batch's own cu_seqlens (host): from 0 to the totals, len_q <= len_k
  if (cu_seqlens_q[0] != 0 || cu_seqlens_k[0] != 0 || cu_seqlens_q[B] != total_q ||
      cu_seqlens_k[B] != total_k)
    return DSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    const int64_t lq = static_cast<int64_t>(cu_seqlens_q[b + 1]) - cu_seqlens_q[b];
    const int64_t lk = static_cast<int64_t>(cu_seqlens_k[b + 1]) - cu_seqlens_k[b];
    if (lq < 0 || lk < lq || lq > max_len_q || lk > max_len_k) return DSA_ERR_INVALID_ARG;
  }
  HostLayout L;
  if (!make_layout(total_k, max_len_k, B, H_I, d_I, H, k, chunk_q, n_streams, L))
    return DSA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DSA_ERR_ALIGNMENT;
  if (total_q == 0 || B == 0) return DSA_OK;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto st = [&](int i) { return static_cast<cudaStream_t>(streams[i]); };
  const cudaStream_t s0 = st(0);
  bool ok = true;
  auto h2d = [&](void* dst, const void* src, size_t bytes, cudaStream_t s) {
    if (ok && bytes) ok = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s) == cudaSuccess;
  };
  auto d2h = [&](void* dst, const void* src, size_t bytes, cudaStream_t s) {
    if (ok && bytes) ok = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess;
  };
  // key-side tensors and the batch's cu_seqlens, once, on stream 0
  const size_t tk = static_cast<size_t>(total_k);
  h2d(ws + L.cu_q, cu_seqlens_q, static_cast<size_t>(B + 1) * 4, s0);
  h2d(ws + L.cu_k, cu_seqlens_k, static_cast<size_t>(B + 1) * 4, s0);
  h2d(ws + L.k8, k_fp8, tk * d_I, s0);
  h2d(ws + L.k_scale, k_scale, tk * 4, s0);
  h2d(ws + L.kv, kv, tk * 576 * 2, s0);
  cudaEvent_t keys_ready = nullptr;
  if (ok) ok = cudaEventCreateWithFlags(&keys_ready, cudaEventDisableTiming) == cudaSuccess;
  if (ok) ok = cudaEventRecord(keys_ready, s0) == cudaSuccess;
  for (int i = 1; ok && i < n_streams; ++i)
    ok = cudaStreamWaitEvent(st(i), keys_ready, 0) == cudaSuccess;

  dsa_status_t result = DSA_OK;
  const int32_t* cq = cu_seqlens_q;
  const int32_t* ck = cu_seqlens_k;
  const uint8_t* q8_h = static_cast<const uint8_t*>(q_fp8);
  const uint8_t* q_h = static_cast<const uint8_t*>(q);
  uint8_t* out_h = static_cast<uint8_t*>(out);
  int b_first = 0;
  int c = 0;
  for (int64_t r0 = 0; ok && result == DSA_OK && r0 < total_q; r0 += chunk_q, ++c) {
    const int64_t r1 = r0 + chunk_q < total_q ? r0 + chunk_q : total_q;
    const int si = c % n_streams;
    const cudaStream_t s = st(si);
    uint8_t* reg = ws + L.keys_end + static_cast<size_t>(si) * L.per_stream;
    // sequences that own rows of [r0, r1): b_first .. b_last
    while (cq[b_first + 1] <= r0) ++b_first;
    int b_last = b_first;
    while (b_last + 1 < B && cq[b_last + 1] < r1) ++b_last;
    const int nb = b_last - b_first + 1;
    int mlq = 0, mlk = 0;
    for (int b = b_first; b <= b_last; ++b) {
      const int64_t qa = cq[b] > r0 ? cq[b] : r0;
      const int64_t qe = cq[b + 1] < r1 ? cq[b + 1] : r1;
      const int lq = static_cast<int>(qe - qa);
      const int lk = (ck[b + 1] - ck[b]) - (cq[b + 1] - cq[b]) + static_cast<int>(qe - cq[b]);
      if (lq > mlq) mlq = lq;
      if (lk > mlk) mlk = lk;
    }
    if (mlq > mlk) mlk = mlq;
    const int64_t rows = r1 - r0;
    const int64_t k_base = ck[b_first];
    const int64_t k_count = static_cast<int64_t>(ck[b_last] - ck[b_first]) +
                            (ck[b_last + 1] - ck[b_last]) - (cq[b_last + 1] - cq[b_last]) +
                            ((cq[b_last + 1] < r1 ? cq[b_last + 1] : r1) - cq[b_last]);
    // this chunk's query rows
    h2d(reg + L.q8, q8_h + r0 * H_I * d_I, static_cast<size_t>(rows) * H_I * d_I, s);
    h2d(reg + L.q_scale, q_scale + r0 * H_I, static_cast<size_t>(rows) * H_I * 4, s);
    h2d(reg + L.w, w + r0 * H_I, static_cast<size_t>(rows) * H_I * 4, s);
    h2d(reg + L.q, q_h + r0 * H * 1152, static_cast<size_t>(rows) * H * 1152, s);
    if (!ok) break;
    chunk_cu_kernel<<<1, 256, 0, s>>>(reinterpret_cast<const int32_t*>(ws + L.cu_q),
                                      reinterpret_cast<const int32_t*>(ws + L.cu_k), b_first, nb,
                                      r0, r1, reinterpret_cast<int32_t*>(reg + L.ccu_q),
                                      reinterpret_cast<int32_t*>(reg + L.ccu_k));
    if (cudaGetLastError() != cudaSuccess) {
      ok = false;
      break;
    }
    result = dsa_forward(reg + L.q8, reinterpret_cast<const float*>(reg + L.q_scale),
                         reinterpret_cast<const float*>(reg + L.w), ws + L.k8 + k_base * d_I,
                         reinterpret_cast<const float*>(ws + L.k_scale) + k_base,
                         reg + L.q, ws + L.kv + k_base * 1152,
                         reinterpret_cast<const int32_t*>(reg + L.ccu_q),
                         reinterpret_cast<const int32_t*>(reg + L.ccu_k), nb, mlq, mlk, rows,
                         k_count, H_I, d_I, H, d_qk, d_v, k, sm_scale, reg + L.out,
                         lse ? reinterpret_cast<float*>(reg + L.lse) : nullptr, nullptr,
                         reg + L.fws, L.fws_bytes, s);
    d2h(out_h + r0 * H * 1024, reg + L.out, static_cast<size_t>(rows) * H * 1024, s);
    if (lse) d2h(lse + r0 * H, reg + L.lse, static_cast<size_t>(rows) * H * 4, s);
  }
  // the call returns with the outputs in host memory
  for (int i = 0; i < n_streams; ++i)
    if (cudaStreamSynchronize(st(i)) != cudaSuccess) ok = false;
  if (keys_ready) cudaEventDestroy(keys_ready);
  if (result != DSA_OK) return result;
  return ok ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
