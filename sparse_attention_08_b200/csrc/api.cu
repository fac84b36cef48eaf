// api.cu -- the C ABI of libdsa.so (declared in include/dsa.h): argument
// validation, TMA tensor-map encoding, the device error word, and the
// sequencing of the three stages on the caller's stream.
//
// The library allocates no device memory: the error word below is a static
// __device__ variable of the module, and every buffer comes from the caller.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "dsa.h"
#include "internal.h"

namespace {

__device__ unsigned g_dsa_err[2];  // [0] sticky error bits, [1] newest failed launch generation

std::atomic<unsigned> g_generation{1};

// Test hook state (dsa_debug_fault_injection): the wait limit of later
// launches (0 = the default) and a one-shot request for the indexer.
std::atomic<uint64_t> g_wait_limit_ns{0};
std::atomic<unsigned> g_inject_indexer{0};

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  unsigned* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

dsa_status_t device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DSA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dsa_err) != cudaSuccess) return DSA_ERR_CUDA;
    d.err = static_cast<unsigned*>(p);
    d.ready = true;
  }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return DSA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = &d;
  return DSA_OK;
}

dsa::DevErr next_err(const DeviceInfo* d) {
  dsa::DevErr e;
  e.word = d->err;
  e.gen = g_generation.fetch_add(1);
  e.inject = 0;
  const uint64_t lim = g_wait_limit_ns.load();
  e.limit_ns = lim != 0 ? lim : dsa::kWaitLimitNs;
  return e;
}

// Row-major 2D tensor [rows, cols] of `elem` bytes per element, box of
// box_rows x box_cols elements.
dsa_status_t encode_2d(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, uint64_t rows,
                       uint64_t cols, uint64_t elem, uint32_t box_rows, uint32_t box_cols,
                       CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

// Row-major 3D tensor [d2, d1, d0] (d0 innermost) of bf16, box of
// box0 x 1 x box2 elements, 128-byte swizzle.
dsa_status_t encode_3d_bf16(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                            uint32_t box0, uint32_t box2) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {box0, 1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status_t check_varlen(const int32_t* cu_q, const int32_t* cu_k, int B, int max_len_q,
                          int max_len_k, int64_t total_q, int64_t total_k) {
  if (!cu_q || !cu_k || B < 0 || max_len_q < 0 || max_len_k < 0 || total_q < 0 || total_k < 0)
    return DSA_ERR_INVALID_ARG;
  if (max_len_q > max_len_k) return DSA_ERR_INVALID_ARG;
  if (total_q > (int64_t)B * max_len_q || total_k > (int64_t)B * max_len_k)
    return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

dsa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

bool indexer_shape_ok(int H_I, int d_I) {
  const bool h = H_I == 4 || H_I == 8 || H_I == 16 || H_I == 32 || H_I == 64 || H_I == 128;
  return h && (d_I == 64 || d_I == 128);
}

bool mla_heads_ok(int H) { return H == 16 || H == 32 || (H % 64 == 0 && H >= 64 && H <= 256); }

}  // namespace

extern "C" {

const char* dsa_version(void) { return "0.1.0"; }

const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_BOUNDS: return "device bounds check failed";
  }
  return "unknown status";
}

dsa_status_t dsa_indexer_logits(const void* q_fp8, const float* q_scale, const float* w,
                                const void* k_fp8, const float* k_scale,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                                int max_len_q, int max_len_k, int64_t total_q, int64_t total_k,
                                int H_I, int d_I, float* logits, int64_t ld_logits, void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!q_fp8 || !q_scale || !w || !k_fp8 || !k_scale || !logits) return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  if (ld_logits < max_len_k || ld_logits < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(logits) || (ld_logits % 4) != 0)
    return DSA_ERR_ALIGNMENT;
  if (total_q * H_I >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31))
    return DSA_ERR_UNSUPPORTED;
  if (total_q == 0 || total_k == 0 || B == 0) return DSA_OK;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  const CUtensorMapSwizzle swz =
      d_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  // A tile holds 256 (query, head) columns; when every sequence has a single
  // query (decode) and the heads fit, one query of 64 columns instead.
  const int tile_n = (max_len_q <= 1 && H_I >= 16 && H_I <= 64) ? 64 : 256;
  CUtensorMap tq, tk;
  if ((st = encode_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_fp8, total_q * H_I, d_I, 1,
                      static_cast<uint32_t>(tile_n), d_I, swz)) != DSA_OK)
    return st;
  if ((st = encode_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_fp8, total_k, d_I, 1, 128, d_I,
                      swz)) != DSA_OK)
    return st;
  dsa::IndexerArgs a;
  a.q_scale = q_scale;
  a.w = w;
  a.k_scale = k_scale;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.B = B;
  a.max_len_q = max_len_q;
  a.max_len_k = max_len_k;
  a.H_I = H_I;
  a.d_I = d_I;
  a.logits = logits;
  a.ld = ld_logits;
  a.tile_n = tile_n;
  dsa::DevErr err = next_err(dev);
  err.inject = g_inject_indexer.exchange(0);
  return from_cuda(dsa::launch_indexer(tq, tk, a, dev->num_sms, err,
                                       static_cast<cudaStream_t>(stream)));
}

dsa_status_t dsa_topk(const float* logits, int64_t ld_logits, const int32_t* cu_seqlens_q,
                      const int32_t* cu_seqlens_k, int B, int max_len_q, int max_len_k,
                      int64_t total_q, int k, int32_t* idx_out, float* val_out, void* stream) {
  dsa_status_t st =
      check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q, 0);
  if (st != DSA_OK) return st;
  if (!logits || !idx_out) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (max_len_k > (1 << 24)) return DSA_ERR_UNSUPPORTED;
  if (ld_logits < max_len_k || ld_logits < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(idx_out) || (val_out && !aligned16(val_out)) ||
      (ld_logits % 4) != 0)
    return DSA_ERR_ALIGNMENT;
  if (total_q >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (total_q == 0 || B == 0) return DSA_OK;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  dsa::TopkArgs a;
  a.logits = logits;
  a.ld = ld_logits;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.B = B;
  a.max_len_q = max_len_q;
  a.max_len_k = max_len_k;
  a.total_q = total_q;
  a.k = k;
  a.idx = idx_out;
  a.val = val_out;
  return from_cuda(dsa::launch_topk(a, next_err(dev), static_cast<cudaStream_t>(stream)));
}

dsa_status_t dsa_sparse_mla_fwd(const void* q, const void* kv, const int32_t* idx,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                                int max_len_q, int max_len_k, int64_t total_q, int64_t total_k,
                                int H, int d_qk, int d_v, int k, float sm_scale, void* out,
                                float* lse, void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!q || !kv || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (d_qk != 576 || d_v != 512 || !mla_heads_ok(H) || k < 1 || k > 4096)
    return DSA_ERR_UNSUPPORTED;
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return DSA_ERR_ALIGNMENT;
  const int64_t groups = (H + 63) / 64;
  if (total_q * H >= (int64_t(1) << 31) || total_q * groups >= (int64_t(1) << 31) ||
      total_k >= (int64_t(1) << 31))
    return DSA_ERR_UNSUPPORTED;
  if (total_q == 0 || B == 0) return DSA_OK;
  if (total_k == 0) return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  dsa::MlaArgs a;
  a.idx = idx;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.B = B;
  a.max_len_q = max_len_q;
  a.max_len_k = max_len_k;
  a.total_q = total_q;
  a.total_k = total_k;
  a.H = H;
  a.k = k;
  a.sm_scale = sm_scale;
  a.out = out;
  a.lse = lse;
  a.num_sms = dev->num_sms;
  return from_cuda(
      dsa::launch_sparse_mla(q, kv, a, next_err(dev), static_cast<cudaStream_t>(stream)));
}

size_t dsa_masked_mha_workspace_size(int64_t total_q, int max_len_k) {
  if (total_q < 0 || max_len_k < 1 || max_len_k > 131072) return 0;
  return dsa::masked_mha_workspace_bytes(total_q, max_len_k);
}

dsa_status_t dsa_masked_mha_fwd(const void* q, const void* k, const void* v, const int32_t* idx,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                                int max_len_q, int max_len_k, int64_t total_q, int64_t total_k,
                                int H, int d_qk, int d_v, int topk, float sm_scale, void* out,
                                float* lse, void* workspace, size_t workspace_bytes,
                                void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!q || !k || !v || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (d_qk != 192 || d_v != 128 || H < 1 || H > 65535 || topk < 1 || topk > 131072 ||
      max_len_k > 131072)
    return DSA_ERR_UNSUPPORTED;
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(out) ||
      (lse && !aligned16(lse)) || (workspace && !aligned16(workspace)))
    return DSA_ERR_ALIGNMENT;
  if (total_q * H >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31) ||
      (int64_t)B * ((max_len_q + 127) / 128) >= (int64_t(1) << 31))
    return DSA_ERR_UNSUPPORTED;
  if (total_q == 0 || B == 0) return DSA_OK;
  if (total_k == 0) return DSA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < dsa::masked_mha_workspace_bytes(total_q, max_len_k))
    return DSA_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  CUtensorMap tq, tk, tv;
  if ((st = encode_3d_bf16(&tq, q, 192, H, total_q, 64, 128)) != DSA_OK) return st;
  if ((st = encode_3d_bf16(&tk, k, 192, H, total_k, 64, 128)) != DSA_OK) return st;
  if ((st = encode_3d_bf16(&tv, v, 128, H, total_k, 64, 128)) != DSA_OK) return st;
  dsa::MaskedMhaArgs a;
  a.idx = idx;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.B = B;
  a.max_len_q = max_len_q;
  a.max_len_k = max_len_k;
  a.total_q = total_q;
  a.total_k = total_k;
  a.H = H;
  a.k = topk;
  a.sm_scale = sm_scale;
  a.mask = static_cast<uint32_t*>(workspace);
  a.out = out;
  a.lse = lse;
  return from_cuda(dsa::launch_masked_mha(tq, tk, tv, a, next_err(dev),
                                          static_cast<cudaStream_t>(stream)));
}

size_t dsa_indexer_kl_workspace_size(int64_t total_q, int H, int k) {
  if (total_q < 0 || !mla_heads_ok(H) || k < 1 || k > 4096) return 0;
  return dsa::indexer_kl_workspace_bytes(total_q, H, k);
}

dsa_status_t dsa_indexer_kl(const void* q, const void* kv, const int32_t* idx, const float* lse,
                            const float* logits, int64_t ld_logits, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, int B, int max_len_q, int max_len_k,
                            int64_t total_q, int64_t total_k, int H, int d_qk, int k,
                            float sm_scale, float* kl_out, float* grad_out, float* target_out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!q || !kv || !idx || !lse || !logits || !kl_out) return DSA_ERR_INVALID_ARG;
  if (d_qk != 576 || !mla_heads_ok(H) || k < 1 || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (!(sm_scale > 0.f) || sm_scale != sm_scale) return DSA_ERR_INVALID_ARG;
  if (ld_logits < max_len_k || ld_logits < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(workspace)) return DSA_ERR_ALIGNMENT;
  const int64_t groups = (H + 127) / 128;
  if (total_q * H >= (int64_t(1) << 31) || groups * 4 * total_q * k >= (int64_t(1) << 40) ||
      total_k >= (int64_t(1) << 31))
    return DSA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < dsa_indexer_kl_workspace_size(total_q, H, k))
    return DSA_ERR_WORKSPACE;
  if (total_q == 0 || B == 0) return DSA_OK;
  if (total_k == 0) return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  dsa::KlArgs a;
  a.q = q;
  a.kv = kv;
  a.idx = idx;
  a.lse = lse;
  a.logits = logits;
  a.ld = ld_logits;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.B = B;
  a.total_q = total_q;
  a.H = H;
  a.k = k;
  a.sm_scale = sm_scale;
  a.kl = kl_out;
  a.grad = grad_out;
  a.target = target_out;
  a.part = static_cast<float*>(workspace);
  a.num_sms = dev->num_sms;
  return from_cuda(
      dsa::launch_indexer_kl(a, next_err(dev), static_cast<cudaStream_t>(stream)));
}

dsa_status_t dsa_indexer_backward(const void* q_fp8, const float* q_scale, const float* w,
                                  const void* k_fp8, const float* k_scale, const float* g,
                                  int64_t ld_g, const int32_t* cu_seqlens_q,
                                  const int32_t* cu_seqlens_k, int B, int max_len_q,
                                  int max_len_k, int64_t total_q, int64_t total_k, int H_I,
                                  int d_I, float* dq, float* dw, float* dk, void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!q_fp8 || !q_scale || !w || !k_fp8 || !k_scale || !g || !dq || !dw || !dk)
    return DSA_ERR_INVALID_ARG;
  if (H_I != 64 || d_I != 128) return DSA_ERR_UNSUPPORTED;
  if (ld_g < max_len_k || ld_g < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || !aligned16(g) || (ld_g % 4) != 0 ||
      !aligned16(dq) || !aligned16(dk))
    return DSA_ERR_ALIGNMENT;
  if (total_q * H_I >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31) ||
      static_cast<int64_t>(B) * ((max_len_k + 127) / 128) * ((max_len_q + 255) / 256 + 1) >=
          (int64_t(1) << 31))
    return DSA_ERR_UNSUPPORTED;
  if (total_q == 0 || B == 0 || total_k == 0) return DSA_OK;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  CUtensorMap tq, tk;
  if ((st = encode_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_fp8, total_q * H_I, d_I, 1, 256, d_I,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != DSA_OK)
    return st;
  if ((st = encode_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_fp8, total_k, d_I, 1, 128, d_I,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != DSA_OK)
    return st;
  dsa::IndexerBwdArgs a;
  a.g = g;
  a.ldg = ld_g;
  a.w = w;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.B = B;
  a.max_len_q = max_len_q;
  a.max_len_k = max_len_k;
  a.total_k = total_k;
  a.dq = dq;
  a.dw = dw;
  a.dk = dk;
  const dsa::DevErr eq = next_err(dev);
  const dsa::DevErr ek = next_err(dev);
  return from_cuda(dsa::launch_indexer_bwd(tq, tk, a, eq, ek, static_cast<cudaStream_t>(stream)));
}

size_t dsa_forward_workspace_size(int64_t total_q, int max_len_k, int k) {
  if (total_q < 0 || max_len_k < 0 || k < 1) return 0;
  const int64_t ld = (static_cast<int64_t>(max_len_k) + 3) / 4 * 4;
  const int64_t logits = (total_q * ld * 4 + 255) / 256 * 256;
  const int64_t idx = (total_q * static_cast<int64_t>(k) * 4 + 255) / 256 * 256;
  return static_cast<size_t>(logits + idx);
}

dsa_status_t dsa_forward(const void* q_fp8, const float* q_scale, const float* w,
                         const void* k_fp8, const float* k_scale, const void* q, const void* kv,
                         const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                         int max_len_q, int max_len_k, int64_t total_q, int64_t total_k, int H_I,
                         int d_I, int H, int d_qk, int d_v, int k, float sm_scale, void* out,
                         float* lse, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                         void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  if (d_qk != 576 || d_v != 512 || !mla_heads_ok(H) || k < 1 || k > 4096)
    return DSA_ERR_UNSUPPORTED;
  const size_t need = dsa_forward_workspace_size(total_q, max_len_k, k);
  if (!workspace || workspace_bytes < need) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_ALIGNMENT;
  if (total_q == 0 || B == 0) return DSA_OK;
  const int64_t ld = (static_cast<int64_t>(max_len_k) + 3) / 4 * 4;
  float* logits = static_cast<float*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                            (total_q * ld * 4 + 255) / 256 * 256);
  if (idx_out) idx = idx_out;
  st = dsa_indexer_logits(q_fp8, q_scale, w, k_fp8, k_scale, cu_seqlens_q, cu_seqlens_k, B,
                          max_len_q, max_len_k, total_q, total_k, H_I, d_I, logits, ld, stream);
  if (st != DSA_OK) return st;
  st = dsa_topk(logits, ld, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q, k, idx,
                nullptr, stream);
  if (st != DSA_OK) return st;
  return dsa_sparse_mla_fwd(q, kv, idx, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k,
                            total_q, total_k, H, d_qk, d_v, k, sm_scale, out, lse, stream);
}

namespace {

// Regions of the fused forward's workspace, each 256-byte aligned.
struct FusedLayout {
  int64_t ld, ld_s, max_samples;
  size_t logits, idx, k8_s, ks_s, cu_k_s, logits_s, thr, flags, cand_key, cand_pos, total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

FusedLayout fused_layout(int64_t total_q, int64_t total_k, int B, int max_len_k, int k,
                         int d_I) {
  FusedLayout f;
  f.ld = (static_cast<int64_t>(max_len_k) + 3) / 4 * 4;
  const int64_t max_len_s = (static_cast<int64_t>(max_len_k) + dsa::kSampleStride - 1) /
                            dsa::kSampleStride;
  f.ld_s = (max_len_s + 3) / 4 * 4;
  // sum over sequences of ceil(len_k / stride) <= total_k / stride + B
  f.max_samples = total_k / dsa::kSampleStride + B;
  size_t o = 0;
  f.logits = o;   o += align256(static_cast<size_t>(total_q * f.ld) * 4);
  f.idx = o;      o += align256(static_cast<size_t>(total_q) * k * 4);
  f.k8_s = o;     o += align256(static_cast<size_t>(f.max_samples) * d_I);
  f.ks_s = o;     o += align256(static_cast<size_t>(f.max_samples) * 4);
  f.cu_k_s = o;   o += align256(static_cast<size_t>(B + 1) * 4);
  f.logits_s = o; o += align256(static_cast<size_t>(total_q * f.ld_s) * 4);
  f.thr = o;      o += align256(static_cast<size_t>(total_q) * 4);
  f.flags = o;    o += align256(static_cast<size_t>(2 * total_q + 1) * 4);   // cnt, row_on, any
  f.cand_key = o; o += align256(static_cast<size_t>(total_q) * dsa::kFusedCap * 4);
  f.cand_pos = o; o += align256(static_cast<size_t>(total_q) * dsa::kFusedCap * 4);
  f.total = o;
  return f;
}

}  // namespace

size_t dsa_forward_fused_workspace_size(int64_t total_q, int64_t total_k, int B, int max_len_k,
                                        int k, int d_I) {
  if (total_q < 0 || total_k < 0 || B < 0 || max_len_k < 0 || k < 1 || k > 2048 ||
      max_len_k > dsa::kFusedMaxLenK || (d_I != 64 && d_I != 128))
    return 0;
  return fused_layout(total_q, total_k, B, max_len_k, k, d_I).total;
}

dsa_status_t dsa_forward_fused(const void* q_fp8, const float* q_scale, const float* w,
                               const void* k_fp8, const float* k_scale, const void* q,
                               const void* kv, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, int B, int max_len_q, int max_len_k,
                               int64_t total_q, int64_t total_k, int H_I, int d_I, int H, int d_qk,
                               int d_v, int k, float sm_scale, void* out, float* lse,
                               int32_t* idx_out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  dsa_status_t st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k, total_q,
                                 total_k);
  if (st != DSA_OK) return st;
  if (!q_fp8 || !q_scale || !w || !k_fp8 || !k_scale || !q || !kv || !out)
    return DSA_ERR_INVALID_ARG;
  if (!indexer_shape_ok(H_I, d_I) || H_I != 64) return DSA_ERR_UNSUPPORTED;
  if (d_qk != 576 || d_v != 512 || !mla_heads_ok(H) || k < 1 || k > 2048 ||
      max_len_k > dsa::kFusedMaxLenK)
    return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_fp8) || !aligned16(k_fp8) || (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGNMENT;
  if (total_q * H_I >= (int64_t(1) << 31) || total_k >= (int64_t(1) << 31) ||
      total_q * static_cast<int64_t>(dsa::kFusedCap) >= (int64_t(1) << 40))
    return DSA_ERR_UNSUPPORTED;
  const FusedLayout f = fused_layout(total_q, total_k, B, max_len_k, k, d_I);
  if (!workspace || workspace_bytes < f.total) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_ALIGNMENT;
  if (total_q == 0 || B == 0) return DSA_OK;
  if (total_k == 0) return DSA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != DSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* logits = reinterpret_cast<float*>(ws + f.logits);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + f.idx);
  uint8_t* k8_s = ws + f.k8_s;
  float* ks_s = reinterpret_cast<float*>(ws + f.ks_s);
  int32_t* cu_k_s = reinterpret_cast<int32_t*>(ws + f.cu_k_s);
  float* logits_s = reinterpret_cast<float*>(ws + f.logits_s);
  float* thr = reinterpret_cast<float*>(ws + f.thr);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + f.flags);
  uint32_t* row_on = cnt + total_q;
  uint32_t* any_on = row_on + total_q;
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(ws + f.cand_key);
  int32_t* cand_pos = reinterpret_cast<int32_t*>(ws + f.cand_pos);

  if (cudaMemsetAsync(ws + f.flags, 0, static_cast<size_t>(2 * total_q + 1) * 4, s) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  // 1. the sampled keys and every query's scores against them
  dsa::FusedSampleArgs sa;
  sa.k8 = static_cast<const uint8_t*>(k_fp8);
  sa.k_scale = k_scale;
  sa.cu_k = cu_seqlens_k;
  sa.B = B;
  sa.d_I = d_I;
  sa.max_samples = f.max_samples;
  sa.k8_s = k8_s;
  sa.k_scale_s = ks_s;
  sa.cu_k_s = cu_k_s;
  if ((st = from_cuda(dsa::launch_fused_sample(sa, s))) != DSA_OK) return st;
  const CUtensorMapSwizzle swz =
      d_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const int tile_n = (max_len_q <= 1 && H_I >= 16 && H_I <= 64) ? 64 : 256;
  CUtensorMap tq, tk, tk_s;
  if ((st = encode_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_fp8, total_q * H_I, d_I, 1,
                      static_cast<uint32_t>(tile_n), d_I, swz)) != DSA_OK)
    return st;
  if ((st = encode_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_fp8, total_k, d_I, 1, 128, d_I,
                      swz)) != DSA_OK)
    return st;
  if ((st = encode_2d(&tk_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, k8_s, f.max_samples, d_I, 1, 128,
                      d_I, swz)) != DSA_OK)
    return st;
  dsa::IndexerArgs ia;
  ia.q_scale = q_scale;
  ia.w = w;
  ia.k_scale = ks_s;
  ia.cu_q = cu_seqlens_q;
  ia.cu_k = cu_k_s;
  ia.B = B;
  ia.max_len_q = max_len_q;
  ia.max_len_k = static_cast<int>((max_len_k + dsa::kSampleStride - 1) / dsa::kSampleStride);
  ia.H_I = H_I;
  ia.d_I = d_I;
  ia.logits = logits_s;
  ia.ld = f.ld_s;
  ia.tile_n = tile_n;
  ia.mode = dsa::kIdxRect;
  if ((st = from_cuda(dsa::launch_indexer(tq, tk_s, ia, dev->num_sms, next_err(dev), s))) !=
      DSA_OK)
    return st;
  dsa::FusedThresholdArgs ta;
  ta.logits_s = logits_s;
  ta.ld_s = f.ld_s;
  ta.cu_q = cu_seqlens_q;
  ta.cu_k = cu_seqlens_k;
  ta.cu_k_s = cu_k_s;
  ta.B = B;
  ta.total_q = total_q;
  ta.k = k;
  ta.thr = thr;
  if ((st = from_cuda(dsa::launch_fused_threshold(ta, s))) != DSA_OK) return st;
  // 2. every causal score again, only those at or above the threshold kept
  ia.k_scale = k_scale;
  ia.cu_k = cu_seqlens_k;
  ia.max_len_k = max_len_k;
  ia.logits = logits;
  ia.ld = f.ld;
  ia.mode = dsa::kIdxCompact;
  ia.thr = thr;
  ia.cand_key = cand_key;
  ia.cand_pos = cand_pos;
  ia.cnt = cnt;
  ia.cap = dsa::kFusedCap;
  if ((st = from_cuda(dsa::launch_indexer(tq, tk, ia, dev->num_sms, next_err(dev), s))) !=
      DSA_OK)
    return st;
  dsa::TopkCandArgs ca;
  ca.cand_key = cand_key;
  ca.cand_pos = cand_pos;
  ca.cnt = cnt;
  ca.cap = dsa::kFusedCap;
  ca.cu_q = cu_seqlens_q;
  ca.cu_k = cu_seqlens_k;
  ca.B = B;
  ca.max_len_k = max_len_k;
  ca.total_q = total_q;
  ca.k = k;
  ca.idx = idx;
  ca.row_on = row_on;
  ca.any_on = any_on;
  if ((st = from_cuda(dsa::launch_topk_candidates(ca, next_err(dev), s))) != DSA_OK) return st;
  // 3. rows the candidate lists could not settle: the unfused path, on those
  // rows only (both launches return at once when there are none)
  ia.mode = dsa::kIdxCausal;
  ia.row_on = row_on;
  ia.any_on = any_on;
  if ((st = from_cuda(dsa::launch_indexer(tq, tk, ia, dev->num_sms, next_err(dev), s))) !=
      DSA_OK)
    return st;
  dsa::TopkArgs tka;
  tka.logits = logits;
  tka.ld = f.ld;
  tka.cu_q = cu_seqlens_q;
  tka.cu_k = cu_seqlens_k;
  tka.B = B;
  tka.max_len_q = max_len_q;
  tka.max_len_k = max_len_k;
  tka.total_q = total_q;
  tka.k = k;
  tka.idx = idx;
  tka.val = nullptr;
  tka.row_on = row_on;
  tka.any_on = any_on;
  if ((st = from_cuda(dsa::launch_topk(tka, next_err(dev), s))) != DSA_OK) return st;
  return dsa_sparse_mla_fwd(q, kv, idx, cu_seqlens_q, cu_seqlens_k, B, max_len_q, max_len_k,
                            total_q, total_k, H, d_qk, d_v, k, sm_scale, out, lse, stream);
}

void dsa_debug_fault_injection(uint64_t wait_limit_ns, int drop_first_key_load) {
  g_wait_limit_ns.store(wait_limit_ns);
  g_inject_indexer.store(drop_first_key_load ? dsa::kInjectDropFirstKeyLoad : 0u);
}

dsa_status_t dsa_get_device_error(void* stream) {
  DeviceInfo* dev = nullptr;
  dsa_status_t st = device_info(&dev);
  if (st != DSA_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  unsigned bits = 0;
  if (cudaMemcpyFromSymbol(&bits, g_dsa_err, sizeof(unsigned)) != cudaSuccess) return DSA_ERR_CUDA;
  if (bits == 0) return DSA_OK;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_dsa_err, &zero, sizeof(unsigned)) != cudaSuccess) return DSA_ERR_CUDA;
  if (bits & dsa::kErrTimeout) return DSA_ERR_TIMEOUT;
  return DSA_ERR_BOUNDS;
}

}  // extern "C"
