// forward_noalloc.cu -- dsa_forward for callers that cannot allocate device
// memory.
//
// Some callers of this library can't call cudaMalloc.  A serving engine that
// reserves the whole device up front for its own memory pool has no room left
// for an allocation it did not plan, and a cudaMalloc from inside the library
// would fail or break the pool's accounting.  A latency-critical loop (a
// decode step) cannot afford the implicit device synchronisation a cudaMalloc
// or cudaFree brings.  Such callers already own the inputs and outputs, but
// they have no buffer to lend for the path's scratch: the score matrix and
// the selected indices that dsa_forward keeps between its three stages.
//
// dsa_forward_noalloc therefore keeps that scratch in a fixed, file-scope
// device array (kScratchBytes per GPU).  Each GPU on which this library's
// device code is loaded holds the array until the process exits.  Host code
// never passes the array's name to a kernel (in host code that name is only a
// stand-in, not a device address): the first call on a device, with that
// device current, asks the runtime for the array's device address once, and
// every later call on that device reuses it.  Make that first call before any
// stream capture.
//
// Every call shares the one array and leaves its contents behind.  Nothing in
// it needs to start at zero: each stage writes every entry the next one reads.
// Calls that overlap on the GPU (for example on two streams at once) race on
// the array and must be serialised by the caller.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "dsa.h"

namespace {

// 48 MiB: for example a varlen decode batch of 64 sequences with caches of up
// to 131072 tokens and k = 2048 (32.5 MiB), or a prefill of 2048 tokens.
constexpr size_t kScratchBytes = size_t(48) << 20;

static __device__ __align__(256) unsigned char g_forward_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once
// per device, with that device current).
dsa_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_forward_scratch) != cudaSuccess || p == nullptr)
      return DSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" DSA_API dsa_status_t dsa_forward_noalloc(
    const void* q_fp8, const float* q_scale, const float* w, const void* k_fp8,
    const float* k_scale, const void* q, const void* kv, const int32_t* cu_seqlens_q,
    const int32_t* cu_seqlens_k, int B, int max_len_q, int max_len_k, int64_t total_q,
    int64_t total_k, int H_I, int d_I, int H, int d_qk, int d_v, int k, float sm_scale, void* out,
    float* lse, int32_t* idx_out, void* stream) {
  // Refuse work whose scratch would not fit before touching the device.
  if (dsa_forward_workspace_size(total_q, max_len_k, k) > kScratchBytes)
    return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const dsa_status_t st = scratch_address(&scratch);
  if (st != DSA_OK) return st;
  return dsa_forward(q_fp8, q_scale, w, k_fp8, k_scale, q, kv, cu_seqlens_q, cu_seqlens_k, B,
                     max_len_q, max_len_k, total_q, total_k, H_I, d_I, H, d_qk, d_v, k, sm_scale,
                     out, lse, idx_out, scratch, kScratchBytes, stream);
}
