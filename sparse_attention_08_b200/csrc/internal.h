// internal.h -- launchers shared between the C-ABI layer (api.cu) and the
// kernel translation units.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx.cuh"

namespace dsa {

struct IndexerArgs {
  const float* q_scale;
  const float* w;
  const float* k_scale;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, max_len_q, max_len_k;
  int H_I, d_I;
  float* logits;
  int64_t ld;
  int tile_n;   // MMA N of a tile: 256 (four queries x 64 heads) or 64 (decode)
};

struct TopkArgs {
  const float* logits;
  int64_t ld;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, max_len_q, max_len_k;
  int64_t total_q;
  int k;
  int32_t* idx;
  float* val;
};

struct MlaArgs {
  const int32_t* idx;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, max_len_q, max_len_k;
  int64_t total_q, total_k;
  int H, k;
  float sm_scale;
  void* out;
  float* lse;
  int num_sms;   // persistent grid size
};

struct KlArgs {
  const void* q;
  const void* kv;
  const int32_t* idx;
  const float* lse;
  const float* logits;
  int64_t ld;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B;
  int64_t total_q;
  int H, k;
  float sm_scale;
  float* kl;
  float* grad;     // nullable
  float* target;   // nullable
  float* part;     // workspace: per-(head group, sub-partition) partial sums
  int num_sms;
};

// Each returns cudaSuccess or the launch error.
cudaError_t launch_indexer(const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const IndexerArgs& a, int num_sms, DevErr err, cudaStream_t s);
cudaError_t launch_topk(const TopkArgs& a, DevErr err, cudaStream_t s);
cudaError_t launch_sparse_mla(const void* q, const void* kv, const MlaArgs& a, DevErr err,
                              cudaStream_t s);
cudaError_t launch_indexer_kl(const KlArgs& a, DevErr err, cudaStream_t s);

struct MaskedMhaArgs {
  const int32_t* idx;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, max_len_q, max_len_k;
  int64_t total_q, total_k;
  int H, k;
  float sm_scale;
  uint32_t* mask;   // workspace: [total_q, masked_mha_workspace_bytes / total_q / 4] words
  void* out;
  float* lse;
};

struct IndexerBwdArgs {
  const float* g;        // [total_q, ldg] upstream gradient of the scores
  int64_t ldg;
  const float* w;
  const float* q_scale;
  const float* k_scale;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, max_len_q, max_len_k;
  int64_t total_k;
  float* dq;             // [total_q, 64, 128]
  float* dw;             // [total_q, 64]
  float* dk;             // [total_k, 128], zeroed by the launcher first
};

cudaError_t launch_indexer_bwd(const CUtensorMap& tq, const CUtensorMap& tk,
                               const IndexerBwdArgs& a, DevErr err_q, DevErr err_k,
                               cudaStream_t s);

cudaError_t launch_masked_mha(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const MaskedMhaArgs& a, DevErr err, cudaStream_t s);
size_t masked_mha_workspace_bytes(int64_t total_q, int max_len_k);
size_t indexer_kl_workspace_bytes(int64_t total_q, int H, int k);

}  // namespace dsa
