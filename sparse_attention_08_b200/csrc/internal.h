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
  // What the read-out does with a score (kIdxCausal unless set):
  //  kIdxCausal   store the causal scores (key s <= the query's position p);
  //  kIdxRect     store every key's score of the sequence (no causal mask);
  //  kIdxCompact  append (order key, position) of every causal score >= thr[row]
  //               to the row's list of cap entries, counting all of them in cnt.
  int mode = 0;
  const float* thr = nullptr;
  uint32_t* cand_key = nullptr;
  int32_t* cand_pos = nullptr;
  uint32_t* cnt = nullptr;
  int cap = 0;
  // Rows to compute (non-zero entries; null = every row): items without such
  // a row are skipped, and the launch does nothing while *any_on is 0.
  const uint32_t* row_on = nullptr;
  const uint32_t* any_on = nullptr;
};

enum { kIdxCausal = 0, kIdxRect = 1, kIdxCompact = 2 };

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
  // Rows to select (non-zero entries; null = every row); the launch does
  // nothing while *any_on is 0.
  const uint32_t* row_on = nullptr;
  const uint32_t* any_on = nullptr;
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

// ---- fused indexer + top-k (two passes over the keys)
constexpr int kFusedCap = 5120;          // candidate list entries per row
constexpr int kFusedMaxLenK = 131072;    // longest key prefix (position bitmap size)
constexpr int kSampleStride = 32;        // a sequence's keys 0, 32, 64, ... are sampled
constexpr int kFusedAllPass = 4096;      // rows of at most this many scores keep them all

struct TopkCandArgs {
  const uint32_t* cand_key;
  const int32_t* cand_pos;
  const uint32_t* cnt;
  int cap;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int B, max_len_k;
  int64_t total_q;
  int k;
  int32_t* idx;
  uint32_t* row_on;   // out: rows left to the unfused path
  uint32_t* any_on;   // out: set when any row is
};
cudaError_t launch_topk_candidates(const TopkCandArgs& a, DevErr err, cudaStream_t s);

struct FusedSampleArgs {
  const uint8_t* k8;        // [total_k, d_I]
  const float* k_scale;     // [total_k]
  const int32_t* cu_k;      // [B + 1]
  int B, d_I;
  int64_t max_samples;      // rows of the sample buffers
  uint8_t* k8_s;            // out [max_samples, d_I]
  float* k_scale_s;         // out [max_samples]
  int32_t* cu_k_s;          // out [B + 1]
};
cudaError_t launch_fused_sample(const FusedSampleArgs& a, cudaStream_t s);

struct FusedThresholdArgs {
  const float* logits_s;    // [total_q, ld_s]: scores against the sampled keys
  int64_t ld_s;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* cu_k_s;
  int B;
  int64_t total_q;
  int k;
  float* thr;               // out [total_q]
};
cudaError_t launch_fused_threshold(const FusedThresholdArgs& a, cudaStream_t s);
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
