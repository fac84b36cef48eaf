/*
 * dsa.h -- C ABI of libdsa.so, the B200 (sm_100a) hot path of DeepSeek Sparse
 * Attention (DSA): lightning-indexer scores -> per-query top-k -> sparse
 * attention in the MQA mode of MLA.
 *
 * The operation, as the pages state it:
 *  - "DeepSeek V3.2 and the lightning indexer" (montana-research blog),
 *    section "How the lightning indexer works": the score of a query for an
 *    earlier token adds up, over a handful of FP8 indexer heads, ReLU-clipped
 *    dot products scaled by per-head weights; a query's 2,048 highest scores
 *    pick the entries its attention reads, and nothing else; under MLA's MQA
 *    form a latent is shared by all query heads, so one selection serves a
 *    whole query position.
 *  - "DeepSeek-V3.2" (atlas.lewiswon.me), "Design overview": token-level
 *    top-k with k = 2048, main attention cost O(L*k).
 *  - "DeepSeek-V3.2 ... (introducing DSA)" (phantomic12 paper record): the
 *    indexer gives each (query, KV) pair a single scalar and the attention
 *    reads the k best; the indexer touches the whole context, hence FP8.
 *
 * Conventions shared by every call
 * --------------------------------
 *  Pointers marked (device) are CUDA device pointers owned by the caller; the
 *  library allocates no device memory and keeps no pointer after returning.
 *  All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *  the legacy default stream) and nothing synchronises with the host, except
 *  dsa_get_device_error().
 *
 *  Varlen batches: B sequences; cu_seqlens_q / cu_seqlens_k are (device)
 *  int32 arrays of B+1 non-decreasing offsets.  Sequence b owns query rows
 *  cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key rows cu_seqlens_k[b] ..
 *  cu_seqlens_k[b+1]-1, with len_q <= len_k.  Its queries are the LAST len_q
 *  positions of the sequence: local query i sits at absolute position
 *  p = (len_k - len_q) + i and may use the sequence-local keys 0..p (causal,
 *  self included).  Prefill: len_q = len_k.  Chunked prefill: len_q = chunk,
 *  len_k = chunk end.  Decode: len_q = 1.
 *  max_len_q / max_len_k bound the per-sequence lengths; total_q / total_k
 *  are cu_seqlens_q[B] / cu_seqlens_k[B] (the caller knows them; the host
 *  code never reads device memory).
 *
 *  Layouts are row-major and contiguous unless a leading dimension is given.
 *  Every pointer must be 16-byte aligned (DSA_ERR_ALIGNMENT otherwise).
 *
 *  Errors: each call validates its arguments before launching anything and
 *  returns a status; CUDA launch errors map to DSA_ERR_CUDA.  Kernels bound
 *  every wait; a wait that runs out sets a device error word and the kernel
 *  returns early.  dsa_get_device_error() reads and clears that word.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* a size, count or pointer is out of range / NULL */
  DSA_ERR_UNSUPPORTED = 2, /* valid but outside the shapes the library supports */
  DSA_ERR_ALIGNMENT = 3,   /* a pointer or stride breaks the 16-byte rule */
  DSA_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than required */
  DSA_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed */
  DSA_ERR_TIMEOUT = 6,     /* a kernel gave up on a bounded wait */
  DSA_ERR_BOUNDS = 7       /* a kernel found an index outside its tensor */
} dsa_status_t;

/*
 * Lightning-indexer scores (blog, "How the lightning indexer works"):
 *
 *   logits[q_row, s] = k_scale[k_row] *
 *                      sum_j (w[q_row,j] * q_scale[q_row,j]) * ReLU(q8[q_row,j,:] . k8[k_row,:])
 *
 * for every causal pair (s <= p), where q_row is the global query row, s the
 * sequence-local key position and k_row = cu_seqlens_k[b] + s.  This equals
 * sum_j w * ReLU(qhat . khat) on the dequantised vectors qhat = q8 * q_scale,
 * khat = k8 * k_scale whenever the scales are positive.
 *
 *  q_fp8    (device) e4m3 bytes [total_q, H_I, d_I]
 *  q_scale  (device) f32 [total_q, H_I]   (> 0; a per-token scale is replicated)
 *  w        (device) f32 [total_q, H_I]   indexer head weights (any sign)
 *  k_fp8    (device) e4m3 bytes [total_k, d_I]  (one head, shared by all H_I)
 *  k_scale  (device) f32 [total_k]        (> 0)
 *  logits   (device) f32, row q_row at logits + q_row * ld_logits, column s;
 *           ld_logits >= max_len_k and a multiple of 4.  Only entries with
 *           s <= p are written; the rest are left untouched.
 *  Supported: d_I in {64, 128}; H_I in {4, 8, 16, 32, 64, 128}.
 *  Arithmetic: FP8 products accumulated by the tensor core, fp32 epilogue.
 */
DSA_API dsa_status_t dsa_indexer_logits(const void* q_fp8, const float* q_scale, const float* w,
                                const void* k_fp8, const float* k_scale,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                                int max_len_q, int max_len_k, int64_t total_q, int64_t total_k,
                                int H_I, int d_I, float* logits, int64_t ld_logits, void* stream);

/*
 * Per-query top-k (blog, "How the lightning indexer works"; atlas,
 * "Design overview": token-level selection of the k best entries per query).
 *
 * For each query row, reads logits[q_row, 0..p] and writes to idx_out[q_row,
 * 0..k) the sequence-local positions of the min(k, p+1) largest scores in
 * ascending position order, padded with -1.  Ties go to the lower position;
 * -0.0 and +0.0 are equal.  NaN scores are not supported.
 *
 *  logits   (device) f32, layout as produced by dsa_indexer_logits (16-byte
 *           aligned, ld_logits a multiple of 4, else DSA_ERR_ALIGNMENT)
 *  idx_out  (device) int32 [total_q, k]
 *  val_out  (device, nullable) f32 [total_q, k]: the selected scores (NaN in
 *           padding slots)
 *  Supported: 1 <= k <= 4096, max_len_k <= 2^24.
 */
DSA_API dsa_status_t dsa_topk(const float* logits, int64_t ld_logits, const int32_t* cu_seqlens_q,
                      const int32_t* cu_seqlens_k, int B, int max_len_q, int max_len_k,
                      int64_t total_q, int k, int32_t* idx_out, float* val_out, void* stream);

/*
 * Sparse attention in the MQA mode of MLA (blog, "How the lightning indexer
 * works": each selected latent is shared by all query heads; atlas,
 * "Inference efficiency": attention touches only the selected latents).
 *
 *   out[q_row, h, :] = sum_{s in S} softmax_s(sm_scale * q[q_row,h,:] . kv[k_row(s),:])
 *                                  * kv[k_row(s), 0:d_v]
 *   lse[q_row, h]    = log sum_{s in S} exp(sm_scale * q[q_row,h,:] . kv[k_row(s),:])
 *
 * S is the set of entries among the FIRST min(k, p+1) of idx[q_row, :] that
 * satisfy 0 <= s <= p; other entries are skipped (dsa_topk fills exactly that
 * prefix).  A row with an empty S gets out = 0 and lse = -inf.
 *
 *  q        (device) bf16 [total_q, H, d_qk]
 *  kv       (device) bf16 [total_k, d_qk]; the first d_v dims are the value
 *  idx      (device) int32 [total_q, k]
 *  out      (device) bf16 [total_q, H, d_v]
 *  lse      (device, nullable) f32 [total_q, H] (natural log)
 *  Supported: d_qk = 576, d_v = 512, H in {16, 32} or a multiple of 64 up to
 *  256, 1 <= k <= 4096.
 *  Arithmetic: bf16 tensor-core products, fp32 accumulation and softmax.
 */
DSA_API dsa_status_t dsa_sparse_mla_fwd(const void* q, const void* kv, const int32_t* idx,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                                int max_len_q, int max_len_k, int64_t total_q, int64_t total_k,
                                int H, int d_qk, int d_v, int k, float sm_scale, void* out,
                                float* lse, void* stream);

/*
 * The whole path on one stream: dsa_indexer_logits -> dsa_topk ->
 * dsa_sparse_mla_fwd, with the scores and indices kept in the caller's
 * workspace (size from dsa_forward_workspace_size).  idx_out (nullable)
 * receives a copy of the selected indices [total_q, k].
 */
DSA_API dsa_status_t dsa_forward(const void* q_fp8, const float* q_scale, const float* w,
                         const void* k_fp8, const float* k_scale, const void* q, const void* kv,
                         const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B,
                         int max_len_q, int max_len_k, int64_t total_q, int64_t total_k, int H_I,
                         int d_I, int H, int d_qk, int d_v, int k, float sm_scale, void* out,
                         float* lse, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * Device workspace bytes for dsa_forward_fused (0 for unsupported sizes:
 * k > 2048, max_len_k > 131072, d_I not 64 or 128).
 */
DSA_API size_t dsa_forward_fused_workspace_size(int64_t total_q, int64_t total_k, int B,
                                                int max_len_k, int k, int d_I);

/*
 * dsa_forward with the indexer and the top-k fused into two passes over the
 * keys, so the causal score matrix is not written to HBM and read back (blog,
 * "What we would test": at long context the indexer's quadratic term is the
 * cost that remains).  Same arguments, same results: idx, out and lse equal
 * dsa_forward's bit for bit.
 *
 *  1. Every query is scored against a 1/32 sample of its sequence's keys
 *     (positions 0, 32, 64, ...), and each row's threshold is the r0-th
 *     largest score among the S samples it may see, r0 = E + 4 sqrt(E) + 8
 *     with E = S k / (p + 1); rows of at most 4096 scores keep every score.
 *  2. Every causal score is computed again (the same arithmetic as
 *     dsa_indexer_logits) and only those at or above the row's threshold are
 *     appended to the row's list of at most 5120 candidates.
 *  3. A row with at least k candidates (and no more than the list holds) has
 *     all of its k best scores in the list, ties included, and is selected
 *     from it.  Any other row, and a row of massive ties, is recomputed on the
 *     unfused path (dsa_indexer_logits and dsa_topk on those rows only).
 *  4. dsa_sparse_mla_fwd on the indices.
 *
 *  workspace (device) dsa_forward_fused_workspace_size bytes, 16-byte aligned:
 *           the sampled keys and their scores, thresholds, candidate lists,
 *           and a full score matrix that only the recomputed rows touch.
 *  Supported: as dsa_forward with H_I = 64, k <= 2048 and max_len_k <= 131072.
 *  Errors: as dsa_forward; DSA_ERR_WORKSPACE for a missing or short workspace.
 */
DSA_API dsa_status_t dsa_forward_fused(const void* q_fp8, const float* q_scale, const float* w,
                                       const void* k_fp8, const float* k_scale, const void* q,
                                       const void* kv, const int32_t* cu_seqlens_q,
                                       const int32_t* cu_seqlens_k, int B, int max_len_q,
                                       int max_len_k, int64_t total_q, int64_t total_k, int H_I,
                                       int d_I, int H, int d_qk, int d_v, int k, float sm_scale,
                                       void* out, float* lse, int32_t* idx_out, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * dsa_forward for callers that cannot allocate device memory.  The pages have
 * no counterpart to this call; it exists for users of this library.
 *
 * Some callers can't call cudaMalloc: a serving engine that reserves the whole
 * device for its own pool up front, or a latency-critical loop that cannot take
 * the device synchronisation an allocation brings.  They pass inputs and
 * outputs as for dsa_forward but no workspace: the scores and indices live in
 * one fixed device array of 48 MiB per GPU inside the library (held from when
 * the library's device code loads on that GPU until the process exits).
 *
 *  - Returns DSA_ERR_WORKSPACE, without launching anything, when
 *    dsa_forward_workspace_size(total_q, max_len_k, k) exceeds 48 MiB
 *    (e.g. 64 decode queries over 131072-token caches with k = 2048 fit;
 *    a 32768-token prefill does not).
 *  - The first call on a device looks up the array's device address with that
 *    device current; make that first call before any stream capture.
 *  - All calls share the array and leave their data in it; nothing in it
 *    needs to start at zero.  Calls that overlap on the GPU (e.g. on two
 *    streams at once) race on it and must be serialised by the caller.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Other arguments, results and errors are those of dsa_forward.
 */
DSA_API dsa_status_t dsa_forward_noalloc(const void* q_fp8, const float* q_scale, const float* w,
                                         const void* k_fp8, const float* k_scale, const void* q,
                                         const void* kv, const int32_t* cu_seqlens_q,
                                         const int32_t* cu_seqlens_k, int B, int max_len_q,
                                         int max_len_k, int64_t total_q, int64_t total_k, int H_I,
                                         int d_I, int H, int d_qk, int d_v, int k, float sm_scale,
                                         void* out, float* lse, int32_t* idx_out, void* stream);

/*
 * dsa_forward with every input and output in HOST memory: the call copies
 * what the path needs to the GPU, runs it and copies the results back, and
 * returns when `out` and `lse` hold them.  The method's statement (each
 * query's scores, selection and attention read only that query's row and the
 * key-side tensors: "DeepSeek V3.2 and the lightning indexer", section "How
 * the lightning indexer works") lets the query rows go through in chunks of
 * `chunk_q` rows: the key-side tensors (k_fp8, k_scale, kv) are copied once,
 * and chunk c is uploaded, computed and downloaded on streams[c % n_streams],
 * so copies of one chunk overlap the kernels of another.  Results are
 * bitwise those of dsa_forward on the same inputs.
 *
 *  - Every pointer argument except `workspace` and `streams` is a host
 *    pointer, with the layouts of dsa_forward; cu_seqlens_q/k are host
 *    arrays [B+1] that start at 0 and end at total_q / total_k.  Page-locked
 *    (pinned) host memory is needed for the copies to overlap; pageable
 *    memory works but serialises them.
 *  - `workspace`: device memory, 256-byte aligned, of at least
 *    dsa_forward_host_workspace_size(total_k, max_len_k, B, H_I, d_I, H, k,
 *    chunk_q, n_streams) bytes, owned by the caller.
 *  - `streams`: n_streams >= 1 CUDA streams owned by the caller (streams[0]
 *    carries the one-time key copies; the others wait for them).  The call
 *    synchronises all of them before it returns.
 *  - lse may be NULL.  Errors as dsa_forward, plus DSA_ERR_INVALID_ARG for
 *    cu_seqlens that do not describe the batch.
 */
DSA_API dsa_status_t dsa_forward_host(const void* q_fp8, const float* q_scale, const float* w,
                                      const void* k_fp8, const float* k_scale, const void* q,
                                      const void* kv, const int32_t* cu_seqlens_q,
                                      const int32_t* cu_seqlens_k, int B, int max_len_q,
                                      int max_len_k, int64_t total_q, int64_t total_k, int H_I,
                                      int d_I, int H, int d_qk, int d_v, int k, float sm_scale,
                                      void* out, float* lse, int chunk_q, void* workspace,
                                      size_t workspace_bytes, void* const* streams, int n_streams);

/* Device workspace bytes for dsa_forward_host: the key-side tensors once, and
 * per stream one chunk's query rows, outputs and dsa_forward workspace.
 * Returns 0 for invalid sizes. */
DSA_API size_t dsa_forward_host_workspace_size(int64_t total_k, int max_len_k, int B, int H_I,
                                               int d_I, int H, int k, int chunk_q, int n_streams);

/*
 * The indexer's training signal ("DeepSeek V3.2 and the lightning indexer",
 * section "Teaching a dense model to be sparse": the indexer's scores are
 * fitted to the main attention's distribution by minimising a KL divergence;
 * "DeepSeek-V3.2" atlas entry, "Design overview": the target is the head-wise
 * attention distribution summed over heads).  For each query row t with valid
 * selected entries S (idx[t, j] with 0 <= idx <= p, j < min(k, p+1)):
 *   target p[t,s] = (1/H) sum_h exp(sm_scale * q[t,h,:] . kv[s,:] - lse[t,h]),
 *   q_I[t,s]      = softmax over S of logits[t, s],
 *   kl_out[t]     = sum_{s in S} p (log p - log q_I),
 *   grad_out[t,j] = q_I[t,s] - p[t,s]  (the gradient of kl_out[t] with respect
 *                   to logits[t,s], s = idx[t,j]); 0 at invalid entries,
 *   target_out[t,j] = p[t,s]; 0 at invalid entries.
 * Over all causal keys (k >= every p+1) this is the dense warm-up's loss.
 *  - q [total_q, H, d_qk] bf16 and kv [total_k, d_qk] bf16 as for
 *    dsa_sparse_mla_fwd (d_qk = 576); idx [total_q, k] int32 as dsa_topk
 *    writes it; lse [total_q, H] f32, natural-log log-sum-exp of each head's
 *    attention scores over the selection (dsa_sparse_mla_fwd's lse output);
 *    logits [total_q, ld_logits] f32 indexer scores, row = query, column =
 *    sequence-local key (dsa_indexer_logits' output).
 *  - kl_out [total_q] f32; grad_out and target_out [total_q, k] f32, nullable.
 *  - workspace: device memory of dsa_indexer_kl_workspace_size(total_q, H, k)
 *    bytes, 16-byte aligned, owned by the caller.
 * Errors as dsa_sparse_mla_fwd.
 */
DSA_API dsa_status_t dsa_indexer_kl(const void* q, const void* kv, const int32_t* idx,
                                    const float* lse, const float* logits, int64_t ld_logits,
                                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                    int B, int max_len_q, int max_len_k, int64_t total_q,
                                    int64_t total_k, int H, int d_qk, int k, float sm_scale,
                                    float* kl_out, float* grad_out, float* target_out,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Device workspace bytes for dsa_indexer_kl: four partial-sum slices of
 * [total_q, k] f32 per group of 128 heads.  Returns 0 for invalid sizes. */
DSA_API size_t dsa_indexer_kl_workspace_size(int64_t total_q, int H, int k);

/*
 * The indexer's backward ("DeepSeek V3.2 and the lightning indexer", section
 * "Teaching a dense model to be sparse": in the warm-up only the indexer is
 * trained, on the KL signal its scores get; dsa_indexer_kl gives the gradient
 * of that loss with respect to the scores).  With qhat = q8 * q_scale and
 * khat = k8 * k_scale (dequantised) and the scores
 *   I[t,s] = sum_j w[t,j] * ReLU(qhat[t,j,:] . khat[s,:]),   s <= p(t),
 * and an upstream gradient g[t,s] = dL/dI[t,s], it writes
 *   dq[t,j,:] = dL/dqhat[t,j,:] = w[t,j] * sum_s g[t,s] [qhat.khat > 0] khat[s,:]
 *   dw[t,j]   = dL/dw[t,j]      = sum_s g[t,s] ReLU(qhat[t,j,:] . khat[s,:])
 *   dk[s,:]   = dL/dkhat[s,:]   = sum_{t,j} g[t,s] [qhat.khat > 0] w[t,j] qhat[t,j,:]
 * (gradients with respect to the dequantised values: the quantisation is
 * passed straight through; the ReLU's derivative is taken as 0 at 0).
 *
 *  q_fp8, q_scale, w, k_fp8, k_scale: as for dsa_indexer_logits (device)
 *  g        (device) f32 [total_q, ld_g], row = query, column = sequence-local
 *           key; entries past p are ignored.  ld_g >= max_len_k, multiple of 4.
 *  dq       (device) f32 [total_q, H_I, d_I]; dw (device) f32 [total_q, H_I];
 *  dk       (device) f32 [total_k, d_I] (overwritten: the call zeroes it, then
 *           adds every query's share; keys no query sees get 0).
 *  Supported: H_I = 64, d_I = 128.
 *  Arithmetic: the gates from the FP8 tensor-core products; the gated sums on
 *  the bf16 tensor cores (gradient, scales and weights folded into one bf16
 *  operand, the e4m3 codes exact in the other), fp32 accumulation.
 */
DSA_API dsa_status_t dsa_indexer_backward(const void* q_fp8, const float* q_scale,
                                          const float* w, const void* k_fp8,
                                          const float* k_scale, const float* g, int64_t ld_g,
                                          const int32_t* cu_seqlens_q,
                                          const int32_t* cu_seqlens_k, int B, int max_len_q,
                                          int max_len_k, int64_t total_q, int64_t total_k,
                                          int H_I, int d_I, float* dq, float* dw, float* dk,
                                          void* stream);

/*
 * The masked MHA mode ("DeepSeek-V3.2" atlas entry, "Design overview" and
 * "Inference efficiency": short prompts are prefilled with a masked MHA
 * standing in for DSA; the pages give no
 * detail, so it is read as dense attention in the MHA form of MLA -- per-head
 * keys and values -- restricted by a mask to each query's selected set):
 *
 *   out[q_row, h, :] = sum_{s in S} softmax_s(sm_scale * q[q_row,h,:] . k[k_row(s),h,:])
 *                                   * v[k_row(s), h, :]
 *   lse[q_row, h]    = log sum_{s in S} exp(sm_scale * q[q_row,h,:] . k[k_row(s),h,:])
 *
 * S is the SET of entries among the first min(topk, p+1) of idx[q_row, :]
 * with 0 <= s <= p (a repeated entry counts once); keys are visited densely,
 * so the cost is that of causal attention, whatever S holds.  A row with an
 * empty S gets out = 0 and lse = -inf.
 *
 *  q        (device) bf16 [total_q, H, 192]: 128 dims + 64 RoPE dims per head
 *  k        (device) bf16 [total_k, H, 192]
 *  v        (device) bf16 [total_k, H, 128]
 *  idx      (device) int32 [total_q, topk] (dsa_topk's output fits)
 *  out      (device) bf16 [total_q, H, 128]
 *  lse      (device, nullable) f32 [total_q, H] (natural log)
 *  workspace (device) dsa_masked_mha_workspace_size bytes: the selection as a
 *           bitmask, rebuilt by every call
 *  Supported: d_qk = 192, d_v = 128, 1 <= H <= 65535, 1 <= topk <= 131072,
 *  max_len_k <= 131072.
 *  Arithmetic: bf16 tensor-core products, fp32 accumulation and softmax.
 */
DSA_API dsa_status_t dsa_masked_mha_fwd(const void* q, const void* k, const void* v,
                                        const int32_t* idx, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int B, int max_len_q,
                                        int max_len_k, int64_t total_q, int64_t total_k, int H,
                                        int d_qk, int d_v, int topk, float sm_scale, void* out,
                                        float* lse, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* Device workspace bytes for dsa_masked_mha_fwd (0 for invalid sizes). */
DSA_API size_t dsa_masked_mha_workspace_size(int64_t total_q, int max_len_k);

/* Bytes of workspace dsa_forward needs: an f32 score matrix [total_q,
 * round_up(max_len_k, 4)] plus an int32 index matrix [total_q, k], each
 * 256-byte aligned.  Returns 0 for invalid sizes. */
DSA_API size_t dsa_forward_workspace_size(int64_t total_q, int max_len_k, int k);

/* Static text for a status code (never NULL). */
DSA_API const char* dsa_status_string(dsa_status_t status);

/* Synchronises `stream`, then reads and clears the device error word that
 * the kernels set on a timed-out wait (DSA_ERR_TIMEOUT) or a bounds failure
 * (DSA_ERR_BOUNDS).  Returns DSA_OK if it was clear. */
DSA_API dsa_status_t dsa_get_device_error(void* stream);

/*
 * Test hook for the failure detection of the kernels (not for production
 * use; the pages have no counterpart).  Every wait inside a kernel is bounded:
 * a wait that runs out records DSA_ERR_TIMEOUT in the device error word and
 * the kernel winds down and returns, leaving the CUDA context usable.  This
 * call lets a test exercise that path without faulting anything:
 *  - wait_limit_ns: the longest a single wait may take in launches made
 *    after this call (0 restores the default of 2 s);
 *  - drop_first_key_load != 0: the NEXT dsa_indexer_logits launch (only that
 *    one) leaves out the first key-tile load of every CTA, so the MMA
 *    issuer's wait for that tile runs out; that launch's scores are then
 *    incomplete and dsa_get_device_error() returns DSA_ERR_TIMEOUT.
 * Process-wide host state, not thread-safe against concurrent launches.
 */
DSA_API void dsa_debug_fault_injection(uint64_t wait_limit_ns, int drop_first_key_load);

/* Library version, "major.minor.patch". */
DSA_API const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
