// Launchers of the libbgtq kernels (host side), called by the ABI layer after it has
// validated every argument.
#pragma once

#include <cuda_runtime.h>

#include "bgtq_internal.h"

namespace bgtq {

// Plan of one decode call: the units' caches (batch rows x KV heads, max_tiles 64-token
// tiles each) are one sequence of T tiles; CTA c takes tiles [c T / n_ctas, (c+1) T /
// n_ctas) (at most tiles_per_cta, never more than one unit long); a unit meets at most
// n_parts slices, each leaving one partial result.
struct DecodePlan {
  int max_tiles;        // ceil(max_seq_len / 64)
  int tiles_per_cta;
  int n_ctas;
  int n_parts;
  size_t workspace_bytes;
};

// ctas_per_sm <= 0: the most split CTAs that fit an SM (the workspace of any launch plan).
DecodePlan plan_decode(int batch, int h_q, int h_kv, long long max_seq_len, int num_sms, int ctas_per_sm = 0);

// heads (device array of h_kv layouts, or null): KV head h is coded with heads[h] (every
// layout of the array has the same value rate, norm options and tile stride L.tile_bytes;
// L is heads[0] as the host sees it).
cudaError_t launch_tq_encode(const DevLayout& L, const void* k, const void* v, int dtype, int batch,
                             int n_new, int h_kv, const int* seq_lens, const CacheRef& cache, cudaStream_t stream,
                             const DevLayout* heads = nullptr);

// n_q query tokens per row (q [batch][n_q][h_q][128], out likewise), causal among them;
// the plan is made for h_q n_q query columns.
cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, int n_q, const CacheRef& cache, const int* seq_lens, float softmax_scale,
                          float* out, void* workspace, cudaStream_t stream, float* rec = nullptr,
                          const DevLayout* heads = nullptr);

// Merge of partial records over disjoint token ranges: recs [n_rec][columns][130]
// (m, l, o' of each query column), out [columns][128] = R_V^T (log-sum-exp merge of o').
cudaError_t launch_merge_records(const DevLayout& L, const float* recs, int n_rec, long long columns, float* out,
                                 cudaStream_t stream);

// Append n_new tokens at seq_lens_before[b] and attend over seq_lens_before[b] + n_new
// tokens: the encode kernel, then the split kernel as its programmatic dependent (only the
// tile receiving the new tokens waits for the encode), then the combine. n_q = 1: one
// query per row at the newest position; n_q = n_new: the new tokens' own queries.
cudaError_t launch_decode_step(const DevLayout& L, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, int n_new, const int* seq_lens_before, const void* q, int q_dtype,
                               int batch, int h_q, int h_kv, int n_q, const CacheRef& cache, float softmax_scale,
                               float* out, void* workspace, cudaStream_t stream, const DevLayout* heads = nullptr);

// Logits only: scores[(b h_q + hq) scores_ld + t] = softmax_scale q . k_hat_t for every
// cached token t < seq_lens[b] (the q-preparation kernel, then the split kernel in its
// scores-only form).
cudaError_t launch_scores(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch, int h_q,
                          int h_kv, const CacheRef& cache, const int* seq_lens, float softmax_scale, float* scores,
                          long long scores_ld, void* workspace, cudaStream_t stream, const DevLayout* heads = nullptr);

}  // namespace bgtq
