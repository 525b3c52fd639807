// Launchers of the libbgtq kernels (host side), called by the ABI layer after it has
// validated every argument.
#pragma once

#include <cuda_runtime.h>

#include "bgtq_internal.h"

namespace bgtq {

// Split-K plan of one decode call: the cache of each (batch row, KV head) is cut into
// n_splits ranges of tiles_per_split 64-token tiles.
struct DecodePlan {
  int max_tiles;        // ceil(max_seq_len / 64)
  int tiles_per_split;
  int n_splits;
  size_t workspace_bytes;
};

DecodePlan plan_decode(int batch, int h_q, int h_kv, long long max_seq_len, int num_sms);

cudaError_t launch_tq_encode(const DevLayout& L, const void* k, const void* v, int dtype, int batch,
                             int n_new, int h_kv, const int* seq_lens, void* cache, long long n_tiles,
                             cudaStream_t stream);

cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, const void* cache, const int* seq_lens, long long n_tiles,
                          float softmax_scale, float* out, void* workspace, cudaStream_t stream);

// Append n_new tokens at seq_lens_before[b] and attend over seq_lens_before[b] + n_new
// tokens, as one chain of three kernels (append + q preparation, split, combine).
cudaError_t launch_decode_step(const DevLayout& L, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, int n_new, const int* seq_lens_before, const void* q, int q_dtype,
                               int batch, int h_q, int h_kv, void* cache, long long n_tiles, float softmax_scale, float* out, void* workspace,
                               cudaStream_t stream);

}  // namespace bgtq
