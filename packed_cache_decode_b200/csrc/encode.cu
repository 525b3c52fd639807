// tq_encode: TQ-MSE encode-append kernel (device code in encode_body.cuh).
#include <cuda_runtime.h>

#include "bgtq_internal.h"
#include "encode_body.cuh"
#include "kernels.h"

namespace bgtq {

namespace {

template <bool NC>
__global__ void __launch_bounds__(enc::kEncodeThreads) tq_encode_kernel(DevLayout L, const void* __restrict__ k,
                                                                        const void* __restrict__ v, int dtype,
                                                                        int n_new, int h_kv,
                                                                        const int* __restrict__ seq_lens, CacheRef cache) {
  // a split kernel launched as this kernel's programmatic dependent may start streaming
  // the tiles that do not receive the new tokens (it waits before the one that does)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  enc::encode_token_part<NC>(L, k, v, dtype, n_new, h_kv, seq_lens, cache, blockIdx.x / kEncodeParts,
                         blockIdx.x % kEncodeParts, blockIdx.y, blockIdx.z);
}

}  // namespace

cudaError_t launch_tq_encode(const DevLayout& L, const void* k, const void* v, int dtype, int batch,
                             int n_new, int h_kv, const int* seq_lens, const CacheRef& cache, cudaStream_t stream) {
  dim3 grid(n_new * kEncodeParts, batch, h_kv);
  if (!L.norm_correct) {
    tq_encode_kernel<false><<<grid, enc::kEncodeThreads, 0, stream>>>(L, k, v, dtype, n_new, h_kv, seq_lens, cache);
    return cudaGetLastError();
  }
  // norm correction: the four parts of a token form one cluster (they exchange sums)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(enc::kEncodeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kEncodeParts;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tq_encode_kernel<true>, L, k, v, dtype, n_new, h_kv, seq_lens, cache);
}

}  // namespace bgtq
