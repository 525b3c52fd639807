// tq_encode: TQ-MSE encode of new key/value vectors and append into the packed cache.
//
// "TurboQuant: paper algorithm and vLLM engineering implementation" (pipeline diagram):
// input vector x (per-head K or V) -> seeded random rotation -> per-coordinate scalar
// quantisation against a few centroids. "Block-GTQ" abstract, sentence 5: equal-rate RoPE
// blocks are grouped and each group is TQ-MSE coded.
//
// One CTA of 128 threads codes one (token, KV head). Every decision (norm, rotation,
// threshold comparison) is taken in fp64 so that the codes agree with an fp64 reading of
// the method except for values within rounding distance of a threshold.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "bgtq_internal.h"
#include "kernels.h"

namespace bgtq {

namespace {

__device__ __forceinline__ double load_elem(const void* p, int dtype, size_t i) {
  if (dtype == BGTQ_F32) return double(static_cast<const float*>(p)[i]);
  if (dtype == BGTQ_BF16) return double(__bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]));
  return double(__half2float(static_cast<const __half*>(p)[i]));
}

// Position of token j (0..15) inside a 16-token row of packed V codes.
__device__ __forceinline__ int chunk_slot(int j) { return 4 * ((j & 7) >> 1) + 2 * (j >> 3) + (j & 1); }

__device__ __forceinline__ int quantize(double y, const double* thr, int rate) {
  int code = 0;
  const int nthr = (1 << rate) - 1;
  for (int m = 0; m < nthr; ++m) code += (y >= thr[m]) ? 1 : 0;
  return code;
}

// Sets `width` bits at bit offset `bit` of a little-endian word array to `val`, leaving
// the other bits alone (other tokens' codes share these words, possibly concurrently).
__device__ __forceinline__ void put_bits_atomic(unsigned* words, int bit, unsigned val, int width) {
  const unsigned mask = (1u << width) - 1u;
  const int w = bit >> 5, sh = bit & 31;
  atomicAnd(&words[w], ~(mask << sh));
  atomicOr(&words[w], (val & mask) << sh);
  if (sh + width > 32) {
    const int s2 = 32 - sh;
    atomicAnd(&words[w + 1], ~(mask >> s2));
    atomicOr(&words[w + 1], (val & mask) >> s2);
  }
}

__global__ void __launch_bounds__(128) tq_encode_kernel(DevLayout L, const void* __restrict__ k,
                                                        const void* __restrict__ v, int dtype, int n_new,
                                                        int h_kv, const int* __restrict__ seq_lens,
                                                        uint8_t* __restrict__ cache, long long n_tiles) {
  const int t = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int tid = threadIdx.x;
  const long long pos = (long long)seq_lens[b] + t;
  if (pos < 0 || pos >= n_tiles * kTile) {
    if (tid == 0) atomicOr(L.status, BGTQ_STATUS_ENCODE_OVERFLOW);
    return;
  }
  __shared__ double xk[kD], xv[kD], xp[kD];
  __shared__ double gnorm[kMaxGroups + 1];
  __shared__ unsigned kw[17];

  const size_t base = (((size_t)b * n_new + t) * h_kv + h) * kD;
  xk[tid] = load_elem(k, dtype, base + tid);
  xv[tid] = load_elem(v, dtype, base + tid);
  if (tid < 17) kw[tid] = 0u;
  __syncthreads();

  // packed dimension p = tid: its group and row inside the group
  int g = 0;
  while (g + 1 < L.n_kgroups && tid >= L.group_off[g + 1]) ++g;
  xp[tid] = xk[L.packed_coord[tid]];
  __syncthreads();

  if (tid < L.n_kgroups) {
    double s = 0.0;
    const int off = L.group_off[tid], d = L.group_dim[tid];
    for (int i = 0; i < d; ++i) s = fma(xp[off + i], xp[off + i], s);
    gnorm[tid] = sqrt(s);
  } else if (tid == 64) {
    double s = 0.0;
    for (int i = 0; i < kD; ++i) s = fma(xv[i], xv[i], s);
    gnorm[kMaxGroups] = sqrt(s);
  }
  __syncthreads();

  // key code of packed dimension tid
  {
    const int d = L.group_dim[g], off = L.group_off[g], i = tid - off, r = L.group_rate[g];
    const double* row = L.k_rot64[g] + (size_t)i * d;
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc = fma(row[j], xp[off + j], acc);
    const double nrm = gnorm[g];
    const double y = nrm > 0.0 ? sqrt(double(d)) * acc / nrm : 0.0;
    const int code = quantize(y, L.threshold[r], r);
    const int bit = L.group_bitoff[g] + i * r;
    atomicOr(&kw[bit >> 5], unsigned(code) << (bit & 31));
    if ((bit & 31) + r > 32) atomicOr(&kw[(bit >> 5) + 1], unsigned(code) >> (32 - (bit & 31)));
  }
  // value code of dimension tid
  int vcode;
  {
    const double* row = L.v_rot64 + (size_t)tid * kD;
    double acc = 0.0;
    for (int j = 0; j < kD; ++j) acc = fma(row[j], xv[j], acc);
    const double nrm = gnorm[kMaxGroups];
    const double y = nrm > 0.0 ? sqrt(double(kD)) * acc / nrm : 0.0;
    vcode = quantize(y, L.threshold[L.v_rate], L.v_rate);
  }
  __syncthreads();

  const long long tile = pos / kTile;
  const int tt = int(pos % kTile);
  uint8_t* tp = cache + (((size_t)b * h_kv + h) * n_tiles + tile) * (size_t)L.tile_bytes;
  unsigned* rec = reinterpret_cast<unsigned*>(tp + (size_t)tt * L.k_record_bytes);
  if (tid < L.k_record_bytes / 4) rec[tid] = kw[tid];
  unsigned* vchunk = reinterpret_cast<unsigned*>(tp + L.vcode_off + (tt / kChunk) * 256 * L.v_rate);
  put_bits_atomic(vchunk, (kChunk * tid + chunk_slot(tt % kChunk)) * L.v_rate, unsigned(vcode), L.v_rate);
  if (tid < L.n_kgroups) reinterpret_cast<float*>(tp + L.knorm_off)[tid * kTile + tt] = float(gnorm[tid]);
  if (tid == 64) reinterpret_cast<float*>(tp + L.vnorm_off)[tt] = float(gnorm[kMaxGroups]);
}

}  // namespace

cudaError_t launch_tq_encode(const DevLayout& L, const void* k, const void* v, int dtype, int batch,
                             int n_new, int h_kv, const int* seq_lens, void* cache, long long n_tiles,
                             cudaStream_t stream) {
  dim3 grid(n_new, batch, h_kv);
  tq_encode_kernel<<<grid, 128, 0, stream>>>(L, k, v, dtype, n_new, h_kv, seq_lens,
                                             static_cast<uint8_t*>(cache), n_tiles);
  return cudaGetLastError();
}

}  // namespace bgtq
