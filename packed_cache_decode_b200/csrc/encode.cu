// tq_encode: TQ-MSE encode of new key/value vectors and append into the packed cache.
//
// "TurboQuant: paper algorithm and vLLM engineering implementation" (pipeline diagram):
// input vector x (per-head K or V) -> seeded random rotation -> per-coordinate scalar
// quantisation against a few centroids. "Block-GTQ" abstract, sentence 5: equal-rate RoPE
// blocks are grouped and each group is TQ-MSE coded.
//
// Every decision (norm, rotation, threshold comparison) is taken in fp64 so that the
// codes agree with an fp64 reading of the method except for values within rounding
// distance of a threshold.
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

// Sets `width` (<= 64) bits at bit offset `bit` of a little-endian word array to `val`,
// word by word with atomics (other tokens' fields share these words, possibly
// concurrently).
__device__ __forceinline__ void put_field_atomic(unsigned* words, int bit, unsigned long long val, int width) {
  while (width > 0) {
    const int w = bit >> 5, sh = bit & 31;
    const int n = min(width, 32 - sh);
    const unsigned mask = (n == 32 ? 0xffffffffu : ((1u << n) - 1u)) << sh;
    atomicAnd(&words[w], ~mask);
    atomicOr(&words[w], (unsigned(val) << sh) & mask);
    val >>= n;
    bit += n;
    width -= n;
  }
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

// One CTA of 512 threads codes one (token, KV head). Output o = tid % 256 is packed key
// dimension o (o < 128) or value dimension o - 128; the two threads of an output
// (tid / 256 = half) each take half of the rotation row (read from the transposed fp64
// copy: consecutive threads, consecutive addresses), eight loads in flight per round,
// and add their halves through shared memory. The latency of a single appended token
// is what matters in a decode step.
__global__ void __launch_bounds__(512) tq_encode_kernel(DevLayout L, const void* __restrict__ k,
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
  __shared__ double xp[kD], xv[kD], partial[2 * kD];
  __shared__ double gnorm[kMaxGroups + 1];
  __shared__ unsigned long long kfield[kMaxChunks];  // this token's field of every key chunk

  const size_t base = (((size_t)b * n_new + t) * h_kv + h) * kD;
  if (tid < kD) xp[tid] = load_elem(k, dtype, base + L.packed_coord[tid]);  // keys in packed order
  else if (tid < 2 * kD) xv[tid - kD] = load_elem(v, dtype, base + tid - kD);
  if (tid < kMaxChunks) kfield[tid] = 0ull;
  __syncthreads();

  if (tid < L.n_kgroups || tid == kD) {
    const double* x = tid < kD ? xp + L.group_off[tid] : xv;
    const int d = tid < kD ? L.group_dim[tid] : kD;
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    int i = 0;
    for (; i + 4 <= d; i += 4) {
      s0 = fma(x[i], x[i], s0);
      s1 = fma(x[i + 1], x[i + 1], s1);
      s2 = fma(x[i + 2], x[i + 2], s2);
      s3 = fma(x[i + 3], x[i + 3], s3);
    }
    for (; i < d; ++i) s0 = fma(x[i], x[i], s0);
    gnorm[tid < kD ? tid : kMaxGroups] = sqrt((s0 + s1) + (s2 + s3));
  }
  __syncthreads();

  const int o = tid & 255, half = tid >> 8;
  const bool is_key = o < kD;
  const int p = is_key ? o : o - kD;
  int g = 0;
  if (is_key)
    while (g + 1 < L.n_kgroups && p >= L.group_off[g + 1]) ++g;
  const int d = is_key ? L.group_dim[g] : kD;
  const int off = is_key ? L.group_off[g] : 0;
  const int i = p - off;
  const double* col = (is_key ? L.k_rot64[g] : L.v_rot64) + i;  // element (i, j) at j * d + i
  const double* x = is_key ? xp + off : xv;
  const int j0 = half * (d / 2), j1 = half ? d : d / 2;
  double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  int j = j0;
  for (; j + 8 <= j1; j += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = fma(__ldg(col + (size_t)(j + u) * d), x[j + u], a[u]);
  }
  for (; j < j1; ++j) a[0] = fma(__ldg(col + (size_t)j * d), x[j], a[0]);
  const double part = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  if (half) partial[o] = part;
  __syncthreads();
  int code = 0;
  if (!half) {
    const double acc = part + partial[o];
    const double nrm = gnorm[is_key ? g : kMaxGroups];
    const double y = nrm > 0.0 ? sqrt(double(d)) * acc / nrm : 0.0;
    const int r = is_key ? L.group_rate[g] : L.v_rate;
    code = quantize(y, L.threshold[r], r);
    if (is_key) atomicOr(&kfield[L.group_chunk0[g] + (i >> 4)], (unsigned long long)code << ((i & 15) * r));
  }
  __syncthreads();

  const long long tile = pos / kTile;
  const int tt = int(pos % kTile);
  uint8_t* tp = cache + (((size_t)b * h_kv + h) * n_tiles + tile) * (size_t)L.tile_bytes;
  if (half) return;
  if (is_key) {
    // chunk-major keys: this token's field of chunk c sits at bit tt * dims_c * rate_c of
    // the chunk's block
    if (tid < L.n_kchunks) {
      const int w = L.chunk_ndim[tid] * L.group_rate[L.chunk_group[tid]];
      put_field_atomic(reinterpret_cast<unsigned*>(tp + L.chunk_koff[tid]), tt * w, kfield[tid], w);
    }
    if (tid < L.n_kgroups) reinterpret_cast<float*>(tp + L.knorm_off)[tid * kTile + tt] = float(gnorm[tid]);
  } else {
    unsigned* vchunk = reinterpret_cast<unsigned*>(tp + L.vcode_off + (tt / kChunk) * 256 * L.v_rate);
    put_bits_atomic(vchunk, (kChunk * p + chunk_slot(tt % kChunk)) * L.v_rate, unsigned(code), L.v_rate);
    if (p == 0) reinterpret_cast<float*>(tp + L.vnorm_off)[tt] = float(gnorm[kMaxGroups]);
  }
}

}  // namespace

cudaError_t launch_tq_encode(const DevLayout& L, const void* k, const void* v, int dtype, int batch,
                             int n_new, int h_kv, const int* seq_lens, void* cache, long long n_tiles,
                             cudaStream_t stream) {
  dim3 grid(n_new, batch, h_kv);
  tq_encode_kernel<<<grid, 512, 0, stream>>>(L, k, v, dtype, n_new, h_kv, seq_lens,
                                             static_cast<uint8_t*>(cache), n_tiles);
  return cudaGetLastError();
}

}  // namespace bgtq
