// Split-K decode attention over the packed cache, and the log-sum-exp combine.
//
// "Block-GTQ" abstract, sentence 5: attention runs over the packed caches without ever
// materialising a decoded fp16 KV cache; sentence 8: every cached token takes part (no
// fp16 sink or recent window). Because each group's rotation is orthogonal,
//   q . k_hat = sum_g (|k_g| / sqrt(d_g)) (R_g q_g) . c[codes_g]
// and the value sum is accumulated in V's rotated space and rotated back once:
//   o = R_V^T sum_t p_t (|v_t| / sqrt(128)) c[vcodes_t].
//
// decode_split_kernel: one CTA per (split, batch row x KV head), 128 threads. Per 64-token
// tile: threads 0..63 score one token each for the G query heads; warps run the online
// softmax (base-2 exponent, warp shuffles); thread d accumulates rotated value dimension d.
// combine_kernel: one CTA per (batch row, query head): merges the splits by log-sum-exp
// and applies R_V^T.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "bgtq_internal.h"
#include "kernels.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float load_q(const void* p, int dtype, size_t i) {
  if (dtype == BGTQ_F32) return static_cast<const float*>(p)[i];
  if (dtype == BGTQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(static_cast<const __half*>(p)[i]);
}

__device__ __forceinline__ int chunk_slot(int j) { return 4 * ((j & 7) >> 1) + 2 * (j >> 3) + (j & 1); }

// `width` (<= 32) bits at bit offset `bit` of a word array in shared memory.
__device__ __forceinline__ unsigned get_bits(const unsigned* w, int bit, int width) {
  const unsigned long long pair =
      (unsigned long long)w[bit >> 5] | ((unsigned long long)w[(bit >> 5) + 1] << 32);
  return unsigned(pair >> (bit & 31)) & ((1u << width) - 1u);
}

__device__ __forceinline__ float warp_max(float x) {
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

constexpr int kMaxTileBytes = kTile * (64 + 64 + 4 * (kMaxGroups + 1));

template <int G>
__global__ void __launch_bounds__(128) decode_split_kernel(
    DevLayout L, const void* __restrict__ q, int q_dtype, int h_q, int h_kv, const uint8_t* __restrict__ cache,
    const int* __restrict__ seq_lens, long long n_tiles, int max_tiles, int tiles_per_split, int n_splits,
    float qscale, float* __restrict__ part_o, float* __restrict__ part_ml) {
  const int s = blockIdx.x, u = blockIdx.y;
  const int b = u / h_kv, h = u % h_kv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  __shared__ __align__(16) unsigned tile_w[kMaxTileBytes / 4 + 4];
  __shared__ float qs[G][kD];
  __shared__ float qr[G][kD];
  __shared__ float sc[G][kTile];
  __shared__ float m_s[G], l_s[G], corr_s[G];
  __shared__ float cent[5][16];
  __shared__ float vn_s[kTile];

  long long len = seq_lens[b];
  if (len < 0) len = 0;
  if (len > n_tiles * kTile || len > (long long)max_tiles * kTile) {
    if (tid == 0 && s == 0) atomicOr(L.status, BGTQ_STATUS_DECODE_CLAMPED);
    len = min(n_tiles * kTile, (long long)max_tiles * kTile);
  }
  const int len_tiles = int((len + kTile - 1) / kTile);
  const int t0 = s * tiles_per_split;
  const int t1 = min(t0 + tiles_per_split, len_tiles);

  for (int hh = 0; hh < G; ++hh) qs[hh][tid] = load_q(q, q_dtype, ((size_t)b * h_q + (size_t)h * G + hh) * kD + tid);
  if (tid < 80) cent[tid >> 4][tid & 15] = L.centroid[tid >> 4][tid & 15];
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  __syncthreads();

  // q' = R_g q_g per group, in packed order, times scale * log2(e) / sqrt(d_g)
  {
    int g = 0;
    while (g + 1 < L.n_kgroups && tid >= L.group_off[g + 1]) ++g;
    const int d = L.group_dim[g], off = L.group_off[g], i = tid - off;
    const float* row = L.k_rot32[g] + (size_t)i * d;
    const float f = qscale * rsqrtf(float(d));
    for (int hh = 0; hh < G; ++hh) {
      float a = 0.f;
      for (int j = 0; j < d; ++j) a = fmaf(row[j], qs[hh][L.packed_coord[off + j]], a);
      qr[hh][tid] = a * f;
    }
  }
  float acc[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) acc[hh] = 0.f;
  __syncthreads();

  const uint8_t* base = cache + ((size_t)u * n_tiles) * (size_t)L.tile_bytes;
  const int nvec = L.tile_bytes / 16;
  const float vscale = rsqrtf(float(kD));
  const int vrate = L.v_rate;
  const unsigned vmask = (1u << vrate) - 1u;

  for (int tile = t0; tile < t1; ++tile) {
    const uint4* src = reinterpret_cast<const uint4*>(base + (size_t)tile * L.tile_bytes);
    uint4* dst = reinterpret_cast<uint4*>(tile_w);
    for (int i = tid; i < nvec; i += 128) dst[i] = __ldg(src + i);
    __syncthreads();

    const uint8_t* tb = reinterpret_cast<const uint8_t*>(tile_w);
    if (tid < kTile) {
      const long long tok = (long long)tile * kTile + tid;
      const unsigned* rec = reinterpret_cast<const unsigned*>(tb + tid * L.k_record_bytes);
      const float* kn = reinterpret_cast<const float*>(tb + L.knorm_off);
      float sh[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) sh[hh] = 0.f;
      for (int g = 0; g < L.n_kgroups; ++g) {
        const int r = L.group_rate[g], d = L.group_dim[g], off = L.group_off[g], b0 = L.group_bitoff[g];
        float a[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) a[hh] = 0.f;
        for (int i = 0; i < d; ++i) {
          const float c = cent[r][get_bits(rec, b0 + i * r, r)];
#pragma unroll
          for (int hh = 0; hh < G; ++hh) a[hh] = fmaf(qr[hh][off + i], c, a[hh]);
        }
        const float nrm = kn[g * kTile + tid];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) sh[hh] = fmaf(nrm, a[hh], sh[hh]);
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh) sc[hh][tid] = tok < len ? sh[hh] : -INFINITY;
    } else {
      vn_s[tid - kTile] = reinterpret_cast<const float*>(tb + L.vnorm_off)[tid - kTile] * vscale;
    }
    __syncthreads();

    for (int hh = warp; hh < G; hh += 4) {
      const float x0 = sc[hh][lane], x1 = sc[hh][lane + 32];
      const float mx = warp_max(fmaxf(x0, x1));
      const float m_old = m_s[hh];
      const float m_new = fmaxf(m_old, mx);
      float corr = 1.f, p0 = 0.f, p1 = 0.f;
      if (m_new != -INFINITY) {
        corr = exp2f(m_old - m_new);
        p0 = exp2f(x0 - m_new);
        p1 = exp2f(x1 - m_new);
      }
      const float sum = warp_sum(p0 + p1);
      sc[hh][lane] = p0 * vn_s[lane];
      sc[hh][lane + 32] = p1 * vn_s[lane + 32];
      if (lane == 0) {
        l_s[hh] = l_s[hh] * corr + sum;
        m_s[hh] = m_new;
        corr_s[hh] = corr;
      }
    }
    __syncthreads();

    {
      const unsigned* vw = reinterpret_cast<const unsigned*>(tb + L.vcode_off);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) acc[hh] *= corr_s[hh];
      for (int c = 0; c < kTile / kChunk; ++c) {
        const int bit = c * 256 * vrate * 8 + kChunk * tid * vrate;
        const unsigned long long row =
            ((unsigned long long)vw[bit >> 5] | ((unsigned long long)vw[(bit >> 5) + 1] << 32)) >> (bit & 31);
        for (int j = 0; j < kChunk; ++j) {
          const float val = cent[vrate][unsigned(row >> (chunk_slot(j) * vrate)) & vmask];
#pragma unroll
          for (int hh = 0; hh < G; ++hh) acc[hh] = fmaf(sc[hh][c * kChunk + j], val, acc[hh]);
        }
      }
    }
    __syncthreads();
  }

  const size_t pidx = ((size_t)u * n_splits + s) * G;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) part_o[(pidx + hh) * kD + tid] = acc[hh];
  if (tid < G) {
    part_ml[(pidx + tid) * 2] = m_s[tid];
    part_ml[(pidx + tid) * 2 + 1] = l_s[tid];
  }
}

__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml, int n_splits, int G,
                                                      int h_q, int h_kv, const float* __restrict__ v_rot,
                                                      float* __restrict__ out) {
  const int bq = blockIdx.x;
  const int b = bq / h_q, hq = bq % h_q;
  const int u = b * h_kv + hq / G, hh = hq % G;
  const int tid = threadIdx.x;
  __shared__ float op[kD];
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, part_ml[(((size_t)u * n_splits + s) * G + hh) * 2]);
  float l = 0.f, o = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < n_splits; ++s) {
      const size_t idx = ((size_t)u * n_splits + s) * G + hh;
      const float m = part_ml[idx * 2];
      if (m == -INFINITY) continue;
      const float w = exp2f(m - M);
      l = fmaf(w, part_ml[idx * 2 + 1], l);
      o = fmaf(w, part_o[idx * kD + tid], o);
    }
  }
  op[tid] = l > 0.f ? o / l : 0.f;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < kD; ++i) r = fmaf(v_rot[i * kD + tid], op[i], r);
  out[((size_t)b * h_q + hq) * kD + tid] = r;
}

}  // namespace

DecodePlan plan_decode(int batch, int h_q, int h_kv, long long max_seq_len, int num_sms) {
  DecodePlan p{};
  const int G = h_q / h_kv;
  p.max_tiles = int((max_seq_len + kTile - 1) / kTile);
  if (p.max_tiles < 1) p.max_tiles = 1;
  const long long units = (long long)batch * h_kv;
  const long long target = 4LL * num_sms;
  long long splits = (target + units - 1) / units;
  if (splits < 1) splits = 1;
  if (splits > p.max_tiles) splits = p.max_tiles;
  p.tiles_per_split = int((p.max_tiles + splits - 1) / splits);
  p.n_splits = (p.max_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  p.workspace_bytes = (size_t)units * p.n_splits * G * (kD + 2) * sizeof(float);
  return p;
}

cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, const void* cache, const int* seq_lens, long long n_tiles,
                          float softmax_scale, float* out, void* workspace, cudaStream_t stream) {
  const int G = h_q / h_kv;
  const long long units = (long long)batch * h_kv;
  float* part_o = static_cast<float*>(workspace);
  float* part_ml = part_o + (size_t)units * plan.n_splits * G * kD;
  dim3 grid(plan.n_splits, (unsigned)units);
  const float qscale = softmax_scale * kLog2e;
  const uint8_t* c = static_cast<const uint8_t*>(cache);
#define BGTQ_LAUNCH_SPLIT(GG)                                                                          \
  decode_split_kernel<GG><<<grid, 128, 0, stream>>>(L, q, q_dtype, h_q, h_kv, c, seq_lens, n_tiles,    \
                                                    plan.max_tiles, plan.tiles_per_split, plan.n_splits, \
                                                    qscale, part_o, part_ml)
  switch (G) {
    case 1: BGTQ_LAUNCH_SPLIT(1); break;
    case 2: BGTQ_LAUNCH_SPLIT(2); break;
    case 3: BGTQ_LAUNCH_SPLIT(3); break;
    case 4: BGTQ_LAUNCH_SPLIT(4); break;
    case 5: BGTQ_LAUNCH_SPLIT(5); break;
    case 6: BGTQ_LAUNCH_SPLIT(6); break;
    case 7: BGTQ_LAUNCH_SPLIT(7); break;
    case 8: BGTQ_LAUNCH_SPLIT(8); break;
    default: return cudaErrorInvalidValue;
  }
#undef BGTQ_LAUNCH_SPLIT
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<<<batch * h_q, 128, 0, stream>>>(part_o, part_ml, plan.n_splits, G, h_q, h_kv, L.v_rot32, out);
  return cudaGetLastError();
}

}  // namespace bgtq
