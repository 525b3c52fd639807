// Device code of tq_encode shared by the append kernel and the fused decode-step kernel.
//
// "TurboQuant: paper algorithm and vLLM engineering implementation" (pipeline diagram):
// input vector x (per-head K or V) -> seeded random rotation -> per-coordinate scalar
// quantisation against a few centroids. "Block-GTQ" abstract, sentence 5: equal-rate RoPE
// blocks are grouped and each group is TQ-MSE coded.
//
// Every decision (norm, rotation, threshold comparison) is taken in fp64 so that the
// codes agree with an fp64 reading of the method except for values within rounding
// distance of a threshold.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "bgtq_internal.h"

namespace bgtq {
namespace enc {


__device__ __forceinline__ double load_elem(const void* p, int dtype, size_t i) {
  if (dtype == BGTQ_F32) return double(static_cast<const float*>(p)[i]);
  if (dtype == BGTQ_BF16) return double(__bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]));
  return double(__half2float(static_cast<const __half*>(p)[i]));
}

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

// Writes a code field that starts at bit `lb` of a lane's bit string, where the string's
// bits below `split` are stored from block bit a0 and the others from block bit b0 (the
// second plane of rate-3 keys and rate 3-4 values); a field may straddle the split.
__device__ __forceinline__ void put_lane_field(unsigned* blk, int lb, unsigned val, int width, int split, int a0,
                                               int b0) {
  if (lb + width <= split) {
    put_bits_atomic(blk, a0 + lb, val, width);
  } else if (lb >= split) {
    put_bits_atomic(blk, b0 + lb - split, val, width);
  } else {
    const int n = split - lb;
    put_bits_atomic(blk, a0 + lb, val, n);
    put_bits_atomic(blk, b0, val >> n, width - n);
  }
}

// Fragment-major placement of the code of token tt (0..63 in its tile).
// Key packed dim at offset i of group g (rate r): quad Q = group_quad0[g] + i / 8 with P
// pairs; pair e = (i % 8) / 2, hi = i & 1; lane = (tt % 8) P + e, slot m = tt / 8. The
// lane's string: rate 1: bit m (lo) or 8 + m (hi); rates 2-4: field 2 r m + r hi. Stored
// at 16 r lane bits into the quad block (rate 3: bits 0..31 at 32 lane, bits 32..47 at
// 256 P + 16 lane).
__device__ __forceinline__ void put_key_code(const DevLayout& L, uint8_t* tile, int g, int i, int tt, unsigned code) {
  const int r = L.group_rate[g];
  const int Q = L.group_quad0[g] + (i >> 3), P = L.quad_np[Q];
  const int e = (i & 7) >> 1, hi = i & 1;
  const int lane = (tt & 7) * P + e, m = tt >> 3;
  unsigned* blk = reinterpret_cast<unsigned*>(tile + L.quad_off[Q]);
  if (r == 1) {
    put_bits_atomic(blk, 16 * lane + 8 * hi + m, code, 1);
  } else if (r == 3) {
    put_lane_field(blk, 6 * m + 3 * hi, code, 3, 32, 32 * lane, 256 * P + 16 * lane);
  } else {
    put_bits_atomic(blk, 16 * r * lane + 2 * r * m + r * hi, code, r);
  }
}

// Value dim d of token tt: chunk c = tt / 16, jj = tt % 16; lane = 4 (d / 16) + (jj % 8) / 2,
// field n = 4 ((d % 16) / 2) + 2 (jj / 8) + (d % 2), hi = jj % 2. The lane's string: rate
// 1: word n / 16, bit n % 16 (+ 16 for hi); rates 2-4: field 2 b n + b hi. Stored at 64 b
// lane bits into the chunk block (rates 3-4: bits 0..127 at 128 lane, the rest at
// 4096 + (64 b - 128) lane).
__device__ __forceinline__ void put_value_code(const DevLayout& L, uint8_t* tile, int d, int tt, unsigned code) {
  const int br = L.v_rate;
  const int jj = tt & 15;
  const int lane = 4 * (d >> 4) + ((jj & 7) >> 1);
  const int n = 4 * ((d & 15) >> 1) + 2 * (jj >> 3) + (d & 1), hi = jj & 1;
  unsigned* blk = reinterpret_cast<unsigned*>(tile + L.vcode_off + (tt >> 4) * 256 * br);
  if (br == 1) {
    put_bits_atomic(blk, 64 * lane + 32 * (n >> 4) + 16 * hi + (n & 15), code, 1);
  } else if (br == 2) {
    put_bits_atomic(blk, 128 * lane + 4 * n + 2 * hi, code, 2);
  } else {
    put_lane_field(blk, 2 * br * n + br * hi, code, br, 128, 128 * lane, 4096 + (64 * br - 128) * lane);
  }
}

// Entry of token tt (0..63 in its tile) in a row of 64 norms: token g + 8 m at 8 g + m, so
// the eight tokens of a lane's tensor-core rows are consecutive.
__device__ __forceinline__ int norm_entry(int tt) { return (tt & 7) * 8 + (tt >> 3); }

// Stores norm s of entry i of a tile's norm area: fp32, or fp16 rounded to nearest even
// and saturated at the largest finite fp16.
__device__ __forceinline__ void store_norm(const DevLayout& L, uint8_t* area, int i, double s) {
  if (L.norm_fp16) reinterpret_cast<__half*>(area)[i] = __double2half(fmin(s, 65504.0));
  else reinterpret_cast<float*>(area)[i] = float(s);
}

// Four CTAs of 256 threads code one (token, KV head); CTA `part` owns packed key
// dimensions and value dimensions [32 part, 32 part + 32). Each of its 64 outputs is
// computed by four consecutive threads, each over a quarter of the rotation row (read
// from the transposed fp64 copy: consecutive outputs, consecutive addresses), eight
// loads in flight, summed with two shuffles. Every CTA recomputes the group norms (the
// inputs are 256 values). Codes are written with atomics: the key fields of a chunk and
// the value rows are shared with other tokens and other parts.
//
// Norm correction ("TurboQuant: paper algorithm and vLLM engineering implementation",
// vLLM column, box "NC"): the stored norm is |x| sqrt(d) / |c|, c the vector of the
// centroids the group's coordinates were coded to, so that the decoded vector keeps the
// input's norm. |c|^2 spans the four parts' codes: the four CTAs of a token run as one
// thread-block cluster; each sums the squares of its own centroids per group (fixed
// order), writes the sums into part 0's shared memory, and after the cluster barrier
// part 0 writes the corrected norms. The launch must then use clusters of 4 along x.
constexpr int kEncodeThreads = 256;

// Body of one encode CTA (256 threads): token t of batch row b, KV head h, output part
// `part` (0..3). NC: the layout has norm correction (L.norm_correct), and the launch runs
// the four parts of a token as one cluster.
template <bool NC>
__device__ __forceinline__ void encode_token_part(const DevLayout& L, const void* __restrict__ k,
                                                  const void* __restrict__ v, int dtype, int n_new, int h_kv,
                                                  const int* __restrict__ seq_lens, const CacheRef& cache, int t,
                                                  int part, int b, int h) {
  const int tid = threadIdx.x;
  // a decode step may be launched while the kernel before it still runs (programmatic
  // dependent launch): nothing the caller writes (seq_lens, k, v, the cache, a block
  // table) is read before that kernel has completed (a no-op for a plain launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // from here on a kernel launched as this one's dependent may start (it waits for this
  // grid before it reads the tokens written here)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long pos = (long long)seq_lens[b] + t;
  // both early exits are the same for the four parts of a token (with NC, a whole cluster
  // leaves before its first barrier)
  if (pos < 0 || pos >= cache.n_tiles * kTile) {
    if (tid == 0 && part == 0) atomicOr(L.status, BGTQ_STATUS_ENCODE_OVERFLOW);
    return;
  }
  uint8_t* tp = nullptr;
  if constexpr (NC) {
    tp = tile_ptr(cache, L, b, h, h_kv, pos / kTile);
    if (!tp) return;
    // the cluster's CTAs must all have started before one writes into another's shared
    // memory: arrive now, wait just before that write
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  }
  __shared__ double xp[kD], xv[kD];
  __shared__ double gnorm[kMaxGroups + 1];
  __shared__ double csq[64];                         // NC: squared centroid of each output
  __shared__ double part_sq[kEncodeParts][kMaxGroups + 1];  // NC, part 0: the parts' sums

  const size_t base = (((size_t)b * n_new + t) * h_kv + h) * kD;
  // keys in packed order (packed dims past n_packed belong to rate-0 blocks: not stored)
  if (tid < kD) xp[tid] = tid < L.n_packed ? load_elem(k, dtype, base + L.packed_coord[tid]) : 0.0;
  else xv[tid - kD] = load_elem(v, dtype, base + tid - kD);
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

  // thread = (output o of this part, quarter q of its dot product)
  const int o = tid >> 2, q = tid & 3;
  const bool is_key = o < 32;
  const int p = 32 * part + (o & 31);
  const bool live = !is_key || p < L.n_packed;  // a key output past n_packed does not exist
  int g = 0;
  if (is_key)
    while (g + 1 < L.n_kgroups && p >= L.group_off[g + 1]) ++g;
  const int d = is_key ? L.group_dim[g] : kD;
  const int off = is_key ? L.group_off[g] : 0;
  const int i = p - off;
  const double* col = (is_key ? L.k_rot64[g] : L.v_rot64) + i;  // element (i, j) at j * d + i
  const double* x = is_key ? xp + off : xv;
  const int j0 = live ? (q * d) / 4 : 0, j1 = live ? ((q + 1) * d) / 4 : 0;
  double a[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  int j = j0;
  for (; j + 8 <= j1; j += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = fma(__ldg(col + (size_t)(j + u) * d), x[j + u], a[u]);
  }
  for (; j < j1; ++j) a[0] = fma(__ldg(col + (size_t)j * d), x[j], a[0]);
  double acc = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);

  if constexpr (!NC) {
    if (q != 0 || !live) return;
    const double nrm = gnorm[is_key ? g : kMaxGroups];
    const double y = nrm > 0.0 ? sqrt(double(d)) * acc / nrm : 0.0;
    const int r = is_key ? L.group_rate[g] : L.v_rate;
    const int code = quantize(y, L.threshold[r], r);
    const int tt = int(pos % kTile);
    tp = tile_ptr(cache, L, b, h, h_kv, pos / kTile);
    if (!tp) return;
    if (is_key) {
      put_key_code(L, tp, g, i, tt, unsigned(code));
      if (part == 0 && p < L.n_kgroups) store_norm(L, tp + L.knorm_off, p * kTile + norm_entry(tt), gnorm[p]);
    } else {
      put_value_code(L, tp, p, tt, unsigned(code));
      if (p == 0) store_norm(L, tp + L.vnorm_off, norm_entry(tt), gnorm[kMaxGroups]);
    }
    return;
  }
  const int tt = int(pos % kTile);
  if (q == 0 && !live) csq[o] = 0.0;
  if (q == 0 && live) {
    const double nrm = gnorm[is_key ? g : kMaxGroups];
    const double y = nrm > 0.0 ? sqrt(double(d)) * acc / nrm : 0.0;
    const int r = is_key ? L.group_rate[g] : L.v_rate;
    const int code = quantize(y, L.threshold[r], r);
    if (is_key) put_key_code(L, tp, g, i, tt, unsigned(code));
    else put_value_code(L, tp, p, tt, unsigned(code));
    const double c = L.centroid64[r * 16 + code];
    csq[o] = c * c;
  }
  uint8_t* kna = tp + L.knorm_off;
  uint8_t* vna = tp + L.vnorm_off;
  // ---- norm correction: every thread of the four CTAs reaches every cluster barrier
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (tid <= kMaxGroups) {
    // entry tid < kMaxGroups: key group tid (outputs 0..31 of this part), entry kMaxGroups:
    // the value vector (outputs 32..63)
    double sq = 0.0;
    if (tid == kMaxGroups) {
      for (int oo = 32; oo < 64; ++oo) sq += csq[oo];
    } else if (tid < L.n_kgroups) {
      const int lo = L.group_off[tid], hi = lo + L.group_dim[tid];
      for (int oo = 0; oo < 32; ++oo) {
        const int pp = 32 * part + oo;
        if (pp >= lo && pp < hi) sq += csq[oo];
      }
    }
    double* dst = cluster.map_shared_rank(&part_sq[0][0], 0);
    dst[part * (kMaxGroups + 1) + tid] = sq;
  }
  cluster.sync();
  if (part == 0 && tid <= kMaxGroups && (tid < L.n_kgroups || tid == kMaxGroups)) {
    const double c2 = ((part_sq[0][tid] + part_sq[1][tid]) + (part_sq[2][tid] + part_sq[3][tid]));
    const double dd = tid == kMaxGroups ? double(kD) : double(L.group_dim[tid]);
    const double s = c2 > 0.0 ? gnorm[tid] * sqrt(dd) / sqrt(c2) : 0.0;
    if (tid == kMaxGroups) store_norm(L, vna, norm_entry(tt), s);
    else store_norm(L, kna, tid * kTile + norm_entry(tt), s);
  }
}


}  // namespace enc
}  // namespace bgtq
