// tq_encode: TQ-MSE encode-append kernel (device code in encode_body.cuh).
#include <cuda_runtime.h>

#include "bgtq_internal.h"
#include "async_copy.cuh"
#include "encode_body.cuh"
#include "kernels.h"

namespace bgtq {

namespace {

// The layout of KV head h: the kernel parameter, or (PH) heads[h] in global memory.
template <bool PH>
__device__ __forceinline__ const DevLayout& head_layout(const DevLayout& param, const DevLayout* heads, int h) {
  if constexpr (PH) return heads[h];
  else return param;
}

template <bool NC, bool PH>
__global__ void __launch_bounds__(enc::kEncodeThreads) tq_encode_kernel(DevLayout Lp, const DevLayout* __restrict__ heads,
                                                                        const void* __restrict__ k,
                                                                        const void* __restrict__ v, int dtype,
                                                                        int n_new, int h_kv,
                                                                        const int* __restrict__ seq_lens, CacheRef cache) {
  enc::encode_token_part<NC>(head_layout<PH>(Lp, heads, blockIdx.z), k, v, dtype, n_new, h_kv, seq_lens, cache,
                             blockIdx.x / kEncodeParts, blockIdx.x % kEncodeParts, blockIdx.y, blockIdx.z);
}

// ------------------------------------------------------------------ bulk appends
// One CTA of 512 threads per (pair of touched tiles, batch row, KV head): the tiles are read
// into shared memory, the new tokens' codes and norms are written there (shared atomics
// only: no other CTA touches these tiles) and the tiles are written back. The rotations (transposed
// fp32, every K group's then V's) arrive by bulk copies while the tile and the first
// tokens load. Tokens go in blocks of 32; threads 0-255 take tokens 0-15 of a block and
// threads 256-511 tokens 16-31. In each half, lanes l and l + 16 of warp w share packed
// key dimension p = 16 (w % 8) + l % 16 and value dimension p: each sums half of the j
// range of y_p = sqrt(d) sum_j R_pj x_j / |x| (fp32) for the 16 tokens, so that every
// warp does the same share of the value rotation (d = 128) and its group's share of the
// key rotation; a shuffle adds the halves and each lane decides the codes of 8 tokens.
// The fp32 value can differ from the fp64 one by at most sqrt(d) (d + 1) 2^-24 (an fp32
// sum of d products of a unit row of R with x, in any order: Cauchy-Schwarz bounds
// sum |R_pj x_j| by |x|) plus a few roundings of |y|; a value within twice that (and
// 1e-6) of a threshold is listed and recomputed in fp64 by a whole warp after the block,
// so every code is the one the fp64 computation gives. Norms (and the norm correction)
// are fp64.
constexpr int kBulkTokens = 32;
constexpr int kBulkThreads = 512;         // two halves of 256: tokens 0-15 and 16-31 of a block
constexpr int kCtaTiles = 2;              // most tiles a CTA owns: its blocks of 32 tokens may straddle them
constexpr int kHalfTokens = kBulkTokens / 2;
constexpr int kXsLd = kBulkTokens + 4;    // floats per row of the block's inputs (rows 16-byte aligned)
constexpr int kRotFloats = 2 * kD * kD;   // the K groups' rotations (sum of d_g^2 <= 128^2) and V's
constexpr int kMaxTileBytes = kTile * (2 * kD * 4 / 8 + 4 * (kMaxGroups + 1));  // K4V4, four groups, fp32 norms
constexpr int kThrLd = 17;                // thresholds per rate: -inf, t_0 .. t_{2^r - 2}, +inf padding

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

// n <= N elements p[0], p[stride], ... (zeros past n), all loads issued before the first
// is used.
template <typename T, int N>
__device__ __forceinline__ void load_column(const T* __restrict__ p, size_t stride, int n, float (&x)[N]) {
  T raw[N];
#pragma unroll
  for (int tk = 0; tk < N; ++tk) raw[tk] = tk < n ? p[tk * stride] : T(0.f);
#pragma unroll
  for (int tk = 0; tk < N; ++tk) x[tk] = to_f32(raw[tk]);
}

// Half a dot product for N tokens: acc[t] += sum_{jj < n} r[jj ld] x[jj][t], x rows at
// kXsLd floats. The loop runs n_warp >= n steps, the same for the whole warp: steps past
// the lane's own n read no rotation element and add zero times the lane's last row (its
// own inputs: a non-finite input elsewhere cannot reach this sum).
template <int N>
__device__ __forceinline__ void half_dot(const float* __restrict__ r, int ld, const float* __restrict__ x, int n,
                                         int n_warp, float (&acc)[N]) {
#pragma unroll 4
  for (int jj = 0; jj < n_warp; ++jj, r += ld, x += jj < n ? kXsLd : 0) {
    const float rij = jj < n ? *r : 0.f;
    const float4* xr = reinterpret_cast<const float4*>(x);
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const float4 v = xr[q];
      acc[4 * q] = fmaf(rij, v.x, acc[4 * q]);
      acc[4 * q + 1] = fmaf(rij, v.y, acc[4 * q + 1]);
      acc[4 * q + 2] = fmaf(rij, v.z, acc[4 * q + 2]);
      acc[4 * q + 3] = fmaf(rij, v.w, acc[4 * q + 3]);
    }
  }
}

// Lane h of a pair (lanes l, l ^ 16) keeps tokens h N/2 .. h N/2 + N/2 - 1: its own half
// sum plus the partner's (the same fp32 sum on both sides of the pair).
template <int N>
__device__ __forceinline__ void pair_sum(const float (&acc)[N], int h, float (&out)[N / 2]) {
#pragma unroll
  for (int t = 0; t < N / 2; ++t) {
    const float send = h ? acc[t] : acc[N / 2 + t];
    const float mine = h ? acc[N / 2 + t] : acc[t];
    out[t] = mine + __shfl_xor_sync(0xffffffffu, send, 16);
  }
}

// Codes of M tokens of one output: y = sum sqrt(d) / |x| (0 for a zero vector: y = 0,
// exact), the code = the number of thresholds <= y (binary search over A = {-inf, t_0 ..,
// +inf}); bit t of the result is set when y lies within the bound of a threshold.
template <int M>
__device__ __forceinline__ unsigned decide(const float (&y0)[M], const float* __restrict__ scl,
                                           const float* __restrict__ A, float sd, float bound, int nt16,
                                           unsigned (&cw)[M / 4]) {
  unsigned near = 0;
#pragma unroll
  for (int t = 0; t < M; ++t) {
    const float f = scl[t * (kMaxGroups + 1)];
    const float y = y0[t] * f;
    int c = y >= A[8] ? 8 : 0;
    c += y >= A[c + 4] ? 4 : 0;
    c += y >= A[c + 2] ? 2 : 0;
    c += y >= A[c + 1] ? 1 : 0;
    const float margin = fminf(y - A[c], A[c + 1] - y);
    if (t % 4 == 0) cw[t / 4] = 0;
    cw[t / 4] |= unsigned(c) << (8 * (t % 4));
    if (t < nt16 && f > 0.f && margin <= bound * (1.f + fabsf(y) / sd)) near |= 1u << t;
  }
  return near;
}

// fp64 value sqrt(d) (R x)_i / |x| of output i of a group of dimension d (rows off.. of
// the block's inputs), summed by one warp in a fixed order.
__device__ __forceinline__ double y_fp64_warp(const double* rt64, const float* xs, int d, int off, int i, int tk,
                                              double n64, int lane) {
  double dot = 0.0;
  for (int j = lane; j < d; j += 32) dot = fma(rt64[(size_t)j * d + i], double(xs[(off + j) * kXsLd + tk]), dot);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  return sqrt(double(d)) * dot / n64;
}

template <bool NC, bool PH>
__global__ void __launch_bounds__(kBulkThreads, 1) tq_encode_tile_kernel(DevLayout Lp, const DevLayout* __restrict__ heads,
                                                                                const void* __restrict__ k,
                                                                                const void* __restrict__ v, int dtype,
                                                                                int n_new, int h_kv,
                                                                                const int* __restrict__ seq_lens,
                                                                                CacheRef cache, int cta_tiles) {
  extern __shared__ __align__(16) unsigned char sm[];
  float* rs = reinterpret_cast<float*>(sm);                                  // rotations (transposed fp32)
  float* xs = rs + kRotFloats;                                               // [256 dims][kXsLd]
  double* nrm = reinterpret_cast<double*>(xs + 256 * kXsLd);                // [kBulkTokens][kMaxGroups + 1]
  float* sc = reinterpret_cast<float*>(nrm + kBulkTokens * (kMaxGroups + 1));  // sqrt(d) / |x|, same index
  unsigned char* cd = reinterpret_cast<unsigned char*>(sc + kBulkTokens * (kMaxGroups + 1));  // codes [256][tok]
  unsigned short* s_near = reinterpret_cast<unsigned short*>(cd + kBulkTokens * 256);  // tk << 8 | output
  unsigned char* tile = reinterpret_cast<unsigned char*>(s_near + kBulkTokens * 256);  // the tile (16-byte aligned)
  __shared__ short s_pc[kD];
  __shared__ int s_roff[kMaxGroups + 1];
  __shared__ float s_thr[5 * kThrLd];
  __shared__ __align__(8) unsigned long long s_bar;
  __shared__ int s_nnear;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y, h = blockIdx.z;
  const DevLayout& L = head_layout<PH>(Lp, heads, h);
  pdl_wait();
  const long long pos0 = seq_lens[b];
  // the CTA's tiles: cta_tiles (1 or 2) consecutive tiles from tix0
  const long long tix0 = pos0 / kTile + (long long)cta_tiles * blockIdx.x;
  long long t_lo = max(pos0, tix0 * kTile), t_hi = min(pos0 + n_new, (tix0 + cta_tiles) * kTile);
  if (pos0 < 0 || t_lo >= t_hi) return;
  const long long cap = cache.n_tiles * kTile;
  if (t_hi > cap) {
    if (tid == 0) atomicOr(L.status, BGTQ_STATUS_ENCODE_OVERFLOW);
    t_hi = cap;
    if (t_lo >= t_hi) return;
  }
  // the CTA's tiles (a page outside a paged pool is flagged, its tile left out)
  const int n_t = int((t_hi - 1) / kTile - tix0) + 1;
  uint8_t* gt[kCtaTiles];
#pragma unroll
  for (int i = 0; i < kCtaTiles; ++i) gt[i] = i < n_t ? tile_ptr(cache, L, b, h, h_kv, tix0 + i) : nullptr;
  bool any = false;
#pragma unroll
  for (int i = 0; i < kCtaTiles; ++i) any = any || gt[i] != nullptr;
  if (!any) return;
  const int ng = L.n_kgroups;
  if (tid == 0) {
    // every K group's rotation, then V's: d_g^2 floats each (d_g even: whole 16-byte units)
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    int o = 0;
    for (int gg = 0; gg < ng; ++gg) {
      s_roff[gg] = o;
      o += L.group_dim[gg] * L.group_dim[gg];
    }
    s_roff[kMaxGroups] = o;
    s_nnear = 0;
    mbar_expect_tx(&s_bar, unsigned(o + kD * kD) * 4u);
    const unsigned long long keep = evict_last_policy();
    for (int gg = 0; gg < ng; ++gg)
      bulk_load(rs + s_roff[gg], L.k_rot32t[gg], unsigned(L.group_dim[gg] * L.group_dim[gg]) * 4u, &s_bar, keep);
    bulk_load(rs + o, L.v_rot32t, unsigned(kD * kD) * 4u, &s_bar, keep);
  }
  const int TB = L.tile_bytes;
#pragma unroll
  for (int ti = 0; ti < kCtaTiles; ++ti)
    if (gt[ti])
      for (int i = tid; i < TB / 16; i += kBulkThreads)
        reinterpret_cast<uint4*>(tile + ti * TB)[i] = reinterpret_cast<const uint4*>(gt[ti])[i];
  if (tid < kD) s_pc[tid] = L.packed_coord[tid];
  if (tid < 5 * kThrLd) {
    const int rr = tid / kThrLd, m = tid % kThrLd;
    s_thr[tid] = m == 0 ? -INFINITY : (rr >= 1 && m - 1 < (1 << rr) - 1) ? float(L.threshold[rr][m - 1]) : INFINITY;
  }
  __syncthreads();

  // half tb of the CTA takes tokens 16 tb .. 16 tb + 15 of every block; thread tl of the
  // half loads row tl of the block's inputs (packed key dimension tl, or value dimension
  // tl - 128)
  const int tb = tid >> 8, tl = tid & 255;
  const bool ld_key = tl < kD;
  const bool ld_live = !ld_key || tl < L.n_packed;
  const void* src = ld_key ? k : v;
  const int col = ld_key ? s_pc[tl & (kD - 1)] : tl - kD;
  // compute: packed key dimension p (group g, index i, dimension dk) and value dimension p,
  // half hh of each j range; lane hh keeps tokens tk0 .. tk0 + 7
  const int p = (warp & 7) * 16 + (lane & 15), hh = lane >> 4;
  const int tk0 = kHalfTokens * tb + 8 * hh;
  const bool klive = p < L.n_packed;
  int g = 0;
  while (g + 1 < ng && p >= L.group_off[g + 1]) ++g;
  const int dk = L.group_dim[g], koff = L.group_off[g], ki = p - koff, rk = L.group_rate[g];
  const float sdk = sqrtf(float(dk)), sdv = sqrtf(float(kD));
  const float bound_k = 2.f * (sdk * float(dk + 1) + 8.f) * 5.9604645e-8f + 1e-6f;
  const float bound_v = 2.f * (sdv * float(kD + 1) + 8.f) * 5.9604645e-8f + 1e-6f;
  const int nk_warp = __reduce_max_sync(0xffffffffu, klive ? dk / 2 : 0);  // key steps of the warp
  bool rot_ready = false;

  for (long long t0 = t_lo; t0 < t_hi; t0 += kBulkTokens) {
    const int nt = int(min((long long)kBulkTokens, t_hi - t0));
    // the block's inputs: this thread's column for every token (independent loads), then
    // its row of xs in eight float4 stores
    {
      float xv[kHalfTokens];
      const size_t tstride = (size_t)h_kv * kD;
      const size_t base = (((size_t)b * n_new + (t0 - pos0)) * h_kv + h) * kD + col + kHalfTokens * tb * tstride;
      const int nl = ld_live ? max(0, min(kHalfTokens, nt - kHalfTokens * tb)) : 0;
      if (dtype == BGTQ_BF16) load_column(static_cast<const __nv_bfloat16*>(src) + base, tstride, nl, xv);
      else if (dtype == BGTQ_F16) load_column(static_cast<const __half*>(src) + base, tstride, nl, xv);
      else load_column(static_cast<const float*>(src) + base, tstride, nl, xv);
      __syncthreads();  // the previous block's xs, list and codes are no longer read
#pragma unroll
      for (int q = 0; q < kHalfTokens / 4; ++q)
        *reinterpret_cast<float4*>(xs + tl * kXsLd + kHalfTokens * tb + 4 * q) =
            make_float4(xv[4 * q], xv[4 * q + 1], xv[4 * q + 2], xv[4 * q + 3]);
    }
    __syncthreads();
    // group norms in fp64: warp w takes tokens w, w + 16; a fixed order of sums. Lane i
    // keeps the i-th sum of its warp and takes its square root (in parallel)
    {
      double my_s2 = 0.0;
      int my_e = -1, my_n = 0, slot = 0;
      for (int tk = warp; tk < nt; tk += kBulkThreads / 32) {
        for (int gg = 0; gg <= ng; ++gg, ++slot) {
          const int a = gg < ng ? L.group_off[gg] : kD, n = gg < ng ? L.group_dim[gg] : kD;
          double s2 = 0.0;
          for (int j = lane; j < n; j += 32) {
            const double x = xs[(a + j) * kXsLd + tk];
            s2 = fma(x, x, s2);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
          if (lane == slot) {
            my_s2 = s2;
            my_e = tk * (kMaxGroups + 1) + (gg < ng ? gg : kMaxGroups);
            my_n = n;
          }
        }
      }
      if (my_e >= 0) {
        const double nr = sqrt(my_s2);
        nrm[my_e] = nr;
        sc[my_e] = my_s2 > 0.0 ? sqrtf(float(my_n)) / float(nr) : 0.f;  // sqrt(d) / |x_g|, fp32
      }
    }
    if (!rot_ready) {
      // the rotations' bulk copies (bounded wait; a copy engine that never completes flags
      // the call and leaves the tile as it was, after a second bounded wait for the copies)
      const bool ok = mbar_wait_bounded(&s_bar, 0);
      if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
        mbar_wait_bounded(&s_bar, 0);
        return;
      }
      rot_ready = true;
    } else {
      __syncthreads();
    }
    if (kHalfTokens * tb < nt) {  // (uniform per warp: a half with no tokens left skips)
      // value dimension p: rows j = 64 hh .. 64 hh + 63 of R_V (element (p, j) at j 128 + p),
      // tokens 16 tb ..
      float acc[kHalfTokens], y[kHalfTokens / 2];
      unsigned cw[2];
      const float* xh = xs + kHalfTokens * tb;
#pragma unroll
      for (int t = 0; t < kHalfTokens; ++t) acc[t] = 0.f;
      half_dot(rs + s_roff[kMaxGroups] + (kD / 2) * hh * kD + p, kD, xh + (kD + (kD / 2) * hh) * kXsLd, kD / 2, kD / 2,
               acc);
      pair_sum(acc, hh, y);
      unsigned near = decide(y, sc + tk0 * (kMaxGroups + 1) + kMaxGroups, s_thr + L.v_rate * kThrLd, sdv, bound_v,
                             nt - tk0, cw);
      *reinterpret_cast<uint2*>(cd + (kD + p) * kBulkTokens + tk0) = make_uint2(cw[0], cw[1]);
      while (near) {
        const int t = __ffs(near) - 1;
        near &= near - 1;
        s_near[atomicAdd(&s_nnear, 1)] = (unsigned short)((tk0 + t) << 8 | (kD + p));
      }
      // packed key dimension p: rows j = dk/2 hh .. of its group's rotation
#pragma unroll
      for (int t = 0; t < kHalfTokens; ++t) acc[t] = 0.f;
      half_dot(rs + s_roff[g] + (dk / 2) * hh * dk + ki, dk, xh + (koff + (dk / 2) * hh) * kXsLd, klive ? dk / 2 : 0,
               nk_warp, acc);
      pair_sum(acc, hh, y);
      if (klive) {
        near = decide(y, sc + tk0 * (kMaxGroups + 1) + g, s_thr + rk * kThrLd, sdk, bound_k, nt - tk0, cw);
        *reinterpret_cast<uint2*>(cd + p * kBulkTokens + tk0) = make_uint2(cw[0], cw[1]);
        while (near) {
          const int t = __ffs(near) - 1;
          near &= near - 1;
          s_near[atomicAdd(&s_nnear, 1)] = (unsigned short)((tk0 + t) << 8 | p);
        }
      }
    }
    __syncthreads();
    // the listed near-threshold outputs: one warp each, fp64 (the list holds at most every
    // output of the block)
    const int n_near = s_nnear;
    for (int e = warp; e < n_near; e += kBulkThreads / 32) {
      const int tk = s_near[e] >> 8, o = s_near[e] & 255;
      const bool ok = o < kD;
      int ge = ng;
      if (ok) {
        ge = 0;
        while (ge + 1 < ng && o >= L.group_off[ge + 1]) ++ge;
      }
      const int de = ok ? L.group_dim[ge] : kD, offe = ok ? L.group_off[ge] : kD, ie = o - offe;
      const int re = ok ? L.group_rate[ge] : L.v_rate;
      const double n64 = nrm[tk * (kMaxGroups + 1) + (ok ? ge : kMaxGroups)];
      const double yv = y_fp64_warp(ok ? L.k_rot64[ge] : L.v_rot64, xs, de, offe, ie, tk, n64, lane);
      if (lane == 0) cd[o * kBulkTokens + tk] = (unsigned char)enc::quantize(yv, L.threshold[re], re);
    }
    __syncthreads();
    if (tid == 0) s_nnear = 0;  // next read after the next block's first barrier
    {
      // the codes of this lane's 8 tokens into their tiles (one copy of the packing code)
      const int t1 = min(nt, tk0 + 8);
#pragma unroll 1
      for (int tk = tk0; tk < t1; ++tk) {
        const long long t = t0 + tk;
        unsigned char* tp = tile + int(t / kTile - tix0) * TB;
        const int tt = int(t % kTile);
        enc::put_value_code(L, tp, p, tt, cd[(kD + p) * kBulkTokens + tk]);
        if (klive) enc::put_key_code(L, tp, g, ki, tt, cd[p * kBulkTokens + tk]);
      }
    }
    // norms (with norm correction: |x| sqrt(d) / |c|, |c|^2 summed in a fixed order)
    for (int e = warp; e < nt * (ng + 1); e += kBulkThreads / 32) {
      const int tk = e / (ng + 1), gg = e % (ng + 1);
      const int gq = gg < ng ? gg : kMaxGroups;
      double s = nrm[tk * (kMaxGroups + 1) + gq];
      if constexpr (NC) {
        const int a = gg < ng ? L.group_off[gg] : kD, n = gg < ng ? L.group_dim[gg] : kD;
        const int rr = gg < ng ? L.group_rate[gg] : L.v_rate;
        double c2 = 0.0;
        for (int j = lane; j < n; j += 32) {
          const double c = L.centroid64[rr * 16 + cd[(a + j) * kBulkTokens + tk]];
          c2 = fma(c, c, c2);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c2 += __shfl_xor_sync(0xffffffffu, c2, o);
        s = c2 > 0.0 ? s * sqrt(double(n)) / sqrt(c2) : 0.0;
      }
      if (lane == 0) {
        const long long t = t0 + tk;
        unsigned char* tp = tile + int(t / kTile - tix0) * TB;
        const int ent = enc::norm_entry(int(t % kTile));
        if (gg < ng) enc::store_norm(L, tp + L.knorm_off, gg * kTile + ent, s);
        else enc::store_norm(L, tp + L.vnorm_off, ent, s);
      }
    }
  }
  __syncthreads();
  // a kernel launched as this one's dependent may start (it waits for this grid before it
  // reads the tiles written here)
  pdl_trigger();
#pragma unroll
  for (int ti = 0; ti < kCtaTiles; ++ti)
    if (gt[ti])
      for (int i2 = tid; i2 < TB / 16; i2 += kBulkThreads)
        reinterpret_cast<uint4*>(gt[ti])[i2] = reinterpret_cast<const uint4*>(tile + ti * TB)[i2];
}

size_t bulk_smem_bytes(int tile_bytes) {
  return size_t(kRotFloats) * 4 + size_t(256) * kXsLd * 4 + size_t(kBulkTokens) * (kMaxGroups + 1) * 12 +
         size_t(kBulkTokens) * 256 * 3 + size_t(kCtaTiles) * size_t(tile_bytes);
}

}  // namespace

cudaError_t launch_tq_encode(const DevLayout& L, const void* k, const void* v, int dtype, int batch,
                             int n_new, int h_kv, const int* seq_lens, const CacheRef& cache, cudaStream_t stream,
                             const DevLayout* heads) {
  const bool ph = heads != nullptr, nc = L.norm_correct != 0;
  // the bulk encoder's cost hardly grows with the tokens a row appends, the per-token
  // encoder's grows with every token: measured crossover at 4 tokens, 2 for 256 rows x heads
  if (n_new >= kBulkMinTokens || (n_new >= 2 && (long long)batch * h_kv >= 256)) {
    // bulk appends: one CTA per pair of touched tiles
    const size_t smem = bulk_smem_bytes(L.tile_bytes);
    static bool configured[64][4] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int vi = (nc ? 1 : 0) + (ph ? 2 : 0);
    auto kern = nc ? (ph ? tq_encode_tile_kernel<true, true> : tq_encode_tile_kernel<true, false>)
                   : (ph ? tq_encode_tile_kernel<false, true> : tq_encode_tile_kernel<false, false>);
    if (dev < 64 && !configured[dev][vi]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bulk_smem_bytes(kMaxTileBytes)));
      if (e != cudaSuccess) return e;
      configured[dev][vi] = true;
    }
    // a row's new tokens touch at most ceil(n_new / 64) + 1 tiles: two per CTA (a block of
    // 32 tokens may then straddle them) when that still gives every SM a CTA, else one
    static int sms[64] = {};
    if (dev < 64 && !sms[dev]) {
      e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
    }
    const long long tiles = (n_new + kTile - 1) / kTile + 1;
    const int ct = (tiles + 1) / 2 * (long long)batch * h_kv >= (dev < 64 ? sms[dev] : 148) ? kCtaTiles : 1;
    dim3 grid(unsigned((tiles + ct - 1) / ct), batch, h_kv);
    kern<<<grid, kBulkThreads, smem, stream>>>(L, heads, k, v, dtype, n_new, h_kv, seq_lens, cache, ct);
    return cudaGetLastError();
  }
  dim3 grid(n_new * kEncodeParts, batch, h_kv);
  if (!nc) {
    if (ph) tq_encode_kernel<false, true><<<grid, enc::kEncodeThreads, 0, stream>>>(L, heads, k, v, dtype, n_new, h_kv, seq_lens, cache);
    else tq_encode_kernel<false, false><<<grid, enc::kEncodeThreads, 0, stream>>>(L, heads, k, v, dtype, n_new, h_kv, seq_lens, cache);
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
  return ph ? cudaLaunchKernelEx(&cfg, tq_encode_kernel<true, true>, L, heads, k, v, dtype, n_new, h_kv, seq_lens, cache)
            : cudaLaunchKernelEx(&cfg, tq_encode_kernel<true, false>, L, heads, k, v, dtype, n_new, h_kv, seq_lens, cache);
}

}  // namespace bgtq
