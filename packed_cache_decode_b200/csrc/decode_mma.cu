// Decode attention over the packed cache on tensor cores (sm_100a).
//
// "Block-GTQ" abstract, sentence 5: attention reads the packed codes directly, no decoded
// fp16 KV cache is ever written. With R_g orthogonal,
//   q . k_hat   = sum_g (|k_g| / sqrt(d_g)) (R_g q_g) . c[codes_g]
//   o           = R_V^T sum_t p_t (|v_t| / sqrt(128)) c[vcodes_t] / sum_t p_t.
//
// Three kernels per call:
//  * qprep_kernel (one CTA per batch row x KV head): q' = R_g q_g for the G query heads,
//    scaled by softmax_scale * log2(e) / sqrt(d_g), split into fp16 hi + lo parts and laid
//    out as mma B fragments; also clears the per-unit completion counters.
//  * split_kernel (one CTA per (split, unit), 4 warps): 64-token tiles arrive by 1-D bulk
//    async copies (cp.async.bulk + mbarrier, no multicast) into a 4-stage ring. Warp w
//    takes tokens 16w..16w+15 of each tile. Scores: for every 16-dimension chunk of a key
//    group, the thread's code pairs index a pair table in shared memory (fp16 values, exact
//    for rates 1-2 after a per-rate scale; hi + lo parts for rates 3-4) and mma.m16n8k16
//    multiplies them with q' hi and lo (fp32 accumulators per group, then times the group
//    norm). Online softmax in base 2 with warp shuffles. Values: the probabilities times
//    |v|/sqrt(128) in fp16, transposed with movmatrix, against value-code pair lookups,
//    accumulated in V's rotated space (fp32). The four warps merge, the CTA writes its
//    partial (o', m, l); the last CTA of the unit to finish (atomic counter, no waiting)
//    merges all splits by log-sum-exp and applies R_V^T.
//
// Every mbarrier wait is bounded; on timeout the kernel records BGTQ_STATUS_TIMEOUT, waits
// (bounded) for its own copies in flight and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "bgtq_internal.h"
#include "kernels.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStages = 4;
constexpr int kWarps = 4;
constexpr unsigned kWaitLimit = 1u << 22;
constexpr int kMaxSplitHeads = 1536;  // n_splits * G cap: the merging CTA stages S x G values
// shared floats of the merge area: the four warps' [8][128] partials, and later the
// split merge (3 S G staged values, 2 x 8 per-head scalars, G x 128 outputs)
constexpr int kMergeFloats = 3 * kMaxSplitHeads + 16 + kMaxG * kD;

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ unsigned smem_addr(const void* p) { return unsigned(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, unsigned long long* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long* bar, unsigned parity) {
  for (unsigned i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void mma16816(float (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3,
                                         unsigned b0, unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ unsigned movmatrix_trans(unsigned x) {
  unsigned y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ unsigned pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<unsigned*>(&h);
}
// 32 bits of a little-endian word array starting at bit `bit`.
__device__ __forceinline__ unsigned bits32(const unsigned* w, int bit) {
  return __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31);
}
__device__ __forceinline__ float load_q(const void* p, int dtype, size_t i) {
  if (dtype == BGTQ_F32) return static_cast<const float*>(p)[i];
  if (dtype == BGTQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(static_cast<const __half*>(p)[i]);
}

// Workspace layout of one call (all offsets 256-byte aligned).
struct Workspace {
  unsigned* counters;  // [units]
  uint2* qfrag;        // [units][kMaxChunks][2][32]
  float* part_ml;      // [units][splits][G][2]
  float* part_o;       // [units][splits][G][128]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline Workspace carve(void* base, long long units, int splits, int G) {
  Workspace w;
  char* p = static_cast<char*>(base);
  w.counters = reinterpret_cast<unsigned*>(p);
  p += align256(units * sizeof(unsigned));
  w.qfrag = reinterpret_cast<uint2*>(p);
  p += align256(size_t(units) * kMaxChunks * 2 * 32 * sizeof(uint2));
  w.part_ml = reinterpret_cast<float*>(p);
  p += align256(size_t(units) * splits * G * 2 * sizeof(float));
  w.part_o = reinterpret_cast<float*>(p);
  return w;
}

inline size_t workspace_size(long long units, int splits, int G) {
  return align256(units * sizeof(unsigned)) + align256(size_t(units) * kMaxChunks * 2 * 32 * sizeof(uint2)) +
         align256(size_t(units) * splits * G * 2 * sizeof(float)) + size_t(units) * splits * G * kD * sizeof(float);
}

// ------------------------------------------------------------------ q preparation
__global__ void __launch_bounds__(128) qprep_kernel(DevLayout L, const void* __restrict__ q, int q_dtype, int h_q,
                                                    int h_kv, int G, float qscale, Workspace ws) {
  const int u = blockIdx.x, b = u / h_kv, h = u % h_kv;
  const int tid = threadIdx.x;
  __shared__ float qs[kMaxG][kD];
  __shared__ float qr[kMaxG][kD];
  for (int hh = 0; hh < kMaxG; ++hh)
    qs[hh][tid] = hh < G ? load_q(q, q_dtype, ((size_t)b * h_q + (size_t)h * G + hh) * kD + tid) : 0.f;
  if (tid == 0) ws.counters[u] = 0u;
  __syncthreads();
  {
    int g = 0;
    while (g + 1 < L.n_kgroups && tid >= L.group_off[g + 1]) ++g;
    const int d = L.group_dim[g], off = L.group_off[g], i = tid - off;
    const float* col = L.k_rot32t[g] + i;  // transposed: element (i, j) at j * d + i
    const float f = qscale * rsqrtf(float(d));
    float acc[kMaxG];
#pragma unroll
    for (int hh = 0; hh < kMaxG; ++hh) acc[hh] = 0.f;
#pragma unroll 4
    for (int j = 0; j < d; ++j) {
      const float rj = __ldg(col + (size_t)j * d);
      const int c = L.packed_coord[off + j];
#pragma unroll
      for (int hh = 0; hh < kMaxG; ++hh) acc[hh] = fmaf(rj, qs[hh][c], acc[hh]);
    }
#pragma unroll
    for (int hh = 0; hh < kMaxG; ++hh) qr[hh][tid] = acc[hh] * f;
  }
  __syncthreads();
  // B fragments: lane (g = lane/4 -> head, t = lane%4). k-slots 2t, 2t+1 -> chunk dims 4t, 4t+1;
  // k-slots 2t+8, 2t+9 -> chunk dims 4t+2, 4t+3. Dims beyond the group are zero.
  for (int e = tid; e < L.n_kchunks * 32; e += 128) {
    const int ci = e >> 5, lane = e & 31, hh = lane >> 2, t = lane & 3;
    const int d0 = L.chunk_dim0[ci], nd = L.chunk_ndim[ci];
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = (4 * t + j < nd) ? qr[hh][d0 + 4 * t + j] : 0.f;
    float hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      hi[j] = __half2float(__float2half_rn(v[j]));
      lo[j] = v[j] - hi[j];
    }
    uint2* dst = ws.qfrag + ((size_t)u * kMaxChunks + ci) * 2 * 32;
    dst[lane] = make_uint2(pack_h2(hi[0], hi[1]), pack_h2(hi[2], hi[3]));
    dst[32 + lane] = make_uint2(pack_h2(lo[0], lo[1]), pack_h2(lo[2], lo[3]));
  }
  __syncthreads();
  pdl_trigger();
}

// ------------------------------------------------------------------ split kernel
struct SplitArgs {
  const uint8_t* cache;
  const int* seq_lens;
  long long n_tiles;
  int max_tiles;
  int tiles_per_split;
  int n_splits;
  int h_q, h_kv, G;
  Workspace ws;
  float* out;
};

// fields of value codes: 4 codes of dimension d, tokens 2t, 2t+1, 2t+8, 2t+9 of a chunk
template <int VR>
__device__ __forceinline__ unsigned vfield(const unsigned* chunk_words, int d, int t) {
  return bits32(chunk_words, (16 * d + 4 * t) * VR);
}

template <int VR>
__global__ void __launch_bounds__(128, 3) split_kernel(DevLayout L, SplitArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int s = blockIdx.x, u = blockIdx.y;
  const int b = u / a.h_kv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int TB = L.tile_bytes;

  // shared memory carve-up
  unsigned long long* full = reinterpret_cast<unsigned long long*>(smem);
  unsigned char* ring = smem + 128;
  uint2* qf = reinterpret_cast<uint2*>(ring + kStages * TB + 64);
  unsigned* klut12 = reinterpret_cast<unsigned*>(qf + kMaxChunks * 2 * 32);
  uint2* klut34 = reinterpret_cast<uint2*>(klut12 + 32);
  unsigned* vlut = reinterpret_cast<unsigned*>(klut34 + 320);
  float* mo = reinterpret_cast<float*>(vlut + 256);  // merge: [warp][8][128]
  float* mm = mo + kMergeFloats;                      // [warp][8]
  float* ml = mm + kWarps * 8;                        // [warp][8]
  __shared__ int s_last;

  long long len = a.seq_lens[b];
  if (len < 0) len = 0;
  const long long cap_tokens = min(a.n_tiles, (long long)a.max_tiles) * kTile;
  if (len > cap_tokens) {
    if (tid == 0 && s == 0) atomicOr(L.status, BGTQ_STATUS_DECODE_CLAMPED);
    len = cap_tokens;
  }
  const int len_tiles = int((len + kTile - 1) / kTile);
  const int t0 = s * a.tiles_per_split;
  const int t1 = min(t0 + a.tiles_per_split, len_tiles);
  const int ntiles = max(0, t1 - t0);
  const uint8_t* src = a.cache + ((size_t)u * a.n_tiles + t0) * (size_t)TB;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    for (int i = 0; i < min(kStages, ntiles); ++i) {
      mbar_expect_tx(&full[i], TB);
      bulk_load(ring + i * TB, src + (size_t)i * TB, TB, &full[i]);
    }
  }
  // constant tables (written by the layout upload, not by the previous kernel)
  for (int i = tid; i < 20; i += 128) klut12[i] = L.klut12[i];
  for (int i = tid; i < 320; i += 128)
    klut34[i] = make_uint2(L.klut34[2 * i], L.klut34[2 * i + 1]);
  for (int i = tid; i < (1 << (2 * VR)); i += 128) vlut[i] = L.vlut[i];
  pdl_wait();  // q fragments and counters come from qprep_kernel
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(a.ws.qfrag + (size_t)u * kMaxChunks * 2 * 32);
    uint4* qdst = reinterpret_cast<uint4*>(qf);
    for (int i = tid; i < L.n_kchunks * 32; i += 128) qdst[i] = qsrc[i];
  }
  __syncthreads();

  const float vscale = rsqrtf(float(kD)) / L.kappa_v;

  float O[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) O[mt][j] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  bool ok = true;

  for (int it = 0; it < ntiles; ++it) {
    const int stage = it % kStages;
    // A timed-out wait still runs the tile on whatever is in shared memory (every index
    // stays in bounds); the CTA-wide vote at the end of the tile then stops the loop.
    if (!mbar_wait_bounded(&full[stage], (it / kStages) & 1)) ok = false;
    const unsigned char* tb = ring + stage * TB;
    const int tok0 = 16 * warp + g;  // token rows g and g+8 of this warp's chunk
    const long long gtok = (long long)(t0 + it) * kTile + tok0;

    // ---------------- scores
    const unsigned* rec0 = reinterpret_cast<const unsigned*>(tb + tok0 * L.k_record_bytes);
    const unsigned* rec1 = reinterpret_cast<const unsigned*>(tb + (tok0 + 8) * L.k_record_bytes);
    const float* kn = reinterpret_cast<const float*>(tb + L.knorm_off);
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int gi = 0; gi < L.n_kgroups; ++gi) {
      const int r = L.group_rate[gi];
      const int c0 = L.group_chunk0[gi], c1 = c0 + L.group_nchunks[gi];
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (r <= 2) {
        const unsigned* lut = klut12 + (r == 1 ? 0 : 4);
        const unsigned msk = (1u << (2 * r)) - 1u;
        for (int ci = c0; ci < c1; ++ci) {
          const int bit = L.chunk_bit[ci] + 4 * t * r;
          const unsigned f0 = bits32(rec0, bit), f1 = bits32(rec1, bit);
          const unsigned a0 = lut[f0 & msk], a2 = lut[(f0 >> (2 * r)) & msk];
          const unsigned a1 = lut[f1 & msk], a3 = lut[(f1 >> (2 * r)) & msk];
          const uint2 bh = qf[ci * 64 + lane], bl = qf[ci * 64 + 32 + lane];
          mma16816(acc, a0, a1, a2, a3, bh.x, bh.y);
          mma16816(acc, a0, a1, a2, a3, bl.x, bl.y);
        }
      } else {
        const uint2* lut = klut34 + (r == 3 ? 0 : 64);
        const unsigned msk = (1u << (2 * r)) - 1u;
        for (int ci = c0; ci < c1; ++ci) {
          const int bit = L.chunk_bit[ci] + 4 * t * r;
          const unsigned f0 = bits32(rec0, bit), f1 = bits32(rec1, bit);
          const uint2 e0 = lut[f0 & msk], e2 = lut[(f0 >> (2 * r)) & msk];
          const uint2 e1 = lut[f1 & msk], e3 = lut[(f1 >> (2 * r)) & msk];
          const uint2 bh = qf[ci * 64 + lane], bl = qf[ci * 64 + 32 + lane];
          mma16816(acc, e0.x, e1.x, e2.x, e3.x, bh.x, bh.y);
          mma16816(acc, e0.x, e1.x, e2.x, e3.x, bl.x, bl.y);
          mma16816(acc, e0.y, e1.y, e2.y, e3.y, bh.x, bh.y);
        }
      }
      const float ik = 1.0f / L.kappa[r];
      const float n0 = kn[gi * kTile + tok0] * ik;
      const float n1 = kn[gi * kTile + tok0 + 8] * ik;
      sc[0] = fmaf(acc[0], n0, sc[0]);
      sc[1] = fmaf(acc[1], n0, sc[1]);
      sc[2] = fmaf(acc[2], n1, sc[2]);
      sc[3] = fmaf(acc[3], n1, sc[3]);
    }
    if (gtok >= len) sc[0] = sc[1] = -INFINITY;
    if (gtok + 8 >= len) sc[2] = sc[3] = -INFINITY;

    // ---------------- online softmax (heads 2t and 2t+1; rows g and g+8)
    float x0 = fmaxf(sc[0], sc[2]), x1 = fmaxf(sc[1], sc[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
    }
    const float n0m = fmaxf(m0, x0), n1m = fmaxf(m1, x1);
    const float corr0 = n0m == -INFINITY ? 1.f : exp2f(m0 - n0m);
    const float corr1 = n1m == -INFINITY ? 1.f : exp2f(m1 - n1m);
    const float p0 = n0m == -INFINITY ? 0.f : exp2f(sc[0] - n0m);
    const float p1 = n1m == -INFINITY ? 0.f : exp2f(sc[1] - n1m);
    const float p2 = n0m == -INFINITY ? 0.f : exp2f(sc[2] - n0m);
    const float p3 = n1m == -INFINITY ? 0.f : exp2f(sc[3] - n1m);
    m0 = n0m;
    m1 = n1m;
    l0 = fmaf(l0, corr0, p0 + p2);
    l1 = fmaf(l1, corr1, p1 + p3);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      O[mt][0] *= corr0;
      O[mt][1] *= corr1;
      O[mt][2] *= corr0;
      O[mt][3] *= corr1;
    }
    const float* vn = reinterpret_cast<const float*>(tb + L.vnorm_off);
    const float av0 = vn[tok0] * vscale, av1 = vn[tok0 + 8] * vscale;
    const unsigned pb0 = movmatrix_trans(pack_h2(p0 * av0, p1 * av0));
    const unsigned pb1 = movmatrix_trans(pack_h2(p2 * av1, p3 * av1));

    // ---------------- values
    const unsigned* vw = reinterpret_cast<const unsigned*>(tb + L.vcode_off + warp * 256 * VR);
    constexpr unsigned vm = (1u << (2 * VR)) - 1u;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const unsigned f0 = vfield<VR>(vw, 16 * mt + g, t);
      const unsigned f1 = vfield<VR>(vw, 16 * mt + g + 8, t);
      mma16816(O[mt], vlut[f0 & vm], vlut[f1 & vm], vlut[(f0 >> (2 * VR)) & vm], vlut[(f1 >> (2 * VR)) & vm], pb0,
               pb1);
    }

    // every warp is done with this stage
    if (!__syncthreads_and(ok)) {
      // A copy never completed: record it, wait (bounded) for the copies this CTA still
      // has in flight, and leave without a result for this unit.
      if (tid == 0) {
        atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
        for (int j = it; j < min(it + kStages, ntiles); ++j) mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1);
      }
      return;
    }
    if (tid == 0 && it + kStages < ntiles) {
      mbar_expect_tx(&full[stage], TB);
      bulk_load(ring + stage * TB, src + (size_t)(it + kStages) * TB, TB, &full[stage]);
    }
  }

  // ---------------- merge the warps
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  float* mow = mo + warp * 8 * kD;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    mow[(2 * t) * kD + 16 * mt + g] = O[mt][0];
    mow[(2 * t + 1) * kD + 16 * mt + g] = O[mt][1];
    mow[(2 * t) * kD + 16 * mt + g + 8] = O[mt][2];
    mow[(2 * t + 1) * kD + 16 * mt + g + 8] = O[mt][3];
  }
  if (g == 0) {
    mm[warp * 8 + 2 * t] = m0;
    mm[warp * 8 + 2 * t + 1] = m1;
    ml[warp * 8 + 2 * t] = l0;
    ml[warp * 8 + 2 * t + 1] = l1;
  }
  __syncthreads();
  const int G = a.G;
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * 8 + hh]);
    float o = 0.f, l = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = exp2f(mm[w * 8 + hh] - M);
        o = fmaf(f, mo[(w * 8 + hh) * kD + tid], o);
        l = fmaf(f, ml[w * 8 + hh], l);
      }
    }
    const size_t idx = ((size_t)u * a.n_splits + s) * G + hh;
    a.ws.part_o[idx * kD + tid] = o;
    if (tid == 0) {
      a.ws.part_ml[idx * 2] = M;
      a.ws.part_ml[idx * 2 + 1] = l;
    }
  }

  // ---------------- the last CTA of this unit merges the splits
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.ws.counters[u], 1u) == unsigned(a.n_splits - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // stage every split's (m, l) of this unit, then the per-split weights exp2(m_s - M)
  const int S = a.n_splits;
  float* sml = mo;                    // [S][G][2]  (S * G <= kMaxSplitHeads)
  float* sw = mo + 2 * S * G;         // [S][G] weights, then [G] sums l
  float* op = sw + S * G + 2 * kMaxG; // [G][128] normalised rotated outputs
  {
    const float* src_ml = a.ws.part_ml + (size_t)u * S * G * 2;
    for (int i = tid; i < S * G * 2; i += 128) sml[i] = __ldcg(src_ml + i);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int sp = 0; sp < S; ++sp) M = fmaxf(M, sml[(sp * G + tid) * 2]);
    float l = 0.f;
    for (int sp = 0; sp < S; ++sp) {
      const float m = sml[(sp * G + tid) * 2];
      const float w = (M == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - M);
      sw[sp * G + tid] = w;
      l = fmaf(w, sml[(sp * G + tid) * 2 + 1], l);
    }
    sw[S * G + tid] = l;
  }
  __syncthreads();
  {
    const float* po = a.ws.part_o + (size_t)u * S * G * kD + tid;
    for (int hh = 0; hh < G; ++hh) {
      float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
      int sp = 0;
      for (; sp + 4 <= S; sp += 4) {
        o0 = fmaf(sw[(sp + 0) * G + hh], __ldcg(po + ((size_t)(sp + 0) * G + hh) * kD), o0);
        o1 = fmaf(sw[(sp + 1) * G + hh], __ldcg(po + ((size_t)(sp + 1) * G + hh) * kD), o1);
        o2 = fmaf(sw[(sp + 2) * G + hh], __ldcg(po + ((size_t)(sp + 2) * G + hh) * kD), o2);
        o3 = fmaf(sw[(sp + 3) * G + hh], __ldcg(po + ((size_t)(sp + 3) * G + hh) * kD), o3);
      }
      for (; sp < S; ++sp) o0 = fmaf(sw[sp * G + hh], __ldcg(po + ((size_t)sp * G + hh) * kD), o0);
      const float l = sw[S * G + hh];
      op[hh * kD + tid] = l > 0.f ? ((o0 + o1) + (o2 + o3)) / l : 0.f;
    }
  }
  __syncthreads();
  float r[kMaxG];
#pragma unroll
  for (int hh = 0; hh < kMaxG; ++hh) r[hh] = 0.f;
#pragma unroll 4
  for (int i = 0; i < kD; ++i) {
    const float rv = __ldg(L.v_rot32 + i * kD + tid);
#pragma unroll
    for (int hh = 0; hh < kMaxG; ++hh) r[hh] = fmaf(rv, op[(hh < G ? hh : 0) * kD + i], r[hh]);
  }
  const int h = u % a.h_kv;
  for (int hh = 0; hh < G; ++hh) a.out[((size_t)b * a.h_q + (size_t)h * G + hh) * kD + tid] = r[hh];
  if (tid == 0) a.ws.counters[u] = 0u;
}

size_t split_smem_bytes(int tile_bytes) {
  return 128 + size_t(kStages) * tile_bytes + 64 + kMaxChunks * 2 * 32 * sizeof(uint2) + 32 * 4 + 320 * 8 +
         256 * 4 + (kMergeFloats + 2 * kWarps * 8) * sizeof(float);
}

template <int VR>
cudaError_t launch_split(const DevLayout& L, const SplitArgs& a, dim3 grid, cudaStream_t stream) {
  const size_t smem = split_smem_bytes(L.tile_bytes);
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(split_kernel<VR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(split_smem_bytes(kTile * (64 + 64 + 4 * (kMaxGroups + 1)))));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_kernel<VR>, L, a);
}

}  // namespace

DecodePlan plan_decode(int batch, int h_q, int h_kv, long long max_seq_len, int num_sms) {
  DecodePlan p{};
  const int G = h_q / h_kv;
  p.max_tiles = int((max_seq_len + kTile - 1) / kTile);
  if (p.max_tiles < 1) p.max_tiles = 1;
  const long long units = (long long)batch * h_kv;
  const long long target = 3LL * num_sms;
  long long splits = (target + units - 1) / units;
  if (splits < 1) splits = 1;
  if (splits > p.max_tiles) splits = p.max_tiles;
  if (splits * G > kMaxSplitHeads) splits = kMaxSplitHeads / G;
  p.tiles_per_split = int((p.max_tiles + splits - 1) / splits);
  p.n_splits = (p.max_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  p.workspace_bytes = workspace_size(units, p.n_splits, G);
  return p;
}

cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, const void* cache, const int* seq_lens, long long n_tiles,
                          float softmax_scale, float* out, void* workspace, cudaStream_t stream) {
  const int G = h_q / h_kv;
  const long long units = (long long)batch * h_kv;
  Workspace ws = carve(workspace, units, plan.n_splits, G);
  qprep_kernel<<<unsigned(units), 128, 0, stream>>>(L, q, q_dtype, h_q, h_kv, G, softmax_scale * kLog2e, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  SplitArgs a;
  a.cache = static_cast<const uint8_t*>(cache);
  a.seq_lens = seq_lens;
  a.n_tiles = n_tiles;
  a.max_tiles = plan.max_tiles;
  a.tiles_per_split = plan.tiles_per_split;
  a.n_splits = plan.n_splits;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.G = G;
  a.ws = ws;
  a.out = out;
  dim3 grid(plan.n_splits, unsigned(units));
  switch (L.v_rate) {
    case 1: return launch_split<1>(L, a, grid, stream);
    case 2: return launch_split<2>(L, a, grid, stream);
    case 3: return launch_split<3>(L, a, grid, stream);
    case 4: return launch_split<4>(L, a, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace bgtq
