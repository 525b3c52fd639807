// Decode attention over the packed cache on tensor cores (sm_100a).
//
// "Block-GTQ" abstract, sentence 5: attention reads the packed codes directly, no decoded
// fp16 KV cache is ever written. With R_g orthogonal,
//   q . k_hat   = sum_g (|k_g| / sqrt(d_g)) (R_g q_g) . c[codes_g]
//   o           = R_V^T sum_t p_t (|v_t| / sqrt(128)) c[vcodes_t] / sum_t p_t.
//
// Three kernels per call (a decode step that also appends the new token fuses the append
// into the first one: step_prep_kernel runs the encode CTAs and the q-preparation CTAs):
//  * qprep_kernel (one CTA per batch row x KV head): q' = R_g q_g for the G query heads
//    (rotations staged in shared memory), scaled by softmax_scale * log2(e) / sqrt(d_g),
//    split into fp16 hi + lo parts and laid out as mma B fragments.
//  * split_kernel (one CTA per (split, unit), 4 consumer warps + 1 producer warp): 64-token
//    tiles arrive by 1-D bulk async copies (cp.async.bulk + mbarrier, no multicast) into an
//    8-stage ring; consumer warp w takes tiles w, w+4, ... whole, as four 16-token row
//    blocks. Scores: for every 16-dimension chunk of a key group, the thread's code pairs
//    index a pair table in shared memory (fp16 values, exact for rates 1-2 after a per-rate
//    scale; hi + lo parts for rates 3-4) and mma.m16n8k16 multiplies them with q' hi and lo
//    (fp32 accumulators per group, then times the group norm). Online softmax in base 2
//    with warp shuffles. Values: the probabilities times |v|/sqrt(128) in fp16, transposed
//    with movmatrix, against value-code pair lookups, accumulated in V's rotated space
//    (fp32). The four warps merge and the CTA writes its partial (o', m, l).
//  * combine_kernel (one CTA per batch row x query head, 512 threads): log-sum-exp merge
//    of the splits and o = R_V^T o'.
// The three launches are chained with programmatic dependent launch, so each kernel's
// set-up (and, when the first kernel does not write the cache, the split kernel's first
// tile copies) overlaps the previous kernel.
//
// Every mbarrier wait is bounded; on timeout the kernel records BGTQ_STATUS_TIMEOUT, waits
// (bounded) for its own copies in flight and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "bgtq_internal.h"
#include "encode_body.cuh"
#include "kernels.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStages = 8;
constexpr int kWarps = 4;
constexpr unsigned kWaitLimit = 1u << 22;

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
  uint2* qfrag;        // [units][kMaxChunks][2][32]
  float* part_ml;      // [units][splits][G][2]
  float* part_o;       // [units][splits][G][128]
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline Workspace carve(void* base, long long units, int splits, int G) {
  Workspace w;
  char* p = static_cast<char*>(base);
  w.qfrag = reinterpret_cast<uint2*>(p);
  p += align256(size_t(units) * kMaxChunks * 2 * 32 * sizeof(uint2));
  w.part_ml = reinterpret_cast<float*>(p);
  p += align256(size_t(units) * splits * G * 2 * sizeof(float));
  w.part_o = reinterpret_cast<float*>(p);
  return w;
}

inline size_t workspace_size(long long units, int splits, int G) {
  return align256(size_t(units) * kMaxChunks * 2 * 32 * sizeof(uint2)) +
         align256(size_t(units) * splits * G * 2 * sizeof(float)) + size_t(units) * splits * G * kD * sizeof(float);
}

// ------------------------------------------------------------------ q preparation
constexpr int kPrepThreads = 256;
static_assert(kPrepThreads == enc::kEncodeThreads, "the fused step kernel runs both bodies");

__device__ __forceinline__ void qprep_unit(const DevLayout& L, const void* __restrict__ q, int q_dtype, int h_q,
                                           int h_kv, int G, float qscale, const Workspace& ws, int u,
                                           float* prep_smem) {
  const int b = u / h_kv, h = u % h_kv;
  const int tid = threadIdx.x;
  float* rot = prep_smem;                       // the K-group rotations, transposed, back to back
  float* qs = rot + L.k_rot32t_floats;          // [8][128] q in original coordinates
  float* qr = qs + kMaxG * kD;                  // [8][128] q' in packed order
  {
    const float4* src = reinterpret_cast<const float4*>(L.k_rot32t[0]);
    float4* dst = reinterpret_cast<float4*>(rot);
    const int n4 = L.k_rot32t_floats / 4;
#pragma unroll 4
    for (int i = tid; i < n4; i += kPrepThreads) dst[i] = __ldg(src + i);
  }
  // q in packed order: qs[hh][p] = q[hh][packed_coord[p]]
  for (int e = tid; e < kMaxG * kD; e += kPrepThreads) {
    const int hh = e / kD, p = e % kD;
    qs[e] = hh < G ? load_q(q, q_dtype, ((size_t)b * h_q + (size_t)h * G + hh) * kD + L.packed_coord[p]) : 0.f;
  }
  __syncthreads();
  {
    // thread = (packed dimension p, half of the heads)
    const int p = tid & (kD - 1), hbase = (tid >> 7) * (kMaxG / 2);
    int g = 0;
    while (g + 1 < L.n_kgroups && p >= L.group_off[g + 1]) ++g;
    const int d = L.group_dim[g], off = L.group_off[g], i = p - off;
    const float* col = rot + L.k_rot32t_off[g] + i;  // element (i, j) at j * d + i
    const float f = qscale * rsqrtf(float(d));
    float acc[kMaxG / 2];
#pragma unroll
    for (int k = 0; k < kMaxG / 2; ++k) acc[k] = 0.f;
    const float* qg = qs + hbase * kD + off;
#pragma unroll 4
    for (int j = 0; j < d; ++j) {
      const float rj = col[j * d];
#pragma unroll
      for (int k = 0; k < kMaxG / 2; ++k) acc[k] = fmaf(rj, qg[k * kD + j], acc[k]);
    }
#pragma unroll
    for (int k = 0; k < kMaxG / 2; ++k) qr[(hbase + k) * kD + p] = acc[k] * f;
  }
  __syncthreads();
  // B fragments: lane (g = lane/4 -> head, t = lane%4). k-slots 2t, 2t+1 -> chunk dims 4t, 4t+1;
  // k-slots 2t+8, 2t+9 -> chunk dims 4t+2, 4t+3. Dims beyond the group are zero.
  for (int e = tid; e < L.n_kchunks * 32; e += kPrepThreads) {
    const int ci = e >> 5, lane = e & 31, hh = lane >> 2, t = lane & 3;
    const int d0 = L.chunk_dim0[ci], nd = L.chunk_ndim[ci];
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = (4 * t + j < nd) ? qr[hh * kD + d0 + 4 * t + j] : 0.f;
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
}

__global__ void __launch_bounds__(kPrepThreads) qprep_kernel(DevLayout L, const void* __restrict__ q, int q_dtype,
                                                             int h_q, int h_kv, int G, float qscale, Workspace ws) {
  extern __shared__ __align__(16) float prep_smem[];
  qprep_unit(L, q, q_dtype, h_q, h_kv, G, qscale, ws, blockIdx.x, prep_smem);
  __syncthreads();
  pdl_trigger();
}

// Fused first kernel of a decode step: blocks [0, n_enc) append the new tokens (four
// blocks per token and KV head), the remaining blocks prepare q' for one unit each.
// It lets the attention kernels launch at once (they wait for it before reading).
__global__ void __launch_bounds__(kPrepThreads) step_prep_kernel(DevLayout L, const void* __restrict__ k,
                                                                 const void* __restrict__ v, int kv_dtype, int n_new,
                                                                 int batch, long long n_tiles,
                                                                 const int* __restrict__ seq_lens_before,
                                                                 uint8_t* __restrict__ cache,
                                                                 const void* __restrict__ q, int q_dtype, int h_q,
                                                                 int h_kv, int G, float qscale, Workspace ws,
                                                                 int n_enc) {
  extern __shared__ __align__(16) float prep_smem[];
  pdl_trigger();
  const int e = blockIdx.x;
  if (e < n_enc) {
    const int part = e % kEncodeParts;
    int rest = e / kEncodeParts;
    const int t = rest % n_new;
    rest /= n_new;
    const int b = rest % batch, h = rest / batch;
    enc::encode_token_part(L, k, v, kv_dtype, n_new, h_kv, seq_lens_before, cache, n_tiles, t, part, b, h);
  } else {
    qprep_unit(L, q, q_dtype, h_q, h_kv, G, qscale, ws, e - n_enc, prep_smem);
  }
}

size_t prep_smem_bytes(const DevLayout& L) { return (size_t(L.k_rot32t_floats) + 2 * kMaxG * kD) * sizeof(float); }

// ------------------------------------------------------------------ combine
constexpr int kCombThreads = 512;
constexpr int kMaxSplits = 1024;

// One CTA per (batch row, query head): log-sum-exp merge of the splits, then o = R_V^T o'.
// Four threads per output dimension. R_V (not written by the split kernel) is read into
// registers before waiting for the split kernel to finish.
__global__ void __launch_bounds__(kCombThreads, 1) combine_kernel(const float* __restrict__ part_ml,
                                                              const float* __restrict__ part_o, int S, int G,
                                                              int h_q, int h_kv, const float* __restrict__ v_rot,
                                                              float* __restrict__ out) {
  const int bq = blockIdx.x, b = bq / h_q, hq = bq % h_q;
  const int u = b * h_kv + hq / G, hh = hq % G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = tid & (kD - 1), qtr = tid >> 7;
  __shared__ float w[kMaxSplits];
  __shared__ float red[2][kCombThreads / 32];
  __shared__ float part[4][kD];
  __shared__ float op[kD];
  float rv[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) rv[i] = __ldg(v_rot + (size_t)(qtr * 32 + i) * kD + d);
  pdl_wait();  // partials come from split_kernel
  const float2* ml = reinterpret_cast<const float2*>(part_ml) + (size_t)u * S * G + hh;  // split sp at ml[sp * G]
  float mloc[2], lloc[2];
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int sp = tid + k * kCombThreads;
    const float2 v = sp < S ? ml[(size_t)sp * G] : make_float2(-INFINITY, 0.f);
    mloc[k] = v.x;
    lloc[k] = v.y;
    M = fmaxf(M, v.x);
  }
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[0][warp] = M;
  __syncthreads();
  M = -INFINITY;
#pragma unroll
  for (int i = 0; i < kCombThreads / 32; ++i) M = fmaxf(M, red[0][i]);
  float l = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int sp = tid + k * kCombThreads;
    if (sp < S) {
      const float wt = (M == -INFINITY || mloc[k] == -INFINITY) ? 0.f : exp2f(mloc[k] - M);
      w[sp] = wt;
      l = fmaf(wt, lloc[k], l);
    }
  }
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[1][warp] = l;
  __syncthreads();
  l = 0.f;
#pragma unroll
  for (int i = 0; i < kCombThreads / 32; ++i) l += red[1][i];
  {
    const float* po = part_o + ((size_t)u * S * G + hh) * kD + d;  // split sp at po[sp * G * kD]
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    int sp = qtr;
    for (; sp + 12 < S; sp += 16) {
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] = fmaf(w[sp + 4 * k], __ldg(po + (size_t)(sp + 4 * k) * G * kD), o[k]);
    }
    for (; sp < S; sp += 4) o[0] = fmaf(w[sp], __ldg(po + (size_t)sp * G * kD), o[0]);
    part[qtr][d] = (o[0] + o[1]) + (o[2] + o[3]);
  }
  __syncthreads();
  if (tid < kD) op[tid] = l > 0.f ? ((part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid])) / l : 0.f;
  __syncthreads();
  float r0 = 0.f, r1 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    r0 = fmaf(rv[i], op[qtr * 32 + i], r0);
    r1 = fmaf(rv[i + 1], op[qtr * 32 + i + 1], r1);
  }
  part[qtr][d] = r0 + r1;
  __syncthreads();
  if (tid < kD) out[((size_t)b * h_q + hq) * kD + tid] = (part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid]);
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
  int len_add;           // tokens appended by the previous kernel: row b attends over seq_lens[b] + len_add
  int wait_before_copy;  // the previous kernel writes the cache: wait for it before copying
};

constexpr int kConsumers = 4;                 // consumer warps, one 16-token slice of a tile each
constexpr int kThreads = 32 * (kConsumers + 1);  // + one producer warp

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Scores of one key group with compile-time rate R: for each 16-dimension chunk, the
// thread's four codes (dims 4t..4t+3 of the chunk) of tokens g and g+8 index the pair
// tables; q' hi and lo are the B operands. The bit offset advances 16 R per chunk.
// Per chunk the thread forms its A fragments from the four codes (dims 4t..4t+3 of the
// chunk) of its two tokens in each of the tile's four 16-token row blocks, and multiplies
// them with the q' hi and lo fragments (and, for rates 3-4, the centroid low parts).
// The four row blocks are independent accumulation chains.
template <int R>
__device__ __forceinline__ void key_chunk(float (&acc)[4], unsigned f0, unsigned f1, uint2 bh, uint2 bl,
                                          const unsigned* klut12, const uint2* klut1q, const uint2* klut34) {
  constexpr unsigned M = (1u << (2 * R)) - 1u;
  if constexpr (R == 1) {
    // the four 1-bit codes of a token index one entry: {pair (4t, 4t+1), pair (4t+2, 4t+3)}
    const uint2 e0 = klut1q[f0 & 15u], e1 = klut1q[f1 & 15u];
    mma16816(acc, e0.x, e1.x, e0.y, e1.y, bh.x, bh.y);
    mma16816(acc, e0.x, e1.x, e0.y, e1.y, bl.x, bl.y);
  } else if constexpr (R == 2) {
    const unsigned* lut = klut12 + 4;
    const unsigned a0 = lut[f0 & M], a2 = lut[(f0 >> 4) & M];
    const unsigned a1 = lut[f1 & M], a3 = lut[(f1 >> 4) & M];
    mma16816(acc, a0, a1, a2, a3, bh.x, bh.y);
    mma16816(acc, a0, a1, a2, a3, bl.x, bl.y);
  } else {
    const uint2* lut = klut34 + (R == 3 ? 0 : 64);
    const uint2 e0 = lut[f0 & M], e2 = lut[(f0 >> (2 * R)) & M];
    const uint2 e1 = lut[f1 & M], e3 = lut[(f1 >> (2 * R)) & M];
    mma16816(acc, e0.x, e1.x, e2.x, e3.x, bh.x, bh.y);
    mma16816(acc, e0.x, e1.x, e2.x, e3.x, bl.x, bl.y);
    mma16816(acc, e0.y, e1.y, e2.y, e3.y, bh.x, bh.y);
  }
}

// Keys are chunk-major inside a tile: chunk c's block holds the 64 tokens' fields of
// dims_c * R bits back to back. For a full chunk (16 dims) the thread's four codes of
// token j sit in one word: R = 1: word j/2 at bit 16 (j%2) + 4t; R = 2: word j at 8t;
// R = 4: word 2j + t/2 at 16 (t%2). Rate 3 and partial chunks use a 64-bit window.
template <int R>
__device__ __forceinline__ void key_group(float (&acc)[4][4], const unsigned char* tb, const DevLayout& L,
                                          const uint2* qf, int c0, int c1, int lane, const unsigned* klut12,
                                          const uint2* klut1q, const uint2* klut34) {
  const int g = lane >> 2, t = lane & 3;
  const uint2* qp = qf + c0 * 64 + lane;
  for (int ci = c0; ci < c1; ++ci, qp += 64) {
    const uint2 bh = qp[0], bl = qp[32];
    const unsigned* blk = reinterpret_cast<const unsigned*>(tb + L.chunk_koff[ci]);
    const int nd = L.chunk_ndim[ci];
    if (R != 3 && nd == 16) {
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const int j0 = 16 * rt + g, j1 = j0 + 8;
        unsigned f0, f1;
        if constexpr (R == 1) {
          f0 = blk[j0 >> 1] >> (16 * (g & 1) + 4 * t);
          f1 = blk[j1 >> 1] >> (16 * (g & 1) + 4 * t);
        } else if constexpr (R == 2) {
          f0 = blk[j0] >> (8 * t);
          f1 = blk[j1] >> (8 * t);
        } else {
          f0 = blk[2 * j0 + (t >> 1)] >> (16 * (t & 1));
          f1 = blk[2 * j1 + (t >> 1)] >> (16 * (t & 1));
        }
        key_chunk<R>(acc[rt], f0, f1, bh, bl, klut12, klut1q, klut34);
      }
    } else {
      const int w = nd * R;
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const int j0 = 16 * rt + g;
        const unsigned f0 = bits32(blk, j0 * w + 4 * t * R), f1 = bits32(blk, (j0 + 8) * w + 4 * t * R);
        key_chunk<R>(acc[rt], f0, f1, bh, bl, klut12, klut1q, klut34);
      }
    }
  }
}

// Value codes for the PV product. MMA row r of m-tile mt stands for value dimension
// 16 (r % 8) + 2 mt + r / 8, so thread g owns the contiguous dimensions 16g .. 16g+15 of
// the 16-token chunk (16 rows of 16 VR bits starting at word 8 VR g). For m-tile mt the
// thread needs rows 2mt (MMA row g) and 2mt+1 (row g+8), and in each row the 4 VR bits of
// tokens 2t, 2t+1, 2t+8, 2t+9 (slots 4t..4t+3). Rates 1 and 2 keep all 16 rows in
// registers (one tile load); rates 3 and 4 read the two rows per m-tile.
template <int VR>
struct ValueRows {
  unsigned w[VR <= 2 ? 8 * VR : 1];
  const unsigned* base;
  int t;
  __device__ __forceinline__ void load(const unsigned* chunk, int g, int t_) {
    t = t_;
    base = chunk + 8 * VR * g;
    if constexpr (VR <= 2) {
      const uint4* p = reinterpret_cast<const uint4*>(base);
#pragma unroll
      for (int i = 0; i < 2 * VR; ++i) {
        const uint4 v = p[i];
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
    }
  }
  __device__ __forceinline__ void fields(int mt, unsigned& fx, unsigned& fy) const {
    if constexpr (VR == 1) {
      fx = w[mt] >> (4 * t);
      fy = w[mt] >> (16 + 4 * t);
    } else if constexpr (VR == 2) {
      fx = w[2 * mt] >> (8 * t);
      fy = w[2 * mt + 1] >> (8 * t);
    } else if constexpr (VR == 3) {
      const unsigned w0 = base[3 * mt], w1 = base[3 * mt + 1], w2 = base[3 * mt + 2];
      fx = unsigned((((unsigned long long)w1 << 32) | w0) >> (12 * t));
      fy = unsigned((((unsigned long long)w2 << 32) | w1) >> (16 + 12 * t));
    } else {
      const uint4 v = reinterpret_cast<const uint4*>(base)[mt];
      const int sh = 16 * (t & 1);
      fx = ((t < 2) ? v.x : v.y) >> sh;
      fy = ((t < 2) ? v.z : v.w) >> sh;
    }
  }
};

template <int VR>
__global__ void __launch_bounds__(kThreads, 3) split_kernel(DevLayout L, SplitArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int s = blockIdx.x, u = blockIdx.y;
  const int b = u / a.h_kv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int TB = L.tile_bytes;

  unsigned long long* full = reinterpret_cast<unsigned long long*>(smem);
  unsigned long long* empty = full + kStages;
  unsigned char* ring = smem + 128;
  uint2* qf = reinterpret_cast<uint2*>(ring + kStages * TB + 64);
  unsigned* klut12 = reinterpret_cast<unsigned*>(qf + kMaxChunks * 2 * 32);
  uint2* klut34 = reinterpret_cast<uint2*>(klut12 + 32);
  uint2* klut1q = klut34 + 320;                       // rate 1, four codes per entry
  unsigned* vlut = reinterpret_cast<unsigned*>(klut1q + 16);
  float* mm = reinterpret_cast<float*>(vlut + 256);  // [warp][8]
  float* ml = mm + kConsumers * 8;                    // [warp][8]
  // the warps' [8][128] partials reuse the ring once every tile has been consumed
  float* mo = reinterpret_cast<float*>(ring);
  __shared__ int s_timeout;

  long long len = (long long)a.seq_lens[b] + a.len_add;
  if (len < 0) len = 0;
  const long long cap_tokens = min(a.n_tiles, (long long)a.max_tiles) * kTile;
  if (len > cap_tokens) {
    if (tid == 0 && s == 0) atomicOr(L.status, BGTQ_STATUS_DECODE_CLAMPED);
    len = cap_tokens;
  }
  const int len_tiles = int((len + kTile - 1) / kTile);
  const int t0 = s * a.tiles_per_split;
  const int ntiles = max(0, min(t0 + a.tiles_per_split, len_tiles) - t0);
  const uint8_t* src = a.cache + ((size_t)u * a.n_tiles + t0) * (size_t)TB;

  if (tid == kConsumers * 32) {
    // the producer lane: barriers, then the first copies before anything else
    s_timeout = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    fence_mbar_init();
    if (a.wait_before_copy) pdl_wait();
    for (int it = 0; it < min(kStages, ntiles); ++it) {
      mbar_expect_tx(&full[it], TB);
      bulk_load(ring + it * TB, src + (size_t)it * TB, TB, &full[it]);
    }
  }
  for (int i = tid; i < 20; i += kThreads) klut12[i] = L.klut12[i];
  for (int i = tid; i < 320; i += kThreads) klut34[i] = make_uint2(L.klut34[2 * i], L.klut34[2 * i + 1]);
  for (int i = tid; i < 16; i += kThreads) klut1q[i] = make_uint2(L.klut1q[2 * i], L.klut1q[2 * i + 1]);
  for (int i = tid; i < (1 << (2 * VR)); i += kThreads) vlut[i] = L.vlut[i];
  __syncthreads();

  if (warp == kConsumers) {
    // ------------------------------------------------ producer warp: one lane streams tiles
    if (lane == 0) {
      int issued = min(kStages, ntiles);
      for (int it = issued; it < ntiles; ++it) {
        const int stage = it % kStages;
        if (it >= kStages && !mbar_wait_bounded(&empty[stage], ((it / kStages) - 1) & 1)) {
          atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
          break;
        }
        mbar_expect_tx(&full[stage], TB);
        bulk_load(ring + stage * TB, src + (size_t)it * TB, TB, &full[stage]);
        issued = it + 1;
      }
      // do not leave while copies into this CTA's shared memory are still in flight
      for (int j = max(0, issued - kStages); j < issued; ++j) mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1);
    }
    return;
  }

  // ---------------------------------------------------- consumer warps
  pdl_wait();  // q fragments come from qprep_kernel
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(a.ws.qfrag + (size_t)u * kMaxChunks * 2 * 32);
    uint4* qdst = reinterpret_cast<uint4*>(qf);
    for (int i = tid; i < L.n_kchunks * 32; i += 128) qdst[i] = qsrc[i];
  }
  consumer_sync();

  const float vscale = rsqrtf(float(kD)) / L.kappa_v;
  float O[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) O[mt][j] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  // warp w takes tiles w, w+4, w+8, ... of this split; a whole 64-token tile per warp
  for (int it = warp; it < ntiles; it += kConsumers) {
    const int stage = it % kStages;
    if (!mbar_wait_bounded(&full[stage], (it / kStages) & 1)) {
      // stop consuming; the producer waits for its own copies and this unit's result
      // is not written (every consumer warp still reaches the merge barriers below)
      if (lane == 0) {
        atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
        s_timeout = 1;
      }
      break;
    }
    const unsigned char* tb = ring + stage * TB;
    const long long gt0 = (long long)(t0 + it) * kTile + g;  // token of row g in row block 0

    // ---------------- scores of the tile's 64 tokens: per key group (rate as a template
    // parameter), per chunk, four row blocks; then times the group norms
    const float* kn = reinterpret_cast<const float*>(tb + L.knorm_off);
    float sc[4][4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[rt][j] = 0.f;
    for (int gi = 0; gi < L.n_kgroups; ++gi) {
      float acc[4][4];
#pragma unroll
      for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[rt][j] = 0.f;
      const int r = L.group_rate[gi], c0 = L.group_chunk0[gi], c1 = c0 + L.group_nchunks[gi];
      switch (r) {
        case 1: key_group<1>(acc, tb, L, qf, c0, c1, lane, klut12, klut1q, klut34); break;
        case 2: key_group<2>(acc, tb, L, qf, c0, c1, lane, klut12, klut1q, klut34); break;
        case 3: key_group<3>(acc, tb, L, qf, c0, c1, lane, klut12, klut1q, klut34); break;
        default: key_group<4>(acc, tb, L, qf, c0, c1, lane, klut12, klut1q, klut34); break;
      }
      const float ik = L.inv_kappa_group[gi];
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const float n0 = kn[gi * kTile + 16 * rt + g] * ik;
        const float n1 = kn[gi * kTile + 16 * rt + g + 8] * ik;
        sc[rt][0] = fmaf(acc[rt][0], n0, sc[rt][0]);
        sc[rt][1] = fmaf(acc[rt][1], n0, sc[rt][1]);
        sc[rt][2] = fmaf(acc[rt][2], n1, sc[rt][2]);
        sc[rt][3] = fmaf(acc[rt][3], n1, sc[rt][3]);
      }
    }
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      if (gt0 + 16 * rt >= len) sc[rt][0] = sc[rt][1] = -INFINITY;
      if (gt0 + 16 * rt + 8 >= len) sc[rt][2] = sc[rt][3] = -INFINITY;
    }

    // ---------------- online softmax over the 64 tokens (heads 2t, 2t+1), base 2
    float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      x0 = fmaxf(x0, fmaxf(sc[rt][0], sc[rt][2]));
      x1 = fmaxf(x1, fmaxf(sc[rt][1], sc[rt][3]));
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
      x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
    }
    const float n0m = fmaxf(m0, x0), n1m = fmaxf(m1, x1);
    // rows that are still all -inf keep a zero weight and leave the accumulators alone
    const float b0m = n0m == -INFINITY ? 0.f : n0m, b1m = n1m == -INFINITY ? 0.f : n1m;
    const float corr0 = fast_exp2(m0 - b0m), corr1 = fast_exp2(m1 - b1m);
    const bool rescale = !__all_sync(0xffffffffu, n0m == m0 && n1m == m1);
    m0 = n0m;
    m1 = n1m;
    if (rescale) {
      l0 *= corr0;
      l1 *= corr1;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        O[mt][0] *= corr0;
        O[mt][1] *= corr1;
        O[mt][2] *= corr0;
        O[mt][3] *= corr1;
      }
    }
    const float* vn = reinterpret_cast<const float*>(tb + L.vnorm_off);

    // ---------------- values: row block rt is value chunk rt of the tile
#pragma unroll
    for (int rt = 0; rt < 4; ++rt) {
      const float p0 = fast_exp2(sc[rt][0] - b0m), p1 = fast_exp2(sc[rt][1] - b1m);
      const float p2 = fast_exp2(sc[rt][2] - b0m), p3 = fast_exp2(sc[rt][3] - b1m);
      l0 += p0 + p2;
      l1 += p1 + p3;
      const float av0 = vn[16 * rt + g] * vscale, av1 = vn[16 * rt + g + 8] * vscale;
      const unsigned pb0 = movmatrix_trans(pack_h2(p0 * av0, p1 * av0));
      const unsigned pb1 = movmatrix_trans(pack_h2(p2 * av1, p3 * av1));
      ValueRows<VR> vr;
      vr.load(reinterpret_cast<const unsigned*>(tb + L.vcode_off + rt * 256 * VR), g, t);
      constexpr unsigned vm = (1u << (2 * VR)) - 1u;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        unsigned fx, fy;
        vr.fields(mt, fx, fy);
        mma16816(O[mt], vlut[fx & vm], vlut[fy & vm], vlut[(fx >> (2 * VR)) & vm], vlut[(fy >> (2 * VR)) & vm],
                 pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }

  pdl_trigger();
  // ---------------- merge the consumer warps (their partials reuse the ring: wait until
  // every warp is done with its tiles; after a timeout copies may still be in flight)
  consumer_sync();
  if (*static_cast<volatile int*>(&s_timeout)) return;  // uniform over the consumer warps
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  float* mow = mo + warp * 8 * kD;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {  // row g -> dim 16g + 2mt, row g+8 -> dim 16g + 2mt + 1
    mow[(2 * t) * kD + 16 * g + 2 * mt] = O[mt][0];
    mow[(2 * t + 1) * kD + 16 * g + 2 * mt] = O[mt][1];
    mow[(2 * t) * kD + 16 * g + 2 * mt + 1] = O[mt][2];
    mow[(2 * t + 1) * kD + 16 * g + 2 * mt + 1] = O[mt][3];
  }
  if (g == 0) {
    mm[warp * 8 + 2 * t] = m0;
    mm[warp * 8 + 2 * t + 1] = m1;
    ml[warp * 8 + 2 * t] = l0;
    ml[warp * 8 + 2 * t + 1] = l1;
  }
  consumer_sync();
  const int G = a.G;
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, mm[w * 8 + hh]);
    float o = 0.f, l = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
        const float f = fast_exp2(mm[w * 8 + hh] - M);
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
}

size_t split_smem_bytes(int tile_bytes) {
  return 128 + size_t(kStages) * tile_bytes + 64 + kMaxChunks * 2 * 32 * sizeof(uint2) + 32 * 4 + 320 * 8 + 16 * 8 +
         256 * 4 + 2 * kConsumers * 8 * sizeof(float);
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
  cfg.blockDim = dim3(kThreads);
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
  if (splits > kMaxSplits) splits = kMaxSplits;
  p.tiles_per_split = int((p.max_tiles + splits - 1) / splits);
  p.n_splits = (p.max_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  p.workspace_bytes = workspace_size(units, p.n_splits, G);
  return p;
}

namespace {

cudaError_t set_prep_smem(const void* fn) {
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, fn);
  if (e != cudaSuccess) return e;
  if (attr.maxDynamicSharedSizeBytes >= int((kD * kD + 2 * kMaxG * kD) * sizeof(float))) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int((kD * kD + 2 * kMaxG * kD) * sizeof(float)));
}

cudaError_t launch_attention(const DevLayout& L, const DecodePlan& plan, int batch, int h_q, int h_kv,
                             const void* cache, const int* seq_lens, long long n_tiles, float* out,
                             const Workspace& ws, int len_add, int wait_before_copy, cudaStream_t stream) {
  const int G = h_q / h_kv;
  const long long units = (long long)batch * h_kv;
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
  a.len_add = len_add;
  a.wait_before_copy = wait_before_copy;
  dim3 grid(plan.n_splits, unsigned(units));
  cudaError_t e;
  switch (L.v_rate) {
    case 1: e = launch_split<1>(L, a, grid, stream); break;
    case 2: e = launch_split<2>(L, a, grid, stream); break;
    case 3: e = launch_split<3>(L, a, grid, stream); break;
    case 4: e = launch_split<4>(L, a, grid, stream); break;
    default: e = cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(batch * h_q));
  cfg.blockDim = dim3(kCombThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, (const float*)ws.part_ml, (const float*)ws.part_o, plan.n_splits,
                            G, h_q, h_kv, L.v_rot32, out);
}

}  // namespace

cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, const void* cache, const int* seq_lens, long long n_tiles,
                          float softmax_scale, float* out, void* workspace, cudaStream_t stream) {
  const int G = h_q / h_kv;
  const long long units = (long long)batch * h_kv;
  Workspace ws = carve(workspace, units, plan.n_splits, G);
  cudaError_t e = set_prep_smem((const void*)qprep_kernel);
  if (e != cudaSuccess) return e;
  qprep_kernel<<<unsigned(units), kPrepThreads, prep_smem_bytes(L), stream>>>(L, q, q_dtype, h_q, h_kv, G,
                                                                              softmax_scale * kLog2e, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the cache is not written by qprep: the split kernel may start copying tiles at once
  return launch_attention(L, plan, batch, h_q, h_kv, cache, seq_lens, n_tiles, out, ws, 0, 0, stream);
}

cudaError_t launch_decode_step(const DevLayout& L, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, int n_new, const int* seq_lens_before, const void* q, int q_dtype,
                               int batch, int h_q, int h_kv, void* cache, long long n_tiles, float softmax_scale, float* out, void* workspace,
                               cudaStream_t stream) {
  const int G = h_q / h_kv;
  const long long units = (long long)batch * h_kv;
  Workspace ws = carve(workspace, units, plan.n_splits, G);
  cudaError_t e = set_prep_smem((const void*)step_prep_kernel);
  if (e != cudaSuccess) return e;
  const long long n_enc = (long long)n_new * kEncodeParts * batch * h_kv;
  step_prep_kernel<<<unsigned(n_enc + units), kPrepThreads, prep_smem_bytes(L), stream>>>(
      L, k_new, v_new, kv_dtype, n_new, batch, n_tiles, seq_lens_before, static_cast<uint8_t*>(cache), q, q_dtype,
      h_q, h_kv, G, softmax_scale * kLog2e, ws, int(n_enc));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, cache, seq_lens_before, n_tiles, out, ws, n_new, 1, stream);
}

}  // namespace bgtq
