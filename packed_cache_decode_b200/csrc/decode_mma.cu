// Decode attention over the packed cache on tensor cores (sm_100a).
//
// "Block-GTQ" abstract, sentence 5: attention reads the packed codes directly, no decoded
// fp16 KV cache is ever written. With R_g orthogonal,
//   q . k_hat   = sum_g (|k_g| / sqrt(d_g)) (R_g q_g) . c[codes_g]
//   o           = R_V^T sum_t p_t (|v_t| / sqrt(128)) c[vcodes_t] / sum_t p_t.
//
// Three kernels per call, chained by programmatic dependent launch:
//  * qprep_kernel (one CTA per batch row x KV head; in a decode step, step_prep_kernel also
//    runs the encode CTAs of the new tokens): q' = R_g q_g for the G query columns of the
//    KV head (fp32, scaled by softmax_scale * log2(e) / (sqrt(d_g) kappa_g)), split into
//    fp16 hi + lo parts and laid out as mma B fragments. A column is one query head at
//    one query token: G = query heads per KV head x n_q query tokens (n_q = 1 except in
//    multi-token calls).
//  * split_kernel: the (batch row, KV head) caches are laid end to end as one sequence of
//    64-token tiles and every CTA takes an equal slice of it (one or two units' worth), so
//    the grid is one balanced wave. 4 warps, no producer warp: warp w streams its own tiles
//    w, w+4, ... through a private pair of ring stages with 1-D bulk async copies
//    (cp.async.bulk + mbarrier, L2 evict-first, no multicast), contiguous or paged; one or
//    two tiles left over after a multiple of four go out as half tiles (row blocks 0-1 and
//    2-3 to two warps). The CTA starts (tables, first copies) while q-prep runs and waits
//    only before loading the q' fragments. Keys: per quad of 4 dimension pairs one load
//    gives the lane its codes for its 8 tokens (fragment-major format); rate 1 turns into
//    +-1 pairs with bit operations, rates 2-4 index pair tables in shared memory
//    (lane-private for rate 2, hi + lo parts for rates 3-4); a group's quads go in pairs
//    into mma.m16n8k16 (for G <= 4 the q' hi and lo parts are the eight columns of one
//    product). fp32 accumulators per group, then times the group norm (fp32 or fp16, a
//    template variant). Each column masks the tokens past its own position (the row's
//    last tiles only). Online softmax in base 2 with warp shuffles. Values: the
//    probabilities times |v|/sqrt(128) in fp16, transposed with movmatrix, against
//    value-code pair lookups in m16n8k16 products, accumulated in V's rotated space
//    (fp32). Per unit the four warps merge and the CTA writes its partial (o', m, l). A
//    scores-only form writes the logits instead.
//  * combine_kernel (one CTA per batch row x query column, 512 threads): log-sum-exp merge
//    of the unit's partials and o = R_V^T o', written to out[b][token][head].
// After an append (bgtq_decode_step) only the tile that receives the new tokens waits for
// the encode before it is copied. With norm correction the step's encode CTAs run as
// clusters of four (their launch pads the grid to whole clusters).
//
// Every mbarrier wait is bounded; on timeout the kernel records BGTQ_STATUS_TIMEOUT, waits
// (bounded) for its own copies in flight and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <utility>

#include "bgtq_internal.h"
#include "encode_body.cuh"
#include "kernels.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
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
// L2 policy for data read once per step (the packed tiles): evicted first, so that the
// small per-layer constants (rotations) stay in L2 from one step to the next.
__device__ __forceinline__ unsigned long long evict_first_policy() {
  unsigned long long pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, unsigned long long* bar,
                                          unsigned long long policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
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
__device__ __forceinline__ float load_q(const void* p, int dtype, size_t i) {
  if (dtype == BGTQ_F32) return static_cast<const float*>(p)[i];
  if (dtype == BGTQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(static_cast<const __half*>(p)[i]);
}

constexpr int kMaxParts = 1024;      // partial slots per unit the combine can merge
constexpr int kCtasPerSm = 3;        // split CTAs resident per SM (registers, shared memory)
constexpr int kMaxTileBytes = kTile * (2 * kD * 4 / 8 + 4 * (kMaxGroups + 1));  // K4V4, four groups

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline size_t qfrag_bytes(long long units) { return align256(size_t(units) * kMaxQuads * 64 * sizeof(unsigned)); }

// ------------------------------------------------------------------ split kernel
struct SplitArgs {
  CacheRef cache;
  const int* seq_lens;
  const unsigned* qfrag;  // [units][kMaxQuads][2][32] q' B fragments from the preparation kernel
  int max_tiles;          // M: tiles per unit covered by the plan
  int n_ctas;             // CTAs; CTA c takes tiles [c T / n_ctas, (c+1) T / n_ctas) of the sequence
  int n_parts;            // partial slots per unit
  long long total_tiles;  // units x M
  int h_q, h_kv, G;       // G: query columns per KV head (query heads per KV head x n_q)
  int n_q;                // query tokens per row; column n is query token n % n_q
  float* part_ml;         // [units][n_parts][G][2]
  float* part_o;          // [units][n_parts][G][128]
  float* scores;          // scores-only mode: [batch][h_q][scores_ld] logits (softmax_scale q.k_hat)
  long long scores_ld;
  int len_add;            // tokens appended by the previous kernel: row b attends over seq_lens[b] + len_add
  int wait_new;           // the previous kernel appends at seq_lens[b]: wait for it before copying that tile
};

constexpr int kWarps = 4;                        // warps, one whole 64-token tile at a time each
constexpr int kThreads = 32 * kWarps;
constexpr int kRing = 2 * kWarps;                // ring stages: two per warp
constexpr int kQsLd = kD + 16;                   // row of q staged per group at 16-byte aligned offsets

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void mma1688(float (&c)[4], unsigned a0, unsigned a1, unsigned b0) {
  asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(b0));
}

// +-1 pair from two 1-bit codes sitting at bits 15 and 31 of x (bit 1 -> +1, 0 -> -1):
// the sign bit is the inverted code, the magnitude is fp16 1.0.
__device__ __forceinline__ unsigned sign_pair(unsigned x) { return (~x & 0x80008000u) | 0x3C003C00u; }
__device__ __forceinline__ unsigned prmt(unsigned a, unsigned b, unsigned sel) {
  unsigned d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Table reads at a byte offset. Lane-private tables keep entry e of lane l at word
// 32 e + l, so the 32 lanes of a lookup always hit 32 different banks.
__device__ __forceinline__ unsigned lds_u32(const unsigned* base, unsigned boff) {
  return *reinterpret_cast<const unsigned*>(reinterpret_cast<const unsigned char*>(base) + boff);
}
__device__ __forceinline__ uint2 lds_u64(const uint2* base, unsigned boff) {
  return *reinterpret_cast<const uint2*>(reinterpret_cast<const unsigned char*>(base) + boff);
}
// x >> s for an s that is known after unrolling and may be negative (a left shift).
__device__ __forceinline__ unsigned shr(unsigned x, int s) { return s >= 0 ? x >> s : x << -s; }

// Shared-memory tables of one CTA.
// A compile-time int carried as a value (row blocks per work item).
template <int N>
struct IntC {
  static constexpr int value = N;
};

template <int VR>
struct Luts {
  static constexpr int kV = VR == 2 ? 16 * 32 : VR == 3 ? 64 * 32 : VR == 4 ? 256 : 1;
  unsigned k2[16 * 32];  // rate-2 key pairs, lane-private
  uint2 k3[64];          // rate-3 key pairs {hi, lo}
  uint2 k4[256];         // rate-4 key pairs {hi, lo}
  unsigned v[kV];        // value pairs: rates 2-3 lane-private, rate 4 shared
};

// The lane's codes of one quad: Kq<R>::load reads them (rate 3: two planes) at the lane's
// precomputed byte offsets, a(m) gives the fp16 pair (hi part for rates 3-4) of slot m
// (token g + 8 m of the tile, dims 2t and 2t+1 of the quad), lo(m) the low parts.
template <int R, int VR>
struct Kq;
template <int VR>
struct Kq<1, VR> {
  unsigned w;  // lo codes in bits 8-15, hi codes in bits 24-31
  __device__ __forceinline__ void load(const unsigned char* tb, unsigned off, bool up = false) {
    w = prmt(*reinterpret_cast<const unsigned short*>(tb + (off & 0xffffu)), 0u, 0x1404u);
    if (up) w >>= 4;
  }
  __device__ __forceinline__ unsigned a(int m, const Luts<VR>&, unsigned) const { return sign_pair(w << (7 - m)); }
  __device__ __forceinline__ unsigned lo(int, const Luts<VR>&) const { return 0u; }
};
template <int VR>
struct Kq<2, VR> {
  unsigned w;  // nibble m = lo | hi << 2
  __device__ __forceinline__ void load(const unsigned char* tb, unsigned off, bool up = false) {
    w = *reinterpret_cast<const unsigned*>(tb + (off & 0xffffu));
    if (up) w >>= 16;
  }
  __device__ __forceinline__ unsigned a(int m, const Luts<VR>& T, unsigned lane4) const {
    return lds_u32(T.k2, (shr(w, 4 * m - 7) & 0x780u) | lane4);  // entry at 128 nibble + 4 lane
  }
  __device__ __forceinline__ unsigned lo(int, const Luts<VR>&) const { return 0u; }
};
template <int VR>
struct Kq<3, VR> {
  unsigned f[8];  // byte offsets (8 x field) of the eight 6-bit fields in the pair table
  uint2 e[8];
  __device__ __forceinline__ void load(const unsigned char* tb, unsigned off, bool up = false) {
    unsigned wa = *reinterpret_cast<const unsigned*>(tb + (off & 0xffffu));
    const unsigned wb = *reinterpret_cast<const unsigned short*>(tb + (off >> 16));
    if (up) wa = (wa >> 24) | (wb << 8);  // fields 4..7 to 0..3 (only those are used then)
    f[0] = (wa << 3) & 0x1f8u;
    f[1] = (wa >> 3) & 0x1f8u;
    f[2] = (wa >> 9) & 0x1f8u;
    f[3] = (wa >> 15) & 0x1f8u;
    f[4] = (wa >> 21) & 0x1f8u;
    f[5] = (__funnelshift_r(wa, wb, 30) << 3) & 0x1f8u;
    f[6] = (wb >> 1) & 0x1f8u;
    f[7] = (wb >> 7) & 0x1f8u;
  }
  __device__ __forceinline__ unsigned a(int m, const Luts<VR>& T, unsigned) { e[m] = lds_u64(T.k3, f[m]); return e[m].x; }
  __device__ __forceinline__ unsigned lo(int m, const Luts<VR>&) const { return e[m].y; }
};
template <int VR>
struct Kq<4, VR> {
  uint2 w;  // byte m = lo | hi << 4
  uint2 e[8];
  __device__ __forceinline__ void load(const unsigned char* tb, unsigned off, bool up = false) {
    w = *reinterpret_cast<const uint2*>(tb + (off & 0xffffu));
    if (up) w.x = w.y;
  }
  __device__ __forceinline__ unsigned a(int m, const Luts<VR>& T, unsigned) {
    const unsigned x = m < 4 ? w.x : w.y;
    e[m] = lds_u64(T.k4, shr(x, 8 * (m & 3) - 3) & 0x7f8u);
    return e[m].x;
  }
  __device__ __forceinline__ unsigned lo(int m, const Luts<VR>&) const { return e[m].y; }
};

// Scores of one key group with compile-time rate R over its quads [q0, q1) of a tile.
// Quads go in pairs into m16n8k16 products (quad q: k columns 0-7, quad q+1: 8-15); a
// group's odd last quad takes an m16n8k8 product. Row block rt of the tile: rows g and
// g+8 are slots m = 2 rt and 2 rt + 1. loff[q][lane] = byte offset of the lane's codes in
// the tile (for a lane without a pair of that quad: any code, its q' rows are zero).
// NRT = 4: the whole tile; NRT = 2: the half tile of row blocks 0-1 (up = false) or 2-3.
template <int R, bool NP, int VR, int NRT>
__device__ __forceinline__ void key_group(float (&acc)[NRT][4], const unsigned char* tb, const unsigned* loff,
                                          const unsigned* qf, int q0, int q1, int lane, const Luts<VR>& T,
                                          bool up) {
  const unsigned lane4 = unsigned(lane) << 2;
  int q = q0;
#pragma unroll 1
  for (; q + 1 < q1; q += 2) {
    Kq<R, VR> c0, c1;
    c0.load(tb, loff[q * 32 + lane], NRT < 4 && up);
    c1.load(tb, loff[(q + 1) * 32 + lane], NRT < 4 && up);
    const unsigned bh0 = qf[q * 64 + lane], bh1 = qf[(q + 1) * 64 + lane];
    const unsigned bl0 = NP ? 0u : qf[q * 64 + 32 + lane], bl1 = NP ? 0u : qf[(q + 1) * 64 + 32 + lane];
#pragma unroll
    for (int rt = 0; rt < NRT; ++rt) {
      const unsigned a0 = c0.a(2 * rt, T, lane4), a1 = c0.a(2 * rt + 1, T, lane4);
      const unsigned a2 = c1.a(2 * rt, T, lane4), a3 = c1.a(2 * rt + 1, T, lane4);
      mma16816(acc[rt], a0, a1, a2, a3, bh0, bh1);
      if constexpr (!NP) mma16816(acc[rt], a0, a1, a2, a3, bl0, bl1);
      if constexpr (R >= 3)
        mma16816(acc[rt], c0.lo(2 * rt, T), c0.lo(2 * rt + 1, T), c1.lo(2 * rt, T), c1.lo(2 * rt + 1, T), bh0, bh1);
    }
  }
  if (q < q1) {
    Kq<R, VR> c0;
    c0.load(tb, loff[q * 32 + lane], NRT < 4 && up);
    const unsigned bh = qf[q * 64 + lane], bl = NP ? 0u : qf[q * 64 + 32 + lane];
#pragma unroll
    for (int rt = 0; rt < NRT; ++rt) {
      const unsigned a0 = c0.a(2 * rt, T, lane4), a1 = c0.a(2 * rt + 1, T, lane4);
      mma1688(acc[rt], a0, a1, bh);
      if constexpr (!NP) mma1688(acc[rt], a0, a1, bl);
      if constexpr (R >= 3) mma1688(acc[rt], c0.lo(2 * rt, T), c0.lo(2 * rt + 1, T), bh);
    }
  }
}

// Value A fragments of one 16-token chunk: the lane's 64 VR-bit string (one or two
// loads) holds 32 fields n = 4 mt + k, each the fp16 pair of A register k of m-tile mt.
template <int VR>
struct ValueLane {
  unsigned w[2 * VR];
  __device__ __forceinline__ void load(const unsigned char* vblk, int lane) {
    if constexpr (VR == 1) {
      const uint2 x = reinterpret_cast<const uint2*>(vblk)[lane];
      w[0] = x.x;
      w[1] = x.y;
    } else {
      const uint4 x = reinterpret_cast<const uint4*>(vblk)[lane];
      w[0] = x.x;
      w[1] = x.y;
      w[2] = x.z;
      w[3] = x.w;
      if constexpr (VR == 3) {
        const uint2 y = reinterpret_cast<const uint2*>(vblk + 512)[lane];
        w[4] = y.x;
        w[5] = y.y;
      } else if constexpr (VR == 4) {
        const uint4 y = reinterpret_cast<const uint4*>(vblk + 512)[lane];
        w[4] = y.x;
        w[5] = y.y;
        w[6] = y.z;
        w[7] = y.w;
      }
    }
  }
  // fp16 pair of field n (compile-time after unrolling)
  __device__ __forceinline__ unsigned field(int n, const unsigned* vlut, unsigned lane4) const {
    if constexpr (VR == 1) {
      return sign_pair(w[n >> 4] << (15 - (n & 15)));
    } else if constexpr (VR == 2) {
      return lds_u32(vlut, (shr(w[n >> 3], 4 * (n & 7) - 7) & 0x780u) | lane4);
    } else if constexpr (VR == 3) {
      const int bit = 6 * n, wi = bit >> 5, sh = bit & 31;
      const unsigned x = sh <= 26 ? (w[wi] >> sh) : __funnelshift_r(w[wi], w[wi + 1], sh);
      return lds_u32(vlut, ((x & 63u) << 7) | lane4);
    } else {
      return lds_u32(vlut, shr(w[n >> 2], 8 * (n & 3) - 2) & 0x3fcu);
    }
  }
};

// The slice of CTA c: tiles [c T / C, (c+1) T / C) of the units x M = T tiles laid end to
// end (C CTAs, C <= T, slices at most M long), i.e. one or two segments, each a tile range
// of one unit (clipped to the unit's length when streamed).
__host__ __device__ inline int cta_of_tile(long long x, long long T, long long C) { return int(((x + 1) * C - 1) / T); }

struct Segment {
  int u;        // unit = batch row * h_kv + KV head
  int lt0;      // first tile (inside the unit) of the slice
  int n;        // tiles to stream (after clipping to the unit's length)
  int part;     // partial slot of this CTA for the unit
  long long len;  // tokens of the unit
};

__device__ __forceinline__ int cta_segments(const DevLayout& L, const SplitArgs& a, int c, Segment* seg, int tid) {
  const long long M = a.max_tiles, T = a.total_tiles, C = a.n_ctas;
  const long long g0 = (long long)c * T / C, g1 = (long long)(c + 1) * T / C;
  const int u0 = int(g0 / M), u1 = int((g1 - 1) / M);
  int nseg = 0;
  for (int u = u0; u <= u1 && nseg < 2; ++u, ++nseg) {
    const int b = u / a.h_kv;
    long long len = (long long)a.seq_lens[b] + a.len_add;
    if (len < 0) len = 0;
    const long long cap_tokens = min(a.cache.n_tiles, M) * kTile;
    const long long a0 = max(g0, (long long)u * M) - (long long)u * M;
    const long long a1 = min(g1, (long long)(u + 1) * M) - (long long)u * M;
    if (len > cap_tokens) {
      if (tid == 0 && a0 == 0) atomicOr(L.status, BGTQ_STATUS_DECODE_CLAMPED);
      len = cap_tokens;
    }
    const long long len_tiles = (len + kTile - 1) / kTile;
    seg[nseg].u = u;
    seg[nseg].lt0 = int(a0);
    seg[nseg].n = int(max(0LL, min(a1, len_tiles) - a0));
    seg[nseg].part = c - cta_of_tile((long long)u * M, T, C);
    seg[nseg].len = len;
  }
  return nseg;
}

// q' B fragments of unit u (batch row b, KV head h) into frag[kMaxQuads][2][32] (global),
// by one CTA of kPrepThreads: thread (p = tid % 128, half = tid / 128) computes
// q'[hh][p] = f_g sum_j R_g[i][j] q[hh][off_g + j] for the heads hh = 4 half .. 4 half + 3
// (16-byte rows of R_g from global memory, q staged in shared memory); with G <= 4 the
// two halves take heads 0..3 over the two halves of the row instead (all of a thread's
// row is then loaded before q arrives) and add up in shared memory. Then every fragment
// word is written once. With G <= 4 the eight B columns are heads 0..3 (hi
// parts) and heads 0..3 again (lo parts) in the first array; otherwise the first array
// holds the hi parts of heads 0..7 and the second the lo parts. Missing pairs and heads
// are zero.
constexpr int kPrepThreads = 256;
static_assert(kPrepThreads == enc::kEncodeThreads, "the step kernel runs both bodies");

__device__ __forceinline__ void prep_unit(const DevLayout& L, const void* __restrict__ q, int q_dtype, int h_q,
                                          int h_kv, int G, int n_q, float qscale, int u, unsigned* __restrict__ frag) {
  __shared__ __align__(16) float qs[kMaxG * kQsLd];  // q per group at 16-byte aligned columns
  __shared__ float qr[kMaxG * kD];                   // q' in packed order
  const int tid = threadIdx.x, ng = L.n_kgroups;
  const int b = u / h_kv, h = u % h_kv;
  __shared__ float red[4 * kD];                      // the k-split halves' partial sums
  // this thread's row of R_g (columns [4 c0, 4 c1)): the first 16 float4 are loaded
  // before q arrives
  const int p = tid & (kD - 1), half = tid >> 7;
  const bool ksplit = G <= 4;
  const int h0 = ksplit ? 0 : half * 4;
  int g = 0, pad = 0;
  while (g + 1 < ng && p >= L.group_off[g + 1]) pad += L.k_rot32_ld[g++];
  const int d = L.group_dim[g], i = p - L.group_off[g], ld = L.k_rot32_ld[g];
  // packed dims past n_packed (rate-0 blocks) have no row: no loads, q' = 0
  const int n4 = p < L.n_packed ? ld / 4 : 0, c0 = ksplit ? half * ((n4 + 1) / 2) : 0, c1 = ksplit ? min(n4, c0 + (n4 + 1) / 2) : n4;
  const float4* row = reinterpret_cast<const float4*>(L.k_rot32[g] + (size_t)i * ld) + c0;
  constexpr int kPre = 16;
  float4 r[kPre];
#pragma unroll
  for (int j4 = 0; j4 < kPre; ++j4) r[j4] = c0 + j4 < c1 ? __ldg(row + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int e = tid; e < kMaxG * kQsLd; e += kPrepThreads) qs[e] = 0.f;
  __syncthreads();
  // in a decode step (launched as a programmatic dependent) the CTA got here, rows of R in
  // flight, while the kernel before it ran; q is the caller's: wait for that kernel before
  // reading it. Only then may the split kernel launch: it reads the cache, which that
  // kernel may write. (q-prep alone is a plain launch: both are no-ops there.)
  pdl_wait();
  pdl_trigger();
  for (int e = tid; e < G * kD; e += kPrepThreads) {
    const int hh = e >> 7, pe = e & (kD - 1);
    if (pe >= L.n_packed) continue;
    int ge = 0, pade = 0;
    while (ge + 1 < ng && pe >= L.group_off[ge + 1]) pade += L.k_rot32_ld[ge++];
    // column hh: query head h G / n_q + hh / n_q at query token hh % n_q of q [b][token][head]
    const size_t qrow = ((size_t)b * n_q + hh % n_q) * h_q + (size_t)h * (G / n_q) + hh / n_q;
    qs[hh * kQsLd + pade + pe - L.group_off[ge]] = load_q(q, q_dtype, qrow * kD + L.packed_coord[pe]);
  }
  __syncthreads();
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (h0 < G) {
    const float* qg = qs + h0 * kQsLd + pad + 4 * c0;
#pragma unroll
    for (int j4 = 0; j4 < kPre; ++j4) {
      if (c0 + j4 < c1) {  // q columns past the group's padded row are not read
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 x = *reinterpret_cast<const float4*>(qg + k * kQsLd + 4 * j4);
          acc[k] = fmaf(r[j4].x, x.x, fmaf(r[j4].y, x.y, fmaf(r[j4].z, x.z, fmaf(r[j4].w, x.w, acc[k]))));
        }
      }
    }
#pragma unroll 8
    for (int j4 = kPre; c0 + j4 < c1; ++j4) {
      const float4 rr = __ldg(row + j4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 x = *reinterpret_cast<const float4*>(qg + k * kQsLd + 4 * j4);
        acc[k] = fmaf(rr.x, x.x, fmaf(rr.y, x.y, fmaf(rr.z, x.z, fmaf(rr.w, x.w, acc[k]))));
      }
    }
  }
  if (ksplit) {  // uniform over the CTA
    if (half == 1)
#pragma unroll
      for (int k = 0; k < 4; ++k) red[k * kD + p] = acc[k];
    __syncthreads();
    if (half == 0)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] += red[k * kD + p];
  }
  if (h0 < G && (!ksplit || half == 0)) {
    const float f = qscale * rsqrtf(float(d)) * L.inv_kappa_group[g];  // the key tables carry kappa
#pragma unroll
    for (int k = 0; k < 4; ++k) qr[(h0 + k) * kD + p] = acc[k] * f;
  }
  __syncthreads();
  for (int e = tid; e < L.n_kquads * 64; e += kPrepThreads) {
    const int qi = e >> 6, j = e & 63, lane = j & 31, n = lane >> 2, t = lane & 3;
    const bool lo_half = j >= 32;
    const int d0 = L.quad_dim0[qi] + 2 * t;
    const int hh = G <= 4 ? (n & 3) : n;
    const bool lo = G <= 4 ? n >= 4 : lo_half;
    float v0 = 0.f, v1 = 0.f;
    if (t < L.quad_np[qi] && hh < G && !(G <= 4 && lo_half)) {
      v0 = qr[hh * kD + d0];
      v1 = qr[hh * kD + d0 + 1];
    }
    const float r0 = __half2float(__float2half_rn(v0)), r1 = __half2float(__float2half_rn(v1));
    frag[qi * 64 + j] = lo ? pack_h2(v0 - r0, v1 - r1) : pack_h2(r0, r1);
  }
}

__global__ void __launch_bounds__(kPrepThreads) qprep_kernel(DevLayout L, const void* __restrict__ q, int q_dtype,
                                                             int h_q, int h_kv, int G, int n_q, float qscale,
                                                             unsigned* __restrict__ qfrag) {
  // launched after the kernel before it has completed: the split kernel may start now
  pdl_trigger();
  const int u = blockIdx.x;
  prep_unit(L, q, q_dtype, h_q, h_kv, G, n_q, qscale, u, qfrag + (size_t)u * kMaxQuads * 64);
}

// First kernel of a decode step: blocks [0, n_enc) append the new tokens (four blocks per
// token and KV head), the others prepare q' of one unit each.
template <bool NC>
__global__ void __launch_bounds__(kPrepThreads) step_prep_kernel(DevLayout L, const void* __restrict__ k,
                                                                 const void* __restrict__ v, int kv_dtype, int n_new,
                                                                 int batch, const int* __restrict__ seq_lens_before,
                                                                 CacheRef cache,
                                                                 const void* __restrict__ q, int q_dtype, int h_q,
                                                                 int h_kv, int G, int n_q, float qscale,
                                                                 unsigned* __restrict__ qfrag, int n_enc) {
  // every block triggers its dependent (the split kernel) after its own wait for the
  // kernel before it (in the encode and q-prep bodies; padding blocks by exiting)
  const int e = blockIdx.x;
  if (e < n_enc) {
    const int part = e % kEncodeParts;
    int rest = e / kEncodeParts;
    const int t = rest % n_new;
    rest /= n_new;
    const int b = rest % batch, h = rest / batch;
    enc::encode_token_part<NC>(L, k, v, kv_dtype, n_new, h_kv, seq_lens_before, cache, t, part, b, h);
  } else if (e - n_enc < batch * h_kv) {  // (a cluster launch pads the grid)
    const int u = e - n_enc;
    prep_unit(L, q, q_dtype, h_q, h_kv, G, n_q, qscale, u, qfrag + (size_t)u * kMaxQuads * 64);
  }
}

// Norm i of a tile's norm area, stored as fp16 (NH) or fp32.
template <bool NH>
__device__ __forceinline__ float tile_norm(const unsigned char* area, int i) {
  if constexpr (NH) return __half2float(reinterpret_cast<const __half*>(area)[i]);
  else return reinterpret_cast<const float*>(area)[i];
}

// SC: scores only. The tiles' logits (softmax_scale q . k_hat, natural units) go to
// a.scores; no softmax, values, partials or merge. NH: the layout stores fp16 norms.
// (the scores-only instantiation discards the softmax and value code of the tile body)
#pragma nv_diag_suppress 128
template <int VR, bool NP, bool SC, bool NH>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) split_kernel(DevLayout L, SplitArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(16) Luts<VR> T;
  __shared__ unsigned s_loff[kMaxQuads * 32];  // [quad][lane]: byte offsets of the lane's codes in a tile
  __shared__ int s_group[kMaxGroups][3];      // first quad, end quad, rate
  __shared__ int s_timeout;
  __shared__ Segment s_seg[2];
  __shared__ int s_nseg;
  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int TB = L.tile_bytes;

  unsigned long long* full = reinterpret_cast<unsigned long long*>(smem);  // [kRing]
  unsigned char* ring = smem + 128;                                        // stage s at ring + s TB
  unsigned* qf = reinterpret_cast<unsigned*>(ring + kRing * TB);           // [quad][2][32]
  float* mm = reinterpret_cast<float*>(qf + L.n_kquads * 64);              // [warp][8]
  float* ml = mm + kWarps * 8;                                             // [warp][8]
  // the warps' [8][128] partials reuse the ring once every tile of the segment is consumed
  float* mo = reinterpret_cast<float*>(ring);

  if (tid == 0) {
    s_timeout = 0;
    s_nseg = cta_segments(L, a, c, s_seg, 0);
    for (int i = 0; i < kRing; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  // pair tables from the layout's fp16 codebooks: only those of the rates it uses
  unsigned has = 0;
  for (int gi = 0; gi < L.n_kgroups; ++gi) has |= 1u << L.group_rate[gi];
  if (has & 4u)
    for (int i = tid; i < 16 * 32; i += kThreads) {
      const int e = i >> 5;
      T.k2[i] = unsigned(L.kc2[e & 3]) | (unsigned(L.kc2[e >> 2]) << 16);
    }
  if (has & 8u)
    for (int e = tid; e < 64; e += kThreads)
      T.k3[e] = make_uint2(unsigned(L.kc3[0][e & 7]) | (unsigned(L.kc3[0][e >> 3]) << 16),
                           unsigned(L.kc3[1][e & 7]) | (unsigned(L.kc3[1][e >> 3]) << 16));
  if (has & 16u)
    for (int e = tid; e < 256; e += kThreads)
      T.k4[e] = make_uint2(unsigned(L.kc4[0][e & 15]) | (unsigned(L.kc4[0][e >> 4]) << 16),
                           unsigned(L.kc4[1][e & 15]) | (unsigned(L.kc4[1][e >> 4]) << 16));
  if constexpr (VR == 2 || VR == 3) {
    // lane-private pair tables: entry e of lane l at 32 e + l (no bank conflicts)
    constexpr unsigned vm = (1u << VR) - 1u;
    for (int i = tid; i < Luts<VR>::kV; i += kThreads) {
      const int e = i >> 5;
      T.v[i] = unsigned(L.vc[e & vm]) | (unsigned(L.vc[e >> VR]) << 16);
    }
  } else if constexpr (VR == 4) {
    for (int e = tid; e < 256; e += kThreads) T.v[e] = unsigned(L.vc[e & 15]) | (unsigned(L.vc[e >> 4]) << 16);
  }
  for (int gi = 0; gi < L.n_kgroups; ++gi) {
    const int r = L.group_rate[gi], q0 = L.group_quad0[gi];
    for (int i = tid; i < L.group_nquads[gi] * 32; i += kThreads) {
      // lane (g, t) holds pair t of the quad for tokens g + 8m: its 16 r bits are string
      // li = g P + t of the block (rate 3: plane A word li, plane B halfword li after 8 P words)
      const int qi = q0 + i / 32, ln = i % 32, P = L.quad_np[qi], t = ln & 3;
      const int li = t < P ? (ln >> 2) * P + t : 0;
      const unsigned base = unsigned(L.quad_off[qi]);
      s_loff[qi * 32 + ln] = r == 3 ? (base + 4u * li) | ((base + 32u * P + 2u * li) << 16) : base + 2u * r * li;
    }
  }
  if (tid < L.n_kgroups) {
    s_group[tid][0] = L.group_quad0[tid];
    s_group[tid][1] = L.group_quad0[tid] + L.group_nquads[tid];
    s_group[tid][2] = L.group_rate[tid];
  }
  __syncthreads();
  const int nseg = s_nseg;

  // Warp w streams its own tiles w, w+4, w+8, ... of a segment through the two ring stages
  // w and w+4 (its k-th tile in stage w + 4 (k & 1)): lane 0 issues tile k+2 as soon as
  // the warp is done with tile k, so no other warp ever waits on these stages.
  const int ng = L.n_kgroups;
  const float vscale = rsqrtf(float(kD)) / L.kappa_v;
  const unsigned lane4 = unsigned(lane) << 2;
  const unsigned long long l2_stream = evict_first_policy();
  unsigned phase = 0;   // bit k&1: parity of the next completion of stage w + 4 (k & 1)
  unsigned pend = 0;    // bit k&1: a copy into stage w + 4 (k & 1) is in flight
  bool waited = !a.wait_new;
  for (int si = 0; si < nseg; ++si) {
    const Segment S = s_seg[si];
    const int srow = S.u / a.h_kv, shead = S.u % a.h_kv;
    const long long first_new = waited ? 0 : a.seq_lens[S.u / a.h_kv];
    // Work items of this warp: full tiles w, w+4, ... of the first 4 floor(n/4); of the
    // n % 4 tiles left, one each for warps 0-2 if three are left, else half tiles (row
    // blocks 0-1 or 2-3), so that no warp runs more than half a tile past the others.
    // Both warps of a split tile copy all of it into their own stages.
    const int nfw = S.n >> 2, rem = S.n & 3;
    const bool extra = rem == 3 ? warp < 3 : rem == 2 ? true : rem == 1 ? warp < 2 : false;
    const int mine = nfw + (extra ? 1 : 0);
    auto item_tile = [&](int k) {
      return (k < nfw || rem == 3) ? warp + kWarps * k : kWarps * nfw + (rem == 2 ? (warp >> 1) : 0);
    };
    auto issue = [&](int k) {  // lane 0 only
      const int it = S.lt0 + item_tile(k);
      if (!waited && (long long)(it + 1) * kTile > first_new) {
        pdl_wait();  // this tile receives tokens from the encode kernel
        waited = true;
      }
      const int st = warp + kWarps * (k & 1);
      const uint8_t* src = tile_ptr(a.cache, L, srow, shead, a.h_kv, it);
      if (src) {
        mbar_expect_tx(&full[st], TB);
        bulk_load(ring + st * TB, src, TB, &full[st], l2_stream);
      } else {
        mbar_expect_tx(&full[st], 0);  // a page outside the pool (flagged): the stage keeps old bytes
      }
    };
    if (lane == 0)
      for (int k = 0; k < min(2, mine); ++k) issue(k);
    pend = mine >= 2 ? 3u : mine == 1 ? 1u : 0u;
    if (si == 0) pdl_wait();  // q' fragments come from the preparation kernel
    {
      const uint4* src4 = reinterpret_cast<const uint4*>(a.qfrag + (size_t)S.u * kMaxQuads * 64);
      for (int e = tid; e < L.n_kquads * 16; e += kThreads) reinterpret_cast<uint4*>(qf)[e] = src4[e];
    }
    __syncthreads();

    float O[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int j = 0; j < 4; ++j) O[mt][j] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    // Row blocks rb0 .. rb0 + NRT - 1 of the tile in stage tb; gt0 = token of row g of
    // row block rb0.
    auto rows = [&](auto nrt, const unsigned char* tb, int rb0, long long gt0) {
      constexpr int NRT = decltype(nrt)::value;
      const bool up = rb0 != 0;

      // ---------------- scores: per key group (rate as a template parameter), per quad,
      // NRT row blocks; then times the group norms
      const unsigned char* kna = tb + L.knorm_off;
      float sc[NRT][4];
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[rt][j] = 0.f;
      for (int gi = 0; gi < ng; ++gi) {
        float acc[NRT][4];
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[rt][j] = 0.f;
        const int q0 = s_group[gi][0], q1 = s_group[gi][1];
        switch (s_group[gi][2]) {
          case 1: key_group<1, NP, VR, NRT>(acc, tb, s_loff, qf, q0, q1, lane, T, up); break;
          case 2: key_group<2, NP, VR, NRT>(acc, tb, s_loff, qf, q0, q1, lane, T, up); break;
          case 3: key_group<3, NP, VR, NRT>(acc, tb, s_loff, qf, q0, q1, lane, T, up); break;
          default: key_group<4, NP, VR, NRT>(acc, tb, s_loff, qf, q0, q1, lane, T, up); break;
        }
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt) {
          const int ni = gi * kTile + 16 * (rb0 + rt) + g;
          const float n0 = tile_norm<NH>(kna, ni), n1 = tile_norm<NH>(kna, ni + 8);
          sc[rt][0] = fmaf(acc[rt][0], n0, sc[rt][0]);
          sc[rt][1] = fmaf(acc[rt][1], n0, sc[rt][1]);
          sc[rt][2] = fmaf(acc[rt][2], n1, sc[rt][2]);
          sc[rt][3] = fmaf(acc[rt][3], n1, sc[rt][3]);
        }
      }
      if constexpr (NP) {
        // columns 4..7 carried the lo parts of q': add them to the hi parts (lanes t, t^2)
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
          for (int j = 0; j < 4; ++j) sc[rt][j] += __shfl_xor_sync(0xffffffffu, sc[rt][j], 2);
      }
      // Rows past a column's last visible token get -inf. The row's n_q query tokens are
      // its last n_q cached tokens: column n (query token n % n_q) sees the tokens before
      // S.len - (n_q - 1 - n % n_q). Warp-uniform test: only rows from the first token
      // some column cannot see need the masks (n_q = 1: the end of the row).
      if (gt0 - g + 16 * NRT > S.len - (a.n_q - 1)) {
        const int c0 = NP ? 2 * (t & 1) : 2 * t;  // this lane's columns c0, c0 + 1
        const long long vis0 = S.len - (a.n_q - 1 - c0 % a.n_q), vis1 = S.len - (a.n_q - 1 - (c0 + 1) % a.n_q);
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt) {
          const long long r0 = gt0 + 16 * rt, r1 = r0 + 8;
          if (r0 >= vis0) sc[rt][0] = -INFINITY;
          if (r0 >= vis1) sc[rt][1] = -INFINITY;
          if (r1 >= vis0) sc[rt][2] = -INFINITY;
          if (r1 >= vis1) sc[rt][3] = -INFINITY;
        }
      }

      if constexpr (SC) {
        // column 2t + c holds head 2t + c (G <= 4: lanes t < 2; t >= 2 hold copies)
        const int b = S.u / a.h_kv, hkv = S.u % a.h_kv;
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int head = 2 * t + (j & 1);
            const long long tok = gt0 + 16 * rt + 8 * (j >> 1);
            if ((!NP || t < 2) && head < a.G && tok < S.len)
              a.scores[((size_t)b * a.h_q + (size_t)hkv * a.G + head) * a.scores_ld + tok] = sc[rt][j] * (1.f / kLog2e);
          }
      } else {
      // ---------------- online softmax over the rows (heads of columns 2t, 2t+1), base 2
      float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
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
      const unsigned char* vna = tb + L.vnorm_off;

      // ---------------- values: row block rb0 + rt is value chunk rb0 + rt of the tile.
      // First the probabilities (times |v| / sqrt(128)) as transposed fp16 B fragments,
      // then the m16n8k16 products against the value codes
      unsigned pb[NRT][2];
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        const float p0 = fast_exp2(sc[rt][0] - b0m), p1 = fast_exp2(sc[rt][1] - b1m);
        const float p2 = fast_exp2(sc[rt][2] - b0m), p3 = fast_exp2(sc[rt][3] - b1m);
        l0 += p0 + p2;
        l1 += p1 + p3;
        const float av0 = tile_norm<NH>(vna, 16 * (rb0 + rt) + g) * vscale;
        const float av1 = tile_norm<NH>(vna, 16 * (rb0 + rt) + g + 8) * vscale;
        pb[rt][0] = movmatrix_trans(pack_h2(p0 * av0, p1 * av0));
        pb[rt][1] = movmatrix_trans(pack_h2(p2 * av1, p3 * av1));
      }
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        ValueLane<VR> vl;
        vl.load(tb + L.vcode_off + (rb0 + rt) * 256 * VR, lane);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          mma16816(O[mt], vl.field(4 * mt, T.v, lane4), vl.field(4 * mt + 1, T.v, lane4),
                   vl.field(4 * mt + 2, T.v, lane4), vl.field(4 * mt + 3, T.v, lane4), pb[rt][0], pb[rt][1]);
      }
      }  // not scores-only
    };

    for (int k = 0; k < mine; ++k) {
      const int st = warp + kWarps * (k & 1), i = item_tile(k);
      const bool ok = mbar_wait_bounded(&full[st], (phase >> (k & 1)) & 1u);
      if (ok) {
        phase ^= 1u << (k & 1);
        pend &= ~(1u << (k & 1));
      }
      if (!ok) {
        // stop consuming; this warp waits for its own copies below, no partial is written
        if (lane == 0) {
          atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
          s_timeout = 1;
        }
        break;
      }
      const unsigned char* tb = ring + st * TB;
      const long long gt0 = (long long)(S.lt0 + i) * kTile + g;  // token of row g in row block 0
      // a paged tile without a page (flagged by the copy) is left out
      if (tile_present(a.cache, S.u / a.h_kv, S.lt0 + i)) {
        if (k == nfw && rem != 3) {
          const int rb0 = 2 * (warp & 1);
          rows(IntC<2>{}, tb, rb0, gt0 + 16 * rb0);
        } else {
          rows(IntC<4>{}, tb, 0, gt0);
        }
      }
      __syncwarp();  // every lane is done with the stage before it is refilled
      if (k + 2 < mine) {
        if (lane == 0) issue(k + 2);
        pend |= 1u << (k & 1);
      }
    }

    if (si + 1 == nseg) pdl_trigger();
    // ---------------- merge the warps (their partials reuse the ring: every warp is done
    // with the segment's tiles and has no copy in flight)
    __syncthreads();
    if (*static_cast<volatile int*>(&s_timeout)) break;  // uniform over the CTA
    if constexpr (SC) continue;  // the q' fragments are reloaded for the next segment
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
          const float f = fast_exp2(mm[w * 8 + hh] - M);
          o = fmaf(f, mo[(w * 8 + hh) * kD + tid], o);
          l = fmaf(f, ml[w * 8 + hh], l);
        }
      }
      const size_t idx = ((size_t)S.u * a.n_parts + S.part) * G + hh;
      a.part_o[idx * kD + tid] = o;
      if (tid == 0) {
        a.part_ml[idx * 2] = M;
        a.part_ml[idx * 2 + 1] = l;
      }
    }
    __syncthreads();  // the merge area is the next segment's ring
  }
  // after a timeout: do not leave while this warp's copies into shared memory are in flight
  if (lane == 0)
    for (int h = 0; h < 2; ++h)
      if (pend & (1u << h)) mbar_wait_bounded(&full[warp + kWarps * h], (phase >> h) & 1u);
}
#pragma nv_diag_default 128

size_t split_smem_bytes(int tile_bytes, int n_kquads) {
  return 128 + size_t(kRing) * tile_bytes + size_t(n_kquads) * 64 * sizeof(unsigned) + 2 * kWarps * 8 * sizeof(float);
}

// Once per device and variant, before the occupancy query and the first launch: the
// largest dynamic shared memory any layout needs, and the whole unified L1/shared array as
// shared memory (the occupancy the plan assumes is then the one the launch gets).
template <int VR, bool NP, bool SC, bool NH>
cudaError_t configure_split() {
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev >= 64 || configured[dev]) return e;
  e = cudaFuncSetAttribute(split_kernel<VR, NP, SC, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(split_smem_bytes(kMaxTileBytes, kMaxQuads)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(split_kernel<VR, NP, SC, NH>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             int(cudaSharedmemCarveoutMaxShared));
  if (e == cudaSuccess) configured[dev] = true;
  return e;
}

template <int VR, bool NP, bool SC, bool NH>
cudaError_t launch_split(const SplitArgs& a, const DevLayout& L, unsigned n_ctas, cudaStream_t stream) {
  const size_t smem = split_smem_bytes(L.tile_bytes, L.n_kquads);
  cudaError_t e = configure_split<VR, NP, SC, NH>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_kernel<VR, NP, SC, NH>, L, a);
}

// ------------------------------------------------------------------ combine
constexpr int kCombThreads = 512;

// One CTA per (batch row, query column): log-sum-exp merge of the unit's partials, then
// o = R_V^T o'. Four threads per output dimension. R_V (not written by the split kernel)
// is read into registers before waiting for the split kernel to finish. h_q counts query
// columns (query heads x n_q); column hh of KV head h is query head h G / n_q + hh / n_q
// at query token hh % n_q, written to out[b][token][head].
__global__ void __launch_bounds__(kCombThreads, 1) combine_kernel(const float* __restrict__ part_ml,
                                                              const float* __restrict__ part_o, int S,
                                                              int max_tiles, long long total_tiles, int n_ctas, int G, int h_q,
                                                              int h_kv, int n_q, const float* __restrict__ v_rot,
                                                              float* __restrict__ out) {
  pdl_trigger();  // the next call's first kernel may start its prologue now
  const int bq = blockIdx.x, b = bq / h_q, hq = bq % h_q;
  const int u = b * h_kv + hq / G, hh = hq % G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = tid & (kD - 1), qtr = tid >> 7;
  __shared__ float w[kMaxParts];
  __shared__ float red[2][kCombThreads / 32];
  __shared__ float part[4][kD];
  __shared__ float op[kD];
  float rv[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) rv[i] = __ldg(v_rot + (size_t)(qtr * 32 + i) * kD + d);
  // the CTAs whose slices meet unit u wrote its partial slots 0 .. n-1
  const long long M = max_tiles;
  const int n = cta_of_tile((long long)(u + 1) * M - 1, total_tiles, n_ctas) - cta_of_tile((long long)u * M, total_tiles, n_ctas) + 1;
  pdl_wait();  // partials come from split_kernel
  const float2* ml = reinterpret_cast<const float2*>(part_ml) + (size_t)u * S * G + hh;  // slot sp at ml[sp * G]
  const float* po = part_o + ((size_t)u * S * G + hh) * kD + d;                          // slot sp at po[sp * G * kD]
  // every load of the merge is issued at once: (m, l) of two slots, o' of 16 slots
  constexpr int kPv = 16;
  float pv[kPv];
#pragma unroll
  for (int k = 0; k < kPv; ++k) {
    const int sp = qtr + 4 * k;
    pv[k] = sp < n ? __ldg(po + (size_t)sp * G * kD) : 0.f;
  }
  float mloc[2], lloc[2];
  float Mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int sp = tid + k * kCombThreads;
    const float2 v = sp < n ? ml[(size_t)sp * G] : make_float2(-INFINITY, 0.f);
    mloc[k] = v.x;
    lloc[k] = v.y;
    Mx = fmaxf(Mx, v.x);
  }
  for (int o = 16; o > 0; o >>= 1) Mx = fmaxf(Mx, __shfl_xor_sync(0xffffffffu, Mx, o));
  if (lane == 0) red[0][warp] = Mx;
  __syncthreads();
  Mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kCombThreads / 32; ++i) Mx = fmaxf(Mx, red[0][i]);
  float l = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int sp = tid + k * kCombThreads;
    if (sp < n) {
      const float wt = (Mx == -INFINITY || mloc[k] == -INFINITY) ? 0.f : exp2f(mloc[k] - Mx);
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
    float o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int k = 0; k < kPv; k += 2) {
      if (qtr + 4 * k < n) o0 = fmaf(w[qtr + 4 * k], pv[k], o0);
      if (qtr + 4 * (k + 1) < n) o1 = fmaf(w[qtr + 4 * (k + 1)], pv[k + 1], o1);
    }
    for (int sp = qtr + 4 * kPv; sp < n; sp += 4) o0 = fmaf(w[sp], __ldg(po + (size_t)sp * G * kD), o0);
    part[qtr][d] = o0 + o1;
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
  const int heads = h_q / n_q, head = (hq / G) * (G / n_q) + hh / n_q, tok = hh % n_q;
  if (tid < kD)
    out[(((size_t)b * n_q + tok) * heads + head) * kD + tid] = (part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid]);
}

template <int VR, bool NP, bool SC, bool NH>
int split_occupancy(const DevLayout& L) {
  int n = 0;
  if (configure_split<VR, NP, SC, NH>() != cudaSuccess) return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, split_kernel<VR, NP, SC, NH>, kThreads,
                                                    split_smem_bytes(L.tile_bytes, L.n_kquads)) != cudaSuccess)
    return 1;
  return n < 1 ? 1 : n;
}

// Launch as a programmatic dependent of the kernel before it on the stream: the CTAs may
// start while that kernel runs and wait (griddepcontrol.wait) before reading its results.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block, cudaStream_t stream,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Calls fn(IntC<VR>, IntC<NP>, IntC<SC>, IntC<NH>) with the split-kernel variant of a
// call: value rate (scores only: 1, the value tables are not built), q' in one product
// (G <= 4), scores only, fp16 norms.
template <int VR, int NP, int SC, typename Fn>
auto split_nh(bool nh, Fn&& fn) {
  return nh ? fn(IntC<VR>{}, IntC<NP>{}, IntC<SC>{}, IntC<1>{}) : fn(IntC<VR>{}, IntC<NP>{}, IntC<SC>{}, IntC<0>{});
}
template <int VR, int SC, typename Fn>
auto split_np(bool np, bool nh, Fn&& fn) {
  return np ? split_nh<VR, 1, SC>(nh, fn) : split_nh<VR, 0, SC>(nh, fn);
}
template <typename Fn>
auto split_variant(int v_rate, bool np, bool sc, bool nh, Fn&& fn) {
  if (sc) return split_np<1, 1>(np, nh, fn);
  switch (v_rate) {
    case 1: return split_np<1, 0>(np, nh, fn);
    case 2: return split_np<2, 0>(np, nh, fn);
    case 3: return split_np<3, 0>(np, nh, fn);
    default: return split_np<4, 0>(np, nh, fn);
  }
}

// Split and combine kernels of one call, launched as programmatic dependents of the
// kernel that wrote the q' fragments (and, after an append, the new tokens).
// n_q query tokens per row: the split and combine kernels see h_q n_q query columns,
// G = h_q n_q / h_kv per KV head.
cudaError_t launch_attention(const DevLayout& L, const DecodePlan& wplan, int batch, int h_q, int h_kv, int n_q,
                             const CacheRef& cache, const int* seq_lens, float* out, void* workspace,
                             int len_add, bool after_append, cudaStream_t stream, float* scores = nullptr,
                             long long scores_ld = 0) {
  const int hc = h_q * n_q, G = hc / h_kv;
  // G <= 4: the q' hi and lo parts share one m16n8k8 product (columns 0-3 and 4-7)
  const bool np = G <= 4;
  // the workspace was sized for the most CTAs per SM; shared memory may allow fewer
  // (larger slices, fewer partials per unit)
  const bool sc = scores != nullptr, nh = L.norm_fp16 != 0;
  if (!sc && (L.v_rate < 1 || L.v_rate > 4)) return cudaErrorInvalidValue;
  const int occ = split_variant(L.v_rate, np, sc, nh, [&](auto V, auto P, auto S, auto H) {
    return split_occupancy<decltype(V)::value, decltype(P)::value != 0, decltype(S)::value != 0,
                           decltype(H)::value != 0>(L);
  });
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const DecodePlan plan = plan_decode(batch, hc, h_kv, (long long)wplan.max_tiles * kTile, sms, occ);
  if (plan.n_parts > wplan.n_parts || plan.workspace_bytes > wplan.workspace_bytes) return cudaErrorInvalidValue;
  const long long units = (long long)batch * h_kv;
  SplitArgs a;
  a.cache = cache;
  a.seq_lens = seq_lens;
  a.max_tiles = plan.max_tiles;
  a.n_ctas = plan.n_ctas;
  a.n_parts = plan.n_parts;
  a.total_tiles = units * plan.max_tiles;
  a.h_q = hc;
  a.h_kv = h_kv;
  a.G = G;
  a.n_q = n_q;
  // q' fragments first, then the partials in the launch plan's layout (never larger than
  // the workspace plan's)
  char* ws = static_cast<char*>(workspace);
  a.qfrag = reinterpret_cast<const unsigned*>(ws);
  ws += qfrag_bytes(units);
  a.part_ml = reinterpret_cast<float*>(ws);
  a.part_o = reinterpret_cast<float*>(ws + align256(size_t(units) * plan.n_parts * G * 2 * sizeof(float)));
  a.scores = scores;
  a.scores_ld = scores_ld;
  a.len_add = len_add;
  a.wait_new = after_append ? 1 : 0;
  const unsigned n_ctas = unsigned(plan.n_ctas);
  e = split_variant(L.v_rate, np, sc, nh, [&](auto V, auto P, auto S, auto H) {
    return launch_split<decltype(V)::value, decltype(P)::value != 0, decltype(S)::value != 0,
                        decltype(H)::value != 0>(a, L, n_ctas, stream);
  });
  if (sc) return e;  // scores only: no merge
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(batch * hc));
  cfg.blockDim = dim3(kCombThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, (const float*)a.part_ml, (const float*)a.part_o, plan.n_parts,
                            plan.max_tiles, a.total_tiles, plan.n_ctas, G, hc, h_kv, n_q, L.v_rot32, out);
}

}  // namespace

DecodePlan plan_decode(int batch, int h_q, int h_kv, long long max_seq_len, int num_sms, int ctas_per_sm) {
  DecodePlan p{};
  if (ctas_per_sm <= 0 || ctas_per_sm > kCtasPerSm) ctas_per_sm = kCtasPerSm;
  const int G = h_q / h_kv;
  p.max_tiles = int((max_seq_len + kTile - 1) / kTile);
  if (p.max_tiles < 1) p.max_tiles = 1;
  const long long units = (long long)batch * h_kv;
  const long long total = units * p.max_tiles;
  // one wave of ctas_per_sm CTAs per SM with slices of equal length (+-1 tile), no longer
  // than a unit; more units than CTA slots: one CTA per unit
  const long long slots = (long long)ctas_per_sm * num_sms;
  long long C = units >= slots ? units : std::min(slots, total);
  // a unit meets at most ceil(C / units) + 1 slices; the combine merges up to kMaxParts
  while ((C + units - 1) / units + 1 > kMaxParts) C -= units;
  p.n_ctas = int(C);
  p.tiles_per_cta = int((total + C - 1) / C);
  p.n_parts = int((C + units - 1) / units + 1);
  p.workspace_bytes = qfrag_bytes(units) + align256(size_t(units) * p.n_parts * G * 2 * sizeof(float)) +
                      size_t(units) * p.n_parts * G * kD * sizeof(float);
  return p;
}

cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, int n_q, const CacheRef& cache, const int* seq_lens, float softmax_scale,
                          float* out, void* workspace, cudaStream_t stream) {
  const int G = h_q * n_q / h_kv;
  // a plain launch: the split kernel, launched as soon as this kernel starts, reads the
  // cache, which the kernel before this one may write
  qprep_kernel<<<unsigned(batch * h_kv), kPrepThreads, 0, stream>>>(
      L, q, q_dtype, h_q, h_kv, G, n_q, softmax_scale * kLog2e, static_cast<unsigned*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, n_q, cache, seq_lens, out, workspace, 0, false, stream);
}

cudaError_t launch_scores(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch, int h_q,
                          int h_kv, const CacheRef& cache, const int* seq_lens, float softmax_scale, float* scores,
                          long long scores_ld, void* workspace, cudaStream_t stream) {
  const int G = h_q / h_kv;
  qprep_kernel<<<unsigned(batch * h_kv), kPrepThreads, 0, stream>>>(
      L, q, q_dtype, h_q, h_kv, G, 1, softmax_scale * kLog2e, static_cast<unsigned*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, 1, cache, seq_lens, nullptr, workspace, 0, false, stream,
                          scores, scores_ld);
}

cudaError_t launch_decode_step(const DevLayout& L, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, int n_new, const int* seq_lens_before, const void* q, int q_dtype,
                               int batch, int h_q, int h_kv, int n_q, const CacheRef& cache, float softmax_scale,
                               float* out, void* workspace, cudaStream_t stream) {
  const int G = h_q * n_q / h_kv;
  const long long n_enc = (long long)n_new * kEncodeParts * batch * h_kv;
  cudaError_t e;
  if (!L.norm_correct) {
    e = launch_dependent(step_prep_kernel<false>, unsigned(n_enc + batch * h_kv), kPrepThreads, stream, L, k_new,
                         v_new, kv_dtype, n_new, batch, seq_lens_before, cache, q, q_dtype, h_q, h_kv, G, n_q,
                         softmax_scale * kLog2e, static_cast<unsigned*>(workspace), int(n_enc));
  } else {
    // norm correction: clusters of the four encode parts of a token; the q' blocks
    // follow, padded to a whole cluster (the padding blocks return at once)
    const long long n_blocks = (n_enc + batch * h_kv + kEncodeParts - 1) / kEncodeParts * kEncodeParts;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(n_blocks));
    cfg.blockDim = dim3(kPrepThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kEncodeParts;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, step_prep_kernel<true>, L, k_new, v_new, kv_dtype, n_new, batch, seq_lens_before, cache,
                           q, q_dtype, h_q, h_kv, G, n_q, softmax_scale * kLog2e, static_cast<unsigned*>(workspace),
                           int(n_enc));
  }
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, n_q, cache, seq_lens_before, out, workspace, n_new,
                          n_new > 0, stream);
}

}  // namespace bgtq
