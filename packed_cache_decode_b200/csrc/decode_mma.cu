// Decode attention over the packed cache on tensor cores (sm_100a).
//
// "Block-GTQ" abstract, sentence 5: attention reads the packed codes directly, no decoded
// fp16 KV cache is ever written. With R_g orthogonal,
//   q . k_hat   = sum_g (|k_g| / sqrt(d_g)) (R_g q_g) . c[codes_g]
//   o           = R_V^T sum_t p_t (|v_t| / sqrt(128)) c[vcodes_t] / sum_t p_t.
//
// Three kernels per call, chained by programmatic dependent launch:
//  * qprep_kernel (one CTA per unit; in a decode step, step_prep_kernel also runs the
//    encode CTAs of the new tokens): q' = R_g q_g for the unit's query columns (fp32,
//    scaled by softmax_scale * log2(e) / (sqrt(d_g) kappa_g)), split into fp16 hi + lo
//    parts and laid out as mma B fragments, plus the column sums of the rate-1 group's
//    fragments. A column is one query head at one query token: a KV head has Gt = query
//    heads per KV head x n_q columns (n_q = 1 except in multi-token calls), taken 8 at a
//    time: a unit is (batch row, KV head, column tile of up to 8 columns).
//  * split_kernel: one CTA per SM, 8 to 12 warps. The (batch row, KV head) caches are
//    laid end to end as one sequence of 64-token tiles and every CTA takes an equal slice
//    of it (one wave). Inside a slice, unit by unit, warp w streams its own tiles w, w+W,
//    ... through a private pair of ring stages with 1-D bulk async copies (cp.async.bulk +
//    mbarrier, L2 evict-first, no multicast), contiguous or paged; the tiles left over after
//    a multiple of W go out whole or as half tiles (row blocks 0-1 and 2-3) so that no warp
//    runs more than half a tile past the others. Keys: per quad of 4 dimension pairs one
//    load gives the lane its codes for its 8 tokens (fragment-major format); rate 1 gives
//    0/1 operands straight from the code bits (an fp16 subnormal 2^(m-24) or 0, exact),
//    turned into +-1 codes afterwards with the rate-1 column sums of q'; rates 2 and 4
//    look up byte-indexed tables (one prmt builds the address from a code byte, one
//    64-bit shared load returns two A registers, or a hi + lo pair at rate 4); rate 3
//    indexes a 6-bit pair table. Rates 3 and 4 put a slot's centroid hi parts in rows g
//    and their lo parts in rows g+8 of one product, summed afterwards. The tables are
//    built once per layout (at upload), fetched by one bulk copy per CTA, and hold 16
//    copies of every entry, lane l reading copy l % 16, so a half-warp's 64-bit loads
//    never share a bank. A group's quads go in pairs into mma.m16n8k16 (for units of at
//    most 4 columns the q' hi and lo parts are the eight columns of one product). fp32
//    accumulators per group (started by the group's first products), then times the
//    group norm (fp32 or fp16, a template variant). With one layout per KV head (a
//    layout set) the CTA reloads the layout and its tables when its segment's head
//    changes. Each column masks the tokens past its own position (the row's last tiles
//    only). Online softmax in base 2 with warp shuffles. Values: the probabilities times
//    |v|/sqrt(128) in fp16, transposed with movmatrix, against value codes turned into A
//    registers the same way (rate 2: the byte table), accumulated in V's rotated space
//    (fp32). At the end of a unit the warps merge and the CTA writes its partial
//    (o', m, l). A scores-only form writes the logits instead.
//  * combine_kernel (one CTA per batch row x query column, 512 threads): log-sum-exp merge
//    of the unit's partials and o = R_V^T o', written to out[b][token][head] (or, for a
//    call over one token range of a split sequence, the merged record (m, l, o')).
// After an append (bgtq_decode_step) only the tile that receives the new tokens waits for
// the encode before it is copied. With norm correction the step's encode CTAs run as
// clusters of four (their launch pads the grid to whole clusters).
//
// Every mbarrier wait is bounded; on timeout the kernel records BGTQ_STATUS_TIMEOUT, drops
// the warp's partial (m = -inf, l = 0), waits (bounded) for its own copies in flight and
// goes on; the call's output is then invalid and the status says so.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <type_traits>
#include <utility>

#include "bgtq_internal.h"
#include "encode_body.cuh"
#include "async_copy.cuh"
#include "kernels.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void mma16816(float (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3,
                                         unsigned b0, unsigned b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ unsigned movmatrix_trans(unsigned x) {
  unsigned y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
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

constexpr int kMaxParts = 1024;      // partial slots per unit the merge can take


__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// per unit: the q' B fragments [kMaxQuads][2][32] words, then the 8 column sums of the
// rate-1 group's fragments (and padding to 16 bytes)
constexpr int kQfragWords = kMaxQuads * 64 + 16;
inline size_t qfrag_bytes(long long units) { return align256(size_t(units) * kQfragWords * sizeof(unsigned)); }

// ------------------------------------------------------------------ split kernel
struct SplitArgs {
  CacheRef cache;
  const int* seq_lens;
  const unsigned* qfrag;  // [units][kMaxQuads][2][32] q' B fragments from the preparation kernel
  int max_tiles;          // M: tiles per unit covered by the plan
  int n_ctas;             // CTAs; CTA c takes tiles [c T / n_ctas, (c+1) T / n_ctas) of the sequence
  int n_parts;            // partial slots per unit
  long long total_tiles;  // units x M
  int h_q, h_kv, Gt;      // Gt: query columns per KV head (query heads per KV head x n_q)
  int G;                  // columns of a unit's tile: Gt when CT = 1, else 8 (the last tile may hold fewer)
  int n_q;                // query tokens per row; column n of KV head h is query token n % n_q
  int CT;                 // column tiles per (batch row, KV head): unit u = cache unit u / CT, tile u % CT
  float* part_ml;         // [units][n_parts][G][2]
  float* part_o;          // [units][n_parts][G][128]
  float* scores;          // scores-only mode: [batch][h_q][scores_ld] logits (softmax_scale q.k_hat)
  long long scores_ld;
  int len_add;            // tokens appended by the previous kernel: row b attends over seq_lens[b] + len_add
  int wait_new;           // the previous kernel appends at seq_lens[b]: wait for it before copying that tile
  const DevLayout* heads; // per-KV-head layouts (device array of h_kv), or null: one layout for all heads
};

// The layout a kernel works with: the by-value kernel parameter, or (PH: one layout per KV
// head) a copy in shared memory of the current head's layout.
template <bool PH>
__device__ __forceinline__ const DevLayout& pick_layout(const DevLayout& param, const unsigned char* copy) {
  if constexpr (PH) return *reinterpret_cast<const DevLayout*>(copy);
  else return param;
}

constexpr int kQsLd = kD + 16;                   // row of q staged per group at 16-byte aligned columns

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void mma1688(float (&c)[4], unsigned a0, unsigned a1, unsigned b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(b0));
}
// The same products with Z: the accumulator starts at zero (C = 0, c not read).
template <bool Z>
__device__ __forceinline__ void mma16816s(float (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3,
                                          unsigned b0, unsigned b1) {
  if constexpr (Z)
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
  else
    mma16816(c, a0, a1, a2, a3, b0, b1);
}
template <bool Z>
__device__ __forceinline__ void mma1688s(float (&c)[4], unsigned a0, unsigned a1, unsigned b0) {
  if constexpr (Z)
    asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};\n"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(b0), "f"(0.f));
  else
    mma1688(c, a0, a1, b0);
}

// +-1 pair from two 1-bit codes sitting at bits 15 and 31 of x (bit 1 -> +1, 0 -> -1):
// the sign bit is the inverted code, the magnitude is fp16 1.0.
__device__ __forceinline__ unsigned sign_pair(unsigned x) { return (~x & 0x80008000u) | 0x3C003C00u; }
__device__ __forceinline__ unsigned prmt(unsigned a, unsigned b, unsigned sel) {
  unsigned d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Shared loads at 32-bit shared-window addresses. They are pure (no side effects, so the
// compiler may schedule them freely): every address they get derives from a value passed
// through launder() after the wait or barrier that made the data valid (a tile's copy, the
// q' fragments of a unit, the tables), which keeps them after it.
__device__ __forceinline__ unsigned launder(unsigned x) {
  unsigned y;
  asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x) : "memory");
  return y;
}
__device__ __forceinline__ unsigned ld_s16(unsigned a) {
  unsigned short v;
  asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ unsigned ld_s32(unsigned a) {
  unsigned v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 ld_s64(unsigned a) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 ld_s128(unsigned a) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
// x >> s for an s that is known after unrolling and may be negative (a left shift).
__device__ __forceinline__ unsigned shr(unsigned x, int s) { return s >= 0 ? x >> s : x << -s; }

// Byte-indexed tables (16 copies of each 8-byte entry, 256 rows of 256 bytes): the row of
// code byte `byte` of w, plus the lane's copy offset c8 = 8 (lane % 16) < 128, in one prmt
// (byte 0 of the result from c8, byte 1 from w, bytes 2-3 zero).
__device__ __forceinline__ unsigned row8(unsigned w, unsigned c8, int byte) {
  return prmt(w, c8, 0x5504u | (unsigned(byte) << 4));
}

// Dynamic shared memory of a split CTA, at offsets fixed at compile time (so that every
// table lookup is one shared load with an immediate offset): mbarriers, the byte table,
// the rate-3 table, the value table of the value rate VR (rate 3: 64 lane-private
// entries, rate 4: 256 shared ones), the q' fragments [pair slot][lane] (hi, hi, lo, lo),
// then the ring of 2 stages per warp (its size depends on the layout's tile bytes).
constexpr int kSmT8 = 256;
constexpr int kSmT3 = kSmT8 + kTbl8Bytes;
constexpr int kSmVt = kSmT3 + kTbl3Bytes;
template <int VR>
__host__ __device__ constexpr int vtab_bytes() { return VR == 3 ? 64 * 32 * 4 : VR == 4 ? 256 * 4 : 0; }
constexpr int kPairSlots = kMaxQuads / 2 + kMaxGroups;  // quad pairs of all groups (a group's odd quad alone)
template <int VR>
__host__ __device__ constexpr int sm_qf() { return kSmVt + vtab_bytes<VR>(); }
template <int VR>
__host__ __device__ constexpr int sm_ring() { return (sm_qf<VR>() + kPairSlots * 32 * 16 + 127) / 128 * 128; }

// A compile-time int carried as a value (row blocks per work item).
template <int N>
struct IntC {
  static constexpr int value = N;
};

// The lane's codes of one quad of a key group with rate R: load() reads them at the lane's
// byte offset (rate 3: two planes); `up` moves slots 4-7 to 0-3 (the upper half tile).
template <int R>
struct KCodes;
template <>
struct KCodes<1> {
  unsigned w;  // lo codes in bits 0-7, hi codes in bits 16-23 (slot m at bits m, 16 + m)
  __device__ __forceinline__ void load(unsigned tb, unsigned off, bool up) {
    w = prmt(ld_s16(tb + (off & 0xffffu)), 0u, 0x4140u);
    if (up) w >>= 4;
  }
  // fp16 pair of slot m: 0 or 2^(m - 24) per half (fp16 subnormals, exact on the tensor
  // cores); the code c = +-a is 2 a bit - a, so the group's scores come out as
  // 2^(25 - m) acc - sum of the B column (applied after the products)
  __device__ __forceinline__ unsigned a(int m) const { return w & (0x00010001u << m); }
};
template <>
struct KCodes<2> {
  unsigned w;  // nibble m = lo | hi << 2; byte j = slots 2j, 2j+1
  __device__ __forceinline__ void load(unsigned tb, unsigned off, bool up) {
    w = ld_s32(tb + (off & 0xffffu));
    if (up) w >>= 16;
  }
};
template <>
struct KCodes<3> {
  unsigned wa, wb;  // 48-bit string: field m (6 bits) at bit 6 m; plane B holds bits 32..47
  __device__ __forceinline__ void load(unsigned tb, unsigned off, bool up) {
    wa = ld_s32(tb + (off & 0xffffu));
    wb = ld_s16(tb + (off >> 16));
    if (up) {  // fields 4..7 to 0..3 (only those are used then)
      wa = (wa >> 24) | (wb << 8);
      wb = 0;
    }
  }
  // row offset (field x 128) plus the lane's copy offset
  __device__ __forceinline__ unsigned row(int m, unsigned c8) const {
    const int p = 6 * m;
    unsigned x;
    if (p + 6 <= 32) x = shr(wa, p - 7);
    else if (p >= 32) x = shr(wb, p - 32 - 7);
    else x = __funnelshift_r(wa, wb, p) << 7;
    return (x & 0x1F80u) | c8;
  }
};
template <>
struct KCodes<4> {
  uint2 w;  // byte m = lo | hi << 4
  __device__ __forceinline__ void load(unsigned tb, unsigned off, bool up) {
    w = ld_s64(tb + (off & 0xffffu));
    if (up) w.x = w.y;
  }
};

// Scores of one key group with compile-time rate R over its nq quads of a tile. Quads go in
// pairs into m16n8k16 products (quad 2i: k columns 0-7, quad 2i+1: 8-15); a group's odd
// last quad takes an m16n8k8 product. The lane's codes of quad j of the group sit at kb +
// 64 R j + lo_full (the last quad, which may hold fewer pairs: at off_last); a lane without
// a pair of that quad reads any code, its q' rows are zero. qf4 + 512 (j / 2) = the lane's
// (hi, hi, lo, lo) B fragments of quad pair j / 2 (a single last quad: (hi, 0, lo, 0)).
// Rates 1-2: row block rt of the work item: rows g and g+8 are slots m = 2 rt and 2 rt + 1;
// acc[rt] holds them. Rates 3-4 (centroids as fp16 hi + lo parts): one product per slot m,
// its hi parts in row g and its lo parts in row g+8 (one 64-bit table load gives the lane
// both, in operand order); acc[m] then holds the slot's two halves, summed afterwards.
// NRT = 4: the whole tile; NRT = 2: the half tile of row blocks 0-1 (up = false) or 2-3.
template <int R, bool NP, int NRT>
__device__ __forceinline__ void key_group(float (&acc)[R >= 3 ? 2 * NRT : NRT][4], unsigned tb, unsigned kb,
                                          unsigned lo_full, unsigned off_last, int nq, unsigned qf4, bool up,
                                          unsigned t8, unsigned t3, unsigned c8) {
  // a full quad block is 16 x 4 pairs x R bytes; rate-3 offsets hold both planes' offsets
  // (low and high halfword), so a step moves both
  constexpr unsigned kQuadBytes = R == 3 ? 64u * R * 0x10001u : 64u * R;
  unsigned off = kb * (R == 3 ? 0x10001u : 1u) + lo_full;
  // (hi, lo) table entry of slot m of a quad's codes
  auto entry = [&](const KCodes<R>& c, int m) -> uint2 {
    if constexpr (R == 3) return ld_s64(t3 + c.row(m, c8));
    else if constexpr (R == 4) return ld_s64(t8 + 128 + row8(m < 4 ? c.w.x : c.w.y, c8, m & 3));
    else return make_uint2(0u, 0u);
  };
  // quads 2i, 2i+1 (codes at o0, o1, B fragments of pair i); Z: the group's first
  // products, which start the accumulators at zero
  auto pair = [&](auto zc, unsigned o0, unsigned o1, int i) {
    constexpr bool Z = decltype(zc)::value;
    KCodes<R> c0, c1;
    c0.load(tb, o0, NRT < 4 && up);
    c1.load(tb, o1, NRT < 4 && up);
    const uint4 f = ld_s128(qf4 + i * 512);
    if constexpr (R <= 2) {
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        unsigned a0, a1, a2, a3;
        if constexpr (R == 1) {
          const int m = 2 * rt;
          a0 = c0.a(m);
          a1 = c0.a(m + 1);
          a2 = c1.a(m);
          a3 = c1.a(m + 1);
        } else {
          const uint2 e0 = ld_s64(t8 + row8(c0.w, c8, rt)), e1 = ld_s64(t8 + row8(c1.w, c8, rt));
          a0 = e0.x;
          a1 = e0.y;
          a2 = e1.x;
          a3 = e1.y;
        }
        mma16816s<Z>(acc[rt], a0, a1, a2, a3, f.x, f.y);
        if constexpr (!NP) mma16816(acc[rt], a0, a1, a2, a3, f.z, f.w);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 2 * NRT; ++m) {
        const uint2 e0 = entry(c0, m), e1 = entry(c1, m);
        mma16816s<Z>(acc[m], e0.x, e0.y, e1.x, e1.y, f.x, f.y);
        if constexpr (!NP) mma16816(acc[m], e0.x, e0.y, e1.x, e1.y, f.z, f.w);
      }
    }
  };
  // an odd last quad j (codes at o0): m16n8k8 products
  auto single = [&](auto zc, unsigned o0, int j) {
    constexpr bool Z = decltype(zc)::value;
    KCodes<R> c0;
    c0.load(tb, o0, NRT < 4 && up);
    const uint4 f = ld_s128(qf4 + (j >> 1) * 512);
    if constexpr (R <= 2) {
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        unsigned a0, a1;
        if constexpr (R == 1) {
          const int m = 2 * rt;
          a0 = c0.a(m);
          a1 = c0.a(m + 1);
        } else {
          const uint2 e0 = ld_s64(t8 + row8(c0.w, c8, rt));
          a0 = e0.x;
          a1 = e0.y;
        }
        mma1688s<Z>(acc[rt], a0, a1, f.x);
        if constexpr (!NP) mma1688(acc[rt], a0, a1, f.z);
      }
    } else {
#pragma unroll
      for (int m = 0; m < 2 * NRT; ++m) {
        const uint2 e0 = entry(c0, m);
        mma1688s<Z>(acc[m], e0.x, e0.y, f.x);
        if constexpr (!NP) mma1688(acc[m], e0.x, e0.y, f.z);
      }
    }
  };
  if (nq == 1) {
    single(std::true_type{}, off_last, 0);
    return;
  }
  pair(std::true_type{}, off, nq == 2 ? off_last : off + kQuadBytes, 0);
  int j = 2;
  off += 2 * kQuadBytes;
#pragma unroll 1
  for (; j + 1 < nq; j += 2, off += 2 * kQuadBytes) pair(std::false_type{}, off, j + 2 == nq ? off_last : off + kQuadBytes, j >> 1);
  if (j < nq) single(std::false_type{}, off_last, j);
}

// Value A fragments of one 16-token chunk: the lane's 64 VR-bit string (one or two
// loads) holds 32 fields n = 4 mt + k, each the fp16 pair of A register k of m-tile mt.
template <int VR>
struct ValueLane {
  unsigned w[2 * VR];
  __device__ __forceinline__ void load(unsigned vblk, int lane) {
    if constexpr (VR == 1) {
      const uint2 x = ld_s64(vblk + 8 * lane);
      w[0] = x.x;
      w[1] = x.y;
    } else {
      const uint4 x = ld_s128(vblk + 16 * lane);
      w[0] = x.x;
      w[1] = x.y;
      w[2] = x.z;
      w[3] = x.w;
      if constexpr (VR == 3) {
        const uint2 y = ld_s64(vblk + 512 + 8 * lane);
        w[4] = y.x;
        w[5] = y.y;
      } else if constexpr (VR == 4) {
        const uint4 y = ld_s128(vblk + 512 + 16 * lane);
        w[4] = y.x;
        w[5] = y.y;
        w[6] = y.z;
        w[7] = y.w;
      }
    }
  }
  // the four A registers of m-tile mt (compile-time after unrolling). Rate 2: byte 2 mt
  // (fields 4 mt, 4 mt + 1) and byte 2 mt + 1 of the string, each one row of the byte table.
  __device__ __forceinline__ void regs(int mt, unsigned t8, unsigned vlut, unsigned c8, unsigned lane4,
                                       unsigned (&a)[4]) const {
    if constexpr (VR == 2) {
      const uint2 e0 = ld_s64(t8 + row8(w[mt >> 1], c8, 2 * (mt & 1)));
      const uint2 e1 = ld_s64(t8 + row8(w[mt >> 1], c8, 2 * (mt & 1) + 1));
      a[0] = e0.x;
      a[1] = e0.y;
      a[2] = e1.x;
      a[3] = e1.y;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) a[k] = field(4 * mt + k, vlut, lane4);
    }
  }
  __device__ __forceinline__ unsigned field(int n, unsigned vlut, unsigned lane4) const {
    if constexpr (VR == 1) {
      return sign_pair(w[n >> 4] << (15 - (n & 15)));
    } else if constexpr (VR == 3) {
      const int bit = 6 * n, wi = bit >> 5, sh = bit & 31;
      const unsigned x = sh <= 26 ? (w[wi] >> sh) : __funnelshift_r(w[wi], w[wi + 1], sh);
      return ld_s32(vlut + (((x & 63u) << 7) | lane4));
    } else {
      return ld_s32(vlut + (shr(w[n >> 2], 8 * (n & 3) - 2) & 0x3fcu));
    }
  }
};

// The slice of CTA c: tiles [c T / C, (c+1) T / C) of the units x M = T tiles laid end to
// end, i.e. a run of segments, each a tile range of one unit (clipped to the unit's length
// when streamed).
__host__ __device__ inline int cta_of_tile(long long x, long long T, long long C) { return int(((x + 1) * C - 1) / T); }

struct Segment {
  int u;          // unit = batch row * h_kv + KV head
  int lt0;        // first tile (inside the unit) of the slice
  int n;          // tiles to stream (after clipping to the unit's length)
  int part;       // partial slot of this CTA for the unit
  long long len;  // tokens of the unit
};

__device__ __forceinline__ Segment make_segment(const DevLayout& L, const SplitArgs& a, int c, int u, bool flag) {
  const long long M = a.max_tiles, T = a.total_tiles, C = a.n_ctas;
  const long long g0 = (long long)c * T / C, g1 = (long long)(c + 1) * T / C;
  const int b = u / a.CT / a.h_kv;
  long long len = (long long)a.seq_lens[b] + a.len_add;
  if (len < 0) len = 0;
  const long long cap_tokens = min(a.cache.n_tiles, M) * kTile;
  const long long a0 = max(g0, (long long)u * M) - (long long)u * M;
  const long long a1 = min(g1, (long long)(u + 1) * M) - (long long)u * M;
  if (len > cap_tokens) {
    if (flag && a0 == 0) atomicOr(L.status, BGTQ_STATUS_DECODE_CLAMPED);
    len = cap_tokens;
  }
  const long long len_tiles = (len + kTile - 1) / kTile;
  Segment s;
  s.u = u;
  s.lt0 = int(a0);
  s.n = int(max(0LL, min(a1, len_tiles) - a0));
  s.part = c - cta_of_tile((long long)u * M, T, C);
  s.len = len;
  return s;
}

// The norms of slots s0 .. s0 + 2 NRT - 1 of row g (tokens g + 8 s) from the row's 8
// consecutive entries at `row` (entry 8 g + m holds token g + 8 m): 128-bit loads.
template <bool NH, int NRT>
__device__ __forceinline__ void row_norms(unsigned row, int s0, float (&n)[2 * NRT]) {
  if constexpr (NH) {
    const uint4 x = ld_s128(row);  // all 8 fp16 entries
    const unsigned w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 2 * NRT; i += 2) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[(s0 + i) >> 1]));
      n[i] = f.x;
      n[i + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2 * NRT; i += 4) {
      const uint4 x = ld_s128(row + 4 * (s0 + i));
      n[i] = __uint_as_float(x.x);
      n[i + 1] = __uint_as_float(x.y);
      n[i + 2] = __uint_as_float(x.z);
      n[i + 3] = __uint_as_float(x.w);
    }
  }
}

// SC: scores only. The tiles' logits (softmax_scale q . k_hat, natural units) go to
// a.scores; no softmax, values, partials or merge. NH: the layout stores fp16 norms.
// W: warps per CTA (one CTA per SM).
// (the scores-only instantiation discards the softmax and value code of the tile body)
#pragma nv_diag_suppress 128
template <int VR, bool NP, bool SC, bool NH, int W, bool PH>
__global__ void __launch_bounds__(32 * W, 1) split_kernel(DevLayout Lp, SplitArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  // per key rate r (1..4): its group (-1: none), quads, byte offset of its first quad in a
  // tile, first q' pair slot; per lane: its offset inside a full quad and the offset of
  // its codes in the group's last quad
  __shared__ int s_gi[5], s_gnq[5], s_gkb[5], s_gslot[5];
  __shared__ unsigned s_lof[5][32], s_olast[5][32];
  __shared__ int s_timeout;
  __shared__ float s_mm[W][8], s_ml[W][8];
  __shared__ __align__(16) unsigned char s_layout[PH ? sizeof(DevLayout) : 16];
  const DevLayout& L = pick_layout<PH>(Lp, s_layout);
  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int TB = Lp.tile_bytes;  // (the same for every head's layout)

  unsigned long long* full = reinterpret_cast<unsigned long long*>(smem);  // [2 W]
  unsigned char* t8 = smem + kSmT8;
  uint4* qf4 = reinterpret_cast<uint4*>(smem + sm_qf<VR>());         // [pair slot][lane]
  unsigned char* ring = smem + sm_ring<VR>();                           // stage s at ring + s TB
  float* mo = reinterpret_cast<float*>(ring);  // the warps' [8][128] partials reuse the ring

  __shared__ __align__(8) unsigned long long s_tbar;
  if (tid == 0) {
    s_timeout = 0;
    for (int i = 0; i < 2 * W; ++i) mbar_init(&full[i], 1);
    mbar_init(&s_tbar, 1);
    fence_mbar_init();
  }
  // The layout's decode state: its prebuilt tables (value table of this variant's value
  // rate included) by one bulk copy, the group table and the lanes' code offsets. Once per
  // CTA, and with per-head layouts again whenever a segment's head differs from the last
  // one (every warp is then past the previous segment's merge: tables and ring are free).
  constexpr unsigned kTblCopy = unsigned(sm_qf<VR>() - kSmT8);
  auto load_layout = [&](int head, unsigned tphase) {
    if constexpr (PH) {
      static_assert(sizeof(DevLayout) % 16 == 0, "layout copied in 16-byte units");
      const uint4* src = reinterpret_cast<const uint4*>(a.heads + head);
      for (int i = tid; i < int(sizeof(DevLayout) / 16); i += 32 * W) reinterpret_cast<uint4*>(s_layout)[i] = src[i];
    }
    __syncthreads();
    if (tid == 0) {
      mbar_expect_tx(&s_tbar, kTblCopy);
      bulk_load(t8, L.tables, kTblCopy, &s_tbar, evict_last_policy());
    }
    if (tid < 5) s_gi[tid] = -1;
    __syncthreads();
    if (tid < L.n_kgroups) {
      // groups are in descending rate order: the pair slots of the groups before this one
      int slot = 0;
      for (int gj = 0; gj < tid; ++gj) slot += (L.group_nquads[gj] + 1) >> 1;
      const int r = L.group_rate[tid];
      s_gi[r] = tid;
      s_gnq[r] = L.group_nquads[tid];
      s_gkb[r] = L.quad_off[L.group_quad0[tid]];
      s_gslot[r] = slot;
    }
    for (int i = tid; i < L.n_kgroups * 32; i += 32 * W) {
      // lane (g, t) holds pair t of a quad for tokens g + 8m: its 16 r bits are string
      // li = g P + t of the quad's block (rate 3: plane A word li, plane B halfword li after
      // 8 P words). Full quads have P = 4 (li = lane).
      const int gi = i >> 5, ln = i & 31, r = L.group_rate[gi];
      const int ql = L.group_quad0[gi] + L.group_nquads[gi] - 1, P = L.quad_np[ql], tt = ln & 3;
      const int li = tt < P ? (ln >> 2) * P + tt : 0;
      const unsigned fl = r == 3 ? 4u * ln | ((128u + 2u * ln) << 16) : 2u * r * ln;
      const unsigned base = unsigned(L.quad_off[ql]);
      s_lof[r][ln] = fl;
      s_olast[r][ln] = r == 3 ? (base + 4u * li) | ((base + 32u * P + 2u * li) << 16) : base + 2u * r * li;
    }
    // every thread waits (bounded) for the tables; on a timeout the status says so and the
    // decode goes on with whatever the tables hold (the call's output is then invalid)
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_tbar, tphase)) && lane == 0)
      atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
    __syncthreads();
  };
  const long long M0 = a.max_tiles, T0 = a.total_tiles, C0 = a.n_ctas;
  int cur_head = int(((long long)c * T0 / C0) / M0 / a.CT % a.h_kv);
  unsigned n_loads = 0;  // completed phases of s_tbar
  load_layout(cur_head, n_loads++ & 1u);

  const float vscale = rsqrtf(float(kD)) / L.kappa_v;
  const unsigned lane4 = unsigned(lane) << 2;
  // 32-bit shared-window addresses of the tables (valid from here on) and of the ring
  const unsigned sbase = smem_addr(smem);
  const unsigned t8a = launder(sbase + kSmT8), t3a = launder(sbase + kSmT3), vluta = launder(sbase + kSmVt);
  const unsigned ringa = sbase + sm_ring<VR>();
  const unsigned c8 = unsigned(lane & 15) << 3;
  const unsigned long long l2_stream = evict_first_policy();
  const long long M = a.max_tiles, T = a.total_tiles, C = a.n_ctas;
  const long long g0 = (long long)c * T / C, g1 = (long long)(c + 1) * T / C;
  const int u_first = int(g0 / M), u_last = int((g1 - 1) / M);
  unsigned phase = 0;   // bit k&1: parity of the next completion of stage w + W (k & 1)
  bool waited = !a.wait_new;
  bool q_ready = false;

  for (int u = u_first; u <= u_last; ++u) {
    if (s_timeout) {
      // a copy engine stalled earlier in this CTA: it is not waited on again, and the CTA's
      // remaining units get empty partials (m = -inf, l = 0, o' = 0), which the merge ignores
      const Segment S = make_segment(L, a, c, u, false);
      for (int it = tid; it < a.G * kD; it += 32 * W) {
        const int hh = it >> 7, d = it & (kD - 1);
        const size_t idx = ((size_t)S.u * a.n_parts + S.part) * a.G + hh;
        a.part_o[idx * kD + d] = 0.f;
        if (d == 0) {
          a.part_ml[idx * 2] = -INFINITY;
          a.part_ml[idx * 2 + 1] = 0.f;
        }
      }
      continue;
    }
    if constexpr (PH) {
      const int head = u / a.CT % a.h_kv;  // uniform over the CTA
      if (head != cur_head) {
        cur_head = head;
        load_layout(head, n_loads++ & 1u);
      }
    }
    const Segment S = make_segment(L, a, c, u, tid == 0);
    const int srow = S.u / a.CT / a.h_kv, shead = S.u / a.CT % a.h_kv;
    const int col0 = S.u % a.CT * kMaxG;  // first column of this unit's tile in its KV head
    const long long first_new = waited ? 0 : a.seq_lens[srow];
    // Work items of this warp: full tiles w, w+W, ... of the first W floor(n/W); the
    // rem = n % W tiles left go one to each of the first rem warps, or, when 2 rem <= W,
    // as half tiles (row blocks 0-1 and 2-3) to the first 2 rem warps. Both warps of a
    // split tile copy all of it into their own stages.
    const int nfw = S.n / W, rem = S.n % W;
    const bool halves = rem > 0 && 2 * rem <= W;
    const bool extra = halves ? warp < 2 * rem : warp < rem;
    const int mine = nfw + (extra ? 1 : 0);
    auto item_tile = [&](int k) { return k < nfw ? warp + W * k : W * nfw + (halves ? (warp >> 1) : warp); };
    auto issue = [&](int k) {  // lane 0 only
      const int it = S.lt0 + item_tile(k);
      if (!waited && (long long)(it + 1) * kTile > first_new) {
        pdl_wait();  // this tile receives tokens from the encode kernel
        waited = true;
      }
      const int st = warp + W * (k & 1);
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
    unsigned pend = mine >= 2 ? 3u : mine == 1 ? 1u : 0u;  // bit k&1: a copy into that stage is in flight
    if (!q_ready) {
      pdl_wait();  // q' fragments come from the preparation kernel
      q_ready = true;
    }
    const unsigned* src = a.qfrag + (size_t)S.u * kQfragWords;
    {
      // q' fragments of the unit, re-laid per group by quad pair: [slot][lane] = (hi of
      // quad 2k, hi of 2k+1, lo of 2k, lo of 2k+1), zeros for a missing odd partner
      int slot = 0;
      for (int gi = 0; gi < L.n_kgroups; ++gi) {
        const int q0 = L.group_quad0[gi], nq = L.group_nquads[gi];
        for (int e = tid; e < ((nq + 1) >> 1) * 32; e += 32 * W) {
          const int k = e >> 5, ln = e & 31, qa = q0 + 2 * k;
          const bool pair = 2 * k + 1 < nq;
          qf4[(slot + k) * 32 + ln] = make_uint4(src[qa * 64 + ln], pair ? src[(qa + 1) * 64 + ln] : 0u,
                                                 src[qa * 64 + 32 + ln], pair ? src[(qa + 1) * 64 + 32 + ln] : 0u);
        }
        slot += (nq + 1) >> 1;
      }
    }
    // column sums of the rate-1 group's B fragments (its 0/1 operands need them)
    const int sbc = 2 * t;  // this lane's B columns 2t, 2t+1
    const float sb0 = s_gi[1] >= 0 ? reinterpret_cast<const float*>(src + kMaxQuads * 64)[sbc] : 0.f;
    const float sb1 = s_gi[1] >= 0 ? reinterpret_cast<const float*>(src + kMaxQuads * 64)[sbc + 1] : 0.f;
    __syncthreads();
    const unsigned qf4a = launder(sbase + sm_qf<VR>());  // the unit's fragments are in

    float O[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int j = 0; j < 4; ++j) O[mt][j] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    // Row blocks rb0 .. rb0 + NRT - 1 of the tile in stage tb; gt0 = token of row g of
    // row block rb0.
    auto rows = [&](auto nrt, unsigned tb, int rb0, long long gt0) {
      constexpr int NRT = decltype(nrt)::value;
      const bool up = rb0 != 0;

      // ---------------- scores: per key group (rate as a template parameter), per quad,
      // NRT row blocks; then times the group norms
      const unsigned kna = tb + L.knorm_off;
      float sc[NRT][4];
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[rt][j] = 0.f;
      // key groups in a fixed rate order (rate known at compile time); a rate the layout
      // does not use has no group
      auto group = [&](auto rc) {
        constexpr int R = decltype(rc)::value;
        const int gi = s_gi[R];
        if (gi < 0) return;
        constexpr int NA = R >= 3 ? 2 * NRT : NRT;
        float acc[NA][4];  // started by the group's first products
        key_group<R, NP, NRT>(acc, tb, unsigned(s_gkb[R]), s_lof[R][lane], s_olast[R][lane], s_gnq[R],
                              qf4a + s_gslot[R] * 512 + 16 * lane, up, t8a, t3a, c8);
        if constexpr (R >= 3) {
          // slot 2rt + i: rows g (hi parts) + g+8 (lo parts) of acc[2rt + i] -> row g + 8i of rt
#pragma unroll
          for (int rt = 0; rt < NRT; ++rt) {
            const float h00 = acc[2 * rt][0] + acc[2 * rt][2], h01 = acc[2 * rt][1] + acc[2 * rt][3];
            const float h10 = acc[2 * rt + 1][0] + acc[2 * rt + 1][2], h11 = acc[2 * rt + 1][1] + acc[2 * rt + 1][3];
            acc[rt][0] = h00;
            acc[rt][1] = h01;
            acc[rt][2] = h10;
            acc[rt][3] = h11;
          }
        }
        float nrm[2 * NRT];
        row_norms<NH, NRT>(kna + (NH ? 2 : 4) * (gi * kTile + 8 * g), 2 * rb0, nrm);
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt) {
          const float n0 = nrm[2 * rt], n1 = nrm[2 * rt + 1];
          if constexpr (R == 1) {
            // 0/1 operands of value 2^(m - 24) (rows g, g+8 = positions 2rt, 2rt + 1):
            // sum_i B_i c_i = 2^(25 - m) acc - (column sum of B)
            const float s0 = n0 * __int_as_float((127 + 25 - 2 * rt) << 23);
            const float s1 = n1 * __int_as_float((127 + 24 - 2 * rt) << 23);
            sc[rt][0] = fmaf(acc[rt][0], s0, fmaf(-sb0, n0, sc[rt][0]));
            sc[rt][1] = fmaf(acc[rt][1], s0, fmaf(-sb1, n0, sc[rt][1]));
            sc[rt][2] = fmaf(acc[rt][2], s1, fmaf(-sb0, n1, sc[rt][2]));
            sc[rt][3] = fmaf(acc[rt][3], s1, fmaf(-sb1, n1, sc[rt][3]));
          } else {
            sc[rt][0] = fmaf(acc[rt][0], n0, sc[rt][0]);
            sc[rt][1] = fmaf(acc[rt][1], n0, sc[rt][1]);
            sc[rt][2] = fmaf(acc[rt][2], n1, sc[rt][2]);
            sc[rt][3] = fmaf(acc[rt][3], n1, sc[rt][3]);
          }
        }
      };
      group(IntC<4>{});
      group(IntC<3>{});
      group(IntC<2>{});
      group(IntC<1>{});
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
        const long long vis0 = S.len - (a.n_q - 1 - (col0 + c0) % a.n_q);
        const long long vis1 = S.len - (a.n_q - 1 - (col0 + c0 + 1) % a.n_q);
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
        // column 2t + c holds head col0 + 2t + c of the KV head (G <= 4: lanes t < 2; t >= 2 hold copies)
        const int b = srow, hkv = shead;
#pragma unroll
        for (int rt = 0; rt < NRT; ++rt)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int head = col0 + 2 * t + (j & 1);
            const long long tok = gt0 + 16 * rt + 8 * (j >> 1);
            if ((!NP || t < 2) && head < a.Gt && tok < S.len)
              a.scores[((size_t)b * a.h_q + (size_t)hkv * a.Gt + head) * a.scores_ld + tok] = sc[rt][j] * (1.f / kLog2e);
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
      const unsigned vna = tb + L.vnorm_off;

      // ---------------- values: row block rb0 + rt is value chunk rb0 + rt of the tile.
      // First the probabilities (times |v| / sqrt(128)) as transposed fp16 B fragments,
      // then the m16n8k16 products against the value codes
      unsigned pb[NRT][2];
      float vnr[2 * NRT];
      row_norms<NH, NRT>(vna + (NH ? 2 : 4) * 8 * g, 2 * rb0, vnr);
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        const float p0 = fast_exp2(sc[rt][0] - b0m), p1 = fast_exp2(sc[rt][1] - b1m);
        const float p2 = fast_exp2(sc[rt][2] - b0m), p3 = fast_exp2(sc[rt][3] - b1m);
        l0 += p0 + p2;
        l1 += p1 + p3;
        const float av0 = vnr[2 * rt] * vscale, av1 = vnr[2 * rt + 1] * vscale;
        pb[rt][0] = movmatrix_trans(pack_h2(p0 * av0, p1 * av0));
        pb[rt][1] = movmatrix_trans(pack_h2(p2 * av1, p3 * av1));
      }
#pragma unroll
      for (int rt = 0; rt < NRT; ++rt) {
        ValueLane<VR> vl;
        vl.load(tb + L.vcode_off + (rb0 + rt) * 256 * VR, lane);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          unsigned av[4];
          vl.regs(mt, t8a, vluta, c8, lane4, av);
          mma16816(O[mt], av[0], av[1], av[2], av[3], pb[rt][0], pb[rt][1]);
        }
      }
      }  // not scores-only
    };

    for (int k = 0; k < mine; ++k) {
      const int st = warp + W * (k & 1), i = item_tile(k);
      // warp-uniform decision: every lane waits, the warp goes on only if all saw the copy
      const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[st], (phase >> (k & 1)) & 1u));
      if (!ok) {
        // stop consuming; this warp's partial is dropped (m = -inf, l = 0) and it waits for
        // its own copies below
        if (lane == 0) {
          atomicOr(L.status, BGTQ_STATUS_TIMEOUT);
          s_timeout = 1;
        }
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
        break;
      }
      phase ^= 1u << (k & 1);
      pend &= ~(1u << (k & 1));
      const unsigned tb = launder(ringa + unsigned(st * TB));  // after the wait: the tile is in
      const long long gt0 = (long long)(S.lt0 + i) * kTile + g;  // token of row g in row block 0
      // a paged tile without a page (flagged by the copy) is left out
      if (tile_present(a.cache, srow, S.lt0 + i)) {
        if (k == nfw && halves) {
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
    // after a timeout: the ring is reused below, so wait (bounded) for this warp's copies
    // still in flight; only a second timeout here can leave one landing in shared memory
    if (pend && lane == 0)
      for (int h = 0; h < 2; ++h)
        if (pend & (1u << h)) mbar_wait_bounded(&full[warp + W * h], (phase >> h) & 1u);
    __syncwarp();
    if (pend) phase ^= pend;  // the stages with a copy awaited above completed a phase
    if (u == u_last) pdl_trigger();
    // ---------------- merge the warps (their partials reuse the ring: every warp is done
    // with the segment's tiles and has no copy in flight)
    __syncthreads();
    if constexpr (SC) {
      __syncthreads();  // the q' fragments are reloaded for the next segment
      continue;
    }
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
      s_mm[warp][2 * t] = m0;
      s_mm[warp][2 * t + 1] = m1;
      s_ml[warp][2 * t] = l0;
      s_ml[warp][2 * t + 1] = l1;
    }
    __syncthreads();
    const int G = a.G;
    for (int it = tid; it < G * kD; it += 32 * W) {
      const int hh = it >> 7, d = it & (kD - 1);
      float Mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) Mx = fmaxf(Mx, s_mm[w][hh]);
      float o = 0.f, l = 0.f;
      if (Mx != -INFINITY) {
#pragma unroll
        for (int w = 0; w < W; ++w) {
          const float f = fast_exp2(s_mm[w][hh] - Mx);
          o = fmaf(f, mo[(w * 8 + hh) * kD + d], o);
          l = fmaf(f, s_ml[w][hh], l);
        }
      }
      const size_t idx = ((size_t)S.u * a.n_parts + S.part) * G + hh;
      a.part_o[idx * kD + d] = o;
      if (d == 0) {
        a.part_ml[idx * 2] = Mx;
        a.part_ml[idx * 2 + 1] = l;
      }
    }
    __syncthreads();  // the merge area is the next segment's ring (s_timeout is uniform from here)
  }
}
#pragma nv_diag_default 128

// ------------------------------------------------------------------ combine
constexpr int kCombThreads = 512;

// One CTA per (batch row, query column): log-sum-exp merge of the unit's partials, then
// o = R_V^T o' (or, with rec, the merged record (m, l, o') of the column: the partial of a
// call over one token range, merged later with other ranges' records). Four threads per output dimension. R_V (not written by the split kernel)
// is read into registers before waiting for the split kernel to finish. h_q counts query
// columns (query heads x n_q); column gc of KV head h is query head h Gt / n_q + gc / n_q
// at query token gc % n_q, written to out[b][token][head]. G: columns per unit tile.
__global__ void __launch_bounds__(kCombThreads, 1) combine_kernel(const float* __restrict__ part_ml,
                                                              const float* __restrict__ part_o, int S,
                                                              int max_tiles, long long total_tiles, int n_ctas, int G, int h_q,
                                                              int h_kv, int n_q, const float* __restrict__ v_rot,
                                                              float* __restrict__ out, float* __restrict__ rec) {
  pdl_trigger();  // the next call's first kernel may start its prologue now
  // column hq of row b: KV head h = hq / Gt, column gc = hq % Gt of the head, in column tile
  // gc / 8 (unit (b h_kv + h) CT + gc / 8) as its column gc % 8 (G columns per unit)
  const int bq = blockIdx.x, b = bq / h_q, hq = bq % h_q;
  const int Gt = h_q / h_kv, CT = (Gt + kMaxG - 1) / kMaxG, gc = hq % Gt;
  const int u = (b * h_kv + hq / Gt) * CT + gc / kMaxG, hh = gc % kMaxG;
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
  const int heads = h_q / n_q, head = (hq / Gt) * (Gt / n_q) + gc / n_q, tok = gc % n_q;
  if (rec) {  // uniform over the grid
    float* r = rec + (((size_t)b * n_q + tok) * heads + head) * (kD + 2);
    if (tid == 0) {
      r[0] = Mx;
      r[1] = l;
    }
    if (tid < kD) r[2 + tid] = op[tid];
    return;
  }
  __syncthreads();
  float r0 = 0.f, r1 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    r0 = fmaf(rv[i], op[qtr * 32 + i], r0);
    r1 = fmaf(rv[i + 1], op[qtr * 32 + i + 1], r1);
  }
  part[qtr][d] = r0 + r1;
  __syncthreads();
  if (tid < kD)
    out[(((size_t)b * n_q + tok) * heads + head) * kD + tid] = (part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid]);
}

// Dynamic shared memory of one split CTA: the fixed part for the value rate plus the ring
// (which the warps' merge and, through it, the combine's partials reuse).
inline int split_smem_bytes(int v_rate, int tile_bytes, int warps) {
  const int fixed = v_rate == 3 ? sm_ring<3>() : v_rate == 4 ? sm_ring<4>() : sm_ring<2>();
  const size_t ring = size_t(2 * warps) * tile_bytes;
  return fixed + int(std::max(ring, size_t(warps) * 8 * kD * 4));
}

// Once per device and variant: the largest dynamic shared memory the kernel may use (the
// device's per-block opt-in limit minus the kernel's static shared memory), set as the
// kernel's limit together with the whole unified L1/shared array as shared memory.
template <int VR, bool NP, bool SC, bool NH, int W, bool PH>
cudaError_t configure_split(int* dyn_limit) {
  static int limit[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!limit[dev]) {
    int optin = 0;
    cudaFuncAttributes fa{};
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, split_kernel<VR, NP, SC, NH, W, PH>);
    if (e != cudaSuccess) return e;
    const int dyn = optin - int(fa.sharedSizeBytes);
    e = cudaFuncSetAttribute(split_kernel<VR, NP, SC, NH, W, PH>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(split_kernel<VR, NP, SC, NH, W, PH>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    limit[dev] = dyn;
  }
  *dyn_limit = limit[dev];
  return cudaSuccess;
}

template <int VR, bool NP, bool SC, bool NH, int W, bool PH>
cudaError_t launch_split(const SplitArgs& a, const DevLayout& L, unsigned n_ctas, int smem, cudaStream_t stream) {
  int limit = 0;
  cudaError_t e = configure_split<VR, NP, SC, NH, W, PH>(&limit);
  if (e != cudaSuccess) return e;
  if (smem > limit) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_ctas);
  cfg.blockDim = dim3(32 * W);
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_kernel<VR, NP, SC, NH, W, PH>, L, a);
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
static_assert(kPrepThreads == 8 * 32, "q-prep sums one B column per warp");

// Word j (0..63) of quad qi's B fragments from q' (qr [head][packed dim], fp32): lane =
// j % 32 = 4 n + t holds column n, dims 2t and 2t+1 of the quad; j < 32: the hi parts
// (with G <= 4: hi parts of heads 0..3 in columns 0-3, lo parts in columns 4-7), j >= 32:
// the lo parts (zero with G <= 4). Missing pairs and heads are zero.
__device__ __forceinline__ unsigned frag_word(const DevLayout& L, const float* qr, int G, int qi, int j) {
  const int lane = j & 31, n = lane >> 2, t = lane & 3;
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
  return lo ? pack_h2(v0 - r0, v1 - r1) : pack_h2(r0, r1);
}

// Gt: query columns of a KV head (query heads per KV head x n_q); a unit holds at most 8 of
// them (column tile ct = u % CT of cache unit u / CT, CT = ceil(Gt / 8)); G: the unit's
// fragment columns (Gt when CT = 1, else 8; columns past Gt stay zero).
__device__ __forceinline__ void prep_unit(const DevLayout& L, const void* __restrict__ q, int q_dtype, int h_q,
                                          int h_kv, int Gt, int n_q, float qscale, int u, unsigned* __restrict__ frag) {
  __shared__ __align__(16) float qs[kMaxG * kQsLd];  // q per group at 16-byte aligned columns
  __shared__ float qr[kMaxG * kD];                   // q' in packed order
  const int tid = threadIdx.x, ng = L.n_kgroups;
  const int CT = (Gt + kMaxG - 1) / kMaxG, G = CT == 1 ? Gt : kMaxG;
  const int cu = u / CT, ct = u % CT;
  const int b = cu / h_kv, h = cu % h_kv;
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
  // the packed-to-original coordinate map in shared memory (a parameter-bank read with a
  // different index in every lane would serialise)
  __shared__ short s_pc[kD];
  if (tid < kD) s_pc[tid] = L.packed_coord[tid];
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
    // column hh of the tile = column gc of the KV head: query head h Gt / n_q + gc / n_q at
    // query token gc % n_q of q [b][token][head]
    const int gc = ct * kMaxG + hh;
    if (gc >= Gt) continue;
    const size_t qrow = ((size_t)b * n_q + gc % n_q) * h_q + (size_t)h * (Gt / n_q) + gc / n_q;
    qs[hh * kQsLd + pade + pe - L.group_off[ge]] = load_q(q, q_dtype, qrow * kD + s_pc[pe]);
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
  for (int e = tid; e < L.n_kquads * 64; e += kPrepThreads) frag[e] = frag_word(L, qr, G, e >> 6, e & 63);
  // Column sums of the rate-1 group's B fragments, as the products see them (the sum of
  // both fp16 halves of every word of the column, hi and lo arrays): the split kernel
  // turns the group's 0/1 operands into +-1 codes with them. Warp n sums column n in a
  // fixed order (deterministic).
  int g1 = -1;
  for (int gi = 0; gi < ng; ++gi)
    if (L.group_rate[gi] == 1) g1 = gi;
  if (g1 >= 0) {
    const int n = tid >> 5, ln = tid & 31;   // 8 warps, one per B column
    const int q0 = L.group_quad0[g1], nw = L.group_nquads[g1] * 8;  // 8 words of column n per quad
    float acc = 0.f;
    for (int w = ln; w < nw; w += 32) {
      const int qi = q0 + (w >> 3), k = w & 7, j = (k >> 2) * 32 + 4 * n + (k & 3);
      const unsigned x = frag_word(L, qr, G, qi, j);
      acc += __half2float(__ushort_as_half((unsigned short)(x & 0xffffu))) +
             __half2float(__ushort_as_half((unsigned short)(x >> 16)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (ln == 0) reinterpret_cast<float*>(frag + kMaxQuads * 64)[n] = acc;
  }
}

// The KV head of q' unit u (column tiles of ceil(Gt / 8) per cache unit).
__device__ __forceinline__ int unit_head(int u, int h_kv, int Gt) { return u / ((Gt + kMaxG - 1) / kMaxG) % h_kv; }

// PH: heads[h] is the layout of KV head h (else L for every head).
template <bool PH>
__global__ void __launch_bounds__(kPrepThreads) qprep_kernel(DevLayout L, const DevLayout* __restrict__ heads,
                                                             const void* __restrict__ q, int q_dtype,
                                                             int h_q, int h_kv, int Gt, int n_q, float qscale,
                                                             unsigned* __restrict__ qfrag) {
  // launched after the kernel before it has completed: the split kernel may start now
  pdl_trigger();
  const int u = blockIdx.x;
  if constexpr (PH)
    prep_unit(heads[unit_head(u, h_kv, Gt)], q, q_dtype, h_q, h_kv, Gt, n_q, qscale, u, qfrag + (size_t)u * kQfragWords);
  else
    prep_unit(L, q, q_dtype, h_q, h_kv, Gt, n_q, qscale, u, qfrag + (size_t)u * kQfragWords);
}

// First kernel of a decode step: blocks [0, n_enc) append the new tokens (four blocks per
// token and KV head), the others prepare q' of one unit each. PH: heads[h] is the layout of
// KV head h (else L for every head).
template <bool NC, bool PH>
__global__ void __launch_bounds__(kPrepThreads) step_prep_kernel(DevLayout L, const DevLayout* __restrict__ heads,
                                                                 const void* __restrict__ k,
                                                                 const void* __restrict__ v, int kv_dtype, int n_new,
                                                                 int batch, const int* __restrict__ seq_lens_before,
                                                                 CacheRef cache,
                                                                 const void* __restrict__ q, int q_dtype, int h_q,
                                                                 int h_kv, int Gt, int n_q, float qscale,
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
    if constexpr (PH)
      enc::encode_token_part<NC>(heads[h], k, v, kv_dtype, n_new, h_kv, seq_lens_before, cache, t, part, b, h);
    else
      enc::encode_token_part<NC>(L, k, v, kv_dtype, n_new, h_kv, seq_lens_before, cache, t, part, b, h);
  } else if (e - n_enc < batch * h_kv * ((Gt + kMaxG - 1) / kMaxG)) {  // (a cluster launch pads the grid)
    const int u = e - n_enc;
    if constexpr (PH)
      prep_unit(heads[unit_head(u, h_kv, Gt)], q, q_dtype, h_q, h_kv, Gt, n_q, qscale, u,
                qfrag + (size_t)u * kQfragWords);
    else
      prep_unit(L, q, q_dtype, h_q, h_kv, Gt, n_q, qscale, u, qfrag + (size_t)u * kQfragWords);
  }
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

// Dynamic shared memory a split CTA may use: the device's per-block opt-in limit less a
// reserve for the kernel's static shared memory (a few KB: group table, merge scalars).
constexpr int kStaticReserve = 6 * 1024;
int split_smem_limit() {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  return optin - kStaticReserve;
}

// Warps per split CTA: the most, up to 12, whose ring stages fit next to the tables (8 at
// least). Up to 12 warps a scheduler holds at most 3 of them, so every count keeps the
// 168-register budget (and 8 warps have up to 255).
int split_warps(int v_rate, int tile_bytes, int limit) {
  for (int w = 12; w > 8; --w)
    if (split_smem_bytes(v_rate, tile_bytes, w) <= limit) return w;
  return 8;
}

// The split kernel of one call (and, unless scores only, the merge in its last CTA per
// unit), launched as a programmatic dependent of the kernel that wrote the q' fragments
// (and, after an append, the new tokens). n_q query tokens per row: h_q n_q query columns,
// G = h_q n_q / h_kv per KV head.
cudaError_t launch_attention(const DevLayout& L, const DecodePlan& plan, int batch, int h_q, int h_kv, int n_q,
                             const CacheRef& cache, const int* seq_lens, float* out, void* workspace,
                             int len_add, bool after_append, cudaStream_t stream, float* scores = nullptr,
                             long long scores_ld = 0, float* rec = nullptr, const DevLayout* heads = nullptr) {
  const int hc = h_q * n_q, Gt = hc / h_kv, CT = (Gt + kMaxG - 1) / kMaxG, G = CT == 1 ? Gt : kMaxG;
  // G <= 4: the q' hi and lo parts share one m16n8k8 product (columns 0-3 and 4-7)
  const bool np = G <= 4;
  const bool sc = scores != nullptr, nh = L.norm_fp16 != 0;
  if (!sc && (L.v_rate < 1 || L.v_rate > 4)) return cudaErrorInvalidValue;
  const int limit = split_smem_limit();
  const int vr = sc ? 1 : L.v_rate;  // the scores-only variant builds no value table
  // 9-11 warps only for value rates 1-2: the rate-3/4 value path needs more registers
  // than 168 and spills there (measured slower than 8 warps); the scores-only form, off the
  // decode path, keeps to 12 or 8 warps too
  const int Wf = split_warps(vr, L.tile_bytes, limit), W = (sc || vr >= 3) && Wf < 12 ? 8 : Wf;
  const int smem = split_smem_bytes(vr, L.tile_bytes, W);
  if (smem > limit) return cudaErrorInvalidValue;
  const long long units = (long long)batch * h_kv * CT;
  SplitArgs a;
  a.cache = cache;
  a.seq_lens = seq_lens;
  a.max_tiles = plan.max_tiles;
  a.n_ctas = plan.n_ctas;
  a.n_parts = plan.n_parts;
  a.total_tiles = units * plan.max_tiles;
  a.h_q = hc;
  a.h_kv = h_kv;
  a.Gt = Gt;
  a.G = G;
  a.n_q = n_q;
  a.CT = CT;
  // q' fragments, the unit counters, then the partials
  char* ws = static_cast<char*>(workspace);
  a.qfrag = reinterpret_cast<const unsigned*>(ws);
  ws += qfrag_bytes(units);
  a.part_ml = reinterpret_cast<float*>(ws);
  a.part_o = reinterpret_cast<float*>(ws + align256(size_t(units) * plan.n_parts * G * 2 * sizeof(float)));
  a.scores = scores;
  a.scores_ld = scores_ld;
  a.len_add = len_add;
  a.wait_new = after_append ? 1 : 0;
  a.heads = heads;
  const unsigned n_ctas = unsigned(plan.n_ctas);
  cudaError_t e = split_variant(L.v_rate, np, sc, nh, [&](auto V, auto P, auto S, auto H) {
    constexpr int VR = decltype(V)::value;
    constexpr bool NPv = decltype(P)::value != 0, SCv = decltype(S)::value != 0, NHv = decltype(H)::value != 0;
    auto go = [&](auto ph) {
      constexpr bool PHv = decltype(ph)::value;
      if constexpr (!SCv && VR <= 2) {
        if (W == 11) return launch_split<VR, NPv, SCv, NHv, 11, PHv>(a, L, n_ctas, smem, stream);
        if (W == 10) return launch_split<VR, NPv, SCv, NHv, 10, PHv>(a, L, n_ctas, smem, stream);
        if (W == 9) return launch_split<VR, NPv, SCv, NHv, 9, PHv>(a, L, n_ctas, smem, stream);
      }
      return W == 12 ? launch_split<VR, NPv, SCv, NHv, 12, PHv>(a, L, n_ctas, smem, stream)
                     : launch_split<VR, NPv, SCv, NHv, 8, PHv>(a, L, n_ctas, smem, stream);
    };
    return heads ? go(std::true_type{}) : go(std::false_type{});
  });
  if (sc || e != cudaSuccess) return e;  // scores only: no merge
  return launch_dependent(combine_kernel, unsigned(batch * hc), kCombThreads, stream, (const float*)a.part_ml,
                          (const float*)a.part_o, plan.n_parts, plan.max_tiles, a.total_tiles, plan.n_ctas, G, hc,
                          h_kv, n_q, L.v_rot32, out, rec);
}

}  // namespace

DecodePlan plan_decode(int batch, int h_q, int h_kv, long long max_seq_len, int num_sms, int /*ctas_per_sm*/) {
  DecodePlan p{};
  // h_q counts query columns; more than 8 per KV head are split into column tiles
  const int Gt = h_q / h_kv, CT = (Gt + kMaxG - 1) / kMaxG, G = CT == 1 ? Gt : kMaxG;
  p.max_tiles = int((max_seq_len + kTile - 1) / kTile);
  if (p.max_tiles < 1) p.max_tiles = 1;
  const long long units = (long long)batch * h_kv * CT;
  const long long total = units * p.max_tiles;
  // one CTA per SM, slices of equal length (+-1 tile); a slice may span several units
  long long C = std::min<long long>(num_sms, total);
  // a unit meets at most ceil(C / units) + 1 slices; the merge takes up to kMaxParts
  while (C > 1 && (C + units - 1) / units + 1 > kMaxParts) --C;
  p.n_ctas = int(C);
  p.tiles_per_cta = int((total + C - 1) / C);
  p.n_parts = int((C + units - 1) / units + 1);
  p.workspace_bytes = qfrag_bytes(units) +
                      align256(size_t(units) * p.n_parts * G * 2 * sizeof(float)) +
                      size_t(units) * p.n_parts * G * kD * sizeof(float);
  return p;
}

cudaError_t launch_decode(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch,
                          int h_q, int h_kv, int n_q, const CacheRef& cache, const int* seq_lens, float softmax_scale,
                          float* out, void* workspace, cudaStream_t stream, float* rec, const DevLayout* heads) {
  const int Gt = h_q * n_q / h_kv;
  const long long units = (long long)batch * h_kv * ((Gt + kMaxG - 1) / kMaxG);
  // a plain launch: the split kernel, launched as soon as this kernel starts, reads the
  // cache, which the kernel before this one may write
  if (heads)
    qprep_kernel<true><<<unsigned(units), kPrepThreads, 0, stream>>>(
        L, heads, q, q_dtype, h_q, h_kv, Gt, n_q, softmax_scale * kLog2e, static_cast<unsigned*>(workspace));
  else
    qprep_kernel<false><<<unsigned(units), kPrepThreads, 0, stream>>>(
        L, nullptr, q, q_dtype, h_q, h_kv, Gt, n_q, softmax_scale * kLog2e, static_cast<unsigned*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, n_q, cache, seq_lens, out, workspace, 0, false, stream,
                          nullptr, 0, rec, heads);
}

namespace {
// One CTA of 128 threads per (batch row, query column): log-sum-exp merge of n_rec partial
// records (m, l, o') of the same column over disjoint token ranges, then o = R_V^T o'.
__global__ void __launch_bounds__(kD) merge_records_kernel(const float* __restrict__ recs, int n_rec,
                                                           long long rec_stride, const float* __restrict__ v_rot,
                                                           float* __restrict__ out) {
  const int col = blockIdx.x, d = threadIdx.x;
  __shared__ float op[kD];
  const float* r0 = recs + (size_t)col * (kD + 2);
  float M = -INFINITY;
  for (int r = 0; r < n_rec; ++r) M = fmaxf(M, r0[(size_t)r * rec_stride]);
  float den = 0.f, o = 0.f;
  if (M != -INFINITY)
    for (int r = 0; r < n_rec; ++r) {
      const float* x = r0 + (size_t)r * rec_stride;
      const float w = x[0] == -INFINITY ? 0.f : exp2f(x[0] - M) * x[1];
      den += w;
      o = fmaf(w, x[2 + d], o);
    }
  op[d] = den > 0.f ? o / den : 0.f;
  __syncthreads();
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
  for (int i = 0; i < kD; i += 2) {
    acc0 = fmaf(__ldg(v_rot + (size_t)i * kD + d), op[i], acc0);
    acc1 = fmaf(__ldg(v_rot + (size_t)(i + 1) * kD + d), op[i + 1], acc1);
  }
  out[(size_t)col * kD + d] = acc0 + acc1;
}
}  // namespace

cudaError_t launch_merge_records(const DevLayout& L, const float* recs, int n_rec, long long columns, float* out,
                                 cudaStream_t stream) {
  merge_records_kernel<<<unsigned(columns), kD, 0, stream>>>(recs, n_rec, columns * (kD + 2), L.v_rot32, out);
  return cudaGetLastError();
}

cudaError_t launch_scores(const DevLayout& L, const DecodePlan& plan, const void* q, int q_dtype, int batch, int h_q,
                          int h_kv, const CacheRef& cache, const int* seq_lens, float softmax_scale, float* scores,
                          long long scores_ld, void* workspace, cudaStream_t stream, const DevLayout* heads) {
  const int Gt = h_q / h_kv;
  const long long units = (long long)batch * h_kv * ((Gt + kMaxG - 1) / kMaxG);
  if (heads)
    qprep_kernel<true><<<unsigned(units), kPrepThreads, 0, stream>>>(
        L, heads, q, q_dtype, h_q, h_kv, Gt, 1, softmax_scale * kLog2e, static_cast<unsigned*>(workspace));
  else
    qprep_kernel<false><<<unsigned(units), kPrepThreads, 0, stream>>>(
        L, nullptr, q, q_dtype, h_q, h_kv, Gt, 1, softmax_scale * kLog2e, static_cast<unsigned*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, 1, cache, seq_lens, nullptr, workspace, 0, false, stream,
                          scores, scores_ld, nullptr, heads);
}

cudaError_t launch_decode_step(const DevLayout& L, const DecodePlan& plan, const void* k_new, const void* v_new,
                               int kv_dtype, int n_new, const int* seq_lens_before, const void* q, int q_dtype,
                               int batch, int h_q, int h_kv, int n_q, const CacheRef& cache, float softmax_scale,
                               float* out, void* workspace, cudaStream_t stream, const DevLayout* heads) {
  const int Gt = h_q * n_q / h_kv;
  const long long cache_units = (long long)batch * h_kv;
  const long long units = cache_units * ((Gt + kMaxG - 1) / kMaxG);  // q' units (column tiles)
  const long long n_enc = (long long)n_new * kEncodeParts * cache_units;
  cudaError_t e;
  if (!L.norm_correct) {
    e = launch_dependent(heads ? step_prep_kernel<false, true> : step_prep_kernel<false, false>,
                         unsigned(n_enc + units), kPrepThreads, stream, L, heads, k_new,
                         v_new, kv_dtype, n_new, batch, seq_lens_before, cache, q, q_dtype, h_q, h_kv, Gt, n_q,
                         softmax_scale * kLog2e, static_cast<unsigned*>(workspace), int(n_enc));
  } else {
    // norm correction: clusters of the four encode parts of a token; the q' blocks
    // follow, padded to a whole cluster (the padding blocks return at once)
    const long long n_blocks = (n_enc + units + kEncodeParts - 1) / kEncodeParts * kEncodeParts;
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
    e = cudaLaunchKernelEx(&cfg, heads ? step_prep_kernel<true, true> : step_prep_kernel<true, false>, L, heads,
                           k_new, v_new, kv_dtype, n_new, batch, seq_lens_before, cache, q, q_dtype, h_q, h_kv, Gt,
                           n_q, softmax_scale * kLog2e, static_cast<unsigned*>(workspace), int(n_enc));
  }
  if (e != cudaSuccess) return e;
  return launch_attention(L, plan, batch, h_q, h_kv, n_q, cache, seq_lens_before, out, workspace, n_new,
                          n_new > 0, stream, nullptr, 0, nullptr, heads);
}

}  // namespace bgtq
