// Internal types shared by the host planner, the ABI layer and the kernels of libbgtq.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/bgtq.h"

namespace bgtq {

constexpr int kD = BGTQ_HEAD_DIM;        // 128
constexpr int kBlocks = BGTQ_N_BLOCKS;   // 64
constexpr int kTile = BGTQ_TILE_TOKENS;  // 64 tokens per tile
constexpr int kChunk = 16;               // tokens per V-code chunk
constexpr int kMaxG = 8;                 // query columns of one unit's tensor-core tile
constexpr int kMaxCols = BGTQ_MAX_GQA;   // query columns per KV head: column tiles of 8
constexpr int kMaxGroups = BGTQ_MAX_KGROUPS;
constexpr int kMaxQuads = 20;            // sum over groups of ceil(d_g / 8) <= 128/8 + 3
constexpr int kEncodeParts = 4;          // encode CTAs per (token, KV head), 32 outputs each
constexpr int kBulkMinTokens = 4;        // appends of this many tokens per row or more (2 or more when
                                         // batch x KV heads >= 256): the bulk encoder

// Decode lookup tables, built once per layout (host, at upload) in the order the split
// kernel keeps them in shared memory: 256 rows of 256 bytes (bytes 0-127: 16 copies of the
// rate-2 entry of a code byte, two slots' fp16 pairs; bytes 128-255: 16 copies of the rate-4
// entry, the hi and lo fp16 pairs of one slot), then 64 rows of 128 bytes (16 copies of the
// rate-3 hi and lo pairs of a 6-bit field), then the value table (rate 3: 64 entries x 32
// lanes, rate 4: 256 shared entries; 4 bytes each).
constexpr int kTbl8Bytes = 256 * 256;
constexpr int kTbl3Bytes = 64 * 128;
constexpr int kTblVBytes = 64 * 32 * 4;
constexpr int kTablesBytes = kTbl8Bytes + kTbl3Bytes + kTblVBytes;

// Everything a kernel needs about one layer's packing, passed by value.
struct alignas(16) DevLayout {  // (16-byte multiple: copied to shared memory in 16-byte units)
  int n_kgroups;
  int n_packed;         // stored key dimensions (packed dims n_packed..127 do not exist)
  int v_rate;
  int k_record_bytes;   // Kb
  int tile_bytes;
  int vcode_off;        // byte offsets inside a tile
  int knorm_off;
  int vnorm_off;
  int norm_fp16;        // norms stored as fp16 (else fp32)
  int norm_correct;     // NC: stored norm |x| sqrt(d) / |c|
  int group_rate[kMaxGroups];
  int group_dim[kMaxGroups];
  int group_off[kMaxGroups];     // first packed dimension of the group
  int group_bitoff[kMaxGroups];  // first bit of the group inside a K record
  short packed_coord[kD];        // packed key dimension -> original coordinate
  double threshold[5][16];       // [rate][k], fp64 (2^rate - 1 used)

  const double* k_rot64[kMaxGroups];  // d_g x d_g, TRANSPOSED: element (i, j) of R at j * d + i
  const double* v_rot64;              // 128 x 128, transposed likewise
  const float* k_rot32[kMaxGroups];  // row-major, rows padded to k_rot32_ld[g] floats (a multiple of 4)
  const float* k_rot32t[kMaxGroups]; // d_g x d_g fp32, transposed like k_rot64 (the bulk encoder)
  const float* v_rot32t;             // 128 x 128 fp32, transposed
  int k_rot32_ld[kMaxGroups];
  const float* v_rot32;
  const double* centroid64;      // [rate][code] at rate * 16 + code, fp64 (norm correction)
  unsigned* status;
  // Fragment-major K area: each group's packed dims cut into quads of 4 pairs (8 dims),
  // the last quad of a group holding the remaining 1-3 pairs.
  int n_kquads;
  int group_quad0[kMaxGroups];
  int group_nquads[kMaxGroups];
  int quad_off[kMaxQuads];       // byte offset of the quad's block inside a tile
  int quad_np[kMaxQuads];        // pairs in the quad (1..4)
  int quad_dim0[kMaxQuads];      // first packed dimension of the quad
  float inv_kappa_group[kMaxGroups];  // 1 / kappa of each group's rate
  float kappa[5];                // per-rate scale making the rate-1/2 fp16 key codebooks exact
  float kappa_v;                 // scale of the fp16 value codebook
  // fp16 bit patterns of the codebooks the decode kernels build their pair tables from:
  // keys of rates 1-2 scaled by kappa (exact), rates 3-4 as hi + lo parts (kappa 1);
  // values scaled by kappa_v.
  unsigned short kc2[4];
  unsigned short kc3[2][8];      // [hi, lo][code]
  unsigned short kc4[2][16];
  unsigned short vc[16];
  const unsigned char* tables;   // the decode lookup tables (kTablesBytes, 16-byte aligned)
};

// Where the packed tiles of a call live. Contiguous: [batch][h_kv][n_tiles][tile].
// Paged: a pool of num_pages pages, page p = [h_kv][tile] (one 64-token span of one row),
// and table[b * n_tiles + i] = the page of tile i of row b.
struct CacheRef {
  uint8_t* base;
  const int* table;      // paged: [batch][n_tiles] page ids; nullptr: contiguous
  long long n_tiles;     // tiles a row can hold (contiguous: capacity / 64; paged: table width)
  long long num_pages;   // paged: pages in the pool
};

#ifdef __CUDACC__
// Tile i of row b, KV head h. A page id outside the pool sets BGTQ_STATUS_BAD_PAGE and
// gives nullptr (the caller skips the tile).
__device__ __forceinline__ uint8_t* tile_ptr(const CacheRef& c, const DevLayout& L, int b, int h, int h_kv,
                                             long long i) {
  if (!c.table) return c.base + (((size_t)b * h_kv + h) * c.n_tiles + i) * (size_t)L.tile_bytes;
  const long long p = c.table[(size_t)b * c.n_tiles + i];
  if (p < 0 || p >= c.num_pages) {
    atomicOr(L.status, BGTQ_STATUS_BAD_PAGE);
    return nullptr;
  }
  return c.base + ((size_t)p * h_kv + h) * (size_t)L.tile_bytes;
}
// Whether tile i of row b has a page in the pool (contiguous caches: always).
__device__ __forceinline__ bool tile_present(const CacheRef& c, int b, long long i) {
  if (!c.table) return true;
  const long long p = c.table[(size_t)b * c.n_tiles + i];
  return p >= 0 && p < c.num_pages;
}
#endif

}  // namespace bgtq

struct bgtq_layout {
  int k_rates[bgtq::kBlocks];
  int v_rate;
  unsigned long long seed;
  int n_kgroups;
  int group_rate[bgtq::kMaxGroups];
  int group_dim[bgtq::kMaxGroups];
  int group_off[bgtq::kMaxGroups];
  int group_bitoff[bgtq::kMaxGroups];
  int packed_coord[bgtq::kD];
  std::vector<double> rot[bgtq::kMaxGroups + 1];  // K groups, then V at index n_kgroups
  double centroid[5][16];
  double threshold[5][16];
  double mse[5];
  int k_record_bytes, v_record_bytes, bytes_per_token, tile_bytes;
  unsigned flags;   // BGTQ_LAYOUT_* options
  int norm_bytes;   // 4 or 2
  int n_packed;     // stored key dimensions: 128 minus two per rate-0 block
  // device copy
  int device = -1;
  void* dev_block = nullptr;
  bgtq::DevLayout dev{};
};

// One layout per KV head (bgtq_layout_set_create): the device array of their DevLayouts,
// each with the common tile stride and the set's status word.
struct bgtq_layout_set {
  int n = 0;                   // KV heads
  int device = -1;
  int tile_stride = 0;         // bytes per tile of every head (the largest tile of the layouts)
  void* dev_block = nullptr;   // status word, then DevLayout[n]
  bgtq::DevLayout* heads = nullptr;
  bgtq::DevLayout head0{};     // heads[0] as the host passes it by value
};

namespace bgtq {
void set_error(const std::string& msg);
bgtq_status fail(bgtq_status s, const std::string& msg);
// Host Lloyd-Max, also used by the layout builder.
void lloyd_max_host(int bits, double* centroids, double* thresholds, double* mse);
}  // namespace bgtq
