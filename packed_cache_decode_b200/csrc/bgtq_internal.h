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
constexpr int kMaxG = BGTQ_MAX_GQA;
constexpr int kMaxGroups = BGTQ_MAX_KGROUPS;
constexpr int kMaxChunks = 12;           // sum over groups of ceil(d_g / 16) <= 128/16 + 4
constexpr int kEncodeParts = 4;          // encode CTAs per (token, KV head), 32 outputs each

// Everything a kernel needs about one layer's packing, passed by value.
struct DevLayout {
  int n_kgroups;
  int v_rate;
  int k_record_bytes;   // Kb
  int tile_bytes;
  int vcode_off;        // byte offsets inside a tile
  int knorm_off;
  int vnorm_off;
  int group_rate[kMaxGroups];
  int group_dim[kMaxGroups];
  int group_off[kMaxGroups];     // first packed dimension of the group
  int group_bitoff[kMaxGroups];  // first bit of the group inside a K record
  short packed_coord[kD];        // packed key dimension -> original coordinate
  float centroid[5][16];         // [rate][code], fp32
  double threshold[5][16];       // [rate][k], fp64 (2^rate - 1 used)
  const double* k_rot64[kMaxGroups];  // d_g x d_g, TRANSPOSED: element (i, j) of R at j * d + i
  const double* v_rot64;              // 128 x 128, transposed likewise
  const float* k_rot32[kMaxGroups];
  const float* k_rot32t[kMaxGroups];  // transposed copies (column-major), back to back
  int k_rot32t_off[kMaxGroups];       // float offset of group g's copy from k_rot32t[0]
  int k_rot32t_floats;                // sum of d_g^2
  const float* v_rot32;
  unsigned* status;
  // Tensor-core decode: 16-dimension chunks of the K record, per group.
  int n_kchunks;
  int group_chunk0[kMaxGroups];
  int group_nchunks[kMaxGroups];
  int chunk_koff[kMaxChunks];    // byte offset of the chunk's block inside a tile (chunk-major keys)
  int chunk_dim0[kMaxChunks];    // first packed dimension of the chunk
  int chunk_ndim[kMaxChunks];    // valid dimensions in the chunk (<= 16)
  int chunk_group[kMaxChunks];
  int chunk_rate[kMaxChunks];
  float inv_kappa_group[kMaxGroups];  // 1 / kappa of each group's rate
  float kappa[5];                // per-rate scale making the rate-1/2 fp16 key codebooks exact
  float kappa_v;                 // scale of the fp16 value codebook
  // Pair tables: entry (a | b << r) holds the fp16 pair (value(a), value(b)).
  const unsigned* klut12;        // rate 1: 4 entries at 0; rate 2: 16 entries at 4 (kappa-scaled)
  const unsigned* klut34;        // rate 3: 64 entries at 0; rate 4: 256 at 64; entry = {hi pair, lo pair}
  const unsigned* klut1q;        // rate 1, 16 entries: four codes -> {pair (0,1), pair (2,3)} (kappa-scaled)
  const unsigned* vlut;          // value codebook pairs, 2^(2 v_rate) entries (fp16, times kappa_v)
};

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
  // device copy
  int device = -1;
  void* dev_block = nullptr;
  bgtq::DevLayout dev{};
};

namespace bgtq {
void set_error(const std::string& msg);
bgtq_status fail(bgtq_status s, const std::string& msg);
// Host Lloyd-Max, also used by the layout builder.
void lloyd_max_host(int bits, double* centroids, double* thresholds, double* mse);
}  // namespace bgtq
