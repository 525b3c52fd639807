// Host-side planning of libbgtq: seeded rotations, Lloyd-Max tables, block energy, rate
// allocation and the per-layer packing layout. Pure C++17 + libm, no CUDA.
//
// Sources: "Block-GTQ: RoPE-Block Rate Allocation for KV-Cache Quantization" (abstract,
// sentences 2-5) and the TurboQuant pipeline diagram ("random rotation", "per-coordinate
// MSE scalar quantisation"). Random draws: Philox4x32-10 (Salmon et al., SC'11) and the
// Box-Muller transform.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>

#include "bgtq_internal.h"

namespace bgtq {

namespace {
thread_local std::string g_err;
}

void set_error(const std::string& msg) { g_err = msg; }

bgtq_status fail(bgtq_status s, const std::string& msg) {
  g_err = msg;
  return s;
}

// ---------------------------------------------------------------- Philox + Gaussians
namespace {

struct Philox4 {
  uint32_t w[4];
};

// Ten Philox4x32 rounds: two 32x32->64 products with the Philox multipliers, the high
// halves xor-ed with the other counter words and the round key, the key bumped by the
// Weyl increments between rounds.
Philox4 philox4x32_10(Philox4 c, uint32_t k0, uint32_t k1) {
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t a = uint64_t(0xD2511F53u) * c.w[0];
    const uint64_t b = uint64_t(0xCD9E8D57u) * c.w[2];
    Philox4 n;
    n.w[0] = uint32_t(b >> 32) ^ c.w[1] ^ k0;
    n.w[1] = uint32_t(b);
    n.w[2] = uint32_t(a >> 32) ^ c.w[3] ^ k1;
    n.w[3] = uint32_t(a);
    c = n;
  }
  return c;
}

double unit_open(uint32_t hi, uint32_t lo) {
  return (double(hi >> 5) * 67108864.0 + double(lo >> 6) + 0.5) * (1.0 / 9007199254740992.0);
}

// Draws 0..count-1 of the N(0,1) stream (seed, stream): block n of Philox (counter
// n_lo, n_hi, stream, 0; key = seed halves) yields draws 2n and 2n+1 by Box-Muller.
void gaussian_stream(unsigned long long seed, uint32_t stream, long long count, double* out) {
  const uint32_t k0 = uint32_t(seed & 0xFFFFFFFFull), k1 = uint32_t(seed >> 32);
  const double two_pi = 6.283185307179586476925286766559;
  for (long long n = 0; 2 * n < count; ++n) {
    Philox4 c{{uint32_t(uint64_t(n) & 0xFFFFFFFFu), uint32_t(uint64_t(n) >> 32), stream, 0u}};
    Philox4 r = philox4x32_10(c, k0, k1);
    const double u1 = unit_open(r.w[0], r.w[1]);
    const double u2 = unit_open(r.w[2], r.w[3]);
    const double rad = std::sqrt(-2.0 * std::log(u1));
    out[2 * n] = rad * std::cos(two_pi * u2);
    if (2 * n + 1 < count) out[2 * n + 1] = rad * std::sin(two_pi * u2);
  }
}

// Rotation R (d x d, row-major, y = R x): the orthonormal factor Q of A = Q T, with T
// upper triangular and positive on its diagonal, where A[i][j] is draw i*d + j. The
// columns of A are orthonormalised left to right by Gram-Schmidt with one full
// re-orthogonalisation pass; the diagonal of T is then each column's remaining length,
// positive by construction.
void haar_rotation(unsigned long long seed, uint32_t stream, int d, std::vector<double>& r) {
  std::vector<double> a(size_t(d) * d);
  gaussian_stream(seed, stream, (long long)d * d, a.data());
  std::vector<double> q(size_t(d) * d, 0.0);  // column-major: q[col*d + row]
  std::vector<double> v(d);
  for (int j = 0; j < d; ++j) {
    for (int i = 0; i < d; ++i) v[i] = a[size_t(i) * d + j];
    for (int pass = 0; pass < 2; ++pass) {
      for (int c = 0; c < j; ++c) {
        const double* qc = &q[size_t(c) * d];
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += qc[i] * v[i];
        for (int i = 0; i < d; ++i) v[i] -= dot * qc[i];
      }
    }
    double nrm = 0.0;
    for (int i = 0; i < d; ++i) nrm += v[i] * v[i];
    nrm = std::sqrt(nrm);
    for (int i = 0; i < d; ++i) q[size_t(j) * d + i] = v[i] / nrm;
  }
  r.assign(size_t(d) * d, 0.0);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) r[size_t(i) * d + j] = q[size_t(j) * d + i];
}

double gauss_pdf(double x) {
  return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) * 0.39894228040143267793994605993438;
}
double gauss_tail(double x) {  // P(X > x)
  return std::isinf(x) ? (x > 0 ? 0.0 : 1.0) : 0.5 * std::erfc(x * 0.70710678118654752440084436210485);
}

}  // namespace

// Lloyd-Max for N(0,1) with 2^bits levels. Both optimality conditions are applied in
// turn until the thresholds stop moving: centroid = mean of the density over its cell,
// threshold = midpoint of adjacent centroids. By symmetry the positive half is solved
// (cell edges 0 = e_0 < e_1 < ... < e_m = inf) and mirrored.
void lloyd_max_host(int bits, double* centroids, double* thresholds, double* mse) {
  const int m = 1 << (bits - 1);
  double e[17], c[16];
  e[0] = 0.0;
  e[m] = INFINITY;
  for (int i = 1; i < m; ++i) e[i] = 2.5 * i / m;
  for (int it = 0; it < 1000000; ++it) {
    for (int i = 0; i < m; ++i)
      c[i] = (gauss_pdf(e[i]) - gauss_pdf(e[i + 1])) / (gauss_tail(e[i]) - gauss_tail(e[i + 1]));
    double moved = 0.0;
    for (int i = 1; i < m; ++i) {
      const double ne = 0.5 * (c[i - 1] + c[i]);
      moved = std::max(moved, std::fabs(ne - e[i]));
      e[i] = ne;
    }
    if (moved < 1e-15) break;
  }
  double err = 1.0;
  for (int i = 0; i < m; ++i) {
    c[i] = (gauss_pdf(e[i]) - gauss_pdf(e[i + 1])) / (gauss_tail(e[i]) - gauss_tail(e[i + 1]));
    err -= 2.0 * (gauss_tail(e[i]) - gauss_tail(e[i + 1])) * c[i] * c[i];
  }
  if (centroids)
    for (int i = 0; i < m; ++i) {
      centroids[m + i] = c[i];
      centroids[m - 1 - i] = -c[i];
    }
  if (thresholds) {
    thresholds[m - 1] = 0.0;
    for (int i = 1; i < m; ++i) {
      thresholds[m - 1 + i] = e[i];
      thresholds[m - 1 - i] = -e[i];
    }
  }
  if (mse) *mse = err;
}

const char* last_error() { return g_err.c_str(); }

}  // namespace bgtq

using namespace bgtq;

namespace {

bool valid_rate(int r) { return r >= 1 && r <= 4; }

}  // namespace

extern "C" {

const char* bgtq_last_error_string(void) { return bgtq::last_error(); }

// 200: layout options, n_packed and flags in bgtq_layout_info, multi-token calls
int bgtq_version(void) { return 200; }

bgtq_status bgtq_lloyd_max(int bits, double* centroids, double* thresholds, double* mse) {
  if (!valid_rate(bits)) return fail(BGTQ_ERR_INVALID, "lloyd_max: bits must be 1..4");
  lloyd_max_host(bits, centroids, thresholds, mse);
  return BGTQ_OK;
}

namespace {
// Energy score of every KV head [BGTQ s3]: per_head[h * 64 + j].
bgtq_status energy_per_head(const char* who, const float* q_cal, long long n_q, int h_q, const float* k_cal,
                            long long n_k, int h_kv, double* per_head) {
  if (!q_cal || !k_cal || !per_head) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null pointer");
  if (n_q <= 0 || n_k <= 0 || h_q <= 0 || h_kv <= 0 || h_q % h_kv)
    return fail(BGTQ_ERR_INVALID, std::string(who) + ": need n_q, n_k > 0 and h_q a multiple of h_kv");
  const int grp = h_q / h_kv;
  std::vector<double> qe(kBlocks), ke(kBlocks);
  for (int h = 0; h < h_kv; ++h) {
    std::fill(qe.begin(), qe.end(), 0.0);
    std::fill(ke.begin(), ke.end(), 0.0);
    for (long long n = 0; n < n_q; ++n)
      for (int g = 0; g < grp; ++g) {
        const float* x = q_cal + (size_t(n) * h_q + size_t(h) * grp + g) * kD;
        for (int j = 0; j < kBlocks; ++j)
          qe[j] += double(x[j]) * x[j] + double(x[j + kBlocks]) * x[j + kBlocks];
      }
    for (long long n = 0; n < n_k; ++n) {
      const float* x = k_cal + (size_t(n) * h_kv + h) * kD;
      for (int j = 0; j < kBlocks; ++j)
        ke[j] += double(x[j]) * x[j] + double(x[j + kBlocks]) * x[j + kBlocks];
    }
    for (int j = 0; j < kBlocks; ++j)
      per_head[size_t(h) * kBlocks + j] = (qe[j] / (double(n_q) * grp)) * (ke[j] / double(n_k));
  }
  return BGTQ_OK;
}
}  // namespace

bgtq_status bgtq_block_energy(const float* q_cal, long long n_q, int h_q, const float* k_cal,
                              long long n_k, int h_kv, double* score_out) {
  if (!score_out) return fail(BGTQ_ERR_INVALID, "block_energy: null pointer");
  std::vector<double> per(size_t(h_kv > 0 ? h_kv : 0) * kBlocks);
  const bgtq_status st = energy_per_head("block_energy", q_cal, n_q, h_q, k_cal, n_k, h_kv, per.data());
  if (st != BGTQ_OK) return st;
  for (int j = 0; j < kBlocks; ++j) {
    score_out[j] = 0.0;
    for (int h = 0; h < h_kv; ++h) score_out[j] += per[size_t(h) * kBlocks + j];
  }
  return BGTQ_OK;
}

bgtq_status bgtq_block_energy_heads(const float* q_cal, long long n_q, int h_q, const float* k_cal,
                                    long long n_k, int h_kv, double* score_out) {
  return energy_per_head("block_energy_heads", q_cal, n_q, h_q, k_cal, n_k, h_kv, score_out);
}

bgtq_status bgtq_allocate_rates(const double* score, int n_blocks, int min_rate, int max_rate,
                                long long total_bits, const double* distortion, int* rates_out) {
  if (!score || !rates_out || n_blocks <= 0) return fail(BGTQ_ERR_INVALID, "allocate_rates: bad arguments");
  if (min_rate < 0 || !valid_rate(max_rate) || min_rate > max_rate)
    return fail(BGTQ_ERR_INVALID, "allocate_rates: need 0 <= min_rate <= max_rate <= 4, max_rate >= 1");
  if (total_bits < (long long)n_blocks * min_rate || total_bits > (long long)n_blocks * max_rate)
    return fail(BGTQ_ERR_INFEASIBLE, "allocate_rates: budget outside [n*min_rate, n*max_rate]");
  double D[6] = {0, 0, 0, 0, 0, 0};
  for (int r = min_rate; r <= max_rate; ++r) {
    if (distortion) D[r] = distortion[r];
    else if (r == 0) D[r] = 1.0;  // an uncoded N(0,1) coordinate decodes to 0: its variance
    else lloyd_max_host(r, nullptr, nullptr, &D[r]);
  }
  for (int j = 0; j < n_blocks; ++j) {
    if (!std::isfinite(score[j])) return fail(BGTQ_ERR_INVALID, "allocate_rates: non-finite score");
    rates_out[j] = min_rate;
  }
  for (long long step = (long long)n_blocks * min_rate; step < total_bits; ++step) {
    int best = -1;
    double best_gain = -INFINITY;
    for (int j = 0; j < n_blocks; ++j) {
      if (rates_out[j] >= max_rate) continue;
      const double gain = score[j] * (D[rates_out[j]] - D[rates_out[j] + 1]);
      if (gain > best_gain) {
        best_gain = gain;
        best = j;
      }
    }
    rates_out[best] += 1;
  }
  return BGTQ_OK;
}

bgtq_status bgtq_layout_create(const int* k_rates, int v_rate, unsigned long long seed, bgtq_layout** out) {
  return bgtq_layout_create_ex(k_rates, v_rate, seed, 0u, out);
}

bgtq_status bgtq_layout_create_ex(const int* k_rates, int v_rate, unsigned long long seed, unsigned flags,
                                  bgtq_layout** out) {
  if (!k_rates || !out) return fail(BGTQ_ERR_INVALID, "layout_create: null pointer");
  *out = nullptr;
  if (flags & ~(BGTQ_LAYOUT_NORM_CORRECT | BGTQ_LAYOUT_NORM_FP16))
    return fail(BGTQ_ERR_INVALID, "layout_create: unknown option flag");
  int sum = 0;
  for (int j = 0; j < kBlocks; ++j) {
    if (k_rates[j] < 0 || k_rates[j] > 4) return fail(BGTQ_ERR_INVALID, "layout_create: key rates must be 0..4");
    sum += k_rates[j];
  }
  if ((2 * sum) % 8) return fail(BGTQ_ERR_INVALID, "layout_create: key rates must sum to a multiple of 4");
  if (sum == 0) return fail(BGTQ_ERR_INVALID, "layout_create: at least one key block must be coded");
  if (!valid_rate(v_rate)) return fail(BGTQ_ERR_INVALID, "layout_create: v_rate must be 1..4");
  bgtq_layout* L = new (std::nothrow) bgtq_layout();
  if (!L) return fail(BGTQ_ERR_NOMEM, "layout_create: out of host memory");
  std::memcpy(L->k_rates, k_rates, sizeof(L->k_rates));
  L->v_rate = v_rate;
  L->seed = seed;
  L->flags = flags;
  L->norm_bytes = (flags & BGTQ_LAYOUT_NORM_FP16) ? 2 : 4;
  // Equal-rate blocks form one group; groups by descending rate, blocks ascending,
  // coordinate j before j + 64.
  int ng = 0, pd = 0, bit = 0;
  for (int r = 4; r >= 1; --r) {
    int count = 0;
    for (int j = 0; j < kBlocks; ++j)
      if (k_rates[j] == r) {
        L->packed_coord[pd + 2 * count] = j;
        L->packed_coord[pd + 2 * count + 1] = j + kBlocks;
        ++count;
      }
    if (!count) continue;
    L->group_rate[ng] = r;
    L->group_dim[ng] = 2 * count;
    L->group_off[ng] = pd;
    L->group_bitoff[ng] = bit;
    pd += 2 * count;
    bit += 2 * count * r;
    ++ng;
  }
  L->n_kgroups = ng;
  L->n_packed = pd;  // rate-0 blocks are in no group: their coordinates are not stored
  for (int p = pd; p < kD; ++p) L->packed_coord[p] = 0;
  for (int g = ng; g < kMaxGroups; ++g) L->group_rate[g] = L->group_dim[g] = L->group_off[g] = L->group_bitoff[g] = 0;
  for (int g = 0; g < ng; ++g) haar_rotation(seed, uint32_t(L->group_rate[g]), L->group_dim[g], L->rot[g]);
  haar_rotation(seed, 0u, kD, L->rot[ng]);
  for (int r = 0; r < 5; ++r)
    for (int i = 0; i < 16; ++i) L->centroid[r][i] = L->threshold[r][i] = 0.0;
  L->mse[0] = 0.0;
  for (int r = 1; r <= 4; ++r) lloyd_max_host(r, L->centroid[r], L->threshold[r], &L->mse[r]);
  for (int r = 1; r <= 4; ++r)
    for (int i = (1 << r) - 1; i < 16; ++i) L->threshold[r][i] = INFINITY;
  L->k_record_bytes = bit / 8;
  L->v_record_bytes = 16 * v_rate;
  L->bytes_per_token = L->k_record_bytes + L->v_record_bytes + L->norm_bytes * (ng + 1);
  L->tile_bytes = kTile * L->bytes_per_token;
  *out = L;
  return BGTQ_OK;
}

bgtq_status bgtq_layout_get_info(const bgtq_layout* L, bgtq_layout_info* info) {
  if (!L || !info) return fail(BGTQ_ERR_INVALID, "layout_get_info: null pointer");
  info->head_dim = kD;
  info->n_blocks = kBlocks;
  info->n_kgroups = L->n_kgroups;
  for (int g = 0; g < kMaxGroups; ++g) {
    info->group_rate[g] = L->group_rate[g];
    info->group_dim[g] = L->group_dim[g];
  }
  info->v_rate = L->v_rate;
  info->k_record_bytes = L->k_record_bytes;
  info->v_record_bytes = L->v_record_bytes;
  info->bytes_per_token = L->bytes_per_token;
  info->tile_tokens = kTile;
  info->tile_bytes = L->tile_bytes;
  info->seed = L->seed;
  info->flags = L->flags;
  info->norm_bytes = L->norm_bytes;
  info->n_packed = L->n_packed;
  return BGTQ_OK;
}

bgtq_status bgtq_layout_rotation(const bgtq_layout* L, int group, double* out, long long max_elems) {
  if (!L || !out) return fail(BGTQ_ERR_INVALID, "layout_rotation: null pointer");
  if (group < 0 || group > L->n_kgroups) return fail(BGTQ_ERR_INVALID, "layout_rotation: bad group");
  const std::vector<double>& r = L->rot[group];
  if ((long long)r.size() > max_elems) return fail(BGTQ_ERR_INVALID, "layout_rotation: output too small");
  std::memcpy(out, r.data(), r.size() * sizeof(double));
  return BGTQ_OK;
}

bgtq_status bgtq_layout_coords(const bgtq_layout* L, int* packed_to_coord) {
  if (!L || !packed_to_coord) return fail(BGTQ_ERR_INVALID, "layout_coords: null pointer");
  std::memcpy(packed_to_coord, L->packed_coord, sizeof(L->packed_coord));
  return BGTQ_OK;
}

long long bgtq_cache_bytes(const bgtq_layout* L, int batch, int h_kv, long long tokens) {
  if (!L || batch < 0 || h_kv < 0 || tokens < 0) {
    set_error("cache_bytes: bad arguments");
    return -1;
  }
  const long long tiles = (tokens + kTile - 1) / kTile;
  return (long long)batch * h_kv * tiles * L->tile_bytes;
}

}  // extern "C"
