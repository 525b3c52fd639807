// Device-side entry points of the C ABI (include/bgtq.h): layout upload, encode-append,
// decode attention, workspace sizing and the device status word. Every argument is
// checked before anything is launched; CUDA errors are mapped to BGTQ_ERR_CUDA.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <new>
#include <cstring>
#include <string>
#include <vector>

#include "bgtq_internal.h"
#include "kernels.h"

using namespace bgtq;

namespace {

bgtq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BGTQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool valid_dtype(int d) { return d == BGTQ_F32 || d == BGTQ_BF16 || d == BGTQ_F16; }

// Nearest fp16 value of v (round half to even), as a double.
double round_fp16(double v) {
  if (v == 0.0) return 0.0;
  const double a = std::fabs(v);
  const int e = std::max(int(std::floor(std::log2(a))), -14);
  const double ulp = std::ldexp(1.0, e - 10);
  return std::copysign(std::nearbyint(a / ulp) * ulp, v);
}

unsigned short fp16_bits(double v) {
  __half h = __float2half_rn(float(v));
  return *reinterpret_cast<unsigned short*>(&h);
}


// Scale kappa_r such that fp16(kappa_r * c) represents the rate-r codebook as exactly as
// possible: +-1 for rate 1; otherwise the best of the 1024 scales that map the outer
// magnitude to [1, 2) (fp16 values with 10 fraction bits: max relative error 2.3e-7 at
// rate 2, 1.8e-5 at rate 3, 9.3e-5 at rate 4). Scaled values stay near 1, so 1/kappa can
// be folded into fp16 operands without leaving the normal range.
double codebook_kappa(const double* c, int r) {
  const int m = 1 << (r - 1);
  if (r == 1) return 1.0 / c[m];
  double best = 1.0, best_err = INFINITY;
  for (int A = 1024; A < 2048; ++A) {
    const double k = (A / 1024.0) / c[2 * m - 1];
    double err = 0.0;
    for (int i = m; i < 2 * m; ++i) {
      const double v = k * c[i];
      err = std::max(err, std::fabs(round_fp16(v) - v) / v);
    }
    if (err < best_err) {
      best_err = err;
      best = k;
    }
  }
  return best;
}

bgtq_status check_device(const bgtq_layout* L, const char* who) {
  if (!L) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null layout");
  if (L->device < 0 || !L->dev_block)
    return fail(BGTQ_ERR_DEVICE, std::string(who) + ": layout not uploaded (bgtq_layout_upload)");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, who);
  if (cur != L->device) return fail(BGTQ_ERR_DEVICE, std::string(who) + ": layout lives on another device");
  return BGTQ_OK;
}

}  // namespace

extern "C" {

void bgtq_layout_destroy(bgtq_layout* L) {
  if (!L) return;
  if (L->dev_block) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != L->device) cudaSetDevice(L->device);
    cudaFree(L->dev_block);
    if (cur >= 0 && cur != L->device) cudaSetDevice(cur);
  }
  delete L;
}

bgtq_status bgtq_layout_upload(bgtq_layout* L, int device) {
  if (!L) return fail(BGTQ_ERR_INVALID, "layout_upload: null layout");
  if (L->dev_block) return fail(BGTQ_ERR_INVALID, "layout_upload: already uploaded");
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e, "layout_upload");
  if (device < 0 || device >= ndev) return fail(BGTQ_ERR_INVALID, "layout_upload: bad device");
  int cur = -1;
  cudaGetDevice(&cur);
  if (cur != device && (e = cudaSetDevice(device)) != cudaSuccess) return cuda_fail(e, "layout_upload");

  const int ng = L->n_kgroups;
  size_t n64 = 0;
  for (int g = 0; g <= ng; ++g) n64 += L->rot[g].size();
  const size_t bytes = 256 + n64 * sizeof(double) + (2 * n64 + 3 * kD) * sizeof(float) + 256 + 5 * 16 * sizeof(double) +
                       kTablesBytes + 16;
  std::vector<unsigned char> host(bytes, 0);
  void* dblock = nullptr;
  if ((e = cudaMalloc(&dblock, bytes)) != cudaSuccess) {
    if (cur != device) cudaSetDevice(cur);
    return fail(BGTQ_ERR_NOMEM, std::string("layout_upload: ") + cudaGetErrorString(e));
  }
  DevLayout& D = L->dev;
  std::memset(&D, 0, sizeof(D));
  unsigned char* dptr = static_cast<unsigned char*>(dblock);
  size_t off = 256;  // status word first
  D.status = reinterpret_cast<unsigned*>(dptr);
  for (int g = 0; g <= ng; ++g) {
    // fp64 copies are stored transposed (element (i, j) at j * d + i) for coalesced reads
    const int d = int(std::lround(std::sqrt(double(L->rot[g].size()))));
    double* h64 = reinterpret_cast<double*>(host.data() + off);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) h64[size_t(j) * d + i] = L->rot[g][size_t(i) * d + j];
    const double* p = reinterpret_cast<const double*>(dptr + off);
    if (g < ng) D.k_rot64[g] = p; else D.v_rot64 = p;
    off += L->rot[g].size() * sizeof(double);
  }
  for (int g = 0; g <= ng; ++g) {
    // fp32 copies, row-major; key rows padded to a multiple of 4 floats (16-byte rows)
    const int d = int(std::lround(std::sqrt(double(L->rot[g].size()))));
    const int ld = g < ng ? (d + 3) / 4 * 4 : d;
    float* h32 = reinterpret_cast<float*>(host.data() + off);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < ld; ++j) h32[size_t(i) * ld + j] = j < d ? float(L->rot[g][size_t(i) * d + j]) : 0.f;
    const float* p = reinterpret_cast<const float*>(dptr + off);
    if (g < ng) {
      D.k_rot32[g] = p;
      D.k_rot32_ld[g] = ld;
    } else {
      D.v_rot32 = p;
    }
    off += size_t(d) * ld * sizeof(float);
  }
  off = (off + 15) / 16 * 16;  // 16-byte aligned: the bulk encoder fetches them with bulk copies
  for (int g = 0; g <= ng; ++g) {
    // fp32 copies transposed like the fp64 ones (element (i, j) at j * d + i); d is even, so
    // every copy is a multiple of 16 bytes and the next one stays aligned
    const int d = int(std::lround(std::sqrt(double(L->rot[g].size()))));
    float* h32 = reinterpret_cast<float*>(host.data() + off);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) h32[size_t(j) * d + i] = float(L->rot[g][size_t(i) * d + j]);
    const float* p = reinterpret_cast<const float*>(dptr + off);
    if (g < ng) D.k_rot32t[g] = p; else D.v_rot32t = p;
    off += size_t(d) * d * sizeof(float);
  }
  {
    // fp64 centroids (the norm correction sums the squares of a token's centroids)
    off = (off + 15) / 16 * 16;
    double* hc = reinterpret_cast<double*>(host.data() + off);
    for (int r = 0; r < 5; ++r)
      for (int i = 0; i < 16; ++i) hc[r * 16 + i] = r >= 1 && i < (1 << r) ? L->centroid[r][i] : 0.0;
    D.centroid64 = reinterpret_cast<const double*>(dptr + off);
    off += 5 * 16 * sizeof(double);
  }
  {
    // codebooks of the tensor-core decode: keys of rates 1-2 scaled (exact in fp16), rates
    // 3-4 as explicit hi + lo parts (kappa 1); values: one fp16 table scaled by the best
    // kappa of the value rate
    double kap[5] = {1, 1, 1, 1, 1};
    for (int r = 1; r <= 2; ++r) kap[r] = codebook_kappa(L->centroid[r], r);
    const double kap_v = codebook_kappa(L->centroid[L->v_rate], L->v_rate);
    for (int i = 0; i < 4; ++i) D.kc2[i] = fp16_bits(kap[2] * L->centroid[2][i]);
    for (int i = 0; i < 8; ++i) {
      D.kc3[0][i] = fp16_bits(round_fp16(L->centroid[3][i]));
      D.kc3[1][i] = fp16_bits(L->centroid[3][i] - round_fp16(L->centroid[3][i]));
    }
    for (int i = 0; i < 16; ++i) {
      D.kc4[0][i] = fp16_bits(round_fp16(L->centroid[4][i]));
      D.kc4[1][i] = fp16_bits(L->centroid[4][i] - round_fp16(L->centroid[4][i]));
    }
    for (int i = 0; i < (1 << L->v_rate); ++i) D.vc[i] = fp16_bits(kap_v * L->centroid[L->v_rate][i]);
    for (int r = 0; r < 5; ++r) D.kappa[r] = float(kap[r]);
    D.kappa_v = float(kap_v);
    for (int g = 0; g < ng; ++g) D.inv_kappa_group[g] = float(1.0 / kap[L->group_rate[g]]);
  }
  {
    // the decode lookup tables, in the split kernel's shared-memory order (16 copies of
    // every entry so that the lanes of a half-warp never share a bank)
    off = (off + 15) / 16 * 16;
    unsigned char* tb = host.data() + off;
    bool has[5] = {false, false, false, false, false};
    for (int g = 0; g < ng; ++g) has[L->group_rate[g]] = true;
    const unsigned short* c2 = has[2] ? D.kc2 : D.vc;  // equal when both are used (same rate, same kappa)
    auto put2 = [&](size_t at, unsigned x, unsigned y) {
      std::memcpy(tb + at, &x, 4);
      std::memcpy(tb + at + 4, &y, 4);
    };
    for (int e = 0; e < 256; ++e)
      for (int cp = 0; cp < 16; ++cp) {
        if (has[2] || L->v_rate == 2)
          put2(size_t(e) * 256 + cp * 8, c2[e & 3] | (unsigned(c2[(e >> 2) & 3]) << 16),
               c2[(e >> 4) & 3] | (unsigned(c2[e >> 6]) << 16));
        put2(size_t(e) * 256 + 128 + cp * 8, D.kc4[0][e & 15] | (unsigned(D.kc4[0][e >> 4]) << 16),
             D.kc4[1][e & 15] | (unsigned(D.kc4[1][e >> 4]) << 16));
      }
    for (int e = 0; e < 64; ++e)
      for (int cp = 0; cp < 16; ++cp)
        put2(size_t(kTbl8Bytes) + size_t(e) * 128 + cp * 8, D.kc3[0][e & 7] | (unsigned(D.kc3[0][e >> 3]) << 16),
             D.kc3[1][e & 7] | (unsigned(D.kc3[1][e >> 3]) << 16));
    unsigned* vt = reinterpret_cast<unsigned*>(tb + kTbl8Bytes + kTbl3Bytes);
    if (L->v_rate == 3)  // lane-private: entry e of lane l at word 32 e + l
      for (int i = 0; i < 64 * 32; ++i) vt[i] = D.vc[(i >> 5) & 7] | (unsigned(D.vc[(i >> 5) >> 3]) << 16);
    else if (L->v_rate == 4)
      for (int e = 0; e < 256; ++e) vt[e] = D.vc[e & 15] | (unsigned(D.vc[e >> 4]) << 16);
    D.tables = dptr + off;
    off += kTablesBytes;
  }
  {
    int qi = 0, koff = 0;
    for (int g = 0; g < ng; ++g) {
      const int r = L->group_rate[g], d = L->group_dim[g];
      D.group_quad0[g] = qi;
      D.group_nquads[g] = (d + 7) / 8;
      for (int c0 = 0; c0 < d; c0 += 8, ++qi) {
        const int np = std::min(8, d - c0) / 2;
        D.quad_off[qi] = koff;
        D.quad_np[qi] = np;
        D.quad_dim0[qi] = L->group_off[g] + c0;
        koff += 16 * np * r;
      }
    }
    D.n_kquads = qi;
  }
  D.n_kgroups = ng;
  D.n_packed = L->n_packed;
  D.v_rate = L->v_rate;
  D.k_record_bytes = L->k_record_bytes;
  D.tile_bytes = L->tile_bytes;
  D.vcode_off = kTile * L->k_record_bytes;
  D.knorm_off = D.vcode_off + kTile * L->v_record_bytes;
  D.vnorm_off = D.knorm_off + L->norm_bytes * kTile * ng;
  D.norm_fp16 = (L->flags & BGTQ_LAYOUT_NORM_FP16) ? 1 : 0;
  D.norm_correct = (L->flags & BGTQ_LAYOUT_NORM_CORRECT) ? 1 : 0;
  for (int g = 0; g < kMaxGroups; ++g) {
    D.group_rate[g] = L->group_rate[g];
    D.group_dim[g] = L->group_dim[g];
    D.group_off[g] = L->group_off[g];
    D.group_bitoff[g] = L->group_bitoff[g];
  }
  for (int p = 0; p < kD; ++p) D.packed_coord[p] = short(L->packed_coord[p]);
  for (int r = 0; r < 5; ++r)
    for (int i = 0; i < 16; ++i) D.threshold[r][i] = L->threshold[r][i];
  e = cudaMemcpy(dblock, host.data(), bytes, cudaMemcpyHostToDevice);
  if (cur != device) cudaSetDevice(cur);
  if (e != cudaSuccess) {
    cudaFree(dblock);
    return cuda_fail(e, "layout_upload");
  }
  L->dev_block = dblock;
  L->device = device;
  return BGTQ_OK;
}

}  // extern "C"

namespace {

// The checks and launches shared by the contiguous and the paged entry points; the
// caller has checked the cache description and passes it as a CacheRef.
bgtq_status encode_impl(const DevLayout& D, const char* who, const void* k, const void* v, int dtype, int batch,
                        int n_new, int h_kv, const int* seq_lens_dev, const CacheRef& c, void* stream,
                        const DevLayout* heads = nullptr) {
  if (!valid_dtype(dtype)) return fail(BGTQ_ERR_INVALID, std::string(who) + ": bad dtype");
  if (batch <= 0 || batch > 65535 || h_kv <= 0 || h_kv > 65535 || n_new < 0)
    return fail(BGTQ_ERR_INVALID, std::string(who) + ": bad batch / h_kv / n_new");
  if (n_new == 0) return BGTQ_OK;
  if (!k || !v || !seq_lens_dev) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null pointer");
  cudaError_t e = launch_tq_encode(D, k, v, dtype, batch, n_new, h_kv, seq_lens_dev, c,
                                   static_cast<cudaStream_t>(stream), heads);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return BGTQ_OK;
}

// Shape checks of the attention calls; on success *plan is the launch plan.
bgtq_status attention_checks(const char* who, int q_dtype, int batch, int h_q, int h_kv,
                             int n_q, long long row_tokens, long long max_seq_len, float softmax_scale, const void* q,
                             const int* seq_lens_dev, const void* out, void* workspace, size_t workspace_bytes,
                             DecodePlan* plan) {
  const std::string w(who);
  if (!valid_dtype(q_dtype)) return fail(BGTQ_ERR_INVALID, w + ": bad dtype");
  if (batch <= 0 || h_kv <= 0 || h_q <= 0 || h_q % h_kv || h_q / h_kv > kMaxCols)
    return fail(BGTQ_ERR_INVALID, w + ": need h_q = G * h_kv with G in 1..32");
  if (n_q < 1 || (h_q / h_kv) * n_q > kMaxCols)
    return fail(BGTQ_ERR_INVALID, w + ": need (h_q / h_kv) * n_q in 1..32");
  const int ct = ((h_q / h_kv) * n_q + kMaxG - 1) / kMaxG;
  if ((long long)batch * h_kv * ct > 65535) return fail(BGTQ_ERR_INVALID, w + ": too many units (batch * h_kv * column tiles > 65535)");
  if (max_seq_len < 0 || max_seq_len > row_tokens)
    return fail(BGTQ_ERR_CAPACITY, w + ": max_seq_len must be in [0, capacity]");
  if (!std::isfinite(softmax_scale)) return fail(BGTQ_ERR_INVALID, w + ": bad softmax_scale");
  if (!q || !seq_lens_dev || !out) return fail(BGTQ_ERR_INVALID, w + ": null pointer");
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, who);
  *plan = plan_decode(batch, h_q * n_q, h_kv, max_seq_len, sms);
  if (!workspace || workspace_bytes < plan->workspace_bytes)
    return fail(BGTQ_ERR_WORKSPACE, w + ": workspace missing or smaller than bgtq_workspace_bytes()");
  return BGTQ_OK;
}

// rec non-null: partial records (m, l, o') instead of outputs (out is then rec).
bgtq_status decode_impl(const DevLayout& D, const char* who, const void* q, int q_dtype, int batch, int h_q,
                        int h_kv, int n_q, const CacheRef& c, const int* seq_lens_dev, long long max_seq_len,
                        float softmax_scale, float* out, void* workspace, size_t workspace_bytes, void* stream,
                        float* rec = nullptr, const DevLayout* heads = nullptr) {
  DecodePlan plan;
  bgtq_status st = attention_checks(who, q_dtype, batch, h_q, h_kv, n_q, c.n_tiles * kTile, max_seq_len,
                                    softmax_scale, q, seq_lens_dev, out, workspace, workspace_bytes, &plan);
  if (st != BGTQ_OK) return st;
  cudaError_t e = launch_decode(D, plan, q, q_dtype, batch, h_q, h_kv, n_q, c, seq_lens_dev, softmax_scale, out,
                                workspace, static_cast<cudaStream_t>(stream), rec, heads);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return BGTQ_OK;
}

// n_q = 1: one query per row at the newest position; n_q = n_new: the new tokens' queries.
bgtq_status step_impl(const DevLayout& D, const char* who, const void* k_new, const void* v_new, int kv_dtype,
                      int n_new, const void* q, int q_dtype, int batch, int h_q, int h_kv, int n_q, const CacheRef& c,
                      const int* seq_lens_dev, long long max_seq_len, float softmax_scale, float* out,
                      void* workspace, size_t workspace_bytes, void* stream, const DevLayout* heads = nullptr) {
  if (!valid_dtype(kv_dtype)) return fail(BGTQ_ERR_INVALID, std::string(who) + ": bad dtype");
  if (n_new < 0 || (long long)n_new * kEncodeParts * batch * h_kv + (long long)batch * h_kv > 0x7fffffffLL)
    return fail(BGTQ_ERR_INVALID, std::string(who) + ": bad n_new");
  if (n_new > 0 && (!k_new || !v_new)) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null pointer");
  DecodePlan plan;
  bgtq_status st = attention_checks(who, q_dtype, batch, h_q, h_kv, n_q, c.n_tiles * kTile, max_seq_len,
                                    softmax_scale, q, seq_lens_dev, out, workspace, workspace_bytes, &plan);
  if (st != BGTQ_OK) return st;
  cudaError_t e = launch_decode_step(D, plan, k_new, v_new, kv_dtype, n_new, seq_lens_dev, q, q_dtype, batch,
                                     h_q, h_kv, n_q, c, softmax_scale, out, workspace,
                                     static_cast<cudaStream_t>(stream), heads);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return BGTQ_OK;
}

bgtq_status contiguous(const char* who, void* cache, long long capacity, CacheRef* c) {
  if (capacity <= 0 || capacity % kTile)
    return fail(BGTQ_ERR_CAPACITY, std::string(who) + ": capacity must be a positive multiple of 64");
  if (!cache) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null pointer");
  *c = CacheRef{static_cast<uint8_t*>(cache), nullptr, capacity / kTile, 0};
  return BGTQ_OK;
}

bgtq_status paged(const char* who, void* pool, long long num_pages, const int* block_table, long long max_pages,
                  CacheRef* c) {
  if (num_pages <= 0 || max_pages <= 0)
    return fail(BGTQ_ERR_CAPACITY, std::string(who) + ": num_pages and max_pages must be positive");
  if (!pool || !block_table) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null pointer");
  *c = CacheRef{static_cast<uint8_t*>(pool), block_table, max_pages, num_pages};
  return BGTQ_OK;
}

}  // namespace

extern "C" {

bgtq_status bgtq_encode_append(const bgtq_layout* L, const void* k, const void* v, int dtype, int batch,
                               int n_new, int h_kv, const int* seq_lens_dev, void* cache, long long capacity,
                               void* stream) {
  bgtq_status st = check_device(L, "encode_append");
  CacheRef c{};
  if (st == BGTQ_OK) st = contiguous("encode_append", cache, capacity, &c);
  if (st != BGTQ_OK) return st;
  return encode_impl(L->dev, "encode_append", k, v, dtype, batch, n_new, h_kv, seq_lens_dev, c, stream);
}

size_t bgtq_workspace_bytes(const bgtq_layout* L, int batch, int h_q, int h_kv, long long max_seq_len) {
  if (!L || batch <= 0 || h_kv <= 0 || h_q <= 0 || h_q % h_kv || h_q / h_kv > kMaxCols || max_seq_len < 0) {
    set_error("workspace_bytes: bad arguments");
    return 0;
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    set_error("workspace_bytes: no CUDA device");
    return 0;
  }
  return plan_decode(batch, h_q, h_kv, max_seq_len, sms).workspace_bytes;
}

bgtq_status bgtq_decode_attention(const bgtq_layout* L, const void* q, int q_dtype, int batch, int h_q, int h_kv,
                                  const void* cache, const int* seq_lens_dev, long long capacity,
                                  long long max_seq_len, float softmax_scale, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  bgtq_status st = check_device(L, "decode_attention");
  CacheRef c{};
  if (st == BGTQ_OK) st = contiguous("decode_attention", const_cast<void*>(cache), capacity, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(L->dev, "decode_attention", q, q_dtype, batch, h_q, h_kv, 1, c, seq_lens_dev, max_seq_len,
                     softmax_scale, out, workspace, workspace_bytes, stream);
}

bgtq_status bgtq_decode_attention_partial(const bgtq_layout* L, const void* q, int q_dtype, int batch, int h_q,
                                          int h_kv, const void* cache, const int* seq_lens_dev, long long capacity,
                                          long long max_seq_len, float softmax_scale, float* partial, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  bgtq_status st = check_device(L, "decode_attention_partial");
  CacheRef c{};
  if (st == BGTQ_OK) st = contiguous("decode_attention_partial", const_cast<void*>(cache), capacity, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(L->dev, "decode_attention_partial", q, q_dtype, batch, h_q, h_kv, 1, c, seq_lens_dev, max_seq_len,
                     softmax_scale, partial, workspace, workspace_bytes, stream, partial);
}

bgtq_status bgtq_merge_partials(const bgtq_layout* L, const float* partials, int n_parts, int batch, int h_q,
                                float* out, void* stream) {
  bgtq_status st = check_device(L, "merge_partials");
  if (st != BGTQ_OK) return st;
  if (n_parts < 1 || batch <= 0 || h_q <= 0 || (long long)batch * h_q > 0x7fffffffLL)
    return fail(BGTQ_ERR_INVALID, "merge_partials: bad n_parts / batch / h_q");
  if (!partials || !out) return fail(BGTQ_ERR_INVALID, "merge_partials: null pointer");
  cudaError_t e = launch_merge_records(L->dev, partials, n_parts, (long long)batch * h_q, out,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge_partials");
  return BGTQ_OK;
}

bgtq_status bgtq_decode_step(const bgtq_layout* L, const void* k_new, const void* v_new, int kv_dtype, int n_new,
                             const void* q, int q_dtype, int batch, int h_q, int h_kv, void* cache,
                             const int* seq_lens_dev, long long capacity, long long max_seq_len,
                             float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                             void* stream) {
  bgtq_status st = check_device(L, "decode_step");
  CacheRef c{};
  if (st == BGTQ_OK) st = contiguous("decode_step", cache, capacity, &c);
  if (st != BGTQ_OK) return st;
  return step_impl(L->dev, "decode_step", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, h_kv, 1, c, seq_lens_dev,
                   max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream);
}

long long bgtq_paged_pool_bytes(const bgtq_layout* L, int h_kv, long long num_pages) {
  if (!L || h_kv <= 0 || num_pages < 0) {
    set_error("paged_pool_bytes: bad arguments");
    return -1;
  }
  return num_pages * h_kv * (long long)L->tile_bytes;
}

bgtq_status bgtq_encode_append_paged(const bgtq_layout* L, const void* k, const void* v, int dtype, int batch,
                                     int n_new, int h_kv, const int* seq_lens_dev, void* pool, long long num_pages,
                                     const int* block_table_dev, long long max_pages, void* stream) {
  bgtq_status st = check_device(L, "encode_append_paged");
  CacheRef c{};
  if (st == BGTQ_OK) st = paged("encode_append_paged", pool, num_pages, block_table_dev, max_pages, &c);
  if (st != BGTQ_OK) return st;
  return encode_impl(L->dev, "encode_append_paged", k, v, dtype, batch, n_new, h_kv, seq_lens_dev, c, stream);
}

bgtq_status bgtq_decode_attention_paged(const bgtq_layout* L, const void* q, int q_dtype, int batch, int h_q,
                                        int h_kv, const void* pool, long long num_pages, const int* block_table_dev,
                                        long long max_pages, const int* seq_lens_dev, long long max_seq_len,
                                        float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  bgtq_status st = check_device(L, "decode_attention_paged");
  CacheRef c{};
  if (st == BGTQ_OK) st = paged("decode_attention_paged", const_cast<void*>(pool), num_pages, block_table_dev,
                                max_pages, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(L->dev, "decode_attention_paged", q, q_dtype, batch, h_q, h_kv, 1, c, seq_lens_dev, max_seq_len,
                     softmax_scale, out, workspace, workspace_bytes, stream);
}

bgtq_status bgtq_decode_step_paged(const bgtq_layout* L, const void* k_new, const void* v_new, int kv_dtype,
                                   int n_new, const void* q, int q_dtype, int batch, int h_q, int h_kv, void* pool,
                                   long long num_pages, const int* block_table_dev, long long max_pages,
                                   const int* seq_lens_dev, long long max_seq_len, float softmax_scale, float* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  bgtq_status st = check_device(L, "decode_step_paged");
  CacheRef c{};
  if (st == BGTQ_OK) st = paged("decode_step_paged", pool, num_pages, block_table_dev, max_pages, &c);
  if (st != BGTQ_OK) return st;
  return step_impl(L->dev, "decode_step_paged", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, h_kv, 1, c,
                   seq_lens_dev, max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream);
}

bgtq_status bgtq_decode_attention_multi(const bgtq_layout* L, const void* q, int q_dtype, int batch, int n_q,
                                        int h_q, int h_kv, const void* cache, const int* seq_lens_dev,
                                        long long capacity, long long max_seq_len, float softmax_scale, float* out,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  bgtq_status st = check_device(L, "decode_attention_multi");
  CacheRef c{};
  if (st == BGTQ_OK) st = contiguous("decode_attention_multi", const_cast<void*>(cache), capacity, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(L->dev, "decode_attention_multi", q, q_dtype, batch, h_q, h_kv, n_q, c, seq_lens_dev, max_seq_len,
                     softmax_scale, out, workspace, workspace_bytes, stream);
}

bgtq_status bgtq_decode_step_multi(const bgtq_layout* L, const void* k_new, const void* v_new, int kv_dtype,
                                   int n_new, const void* q, int q_dtype, int batch, int h_q, int h_kv, void* cache,
                                   const int* seq_lens_dev, long long capacity, long long max_seq_len,
                                   float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  bgtq_status st = check_device(L, "decode_step_multi");
  CacheRef c{};
  if (st == BGTQ_OK) st = contiguous("decode_step_multi", cache, capacity, &c);
  if (st != BGTQ_OK) return st;
  if (n_new < 1) return fail(BGTQ_ERR_INVALID, "decode_step_multi: n_new must be >= 1");
  return step_impl(L->dev, "decode_step_multi", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, h_kv, n_new, c,
                   seq_lens_dev, max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream);
}

bgtq_status bgtq_decode_step_multi_paged(const bgtq_layout* L, const void* k_new, const void* v_new, int kv_dtype,
                                         int n_new, const void* q, int q_dtype, int batch, int h_q, int h_kv,
                                         void* pool, long long num_pages, const int* block_table_dev,
                                         long long max_pages, const int* seq_lens_dev, long long max_seq_len,
                                         float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  bgtq_status st = check_device(L, "decode_step_multi_paged");
  CacheRef c{};
  if (st == BGTQ_OK) st = paged("decode_step_multi_paged", pool, num_pages, block_table_dev, max_pages, &c);
  if (st != BGTQ_OK) return st;
  if (n_new < 1) return fail(BGTQ_ERR_INVALID, "decode_step_multi_paged: n_new must be >= 1");
  return step_impl(L->dev, "decode_step_multi_paged", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, h_kv, n_new,
                   c, seq_lens_dev, max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {
bgtq_status scores_impl(const DevLayout& D, const char* who, const void* q, int q_dtype, int batch, int h_q,
                        int h_kv, const void* cache, const int* seq_lens_dev, long long capacity,
                        long long max_seq_len, float softmax_scale, float* scores, long long scores_ld,
                        void* workspace, size_t workspace_bytes, void* stream, const DevLayout* heads = nullptr) {
  const std::string w(who);
  if (!valid_dtype(q_dtype)) return fail(BGTQ_ERR_INVALID, w + ": bad dtype");
  if (batch <= 0 || h_kv <= 0 || h_q <= 0 || h_q % h_kv || h_q / h_kv > kMaxCols)
    return fail(BGTQ_ERR_INVALID, w + ": need h_q = G * h_kv with G in 1..32");
  if ((long long)batch * h_kv * ((h_q / h_kv + kMaxG - 1) / kMaxG) > 65535)
    return fail(BGTQ_ERR_INVALID, w + ": too many units (batch * h_kv * column tiles > 65535)");
  if (capacity <= 0 || capacity % kTile)
    return fail(BGTQ_ERR_CAPACITY, w + ": capacity must be a positive multiple of 64");
  if (max_seq_len < 0 || max_seq_len > capacity)
    return fail(BGTQ_ERR_CAPACITY, w + ": max_seq_len must be in [0, capacity]");
  if (scores_ld < max_seq_len) return fail(BGTQ_ERR_INVALID, w + ": scores_ld < max_seq_len");
  if (!std::isfinite(softmax_scale)) return fail(BGTQ_ERR_INVALID, w + ": bad softmax_scale");
  if (!q || !cache || !seq_lens_dev || !scores) return fail(BGTQ_ERR_INVALID, w + ": null pointer");
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, who);
  const DecodePlan plan = plan_decode(batch, h_q, h_kv, max_seq_len, sms);
  if (!workspace || workspace_bytes < plan.workspace_bytes)
    return fail(BGTQ_ERR_WORKSPACE, w + ": workspace missing or smaller than bgtq_workspace_bytes()");
  const CacheRef c{static_cast<uint8_t*>(const_cast<void*>(cache)), nullptr, capacity / kTile, 0};
  e = launch_scores(D, plan, q, q_dtype, batch, h_q, h_kv, c, seq_lens_dev, softmax_scale, scores, scores_ld,
                    workspace, static_cast<cudaStream_t>(stream), heads);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return BGTQ_OK;
}
}  // namespace

extern "C" {

bgtq_status bgtq_decode_scores(const bgtq_layout* L, const void* q, int q_dtype, int batch, int h_q, int h_kv,
                               const void* cache, const int* seq_lens_dev, long long capacity, long long max_seq_len,
                               float softmax_scale, float* scores, long long scores_ld, void* workspace,
                               size_t workspace_bytes, void* stream) {
  bgtq_status st = check_device(L, "decode_scores");
  if (st != BGTQ_OK) return st;
  return scores_impl(L->dev, "decode_scores", q, q_dtype, batch, h_q, h_kv, cache, seq_lens_dev, capacity,
                     max_seq_len, softmax_scale, scores, scores_ld, workspace, workspace_bytes, stream);
}

bgtq_status bgtq_device_status(const bgtq_layout* L, unsigned* flags, int clear) {
  bgtq_status st = check_device(L, "device_status");
  if (st != BGTQ_OK) return st;
  if (!flags) return fail(BGTQ_ERR_INVALID, "device_status: null pointer");
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(flags, L->dev.status, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(L->dev.status, 0, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_fail(e, "device_status");
  return BGTQ_OK;
}

// ------------------------------------------------------------------ one layout per KV head
namespace {
bgtq_status check_set(const bgtq_layout_set* S, const char* who) {
  if (!S) return fail(BGTQ_ERR_INVALID, std::string(who) + ": null layout set");
  int cur = -1;
  cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, who);
  if (cur != S->device) return fail(BGTQ_ERR_DEVICE, std::string(who) + ": layout set lives on another device");
  return BGTQ_OK;
}
}  // namespace

bgtq_status bgtq_layout_set_create(const bgtq_layout* const* layouts, int n, bgtq_layout_set** out) {
  if (!out) return fail(BGTQ_ERR_INVALID, "layout_set_create: null output");
  *out = nullptr;
  if (!layouts || n < 1 || n > 65535) return fail(BGTQ_ERR_INVALID, "layout_set_create: need 1..65535 layouts");
  for (int h = 0; h < n; ++h) {
    bgtq_status st = check_device(layouts[h], "layout_set_create");
    if (st != BGTQ_OK) return st;
    const bgtq_layout* a = layouts[0];
    const bgtq_layout* b = layouts[h];
    if (b->v_rate != a->v_rate || b->flags != a->flags || b->seed != a->seed)
      return fail(BGTQ_ERR_INVALID, "layout_set_create: layouts differ in value rate, options or seed");
  }
  auto* S = new (std::nothrow) bgtq_layout_set;
  if (!S) return fail(BGTQ_ERR_NOMEM, "layout_set_create: out of host memory");
  S->n = n;
  S->device = layouts[0]->device;
  for (int h = 0; h < n; ++h) S->tile_stride = std::max(S->tile_stride, layouts[h]->tile_bytes);
  const size_t bytes = 256 + sizeof(DevLayout) * size_t(n);
  cudaError_t e = cudaMalloc(&S->dev_block, bytes);
  if (e != cudaSuccess) {
    delete S;
    return cuda_fail(e, "layout_set_create");
  }
  unsigned* status = static_cast<unsigned*>(S->dev_block);
  S->heads = reinterpret_cast<DevLayout*>(static_cast<char*>(S->dev_block) + 256);
  std::vector<DevLayout> host(static_cast<size_t>(n) + 0);
  for (int h = 0; h < n; ++h) {
    host[h] = layouts[h]->dev;     // device pointers of the layout's own tables stay valid
    host[h].tile_bytes = S->tile_stride;
    host[h].status = status;
  }
  S->head0 = host[0];
  e = cudaMemset(status, 0, sizeof(unsigned));
  if (e == cudaSuccess) e = cudaMemcpy(S->heads, host.data(), sizeof(DevLayout) * size_t(n), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(S->dev_block);
    delete S;
    return cuda_fail(e, "layout_set_create");
  }
  *out = S;
  return BGTQ_OK;
}

void bgtq_layout_set_destroy(bgtq_layout_set* S) {
  if (!S) return;
  if (S->dev_block) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != S->device) cudaSetDevice(S->device);
    cudaFree(S->dev_block);
    if (cur >= 0 && cur != S->device) cudaSetDevice(cur);
  }
  delete S;
}

int bgtq_layout_set_tile_bytes(const bgtq_layout_set* S) { return S ? S->tile_stride : 0; }

size_t bgtq_layout_set_cache_bytes(const bgtq_layout_set* S, int batch, long long capacity) {
  if (!S || batch <= 0 || capacity <= 0 || capacity % kTile) {
    set_error("layout_set_cache_bytes: bad arguments");
    return 0;
  }
  return size_t(batch) * size_t(S->n) * size_t(capacity / kTile) * size_t(S->tile_stride);
}

bgtq_status bgtq_encode_append_heads(const bgtq_layout_set* S, const void* k, const void* v, int dtype, int batch,
                                     int n_new, const int* seq_lens_dev, void* cache, long long capacity,
                                     void* stream) {
  CacheRef c;
  bgtq_status st = check_set(S, "encode_append_heads");
  if (st == BGTQ_OK) st = contiguous("encode_append_heads", cache, capacity, &c);
  if (st != BGTQ_OK) return st;
  return encode_impl(S->head0, "encode_append_heads", k, v, dtype, batch, n_new, S->n, seq_lens_dev, c, stream,
                     S->heads);
}

bgtq_status bgtq_decode_attention_heads(const bgtq_layout_set* S, const void* q, int q_dtype, int batch, int h_q,
                                        const void* cache, const int* seq_lens_dev, long long capacity,
                                        long long max_seq_len, float softmax_scale, float* out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  CacheRef c;
  bgtq_status st = check_set(S, "decode_attention_heads");
  if (st == BGTQ_OK) st = contiguous("decode_attention_heads", const_cast<void*>(cache), capacity, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(S->head0, "decode_attention_heads", q, q_dtype, batch, h_q, S->n, 1, c, seq_lens_dev,
                     max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream, nullptr, S->heads);
}

bgtq_status bgtq_decode_attention_multi_heads(const bgtq_layout_set* S, const void* q, int q_dtype, int batch,
                                              int n_q, int h_q, const void* cache, const int* seq_lens_dev,
                                              long long capacity, long long max_seq_len, float softmax_scale,
                                              float* out, void* workspace, size_t workspace_bytes, void* stream) {
  CacheRef c;
  bgtq_status st = check_set(S, "decode_attention_multi_heads");
  if (st == BGTQ_OK) st = contiguous("decode_attention_multi_heads", const_cast<void*>(cache), capacity, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(S->head0, "decode_attention_multi_heads", q, q_dtype, batch, h_q, S->n, n_q, c, seq_lens_dev,
                     max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream, nullptr, S->heads);
}

bgtq_status bgtq_decode_scores_heads(const bgtq_layout_set* S, const void* q, int q_dtype, int batch, int h_q,
                                     const void* cache, const int* seq_lens_dev, long long capacity,
                                     long long max_seq_len, float softmax_scale, float* scores, long long scores_ld,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  bgtq_status st = check_set(S, "decode_scores_heads");
  if (st != BGTQ_OK) return st;
  return scores_impl(S->head0, "decode_scores_heads", q, q_dtype, batch, h_q, S->n, cache, seq_lens_dev, capacity,
                     max_seq_len, softmax_scale, scores, scores_ld, workspace, workspace_bytes, stream, S->heads);
}

bgtq_status bgtq_decode_step_heads(const bgtq_layout_set* S, const void* k_new, const void* v_new, int kv_dtype,
                                   int n_new, const void* q, int q_dtype, int batch, int h_q, void* cache,
                                   const int* seq_lens_dev, long long capacity, long long max_seq_len,
                                   float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  CacheRef c;
  bgtq_status st = check_set(S, "decode_step_heads");
  if (st == BGTQ_OK) st = contiguous("decode_step_heads", cache, capacity, &c);
  if (st != BGTQ_OK) return st;
  return step_impl(S->head0, "decode_step_heads", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, S->n, 1, c,
                   seq_lens_dev, max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream, S->heads);
}

bgtq_status bgtq_decode_step_multi_heads(const bgtq_layout_set* S, const void* k_new, const void* v_new,
                                         int kv_dtype, int n_new, const void* q, int q_dtype, int batch, int h_q,
                                         void* cache, const int* seq_lens_dev, long long capacity,
                                         long long max_seq_len, float softmax_scale, float* out, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  CacheRef c;
  bgtq_status st = check_set(S, "decode_step_multi_heads");
  if (st == BGTQ_OK) st = contiguous("decode_step_multi_heads", cache, capacity, &c);
  if (st != BGTQ_OK) return st;
  if (n_new < 1) return fail(BGTQ_ERR_INVALID, "decode_step_multi_heads: n_new must be >= 1");
  return step_impl(S->head0, "decode_step_multi_heads", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, S->n,
                   n_new, c, seq_lens_dev, max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream,
                   S->heads);
}

long long bgtq_layout_set_paged_pool_bytes(const bgtq_layout_set* S, long long num_pages) {
  if (!S || num_pages < 0) {
    set_error("layout_set_paged_pool_bytes: bad arguments");
    return -1;
  }
  return num_pages * S->n * (long long)S->tile_stride;
}

bgtq_status bgtq_encode_append_paged_heads(const bgtq_layout_set* S, const void* k, const void* v, int dtype,
                                           int batch, int n_new, const int* seq_lens_dev, void* pool,
                                           long long num_pages, const int* block_table_dev, long long max_pages,
                                           void* stream) {
  CacheRef c{};
  bgtq_status st = check_set(S, "encode_append_paged_heads");
  if (st == BGTQ_OK) st = paged("encode_append_paged_heads", pool, num_pages, block_table_dev, max_pages, &c);
  if (st != BGTQ_OK) return st;
  return encode_impl(S->head0, "encode_append_paged_heads", k, v, dtype, batch, n_new, S->n, seq_lens_dev, c, stream,
                     S->heads);
}

bgtq_status bgtq_decode_attention_paged_heads(const bgtq_layout_set* S, const void* q, int q_dtype, int batch,
                                              int h_q, const void* pool, long long num_pages,
                                              const int* block_table_dev, long long max_pages,
                                              const int* seq_lens_dev, long long max_seq_len, float softmax_scale,
                                              float* out, void* workspace, size_t workspace_bytes, void* stream) {
  CacheRef c{};
  bgtq_status st = check_set(S, "decode_attention_paged_heads");
  if (st == BGTQ_OK)
    st = paged("decode_attention_paged_heads", const_cast<void*>(pool), num_pages, block_table_dev, max_pages, &c);
  if (st != BGTQ_OK) return st;
  return decode_impl(S->head0, "decode_attention_paged_heads", q, q_dtype, batch, h_q, S->n, 1, c, seq_lens_dev,
                     max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream, nullptr, S->heads);
}

bgtq_status bgtq_decode_step_paged_heads(const bgtq_layout_set* S, const void* k_new, const void* v_new,
                                         int kv_dtype, int n_new, const void* q, int q_dtype, int batch, int h_q,
                                         void* pool, long long num_pages, const int* block_table_dev,
                                         long long max_pages, const int* seq_lens_dev, long long max_seq_len,
                                         float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  CacheRef c{};
  bgtq_status st = check_set(S, "decode_step_paged_heads");
  if (st == BGTQ_OK) st = paged("decode_step_paged_heads", pool, num_pages, block_table_dev, max_pages, &c);
  if (st != BGTQ_OK) return st;
  return step_impl(S->head0, "decode_step_paged_heads", k_new, v_new, kv_dtype, n_new, q, q_dtype, batch, h_q, S->n,
                   1, c, seq_lens_dev, max_seq_len, softmax_scale, out, workspace, workspace_bytes, stream, S->heads);
}

bgtq_status bgtq_layout_set_status(const bgtq_layout_set* S, unsigned* flags, int clear) {
  bgtq_status st = check_set(S, "layout_set_status");
  if (st != BGTQ_OK) return st;
  if (!flags) return fail(BGTQ_ERR_INVALID, "layout_set_status: null pointer");
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(flags, S->dev_block, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(S->dev_block, 0, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_fail(e, "layout_set_status");
  return BGTQ_OK;
}

}  // extern "C"
