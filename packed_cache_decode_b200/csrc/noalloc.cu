// bgtq_decode_attention_noalloc: decode attention for callers that cannot allocate.
//
// Some callers are not allowed to call cudaMalloc at all: an inference server that hands
// every byte of device memory to its own pool at start-up, a plugin whose host framework
// forbids allocation inside its enqueue/execute callback, or code whose memory budget
// is fixed and audited. bgtq_decode_attention needs a caller-provided workspace for its
// split-K partials; this variant instead keeps that scratch in one file-scope device
// array of fixed size, so the caller passes only inputs and outputs.
//
// The array lives in every GPU that loads the library until the process exits. Its
// device address is looked up once per device (cudaGetSymbolAddress, with that device
// current) on the first call that runs on it; make that first call before any stream
// capture. All calls share the array: two calls whose kernels overlap on the GPU (for
// example on two streams) race on it and give wrong results. The split kernel writes
// every partial it later reads, so nothing in the array has to start at zero.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "bgtq_internal.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = BGTQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on `device` (which is current). The host-side symbol is
// only a stand-in; the address has to be asked from the runtime once per device.
bgtq_status scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices)
    return bgtq::fail(BGTQ_ERR_DEVICE, "decode_attention_noalloc: device index out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p)
      return bgtq::fail(BGTQ_ERR_CUDA, std::string("decode_attention_noalloc: cudaGetSymbolAddress: ") +
                                           cudaGetErrorString(e));
    g_scratch_addr[device] = p;
  }
  *out = g_scratch_addr[device];
  return BGTQ_OK;
}

}  // namespace

extern "C" {

size_t bgtq_noalloc_scratch_capacity(void) { return kScratchBytes; }

bgtq_status bgtq_decode_attention_noalloc(const bgtq_layout* L, const void* q, int q_dtype, int batch, int h_q,
                                          int h_kv, const void* cache, const int* seq_lens_dev, long long capacity,
                                          long long max_seq_len, float softmax_scale, float* out, void* stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess)
    return bgtq::fail(BGTQ_ERR_CUDA, std::string("decode_attention_noalloc: ") + cudaGetErrorString(e));
  if (!L || batch <= 0 || h_kv <= 0 || h_q <= 0 || h_q % h_kv || h_q / h_kv > bgtq::kMaxCols || max_seq_len < 0)
    return bgtq::fail(BGTQ_ERR_INVALID, "decode_attention_noalloc: bad layout or shape");
  const bgtq::DecodePlan plan = bgtq::plan_decode(batch, h_q, h_kv, max_seq_len, sms);
  if (plan.workspace_bytes > kScratchBytes)
    return bgtq::fail(BGTQ_ERR_WORKSPACE,
                      "decode_attention_noalloc: this shape needs " + std::to_string(plan.workspace_bytes) +
                          " bytes of scratch, more than the fixed " + std::to_string(kScratchBytes) +
                          "; use bgtq_decode_attention with a workspace");
  void* scratch = nullptr;
  bgtq_status st = scratch_address(dev, &scratch);
  if (st != BGTQ_OK) return st;
  // Same argument checks and kernels as bgtq_decode_attention, with the static scratch
  // standing in for the caller's workspace.
  return bgtq_decode_attention(L, q, q_dtype, batch, h_q, h_kv, cache, seq_lens_dev, capacity, max_seq_len,
                               softmax_scale, out, scratch, kScratchBytes, stream);
}

}  // extern "C"
