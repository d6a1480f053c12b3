// sdpa_forward_noalloc: the forward pass for callers that cannot allocate
// device memory.
//
// When the router splits the keys, the attention pass writes fp32 partial
// outputs and log-sum-exp values to scratch memory that the combine kernel
// then reads.  sdpa_forward takes that scratch from the stream-ordered pool
// and sdpa_forward_ws takes it from the caller.  Some callers can do neither:
// code that must not call cudaMalloc/cudaMallocAsync at all (for instance a
// runtime whose device memory is handed out by an allocator it cannot call
// into at this point, or a latency-critical loop where an allocation could
// synchronise the device or grow a pool mid-run).  This entry point serves
// them from a fixed scratch array that lives in the library's device image.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kNoAllocScratchBytes of device memory for it until the
// process exits.  Host code cannot use the variable's name as a device
// address; the address is looked up with cudaGetSymbolAddress on the first
// call made while a device is current (and again if that device's context
// has been replaced since).
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "launch.h"

namespace sdpa {

// Fixed maximum of the shared scratch: 16 MiB per device.
constexpr size_t kNoAllocScratchBytes = 16u << 20;

}  // namespace sdpa

static __device__ __align__(256) unsigned char g_sdpa_noalloc_scratch[sdpa::kNoAllocScratchBytes];

namespace sdpa {
namespace {

constexpr int kMaxDev = 64;
std::mutex g_mu;
void *g_scratch[kMaxDev];
unsigned long long g_scratch_ctx[kMaxDev];  // context the address belongs to

// Device address of the scratch array in the current device's context.  It is
// looked up once per context: on the first call made on a device, and again
// if that device's context was replaced since (after cudaDeviceReset, say, the
// old address would be stale).
sdpa_status scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return set_error(SDPA_ERR_CUDA, std::string("no usable CUDA device: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDev) return set_error(SDPA_ERR_CUDA, "device index too large");
  std::lock_guard<std::mutex> lk(g_mu);
  unsigned long long ctx = 0;
  if (g_scratch[dev] == nullptr || current_context_id(&ctx) != SDPA_OK ||
      ctx != g_scratch_ctx[dev]) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress((void **)&ptr, g_sdpa_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return set_error(SDPA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") +
                                          cudaGetErrorString(e));
    if (current_context_id(&ctx) != SDPA_OK) ctx = 0;
    g_scratch[dev] = ptr;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch[dev];
  return SDPA_OK;
}

}  // namespace
}  // namespace sdpa

using namespace sdpa;

extern "C" SDPA_API sdpa_status sdpa_forward_noalloc(const void *q, const void *k, const void *v,
                                                     void *out, int B, int Hq, int Hkv, int L,
                                                     int S, int Dqk, int Dv, float scale,
                                                     int causal, int window_size,
                                                     sdpa_dtype dtype, sdpa_stream_t stream) {
  set_error(SDPA_OK, "");
  Problem pb;
  pb.B = B; pb.Hq = Hq; pb.Hkv = Hkv; pb.L = L; pb.S = S; pb.Dqk = Dqk; pb.Dv = Dv;
  pb.scale = scale; pb.causal = causal; pb.window = window_size; pb.dtype = dtype;
  pb.q_offset = S - L;  // queries end at the last key
  pb.has_q_offset = 0;
  // host-side checks first, in the same order as sdpa_forward, before any
  // CUDA call
  sdpa_status st = validate_call(pb, q, k, v, out);
  if (st != SDPA_OK) return st;
  Plan pl;
  st = plan_call(pb, SDPA_PATH_AUTO, 0, &pl);
  if (st != SDPA_OK) return st;
  if (pl.ws_bytes > kNoAllocScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "sdpa_forward_noalloc: this problem needs %zu bytes of scratch, above the fixed "
             "maximum of %zu bytes; use sdpa_forward or sdpa_forward_ws",
             pl.ws_bytes, kNoAllocScratchBytes);
    return set_error(SDPA_ERR_RESOURCES, buf);
  }
  void *scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != SDPA_OK) return st;
  // Every element of the scratch the combine reads is written by the
  // attention pass of the same call (empty splits write O = 0, LSE = -inf),
  // so nothing needs clearing between calls.
  return forward_call(pb, q, k, v, out, SDPA_PATH_AUTO, 0, scratch, kNoAllocScratchBytes, false,
                      (cudaStream_t)stream);
}
