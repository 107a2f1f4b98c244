// spa_attention_noalloc: spa_attention for callers that cannot allocate.
//
// spa_attention needs a caller-provided workspace whenever it splits the
// key range (partial softmax states plus per-unit tickets).  Some callers
// cannot obtain one: code that runs while a CUDA graph is being captured in
// relaxed/global capture mode (where cudaMalloc is not permitted), plugins
// hosted by a runtime that owns every device allocation and exposes no
// allocator to them, and tools that must not change the process's
// device-memory footprint after start-up.  This entry point serves them from
// a fixed scratch array that lives in the library itself.
//
// The scratch is a file-scope __device__ array of SPA_NOALLOC_SCRATCH_BYTES;
// every GPU that loads the library holds it until the process exits.  Host
// code never uses the array's name as a device address: the first call on
// each device, with that device current, resolves the address with
// cudaGetSymbolAddress (so that first call should come before any stream
// capture; every later call outside a capture resolves it again), and every
// call passes that pointer to the kernel.  All calls on a
// device share the array and find the previous call's contents in it: the
// tickets that must start at zero are cleared on the stream before each
// launch, and calls that overlap on the GPU (other streams, other threads)
// race on the array.
#include <mutex>

#include "spa_attn.cuh"
#include "spa_plan.h"

namespace spa {
int run_attention(const spa_attention_args_t* a, const Plan& pl, void* ws, cudaStream_t stream);
}

using namespace spa;

static __device__ __align__(256) unsigned char g_noalloc_scratch[SPA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// Device address of the scratch array on the current device.  It is resolved
// with that device current on the first call, and again on every call made
// while `stream` is not being captured, so that a call after a context reset
// (cudaDeviceReset reloads the module, and the array may move) uses the new
// address.  A call made during a capture uses the address the last uncaptured
// call on this device resolved.
int scratch_address(cudaStream_t stream, void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SPA_ERR_CUDA;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    cudaGetLastError();
    cs = cudaStreamCaptureStatusActive;  // unknown: do not resolve during a possible capture
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SPA_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return SPA_OK;
}

}  // namespace

extern "C" int spa_attention_noalloc(const spa_attention_args_t* a, spa_stream_t stream) {
  int rc = validate_attention(a);
  if (rc != SPA_OK) return rc;
  if (a->T == 0 || a->B == 0) return SPA_OK;
  Plan pl;
  if ((rc = make_plan(a, &pl)) != SPA_OK) return rc;
  const size_t need = pl.ws_acc_bytes + pl.ws_ml_bytes + pl.ws_count_bytes;
  if (need > SPA_NOALLOC_SCRATCH_BYTES) return SPA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if ((rc = scratch_address((cudaStream_t)stream, &scratch)) != SPA_OK) return rc;
  if (pl.ws_count_bytes > 0) {
    // split tickets start at zero; the bytes may hold an earlier call's partials
    unsigned char* tickets = static_cast<unsigned char*>(scratch) + pl.ws_acc_bytes + pl.ws_ml_bytes;
    if (cudaMemsetAsync(tickets, 0, pl.ws_count_bytes, (cudaStream_t)stream) != cudaSuccess) {
      cudaGetLastError();
      return SPA_ERR_CUDA;
    }
  }
  return run_attention(a, pl, need > 0 ? scratch : nullptr, (cudaStream_t)stream);
}
