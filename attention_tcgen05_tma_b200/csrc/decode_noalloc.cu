// Allocation-free variant of the decode full-layer entry point.
//
// Some callers cannot allocate device memory at the moment they run a decode step:
// a serving loop that plans all of its device memory up front and forbids later
// cudaMalloc calls (cudaMalloc may synchronise the device and fragments a pre-sized
// pool), or a host integration that owns no allocator at all.  This entry point gives
// them the decode full layer with its split-KV scratch taken from a fixed array that
// the library itself holds in device memory, so the caller passes only inputs and
// outputs.  It calls no cudaMalloc, cudaFree or other allocating routine.
//
// The array has a fixed capacity (kNoAllocScratchBytes).  Every GPU that loads the
// library holds it until the process exits.  Its device address is resolved once per
// device, on the first call made with that device current; under the driver's lazy module
// loading that first call is also when the driver loads this file's module and places the
// array on the device, so the first call may allocate and synchronise and belongs in the
// caller's set-up (before any stream capture).  Later calls allocate nothing.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device (nullptr on failure).  In host
// code the symbol itself is only a host-side stand-in, never a device address.
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" HYS_API hys_status hysparse_full_attn_select_decode_noalloc(const hys_decode_shape* shape,
                                                                       hys_dtype dtype, const void* q,
                                                                       const void* k_cache, const void* v_cache,
                                                                       const int* seqlens, void* o, float* scores,
                                                                       hys_reduce red, hys_stream_t stream) {
  void* ws = scratch_address();
  if (ws == nullptr) return HYS_ERR_CUDA;
  // Shapes whose split-KV scratch exceeds the fixed capacity come back as HYS_ERR_WORKSPACE
  // from the regular entry point's own check; nothing is launched in that case.  Every
  // scratch entry the kernels read is written earlier in the same call, so nothing needs
  // clearing between calls.
  return hysparse_full_attn_select_decode(shape, dtype, q, k_cache, v_cache, seqlens, o, scores, red, ws,
                                          kNoAllocScratchBytes, stream);
}
