// tp_mlp_forward_noalloc: the MLP block with its scratch in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// For callers that cannot allocate device memory: a C or C++ host program
// that embeds libtp.so without PyTorch or any other device memory pool has no
// allocator to carve a workspace from, and a caller running inside a
// framework that has already reserved all device memory for its own pool
// cannot ask cudaMalloc for more (and must not call it on a latency-critical
// path, where it synchronizes the device). Such callers pass only inputs and
// outputs; the intermediates (the column-parallel activations and the N fp32
// partials) live in g_tp_noalloc_ws below.
//
// Properties a caller must know:
//   * The array is TP_NOALLOC_WS_BYTES (include/tp.h) per GPU. It belongs
//     to this file's CUDA module, and the runtime reserves it when it loads
//     the module on a GPU: under lazy module loading (the CUDA 12 default)
//     that is the first call here on that GPU, whose cudaGetSymbolAddress
//     triggers the load; under eager loading, context creation. It stays
//     reserved until the process exits.
//   * A problem whose scratch exceeds it is rejected with TP_ERR_WORKSPACE
//     before anything is launched.
//   * Every call on a device shares the same array and it keeps the last
//     call's contents. Nothing in it has to start at zero: each call writes
//     every scratch byte it later reads. Calls that overlap on the GPU (on
//     different streams, or from different host threads, without ordering
//     between them) race on the array and corrupt each other's results.
//   * The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make
//     that first call before any stream capture begins, and before a memory
//     pool of the caller's takes the free device memory (the lazy module
//     load needs room for the array; without it the call returns
//     TP_ERR_WORKSPACE). After cudaDeviceReset the cached address is stale.
//   * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/tp.h"

namespace {

// Host code must never use this name as a device address (on the host it is
// only a stand-in); the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_tp_noalloc_ws[TP_NOALLOC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};

}  // namespace

extern "C" tp_status tp_mlp_forward_noalloc(const uint16_t* X, int64_t B, int64_t h, int64_t ffn,
                                            int n_shards, const uint16_t* A_shards,
                                            const uint16_t* b1_shards, const uint16_t* B_shards,
                                            const uint16_t* b2, const uint16_t* residual,
                                            uint16_t* Y, void* stream) {
  const size_t need = tp_workspace_bytes(TP_WS_MLP, B, h, ffn, n_shards);
  if (need == 0) return TP_ERR_SHAPE;
  if (need > static_cast<size_t>(TP_NOALLOC_WS_BYTES)) return TP_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TP_ERR_UNSUPPORTED;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_ws_ptr[dev] == nullptr) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_tp_noalloc_ws);
      if (e == cudaErrorMemoryAllocation) {
        cudaGetLastError();  // not sticky: clear it and report the missing room
        return TP_ERR_WORKSPACE;
      }
      if (e != cudaSuccess || p == nullptr) return TP_ERR_CUDA;
      g_ws_ptr[dev] = p;
    }
    ws = g_ws_ptr[dev];
  }
  return tp_mlp_forward(X, B, h, ffn, n_shards, A_shards, b1_shards, B_shards, b2, residual, ws,
                        static_cast<size_t>(TP_NOALLOC_WS_BYTES), Y, stream);
}
