// mls_junction_bwd_noalloc: the junction backward pass for callers that cannot
// hand the library a device buffer.
//
// mls_junction_bwd needs scratch space for the residual-table gradient (the
// id grouping of the tokens).  Its ordinary form takes that space from the
// caller.  Some callers cannot produce it at the point of the call: code that
// runs while a stream is being captured into a CUDA graph (cudaMalloc is not
// a stream operation and cannot be captured), code that must never block on
// the device (cudaMalloc and cudaFree may synchronise), and programs whose
// device memory is handed out up front by another allocator.  This entry point
// serves them from one fixed array in the library's own device memory.
//
// The array is a file-scope __device__ object of kNoallocScratchBytes bytes;
// every GPU that loads the library holds one copy of it until the process
// exits.  Host code cannot use the array's name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress
// (with that device current) and caches it; that first call should therefore
// happen before any stream capture begins.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "mls.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;   // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

mls_status mls_junction_bwd_noalloc(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                    int64_t V, int64_t delta, const void* dy, void* do_m, void* de_rows,
                                    float* dE_table, int accumulate_dE, mls_dtype dt, int32_t* dev_status,
                                    void* stream) {
  if (dE_table == nullptr) {
    // no table gradient requested: no scratch is used at all
    return mls_junction_bwd(x, T, o_m, D_m, e_next, V, delta, dy, do_m, de_rows, nullptr, accumulate_dE, nullptr,
                            0, dt, dev_status, stream);
  }
  size_t need = 0;
  mls_status st = mls_junction_bwd_workspace(T, V, &need);
  if (st != MLS_OK) return st;
  if (need > kNoallocScratchBytes) return MLS_ERR_UNSUPPORTED;   // (T, V) too large for the fixed array
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return MLS_ERR_CUDA;
  }
  return mls_junction_bwd(x, T, o_m, D_m, e_next, V, delta, dy, do_m, de_rows, dE_table, accumulate_dE, scratch,
                          kNoallocScratchBytes, dt, dev_status, stream);
}

}  // extern "C"
