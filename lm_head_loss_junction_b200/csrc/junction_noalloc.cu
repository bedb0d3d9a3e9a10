// mls_junction_bwd_noalloc: the junction backward pass for callers that cannot
// hand the library a device buffer.
//
// mls_junction_bwd needs scratch space for the residual-table gradient (the
// id grouping of the tokens).  Its ordinary form takes that space from the
// caller.  Some callers cannot allocate device memory where they call it:
// programs whose device memory is handed out up front by another allocator
// (a framework's caching allocator or a fixed pool that owns the whole
// device), and latency-critical paths that must not call cudaMalloc or
// cudaFree, which can synchronise the whole device.  This entry point serves
// them from one fixed array in the library's own device memory.
//
// The array is a file-scope __device__ object of kNoallocScratchBytes bytes;
// every GPU that loads the library holds one copy of it until the process
// exits.  In host code the array's name is only a host-side stand-in, not a
// device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and keeps it together with
// the identity of the device's CUDA context.  If that context is destroyed
// and created again (cudaDeviceReset), the next call sees a new context and
// looks the address up again instead of using a stale one.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "mls.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;   // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct ScratchSlot {
  unsigned long long ctx_id;   // context the address belongs to (0: unknown)
  void* addr;
};

std::mutex g_noalloc_mu;
ScratchSlot g_noalloc_slot[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context (never reused within a process), or
// 0 when there is no current context or the driver does not provide one.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device: looked up once
// per device and context, and again whenever the context is not the one the
// cached address belongs to (or its identity cannot be read).
cudaError_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchSlot& slot = g_noalloc_slot[dev];
  if (slot.addr == nullptr || ctx == 0 || slot.ctx_id != ctx) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    slot.addr = p;
    slot.ctx_id = current_context_id();   // the lookup makes the device's context current
  }
  *out = slot.addr;
  return cudaSuccess;
}

}  // namespace

extern "C" {

mls_status mls_junction_bwd_noalloc(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                    int64_t V, int64_t delta, const void* dy, void* do_m, void* de_rows,
                                    float* dE_table, int accumulate_dE, mls_dtype dt, int32_t* dev_status,
                                    void* stream) {
  // the checks of mls_junction_bwd come first, so errors are reported as that call reports them
  mls_status st = mls::check_junction_bwd_args(x, T, o_m, D_m, e_next, V, delta, dy, do_m, de_rows, dE_table,
                                               MLS_JUNCTION_STANDARD, dt);
  if (st != MLS_OK) return st;
  if (dE_table == nullptr) {
    // no table gradient requested: no scratch is used at all
    return mls_junction_bwd(x, T, o_m, D_m, e_next, V, delta, dy, do_m, de_rows, nullptr, accumulate_dE, nullptr,
                            0, dt, dev_status, stream);
  }
  size_t need = 0;
  st = mls_junction_bwd_workspace(T, V, &need);
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
