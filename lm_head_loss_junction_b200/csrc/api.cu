// C ABI of libmls: argument checking, workspace sizing and kernel launch on
// the caller's stream.  Every declaration, its meaning and its error behaviour
// is documented in include/mls.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <climits>
#include <cstdint>

#include "kernels.h"
#include "mls.h"

namespace mls {
namespace {
std::atomic<uint64_t> g_launches{0};
}
void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
}  // namespace mls

namespace {

using mls::LossProblem;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr uint32_t kKnownVariants = MLS_JUNCTION_NO_RESCALE | MLS_JUNCTION_ZERO_FILL | MLS_JUNCTION_STOP_GRAD;

// Returns MLS_OK when the current device is a compute-capability 10.0 GPU
// (the only target this library is built for).
mls_status device_ok() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MLS_ERR_NO_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return MLS_ERR_NO_DEVICE;
  }
  if (major != 10 || minor != 0) return MLS_ERR_NO_DEVICE;
  return MLS_OK;
}

mls_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MLS_OK : MLS_ERR_CUDA; }

mls_status check_junction_shape(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                int64_t V, int64_t delta, mls_dtype dt) {
  if (x == nullptr || o_m == nullptr || e_next == nullptr) return MLS_ERR_INVALID_ARG;
  if (T <= 0 || D_m <= 0 || V <= 0 || delta <= 0) return MLS_ERR_INVALID_ARG;
  if (dt != MLS_F32 && dt != MLS_BF16) return MLS_ERR_INVALID_ARG;
  const int64_t per_vec = dt == MLS_BF16 ? 8 : 4;
  if (D_m % per_vec != 0 || delta % per_vec != 0) return MLS_ERR_UNSUPPORTED;
  if ((D_m + delta) / per_vec > INT_MAX || V > INT_MAX || T > (int64_t(1) << 40)) return MLS_ERR_UNSUPPORTED;
  if (!aligned16(o_m) || !aligned16(e_next)) return MLS_ERR_UNSUPPORTED;
  return MLS_OK;
}

// Shape checks shared by every loss entry point (no pointers involved).
mls_status check_loss_shape(int M, int64_t T, int64_t V, const int64_t* D, mls_dtype dt) {
  if (M < 1 || M > mls::kMaxExits) return M < 1 ? MLS_ERR_INVALID_ARG : MLS_ERR_UNSUPPORTED;
  if (D == nullptr) return MLS_ERR_INVALID_ARG;
  if (T <= 0 || V <= 0) return MLS_ERR_INVALID_ARG;
  if (dt != MLS_F32 && dt != MLS_BF16) return MLS_ERR_INVALID_ARG;
  for (int m = 0; m < M; ++m) {
    if (D[m] <= 0) return MLS_ERR_INVALID_ARG;
    if (m > 0 && D[m] <= D[m - 1]) return MLS_ERR_INVALID_ARG;   // widths strictly increase
  }
  if (T > INT_MAX || V > INT_MAX) return MLS_ERR_UNSUPPORTED;
  if (dt == MLS_BF16) {
    if (V % 128 != 0) return MLS_ERR_UNSUPPORTED;
    for (int m = 0; m < M; ++m)
      if (D[m] % 64 != 0 || D[m] > 65536) return MLS_ERR_UNSUPPORTED;
    if (static_cast<double>(V) * static_cast<double>(T) >= 9.0e15) return MLS_ERR_UNSUPPORTED;
  }
  return MLS_OK;
}

// Shape-only problem description, for the workspace queries.
LossProblem shape_problem(int M, int64_t T, int64_t V, const int64_t* D) {
  LossProblem p{};
  p.M = M;
  p.T = T;
  p.V = V;
  for (int m = 0; m < M; ++m) p.D[m] = D[m];
  for (int m = 0; m < mls::kMaxExits; ++m) p.exit_w[m] = 1.f;
  return p;
}

mls_status build_problem(int M, int64_t T, int64_t V, const int64_t* D, const int32_t* y, const void* const* h,
                         const void* const* W, float alpha_d, mls_dtype dt, int32_t* status, LossProblem* p) {
  mls_status st = check_loss_shape(M, T, V, D, dt);
  if (st != MLS_OK) return st;
  if (h == nullptr || W == nullptr || y == nullptr) return MLS_ERR_INVALID_ARG;
  if (!(alpha_d == alpha_d)) return MLS_ERR_INVALID_ARG;   // NaN
  for (int m = 0; m < M; ++m) {
    if (h[m] == nullptr || W[m] == nullptr) return MLS_ERR_INVALID_ARG;
    if (!aligned16(h[m]) || !aligned16(W[m])) return MLS_ERR_UNSUPPORTED;
  }
  *p = shape_problem(M, T, V, D);
  for (int m = 0; m < M; ++m) {
    p->h[m] = h[m];
    p->W[m] = W[m];
  }
  p->y = y;
  p->alpha_d = alpha_d;
  p->status = status;
  return MLS_OK;
}

mls_status apply_options(const mls_loss_options* opts, LossProblem* p) {
  if (opts == nullptr) return MLS_OK;
  if (opts->distill != MLS_DISTILL_CE && opts->distill != MLS_DISTILL_REVERSE_KL && opts->distill != MLS_DISTILL_JS &&
      opts->distill != MLS_DISTILL_ACCEPT)
    return MLS_ERR_INVALID_ARG;
  p->distill = opts->distill;
  if (opts->teacher_grad != 0 && opts->teacher_grad != 1) return MLS_ERR_INVALID_ARG;
  p->teacher_grad = opts->teacher_grad;
  if (opts->exit_weights != nullptr) {
    for (int m = 0; m < p->M; ++m) {
      const float w = opts->exit_weights[m];
      if (!(w == w) || w == INFINITY || w == -INFINITY) return MLS_ERR_INVALID_ARG;
      p->exit_w[m] = w;
    }
  }
  return MLS_OK;
}

}  // namespace

namespace mls {

mls_status check_junction_bwd_args(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                   int64_t V, int64_t delta, const void* dy, const void* do_m, const void* de_rows,
                                   const float* dE_table, uint32_t variant, mls_dtype dt) {
  if (variant & ~kKnownVariants) return MLS_ERR_INVALID_ARG;
  mls_status st = check_junction_shape(x, T, o_m, D_m, e_next, V, delta, dt);
  if (st != MLS_OK) return st;
  if (dy == nullptr || do_m == nullptr) return MLS_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(do_m) || (de_rows != nullptr && !aligned16(de_rows)) ||
      (dE_table != nullptr && !aligned16(dE_table)))
    return MLS_ERR_UNSUPPORTED;
  if (T > INT_MAX) return MLS_ERR_UNSUPPORTED;
  return MLS_OK;
}

}  // namespace mls

extern "C" {

int mls_version(void) { return 100; }

uint64_t mls_kernel_launches(void) { return mls::g_launches.load(std::memory_order_relaxed); }

const char* mls_status_string(mls_status s) {
  switch (s) {
    case MLS_OK: return "ok";
    case MLS_ERR_INVALID_ARG: return "invalid argument";
    case MLS_ERR_UNSUPPORTED: return "unsupported shape, dtype or alignment";
    case MLS_ERR_WORKSPACE: return "workspace missing or too small";
    case MLS_ERR_CUDA: return "CUDA runtime error";
    case MLS_ERR_BAD_ID: return "token id or target outside [0, V)";
    case MLS_ERR_DEVICE_TIMEOUT: return "a device-side wait ran past its limit";
    case MLS_ERR_NO_DEVICE: return "no compute-capability 10.0 device is current";
  }
  return "unknown status";
}

mls_status mls_junction_fwd(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                            int64_t V, int64_t delta, void* y, float* scale_out, mls_dtype dt,
                            int32_t* dev_status, void* stream) {
  return mls_junction_fwd_variant(x, T, o_m, D_m, e_next, V, delta, y, scale_out, MLS_JUNCTION_STANDARD, dt,
                                  dev_status, stream);
}

mls_status mls_junction_fwd_variant(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                    int64_t V, int64_t delta, void* y, float* scale_out, uint32_t variant,
                                    mls_dtype dt, int32_t* dev_status, void* stream) {
  if (variant & ~kKnownVariants) return MLS_ERR_INVALID_ARG;
  mls_status st = check_junction_shape(x, T, o_m, D_m, e_next, V, delta, dt);
  if (st != MLS_OK) return st;
  if (y == nullptr) return MLS_ERR_INVALID_ARG;
  if (!aligned16(y)) return MLS_ERR_UNSUPPORTED;
  if ((st = device_ok()) != MLS_OK) return st;
  mls::JunctionArgs a{};
  a.bf16 = dt == MLS_BF16;
  a.x = x;
  a.T = T;
  a.D = D_m;
  a.V = V;
  a.delta = delta;
  a.o = o_m;
  a.E = e_next;
  a.y = y;
  a.scale_out = scale_out;
  a.status = dev_status;
  a.variant = variant;
  return from_cuda(mls::launch_junction_fwd(a, static_cast<cudaStream_t>(stream)));
}

mls_status mls_junction_bwd_workspace(int64_t T, int64_t V, size_t* bytes) {
  if (bytes == nullptr || T <= 0 || V <= 0) return MLS_ERR_INVALID_ARG;
  *bytes = mls::junction_scatter_bytes(T, V);
  return MLS_OK;
}

mls_status mls_junction_bwd(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                            int64_t V, int64_t delta, const void* dy, void* do_m, void* de_rows, float* dE_table,
                            int accumulate_dE, void* workspace, size_t ws_bytes, mls_dtype dt,
                            int32_t* dev_status, void* stream) {
  return mls_junction_bwd_variant(x, T, o_m, D_m, e_next, V, delta, dy, do_m, de_rows, dE_table, accumulate_dE,
                                  workspace, ws_bytes, MLS_JUNCTION_STANDARD, dt, dev_status, stream);
}

mls_status mls_junction_bwd_variant(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                    int64_t V, int64_t delta, const void* dy, void* do_m, void* de_rows,
                                    float* dE_table, int accumulate_dE, void* workspace, size_t ws_bytes,
                                    uint32_t variant, mls_dtype dt, int32_t* dev_status, void* stream) {
  mls_status st = mls::check_junction_bwd_args(x, T, o_m, D_m, e_next, V, delta, dy, do_m, de_rows, dE_table,
                                               variant, dt);
  if (st != MLS_OK) return st;
  if (dE_table != nullptr) {
    if (workspace == nullptr || ws_bytes < mls::junction_scatter_bytes(T, V)) return MLS_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLS_ERR_UNSUPPORTED;
  }
  if ((st = device_ok()) != MLS_OK) return st;
  mls::JunctionArgs a{};
  a.bf16 = dt == MLS_BF16;
  a.x = x;
  a.T = T;
  a.D = D_m;
  a.V = V;
  a.delta = delta;
  a.o = o_m;
  a.E = e_next;
  a.dy = dy;
  a.do_out = do_m;
  a.de_out = de_rows;
  a.dE = dE_table;
  a.accumulate_dE = accumulate_dE;
  a.workspace = workspace;
  a.status = dev_status;
  a.variant = variant;
  return from_cuda(mls::launch_junction_bwd(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Shared checks of the multi-junction calls; fills the per-junction shapes.
mls_status check_multi(const int32_t* x, int64_t T, int64_t V, int J, const int64_t* D, const void* const* o,
                       const void* const* e_next, mls_dtype dt, mls::JunctionArgs* js, int32_t* status) {
  if (J < 1 || J > mls::kMaxExits - 1) return J < 1 ? MLS_ERR_INVALID_ARG : MLS_ERR_UNSUPPORTED;
  if (D == nullptr || o == nullptr || e_next == nullptr) return MLS_ERR_INVALID_ARG;
  for (int k = 0; k < J; ++k) {
    if (D[k + 1] <= D[k]) return MLS_ERR_INVALID_ARG;
    const mls_status st = check_junction_shape(x, T, o[k], D[k], e_next[k], V, D[k + 1] - D[k], dt);
    if (st != MLS_OK) return st;
    js[k] = mls::JunctionArgs{};
    js[k].bf16 = dt == MLS_BF16;
    js[k].x = x;
    js[k].T = T;
    js[k].D = D[k];
    js[k].V = V;
    js[k].delta = D[k + 1] - D[k];
    js[k].o = o[k];
    js[k].E = e_next[k];
    js[k].status = status;
  }
  return MLS_OK;
}

}  // namespace

extern "C" {

mls_status mls_junction_fwd_multi(const int32_t* x, int64_t T, int64_t V, int J, const int64_t* D,
                                  const void* const* o, const void* const* e_next, void* const* y,
                                  float* const* scale_out, mls_dtype dt, int32_t* dev_status, void* stream) {
  mls::JunctionArgs js[mls::kMaxExits - 1];
  mls_status st = check_multi(x, T, V, J, D, o, e_next, dt, js, dev_status);
  if (st != MLS_OK) return st;
  if (y == nullptr) return MLS_ERR_INVALID_ARG;
  for (int k = 0; k < J; ++k) {
    if (y[k] == nullptr) return MLS_ERR_INVALID_ARG;
    if (!aligned16(y[k])) return MLS_ERR_UNSUPPORTED;
    js[k].y = y[k];
    js[k].scale_out = scale_out != nullptr ? scale_out[k] : nullptr;
  }
  if ((st = device_ok()) != MLS_OK) return st;
  return from_cuda(mls::launch_junction_fwd_multi(js, J, static_cast<cudaStream_t>(stream)));
}

mls_status mls_junction_bwd_multi_workspace(int64_t T, int64_t V, int J, size_t* bytes) {
  if (bytes == nullptr || T <= 0 || V <= 0 || J < 1) return MLS_ERR_INVALID_ARG;
  if (J > mls::kMaxExits - 1) return MLS_ERR_UNSUPPORTED;
  *bytes = mls::junction_multi_scatter_bytes(T, V, J);
  return MLS_OK;
}

mls_status mls_junction_bwd_multi(const int32_t* x, int64_t T, int64_t V, int J, const int64_t* D,
                                  const void* const* o, const void* const* e_next, const void* const* dy,
                                  void* const* do_m, void* const* de_rows, float* const* dE_table, int accumulate_dE,
                                  void* workspace, size_t ws_bytes, mls_dtype dt, int32_t* dev_status, void* stream) {
  mls::JunctionArgs js[mls::kMaxExits - 1];
  mls_status st = check_multi(x, T, V, J, D, o, e_next, dt, js, dev_status);
  if (st != MLS_OK) return st;
  if (dy == nullptr || do_m == nullptr) return MLS_ERR_INVALID_ARG;
  if (T > INT_MAX) return MLS_ERR_UNSUPPORTED;
  bool any_table = false;
  for (int k = 0; k < J; ++k) {
    void* de = de_rows != nullptr ? de_rows[k] : nullptr;
    float* dE = dE_table != nullptr ? dE_table[k] : nullptr;
    if (dy[k] == nullptr || do_m[k] == nullptr) return MLS_ERR_INVALID_ARG;
    if (!aligned16(dy[k]) || !aligned16(do_m[k]) || (de != nullptr && !aligned16(de)) ||
        (dE != nullptr && !aligned16(dE)))
      return MLS_ERR_UNSUPPORTED;
    js[k].dy = dy[k];
    js[k].do_out = do_m[k];
    js[k].de_out = de;
    js[k].dE = dE;
    js[k].accumulate_dE = accumulate_dE;
    any_table = any_table || dE != nullptr;
  }
  if (any_table) {
    if (workspace == nullptr || ws_bytes < mls::junction_multi_scatter_bytes(T, V, J)) return MLS_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLS_ERR_UNSUPPORTED;
  }
  if ((st = device_ok()) != MLS_OK) return st;
  return from_cuda(mls::launch_junction_bwd_multi(js, J, any_table, workspace, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

extern "C" {

mls_status mls_multiexit_loss_workspace(int M, int64_t T, const int64_t* D, int64_t V, mls_dtype dt,
                                        size_t* fwd_bytes, size_t* bwd_bytes) {
  if (fwd_bytes == nullptr || bwd_bytes == nullptr) return MLS_ERR_INVALID_ARG;
  const mls_status st = check_loss_shape(M, T, V, D, dt);
  if (st != MLS_OK) return st;
  const LossProblem p = shape_problem(M, T, V, D);
  if (dt == MLS_BF16) {
    *fwd_bytes = mls::loss_tc_fwd_bytes(p);
    *bwd_bytes = mls::loss_tc_bwd_bytes(p);
  } else {
    *fwd_bytes = mls::loss_simt_fwd_bytes(p);
    *bwd_bytes = mls::loss_simt_bwd_bytes(p);
  }
  return MLS_OK;
}

mls_status mls_multiexit_loss_bwd_plan(int M, int64_t T, const int64_t* D, int64_t V, mls_dtype dt,
                                       size_t ws_bytes, int64_t* Tb, int64_t* Vc, size_t* min_bytes) {
  if (Tb == nullptr || Vc == nullptr || min_bytes == nullptr) return MLS_ERR_INVALID_ARG;
  const mls_status st = check_loss_shape(M, T, V, D, dt);
  if (st != MLS_OK) return st;
  const LossProblem p = shape_problem(M, T, V, D);
  if (dt != MLS_BF16) {
    *Tb = T;
    *Vc = V;
    *min_bytes = mls::loss_simt_bwd_bytes(p);
    return MLS_OK;
  }
  *min_bytes = mls::loss_tc_bwd_min_bytes(p);
  if (ws_bytes < *min_bytes) {
    *Tb = 0;
    *Vc = 0;
    return MLS_OK;
  }
  mls::loss_tc_bwd_plan(p, ws_bytes, Tb, Vc);
  return MLS_OK;
}

mls_status mls_multiexit_loss_fwd(int M, int64_t T, int64_t V, const int64_t* D, const int32_t* y_targets,
                                  const void* const* h, const void* const* W, float alpha_d, mls_dtype dt,
                                  float* losses, float* stats, void* workspace, size_t ws_bytes,
                                  int32_t* dev_status, void* stream) {
  return mls_multiexit_loss_fwd_opts(M, T, V, D, y_targets, h, W, alpha_d, dt, losses, stats, workspace, ws_bytes,
                                     nullptr, dev_status, stream);
}

mls_status mls_multiexit_loss_fwd_opts(int M, int64_t T, int64_t V, const int64_t* D, const int32_t* y_targets,
                                       const void* const* h, const void* const* W, float alpha_d, mls_dtype dt,
                                       float* losses, float* stats, void* workspace, size_t ws_bytes,
                                       const mls_loss_options* opts, int32_t* dev_status, void* stream) {
  LossProblem p{};
  mls_status st = build_problem(M, T, V, D, y_targets, h, W, alpha_d, dt, dev_status, &p);
  if (st != MLS_OK) return st;
  if ((st = apply_options(opts, &p)) != MLS_OK) return st;
  if (losses == nullptr || stats == nullptr) return MLS_ERR_INVALID_ARG;
  if (!aligned16(stats)) return MLS_ERR_UNSUPPORTED;
  const size_t need = dt == MLS_BF16 ? mls::loss_tc_fwd_bytes(p) : mls::loss_simt_fwd_bytes(p);
  if (workspace == nullptr || ws_bytes < need) return MLS_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLS_ERR_UNSUPPORTED;
  if ((st = device_ok()) != MLS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dt == MLS_BF16) {
    if (!mls::tensor_map_encoder_available()) return MLS_ERR_CUDA;
    return from_cuda(mls::loss_tc_fwd(p, losses, stats, workspace, s));
  }
  return from_cuda(mls::loss_simt_fwd(p, losses, stats, workspace, s));
}

mls_status mls_multiexit_loss_bwd(int M, int64_t T, int64_t V, const int64_t* D, const int32_t* y_targets,
                                  const void* const* h, const void* const* W, float alpha_d, mls_dtype dt,
                                  const float* stats, float grad_scale, void* const* dh, float* const* dW,
                                  int accumulate_dW, void* workspace, size_t ws_bytes, int32_t* dev_status,
                                  void* stream) {
  return mls_multiexit_loss_bwd_opts(M, T, V, D, y_targets, h, W, alpha_d, dt, stats, grad_scale, dh, dW,
                                     accumulate_dW, workspace, ws_bytes, nullptr, dev_status, stream);
}

mls_status mls_multiexit_loss_bwd_opts(int M, int64_t T, int64_t V, const int64_t* D, const int32_t* y_targets,
                                       const void* const* h, const void* const* W, float alpha_d, mls_dtype dt,
                                       const float* stats, float grad_scale, void* const* dh, float* const* dW,
                                       int accumulate_dW, void* workspace, size_t ws_bytes,
                                       const mls_loss_options* opts, int32_t* dev_status, void* stream) {
  LossProblem p{};
  mls_status st = build_problem(M, T, V, D, y_targets, h, W, alpha_d, dt, dev_status, &p);
  if (st != MLS_OK) return st;
  if ((st = apply_options(opts, &p)) != MLS_OK) return st;
  if (stats == nullptr || dh == nullptr || dW == nullptr) return MLS_ERR_INVALID_ARG;
  for (int m = 0; m < M; ++m) {
    if (dh[m] == nullptr || dW[m] == nullptr) return MLS_ERR_INVALID_ARG;
    if (!aligned16(dh[m]) || !aligned16(dW[m])) return MLS_ERR_UNSUPPORTED;
  }
  if (!(grad_scale == grad_scale)) return MLS_ERR_INVALID_ARG;
  const size_t need = dt == MLS_BF16 ? mls::loss_tc_bwd_min_bytes(p) : mls::loss_simt_bwd_bytes(p);
  if (workspace == nullptr || ws_bytes < need) return MLS_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLS_ERR_UNSUPPORTED;
  if ((st = device_ok()) != MLS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dt == MLS_BF16) {
    if (!mls::tensor_map_encoder_available()) return MLS_ERR_CUDA;
    return from_cuda(mls::loss_tc_bwd(p, stats, grad_scale, dh, dW, accumulate_dW, workspace, ws_bytes, s));
  }
  return from_cuda(mls::loss_simt_bwd(p, stats, grad_scale, dh, dW, accumulate_dW, workspace, s));
}

mls_status mls_exit_agreement_workspace(int M, int64_t T, const int64_t* D, int64_t V, mls_dtype dt,
                                        size_t* bytes) {
  if (bytes == nullptr || M < 2) return MLS_ERR_INVALID_ARG;
  const mls_status st = check_loss_shape(M, T, V, D, dt);
  if (st != MLS_OK) return st;
  const LossProblem p = shape_problem(M, T, V, D);
  *bytes = dt == MLS_BF16 ? mls::agree_tc_bytes(p) : mls::agree_simt_bytes(p);
  return MLS_OK;
}

mls_status mls_exit_agreement(int M, int64_t T, int64_t V, const int64_t* D, const void* const* h,
                              const void* const* W, mls_dtype dt, const float* stats, float* metrics,
                              float* per_token, int32_t* top1, void* workspace, size_t ws_bytes,
                              int32_t* dev_status, void* stream) {
  if (M < 2) return MLS_ERR_INVALID_ARG;
  alignas(16) static const int32_t no_targets[4] = {0, 0, 0, 0};
  LossProblem p{};
  mls_status st = build_problem(M, T, V, D, no_targets, h, W, 0.f, dt, dev_status, &p);
  if (st != MLS_OK) return st;
  if (stats == nullptr || metrics == nullptr) return MLS_ERR_INVALID_ARG;
  if (!aligned16(stats) || (per_token != nullptr && !aligned16(per_token)) ||
      (top1 != nullptr && !aligned16(top1)))
    return MLS_ERR_UNSUPPORTED;
  const size_t need = dt == MLS_BF16 ? mls::agree_tc_bytes(p) : mls::agree_simt_bytes(p);
  if (workspace == nullptr || ws_bytes < need) return MLS_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLS_ERR_UNSUPPORTED;
  if ((st = device_ok()) != MLS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dt == MLS_BF16) {
    if (!mls::tensor_map_encoder_available()) return MLS_ERR_CUDA;
    return from_cuda(mls::agree_tc(p, stats, metrics, per_token, top1, workspace, s));
  }
  return from_cuda(mls::agree_simt(p, stats, metrics, per_token, top1, workspace, s));
}

mls_status mls_selftest_wait_timeout(int M, int64_t T, int64_t V, const int64_t* D, const int32_t* y_targets,
                                     const void* const* h, const void* const* W, float* losses, float* stats,
                                     void* workspace, size_t ws_bytes, uint64_t wait_limit_ns,
                                     int32_t* dev_status, void* stream) {
  LossProblem p{};
  mls_status st = build_problem(M, T, V, D, y_targets, h, W, 0.3f, MLS_BF16, dev_status, &p);
  if (st != MLS_OK) return st;
  if (losses == nullptr || stats == nullptr || dev_status == nullptr) return MLS_ERR_INVALID_ARG;
  if (wait_limit_ns < 1000ull || wait_limit_ns > 4000000000ull) return MLS_ERR_INVALID_ARG;
  if (!aligned16(stats)) return MLS_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < mls::loss_tc_fwd_bytes(p)) return MLS_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MLS_ERR_UNSUPPORTED;
  if ((st = device_ok()) != MLS_OK) return st;
  if (!mls::tensor_map_encoder_available()) return MLS_ERR_CUDA;
  p.wait_ns = wait_limit_ns;
  p.withhold_loads = 1;
  return from_cuda(mls::loss_tc_fwd(p, losses, stats, workspace, static_cast<cudaStream_t>(stream)));
}

mls_status mls_status_read(int32_t* dev_status, void* stream, int32_t* host_out) {
  if (dev_status == nullptr || host_out == nullptr) return MLS_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, dev_status, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MLS_ERR_CUDA;
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return MLS_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MLS_ERR_CUDA;
  *host_out = v;
  if (v & MLS_DEVFLAG_TIMEOUT) return MLS_ERR_DEVICE_TIMEOUT;
  if (v & MLS_DEVFLAG_BAD_ID) return MLS_ERR_BAD_ID;
  return MLS_OK;
}

}  // extern "C"
