// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
// Argument checking happens in api.cu; these functions assume valid inputs.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace mls {

constexpr int kMaxExits = 4;

// ------------------------------------------------------------------ junction
struct JunctionArgs {
  bool bf16;
  const int32_t* x;
  int64_t T, D, V, delta;
  const void* o;
  const void* E;
  void* y;            // fwd output
  float* scale_out;   // fwd, optional
  const void* dy;     // bwd input
  void* do_out;       // bwd output
  void* de_out;       // bwd, optional
  float* dE;          // bwd, optional
  int accumulate_dE;
  void* workspace;
  int32_t* status;
};

struct JunctionScatterWs {
  float* coef;
  int32_t *keys0, *keys1, *vals0, *vals1, *hist;
};

size_t junction_scatter_bytes(int64_t T);
JunctionScatterWs junction_scatter_layout(int64_t T, void* base);
cudaError_t launch_junction_fwd(const JunctionArgs& a, cudaStream_t st);
cudaError_t launch_junction_bwd(const JunctionArgs& a, cudaStream_t st);

// ------------------------------------------------------------------ loss
struct LossProblem {
  int M;
  int64_t T, V;
  int64_t D[kMaxExits];
  const int32_t* y;
  const void* h[kMaxExits];
  const void* W[kMaxExits];
  float alpha_d;
  int32_t* status;
};

// Workspace sizes (bytes) of each path.
size_t loss_tc_fwd_bytes(const LossProblem& p);
size_t loss_tc_bwd_bytes(const LossProblem& p);
size_t loss_simt_fwd_bytes(const LossProblem& p);
size_t loss_simt_bwd_bytes(const LossProblem& p);

// Tensor-core (bf16) path.
cudaError_t loss_tc_fwd(const LossProblem& p, float* losses, float* stats, void* ws, cudaStream_t st);
cudaError_t loss_tc_bwd(const LossProblem& p, const float* stats, float grad_scale, void* const* dh,
                        float* const* dW, int accumulate, void* ws, cudaStream_t st);

// CUDA-core (fp32) path.
cudaError_t loss_simt_fwd(const LossProblem& p, float* losses, float* stats, void* ws, cudaStream_t st);
cudaError_t loss_simt_bwd(const LossProblem& p, const float* stats, float grad_scale, void* const* dh,
                          float* const* dW, int accumulate, void* ws, cudaStream_t st);

// Shared: per-token loss terms [2M-1][T] -> losses [2M], fixed-order reduction.
cudaError_t launch_loss_reduce(const float* terms, int M, int64_t T, float alpha_d, float* losses,
                               cudaStream_t st);

// Counts kernel launches issued by the library (diagnostics).
void note_launches(int n);

// Set when the tensor-map encoder could not be obtained from the driver.
bool tensor_map_encoder_available();

}  // namespace mls
