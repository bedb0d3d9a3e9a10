// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
// Argument checking happens in api.cu; these functions assume valid inputs.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "mls.h"

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
  uint32_t variant;   // junction variant bits (0 = the standard junction)
};

// Every argument check of mls_junction_bwd_variant except the workspace's.
mls_status check_junction_bwd_args(const int32_t* x, int64_t T, const void* o_m, int64_t D_m, const void* e_next,
                                   int64_t V, int64_t delta, const void* dy, const void* do_m, const void* de_rows,
                                   const float* dE_table, uint32_t variant, mls_dtype dt);

size_t junction_scatter_bytes(int64_t T, int64_t V);
cudaError_t launch_junction_fwd(const JunctionArgs& a, cudaStream_t st);
cudaError_t launch_junction_bwd(const JunctionArgs& a, cudaStream_t st);
// J junctions sharing x, T and V (standard junction; dtype of js[0] for all).
size_t junction_multi_scatter_bytes(int64_t T, int64_t V, int J);
cudaError_t launch_junction_fwd_multi(const JunctionArgs* js, int J, cudaStream_t st);
cudaError_t launch_junction_bwd_multi(const JunctionArgs* js, int J, bool any_table, void* ws, cudaStream_t st);

// ------------------------------------------------------------------ id-grouped row sums
// Tokens grouped by id (stable in t): the tokens of id v are
// toks[offsets[v] .. ends[v]).  Ids outside [0, V) are left out.
struct SegIndexDev {
  int64_t V;
  const int32_t* ends;
  const int32_t* offsets;
  const int32_t* toks;
  const int32_t* heavy;      // ids with many tokens
  const int32_t* n_heavy;
  int64_t max_heavy;
  const int32_t* light;      // ids with 1..kHeavy tokens (any order)
  const int32_t* n_light;
  int64_t max_light;
};

// A per-device side stream for work that does not depend on the kernels the
// caller's stream runs meanwhile (the id sort beside the junction row kernels,
// the fp16 operand copies beside the loss backward's tensor-core kernels):
// forked from the caller's stream with an event (at construction and at each
// fork()), joined back into it with another (join(), and at destruction), so
// under graph capture it becomes parallel branches.  One scope at a time per
// process (a mutex held for the scope's life); without a side stream
// (creation failed, or built with MLS_SIDE_STREAM=0) stream() is the caller's
// stream and fork()/join() do nothing.
class SideScope {
 public:
  explicit SideScope(cudaStream_t st);
  ~SideScope();
  cudaStream_t stream() const { return side_; }
  cudaError_t fork();
  cudaError_t join();
 private:
  cudaStream_t main_, side_;
  void* slot_;
  bool joined_;
};

size_t segindex_bytes(int64_t T, int64_t V);
cudaError_t build_segindex(const int32_t* ids, int64_t T, int64_t V, void* ws, SegIndexDev* out, cudaStream_t st);
// dE[v] (+)= ge sum_t g_e,t + (sum_t coef_t) E[v]; g_e is the tail of each dy row.
cudaError_t scatter_table_grad(const SegIndexDev& ix, bool bf16, const void* dy, int d_vec, int dl_vec,
                               const float* coef, float ge, const void* E, float* dE, bool accumulate,
                               cudaStream_t st);
// The same for several tables that share the ids (the junctions of one suite), one launch set for all.
struct TableGradJob {
  const void* dy;
  int d_vec, dl_vec;
  const float* coef;
  float ge;
  const void* E;
  float* dE;
};
// The rows of ids with many tokens go to heavy_st (disjoint rows; it may be st).
cudaError_t scatter_table_grads(const SegIndexDev& ix, bool bf16, int njobs, const TableGradJob* jobs, bool accumulate,
                                cudaStream_t st, cudaStream_t heavy_st);
// For every job z < njobs (at most kMaxExits; one launch pair for all):
//   dW[z][v] -= scale[z] * sum_{t: y_t = v} h[z]_t  (bf16 rows of d_vec[z] 16-byte vectors).
// The rows of ids with many tokens go to heavy_st (disjoint rows; it may be st).
cudaError_t scatter_target_rows(const SegIndexDev& ix, int njobs, const void* const* h, const int* d_vec,
                                float* const* dW, const float* scale, cudaStream_t st, cudaStream_t heavy_st);

// ------------------------------------------------------------------ loss
struct LossProblem {
  int M;
  int64_t T, V;
  int64_t D[kMaxExits];
  const int32_t* y;
  const void* h[kMaxExits];
  const void* W[kMaxExits];
  float alpha_d;
  float exit_w[kMaxExits];   // per-exit loss weights (1 = equal weights)
  int distill;               // 0: cross-entropy to the largest exit, 1: KL(q_m || p_M), 2: Jensen-Shannon
  int teacher_grad;          // 1: the largest exit also gets the distillation gradient (no stop-gradient)
  int32_t* status;
  uint64_t wait_ns;          // limit of the tile kernels' barrier waits; 0 = the library default
  int withhold_loads;        // test of the bounded waits only: the tile kernel's producer issues no loads
};

// Workspace sizes (bytes) of each path.
size_t loss_tc_fwd_bytes(const LossProblem& p);
size_t loss_tc_bwd_bytes(const LossProblem& p);
size_t loss_simt_fwd_bytes(const LossProblem& p);
size_t loss_simt_bwd_bytes(const LossProblem& p);

// Tensor-core (bf16) path.  The backward pass runs in (token block x vocabulary
// chunk) pieces sized to the workspace it is given: loss_tc_bwd_bytes is the
// size of the plan for a 1.5 GiB budget (or of the whole problem, when smaller),
// loss_tc_bwd_min_bytes the smallest workspace any plan fits in.
size_t loss_tc_bwd_min_bytes(const LossProblem& p);
void loss_tc_bwd_plan(const LossProblem& p, size_t ws_bytes, int64_t* Tb, int64_t* Vc);
cudaError_t loss_tc_fwd(const LossProblem& p, float* losses, float* stats, void* ws, cudaStream_t st);
cudaError_t loss_tc_bwd(const LossProblem& p, const float* stats, float grad_scale, void* const* dh,
                        float* const* dW, int accumulate, void* ws, size_t ws_bytes, cudaStream_t st);

// CUDA-core (fp32) path.
cudaError_t loss_simt_fwd(const LossProblem& p, float* losses, float* stats, void* ws, cudaStream_t st);
cudaError_t loss_simt_bwd(const LossProblem& p, const float* stats, float grad_scale, void* const* dh,
                          float* const* dW, int accumulate, void* ws, cudaStream_t st);

// Agreement of every smaller exit with the largest: metrics [3(M-1)] = means of
// beta, KL(p_M || q_m) and top-1 agreement; optional per-token rows and top-1 ids.
size_t agree_tc_bytes(const LossProblem& p);
size_t agree_simt_bytes(const LossProblem& p);
cudaError_t agree_tc(const LossProblem& p, const float* stats, float* metrics, float* per_token, int32_t* top1,
                     void* ws, cudaStream_t st);
cudaError_t agree_simt(const LossProblem& p, const float* stats, float* metrics, float* per_token, int32_t* top1,
                       void* ws, cudaStream_t st);

// Shared: rows [Q][T] -> their means over T, fixed-order reduction.
cudaError_t launch_row_means(const float* rows, int Q, int64_t T, float* out, cudaStream_t st);

// Shared: per-token loss terms [2M-1][T] -> losses [2M], fixed-order reduction.
cudaError_t launch_loss_reduce(const float* terms, const LossProblem& p, float* losses, cudaStream_t st);

// Counts kernel launches issued by the library (diagnostics).
void note_launches(int n);

// Set when the tensor-map encoder could not be obtained from the driver.
bool tensor_map_encoder_available();

}  // namespace mls
