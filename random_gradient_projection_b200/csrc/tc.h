// Tensor-core (tcgen05 / TMEM / TMA) path of the DP-GRAPE step for bf16 inputs.
#pragma once
#include <cuda_runtime.h>

#include <string>

#include "kernels.h"

namespace grape {

#ifdef GRAPE_CHECKED
// Bounds-checked build: the error-word bit of a TMA box that would start outside its
// tensor or off the 16-byte rule (the copy is skipped).
constexpr int kTcErrBounds = 8;
#endif

struct TcWorkspace {
  void* base = nullptr;       // library scratch inside the context arena
  size_t bytes = 0;
  void* host_state = nullptr; // tensor maps and launch plans (host memory)
};

bool tc_supported(int device, const grape_layer* layers, int n_layers, int r, int B, int T,
                  std::string* why);
int tc_partials_per_sample(int r, int d_out);
size_t tc_workspace_bytes(const StepShape& sh, const LayerWs* ws);
cudaError_t tc_init(const StepShape& sh, const LayerWs* ws, void* scratch, size_t bytes,
                    TcWorkspace* out);
void tc_release(TcWorkspace* tc);
// Device word where the tensor-core kernels record bounded waits that gave up (0 = none).
int* tc_error_word(const TcWorkspace& tc);
// Self-test of the bounded mbarrier waits (see grape_selftest_wait_timeout): ORs into
// *bits_dev 1 (warp 0 gave up at its limit), 2 (warp 1 left on the abort flag) or 4
// (warp 1 ran to its own limit).
cudaError_t tc_selftest_wait(uint64_t short_ns, uint64_t long_ns, int* bits_dev, cudaStream_t st);
// CUDA-graph replay: the P-generation kernel and the rewrite of its key in a graph.
const void* tc_gen_P_func();
cudaError_t tc_generate_P_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                   const LayerWs* ws, uint32_t key);
// The phases of the tensor-core path; each enqueues on `st`, adds the number of
// kernels it launched to *launches and returns the first CUDA error.
// `key` is the step field of P's Philox counter (the step, or step / refresh period).
cudaError_t tc_generate_P(const StepShape& sh, const LayerWs* ws, const TcWorkspace& tc,
                          uint32_t key, cudaStream_t st, int* launches);
// `first_in_step`: no P was generated this step (it is still valid from an earlier one),
// so the projection is the step's first kernel and is launched as an ordinary launch.
cudaError_t tc_project(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                       const TcWorkspace& tc, cudaStream_t st, int* launches, bool first_in_step);
// The same partials by the ghost identity (two T x T Gram matrices per sample and layer);
// needs T <= 128 (tc_ghost_supported).
bool tc_ghost_supported(const StepShape& sh);
cudaError_t tc_project_norm_ghost(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                                  const TcWorkspace& tc, float* partials, cudaStream_t st, int* launches);
// store_R: also write every R_i (bf16) to ws[l].Rst for tc_aggregate_stored.
cudaError_t tc_project_norm(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                            const TcWorkspace& tc, float* partials, bool store_R, cudaStream_t st,
                            int* launches);
// n_i and c_i; with rescale_ap, AP is also scaled in place by c_i for tc_aggregate.
cudaError_t tc_clip_scale(const StepShape& sh, const LayerWs* ws, const TcWorkspace& tc,
                          const float* partials, float* norms, float* clip, bool rescale_ap,
                          cudaStream_t st, int* launches);
// S = (diag(c) AP)^T Gout over the stacked rows (AP already scaled by c).
cudaError_t tc_aggregate(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                         const TcWorkspace& tc, const float* clip, cudaStream_t st, int* launches);
// S = sum_i c_i R_i over the R_i stored by tc_project_norm(store_R = true).
// The stored aggregation fused with noise + Adam, for a one-process step: S = sum_i
// c_i R_i (written to ws[l].S), then the update of m, v and dR (bf16) as noise_adam
// computes it, with the same bits.  The _func / _set_node pair rewrites the captured
// node's step-dependent arguments on a graph replay.
cudaError_t tc_aggregate_adam(const StepShape& sh, const LayerWs* ws, const UpdateScalars& u, const float* clip,
                              cudaStream_t st, int* launches);
const void* tc_aggregate_adam_func();
cudaError_t tc_aggregate_adam_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                       const LayerWs* ws, const UpdateScalars& u, const float* clip);
cudaError_t tc_aggregate_stored(const StepShape& sh, const LayerWs* ws, const float* clip, cudaStream_t st,
                                int* launches);
cudaError_t tc_backproject(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                           const TcWorkspace& tc, float lr, cudaStream_t st, int* launches);

// Per-sample squared norms of one layer using only the library's static device
// scratch (grape_layer_sqnorms_static).
size_t tc_static_scratch_bytes();
// Whether the driver provides the tensor-map encoder every tensor-core kernel needs.
bool tc_tensor_maps_available();
size_t tc_static_scratch_needed(int d_in, int d_out, int r, int B, int T);
cudaError_t tc_layer_sqnorms_static(const void* A, const void* G, int d_in, int d_out, int r, int B,
                                    int T, uint64_t seed, uint32_t layer, uint32_t step, float* out,
                                    cudaStream_t st);

}  // namespace grape
