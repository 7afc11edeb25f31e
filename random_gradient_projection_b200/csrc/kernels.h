// Internal interface between the C ABI (api.cu) and the kernel files.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/grape.h"

namespace grape {

// Library-owned buffers of one layer (device pointers; unused ones are null).
struct LayerWs {
  int d_in, d_out;
  float* P32;              // d_in x r fp32        (CUDA-core path)
  __nv_bfloat16* P16;      // d_in x r bf16 = P    (tensor-core path: back-projection operand)
  void* AP;                // B*T x r: fp32 (CUDA-core) / bf16 (tensor-core)
  float* S;                // r x d_out  sum_i c_i R_i
  float* m;                // r x d_out  Adam first moment
  float* v;                // r x d_out  Adam second moment
  void* dR;                // r x d_out: fp32 (CUDA-core) / bf16 (tensor-core)
  __nv_bfloat16* Rst;      // B x r x d_out bf16: every R_i, stored for the aggregation
                           // (tensor-core path with GRAPE_AGG_STORE; null otherwise)
  int part_base;           // first norm-partial slot of (this layer, sample 0)
  int part_count;          // norm-partial slots per sample of this layer
};

// Per-step inputs of one layer (caller-owned).
struct LayerIo {
  const void* A;           // B x T x d_in
  const void* G;           // B x T x d_out
  float* W;                // d_in x d_out
};

struct StepShape {
  int L, r, B, T, dtype;   // dtype: GRAPE_F32 / GRAPE_BF16
  uint64_t seed;
  float C;
  float sigma_C;           // sigma * C, the noise standard deviation before the average
  float lr, beta1, beta2, eps;
  float one_minus_beta1, one_minus_beta2;
  int part_stride;         // norm-partial slots per sample over all layers
};

// Per-step scalars of the update.
struct UpdateScalars {
  uint32_t step;           // s (0-based)
  float inv_batch;         // 1 / batch_total
  float inv_bc1;           // 1 / (1 - beta1^t)
  float inv_bc2;           // 1 / (1 - beta2^t)
};

// ---- CUDA-core (SIMT, fp32) kernels: simt.cu --------------------------------
// Each enqueues on `st` and returns cudaGetLastError().
// `key`: the step field of P's Philox counter (the step, or step / refresh period).
cudaError_t simt_generate_P(const StepShape& sh, const LayerWs* ws, uint32_t key, cudaStream_t st);
cudaError_t simt_project_ap(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                            cudaStream_t st);
cudaError_t simt_project_norm(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                              float* partials, cudaStream_t st);
// CUDA-graph replay: the kernels whose arguments change every step, and the rewrite of
// those arguments in an instantiated graph (node = the node of the captured graph).
const void* noise_adam_func();
const void* simt_generate_P_func();
cudaError_t noise_adam_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                const LayerWs* ws, const UpdateScalars& u, bool dR_bf16);
cudaError_t simt_generate_P_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                     const LayerWs* ws, uint32_t key);
// Per-sample squared norms: each sample's partial slots summed in a fixed order (no clip).
cudaError_t sum_partials(const StepShape& sh, const float* partials, float* sqnorms, cudaStream_t st);
cudaError_t finalize_clip(const StepShape& sh, const float* partials, float* norms, float* clip,
                          cudaStream_t st);
cudaError_t simt_aggregate(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                           const float* clip, cudaStream_t st);
// pdl: launch as a programmatic dependent of the previous kernel (tensor-core path).
cudaError_t noise_adam(const StepShape& sh, const LayerWs* ws, const UpdateScalars& u,
                       bool dR_bf16, bool pdl, cudaStream_t st);
cudaError_t simt_backproject(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                             float lr, cudaStream_t st);
int simt_partials_per_sample(int r, int d_out);

// ---- generator entry points: simt.cu ------------------------------------------
cudaError_t launch_philox_words(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                                int64_t n_blocks, uint32_t* out, cudaStream_t st);
cudaError_t launch_gaussian(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                            int64_t n, float* out, cudaStream_t st);

}  // namespace grape
