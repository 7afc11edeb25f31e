// Live-token compaction: the rows of the tokens a loss mask keeps, gathered per sample
// into dense buffers of T_cap rows, so that the projection, the per-sample norms and
// the aggregation run over the kept tokens only.
//
// A masked token contributes nothing to a sample's gradient (the gradient of a linear
// layer is a sum over tokens, A_i^T Gout_i = sum_t a_t^T g_t), so dropping it is an
// exact rewrite of the step of "Metodologia: DP-GRAPE" in the technical summary of
// "Memory-Efficient Differentially Private Training with Gradient Random Projection".
// The pages are silent about masks; they are a property of the workload.
//
// Two kernels:
//   live_index_kernel   one block per sample: an ordered scan of the mask row lists
//                       the kept tokens t_0 < t_1 < ... in idx[i][0 ..), pads the rest
//                       of the T_cap slots with -1, and raises *overflow when a sample
//                       keeps more than T_cap tokens (the first T_cap are listed);
//   gather_rows_kernel  one block per (slot j, sample i, layer l): copies row t_j of
//                       A_l[i] and Gout_l[i] into row j of the compact buffers, or
//                       zeros for a -1 slot (zero rows add nothing to AP^T Gout).
#include <cuda_runtime.h>

#include <cstdint>

#include "compact.h"

namespace grape {
namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) live_index_kernel(const uint8_t* mask, int T_full, int T_cap,
                                                                  int32_t* idx, int32_t* counts, int* overflow) {
  __shared__ int warp_off[kScanThreads / 32];
  __shared__ int chunk_total;
  const int i = blockIdx.x;
  const uint8_t* m = mask + static_cast<size_t>(i) * T_full;
  int32_t* out = idx + static_cast<size_t>(i) * T_cap;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int base = 0;   // kept tokens before this chunk
  for (int t0 = 0; t0 < T_full; t0 += kScanThreads) {
    const int t = t0 + static_cast<int>(threadIdx.x);
    const bool live = t < T_full && m[t] != 0;
    const unsigned ballot = __ballot_sync(0xffffffffu, live);
    const int before_in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_off[wid] = __popc(ballot);
    __syncthreads();
    if (wid == 0) {   // exclusive scan of the 32 warp counts, in warp order
      const int v = warp_off[lane];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      warp_off[lane] = incl - v;
      if (lane == 31) chunk_total = incl;
    }
    __syncthreads();
    const int pos = base + warp_off[wid] + before_in_warp;
    if (live && pos < T_cap) out[pos] = t;
    base += chunk_total;
    __syncthreads();   // warp_off and chunk_total are rewritten by the next chunk
  }
  for (int j = base + static_cast<int>(threadIdx.x); j < T_cap; j += kScanThreads) out[j] = -1;
  if (threadIdx.x == 0) {
    counts[i] = base < T_cap ? base : T_cap;
    if (base > T_cap) atomicOr(overflow, 1);
  }
}

// One row of `row_bytes` bytes: 16-byte vectors when the row allows, else elements.
__device__ __forceinline__ void copy_row(const char* src, char* dst, int row_bytes, int el, bool zero) {
  if ((row_bytes & 15) == 0) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst);
    for (int k = threadIdx.x; k < row_bytes / 16; k += blockDim.x)
      d[k] = zero ? make_uint4(0u, 0u, 0u, 0u) : s[k];
  } else if (el == 4) {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
    uint32_t* d = reinterpret_cast<uint32_t*>(dst);
    for (int k = threadIdx.x; k < row_bytes / 4; k += blockDim.x) d[k] = zero ? 0u : s[k];
  } else {
    const uint16_t* s = reinterpret_cast<const uint16_t*>(src);
    uint16_t* d = reinterpret_cast<uint16_t*>(dst);
    for (int k = threadIdx.x; k < row_bytes / 2; k += blockDim.x) d[k] = zero ? uint16_t(0) : s[k];
  }
}

__global__ void __launch_bounds__(256) gather_rows_kernel(CompactTable tb, const int32_t* idx, int T_full,
                                                          int T_cap, int el) {
  const int j = blockIdx.x, i = blockIdx.y, l = blockIdx.z;
  const int t = idx[static_cast<size_t>(i) * T_cap + j];
  const bool zero = t < 0;
  const size_t src_row = static_cast<size_t>(i) * T_full + (zero ? 0 : t);
  const size_t dst_row = static_cast<size_t>(i) * T_cap + j;
  const int a_bytes = tb.d_in[l] * el, g_bytes = tb.d_out[l] * el;
  copy_row(static_cast<const char*>(tb.A[l]) + src_row * a_bytes, static_cast<char*>(tb.Ac[l]) + dst_row * a_bytes,
           a_bytes, el, zero);
  copy_row(static_cast<const char*>(tb.G[l]) + src_row * g_bytes, static_cast<char*>(tb.Gc[l]) + dst_row * g_bytes,
           g_bytes, el, zero);
}

}  // namespace

cudaError_t compact_live_index(const uint8_t* mask, int B, int T_full, int T_cap, int32_t* idx, int32_t* counts,
                               int* overflow, cudaStream_t st) {
  live_index_kernel<<<B, kScanThreads, 0, st>>>(mask, T_full, T_cap, idx, counts, overflow);
  return cudaGetLastError();
}

cudaError_t compact_gather(const CompactTable& tb, int L, int B, int T_full, int T_cap, int el, const int32_t* idx,
                           cudaStream_t st) {
  gather_rows_kernel<<<dim3(T_cap, B, L), 256, 0, st>>>(tb, idx, T_full, T_cap, el);
  return cudaGetLastError();
}

}  // namespace grape
