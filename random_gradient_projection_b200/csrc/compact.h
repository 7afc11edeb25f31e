// Live-token compaction (compact.cu): host launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "grape.h"

namespace grape {

// Per layer: the full inputs (B x T_full rows) and the compact buffers (B x T_cap rows),
// row-major with samples contiguous, elements of `el` bytes.
struct CompactTable {
  const void* A[GRAPE_MAX_LAYERS];
  const void* G[GRAPE_MAX_LAYERS];
  void* Ac[GRAPE_MAX_LAYERS];
  void* Gc[GRAPE_MAX_LAYERS];
  int d_in[GRAPE_MAX_LAYERS];
  int d_out[GRAPE_MAX_LAYERS];
};

// idx: B x T_cap int32 (kept token of each slot, -1 = padding); counts: B int32 (kept
// tokens listed, at most T_cap); *overflow |= 1 when a sample keeps more than T_cap.
cudaError_t compact_live_index(const uint8_t* mask, int B, int T_full, int T_cap, int32_t* idx, int32_t* counts,
                               int* overflow, cudaStream_t st);
// Copy the listed rows of every layer's A and Gout into the compact buffers (zeros for -1).
cudaError_t compact_gather(const CompactTable& tb, int L, int B, int T_full, int T_cap, int el, const int32_t* idx,
                           cudaStream_t st);

}  // namespace grape
