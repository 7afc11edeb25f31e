// CUDA-core (fp32 FFMA) kernels of the DP-GRAPE step.
//
// This is the exact-fp32 path: it serves fp32 inputs (no reduced-precision
// operand anywhere, so the step stays within fp32 rounding of the fp64
// definition) and any shape.  The tensor-core path (tc.cu) serves bf16
// inputs.  The noise + Adam kernel and the clip finalisation are shared by
// both paths.  Every reduction runs in a fixed order (no float atomics), so a
// step is bitwise reproducible.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "philox.cuh"

namespace grape {
namespace {

constexpr int kTile = 64;     // output tile edge of the CUDA-core GEMMs
constexpr int kTileK = 16;    // K step
constexpr int kThreads = 256; // 16 x 16 threads, 4 x 4 outputs each

struct LayerTable {
  LayerWs ws[GRAPE_MAX_LAYERS];
  LayerIo io[GRAPE_MAX_LAYERS];
};

__device__ __forceinline__ float ld_in(const void* p, size_t i, int dtype) {
  if (dtype == GRAPE_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return static_cast<const float*>(p)[i];
}

// C[m0:m0+64, n0:n0+64] += sum_k A(m, k) B(k, n) with one 4 x 4 block per thread.
// A_K_CONTIG / B_N_CONTIG choose the load order that coalesces the global reads.
template <bool A_K_CONTIG, bool B_N_CONTIG, class FA, class FB>
__device__ __forceinline__ void tile_gemm(const FA& fa, const FB& fb, int M, int N, int K, int m0,
                                          int n0, float (&acc)[4][4]) {
  __shared__ float As[kTileK][kTile + 1];
  __shared__ float Bs[kTileK][kTile + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int k0 = 0; k0 < K; k0 += kTileK) {
    for (int e = tid; e < kTile * kTileK; e += kThreads) {
      const int mm = A_K_CONTIG ? (e >> 4) : (e & 63);
      const int ka = A_K_CONTIG ? (e & 15) : (e >> 6);
      const int m = m0 + mm, k = k0 + ka;
      As[ka][mm] = (m < M && k < K) ? fa(m, k) : 0.0f;
      const int nn = B_N_CONTIG ? (e & 63) : (e >> 4);
      const int kb = B_N_CONTIG ? (e >> 6) : (e & 15);
      const int n = n0 + nn, k2 = k0 + kb;
      Bs[kb][nn] = (n < N && k2 < K) ? fb(k2, n) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTileK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
}

// Fixed-order block sum of one float per thread (kThreads threads).
__device__ __forceinline__ float block_sum(float x) {
  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
  __syncthreads();
  float t = 0.0f;
  if (threadIdx.x == 0)
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  return t;
}

// ---- a1: P_l = z(seed, l, s, stream 0, e) / sqrt(r), e = k*r + j -------------
// One thread per block of four elements; blockIdx.y = layer.
__global__ void __launch_bounds__(256) generate_P_kernel(StepShape sh, LayerTable tab, uint32_t step) {
  const int l = blockIdx.y;
  const LayerWs& w = tab.ws[l];
  const int64_t n = static_cast<int64_t>(w.d_in) * sh.r;
  const int64_t nq = (n + 3) / 4;
  const float scale = rsqrtf(static_cast<float>(sh.r));
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < nq;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 z = gaussian4(sh.seed, static_cast<uint32_t>(l), step, kStreamProjection,
                               static_cast<uint32_t>(q));
    const float zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = 4 * q + u;
      if (e >= n) break;
      w.P32[e] = zz[u] * scale;
    }
  }
}

// ---- a2: AP = A P over the stacked B*T rows (per layer, blockIdx.z) -------------
__global__ void __launch_bounds__(kThreads) project_ap_kernel(StepShape sh, LayerTable tab) {
  const int l = blockIdx.z;
  const LayerWs& w = tab.ws[l];
  const void* A = tab.io[l].A;
  const int M = sh.B * sh.T, N = sh.r, K = w.d_in;
  const int m0 = blockIdx.x * kTile, n0 = blockIdx.y * kTile;
  if (m0 >= M || n0 >= N) return;
  const int dt = sh.dtype;
  const float* P = w.P32;
  float acc[4][4] = {};
  tile_gemm<true, true>([&](int m, int k) { return ld_in(A, static_cast<size_t>(m) * K + k, dt); },
                        [&](int k, int n) { return P[static_cast<size_t>(k) * N + n]; }, M, N, K, m0,
                        n0, acc);
  float* AP = static_cast<float*>(w.AP);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) AP[static_cast<size_t>(m) * N + n] = acc[i][j];
    }
}

// ---- a3: R_i = (A_i P)^T Gout_i tile by tile, keeping only ||tile||^2 -----------
// blockIdx.z = l * B + i; partial slot = i * part_stride + part_base + tile.
__global__ void __launch_bounds__(kThreads) project_norm_kernel(StepShape sh, LayerTable tab,
                                                                float* partials) {
  const int l = blockIdx.z / sh.B, i = blockIdx.z % sh.B;
  const LayerWs& w = tab.ws[l];
  const int M = sh.r, N = w.d_out, K = sh.T;
  const int m0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
  if (n0 >= N) return;
  const float* AP = static_cast<const float*>(w.AP) + static_cast<size_t>(i) * sh.T * sh.r;
  const void* G = tab.io[l].G;
  const size_t g0 = static_cast<size_t>(i) * sh.T * N;
  const int dt = sh.dtype;
  float acc[4][4] = {};
  tile_gemm<false, true>([&](int m, int k) { return AP[static_cast<size_t>(k) * M + m]; },
                         [&](int k, int n) { return ld_in(G, g0 + static_cast<size_t>(k) * N + n, dt); },
                         M, N, K, m0, n0, acc);
  float ss = 0.0f;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) ss = fmaf(acc[a][b], acc[a][b], ss);
  const float tot = block_sum(ss);
  if (threadIdx.x == 0) {
    const int n_tiles = (N + kTile - 1) / kTile;
    const int tile = blockIdx.y * n_tiles + blockIdx.x;
    partials[static_cast<size_t>(i) * sh.part_stride + w.part_base + tile] = tot;
  }
}

// ---- a4: n_i = sqrt(sum of partials), c_i = C/n_i if n_i > C else 1 ----------------
// One block per sample; thread t sums slots t, t + 256, ... and the block sum runs
// in a fixed order, so the result does not depend on scheduling.
__global__ void __launch_bounds__(kThreads) clip_kernel(StepShape sh, const float* partials,
                                                        float* norms, float* clip) {
  const int i = blockIdx.x;
  const float* p = partials + static_cast<size_t>(i) * sh.part_stride;
  float ss = 0.0f;
  for (int k = threadIdx.x; k < sh.part_stride; k += kThreads) ss += p[k];
  const float tot = block_sum(ss);
  if (threadIdx.x == 0) {
    const float n = sqrtf(tot);
    norms[i] = n;
    clip[i] = (n > sh.C) ? sh.C / n : 1.0f;
  }
}

// ---- per-sample squared norms alone (the Hutchinson estimate): the sum of a sample's
// partial slots over all layers, in the same fixed order, with no clip ----------------
__global__ void __launch_bounds__(kThreads) sum_partials_kernel(StepShape sh, const float* partials,
                                                                float* sqnorms) {
  const int i = blockIdx.x;
  const float* p = partials + static_cast<size_t>(i) * sh.part_stride;
  float ss = 0.0f;
  for (int k = threadIdx.x; k < sh.part_stride; k += kThreads) ss += p[k];
  const float tot = block_sum(ss);
  if (threadIdx.x == 0) sqnorms[i] = tot;
}

// ---- a5: S_l = sum_i c_i R_i = sum over stacked rows of c_{row/T} AP[row]^T Gout[row] --
__global__ void __launch_bounds__(kThreads) aggregate_kernel(StepShape sh, LayerTable tab,
                                                             const float* clip) {
  const int l = blockIdx.z;
  const LayerWs& w = tab.ws[l];
  const int M = sh.r, N = w.d_out, K = sh.B * sh.T;
  const int m0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
  if (n0 >= N) return;
  const float* AP = static_cast<const float*>(w.AP);
  const void* G = tab.io[l].G;
  const int T = sh.T, dt = sh.dtype;
  float acc[4][4] = {};
  tile_gemm<false, true>(
      [&](int m, int k) { return clip[k / T] * AP[static_cast<size_t>(k) * M + m]; },
      [&](int k, int n) { return ld_in(G, static_cast<size_t>(k) * N + n, dt); }, M, N, K, m0, n0,
      acc);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int m = m0 + ty * 4 + a, n = n0 + tx * 4 + b;
      if (m < M && n < N) w.S[static_cast<size_t>(m) * N + n] = acc[a][b];
    }
}

// ---- a6: g = (S + sigma C xi) / batch; Adam in the projected space ----------------
// xi_l[e] = z(seed, l, s, stream 1, e), e = j*d_out + n.  A thread unit is a block of
// four consecutive elements of one layer (float4 accesses when the layer's r*d_out is a
// multiple of 4; every buffer of the library's arena starts on a 256-byte boundary).
// Units of all layers are numbered back to back (begin[l] .. begin[l+1]) and a grid of a
// few blocks per SM strides over them, so layers of unequal size keep every SM busy and
// no block is launched without work.
//
// After a programmatic (PDL) launch the aggregation that writes S may still be
// running, so S is read only after griddepcontrol.wait.  m and v were last written by
// this kernel in the previous step, and every step begins with an ordinary launch
// (the generation of P) that waits for all earlier work, so the first unit's m and v --
// and its noise, which depends on nothing -- are read and drawn before the wait.
struct AdamTable {
  float* m[GRAPE_MAX_LAYERS];
  float* v[GRAPE_MAX_LAYERS];
  const float* S[GRAPE_MAX_LAYERS];
  void* dR[GRAPE_MAX_LAYERS];
  int64_t n[GRAPE_MAX_LAYERS];               // elements r * d_out of each layer
  int64_t begin[GRAPE_MAX_LAYERS + 1];       // first unit of each layer; begin[L] = total
};

struct AdamUnit {
  float m[4], v[4], xi[4];
  int cnt;      // elements in this unit (4 except a layer's last unit)
  bool vec;     // float4 accesses
};

__device__ __forceinline__ void adam_load_mv(const AdamTable& t, int l, int64_t q, AdamUnit& a) {
  const int64_t n = t.n[l];
  a.cnt = static_cast<int>((n - 4 * q) < 4 ? (n - 4 * q) : 4);
  a.vec = (n % 4) == 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) a.m[k] = a.v[k] = 0.0f;
  if (a.vec) {
    const float4 m4 = reinterpret_cast<const float4*>(t.m[l])[q];
    const float4 v4 = reinterpret_cast<const float4*>(t.v[l])[q];
    a.m[0] = m4.x; a.m[1] = m4.y; a.m[2] = m4.z; a.m[3] = m4.w;
    a.v[0] = v4.x; a.v[1] = v4.y; a.v[2] = v4.z; a.v[3] = v4.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < a.cnt) {
        a.m[k] = t.m[l][4 * q + k];
        a.v[k] = t.v[l][4 * q + k];
      }
  }
}

__device__ __forceinline__ void adam_noise(const StepShape& sh, int l, uint32_t step, int64_t q, AdamUnit& a) {
  if (sh.sigma_C != 0.0f) {
    const float4 z = gaussian4(sh.seed, static_cast<uint32_t>(l), step, kStreamNoise, static_cast<uint32_t>(q));
    a.xi[0] = z.x; a.xi[1] = z.y; a.xi[2] = z.z; a.xi[3] = z.w;
  } else {
    a.xi[0] = a.xi[1] = a.xi[2] = a.xi[3] = 0.0f;
  }
}

__device__ __forceinline__ void adam_finish(const StepShape& sh, const AdamTable& t, const UpdateScalars& u,
                                            int dR_bf16, int l, int64_t q, AdamUnit& a) {
  float S[4] = {0.f, 0.f, 0.f, 0.f};
  if (a.vec) {
    const float4 s4 = reinterpret_cast<const float4*>(t.S[l])[q];
    S[0] = s4.x; S[1] = s4.y; S[2] = s4.z; S[3] = s4.w;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < a.cnt) S[k] = t.S[l][4 * q + k];
  }
  const float b1 = sh.beta1, b2 = sh.beta2;
  const float ob1 = sh.one_minus_beta1, ob2 = sh.one_minus_beta2;
  float d[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float g = fmaf(sh.sigma_C, a.xi[k], S[k]) * u.inv_batch;
    a.m[k] = fmaf(b1, a.m[k], ob1 * g);
    a.v[k] = fmaf(b2, a.v[k], ob2 * g * g);
    d[k] = (a.m[k] * u.inv_bc1) / (sqrtf(a.v[k] * u.inv_bc2) + sh.eps);
  }
  if (a.vec) {
    reinterpret_cast<float4*>(t.m[l])[q] = make_float4(a.m[0], a.m[1], a.m[2], a.m[3]);
    reinterpret_cast<float4*>(t.v[l])[q] = make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
    if (dR_bf16) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(d[0], d[1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(d[2], d[3]);
      reinterpret_cast<uint2*>(t.dR[l])[q] =
          make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    } else {
      reinterpret_cast<float4*>(t.dR[l])[q] = make_float4(d[0], d[1], d[2], d[3]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= a.cnt) continue;
      const int64_t e = 4 * q + k;
      t.m[l][e] = a.m[k];
      t.v[l][e] = a.v[k];
      if (dR_bf16)
        static_cast<__nv_bfloat16*>(t.dR[l])[e] = __float2bfloat16_rn(d[k]);
      else
        static_cast<float*>(t.dR[l])[e] = d[k];
    }
  }
}

__global__ void __launch_bounds__(256) noise_adam_kernel(StepShape sh, AdamTable t, UpdateScalars u,
                                                         int dR_bf16) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t total = t.begin[sh.L];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t unit = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  int l = 0;
  AdamUnit a;
  if (unit < total) {   // the first unit's m, v and noise do not depend on the running kernel
    while (unit >= t.begin[l + 1]) ++l;
    adam_load_mv(t, l, unit - t.begin[l], a);
    adam_noise(sh, l, u.step, unit - t.begin[l], a);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (bool first = true; unit < total; unit += stride, first = false) {
    while (unit >= t.begin[l + 1]) ++l;   // units only grow, so l only moves forward
    const int64_t q = unit - t.begin[l];
    if (!first) {
      adam_load_mv(t, l, q, a);
      adam_noise(sh, l, u.step, q, a);
    }
    adam_finish(sh, t, u, dR_bf16, l, q, a);
  }
}

// ---- a7: W_l -= lr * P_l dR_l --------------------------------------------------
__global__ void __launch_bounds__(kThreads) backproject_kernel(StepShape sh, LayerTable tab,
                                                               float lr) {
  const int l = blockIdx.z;
  const LayerWs& w = tab.ws[l];
  const int M = w.d_in, N = w.d_out, K = sh.r;
  const int m0 = blockIdx.y * kTile, n0 = blockIdx.x * kTile;
  if (m0 >= M || n0 >= N) return;
  const float* P = w.P32;
  const float* dR = static_cast<const float*>(w.dR);
  float acc[4][4] = {};
  tile_gemm<true, true>([&](int m, int k) { return P[static_cast<size_t>(m) * K + k]; },
                        [&](int k, int n) { return dR[static_cast<size_t>(k) * N + n]; }, M, N, K,
                        m0, n0, acc);
  float* W = tab.io[l].W;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int m = m0 + ty * 4 + a, n = n0 + tx * 4 + b;
      if (m < M && n < N) {
        const size_t o = static_cast<size_t>(m) * N + n;
        W[o] = fmaf(-lr, acc[a][b], W[o]);
      }
    }
}

// ---- generator entry points -------------------------------------------------
__global__ void philox_words_kernel(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                                    int64_t n_blocks, uint32_t* out) {
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < n_blocks;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 w = philox_block(seed, layer, step, stream_id, static_cast<uint32_t>(q));
    reinterpret_cast<uint4*>(out)[q] = w;
  }
}

__global__ void gaussian_kernel(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                                int64_t n, float* out) {
  const int64_t nq = (n + 3) / 4;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < nq;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 z = gaussian4(seed, layer, step, stream_id, static_cast<uint32_t>(q));
    const float zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (4 * q + u < n) out[4 * q + u] = zz[u];
  }
}

LayerTable make_table(const StepShape& sh, const LayerWs* ws, const LayerIo* io) {
  LayerTable t{};
  for (int l = 0; l < sh.L; ++l) {
    t.ws[l] = ws[l];
    if (io) t.io[l] = io[l];
  }
  return t;
}

int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

int max_d_out(const StepShape& sh, const LayerWs* ws) {
  int m = 0;
  for (int l = 0; l < sh.L; ++l) m = ws[l].d_out > m ? ws[l].d_out : m;
  return m;
}
int max_d_in(const StepShape& sh, const LayerWs* ws) {
  int m = 0;
  for (int l = 0; l < sh.L; ++l) m = ws[l].d_in > m ? ws[l].d_in : m;
  return m;
}

}  // namespace

int simt_partials_per_sample(int r, int d_out) { return cdiv(r, kTile) * cdiv(d_out, kTile); }

cudaError_t simt_generate_P(const StepShape& sh, const LayerWs* ws, uint32_t step, cudaStream_t st) {
  const LayerTable t = make_table(sh, ws, nullptr);
  int64_t most = 0;
  for (int l = 0; l < sh.L; ++l) {
    const int64_t q = (static_cast<int64_t>(ws[l].d_in) * sh.r + 3) / 4;
    most = q > most ? q : most;
  }
  if (ws[0].P32 == nullptr) return cudaErrorInvalidValue;   // fp32 P lives on the CUDA-core path only
  dim3 grid(cdiv(most, 256) < 1184 ? cdiv(most, 256) : 1184, sh.L);
  generate_P_kernel<<<grid, 256, 0, st>>>(sh, t, step);
  return cudaGetLastError();
}

cudaError_t simt_project_ap(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                            cudaStream_t st) {
  const LayerTable t = make_table(sh, ws, io);
  dim3 g1(cdiv(static_cast<int64_t>(sh.B) * sh.T, kTile), cdiv(sh.r, kTile), sh.L);
  project_ap_kernel<<<g1, kThreads, 0, st>>>(sh, t);
  return cudaGetLastError();
}

cudaError_t simt_project_norm(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                              float* partials, cudaStream_t st) {
  const LayerTable t = make_table(sh, ws, io);
  dim3 g2(cdiv(max_d_out(sh, ws), kTile), cdiv(sh.r, kTile), sh.L * sh.B);
  project_norm_kernel<<<g2, kThreads, 0, st>>>(sh, t, partials);
  return cudaGetLastError();
}

cudaError_t finalize_clip(const StepShape& sh, const float* partials, float* norms, float* clip,
                          cudaStream_t st) {
  clip_kernel<<<sh.B, kThreads, 0, st>>>(sh, partials, norms, clip);
  return cudaGetLastError();
}

cudaError_t sum_partials(const StepShape& sh, const float* partials, float* sqnorms, cudaStream_t st) {
  sum_partials_kernel<<<sh.B, kThreads, 0, st>>>(sh, partials, sqnorms);
  return cudaGetLastError();
}

cudaError_t simt_aggregate(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                           const float* clip, cudaStream_t st) {
  const LayerTable t = make_table(sh, ws, io);
  dim3 g(cdiv(max_d_out(sh, ws), kTile), cdiv(sh.r, kTile), sh.L);
  aggregate_kernel<<<g, kThreads, 0, st>>>(sh, t, clip);
  return cudaGetLastError();
}

AdamTable make_adam_table(const StepShape& sh, const LayerWs* ws) {
  AdamTable t{};
  int64_t at = 0;
  for (int l = 0; l < sh.L; ++l) {
    t.m[l] = ws[l].m;
    t.v[l] = ws[l].v;
    t.S[l] = ws[l].S;
    t.dR[l] = ws[l].dR;
    t.n[l] = static_cast<int64_t>(sh.r) * ws[l].d_out;
    t.begin[l] = at;
    at += (t.n[l] + 3) / 4;
  }
  t.begin[sh.L] = at;
  return t;
}

// Blocks of the noise + Adam grid: 8 resident 256-thread blocks per SM, never more than
// there are units.
unsigned adam_blocks(const AdamTable& t, int L) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);   // the current device's SM count (the runtime answers from its cache)
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  const int64_t need = (t.begin[L] + 255) / 256;
  const int64_t fill = static_cast<int64_t>(sms) * 8;
  const int64_t b = need < fill ? need : fill;
  return static_cast<unsigned>(b > 0 ? b : 1);
}

cudaError_t noise_adam(const StepShape& sh, const LayerWs* ws, const UpdateScalars& u, bool dR_bf16,
                       bool pdl, cudaStream_t st) {
  const AdamTable t = make_adam_table(sh, ws);
  const dim3 grid(adam_blocks(t, sh.L));
  if (!pdl) {
    noise_adam_kernel<<<grid, 256, 0, st>>>(sh, t, u, dR_bf16 ? 1 : 0);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = a;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, noise_adam_kernel, sh, t, u, dR_bf16 ? 1 : 0);
}

cudaError_t simt_backproject(const StepShape& sh, const LayerWs* ws, const LayerIo* io, float lr,
                             cudaStream_t st) {
  const LayerTable t = make_table(sh, ws, io);
  dim3 g(cdiv(max_d_out(sh, ws), kTile), cdiv(max_d_in(sh, ws), kTile), sh.L);
  backproject_kernel<<<g, kThreads, 0, st>>>(sh, t, lr);
  return cudaGetLastError();
}

// ---- CUDA-graph replay: the step-dependent arguments of captured nodes ----------------
const void* noise_adam_func() { return reinterpret_cast<const void*>(noise_adam_kernel); }
const void* simt_generate_P_func() { return reinterpret_cast<const void*>(generate_P_kernel); }

cudaError_t noise_adam_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                const LayerWs* ws, const UpdateScalars& u, bool dR_bf16) {
  cudaKernelNodeParams p{};
  cudaError_t e = cudaGraphKernelNodeGetParams(node, &p);
  if (e != cudaSuccess) return e;
  StepShape a0 = sh;
  AdamTable a1 = make_adam_table(sh, ws);
  UpdateScalars a2 = u;
  int a3 = dR_bf16 ? 1 : 0;
  void* args[] = {&a0, &a1, &a2, &a3};
  p.kernelParams = args;
  p.extra = nullptr;
  return cudaGraphExecKernelNodeSetParams(exec, node, &p);
}

cudaError_t simt_generate_P_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                     const LayerWs* ws, uint32_t key) {
  cudaKernelNodeParams p{};
  cudaError_t e = cudaGraphKernelNodeGetParams(node, &p);
  if (e != cudaSuccess) return e;
  StepShape a0 = sh;
  LayerTable a1 = make_table(sh, ws, nullptr);
  uint32_t a2 = key;
  void* args[] = {&a0, &a1, &a2};
  p.kernelParams = args;
  p.extra = nullptr;
  return cudaGraphExecKernelNodeSetParams(exec, node, &p);
}

cudaError_t launch_philox_words(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                                int64_t n_blocks, uint32_t* out, cudaStream_t st) {
  const int grid = cdiv(n_blocks, 256) < 1184 ? cdiv(n_blocks, 256) : 1184;
  philox_words_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(seed, layer, step, stream_id, n_blocks, out);
  return cudaGetLastError();
}

cudaError_t launch_gaussian(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                            int64_t n, float* out, cudaStream_t st) {
  const int grid = cdiv((n + 3) / 4, 256) < 1184 ? cdiv((n + 3) / 4, 256) : 1184;
  gaussian_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(seed, layer, step, stream_id, n, out);
  return cudaGetLastError();
}

}  // namespace grape
