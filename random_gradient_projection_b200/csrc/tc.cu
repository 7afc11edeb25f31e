// Tensor-core (tcgen05 / TMEM / TMA) path of the DP-GRAPE step for bf16 inputs.
//
// The step's four dense contractions (the closing paragraph of "Metodologia: DP-GRAPE"
// in the technical summary of "Memory-Efficient Differentially Private Training with
// Gradient Random Projection": per-sample projection, norms for clipping, aggregation,
// and the projected update of the parameters):
//
//   PROJECT    AP   = A P            M = B*T rows, N = r,     K = d_in
//   NORM       ||R_i||^2, R_i = (A_i P)^T Gout_i
//                                    M = r,        N = d_out, K = T  (per sample)
//   AGGREGATE  S    = sum_i c_i R_i  M = r,        N = d_out, K = B*T (split-K)
//   BACKPROJ   W   -= lr P dR        M = d_in,     N = d_out, K = r
//
// run on one warp-specialised UMMA kernel template, tc_gemm_kernel<MODE, BN, STAGES>,
// described below, and on kernels built for the shapes where it is not the fastest:
//
//   tc_project_wide_kernel    PROJECT for r >= 256 in 256-row tiles (two MMAs share
//                             each P stage), on an LPT tile schedule made on the host
//   tc_norm_tmem_kernel       NORM with the R_i store for 256 < T <= 512, the block
//                             of (A_i P)^T resident in TMEM as the MMA's A operand
//   tc_backproj_tmem_kernel   BACKPROJ for r = 512, the block of P resident in TMEM
//   tc_agg_cluster_kernel     AGGREGATE with K split over a cluster (few output tiles)
//
// and CUDA-core kernels: P's generation (gen_P_bf16_kernel), the clip factors
// (clip_scale_kernel), the sum of stored R_i alone (aggregate_stored_kernel) or fused
// with noise + Adam (aggregate_adam_kernel), and the no-allocation entry point's helpers.
//
// tc_gemm_kernel's CTA layout (416 threads, one CTA per SM: the runtime places a single CTA of a kernel
// that allocates TMEM on each SM): four producer warps (0, 10, 11, 12) issue the TMA
// loads into a ring of shared-memory stages (128-byte swizzle), producer p filling the
// stages of k-block iterations it = p (mod 4) -- the TMA stream of one issuing thread
// moves about 25 GB/s of L2-resident data into an SM and four such streams about
// 86 GB/s, so the issue is spread; warp 1 owns the TMEM allocation and one of its
// threads issues tcgen05.mma (M = 128, N = BN, K = 16 per instruction) into one of
// two 128 x BN fp32 TMEM accumulators; warps 2-9 read the accumulator back with
// tcgen05.ld (each warp its 32 TMEM lanes) and run the epilogue.  Stage reuse is
// tracked with mbarriers (TMA completion -> full, tcgen05.commit -> empty); every
// wait is bounded and reports a timeout through an error word.
//
// Operands: A, P (as the A operand of BACKPROJ) are K-major tiles of 128 rows x
// 64 bf16; AP^T (NORM / AGGREGATE) and every B operand (P, Gout, dR) are
// M/N-major: 64-element chunks of 64 K-rows x 128 bytes, one TMA box each.
// Samples with T not a multiple of 64 load through 3-D tensor maps
// (B x T x cols): rows past T are zero-filled by the TMA unit, so no sample
// mixes with the next.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "philox.cuh"
#include "tc.h"
#include "tc_ptx.cuh"

namespace grape {
namespace {

constexpr int kBM = 128;           // UMMA M (one CTA, TMEM lanes)
constexpr int kBK = 64;            // K per stage: one 128-byte swizzle row of bf16
constexpr int kEpiWarps = 8;       // two per TMEM lane quarter, each on half the columns
constexpr int kProducers = 4;                    // TMA-issuing warps: 0 and 10, 11, 12
// A ring of STAGES stages is filled by min(kProducers, STAGES) of them.  An mbarrier
// parity wait tells only adjacent phases apart: a producer waiting for phase u-1 of
// empty[s] must know that phase u-2 is complete, and its own previous wait (kP
// iterations earlier) guarantees that only when kP <= STAGES.
template <int STAGES>
struct RingProducers {
  static constexpr int kCount = STAGES < kProducers ? STAGES : kProducers;
};
constexpr int kThreads = 32 * (2 + kEpiWarps + kProducers - 1);   // 416
// producer index of a warp (0 .. kProducers-1), or -1 for the MMA and epilogue warps
__device__ __forceinline__ int producer_of(int warp) {
  return warp == 0 ? 0 : (warp >= 2 + kEpiWarps ? warp - (2 + kEpiWarps) + 1 : -1);
}
constexpr int kMaxGroup = 16;      // layers per launch
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint64_t kDrainLimitNs = 1000000000ull;   // after an abort: wait for loads in flight

// NORMST: NORM that also stores every tile of R_i (bf16) for the stored aggregation.
enum Mode : int { PROJECT = 0, NORM = 1, AGGREGATE = 2, BACKPROJ = 3, GHOST = 4, NORMST = 5 };

// error word bits
constexpr int kErrTimeoutProducer = 1;
constexpr int kErrTimeoutMma = 2;
constexpr int kErrTimeoutEpilogue = 4;

struct GroupLayer {
  int tiles_begin;   // first tile of this layer in the launch
  int mt, nt, ns;    // m tiles, n tiles, samples (NORM; 1 otherwise)
  int kblocks;       // k-blocks of the whole K extent
  int M, N;          // output extent
  int ldo;           // leading dimension of the output
  void* out;         // PROJECT: AP (bf16); AGGREGATE: S; BACKPROJ: W
  int part_base;     // NORM, GHOST: first partial slot of this layer
  int slots;         // GHOST: partial slots of this layer per sample (the first gets the sum)
  int kfirst;        // GHOST: k-blocks of Gout, loaded before the k-blocks of AP
  int nb;            // GHOST: 128-token blocks of a sample, ceil(T / 128)
};

struct GroupParams {
  CUtensorMap mapA[kMaxGroup];
  CUtensorMap mapB[kMaxGroup];
  CUtensorMap mapW[kMaxGroup];   // BACKPROJ: W as fp32 (32-column x 128-row boxes)
  GroupLayer lay[kMaxGroup];
  int n_layers;
  int total_tiles;
  int part_stride;   // NORM
  float* partials;   // NORM
  float lr;          // BACKPROJ
  int cluster;       // AGGREGATE on a cluster: CTAs per output tile (K split)
  // tc_project_wide_kernel: the launch's tiles in the order CTAs take them (total_tiles
  // ints), then each CTA's first position in that order (grid + 1 ints)
  const int* sched;
  int* err;
#ifdef GRAPE_CHECKED
  int extA[kMaxGroup][3];   // x, y, z extents of the tensors behind mapA, mapB, mapW
  int extB[kMaxGroup][3];
  int extW[kMaxGroup][3];
#endif
};

// Bounds-checked build (GRAPE_CHECKED): before each TMA copy, GRAPE_BOX checks that
// the box starts inside its tensor and that x times the element size is a multiple of
// 16 bytes.  A violation sets kTcErrBounds in the error word and skips the copy; its
// stage then never completes, and the bounded waits end the kernel.  In the default
// build GRAPE_BOX and GRAPE_EXT expand to nothing.
#ifdef GRAPE_CHECKED
__device__ __forceinline__ bool box_ok(int* err, const int (&ext)[3], int el, int x, int y, int z) {
  const bool ok = x >= 0 && y >= 0 && z >= 0 && x < ext[0] && y < ext[1] && z < ext[2] &&
                  (x * el) % 16 == 0;
  if (!ok) atomicOr(err, kTcErrBounds);
  return ok;
}
inline void set_ext(int (&e)[3], int64_t x, int64_t y, int64_t z) {
  e[0] = static_cast<int>(x);
  e[1] = static_cast<int>(y);
  e[2] = static_cast<int>(z);
}
#define GRAPE_BOX(err, ext, el, x, y, z) if (!box_ok(err, ext, el, x, y, z)) {} else
#define GRAPE_EXT(e, x, y, z) set_ext(e, x, y, z);
#else
#define GRAPE_BOX(err, ext, el, x, y, z)
#define GRAPE_EXT(e, x, y, z)
#endif

template <int MODE>
struct ModeTraits {
  static constexpr bool kNorm = (MODE == NORM || MODE == NORMST);
  static constexpr bool kAMn = (kNorm || MODE == AGGREGATE);
  static constexpr bool kB3d = kNorm;
};

template <int BN, int STAGES, int EXTRA = 0, int BCOLS = BN>
struct Smem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BCOLS * kBK * 2;   // 0: one tile per stage serves as A and B
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kBarOff = STAGES * kStage;
  // after the barriers, on a 1024-byte boundary (128-byte-swizzled TMA boxes live there)
  static constexpr int kExtraOff = ((kBarOff + 512 + 1023) / 1024) * 1024;
  static constexpr int kBytes = kExtraOff + EXTRA + 1024;  // + alignment slack
  static_assert(kStage % 1024 == 0 && kExtraOff % 1024 == 0, "swizzled tiles need 1024-byte alignment");
};

// NORMST: one staging box per epilogue warp for its 32 rows x 64 columns of R_i in bf16.
constexpr int kRBox = 32 * 128;
// BACKPROJ: two W tiles (128 rows x 128 fp32 columns, as four 128B-swizzled boxes of
// 32 columns) so the TMA load of the next tile's W overlaps this tile's update.
constexpr int kBnBack = 128;
constexpr int kWBox = kBM * 128;                 // one 32-column box: 16 KB
constexpr int kWTile = (kBnBack / 32) * kWBox;   // 64 KB
template <int MODE>
struct ModeExtra {
  static constexpr int kBytes = (MODE == BACKPROJ) ? 2 * kWTile : (MODE == NORMST) ? kEpiWarps * kRBox : 0;
};
// GHOST stages hold the 128-token blocks a and b of a sample (one block when a == b),
// whose Gram block X_a X_b^T the stage's MMAs accumulate.
template <int MODE, int BN, int STAGES>
using SmemOf = Smem<BN, STAGES, ModeExtra<MODE>::kBytes, BN>;

// GHOST: the pairs of token blocks (a, b), a <= b, of one (sample, layer) tile, in order;
// every other mode has one round per tile.
struct GhostPairs {
  int a = 0, b = 0;
  __device__ __forceinline__ void next(int nb) {
    if (++b == nb) b = ++a;
  }
};
__device__ __forceinline__ int ghost_rounds(int nb) { return nb * (nb + 1) / 2; }

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

struct TileCoord {
  int g, m_t, n_t, s_t, kb0, kb1;
};

__device__ __forceinline__ TileCoord decode_tile(const GroupParams& p, int tile, int mode) {
  TileCoord c;
  int g = 0;
  while (g + 1 < p.n_layers && tile >= p.lay[g + 1].tiles_begin) ++g;
  const GroupLayer& L = p.lay[g];
  int t = tile - L.tiles_begin;
  c.g = g;
  c.n_t = t % L.nt;
  t /= L.nt;
  c.m_t = t % L.mt;
  c.s_t = t / L.mt;
  c.kb0 = 0;
  c.kb1 = L.kblocks;
  (void)mode;
  return c;
}

// Persistent: CTA b handles tiles b, b + gridDim.x, ...  The shared-memory stage ring
// (index `it` counts k-blocks over all of this CTA's tiles) runs across tile
// boundaries, and two TMEM accumulators let the epilogue of one tile overlap the
// loads and MMAs of the next.
template <int MODE, int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ GroupParams p) {
  using T = ModeTraits<MODE>;
  using S = SmemOf<MODE, BN, STAGES>;
  // GHOST keeps two accumulators per tile (Gout Gout^T and AP AP^T), both K-major products
  constexpr uint32_t kAccCols = (MODE == GHOST) ? 2 * BN : BN;
  constexpr uint32_t kTmemCols = 2 * kAccCols;
  constexpr uint32_t kIdesc = (MODE == GHOST) ? ptx::idesc_bf16(kBM, BN, false, false)
                                              : ptx::idesc_bf16(kBM, BN, T::kAMn, true);
  static_assert(MODE != GHOST || BN == kBM, "a Gram tile is 128 x 128");
  static_assert(BN % 128 == 0, "each epilogue warp takes BN/2 columns in 64-column loads");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* accfull = empty + STAGES;       // [2]
  uint64_t* accempty = accfull + 2;         // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 2);
  float* red = reinterpret_cast<float*>(tmem_slot + 2);   // [2][kEpiWarps]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + 2 * kEpiWarps);
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + S::kBarOff + 448);   // BACKPROJ [2]
  uint64_t* wfree = wfull + 2;                                              // BACKPROJ [2]
  static_assert(2 * STAGES * 8 + 4 * 8 + 8 + 2 * kEpiWarps * 4 + 4 <= 448, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitLimitNs, abort_flag);
  };
  ptx::griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&accfull[b], 1);
      ptx::mbar_init(&accempty[b], kEpiWarps);
      ptx::mbar_init(&wfull[b], 1);
      ptx::mbar_init(&wfree[b], 1);
    }
    ptx::fence_mbar_init();
    for (int g = 0; g < p.n_layers; ++g) {
      ptx::prefetch_tmap(&p.mapA[g]);
      ptx::prefetch_tmap(&p.mapB[g]);
      if (MODE == BACKPROJ) ptx::prefetch_tmap(&p.mapW[g]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (producer_of(warp) >= 0) {
    // ---------------- TMA producers ----------------
    constexpr int kNP = RingProducers<STAGES>::kCount;
    static_assert(kNP >= 1 && kNP <= STAGES, "parity waits need at most STAGES producers");
    if (lane == 0 && producer_of(warp) < kNP) {
      const int pi = producer_of(warp);
      // A and Gout stream once per use; P, AP and dR are re-read by other tiles or
      // by the next phase, so they are kept in L2 preferentially.
      // (NORMST: neither AP nor Gout is read again after this kernel, and its R stores
      // share the cache, so both load with the normal priority)
      const uint64_t polA = (MODE == PROJECT || MODE == AGGREGATE || MODE == BACKPROJ)
                                ? ptx::policy_evict_first()
                                : (MODE == NORMST) ? ptx::policy_evict_normal() : ptx::policy_evict_last();
      const uint64_t polB = (MODE == AGGREGATE) ? ptx::policy_evict_first()
                            : (MODE == NORMST) ? ptx::policy_evict_normal() : ptx::policy_evict_last();
      auto load_a = [&](const TileCoord& c, int kb, int s) {
        uint8_t* sa = smem + s * S::kStage;
        const CUtensorMap* mapA = &p.mapA[c.g];
        const int kk = kb * kBK;
        if (MODE == PROJECT || MODE == BACKPROJ) {
          GRAPE_BOX(p.err, p.extA[c.g], 2, kk, c.m_t * kBM, 0)
          ptx::tma_load_2d_hint(sa, mapA, &full[s], kk, c.m_t * kBM, MODE == BACKPROJ ? polB : polA);
        } else if (T::kNorm) {
#pragma unroll
          for (int q = 0; q < kBM / 64; ++q)
            GRAPE_BOX(p.err, p.extA[c.g], 2, c.m_t * kBM + 64 * q, kk, c.s_t)
            ptx::tma_load_3d_hint(sa + q * 8192, mapA, &full[s], c.m_t * kBM + 64 * q, kk, c.s_t, polA);
        } else {
#pragma unroll
          for (int q = 0; q < kBM / 64; ++q)
            GRAPE_BOX(p.err, p.extA[c.g], 2, c.m_t * kBM + 64 * q, kk, 0)
            ptx::tma_load_2d_hint(sa + q * 8192, mapA, &full[s], c.m_t * kBM + 64 * q, kk, polA);
        }
      };
      auto load_b = [&](const TileCoord& c, int kb, int s) {
        uint8_t* sb = smem + s * S::kStage + S::kABytes;
        const CUtensorMap* mapB = &p.mapB[c.g];
        const int kk = kb * kBK;
#pragma unroll
        for (int q = 0; q < BN / 64; ++q) {
          if (T::kB3d)
            GRAPE_BOX(p.err, p.extB[c.g], 2, c.n_t * BN + 64 * q, kk, c.s_t)
            ptx::tma_load_3d_hint(sb + q * 8192, mapB, &full[s], c.n_t * BN + 64 * q, kk, c.s_t, polB);
          else
            GRAPE_BOX(p.err, p.extB[c.g], 2, c.n_t * BN + 64 * q, kk, 0)
            ptx::tma_load_2d_hint(sb + q * 8192, mapB, &full[s], c.n_t * BN + 64 * q, kk, polB);
        }
      };
      auto load_w = [&](const TileCoord& c, int wb) {
        uint8_t* wbuf = smem + S::kExtraOff + wb * kWTile;
        ptx::mbar_arrive_expect_tx(&wfull[wb], kWTile);
#pragma unroll
        for (int q = 0; q < kBnBack / 32; ++q)
          GRAPE_BOX(p.err, p.extW[c.g], 4, c.n_t * kBnBack + 32 * q, c.m_t * kBM, 0)
          ptx::tma_load_2d_hint(wbuf + q * kWBox, &p.mapW[c.g], &wfull[wb], c.n_t * kBnBack + 32 * q,
                                c.m_t * kBM, polA);
      };

      // The operand that predates the step -- A (PROJECT) or Gout (NORM, AGGREGATE) --
      // of a producer's first stage loads before waiting for the previous kernel of the
      // step; P, AP and dR are written earlier in this step and load after the wait.
      // Producer 0 also loads W of the first tile (BACKPROJ) before it, and every W tile.
      bool waited = false;
      auto ensure_wait = [&]() {
        if (!waited) {
          ptx::griddep_wait();
          waited = true;
        }
      };
      uint32_t wissued = 0;
      if (MODE == BACKPROJ && pi == 0 && static_cast<int>(blockIdx.x) < p.total_tiles) {
        load_w(decode_tile(p, blockIdx.x, MODE), 0);
        wissued = 1;
      }

      uint32_t it = 0, tcp = 0, issued_end = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x, ++tcp) {
        const TileCoord c = decode_tile(p, tile, MODE);
        const int rounds = (MODE == GHOST) ? ghost_rounds(p.lay[c.g].nb) : 1;
        GhostPairs gp_;
        if (MODE == BACKPROJ && pi == 0 && tcp > 0) {
          // this tile's W into buffer tcp & 1, once the store of the tile before last
          // has finished reading it
          const int wb = tcp & 1;
          const uint32_t wuse = tcp >> 1;
          if (wuse > 0 && !wait(&wfree[wb], (wuse - 1) & 1)) {
            atomicOr(p.err, kErrTimeoutProducer);
            break;
          }
          load_w(c, wb);
          ++wissued;
        }
        for (int round = 0; ok && round < rounds; ++round) {
        if (MODE == GHOST && round > 0) gp_.next(p.lay[c.g].nb);
        for (int kb = c.kb0; kb < c.kb1; ++kb, ++it) {
          if (static_cast<int>(it % kNP) != pi) continue;
          const int s = it % STAGES;
          const uint32_t use = it / STAGES;
          if (use > 0 && !wait(&empty[s], (use - 1) & 1)) {
            atomicOr(p.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          if (MODE == GHOST) {
            // token blocks a and b of the sample (rows past T: zeros), one box when a == b;
            // Gout's k-blocks first, then AP's (after the wait)
            const int kf = p.lay[c.g].kfirst;
            const int na = gp_.a == gp_.b ? 1 : 2;
            ptx::mbar_arrive_expect_tx(&full[s], na * S::kABytes);
            uint8_t* st_ = smem + s * S::kStage;
            if (kb >= kf) ensure_wait();
            const CUtensorMap* map = kb < kf ? &p.mapB[c.g] : &p.mapA[c.g];
            const int x = (kb < kf ? kb : kb - kf) * kBK;
            const uint64_t pol = kb < kf ? polB : polA;
            for (int k = 0; k < na; ++k) {
              const int y = (k == 0 ? gp_.a : gp_.b) * kBM;
              if (kb < kf)
                GRAPE_BOX(p.err, p.extB[c.g], 2, x, y, c.s_t)
                ptx::tma_load_3d_hint(st_ + k * S::kABytes, map, &full[s], x, y, c.s_t, pol);
              else
                GRAPE_BOX(p.err, p.extA[c.g], 2, x, y, c.s_t)
                ptx::tma_load_3d_hint(st_ + k * S::kABytes, map, &full[s], x, y, c.s_t, pol);
            }
            issued_end = it + 1;
            continue;
          }
          ptx::mbar_arrive_expect_tx(&full[s], S::kStage);
          if (MODE == PROJECT) {
            load_a(c, kb, s);
            ensure_wait();
            load_b(c, kb, s);
          } else if (T::kNorm || MODE == AGGREGATE) {
            load_b(c, kb, s);
            ensure_wait();
            load_a(c, kb, s);
          } else {
            ensure_wait();
            load_a(c, kb, s);
            load_b(c, kb, s);
          }
          issued_end = it + 1;
        }
        }
      }
      if (*abort_flag) {
        // leave none of this thread's TMA loads in flight into this CTA's shared memory
        for (uint32_t k = issued_end > STAGES ? issued_end - STAGES : 0; k < issued_end; ++k)
          if (static_cast<int>(k % kNP) == pi)
            ptx::mbar_wait(&full[k % STAGES], (k / STAGES) & 1, kDrainLimitNs);
        if (MODE == BACKPROJ && pi == 0)
          for (uint32_t k = wissued > 2 ? wissued - 2 : 0; k < wissued; ++k)
            ptx::mbar_wait(&wfull[k & 1], (k >> 1) & 1, kDrainLimitNs);
      }
    }
  } else if (warp == 1) {
    // ---------------- UMMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.total_tiles; tile += gridDim.x) {
        const TileCoord c = decode_tile(p, tile, MODE);
        const int rounds = (MODE == GHOST) ? ghost_rounds(p.lay[c.g].nb) : 1;
        GhostPairs gp_;
        for (int round = 0; ok && round < rounds; ++round, ++tc) {
        if (MODE == GHOST && round > 0) gp_.next(p.lay[c.g].nb);
        const int b = tc & 1;
        const uint32_t use = tc >> 1;
        if (use > 0 && !wait(&accempty[b], (use - 1) & 1)) {
          atomicOr(p.err, kErrTimeoutMma);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + b * kAccCols;
        for (int kb = c.kb0; kb < c.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!wait(&full[s], ph)) {
            atomicOr(p.err, kErrTimeoutMma);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_base = ptx::smem_u32(smem + s * S::kStage);
          const uint32_t b_base = a_base + S::kABytes;
          if (MODE == GHOST) {
            // the stage's blocks X_a, X_b (128 rows, 64 K-major columns each; X_b is X_a
            // when a == b): D += X_a X_b^T, into the Gout Gram block (first accumulator) or
            // the AP Gram block (second)
            const int kf = p.lay[c.g].kfirst;
            const bool second = kb >= kf;
            const uint32_t dd = d + (second ? BN : 0);
            const int kstart = second ? kf : c.kb0;
            const uint32_t bx = gp_.a == gp_.b ? a_base : a_base + S::kABytes;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              ptx::umma_bf16(dd, ptx::desc_sw128(a_base + k * 32, 16, 1024), ptx::desc_sw128(bx + k * 32, 16, 1024),
                             kIdesc, (kb > kstart || k > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              // K-major: the next 16 elements are 32 bytes further along the swizzled row;
              // M/N-major: the next 16 K-rows are 16 x 128 bytes further.
              const uint64_t ad = T::kAMn ? ptx::desc_sw128(a_base + k * 2048, 8192, 1024)
                                          : ptx::desc_sw128(a_base + k * 32, 16, 1024);
              const uint64_t bd = ptx::desc_sw128(b_base + k * 2048, 8192, 1024);
              ptx::umma_bf16(d, ad, bd, kIdesc, (kb > c.kb0 || k > 0) ? 1u : 0u);
            }
          }
          ptx::umma_commit(&empty[s]);
        }
        ptx::umma_commit(&accfull[b]);
        }
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // ---------------- epilogue: warps 2..9 ----------------
    // Warp w reads TMEM lanes 32*(w%4).. (its lane quarter, a hardware rule) and half
    // h = (w-2)/4 of the accumulator's columns, 64 columns per load.
    const int ew = warp - 2;                      // 0..7
    const int q = warp & 3;                       // TMEM lanes 32q .. 32q+31
    const int h = ew >> 2;                        // column half
    const int row = q * 32 + lane;                // accumulator row of this thread
    constexpr int kHalf = BN / 2;
    // The epilogue warps walk every tile even after a failed wait (their waits then
    // return at once), so the named barriers below are always reached by all of them.
    uint32_t tc = 0, tcount = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++tcount) {
      const TileCoord c = decode_tile(p, tile, MODE);
      const GroupLayer& L = p.lay[c.g];
      const int rounds = (MODE == GHOST) ? ghost_rounds(L.nb) : 1;
      GhostPairs gp_;
      float gsum = 0.0f;   // GHOST: this thread's share of the sample's squared norm
      for (int round = 0; round < rounds; ++round, ++tc) {
      if (MODE == GHOST && round > 0) gp_.next(L.nb);
      const int b = tc & 1;
      const uint32_t use = tc >> 1;
      const bool got = wait(&accfull[b], use & 1);
      if (!got) atomicOr(p.err, kErrTimeoutEpilogue);
      ptx::tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kAccCols + h * kHalf;
      const int col0 = c.n_t * BN + h * kHalf;    // first output column of this warp
      const bool have = got && c.kb1 > c.kb0;

      if (MODE == PROJECT) {
        const int m = c.m_t * kBM + row;
        __nv_bfloat16* AP = static_cast<__nv_bfloat16*>(L.out);
#pragma unroll 1
        for (int cc = 0; cc < kHalf; cc += 64) {
          float v[64];
          ptx::tmem_ld64(tbase + cc, v);
          if (have && m < L.M) {
            uint4* dst = reinterpret_cast<uint4*>(AP + static_cast<size_t>(m) * L.ldo + col0 + cc);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              dst[u] = make_uint4(pack_bf16(v[8 * u + 0], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                                  pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
          }
        }
      } else if (T::kNorm) {
        // ||R_i||^2 partial of this tile.  NORMST also stores the tile of R_i as bf16 to
        // [sample][r][d_out] (L.out): each warp stages its 32 rows x 64 columns in its own
        // box (row `lane` at 128-byte row `lane`, 16-byte unit u at u ^ (lane & 7), so the
        // eight lanes writing one unit hit distinct banks), then writes them out four rows
        // per instruction, eight lanes per row: whole 128-byte lines, where each thread
        // storing its own row would scatter 16-byte pieces over 32 lines.
        float ss = 0.0f;
        uint4* rbox = reinterpret_cast<uint4*>(smem + S::kExtraOff + ew * kRBox);
        __nv_bfloat16* Rst = static_cast<__nv_bfloat16*>(L.out);
#pragma unroll 1
        for (int cc = 0; cc < kHalf; cc += 64) {
          float v[64];
          ptx::tmem_ld64(tbase + cc, v);
#pragma unroll
          for (int j = 0; j < 64; ++j) ss = fmaf(v[j], v[j], ss);
          if (MODE == NORMST && have) {
            __syncwarp();   // the previous chunk's rows have been read out of the box
#pragma unroll
            for (int u = 0; u < 8; ++u)
              rbox[lane * 8 + (u ^ (lane & 7))] =
                  make_uint4(pack_bf16(v[8 * u + 0], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                             pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
            __syncwarp();
            const int u = lane & 7;
            __nv_bfloat16* base = Rst + (static_cast<size_t>(c.s_t) * L.M + c.m_t * kBM + q * 32) * L.ldo +
                                  col0 + cc + 8 * u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = 4 * i + (lane >> 3);
              *reinterpret_cast<uint4*>(base + static_cast<size_t>(rr) * L.ldo) = rbox[rr * 8 + (u ^ (rr & 7))];
            }
          }
        }
        if (!have) ss = 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        float* rb = red + (tc & 1) * kEpiWarps;
        if (lane == 0) rb[ew] = ss;
        epi_bar();
        // one partial slot per 128 columns of d_out (the slot layout every norm kernel
        // shares): column half `lane` of the tile is the sum over its four warps
        static_assert(!T::kNorm || BN == 256, "a norm tile is two 128-column slots");
        if (ew == 0 && lane < 2) {
          float tot = 0.0f;
#pragma unroll
          for (int k = 0; k < 4; ++k) tot += rb[4 * lane + k];
          p.partials[static_cast<size_t>(c.s_t) * p.part_stride + L.part_base + c.m_t * (2 * L.nt) +
                     2 * c.n_t + lane] = tot;
        }
      } else if (MODE == GHOST) {
        // this thread's row x 64 columns of (Gout Gram block) * (AP Gram block); an
        // off-diagonal block (a < b) stands for its transpose (b, a) too
        float ss = 0.0f;
#pragma unroll 1
        for (int cc = 0; cc < kHalf; cc += 32) {
          float y[32], x[32];
          ptx::tmem_ld32(tbase + cc, y);
          ptx::tmem_ld32(tbase + BN + cc, x);
#pragma unroll
          for (int j = 0; j < 32; ++j) ss = fmaf(x[j], y[j], ss);
        }
        if (have) gsum = fmaf(gp_.a == gp_.b ? 1.0f : 2.0f, ss, gsum);
      } else if (MODE == AGGREGATE) {
        const int m = c.m_t * kBM + row;
        float* dst = static_cast<float*>(L.out);
#pragma unroll 1
        for (int cc = 0; cc < kHalf; cc += 64) {
          float v[64];
          ptx::tmem_ld64(tbase + cc, v);
          const int n0 = col0 + cc;
          if (m < L.M) {
            float* o = dst + static_cast<size_t>(m) * L.ldo + n0;
            if (n0 + 64 <= L.N) {
#pragma unroll
              for (int u = 0; u < 16; ++u)
                reinterpret_cast<float4*>(o)[u] =
                    have ? make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3])
                         : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
              for (int j = 0; j < 64 && n0 + j < L.N; ++j) o[j] = have ? v[j] : 0.0f;
            }
          }
        }
      } else {  // BACKPROJ: W -= lr * P dR on the W tile in shared memory, then TMA store
        const bool wgot = wait(&wfull[b], use & 1);
        if (!wgot) atomicOr(p.err, kErrTimeoutEpilogue);
        uint8_t* wbuf = smem + S::kExtraOff + b * kWTile;
        const float lr = p.lr;
#pragma unroll 1
        for (int cc = 0; cc < kHalf; cc += 64) {
          float v[64];
          ptx::tmem_ld64(tbase + cc, v);
          if (have && wgot) {
            // columns h*kHalf + cc + [0, 64): two 32-column boxes; 16-byte unit u of
            // row `row` sits at unit u ^ (row & 7) (128-byte swizzle)
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
              uint8_t* box = wbuf + ((h * kHalf + cc) / 32 + bx) * kWBox + row * 128;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                float4* w4 = reinterpret_cast<float4*>(box + ((u ^ (row & 7)) * 16));
                float4 x = *w4;
                const int j = bx * 32 + u * 4;
                x.x = fmaf(-lr, v[j + 0], x.x);
                x.y = fmaf(-lr, v[j + 1], x.y);
                x.z = fmaf(-lr, v[j + 2], x.z);
                x.w = fmaf(-lr, v[j + 3], x.w);
                *w4 = x;
              }
            }
          }
        }
        ptx::fence_proxy_async_smem();   // the W tile is next read by the TMA store
        epi_bar();
        if (ew == 0 && lane == 0) {
          if (have && wgot) {
#pragma unroll
            for (int q2 = 0; q2 < kBnBack / 32; ++q2)
              GRAPE_BOX(p.err, p.extW[c.g], 4, c.n_t * kBnBack + 32 * q2, c.m_t * kBM, 0)
              ptx::tma_store_2d(&p.mapW[c.g], wbuf + q2 * kWBox, c.n_t * kBnBack + 32 * q2, c.m_t * kBM);
            ptx::bulk_commit_group();
            ptx::bulk_wait_group_read0();
          }
          ptx::mbar_arrive(&wfree[b]);
        }
      }
      // this accumulator may be overwritten by the round after next
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&accempty[b]);
      }
      if (MODE == GHOST) {
        // the sample's squared norm for this layer: the sum over the 8 warps, in order
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
        float* rb = red + (tcount & 1) * kEpiWarps;
        if (lane == 0) rb[ew] = gsum;
        epi_bar();
        if (ew == 0) {
          // the layer's first slot holds the norm, its other slots zero (the clip sums them all)
          float* slot = p.partials + static_cast<size_t>(c.s_t) * p.part_stride + L.part_base;
          for (int k = lane; k < L.slots; k += 32) {
            float tot = 0.0f;
            if (k == 0)
#pragma unroll
              for (int w2 = 0; w2 < kEpiWarps; ++w2) tot += rb[w2];
            slot[k] = tot;
          }
        }
      }
    }
  }

  if (MODE == BACKPROJ && warp == 2 && lane == 0) ptx::bulk_wait_group0();   // W stores complete
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- back-projection with P resident in tensor memory -------------------------------
// W -= lr P dR in tiles of 128 rows x 128 columns of W with K = r, with the A operand
// (the 128 x r block of P under the tile) read by the MMA from TMEM instead of shared
// memory.  The layers of a launch are cut into consecutive spans of at least four
// tiles per CTA (a single layer when it is that large).  Span by span, each CTA takes a
// contiguous range of the span's T tiles (numbered layer by layer, row block by row
// block): T / grid of them, one more for T % grid of the CTAs, with the CTAs that take
// the extra tile rotating from span to span, so the whole launch is balanced to within
// one tile and all CTAs work on the same span at once (its P and dR stay in L2).  A
// work unit is the part of a CTA's range in one 128-row block: the block of P is
// written into TMEM once per unit, and per tile only dR (r x 128 bf16, from L2) and W
// (from DRAM) stream through shared memory, which holds nothing but those streams.
// Next to tc_gemm_kernel<BACKPROJ>, which loads P with every tile, this moves 192
// instead of 320 bytes from L2 into the SM per 64 bytes of W read, with the same bytes
// in flight.
//
// The block of P comes by TMA in 64-column chunks (128 rows x 64 bf16, 16 KB, rows past
// d_in zero-filled) through the dR ring: the ring holds, in order, the chunks of unit 0,
// its dR stages, the chunks of unit 1, its dR stages, and so on, so a unit's chunks are
// loaded while the previous unit's last dR stages are consumed.  The writers of a unit's
// block wait until the MMAs of the previous unit are done, which keeps the ring's parity
// waits sound: a consumer waits for a ring position only once the position DRS earlier
// has been loaded (an mbarrier parity wait for phase k returns at once while phase k - 1
// is still open).
//
// W streams through a ring of 32-column boxes (128 rows x 32 fp32, 16 KB) that runs
// ahead of the tiles; each epilogue warp updates its 32 rows of a box in shared memory
// and stores them with a TMA tile store; a box's slot is reloaded once its four row
// quarters have been read out.
//
// TMEM: two 128 x 128 fp32 accumulators (columns 0..255) and the P block of r/2 columns
// (lane = row of P, two bf16 of consecutive k per 32-bit column).
// Warps: 0 loads the ring, P chunks and dR (both written earlier in the step, after
// griddepcontrol.wait); 1 owns TMEM and issues the MMAs; 2-9 are the epilogue (warp w:
// lane quarter w % 4, column half (w - 2) / 4); 10 loads W (written by the previous
// step, whose work every step's first, ordinary launch waits for, so its loads start at
// once); 11-14 write P into TMEM (warp w: lane quarter w % 4, one row of P per thread,
// read from its chunk in shared memory).
struct BptLayer {
  int tiles_begin;   // first tile of this layer in its span
  int M;             // rows of W and of P (d_in)
  int mt, nt;        // 128-row blocks of W, 128-column tiles of W
};

struct BptParams {
  CUtensorMap mapP[kMaxGroup];    // P: bf16 d_in x r, boxes of 64 columns x 128 rows
  CUtensorMap mapDR[kMaxGroup];   // dR: bf16 r x d_out, boxes of 64 x 64
  CUtensorMap mapW[kMaxGroup];    // W: fp32 d_in x d_out, load boxes of 32 columns x 128 rows
  CUtensorMap mapWs[kMaxGroup];   // W, store boxes of 32 columns x 32 rows
  BptLayer lay[kMaxGroup];
  int n_layers;
  int n_spans;
  int span_first[kMaxGroup + 1];   // first layer of each span; span_first[n_spans] = n_layers
  int span_tiles[kMaxGroup];
  int span_rot[kMaxGroup];         // CTA b takes the range of position (b + rot) % grid
  int r;
  float lr;
  int* err;
#ifdef GRAPE_CHECKED
  int extP[kMaxGroup][3];
  int extDR[kMaxGroup][3];
  int extW[kMaxGroup][3];
#endif
};

struct BptUnit {
  int g, m_t, n0, n1;   // layer in the launch, row block (a sample in the norm kernel), tiles [n0, n1)
};

// One position's units in order: span by span, its range of the span's tiles cut at
// the ends of layers and of row blocks.  A position is a CTA (back-projection) or a
// group of CTAs that walk the same tiles (norms); `npos` positions share each span.
// The params need n_spans, span_first, span_tiles, span_rot and per layer
// tiles_begin and nt.
struct SpanWalk {
  int sp, g, cur, t1;   // span, layer, next tile of the span, end of this position's range in it
  int npos, pos;
  template <class Pm>
  __device__ __forceinline__ void range(const Pm& p) {
    const int T = p.span_tiles[sp];
    const int base = T / npos, extra = T % npos;
    const int b = (pos + p.span_rot[sp]) % npos;
    cur = b * base + min(b, extra);
    t1 = cur + base + (b < extra ? 1 : 0);
    g = p.span_first[sp];
  }
  template <class Pm>
  __device__ __forceinline__ void start(const Pm& p, int npos_, int pos_) {
    npos = npos_;
    pos = pos_;
    sp = 0;
    range(p);
  }
  template <class Pm>
  __device__ __forceinline__ void start(const Pm& p) {
    start(p, static_cast<int>(gridDim.x), static_cast<int>(blockIdx.x));
  }
  // The next unit; false when the position has none left.
  template <class Pm>
  __device__ __forceinline__ bool next(const Pm& p, BptUnit& x) {
    while (cur >= t1) {
      if (++sp >= p.n_spans) return false;
      range(p);
    }
    while (g + 1 < p.span_first[sp + 1] && cur >= p.lay[g + 1].tiles_begin) ++g;
    const auto& L = p.lay[g];
    const int t = cur - L.tiles_begin;
    x.g = g;
    x.m_t = t / L.nt;
    x.n0 = t % L.nt;
    x.n1 = min(L.nt, x.n0 + (t1 - cur));
    cur += x.n1 - x.n0;
    return true;
  }
};
using BptWalk = SpanWalk;

// DRS ring stages (dR, or a chunk of P) and NW W boxes in shared memory.
template <int DRS, int NW>
struct BptSmem {
  static constexpr int kDRStage = kBK * kBnBack * 2;        // 64 x 128 bf16: 16 KB (a P chunk too)
  static constexpr int kDROff = 0;
  static constexpr int kWOff = DRS * kDRStage;
  static constexpr int kBarOff = kWOff + NW * kWBox;
  static constexpr int kBytes = kBarOff + 512 + 1024;       // barriers + alignment slack
  static_assert(kBytes <= 232448, "exceeds the shared memory of a CTA");
};
constexpr int kBptThreads = 32 * 15;
constexpr int kBptWProducer = 10;
constexpr int kBptPWriter0 = 11;    // warps 11..14

__device__ __forceinline__ void bpt_writer_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
constexpr uint32_t kBptTmemCols = 512;
constexpr int kBptDRS = 6;
constexpr int kBptNW = 8;

// PK = r / 64 k-blocks: the P block takes PK * 32 TMEM columns.
template <int PK>
__global__ void __launch_bounds__(kBptThreads, 1) tc_backproj_tmem_kernel(const __grid_constant__ BptParams p) {
  constexpr int DRS = kBptDRS, NW = kBptNW;
  using S = BptSmem<DRS, NW>;
  constexpr uint32_t kIdesc = ptx::idesc_bf16(kBM, kBnBack, false, true);   // A K-major (TMEM), dR N-major
  constexpr int kBoxes = kBnBack / 32;                                     // W boxes per tile
  constexpr uint32_t kPCols = PK * 32;                                     // TMEM columns of one P block
  static_assert(2 * kBnBack + kPCols <= kBptTmemCols, "TMEM columns");
  static_assert(S::kDRStage == kBK * kBM * 2, "a P chunk fills one ring stage");
  // A slot of the W ring must only ever hold boxes of one column half, so that the four
  // warps that wait on its wfull barrier have consumed its previous use themselves: a
  // parity wait cannot tell a phase two ahead from the one behind, and a warp of the other
  // half waiting for the slot's next use would pass at once on the previous phase.
  static_assert(NW % kBoxes == 0, "W ring slots must map to one box position of a tile");
  static_assert((2 + 2 * DRS + 4 + 2 * NW) * 8 + 16 <= 512, "barrier area");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + S::kBarOff);   // the P block is in TMEM
  uint64_t* pempty = pfull + 1;                                          // its MMAs are done
  uint64_t* full = pempty + 1;
  uint64_t* empty = full + DRS;
  uint64_t* accfull = empty + DRS;     // [2]
  uint64_t* accempty = accfull + 2;    // [2]
  uint64_t* wfull = accempty + 2;      // [NW]
  uint64_t* wfree = wfull + NW;        // [NW]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfree + NW);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitLimitNs, abort_flag);
  };
  ptx::griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    ptx::mbar_init(pfull, 4);    // the four P-writing warps
    ptx::mbar_init(pempty, 1);
    for (int st = 0; st < DRS; ++st) {
      ptx::mbar_init(&full[st], 1);
      ptx::mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&accfull[b], 1);
      ptx::mbar_init(&accempty[b], kEpiWarps);
    }
    for (int sl = 0; sl < NW; ++sl) {
      ptx::mbar_init(&wfull[sl], 1);
      ptx::mbar_init(&wfree[sl], 4);   // the four row quarters of a box
    }
    ptx::fence_mbar_init();
    for (int g = 0; g < p.n_layers; ++g) {
      ptx::prefetch_tmap(&p.mapP[g]);
      ptx::prefetch_tmap(&p.mapDR[g]);
      ptx::prefetch_tmap(&p.mapW[g]);
      ptx::prefetch_tmap(&p.mapWs[g]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kBptTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_p = tmem + 2 * kBnBack;   // the P block after the two accumulators

  if (warp == 0) {
    // ---------------- the ring: each unit's chunks of P, then its dR stages ----------------
    if (lane == 0) {
      const uint64_t pol = ptx::policy_evict_last();   // dR and P are read by many units
      ptx::griddep_wait();
      uint32_t it = 0, it_issued = 0;
      bool ok = true;
      BptWalk walk;
      walk.start(p);
      BptUnit x;
      while (ok && walk.next(p, x)) {
#pragma unroll 1
        for (int c = 0; c < PK; ++c, ++it) {
          const int st = it % DRS;
          const uint32_t use = it / DRS;
          if (use > 0 && !wait(&empty[st], (use - 1) & 1)) {
            atomicOr(p.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&full[st], S::kDRStage);
          GRAPE_BOX(p.err, p.extP[x.g], 2, c * kBK, x.m_t * kBM, 0)
          ptx::tma_load_2d_hint(smem + S::kDROff + st * S::kDRStage, &p.mapP[x.g], &full[st], c * kBK, x.m_t * kBM,
                                pol);
          it_issued = it + 1;
        }
        for (int n = x.n0; ok && n < x.n1; ++n) {
#pragma unroll 1
          for (int kb = 0; kb < PK; ++kb, ++it) {
            const int st = it % DRS;
            const uint32_t use = it / DRS;
            if (use > 0 && !wait(&empty[st], (use - 1) & 1)) {
              atomicOr(p.err, kErrTimeoutProducer);
              ok = false;
              break;
            }
            uint8_t* ddst = smem + S::kDROff + st * S::kDRStage;
            ptx::mbar_arrive_expect_tx(&full[st], S::kDRStage);
#pragma unroll
            for (int h = 0; h < kBnBack / 64; ++h)
              GRAPE_BOX(p.err, p.extDR[x.g], 2, n * kBnBack + 64 * h, kb * kBK, 0)
              ptx::tma_load_2d_hint(ddst + h * 8192, &p.mapDR[x.g], &full[st], n * kBnBack + 64 * h, kb * kBK, pol);
            it_issued = it + 1;
          }
        }
      }
      if (*abort_flag)   // leave none of this thread's loads in flight into shared memory
        for (uint32_t k = it_issued > DRS ? it_issued - DRS : 0; k < it_issued; ++k)
          ptx::mbar_wait(&full[k % DRS], (k / DRS) & 1, kDrainLimitNs);
    }
  } else if (warp == kBptWProducer) {
    // ---------------- W boxes ----------------
    if (lane == 0) {
      const uint64_t pol = ptx::policy_evict_first();
      uint32_t wi = 0, w_issued = 0;
      bool ok = true;
      BptWalk walk;
      walk.start(p);
      BptUnit x;
      while (ok && walk.next(p, x)) {
        for (int n = x.n0; ok && n < x.n1; ++n) {
#pragma unroll 1
          for (int j = 0; j < kBoxes; ++j, ++wi) {
            const int sl = wi % NW;
            const uint32_t use = wi / NW;
            if (use > 0 && !wait(&wfree[sl], (use - 1) & 1)) {
              atomicOr(p.err, kErrTimeoutProducer);
              ok = false;
              break;
            }
            ptx::mbar_arrive_expect_tx(&wfull[sl], kWBox);
            GRAPE_BOX(p.err, p.extW[x.g], 4, n * kBnBack + 32 * j, x.m_t * kBM, 0)
            ptx::tma_load_2d_hint(smem + S::kWOff + sl * kWBox, &p.mapW[x.g], &wfull[sl], n * kBnBack + 32 * j,
                                  x.m_t * kBM, pol);
            w_issued = wi + 1;
          }
        }
      }
      if (*abort_flag)
        for (uint32_t k = w_issued > NW ? w_issued - NW : 0; k < w_issued; ++k)
          ptx::mbar_wait(&wfull[k % NW], (k / NW) & 1, kDrainLimitNs);
    }
  } else if (warp >= kBptPWriter0) {
    // ---------------- P into TMEM: one row of the block per thread ----------------
    const int q = warp & 3;                       // TMEM lanes 32q .. 32q+31
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int row = q * 32 + lane;                // row of the block
    // The four warps walk every unit even after a failed wait (their waits then return
    // at once), so the named barrier below is always reached by all of them.
    uint32_t ui = 0, it = 0;
    bool ok = true;
    BptWalk walk;
    walk.start(p);
    BptUnit x;
    for (; walk.next(p, x); ++ui) {
      if (ui > 0 && !wait(pempty, (ui - 1) & 1)) {
        atomicOr(p.err, kErrTimeoutProducer);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);   // tcgen05.st is warp-wide: one decision per warp
      ptx::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < PK; ++c, ++it) {
        const int st = it % DRS;
        if (!wait(&full[st], (it / DRS) & 1)) {
          atomicOr(p.err, kErrTimeoutProducer);
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
        // row `row` of the chunk: 16-byte unit uu at uu ^ (row & 7) (128-byte swizzle)
        const uint4* src = reinterpret_cast<const uint4*>(smem + S::kDROff + st * S::kDRStage + row * 128);
        uint32_t v[32];
#pragma unroll
        for (int uu = 0; uu < 8; ++uu) {
          const uint4 w = src[uu ^ (row & 7)];
          v[4 * uu] = w.x;
          v[4 * uu + 1] = w.y;
          v[4 * uu + 2] = w.z;
          v[4 * uu + 3] = w.w;
        }
        bpt_writer_bar();   // all four warps have read the chunk: its slot is free
        if (warp == kBptPWriter0 && lane == 0) ptx::mbar_arrive(&empty[st]);
        if (ok) ptx::tmem_st32(tmem_p + lane_base + c * 32, v);
      }
      it += (x.n1 - x.n0) * PK;   // the unit's dR stages
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) ptx::mbar_arrive(pfull);
    }
  } else if (warp == 1) {
    // ---------------- UMMA issuer ----------------
    if (lane == 0) {
      uint32_t ui = 0, ti = 0, it = 0;
      bool ok = true;
      BptWalk walk;
      walk.start(p);
      BptUnit x;
      for (; ok && walk.next(p, x); ++ui) {
        it += PK;   // the unit's chunks of P, consumed by the TMEM writers
        if (!wait(pfull, ui & 1)) {
          atomicOr(p.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a0 = tmem_p;
        for (int n = x.n0; ok && n < x.n1; ++n, ++ti) {
          const int b = ti & 1;
          const uint32_t use = ti >> 1;
          if (use > 0 && !wait(&accempty[b], (use - 1) & 1)) {
            atomicOr(p.err, kErrTimeoutMma);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem + b * kBnBack;
#pragma unroll 1
          for (int kb = 0; kb < PK; ++kb, ++it) {
            const int st = it % DRS;
            if (!wait(&full[st], (it / DRS) & 1)) {
              atomicOr(p.err, kErrTimeoutMma);
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t b_base = ptx::smem_u32(smem + S::kDROff + st * S::kDRStage);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)   // 16 k per MMA: 8 TMEM columns of A
              ptx::umma_bf16_tmem_a(d, a0 + kb * 32 + k * 8, ptx::desc_sw128(b_base + k * 2048, 8192, 1024),
                                    kIdesc, (kb > 0 || k > 0) ? 1u : 0u);
            ptx::umma_commit(&empty[st]);
          }
          ptx::umma_commit(&accfull[b]);
        }
        ptx::umma_commit(pempty);   // the unit's MMAs, the last readers of the P block
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 ----------------
    const int ew = warp - 2;
    const int q = warp & 3;          // TMEM lanes (rows) 32q .. 32q+31
    const int h = ew >> 2;           // column half of the tile: W boxes 2h, 2h+1
    const int row = q * 32 + lane;
    const float lr = p.lr;
    uint32_t ti = 0;
    BptWalk walk;
    walk.start(p);
    BptUnit x;
    while (walk.next(p, x)) {
      for (int n = x.n0; n < x.n1; ++n, ++ti) {
        const int b = ti & 1;
        const bool got = wait(&accfull[b], (ti >> 1) & 1);
        if (!got) atomicOr(p.err, kErrTimeoutEpilogue);
        ptx::tc_fence_after();
#pragma unroll 1
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * h + jj;
          const uint32_t wi = ti * kBoxes + j;
          const int sl = wi % NW;
          const bool wgot = wait(&wfull[sl], (wi / NW) & 1);
          if (!wgot) atomicOr(p.err, kErrTimeoutEpilogue);
          float v[32];
          ptx::tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kBnBack + j * 32, v);
          uint8_t* box = smem + S::kWOff + sl * kWBox;
          const bool act = got && wgot;
          if (act) {
            // row `row` of the box: 16-byte unit uu at uu ^ (row & 7) (128-byte swizzle)
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {
              float4* w4 = reinterpret_cast<float4*>(box + row * 128 + ((uu ^ (row & 7)) * 16));
              float4 w = *w4;
              w.x = fmaf(-lr, v[4 * uu + 0], w.x);
              w.y = fmaf(-lr, v[4 * uu + 1], w.y);
              w.z = fmaf(-lr, v[4 * uu + 2], w.z);
              w.w = fmaf(-lr, v[4 * uu + 3], w.w);
              *w4 = w;
            }
            ptx::fence_proxy_async_smem();   // the rows are next read by the TMA store
          }
          __syncwarp();
          if (lane == 0) {
            // (a row quarter wholly past the last row of W has nothing to store)
            if (act && x.m_t * kBM + q * 32 < p.lay[x.g].M) {
              GRAPE_BOX(p.err, p.extW[x.g], 4, n * kBnBack + 32 * j, x.m_t * kBM + q * 32, 0)
              ptx::tma_store_2d(&p.mapWs[x.g], box + q * 32 * 128, n * kBnBack + 32 * j, x.m_t * kBM + q * 32);
              ptx::bulk_commit_group();
              ptx::bulk_wait_group_read0();
            }
            ptx::mbar_arrive(&wfree[sl]);
          }
        }
        // this accumulator may be overwritten by the tile after next
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&accempty[b]);
      }
    }
    if (lane == 0) ptx::bulk_wait_group0();   // this warp's W stores complete
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kBptTmemCols);
  }
}

// ---- per-sample norms and stored R_i with (A_i P)^T resident in tensor memory -------
// R_i = (A_i P)^T Gout_i in tiles of 128 rows (a block of the r projection rows) x 256
// columns of d_out with K = T, the A operand -- the 128 x T block of (A_i P)^T -- read
// by the MMA from TMEM.  The mr = r / 128 row blocks of a sample run side by side on mr
// CTAs (a group): CTA b is row block b % mr of group b / mr.  The groups split the
// launch's column tiles (layer, sample, 256 columns of d_out, in that order) into
// contiguous ranges balanced to within one tile, and the CTAs of a group walk the same
// column tiles at the same pace, so a Gout tile is read from DRAM once and from L2 by
// the mr SMs.  A work unit is the part of a range in one sample: its block of
// (A_i P)^T enters TMEM once, and per tile only Gout (T x 256 bf16) streams through
// shared memory.  tc_gemm_kernel<NORMST> moves 128 x T of AP and T x 256 of Gout from L2
// per 128 x 256 tile; this kernel moves the Gout part alone, 512 T instead of 768 T
// bytes per 65536 T flops, and its MMAs, with A from TMEM, issue faster than that
// kernel's with both operands in shared memory.  Every tile's R_i is stored (bf16,
// [sample][r][d_out]) for the stored aggregation.
//
// A unit's block enters TMEM in 64-token chunks, loaded by TMA as two 64-token x 64-row
// boxes of AP (tokens past T zero-filled) through the same ring of stages as Gout: the
// ring holds, in order, the chunks of unit 0, its Gout stages, the chunks of unit 1, its
// Gout stages, and so on, so a unit's chunks load while the previous unit's last Gout
// stages are consumed, and the ring keeps all the shared memory that the R staging
// leaves.  Warps 10-13 read the chunks out of shared memory transposed (thread = row of
// (A_i P)^T, two tokens per 32-bit column) and store them with tcgen05.st.  Gout tokens
// past T are zero-filled too.
//
// TMEM: one 128 x 256 fp32 accumulator (columns 0..255) and the block of (A_i P)^T
// (columns 256..511: T <= 512).  With one accumulator the MMAs of a tile wait until the
// epilogue has loaded the previous tile into registers, which it does first, before any
// other work on it.  The writers of a unit's block wait until the MMAs of the previous
// unit are done, which is also what keeps the shared ring's parity waits sound.  An
// mbarrier parity wait for phase k of a slot returns at once while phase k - 1 is still
// open, so a consumer may wait for a ring position only once the position NS earlier
// has been loaded.  The MMAs' positions follow their unit's chunks, which the writers
// have consumed; the writers' positions follow the previous unit's Gout stages, which
// the MMAs have consumed.  (With a second block the writers would run a unit ahead of
// the MMAs and wait on slots whose previous Gout stage had not been loaded yet.)
//
// Warps: 0 issues the ring's loads (after griddepcontrol.wait: AP is written earlier
// in the step); 1 owns TMEM and issues the MMAs; 2-9 are the epilogue (warp w: lane
// quarter w % 4, 128-column half (w - 2) / 4), which sums the squares of each half into
// its partial slot and writes the tile of R_i; 10-13 write the chunks into TMEM.
constexpr int kNtBN = 256;

struct NtLayer {
  int tiles_begin;   // first column tile of this layer in its span
  int nt;            // 256-column tiles of d_out
  int d_out;
  int part_base;     // first partial slot of this layer
  __nv_bfloat16* Rst;   // R_l as [B][r][d_out] bf16
};

struct NtParams {
  CUtensorMap mapG[kMaxGroup];    // Gout: bf16 (d_out, T, B), boxes of 64 x 64 x 1
  CUtensorMap mapAP[kMaxGroup];   // AP: bf16 (r, T, B), boxes of 64 x 64 x 1
  NtLayer lay[kMaxGroup];
  int n_layers;
  int n_spans;
  int span_first[kMaxGroup + 1];
  int span_tiles[kMaxGroup];
  int span_rot[kMaxGroup];
  int r;
  int mr;        // 128-row blocks of r: CTAs per group
  int groups;
  int kblocks;   // 64-token chunks: ceil(T / 64)
  int part_stride;
  float* partials;
  int* err;
#ifdef GRAPE_CHECKED
  int extG[kMaxGroup][3];
  int extAP[kMaxGroup][3];
#endif
};

struct NtSmem {
  static constexpr int kStage = kBK * kNtBN * 2;   // 64 tokens x 256 columns of Gout: 32 KB
  static constexpr int kAStage = kBK * kBM * 2;    // a chunk, 64 tokens x 128 rows of AP: 16 KB
  static constexpr int kStages = 6;
  static constexpr int kRBoxOff = kStages * kStage;
  static constexpr int kBarOff = kRBoxOff + kEpiWarps * kRBox;
  static constexpr int kBytes = kBarOff + 512 + 1024;   // barriers + alignment slack
  static_assert(kBytes <= 232448, "exceeds the shared memory of a CTA");
};
constexpr int kNtThreads = 32 * 14;
constexpr int kNtAWriter0 = 10;   // warps 10..13
constexpr uint32_t kNtTmemCols = 512;

__device__ __forceinline__ void nt_writer_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

__global__ void __launch_bounds__(kNtThreads, 1) tc_norm_tmem_kernel(const __grid_constant__ NtParams p) {
  using S = NtSmem;
  constexpr int NS = S::kStages;
  constexpr uint32_t kIdesc = ptx::idesc_bf16(kBM, kNtBN, false, true);   // A K-major (TMEM), Gout N-major
  constexpr uint32_t kACols = 256;                                     // the block: 512 tokens at most
  static_assert(kNtBN + kACols <= kNtTmemCols, "TMEM columns");
  static_assert((2 * NS + 4) * 8 + 16 + 2 * kEpiWarps * 4 <= 512, "barrier area");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + NS;
  uint64_t* pfull = empty + NS;      // the block of (A_i P)^T is in TMEM
  uint64_t* pempty = pfull + 1;      // the block's MMAs are done
  uint64_t* accfull = pempty + 1;
  uint64_t* accempty = accfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* red = reinterpret_cast<float*>(tmem_slot + 4);   // [2][kEpiWarps]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mblk = static_cast<int>(blockIdx.x) % p.mr;
  const int group = static_cast<int>(blockIdx.x) / p.mr;
  const int kbn = p.kblocks;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitLimitNs, abort_flag);
  };
  ptx::griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int st = 0; st < NS; ++st) {
      ptx::mbar_init(&full[st], 1);
      ptx::mbar_init(&empty[st], 1);
    }
    ptx::mbar_init(pfull, 4);   // the four TMEM-writing warps
    ptx::mbar_init(pempty, 1);
    ptx::mbar_init(accfull, 1);
    ptx::mbar_init(accempty, kEpiWarps);
    ptx::fence_mbar_init();
    for (int g = 0; g < p.n_layers; ++g) {
      ptx::prefetch_tmap(&p.mapG[g]);
      ptx::prefetch_tmap(&p.mapAP[g]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kNtTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_a = tmem + kNtBN;   // the block of (A_i P)^T after the accumulator

  if (warp == 0) {
    // ---------------- the ring: each unit's chunks of AP, then its Gout stages ----------------
    if (lane == 0) {
      // Gout is read by the group's mr CTAs at about the same time, then never again;
      // AP is not read again in the step
      const uint64_t polG = ptx::policy_evict_normal();
      const uint64_t polA = ptx::policy_evict_first();
      ptx::griddep_wait();   // AP is written earlier in this step
      uint32_t it = 0, it_issued = 0;
      bool ok = true;
      SpanWalk walk;
      walk.start(p, p.groups, group);
      BptUnit x;
      auto next_slot = [&](int& st) {
        st = it % NS;
        const uint32_t use = it / NS;
        if (use > 0 && !wait(&empty[st], (use - 1) & 1)) {
          atomicOr(p.err, kErrTimeoutProducer);
          ok = false;
        }
        return ok;
      };
      while (ok && walk.next(p, x)) {
#pragma unroll 1
        for (int c = 0; c < kbn; ++c, ++it) {
          int st;
          if (!next_slot(st)) break;
          uint8_t* dst = smem + st * S::kStage;
          ptx::mbar_arrive_expect_tx(&full[st], S::kAStage);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            GRAPE_BOX(p.err, p.extAP[x.g], 2, mblk * kBM + 64 * h, c * kBK, x.m_t)
            ptx::tma_load_3d_hint(dst + h * 8192, &p.mapAP[x.g], &full[st], mblk * kBM + 64 * h, c * kBK, x.m_t,
                                  polA);
          it_issued = it + 1;
        }
        for (int n = x.n0; ok && n < x.n1; ++n) {
#pragma unroll 1
          for (int kb = 0; kb < kbn; ++kb, ++it) {
            int st;
            if (!next_slot(st)) break;
            uint8_t* dst = smem + st * S::kStage;
            ptx::mbar_arrive_expect_tx(&full[st], S::kStage);
#pragma unroll
            for (int h = 0; h < kNtBN / 64; ++h)
              GRAPE_BOX(p.err, p.extG[x.g], 2, n * kNtBN + 64 * h, kb * kBK, x.m_t)
              ptx::tma_load_3d_hint(dst + h * 8192, &p.mapG[x.g], &full[st], n * kNtBN + 64 * h, kb * kBK, x.m_t,
                                    polG);
            it_issued = it + 1;
          }
        }
      }
      if (*abort_flag)   // leave none of this thread's loads in flight into shared memory
        for (uint32_t k = it_issued > NS ? it_issued - NS : 0; k < it_issued; ++k)
          ptx::mbar_wait(&full[k % NS], (k / NS) & 1, kDrainLimitNs);
    }
  } else if (warp >= kNtAWriter0) {
    // ---------------- (A_i P)^T into TMEM: one row of the block per thread ----------------
    const int q = warp & 3;                                   // TMEM lanes 32q .. 32q+31
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int j = q * 32 + lane;                              // row of the block: column of AP
    const int box = j >> 6, u = (j & 63) >> 3, e = j & 7;     // its box, 16-byte unit and element
    // The four warps walk every unit even after a failed wait (their waits then return
    // at once), so the named barrier below is always reached by all of them.
    uint32_t ui = 0, it = 0;
    bool ok = true;
    SpanWalk walk;
    walk.start(p, p.groups, group);
    BptUnit x;
    for (; walk.next(p, x); ++ui) {
      if (ui > 0 && !wait(pempty, (ui - 1) & 1)) {
        atomicOr(p.err, kErrTimeoutProducer);
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);   // tcgen05.st is warp-wide: one decision per warp
      ptx::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kbn; ++c, ++it) {
        const int st = it % NS;
        if (!wait(&full[st], (it / NS) & 1)) {
          atomicOr(p.err, kErrTimeoutProducer);
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
        // token t of this column sits in row t of the box, 16-byte unit u ^ (t & 7)
        // (128-byte swizzle); the 32 lanes read 64 consecutive bytes of one row
        const uint8_t* col = smem + st * S::kStage + box * 8192 + e * 2;
        uint32_t v[32];
#pragma unroll
        for (int tt = 0; tt < 32; ++tt) {
          const int t0 = 2 * tt, t1 = 2 * tt + 1;
          const uint32_t lo = *reinterpret_cast<const uint16_t*>(col + t0 * 128 + ((u ^ (t0 & 7)) << 4));
          const uint32_t hi = *reinterpret_cast<const uint16_t*>(col + t1 * 128 + ((u ^ (t1 & 7)) << 4));
          v[tt] = lo | (hi << 16);
        }
        nt_writer_bar();   // all four warps have read the chunk: its slot is free
        if (warp == kNtAWriter0 && lane == 0) ptx::mbar_arrive(&empty[st]);
        if (ok) ptx::tmem_st32(tmem_a + lane_base + c * 32, v);
      }
      it += (x.n1 - x.n0) * kbn;   // the unit's Gout stages
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) ptx::mbar_arrive(pfull);
    }
  } else if (warp == 1) {
    // ---------------- UMMA issuer ----------------
    if (lane == 0) {
      uint32_t ui = 0, ti = 0, it = 0;
      bool ok = true;
      SpanWalk walk;
      walk.start(p, p.groups, group);
      BptUnit x;
      for (; ok && walk.next(p, x); ++ui) {
        it += kbn;   // the unit's chunks of AP, consumed by the TMEM writers
        if (!wait(pfull, ui & 1)) {
          atomicOr(p.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a0 = tmem_a;
        for (int n = x.n0; ok && n < x.n1; ++n, ++ti) {
          // the epilogue has the previous tile in registers
          if (ti > 0 && !wait(accempty, (ti - 1) & 1)) {
            atomicOr(p.err, kErrTimeoutMma);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int kb = 0; kb < kbn; ++kb, ++it) {
            const int st = it % NS;
            if (!wait(&full[st], (it / NS) & 1)) {
              atomicOr(p.err, kErrTimeoutMma);
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t b_base = ptx::smem_u32(smem + st * S::kStage);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)   // 16 tokens per MMA: 8 TMEM columns of A
              ptx::umma_bf16_tmem_a(tmem, a0 + kb * 32 + k * 8, ptx::desc_sw128(b_base + k * 2048, 8192, 1024),
                                    kIdesc, (kb > 0 || k > 0) ? 1u : 0u);
            ptx::umma_commit(&empty[st]);
          }
          ptx::umma_commit(accfull);
        }
        ptx::umma_commit(pempty);   // the unit's MMAs, the last readers of the block
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 ----------------
    const int ew = warp - 2;
    const int q = warp & 3;          // TMEM lanes (rows of the tile) 32q .. 32q+31
    const int h = ew >> 2;           // 128-column half of the tile
    uint4* rbox = reinterpret_cast<uint4*>(smem + S::kRBoxOff + ew * kRBox);
    const uint32_t tsrc = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 128;
    uint32_t ti = 0;
    SpanWalk walk;
    walk.start(p, p.groups, group);
    BptUnit x;
    // The epilogue warps walk every tile even after a failed wait (their waits then
    // return at once), so the named barrier below is always reached by all of them.
    while (walk.next(p, x)) {
      const NtLayer& L = p.lay[x.g];
      const int s = x.m_t;
      for (int n = x.n0; n < x.n1; ++n, ++ti) {
        const bool got = wait(accfull, ti & 1);
        if (!got) atomicOr(p.err, kErrTimeoutEpilogue);
        ptx::tc_fence_after();
        // The MMAs of the next tile wait for this hand-over, so its path is short: load
        // the first 64 columns, square them into four independent sums and stage them as
        // bf16 in this warp's box (row `lane` at 128-byte row `lane`, unit uu at
        // uu ^ (lane & 7)), load the other 64, release the accumulator, and only then
        // work on those.
        float sq[4] = {0.f, 0.f, 0.f, 0.f};
        float v[64];
        ptx::tmem_ld64(tsrc, v);
#pragma unroll
        for (int k = 0; k < 64; ++k) sq[k & 3] = fmaf(v[k], v[k], sq[k & 3]);
        auto stage = [&]() {
          __syncwarp();   // every lane has read the box's previous rows out
#pragma unroll
          for (int uu = 0; uu < 8; ++uu)
            rbox[lane * 8 + (uu ^ (lane & 7))] =
                make_uint4(pack_bf16(v[8 * uu + 0], v[8 * uu + 1]), pack_bf16(v[8 * uu + 2], v[8 * uu + 3]),
                           pack_bf16(v[8 * uu + 4], v[8 * uu + 5]), pack_bf16(v[8 * uu + 6], v[8 * uu + 7]));
          __syncwarp();
        };
        // the box's 32 rows x 64 columns out as whole 128-byte row pieces, four rows per
        // instruction, to columns h * 128 + cc * 64 of the tile
        auto write_out = [&](int cc) {
          const int uu = lane & 7;
          uint4* dst = reinterpret_cast<uint4*>(
              L.Rst + (static_cast<size_t>(s) * p.r + mblk * kBM + q * 32 + (lane >> 3)) * L.d_out + n * kNtBN +
              h * 128 + cc * 64 + 8 * uu);
          const int step = L.d_out / 2;   // four rows of bf16, in 16-byte units
#pragma unroll 2
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + (lane >> 3);
            dst[i * step] = rbox[rr * 8 + (uu ^ (rr & 7))];
          }
        };
        stage();
        ptx::tmem_ld64(tsrc + 64, v);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(accempty);
#pragma unroll
        for (int k = 0; k < 64; ++k) sq[k & 3] = fmaf(v[k], v[k], sq[k & 3]);
        if (got) {
          write_out(0);
          stage();
          write_out(1);
        }
        float ss = (sq[0] + sq[1]) + (sq[2] + sq[3]);
        if (!got) ss = 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        float* rb = red + (ti & 1) * kEpiWarps;
        if (lane == 0) rb[ew] = ss;
        epi_bar();
        // one partial slot per 128 columns: column half `lane` is its four warps' sum
        if (ew == 0 && lane < 2) {
          float tot = 0.0f;
#pragma unroll
          for (int k = 0; k < 4; ++k) tot += rb[4 * lane + k];
          p.partials[static_cast<size_t>(s) * p.part_stride + L.part_base + mblk * (2 * L.nt) + 2 * n + lane] =
              tot;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kNtTmemCols);
  }
}

// ---- the projection in 256-row tiles ------------------------------------------------
// AP = A P for r >= 256 in tiles of 256 stacked rows x 256 columns of r, K = d_in: two
// M = 128 MMAs per 16-wide k step, one per 128-row half of the tile, share the P box of
// the stage.  Against tc_gemm_kernel<PROJECT>'s 128-row tiles, each P block is read from
// L2 by half as many CTAs: per 128 x 256 unit of output, 128 + 256 (here) instead of
// 128 + 512 bytes per k.  The two 128 x 256 fp32 accumulators fill TMEM's 512 columns,
// so the MMAs of a tile wait for the epilogue of the one before; with K = d_in that
// hand-over is small next to a tile's K loop.
//
// Tiles are as long as their layer's d_in, and there are half as many as with 128-row
// tiles, so a plain round robin over CTAs leaves some CTAs a long tile more than others
// (on the 7B slice's launch groups, 31 % above the mean).  The host therefore gives each
// CTA its own list: tiles in descending length, each to the CTA with the least work so
// far (LPT), about 4 % above the mean; tiles of equal length keep their order, so the
// column tiles of one row block run side by side and read its rows of A once from DRAM.
//
// Warps: 0 and 10 load the ring, alternating stages (A, a step input, before
// griddepcontrol.wait; P after it); 1 owns TMEM and issues the MMAs; 2-9 are the
// epilogue (warp w: lane quarter w % 4, 128-row half (w - 2) / 4 of the tile), which
// writes AP as bf16.
constexpr int kPwStages = 3;
constexpr int kPwThreads = 32 * 11;
constexpr int kPwProducer1 = 10;
struct PwSmem {
  static constexpr int kA = kBM * kBK * 2;                 // one 128-row half: 16 KB
  static constexpr int kStage = 2 * kA + 256 * kBK * 2;    // two halves and P (64 x 256): 64 KB
  static constexpr int kBarOff = kPwStages * kStage;
  static constexpr int kBytes = kBarOff + 256 + 1024;      // barriers + alignment slack
  static_assert(kBytes <= 232448, "exceeds the shared memory of a CTA");
};

__global__ void __launch_bounds__(kPwThreads, 1) tc_project_wide_kernel(const __grid_constant__ GroupParams p) {
  using S = PwSmem;
  constexpr int NS = kPwStages;
  constexpr uint32_t kIdesc = ptx::idesc_bf16(kBM, 256, false, true);   // A K-major, P N-major
  static_assert((2 * NS + 2) * 8 + 16 <= 256, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + NS;
  uint64_t* accfull = empty + NS;
  uint64_t* accempty = accfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitLimitNs, abort_flag);
  };
  ptx::griddep_launch_dependents();
  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int st = 0; st < NS; ++st) {
      ptx::mbar_init(&full[st], 1);
      ptx::mbar_init(&empty[st], 1);
    }
    ptx::mbar_init(accfull, 1);
    ptx::mbar_init(accempty, kEpiWarps);
    ptx::fence_mbar_init();
    for (int g = 0; g < p.n_layers; ++g) {
      ptx::prefetch_tmap(&p.mapA[g]);
      ptx::prefetch_tmap(&p.mapB[g]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // this CTA's tiles: positions [k0, k1) of the launch's schedule
  const int k0 = p.sched[p.total_tiles + blockIdx.x], k1 = p.sched[p.total_tiles + blockIdx.x + 1];

  if (warp == 0 || warp == kPwProducer1) {
    // ---------------- TMA producers: stage it is loaded by producer it % 2 ----------------
    if (lane == 0) {
      const int pi = warp == 0 ? 0 : 1;
      const uint64_t polA = ptx::policy_evict_first();   // A is read by the r / 256 column tiles
      const uint64_t polB = ptx::policy_evict_last();    // P is read by every row tile
      bool waited = false, ok = true;
      uint32_t it = 0, issued_end = 0;
      for (int k = k0; ok && k < k1; ++k) {
        const TileCoord c = decode_tile(p, p.sched[k], PROJECT);
        const GroupLayer& L = p.lay[c.g];
        const int m0 = c.m_t * 2 * kBM;
        const bool two = m0 + kBM < L.M;   // the second half has rows of A
        for (int kb = c.kb0; kb < c.kb1; ++kb, ++it) {
          if (static_cast<int>(it & 1) != pi) continue;
          const int st = it % NS;
          const uint32_t use = it / NS;
          if (use > 0 && !wait(&empty[st], (use - 1) & 1)) {
            atomicOr(p.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * S::kStage;
          const int kk = kb * kBK;
          ptx::mbar_arrive_expect_tx(&full[st], (two ? 2 : 1) * S::kA + 256 * kBK * 2);
          GRAPE_BOX(p.err, p.extA[c.g], 2, kk, m0, 0)
          ptx::tma_load_2d_hint(sa, &p.mapA[c.g], &full[st], kk, m0, polA);
          if (two)
            GRAPE_BOX(p.err, p.extA[c.g], 2, kk, m0 + kBM, 0)
            ptx::tma_load_2d_hint(sa + S::kA, &p.mapA[c.g], &full[st], kk, m0 + kBM, polA);
          if (!waited) {
            ptx::griddep_wait();   // P is generated earlier in the step
            waited = true;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            GRAPE_BOX(p.err, p.extB[c.g], 2, c.n_t * 256 + 64 * q, kk, 0)
            ptx::tma_load_2d_hint(sa + 2 * S::kA + q * 8192, &p.mapB[c.g], &full[st], c.n_t * 256 + 64 * q, kk,
                                  polB);
          issued_end = it + 1;
        }
      }
      if (*abort_flag)   // leave none of this thread's loads in flight into shared memory
        for (uint32_t k = issued_end > NS ? issued_end - NS : 0; k < issued_end; ++k)
          if (static_cast<int>(k & 1) == pi) ptx::mbar_wait(&full[k % NS], (k / NS) & 1, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ---------------- UMMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int k = k0; ok && k < k1; ++k, ++tc) {
        const TileCoord c = decode_tile(p, p.sched[k], PROJECT);
        // the epilogue has the previous tile in registers
        if (tc > 0 && !wait(accempty, (tc - 1) & 1)) {
          atomicOr(p.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        for (int kb = c.kb0; kb < c.kb1; ++kb, ++it) {
          const int st = it % NS;
          if (!wait(&full[st], (it / NS) & 1)) {
            atomicOr(p.err, kErrTimeoutMma);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a_base = ptx::smem_u32(smem + st * S::kStage);
          const uint32_t b_base = a_base + 2 * S::kA;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bd = ptx::desc_sw128(b_base + k * 2048, 8192, 1024);
            const uint32_t acc = (kb > c.kb0 || k > 0) ? 1u : 0u;
            ptx::umma_bf16(tmem, ptx::desc_sw128(a_base + k * 32, 16, 1024), bd, kIdesc, acc);
            ptx::umma_bf16(tmem + 256, ptx::desc_sw128(a_base + S::kA + k * 32, 16, 1024), bd, kIdesc, acc);
          }
          ptx::umma_commit(&empty[st]);
        }
        ptx::umma_commit(accfull);
      }
    }
  } else {
    // ---------------- epilogue: warps 2..9 ----------------
    const int ew = warp - 2;
    const int q = warp & 3;          // TMEM lanes (rows of a half) 32q .. 32q+31
    const int h = ew >> 2;           // 128-row half of the tile: accumulator h
    uint32_t tc = 0;
    // The epilogue warps walk every tile even after a failed wait (their waits then
    // return at once).
    for (int k = k0; k < k1; ++k, ++tc) {
      const TileCoord c = decode_tile(p, p.sched[k], PROJECT);
      const GroupLayer& L = p.lay[c.g];
      const bool got = wait(accfull, tc & 1);
      if (!got) atomicOr(p.err, kErrTimeoutEpilogue);
      ptx::tc_fence_after();
      const int m = c.m_t * 2 * kBM + h * kBM + q * 32 + lane;
      __nv_bfloat16* AP = static_cast<__nv_bfloat16*>(L.out);
      const uint32_t tsrc = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 256;
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 64) {
        float v[64];
        ptx::tmem_ld64(tsrc + cc, v);
        if (cc == 192) {   // the whole accumulator is in registers: the next tile may start
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(accempty);
        }
        if (got && m < L.M) {
          uint4* dst = reinterpret_cast<uint4*>(AP + static_cast<size_t>(m) * L.ldo + c.n_t * 256 + cc);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[u] = make_uint4(pack_bf16(v[8 * u + 0], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                                pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---- aggregation with the K split across a thread-block cluster --------------------
// For few output tiles (r x d_out is small next to K = B*T): the CS CTAs of a cluster
// share one 128 x BN output tile of S and each runs 1/CS of the stacked token rows.
// Their fp32 partial tiles meet in shared memory: after a cluster barrier, CTA k sums
// rows [k*128/CS, (k+1)*128/CS) over the CS partials, read through distributed shared
// memory in rank order (a fixed order: the result does not depend on timing), and
// writes them to S.  No partial ever goes to global memory.
template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1) tc_agg_cluster_kernel(const __grid_constant__ GroupParams p) {
  using S = Smem<BN, STAGES>;
  constexpr uint32_t kTmemCols = BN;
  constexpr uint32_t kIdesc = ptx::idesc_bf16(kBM, BN, true, true);
  constexpr int kLd = BN + 4;   // staging row stride (floats): conflict-free row writes
  static_assert(kBM * kLd * 4 <= STAGES * S::kStage, "staging must fit in the stage ring");
  static_assert(BN % 128 == 0, "each epilogue warp stages BN/2 columns in 64-column loads");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* accfull = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CS = p.cluster;
  ptx::griddep_launch_dependents();
  const uint32_t rank = ptx::cluster_ctarank();
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitLimitNs, abort_flag);
  };

  // output tile of this cluster and this CTA's share of K
  const TileCoord c = decode_tile(p, static_cast<int>(blockIdx.x) / CS, NORM);
  const GroupLayer& L = p.lay[c.g];
  const int kb0 = static_cast<int>(static_cast<int64_t>(rank) * L.kblocks / CS);
  const int kb1 = static_cast<int>(static_cast<int64_t>(rank + 1) * L.kblocks / CS);

  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accfull, 1);
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&p.mapA[c.g]);
    ptx::prefetch_tmap(&p.mapB[c.g]);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (producer_of(warp) >= 0) {
    // Producer p fills the stages of iterations it = p (mod kNP).  Gout predates the
    // step and loads before the wait for the clip kernel; AP (rescaled by it) after.
    constexpr int kNP = RingProducers<STAGES>::kCount;
    static_assert(kNP >= 1 && kNP <= STAGES, "parity waits need at most STAGES producers");
    if (lane == 0 && producer_of(warp) < kNP) {
      const int pi = producer_of(warp);
      const uint64_t pol = ptx::policy_evict_first();   // last use of AP and Gout in the step
      const CUtensorMap* mapA = &p.mapA[c.g];
      const CUtensorMap* mapB = &p.mapB[c.g];
      bool waited = false;
      uint32_t issued_end = 0;
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        if (it % kNP != pi) continue;
        const int s = it % STAGES;
        const uint32_t use = it / STAGES;
        if (use > 0 && !wait(&empty[s], (use - 1) & 1)) {
          atomicOr(p.err, kErrTimeoutProducer);
          break;
        }
        uint8_t* sa = smem + s * S::kStage;
        uint8_t* sb = sa + S::kABytes;
        ptx::mbar_arrive_expect_tx(&full[s], S::kStage);
#pragma unroll
        for (int q = 0; q < BN / 64; ++q)
          GRAPE_BOX(p.err, p.extB[c.g], 2, c.n_t * BN + 64 * q, kb * kBK, 0)
          ptx::tma_load_2d_hint(sb + q * 8192, mapB, &full[s], c.n_t * BN + 64 * q, kb * kBK, pol);
        if (!waited) {
          ptx::griddep_wait();
          waited = true;
        }
#pragma unroll
        for (int q = 0; q < kBM / 64; ++q)
          GRAPE_BOX(p.err, p.extA[c.g], 2, c.m_t * kBM + 64 * q, kb * kBK, 0)
          ptx::tma_load_2d_hint(sa + q * 8192, mapA, &full[s], c.m_t * kBM + 64 * q, kb * kBK, pol);
        issued_end = it + 1;
      }
      if (*abort_flag)
        for (uint32_t k2 = issued_end > STAGES ? issued_end - STAGES : 0; k2 < issued_end; ++k2)
          if (static_cast<int>(k2 % kNP) == pi)
            ptx::mbar_wait(&full[k2 % STAGES], (k2 / STAGES) & 1, kDrainLimitNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!wait(&full[s], ph)) {
          atomicOr(p.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a_base = ptx::smem_u32(smem + s * S::kStage);
        const uint32_t b_base = a_base + S::kABytes;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          ptx::umma_bf16(tmem, ptx::desc_sw128(a_base + k * 2048, 8192, 1024),
                         ptx::desc_sw128(b_base + k * 2048, 8192, 1024), kIdesc,
                         (kb > kb0 || k > 0) ? 1u : 0u);
        ptx::umma_commit(&empty[s]);
      }
      ptx::umma_commit(accfull);
    }
  } else if (warp < 2 + kEpiWarps) {
    const int q = warp & 3;                 // TMEM lane quarter
    const int h = (warp - 2) >> 2;          // column half
    const int row = q * 32 + lane;
    // partial tile -> own shared memory (the stage ring is idle once the MMAs are done)
    const bool got = wait(accfull, 0);
    if (!got) atomicOr(p.err, kErrTimeoutEpilogue);
    ptx::tc_fence_after();
    float* stage = reinterpret_cast<float*>(smem);
    const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * (BN / 2);
    const bool have = got && kb1 > kb0;
#pragma unroll 1
    for (int cc = 0; cc < BN / 2; cc += 32) {
      float v[32];
      ptx::tmem_ld32(tbase + cc, v);
      float4* dst = reinterpret_cast<float4*>(stage + row * kLd + h * (BN / 2) + cc);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        dst[u] = have ? make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3])
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  __syncwarp();
  ptx::cluster_sync();   // every partial tile of the cluster is in shared memory

  if (warp >= 2 && warp < 2 + kEpiWarps) {
    const int e = (warp - 2) * 32 + threadIdx.x % 32;
    const int rows_per = kBM / CS;
    const int r0 = static_cast<int>(rank) * rows_per;
    const uint32_t stage_addr = ptx::smem_u32(smem);
    float* Sout = static_cast<float*>(L.out);
    const int n_f4 = rows_per * (BN / 4);
    for (int idx = e; idx < n_f4; idx += 32 * kEpiWarps) {
      const int rr = r0 + idx / (BN / 4);
      const int c4 = idx % (BN / 4);
      const uint32_t off = static_cast<uint32_t>((rr * kLd + c4 * 4) * 4);
      float4 acc = ptx::ld_dsmem_f4(ptx::mapa_shared(stage_addr + off, 0));
      for (int j = 1; j < CS; ++j) {
        const float4 x = ptx::ld_dsmem_f4(ptx::mapa_shared(stage_addr + off, j));
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
      }
      const int m = c.m_t * kBM + rr;
      const int n = c.n_t * BN + c4 * 4;
      if (m < L.M && n + 4 <= L.N)
        *reinterpret_cast<float4*>(Sout + static_cast<size_t>(m) * L.ldo + n) = acc;
    }
  }
  __syncwarp();
  ptx::cluster_sync();   // no CTA leaves while another may still read its shared memory
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- P_l in bf16, row-major d_in x r: element e = k*r + j ----------------------------
// A thread unit is Philox block q of one layer (elements 4q .. 4q+3), its normals from
// the special-function unit's log and sine/cosine (gaussian4_fast): the values are
// rounded to bf16 at once, and the precise functions made the kernel issue-bound on
// them.  The units of all layers are numbered back to back (begin[l] .. begin[l+1]) and
// a grid of a few blocks per SM strides over them, so layers of unequal size keep every
// SM busy.
struct PTable {
  __nv_bfloat16* P16[GRAPE_MAX_LAYERS];
  int64_t begin[GRAPE_MAX_LAYERS + 1];   // first unit of each layer; begin[L] = total
  int L;
};

__global__ void __launch_bounds__(256) gen_P_bf16_kernel(PTable t, uint64_t seed, uint32_t step, int r) {
  ptx::griddep_launch_dependents();
  const float scale = rsqrtf(static_cast<float>(r));
  const int64_t total = t.begin[t.L];
  int l = 0;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    while (u >= t.begin[l + 1]) ++l;   // u only grows, so l only moves forward
    const int64_t q = u - t.begin[l];
    const float4 z = gaussian4_fast(seed, static_cast<uint32_t>(l), step, kStreamProjection,
                                    static_cast<uint32_t>(q));
    reinterpret_cast<uint2*>(t.P16[l])[q] =
        make_uint2(pack_bf16(z.x * scale, z.y * scale), pack_bf16(z.z * scale, z.w * scale));
  }
}

// ---- n_i, c_i, and the clip folded into AP ------------------------------------------
// Block (i, l): n_i = sqrt(sum of sample i's partial slots) in a fixed order (every
// block of sample i computes the same bits), c_i = C/n_i if n_i > C else 1; block
// (i, 0) records n_i and c_i, and block (i, l) rescales sample i's T rows of AP_l by
// c_i in place, so the aggregation that follows is a plain GEMM:
// sum_i c_i (A_i P)^T Gout_i = (diag(c) AP)^T Gout over the stacked rows.
struct ApTable {
  __nv_bfloat16* AP[GRAPE_MAX_LAYERS];
};

__global__ void __launch_bounds__(256) clip_scale_kernel(ApTable t, int r, int T, int part_stride, float C,
                                                         const float* partials, float* norms, float* clip,
                                                         int rescale) {
  __shared__ float red[8];
  __shared__ float c_sh;
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();   // the norm partials, and AP no longer read by the norm kernel
  const int i = blockIdx.x, l = blockIdx.y;
  const float* pp = partials + static_cast<size_t>(i) * part_stride;
  float ss = 0.0f;
  for (int k = threadIdx.x; k < part_stride; k += 256) ss += pp[k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.0f;
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float n = sqrtf(tot);
    const float c = (n > C) ? C / n : 1.0f;
    if (l == 0) {
      norms[i] = n;
      clip[i] = c;
    }
    c_sh = c;
  }
  __syncthreads();
  const float c = c_sh;
  if (c == 1.0f || !rescale) return;
  uint4* rows = reinterpret_cast<uint4*>(t.AP[l] + static_cast<size_t>(i) * T * r);
  const size_t n8 = static_cast<size_t>(T) * r / 8;   // 8 bf16 per 16-byte vector
  constexpr int kBatch = 8;                            // loads in flight per thread
  for (size_t k0 = threadIdx.x; k0 < n8; k0 += 256 * kBatch) {
    uint4 x[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const size_t k = k0 + static_cast<size_t>(u) * 256;
      if (k < n8) x[u] = rows[k];
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const size_t k = k0 + static_cast<size_t>(u) * 256;
      if (k >= n8) continue;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&x[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        h[e] = __floats2bfloat162_rn(f.x * c, f.y * c);
      }
      rows[k] = x[u];
    }
  }
}

// ---- S_l = sum_i c_i R_i over the R_i the norm kernel stored ------------------------
// The stored variant of the aggregation: every R_{i,l} (r x d_out) was written as bf16
// by the norm kernel to [sample][r][d_out], so S is a c-weighted sum of B streams, an
// HBM-bound pass over B*r*d_out*2 bytes instead of a second contraction over the B*T
// stacked rows.  Thread unit u covers 8 consecutive elements of one layer (16 bytes per
// sample); units of all layers are numbered back to back (begin[l] .. begin[l+1]) so
// the grid covers layers of unequal size evenly.  Samples are summed in order 0..B-1
// with fmaf, so the result does not depend on timing.
struct StoredAggTable {
  const __nv_bfloat16* R[GRAPE_MAX_LAYERS];   // [B][r][d_out] bf16
  float* S[GRAPE_MAX_LAYERS];                  // [r][d_out] fp32
  int64_t begin[GRAPE_MAX_LAYERS + 1];         // first unit of each layer; begin[L] = total
};

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& x, float c) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    acc[2 * e] = fmaf(c, f.x, acc[2 * e]);
    acc[2 * e + 1] = fmaf(c, f.y, acc[2 * e + 1]);
  }
}

__global__ void __launch_bounds__(256) aggregate_stored_kernel(StoredAggTable t, int L, int B,
                                                               const float* clip) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();   // R_i from the norm kernel, c_i from the clip kernel
  const int64_t total = t.begin[L];
  int l = 0;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    while (u >= t.begin[l + 1]) ++l;   // u only grows, so l only moves forward
    const int64_t e = u - t.begin[l];                       // unit within the layer
    const int64_t n8 = t.begin[l + 1] - t.begin[l];         // units per sample
    const uint4* R = reinterpret_cast<const uint4*>(t.R[l]) + e;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    constexpr int kBatch = 8;   // loads in flight per thread
    int i = 0;
    for (; i + kBatch <= B; i += kBatch) {
      uint4 x[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) x[k] = __ldcs(R + static_cast<int64_t>(i + k) * n8);
#pragma unroll
      for (int k = 0; k < kBatch; ++k) acc_bf16x8(acc, x[k], __ldg(clip + i + k));
    }
    for (; i < B; ++i) acc_bf16x8(acc, __ldcs(R + static_cast<int64_t>(i) * n8), __ldg(clip + i));
    float4* S = reinterpret_cast<float4*>(t.S[l]) + 2 * e;
    S[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    S[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// ---- the stored aggregation fused with noise + projected Adam (one-process step) ----
// S = sum_i c_i R_i, then g = (S + sigma C xi) / batch and the Adam update, per unit of
// eight consecutive elements of one layer's r x d_out: the same per-element arithmetic,
// in the same order, as aggregate_stored_kernel followed by noise_adam_kernel (the noise
// of elements 8e .. 8e+7 is Philox blocks 2e and 2e+1 of the noise stream), so the two
// forms give the same bits.  S is still written, for grape_debug; what the fusion saves
// is S's re-read and a launch, and the noise's Philox and Box-Muller work runs under
// the R_i stream instead of after it.  The unit's m, v and noise, which depend on no
// kernel of the step, are fetched before griddepcontrol.wait for the first unit.
struct AggAdamTable {
  const __nv_bfloat16* R[GRAPE_MAX_LAYERS];   // [B][r][d_out] bf16
  float* S[GRAPE_MAX_LAYERS];                  // [r][d_out] fp32
  float* m[GRAPE_MAX_LAYERS];
  float* v[GRAPE_MAX_LAYERS];
  __nv_bfloat16* dR[GRAPE_MAX_LAYERS];
  int64_t begin[GRAPE_MAX_LAYERS + 1];         // first unit of each layer; begin[L] = total
};

struct AggAdamUnit {
  float m[8], v[8], xi[8];
};

__device__ __forceinline__ void agg_adam_load(const StepShape& sh, const AggAdamTable& t, uint32_t step, int l,
                                              int64_t e, AggAdamUnit& a) {
  const float4* m4 = reinterpret_cast<const float4*>(t.m[l]) + 2 * e;
  const float4* v4 = reinterpret_cast<const float4*>(t.v[l]) + 2 * e;
  const float4 ma = m4[0], mb = m4[1], va = v4[0], vb = v4[1];
  a.m[0] = ma.x; a.m[1] = ma.y; a.m[2] = ma.z; a.m[3] = ma.w;
  a.m[4] = mb.x; a.m[5] = mb.y; a.m[6] = mb.z; a.m[7] = mb.w;
  a.v[0] = va.x; a.v[1] = va.y; a.v[2] = va.z; a.v[3] = va.w;
  a.v[4] = vb.x; a.v[5] = vb.y; a.v[6] = vb.z; a.v[7] = vb.w;
  if (sh.sigma_C != 0.0f) {
    const float4 z0 = gaussian4(sh.seed, static_cast<uint32_t>(l), step, kStreamNoise, static_cast<uint32_t>(2 * e));
    const float4 z1 =
        gaussian4(sh.seed, static_cast<uint32_t>(l), step, kStreamNoise, static_cast<uint32_t>(2 * e + 1));
    a.xi[0] = z0.x; a.xi[1] = z0.y; a.xi[2] = z0.z; a.xi[3] = z0.w;
    a.xi[4] = z1.x; a.xi[5] = z1.y; a.xi[6] = z1.z; a.xi[7] = z1.w;
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) a.xi[k] = 0.0f;
  }
}

__global__ void __launch_bounds__(256) aggregate_adam_kernel(StepShape sh, AggAdamTable t, UpdateScalars u,
                                                             const float* clip) {
  ptx::griddep_launch_dependents();
  const int64_t total = t.begin[sh.L];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t unit = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  int l = 0;
  AggAdamUnit a;
  if (unit < total) {
    while (unit >= t.begin[l + 1]) ++l;
    agg_adam_load(sh, t, u.step, l, unit - t.begin[l], a);
  }
  ptx::griddep_wait();   // R_i from the norm kernel, c_i from the clip kernel
  const int B = sh.B;
  for (bool first = true; unit < total; unit += stride, first = false) {
    while (unit >= t.begin[l + 1]) ++l;   // units only grow, so l only moves forward
    const int64_t e = unit - t.begin[l];                     // unit within the layer
    const int64_t n8 = t.begin[l + 1] - t.begin[l];         // units per sample
    if (!first) agg_adam_load(sh, t, u.step, l, e, a);
    const uint4* R = reinterpret_cast<const uint4*>(t.R[l]) + e;
    float S[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    constexpr int kBatch = 8;   // loads in flight per thread
    int i = 0;
    for (; i + kBatch <= B; i += kBatch) {
      uint4 x[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) x[k] = __ldcs(R + static_cast<int64_t>(i + k) * n8);
#pragma unroll
      for (int k = 0; k < kBatch; ++k) acc_bf16x8(S, x[k], __ldg(clip + i + k));
    }
    for (; i < B; ++i) acc_bf16x8(S, __ldcs(R + static_cast<int64_t>(i) * n8), __ldg(clip + i));
    float4* S4 = reinterpret_cast<float4*>(t.S[l]) + 2 * e;
    S4[0] = make_float4(S[0], S[1], S[2], S[3]);
    S4[1] = make_float4(S[4], S[5], S[6], S[7]);
    const float b1 = sh.beta1, b2 = sh.beta2;
    const float ob1 = sh.one_minus_beta1, ob2 = sh.one_minus_beta2;
    float d[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float g = fmaf(sh.sigma_C, a.xi[k], S[k]) * u.inv_batch;
      a.m[k] = fmaf(b1, a.m[k], ob1 * g);
      a.v[k] = fmaf(b2, a.v[k], ob2 * g * g);
      d[k] = (a.m[k] * u.inv_bc1) / (sqrtf(a.v[k] * u.inv_bc2) + sh.eps);
    }
    float4* m4 = reinterpret_cast<float4*>(t.m[l]) + 2 * e;
    float4* v4 = reinterpret_cast<float4*>(t.v[l]) + 2 * e;
    m4[0] = make_float4(a.m[0], a.m[1], a.m[2], a.m[3]);
    m4[1] = make_float4(a.m[4], a.m[5], a.m[6], a.m[7]);
    v4[0] = make_float4(a.v[0], a.v[1], a.v[2], a.v[3]);
    v4[1] = make_float4(a.v[4], a.v[5], a.v[6], a.v[7]);
    reinterpret_cast<uint4*>(t.dR[l])[e] = make_uint4(pack_bf16(d[0], d[1]), pack_bf16(d[2], d[3]),
                                                     pack_bf16(d[4], d[5]), pack_bf16(d[6], d[7]));
  }
}

// ---------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// bf16 row-major [rows][cols] as a 2-D map with a (box_cols x box_rows) box, 128-byte swizzle.
bool map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_cols,
            uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 row-major [rows][cols] as a 2-D map with a (32 x box_rows) box, 128-byte swizzle.
bool map_2d_f32(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows = kBM) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [B][T][cols] as a 3-D map with a (64 x box_rows x 1) box: rows past T read as zero.
bool map_3d(CUtensorMap* m, const void* ptr, uint64_t B, uint64_t T, uint64_t cols, uint32_t box_rows = 64) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, T, B};
  cuuint64_t strides[2] = {cols * 2, T * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Small cache of encoded maps keyed by base pointer (callers often reuse buffers).
struct MapCache {
  struct Entry { const void* ptr; CUtensorMap map; uint64_t used; };
  std::vector<Entry> e;
  uint64_t tick = 0;
  template <class F>
  bool get(const void* ptr, CUtensorMap* out, F&& make) {
    ++tick;
    for (auto& x : e)
      if (x.ptr == ptr) {
        x.used = tick;
        *out = x.map;
        return true;
      }
    Entry n{ptr, {}, tick};
    if (!make(&n.map)) return false;
    if (e.size() < 8) {
      e.push_back(n);
    } else {
      size_t lru = 0;
      for (size_t k = 1; k < e.size(); ++k)
        if (e[k].used < e[lru].used) lru = k;
      e[lru] = n;
    }
    *out = n.map;
    return true;
  }
};

constexpr int kBnWide = 256;
// One CTA per SM, so each ring takes most of the 227 KB of shared memory.
constexpr int kStagesProject128 = 6;   // 6 x 32 KB
constexpr int kStagesProject256 = 4;   // 4 x 48 KB
constexpr int kStagesNorm = 4;         // 4 x 48 KB
constexpr int kStagesAgg = 4;          // 4 x 48 KB
constexpr int kStagesBack = 3;         // 3 x 32 KB stages + 2 x 64 KB W tiles
constexpr int kBnAggCluster = 128;     // cluster-split aggregation: 6 x 32 KB
constexpr int kStagesAggCluster = 6;
constexpr int kStagesGhost = 6;        // 6 x 32 KB: the two 128-token blocks of a Gram block

struct HostState {
  int L = 0, r = 0, B = 0, T = 0;
  std::vector<int> d_in, d_out;
  // fixed maps (library buffers)
  std::vector<CUtensorMap> mapP_mn;     // P16 as the MN-major B operand of PROJECT
  std::vector<CUtensorMap> mapP_k;      // P16 as the K-major A operand of BACKPROJ
  std::vector<CUtensorMap> mapAP3;      // AP as [B][T][r] (NORM A operand)
  std::vector<CUtensorMap> mapAP3k;     // AP as [B][T][r], 128-row boxes (GHOST)
  std::vector<CUtensorMap> mapAP2;      // AP as [B*T][r] (AGGREGATE A operand)
  std::vector<CUtensorMap> mapDR;       // dR as [r][d_out] (BACKPROJ B operand)
  // per-step maps, cached by pointer
  std::vector<MapCache> cacheA, cacheG3, cacheG2, cacheW, cacheG3k, cacheWs;
  int* err = nullptr;
  int bn_project = 128;
  GroupParams gp;   // host staging of one launch's kernel parameters
  BptParams bp;     // the same for tc_backproj_tmem_kernel
  NtParams np;      // the same for tc_norm_tmem_kernel
  // GRAPE_NORM_TMEM in the environment when the context is created: 0 runs the norms on
  // tc_gemm_kernel<NORM / NORMST> for every T, 1 runs tc_norm_tmem_kernel wherever it
  // can (stored R_i, T <= 512); unset, tc_norm_a_in_tmem decides by T (a measurement
  // and test knob: both kernels compute the same partial slots and R_i)
  int norm_tmem = -1;
  // GRAPE_PROJECT_WIDE=0 at context creation keeps the projection on 128-row tiles
  // (tc_gemm_kernel<PROJECT>) at every r; by default r >= 256 runs tc_project_wide_kernel
  bool project_wide = true;
  std::vector<const int*> sched;   // per launch group: the wide projection's schedule
  std::vector<int> sched_grid;     // and the grid it was built for
};

int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// A programmatic dependent launch of `kernel` after the previous kernel in the stream when
// `pdl` (the kernel itself waits with griddepcontrol.wait before it reads that kernel's
// outputs), else an ordinary one: the first kernel of a step is ordinary, so it waits for
// all earlier work, which the early loads of the later kernels rely on.
template <class Kern, class... Args>
cudaError_t launch_maybe_pdl(bool pdl, Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = a;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <class Kern, class... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  return launch_maybe_pdl(true, kernel, grid, block, smem, st, args...);
}

// Launch configuration that belongs to a device: its SM count, and per kernel the
// opt-in to more than 48 KB of dynamic shared memory (cudaFuncSetAttribute acts on the
// current device only) with the residency that follows from it.  Each entry is taken
// once per (device, kernel, key) under one lock, so host threads driving several GPUs
// launch every kernel with its attribute set on the device it runs on.
std::mutex g_launch_cfg_mu;
std::map<std::tuple<int, const void*, int>, int> g_launch_cfg;   // (device, kernel, key) -> value

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  return dev;
}

int sm_count() {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_launch_cfg_mu);
  int& n = g_launch_cfg[std::make_tuple(dev, static_cast<const void*>(nullptr), 0)];
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Sets `kernel`'s dynamic shared memory to `smem` bytes on the current device (once per
// device) and returns in *per_sm how many of its CTAs of `threads` threads an SM holds.
cudaError_t configure_kernel(const void* kernel, int smem, int threads, int* per_sm) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_launch_cfg_mu);
  int& n = g_launch_cfg[std::make_tuple(dev, kernel, 1)];
  if (n == 0) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int got = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&got, kernel, threads, smem);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return e;
    }
    if (got < 1) return cudaErrorInvalidConfiguration;   // does not fit on an SM
    n = got;
  }
  *per_sm = n;
  return cudaSuccess;
}

// Persistent launch: as many CTAs as the runtime keeps resident at once (one per SM
// for a kernel that allocates TMEM), never more than there are tiles.  A larger grid
// would run its surplus CTAs as a second wave behind the first.
template <int MODE, int BN, int STAGES>
cudaError_t launch_group(GroupParams& gp, int tiles, cudaStream_t st, bool pdl = true) {
  using S = SmemOf<MODE, BN, STAGES>;
  int per_sm = 0;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(tc_gemm_kernel<MODE, BN, STAGES>), S::kBytes,
                                   kThreads, &per_sm);
  if (e != cudaSuccess) return e;
  gp.total_tiles = tiles;
  if (tiles <= 0) return cudaSuccess;
  int grid = sm_count() * per_sm;
  grid = grid < tiles ? grid : tiles;
  return launch_maybe_pdl(pdl, tc_gemm_kernel<MODE, BN, STAGES>, dim3(grid), dim3(kThreads), S::kBytes, st, gp);
}

// Build and launch the groups of one mode.  fill(g, l, gp) sets maps and the layer record
// (except tiles_begin) and returns the tile count of layer l.
// `pdl_first` = false makes the first launch an ordinary one (used when it is the step's
// first kernel); later groups always follow a kernel of the same step.
template <int MODE, int BN, int STAGES, class Fill>
cudaError_t run_mode(const HostState& hs, int L, cudaStream_t st, int* launches, const Fill& fill,
                     GroupParams& gp, bool pdl_first = true) {
  for (int l0 = 0; l0 < L; l0 += kMaxGroup) {
    const int n = (L - l0) < kMaxGroup ? (L - l0) : kMaxGroup;
    gp.n_layers = n;
    int tiles = 0;
    for (int g = 0; g < n; ++g) {
      int t = 0;
      if (!fill(g, l0 + g, &t)) return cudaErrorInvalidValue;
      gp.lay[g].tiles_begin = tiles;
      tiles += t;
    }
    cudaError_t e = launch_group<MODE, BN, STAGES>(gp, tiles, st, l0 == 0 ? pdl_first : true);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  (void)hs;
  return cudaSuccess;
}

}  // namespace

bool tc_supported(int device, const grape_layer* layers, int n_layers, int r, int B, int T,
                  std::string* why) {
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  if (major != 10 || minor != 0) {
    if (why) *why = "the tensor-core kernels are built for sm_100a (B200)";
    return false;
  }
  if (!encode_fn()) {
    if (why) *why = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  // Every TMA box starts inside its tensor (no box lies wholly out of bounds): the
  // projection width r tiles by 128 (and by 256 above 256), d_out by 256.
  if (r % 128 != 0 || (r > 256 && r % 256 != 0)) {
    if (why) *why = "the tensor-core path needs r to be a multiple of 128 (and of 256 above 256)";
    return false;
  }
  for (int l = 0; l < n_layers; ++l)
    if (layers[l].d_in % 8 != 0 || layers[l].d_out % 256 != 0) {
      if (why) *why = "the tensor-core path needs d_in % 8 == 0 and d_out % 256 == 0";
      return false;
    }
  (void)B;
  (void)T;
  return true;
}

// One slot per 128 x 128 tile of R_i (row block of r, 128 columns of d_out).
int tc_partials_per_sample(int r, int d_out) { return cdiv(r, kBM) * cdiv(d_out, 128); }

namespace {

// The wide projection's schedules: one per launch group, sized on the host with no
// device (grape_context_bytes) for at most kMaxSchedCtas CTAs.
constexpr int kMaxSchedCtas = 1024;

bool wide_projection(int r) { return r >= 256 && r % 256 == 0; }

int wide_tiles_of_group(const StepShape& sh, int n_layers) {
  const int64_t rows = static_cast<int64_t>(sh.B) * sh.T;
  return n_layers * cdiv(rows, 2 * kBM) * (sh.r / 256);
}

size_t schedule_bytes(const StepShape& sh) {
  if (!wide_projection(sh.r)) return 0;
  size_t b = 0;
  for (int l0 = 0; l0 < sh.L; l0 += kMaxGroup) {
    const int n = (sh.L - l0) < kMaxGroup ? (sh.L - l0) : kMaxGroup;
    b += static_cast<size_t>(wide_tiles_of_group(sh, n) + kMaxSchedCtas + 1) * 4;
  }
  return (b + 255) & ~size_t(255);
}

// LPT list scheduling of one launch group's tiles over `grid` CTAs: tiles in descending
// k-blocks (stable), each to the CTA with the least k-blocks so far (the lowest index on
// ties); each CTA runs its tiles in the order they were given.  out = the order, then
// the CTAs' first positions (grid + 1 ints).
std::vector<int> lpt_schedule(const std::vector<int>& work, int grid) {
  const int n = static_cast<int>(work.size());
  std::vector<int> idx(n);
  for (int t = 0; t < n; ++t) idx[t] = t;
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return work[a] > work[b]; });
  std::vector<std::vector<int>> lists(grid);
  std::vector<std::pair<int64_t, int>> heap;   // (load, cta), a min-heap
  for (int b = 0; b < grid; ++b) heap.push_back({0, b});
  auto cmp = [](const std::pair<int64_t, int>& x, const std::pair<int64_t, int>& y) { return x > y; };
  std::make_heap(heap.begin(), heap.end(), cmp);
  for (int t : idx) {
    std::pop_heap(heap.begin(), heap.end(), cmp);
    auto& top = heap.back();
    lists[top.second].push_back(t);
    top.first += work[t];
    std::push_heap(heap.begin(), heap.end(), cmp);
  }
  std::vector<int> out;
  out.reserve(n + grid + 1);
  std::vector<int> begin(grid + 1, 0);
  for (int b = 0; b < grid; ++b) {
    begin[b] = static_cast<int>(out.size());
    out.insert(out.end(), lists[b].begin(), lists[b].end());
  }
  begin[grid] = static_cast<int>(out.size());
  out.insert(out.end(), begin.begin(), begin.end());
  return out;
}

}  // namespace

size_t tc_workspace_bytes(const StepShape& sh, const LayerWs*) {
  return 256 + schedule_bytes(sh);  // error word, then the wide projection's schedules
}

cudaError_t tc_init(const StepShape& sh, const LayerWs* ws, void* scratch, size_t bytes,
                    TcWorkspace* out) {
  HostState* hs = new HostState();
  hs->L = sh.L;
  hs->r = sh.r;
  hs->B = sh.B;
  hs->T = sh.T;
  hs->bn_project = sh.r == 128 ? 128 : 256;
  if (const char* v = std::getenv("GRAPE_NORM_TMEM")) hs->norm_tmem = std::strcmp(v, "0") == 0 ? 0 : 1;
  if (const char* v = std::getenv("GRAPE_PROJECT_WIDE")) hs->project_wide = std::strcmp(v, "0") != 0;
  char* base = static_cast<char*>(scratch);
  size_t off = 0;
  hs->err = reinterpret_cast<int*>(base + off);
  off += 256;
  hs->mapP_mn.resize(sh.L);
  hs->mapP_k.resize(sh.L);
  hs->mapAP3.resize(sh.L);
  hs->mapAP3k.resize(sh.L);
  hs->mapAP2.resize(sh.L);
  hs->mapDR.resize(sh.L);
  hs->cacheA.resize(sh.L);
  hs->cacheG3.resize(sh.L);
  hs->cacheG3k.resize(sh.L);
  hs->cacheG2.resize(sh.L);
  hs->cacheW.resize(sh.L);
  hs->cacheWs.resize(sh.L);
  const uint64_t rows = static_cast<uint64_t>(sh.B) * sh.T;
  for (int l = 0; l < sh.L; ++l) {
    hs->d_in.push_back(ws[l].d_in);
    hs->d_out.push_back(ws[l].d_out);
    bool ok = map_2d(&hs->mapP_mn[l], ws[l].P16, ws[l].d_in, sh.r, 64, 64) &&
              map_2d(&hs->mapP_k[l], ws[l].P16, ws[l].d_in, sh.r, 64, kBM) &&
              map_3d(&hs->mapAP3[l], ws[l].AP, sh.B, sh.T, sh.r) &&
              map_3d(&hs->mapAP3k[l], ws[l].AP, sh.B, sh.T, sh.r, kBM) &&
              map_2d(&hs->mapAP2[l], ws[l].AP, rows, sh.r, 64, 64) &&
              map_2d(&hs->mapDR[l], ws[l].dR, sh.r, ws[l].d_out, 64, 64);
    if (!ok) {
      delete hs;
      return cudaErrorInvalidValue;
    }
  }
  if (wide_projection(sh.r)) {
    // the wide projection's LPT schedules, one per launch group, for the grid it will
    // launch (one CTA per SM, never more than there are tiles)
    int per_sm = 0;
    cudaError_t e = configure_kernel(reinterpret_cast<const void*>(tc_project_wide_kernel), PwSmem::kBytes,
                                     kPwThreads, &per_sm);
    if (e != cudaSuccess) {
      delete hs;
      return e;
    }
    const int ctas = std::min(sm_count() * per_sm, kMaxSchedCtas);
    const int64_t rows = static_cast<int64_t>(sh.B) * sh.T;
    char* sb = base + off;
    for (int l0 = 0; l0 < sh.L; l0 += kMaxGroup) {
      const int n = (sh.L - l0) < kMaxGroup ? (sh.L - l0) : kMaxGroup;
      std::vector<int> work;   // k-blocks of each tile, numbered as tc_project numbers them
      for (int g = 0; g < n; ++g)
        work.insert(work.end(), static_cast<size_t>(cdiv(rows, 2 * kBM)) * (sh.r / 256),
                    cdiv(ws[l0 + g].d_in, kBK));
      const int grid = std::min(ctas, static_cast<int>(work.size()));
      const std::vector<int> sched = lpt_schedule(work, grid);
      e = cudaMemcpy(sb, sched.data(), sched.size() * sizeof(int), cudaMemcpyHostToDevice);
      if (e != cudaSuccess) {
        delete hs;
        return e;
      }
      hs->sched.push_back(reinterpret_cast<const int*>(sb));
      hs->sched_grid.push_back(grid);
      sb += static_cast<size_t>(wide_tiles_of_group(sh, n) + kMaxSchedCtas + 1) * 4;
    }
    off += schedule_bytes(sh);
  }
  if (off > bytes) {
    delete hs;
    return cudaErrorInvalidValue;
  }
  out->base = scratch;
  out->bytes = bytes;
  out->host_state = hs;
  return cudaSuccess;
}

void tc_release(TcWorkspace* tc) {
  if (tc && tc->host_state) {
    delete static_cast<HostState*>(tc->host_state);
    tc->host_state = nullptr;
  }
}

int* tc_error_word(const TcWorkspace& tc) {
  return tc.host_state ? static_cast<HostState*>(tc.host_state)->err : nullptr;
}

namespace {
PTable make_p_table(const StepShape& sh, const LayerWs* ws) {
  PTable t{};
  int64_t at = 0;
  for (int l = 0; l < sh.L; ++l) {
    t.P16[l] = ws[l].P16;
    t.begin[l] = at;
    at += static_cast<int64_t>(ws[l].d_in) * sh.r / 4;   // r is a multiple of 64
  }
  t.begin[sh.L] = at;
  t.L = sh.L;
  return t;
}
}  // namespace

cudaError_t tc_generate_P(const StepShape& sh, const LayerWs* ws, const TcWorkspace&, uint32_t step,
                          cudaStream_t st, int* launches) {
  const PTable t = make_p_table(sh, ws);
  // 8 resident 256-thread blocks per SM, never more than there are units
  int64_t gx = (t.begin[sh.L] + 255) / 256;
  const int64_t fill = static_cast<int64_t>(sm_count()) * 8;
  gx = gx < fill ? gx : fill;
  gen_P_bf16_kernel<<<static_cast<unsigned>(gx > 0 ? gx : 1), 256, 0, st>>>(t, sh.seed, step, sh.r);
  ++*launches;
  return cudaGetLastError();
}

const void* tc_gen_P_func() { return reinterpret_cast<const void*>(gen_P_bf16_kernel); }

cudaError_t tc_generate_P_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                   const LayerWs* ws, uint32_t key) {
  cudaKernelNodeParams p{};
  cudaError_t e = cudaGraphKernelNodeGetParams(node, &p);
  if (e != cudaSuccess) return e;
  PTable a0 = make_p_table(sh, ws);
  uint64_t a1 = sh.seed;
  uint32_t a2 = key;
  int a3 = sh.r;
  void* args[] = {&a0, &a1, &a2, &a3};
  p.kernelParams = args;
  p.extra = nullptr;
  return cudaGraphExecKernelNodeSetParams(exec, node, &p);
}

namespace {

// Persistent, on the grid its schedule (gp.sched) was built for at tc_init.
cudaError_t launch_project_wide(GroupParams& gp, int tiles, int grid, cudaStream_t st, bool pdl) {
  int per_sm = 0;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(tc_project_wide_kernel), PwSmem::kBytes,
                                   kPwThreads, &per_sm);
  if (e != cudaSuccess) return e;
  gp.total_tiles = tiles;
  if (tiles <= 0) return cudaSuccess;
  return launch_maybe_pdl(pdl, tc_project_wide_kernel, dim3(grid), dim3(kPwThreads), PwSmem::kBytes, st, gp);
}

}  // namespace

cudaError_t tc_project(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                       const TcWorkspace& tc, cudaStream_t st, int* launches, bool first_in_step) {
  HostState& hs = *static_cast<HostState*>(tc.host_state);
  GroupParams& gp = hs.gp;
  std::memset(&gp, 0, sizeof(gp));
  gp.err = hs.err;
  const int64_t rows = static_cast<int64_t>(sh.B) * sh.T;
  auto fill = [&](int g, int l, int* tiles) {
    if (!hs.cacheA[l].get(io[l].A, &gp.mapA[g], [&](CUtensorMap* m) {
          return map_2d(m, io[l].A, rows, ws[l].d_in, 64, kBM);
        }))
      return false;
    gp.mapB[g] = hs.mapP_mn[l];
    GRAPE_EXT(gp.extA[g], ws[l].d_in, rows, 1)
    GRAPE_EXT(gp.extB[g], sh.r, ws[l].d_in, 1)
    GroupLayer& L = gp.lay[g];
    L.mt = cdiv(rows, kBM);
    L.nt = sh.r / hs.bn_project;
    L.ns = 1;
    L.kblocks = cdiv(ws[l].d_in, kBK);
    L.M = static_cast<int>(rows);
    L.N = sh.r;
    L.ldo = sh.r;
    L.out = ws[l].AP;
    *tiles = L.mt * L.nt;
    return true;
  };
  if (hs.bn_project == 128)
    return run_mode<PROJECT, 128, kStagesProject128>(hs, sh.L, st, launches, fill, gp, !first_in_step);
  if (!hs.project_wide)
    return run_mode<PROJECT, 256, kStagesProject256>(hs, sh.L, st, launches, fill, gp, !first_in_step);
  // 256-row tiles (tc_project_wide_kernel)
  for (int l0 = 0; l0 < sh.L; l0 += kMaxGroup) {
    const int n = (sh.L - l0) < kMaxGroup ? (sh.L - l0) : kMaxGroup;
    gp.n_layers = n;
    int tiles = 0;
    for (int g = 0; g < n; ++g) {
      int t = 0;
      if (!fill(g, l0 + g, &t)) return cudaErrorInvalidValue;
      GroupLayer& L = gp.lay[g];
      L.mt = cdiv(rows, 2 * kBM);
      L.tiles_begin = tiles;
      tiles += L.mt * L.nt;
    }
    const size_t gi = static_cast<size_t>(l0 / kMaxGroup);
    if (gi >= hs.sched.size()) return cudaErrorInvalidValue;
    gp.sched = hs.sched[gi];
    cudaError_t e = launch_project_wide(gp, tiles, hs.sched_grid[gi], st, l0 == 0 ? !first_in_step : true);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

namespace {

cudaError_t launch_norm_tmem(NtParams& np, cudaStream_t st) {
  using S = NtSmem;
  const void* kern = reinterpret_cast<const void*>(tc_norm_tmem_kernel);
  int per_sm = 0;
  cudaError_t e = configure_kernel(kern, S::kBytes, kNtThreads, &per_sm);
  if (e != cudaSuccess) return e;
  int most = 0;   // no more groups than the largest span has column tiles
  for (int k = 0; k < np.n_spans; ++k) most = std::max(most, np.span_tiles[k]);
  if (most <= 0) return cudaSuccess;
  int groups = sm_count() * per_sm / np.mr;   // one CTA per SM (the kernel allocates TMEM)
  groups = std::max(1, std::min(groups, most));
  np.groups = groups;
  int rot = 0;
  for (int k = 0; k < np.n_spans; ++k) {
    np.span_rot[k] = rot;
    rot = ((rot - np.span_tiles[k] % groups) % groups + groups) % groups;
  }
  return launch_maybe_pdl(true, tc_norm_tmem_kernel, dim3(groups * np.mr), dim3(kNtThreads), S::kBytes, st, np);
}

}  // namespace

// The norm kernel with (A_i P)^T in TMEM stores R_i and holds a block of
// ceil(T / 64) * 32 columns next to its accumulator: T up to 512.  Against
// tc_gemm_kernel<NORMST> it measured faster from T = 257 on (7B slice, T = 512: 1.37
// against 1.52 ms per step's norms) and slower at ViT-B's T = 197, where its block
// changes more often per tile.  `mode` is the GRAPE_NORM_TMEM knob: 0 never, 1 for
// every T it can take, -1 (unset) by that measurement.
bool tc_norm_a_in_tmem(int T, bool store_R, int mode) {
  if (!store_R || mode == 0 || T < 1 || T > 512) return false;
  return mode == 1 || T > 256;
}

cudaError_t tc_project_norm(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                            const TcWorkspace& tc, float* partials, bool store_R, cudaStream_t st,
                            int* launches) {
  HostState& hs = *static_cast<HostState*>(tc.host_state);
  if (tc_norm_a_in_tmem(sh.T, store_R, hs.norm_tmem)) {
    NtParams& np = hs.np;
    for (int l0 = 0; l0 < sh.L; l0 += kMaxGroup) {
      const int n = (sh.L - l0) < kMaxGroup ? (sh.L - l0) : kMaxGroup;
      std::memset(&np, 0, sizeof(np));
      np.err = hs.err;
      np.partials = partials;
      np.part_stride = sh.part_stride;
      np.r = sh.r;
      np.mr = cdiv(sh.r, kBM);
      np.kblocks = cdiv(sh.T, kBK);
      np.n_layers = n;
      // one span: the groups share nothing, so each takes one contiguous range of the
      // whole launch (the fewest unit starts)
      np.n_spans = 1;
      np.span_first[0] = 0;
      np.span_first[1] = n;
      int tiles = 0;
      for (int g = 0; g < n; ++g) {
        const int l = l0 + g;
        np.mapAP[g] = hs.mapAP3[l];
        if (!hs.cacheG3[l].get(io[l].G, &np.mapG[g], [&](CUtensorMap* m) {
              return map_3d(m, io[l].G, sh.B, sh.T, ws[l].d_out);
            }))
          return cudaErrorInvalidValue;
        if (!ws[l].Rst) return cudaErrorInvalidValue;
        GRAPE_EXT(np.extAP[g], sh.r, sh.T, sh.B)
        GRAPE_EXT(np.extG[g], ws[l].d_out, sh.T, sh.B)
        NtLayer& L = np.lay[g];
        L.tiles_begin = tiles;
        L.nt = cdiv(ws[l].d_out, kNtBN);   // d_out % 256 == 0 on this path
        L.d_out = ws[l].d_out;
        L.part_base = ws[l].part_base;
        L.Rst = ws[l].Rst;
        tiles += sh.B * L.nt;
      }
      np.span_tiles[0] = tiles;
      cudaError_t e = launch_norm_tmem(np, st);
      if (e != cudaSuccess) return e;
      ++*launches;
    }
    return cudaSuccess;
  }
  GroupParams& gp = hs.gp;
  std::memset(&gp, 0, sizeof(gp));
  gp.err = hs.err;
  gp.partials = partials;
  gp.part_stride = sh.part_stride;
  auto fill = [&](int g, int l, int* tiles) {
    gp.mapA[g] = hs.mapAP3[l];
    if (!hs.cacheG3[l].get(io[l].G, &gp.mapB[g], [&](CUtensorMap* m) {
          return map_3d(m, io[l].G, sh.B, sh.T, ws[l].d_out);
        }))
      return false;
    if (store_R && !ws[l].Rst) return false;
    GRAPE_EXT(gp.extA[g], sh.r, sh.T, sh.B)
    GRAPE_EXT(gp.extB[g], ws[l].d_out, sh.T, sh.B)
    GroupLayer& L = gp.lay[g];
    L.mt = cdiv(sh.r, kBM);
    L.nt = cdiv(ws[l].d_out, kBnWide);
    L.ns = sh.B;
    L.kblocks = cdiv(sh.T, kBK);
    L.M = sh.r;
    L.N = ws[l].d_out;
    L.part_base = ws[l].part_base;
    L.out = store_R ? ws[l].Rst : nullptr;   // R_l as [B][r][d_out] bf16
    L.ldo = ws[l].d_out;
    *tiles = L.mt * L.nt * sh.B;
    return true;
  };
  if (store_R) return run_mode<NORMST, kBnWide, kStagesNorm>(hs, sh.L, st, launches, fill, gp);
  return run_mode<NORM, kBnWide, kStagesNorm>(hs, sh.L, st, launches, fill, gp);
}

bool tc_ghost_supported(const StepShape& sh) { (void)sh; return true; }

// Per-sample squared norms by the ghost identity ||(A_i P)^T Gout_i||^2 =
// <(A_i P)(A_i P)^T, Gout_i Gout_i^T>_F: one tile per (sample, layer), which runs over the
// pairs a <= b of 128-token blocks of the sample, each a 128 x 128 block of both T x T
// Gram matrices (off-diagonal blocks counted twice, for their transposes).
cudaError_t tc_project_norm_ghost(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                                  const TcWorkspace& tc, float* partials, cudaStream_t st, int* launches) {
  HostState& hs = *static_cast<HostState*>(tc.host_state);
  GroupParams& gp = hs.gp;
  std::memset(&gp, 0, sizeof(gp));
  gp.err = hs.err;
  gp.partials = partials;
  gp.part_stride = sh.part_stride;
  auto fill = [&](int g, int l, int* tiles) {
    gp.mapA[g] = hs.mapAP3k[l];
    if (!hs.cacheG3k[l].get(io[l].G, &gp.mapB[g], [&](CUtensorMap* m) {
          return map_3d(m, io[l].G, sh.B, sh.T, ws[l].d_out, kBM);
        }))
      return false;
    GRAPE_EXT(gp.extA[g], sh.r, sh.T, sh.B)
    GRAPE_EXT(gp.extB[g], ws[l].d_out, sh.T, sh.B)
    GroupLayer& L = gp.lay[g];
    L.mt = 1;
    L.nt = 1;
    L.ns = sh.B;
    L.kfirst = cdiv(ws[l].d_out, kBK);
    L.kblocks = L.kfirst + cdiv(sh.r, kBK);
    L.nb = cdiv(sh.T, kBM);
    L.M = sh.T;
    L.N = sh.T;
    L.part_base = ws[l].part_base;
    L.slots = tc_partials_per_sample(sh.r, ws[l].d_out);
    *tiles = sh.B;
    return true;
  };
  return run_mode<GHOST, kBM, kStagesGhost>(hs, sh.L, st, launches, fill, gp);
}

cudaError_t tc_clip_scale(const StepShape& sh, const LayerWs* ws, const TcWorkspace&,
                          const float* partials, float* norms, float* clip, bool rescale_ap,
                          cudaStream_t st, int* launches) {
  ApTable t{};
  for (int l = 0; l < sh.L; ++l) t.AP[l] = static_cast<__nv_bfloat16*>(ws[l].AP);
  ++*launches;
  return launch_pdl(clip_scale_kernel, dim3(sh.B, rescale_ap ? sh.L : 1), dim3(256), 0, st, t, sh.r, sh.T,
                    sh.part_stride, sh.C, partials, norms, clip, rescale_ap ? 1 : 0);
}

cudaError_t tc_aggregate_stored(const StepShape& sh, const LayerWs* ws, const float* clip, cudaStream_t st,
                                int* launches) {
  StoredAggTable t{};
  int64_t at = 0;
  for (int l = 0; l < sh.L; ++l) {
    if (!ws[l].Rst) return cudaErrorInvalidValue;
    t.R[l] = ws[l].Rst;
    t.S[l] = ws[l].S;
    t.begin[l] = at;
    at += static_cast<int64_t>(sh.r) * ws[l].d_out / 8;   // d_out % 256 == 0 on this path
  }
  t.begin[sh.L] = at;
  // enough 256-thread blocks to fill every SM (8 per SM), never more than there are units
  int64_t blocks = (at + 255) / 256;
  const int64_t fill = static_cast<int64_t>(sm_count()) * 8;
  blocks = blocks < fill ? blocks : fill;
  ++*launches;
  return launch_pdl(aggregate_stored_kernel, dim3(static_cast<unsigned>(blocks > 0 ? blocks : 1)), dim3(256), 0,
                    st, t, sh.L, sh.B, clip);
}

namespace {

AggAdamTable make_agg_adam_table(const StepShape& sh, const LayerWs* ws) {
  AggAdamTable t{};
  int64_t at = 0;
  for (int l = 0; l < sh.L; ++l) {
    t.R[l] = ws[l].Rst;
    t.S[l] = ws[l].S;
    t.m[l] = ws[l].m;
    t.v[l] = ws[l].v;
    t.dR[l] = static_cast<__nv_bfloat16*>(ws[l].dR);
    t.begin[l] = at;
    at += static_cast<int64_t>(sh.r) * ws[l].d_out / 8;   // r % 128 == 0 on this path
  }
  t.begin[sh.L] = at;
  return t;
}

// enough 256-thread blocks to fill every SM (8 per SM), never more than there are units
unsigned agg_adam_blocks(const AggAdamTable& t, int L) {
  int64_t blocks = (t.begin[L] + 255) / 256;
  const int64_t fill = static_cast<int64_t>(sm_count()) * 8;
  blocks = blocks < fill ? blocks : fill;
  return static_cast<unsigned>(blocks > 0 ? blocks : 1);
}

}  // namespace

cudaError_t tc_aggregate_adam(const StepShape& sh, const LayerWs* ws, const UpdateScalars& u, const float* clip,
                              cudaStream_t st, int* launches) {
  for (int l = 0; l < sh.L; ++l)
    if (!ws[l].Rst) return cudaErrorInvalidValue;
  const AggAdamTable t = make_agg_adam_table(sh, ws);
  ++*launches;
  return launch_pdl(aggregate_adam_kernel, dim3(agg_adam_blocks(t, sh.L)), dim3(256), 0, st, sh, t, u, clip);
}

const void* tc_aggregate_adam_func() { return reinterpret_cast<const void*>(aggregate_adam_kernel); }

cudaError_t tc_aggregate_adam_set_node(cudaGraphExec_t exec, cudaGraphNode_t node, const StepShape& sh,
                                       const LayerWs* ws, const UpdateScalars& u, const float* clip) {
  cudaKernelNodeParams p{};
  cudaError_t e = cudaGraphKernelNodeGetParams(node, &p);
  if (e != cudaSuccess) return e;
  StepShape a0 = sh;
  AggAdamTable a1 = make_agg_adam_table(sh, ws);
  UpdateScalars a2 = u;
  const float* a3 = clip;
  void* args[] = {&a0, &a1, &a2, &a3};
  p.kernelParams = args;
  p.extra = nullptr;
  return cudaGraphExecKernelNodeSetParams(exec, node, &p);
}

namespace {

// How many clusters of `cs` CTAs of the aggregation kernel the device holds at once.
// (cached per device and cluster size, 0 when the size cannot run)
template <int BN, int STAGES>
int clusters_resident(int cs) {
  if (cs < 1 || cs > 8) return 0;
  using S = Smem<BN, STAGES>;
  const void* kern = reinterpret_cast<const void*>(tc_agg_cluster_kernel<BN, STAGES>);
  int per_sm = 0;
  if (configure_kernel(kern, S::kBytes, kThreads, &per_sm) != cudaSuccess) return 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_launch_cfg_mu);
  int& cached = g_launch_cfg[std::make_tuple(dev, kern, 100 + cs)];   // stored as count + 1
  if (cached == 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = S::kBytes;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = cs;
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, tc_agg_cluster_kernel<BN, STAGES>, &cfg);
    if (e != cudaSuccess) cudaGetLastError();
    cached = 1 + ((e == cudaSuccess) ? n : 0);
  }
  return cached - 1;
}

template <int BN, int STAGES>
cudaError_t launch_agg_cluster(GroupParams& gp, int tiles, int cs, cudaStream_t st) {
  using S = Smem<BN, STAGES>;
  int per_sm = 0;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(tc_agg_cluster_kernel<BN, STAGES>),
                                   S::kBytes, kThreads, &per_sm);
  if (e != cudaSuccess) return e;
  gp.total_tiles = tiles;
  gp.cluster = cs;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(tiles * cs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = S::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute a[2];
  a[0].id = cudaLaunchAttributeClusterDimension;
  a[0].val.clusterDim.x = cs;
  a[0].val.clusterDim.y = 1;
  a[0].val.clusterDim.z = 1;
  a[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = a;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tc_agg_cluster_kernel<BN, STAGES>, gp);
}

}  // namespace

cudaError_t tc_aggregate(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                         const TcWorkspace& tc, const float* clip, cudaStream_t st, int* launches) {
  (void)clip;   // folded into AP by tc_clip_scale
  HostState& hs = *static_cast<HostState*>(tc.host_state);
  GroupParams& gp = hs.gp;
  const int64_t rows = static_cast<int64_t>(sh.B) * sh.T;
  for (int l0 = 0; l0 < sh.L; l0 += kMaxGroup) {
    const int n = (sh.L - l0) < kMaxGroup ? (sh.L - l0) : kMaxGroup;
    // Output tiles of this group at the persistent kernel's width: with at least one
    // tile per SM the persistent kernel runs K whole; with fewer, K is split over a
    // cluster (the largest of 8, 4, 2 whose clusters are all resident at once).
    int wide_tiles = 0;
    for (int g = 0; g < n; ++g) wide_tiles += cdiv(sh.r, kBM) * cdiv(ws[l0 + g].d_out, kBnWide);
    int cs = 1, narrow_tiles = 0;
    if (wide_tiles < sm_count()) {
      for (int g = 0; g < n; ++g) narrow_tiles += cdiv(sh.r, kBM) * cdiv(ws[l0 + g].d_out, kBnAggCluster);
      for (int cand = 8; cand >= 2; cand /= 2)
        if (narrow_tiles <= clusters_resident<kBnAggCluster, kStagesAggCluster>(cand)) {
          cs = cand;
          break;
        }
    }
    const int bn = (cs > 1) ? kBnAggCluster : kBnWide;
    if (std::getenv("GRAPE_DEBUG_PLAN"))
      std::fprintf(stderr, "grape: aggregate layers %d..%d: %d wide tiles, cluster %d (resident clusters of 8/4/2: %d/%d/%d)\n",
                   l0, l0 + n - 1, wide_tiles, cs, clusters_resident<kBnAggCluster, kStagesAggCluster>(8),
                   clusters_resident<kBnAggCluster, kStagesAggCluster>(4),
                   clusters_resident<kBnAggCluster, kStagesAggCluster>(2));
    std::memset(&gp, 0, sizeof(gp));
    gp.err = hs.err;
    gp.n_layers = n;
    int tiles = 0;
    for (int g = 0; g < n; ++g) {
      const int l = l0 + g;
      gp.mapA[g] = hs.mapAP2[l];
      if (!hs.cacheG2[l].get(io[l].G, &gp.mapB[g], [&](CUtensorMap* m) {
            return map_2d(m, io[l].G, rows, ws[l].d_out, 64, 64);
          }))
        return cudaErrorInvalidValue;
      GRAPE_EXT(gp.extA[g], sh.r, rows, 1)
      GRAPE_EXT(gp.extB[g], ws[l].d_out, rows, 1)
      GroupLayer& L = gp.lay[g];
      L.tiles_begin = tiles;
      L.mt = cdiv(sh.r, kBM);
      L.nt = cdiv(ws[l].d_out, bn);
      L.ns = 1;
      L.kblocks = cdiv(rows, kBK);
      L.M = sh.r;
      L.N = ws[l].d_out;
      L.ldo = ws[l].d_out;
      L.out = ws[l].S;
      tiles += L.mt * L.nt;
    }
    cudaError_t e = (cs > 1) ? launch_agg_cluster<kBnAggCluster, kStagesAggCluster>(gp, tiles, cs, st)
                             : launch_group<AGGREGATE, kBnWide, kStagesAgg>(gp, tiles, st);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

namespace {

template <int PK>
cudaError_t launch_backproj_tmem(BptParams& bp, cudaStream_t st) {
  using S = BptSmem<kBptDRS, kBptNW>;
  const void* kern = reinterpret_cast<const void*>(tc_backproj_tmem_kernel<PK>);
  int per_sm = 0;
  cudaError_t e = configure_kernel(kern, S::kBytes, kBptThreads, &per_sm);
  if (e != cudaSuccess) return e;
  int most = 0;   // no more CTAs than the largest span has tiles
  for (int k = 0; k < bp.n_spans; ++k) most = std::max(most, bp.span_tiles[k]);
  if (most <= 0) return cudaSuccess;
  int grid = sm_count() * per_sm;
  grid = grid < most ? grid : most;
  // the CTAs that take a span's extra tiles follow on from those of the span before
  int rot = 0;
  for (int k = 0; k < bp.n_spans; ++k) {
    bp.span_rot[k] = rot;
    rot = ((rot - bp.span_tiles[k] % grid) % grid + grid) % grid;
  }
  return launch_maybe_pdl(true, tc_backproj_tmem_kernel<PK>, dim3(grid), dim3(kBptThreads), S::kBytes, st,
                          bp);
}

}  // namespace

// The kernel with P in TMEM measured faster at r = 512 (the 7B slice: 1.73 against
// 1.81-1.94 ms per step's back-projection) and slower at r = 256 and 128 (ViT-B: 172
// against 150-157 us; long context: 192 against 169-176 us; MLP: 14.7 against
// 13.8-14.8 us), where the streamed kernel's P tile is small.
bool tc_backproj_p_in_tmem(int r) { return r == 512; }

cudaError_t tc_backproject_streamed(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                                    const TcWorkspace& tc, float lr, cudaStream_t st, int* launches);

cudaError_t tc_backproject(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                           const TcWorkspace& tc, float lr, cudaStream_t st, int* launches) {
  if (!tc_backproj_p_in_tmem(sh.r)) return tc_backproject_streamed(sh, ws, io, tc, lr, st, launches);
  HostState& hs = *static_cast<HostState*>(tc.host_state);
  BptParams& bp = hs.bp;
  for (int l0 = 0; l0 < sh.L; l0 += kMaxGroup) {
    const int n = (sh.L - l0) < kMaxGroup ? (sh.L - l0) : kMaxGroup;
    std::memset(&bp, 0, sizeof(bp));
    bp.err = hs.err;
    bp.lr = lr;
    bp.r = sh.r;
    bp.n_layers = n;
    const int grid_full = sm_count();   // one CTA per SM (the kernel allocates TMEM)
    int span_tiles = 0;
    for (int g = 0; g < n; ++g) {
      const int l = l0 + g;
      bp.mapP[g] = hs.mapP_k[l];
      bp.mapDR[g] = hs.mapDR[l];
      if (!hs.cacheW[l].get(io[l].W, &bp.mapW[g], [&](CUtensorMap* m) {
            return map_2d_f32(m, io[l].W, ws[l].d_in, ws[l].d_out);
          }) ||
          !hs.cacheWs[l].get(io[l].W, &bp.mapWs[g], [&](CUtensorMap* m) {
            return map_2d_f32(m, io[l].W, ws[l].d_in, ws[l].d_out, 32);
          }))
        return cudaErrorInvalidValue;
      GRAPE_EXT(bp.extP[g], sh.r, ws[l].d_in, 1)
      GRAPE_EXT(bp.extDR[g], ws[l].d_out, sh.r, 1)
      GRAPE_EXT(bp.extW[g], ws[l].d_out, ws[l].d_in, 1)
      BptLayer& L = bp.lay[g];
      L.M = ws[l].d_in;
      L.mt = cdiv(ws[l].d_in, kBM);
      L.nt = cdiv(ws[l].d_out, kBnBack);
      // spans of at least four tiles per CTA
      if (span_tiles == 0) bp.span_first[bp.n_spans] = g;
      L.tiles_begin = span_tiles;
      span_tiles += L.mt * L.nt;
      if (span_tiles >= 4 * grid_full || g == n - 1) {
        bp.span_tiles[bp.n_spans++] = span_tiles;
        span_tiles = 0;
      }
    }
    bp.span_first[bp.n_spans] = n;
    cudaError_t e = launch_backproj_tmem<8>(bp, st);   // r = 512: a 256-column P block
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

// W -= lr P dR with P loaded by TMA with every tile (tc_gemm_kernel<BACKPROJ>): the
// projection widths whose P block does not fit in TMEM next to the accumulators.
cudaError_t tc_backproject_streamed(const StepShape& sh, const LayerWs* ws, const LayerIo* io,
                                    const TcWorkspace& tc, float lr, cudaStream_t st, int* launches) {
  HostState& hs = *static_cast<HostState*>(tc.host_state);
  GroupParams& gp = hs.gp;
  std::memset(&gp, 0, sizeof(gp));
  gp.err = hs.err;
  gp.lr = lr;
  auto fill = [&](int g, int l, int* tiles) {
    gp.mapA[g] = hs.mapP_k[l];
    gp.mapB[g] = hs.mapDR[l];
    GRAPE_EXT(gp.extA[g], sh.r, ws[l].d_in, 1)
    GRAPE_EXT(gp.extB[g], ws[l].d_out, sh.r, 1)
    GRAPE_EXT(gp.extW[g], ws[l].d_out, ws[l].d_in, 1)
    if (!hs.cacheW[l].get(io[l].W, &gp.mapW[g], [&](CUtensorMap* m) {
          return map_2d_f32(m, io[l].W, ws[l].d_in, ws[l].d_out);
        }))
      return false;
    GroupLayer& L = gp.lay[g];
    L.mt = cdiv(ws[l].d_in, kBM);
    L.nt = cdiv(ws[l].d_out, kBnBack);
    L.ns = 1;
    L.kblocks = cdiv(sh.r, kBK);
    L.M = ws[l].d_in;
    L.N = ws[l].d_out;
    L.ldo = ws[l].d_out;
    L.out = io[l].W;
    *tiles = L.mt * L.nt;
    return true;
  };
  return run_mode<BACKPROJ, kBnBack, kStagesBack>(hs, sh.L, st, launches, fill, gp);
}

// ---------------------------------------------------------------------------------
// Per-sample squared norms of one layer with no allocation (grape_layer_sqnorms_static).
// ---------------------------------------------------------------------------------
namespace {

// The scratch of that entry point: a file-scope device array, present on every GPU
// that loads the library until the process exits.  Layout per call: error word |
// P (d_in x r bf16) | AP (B*T x r bf16) | norm partials (B x slots fp32).
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

// P of one layer with an explicit Philox layer index (the same normals as gen_P_bf16_kernel).
__global__ void __launch_bounds__(256) gen_P_layer_static_kernel(__nv_bfloat16* P16, int d_in, int r,
                                                                 uint64_t seed, uint32_t layer,
                                                                 uint32_t step) {
  const int64_t nq = static_cast<int64_t>(d_in) * r / 4;
  const float scale = rsqrtf(static_cast<float>(r));
  uint2* out = reinterpret_cast<uint2*>(P16);
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < nq;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 z = gaussian4_fast(seed, layer, step, kStreamProjection, static_cast<uint32_t>(q));
    out[q] = make_uint2(pack_bf16(z.x * scale, z.y * scale), pack_bf16(z.z * scale, z.w * scale));
  }
}

// out[i] = sum of sample i's partial slots in slot order; NaN if a bounded wait gave up.
__global__ void sum_slots_static_kernel(const float* partials, int slots, int B, const int* err,
                                        float* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B) return;
  float s = 0.0f;
  for (int k = 0; k < slots; ++k) s += partials[static_cast<size_t>(i) * slots + k];
  out[i] = (*err == 0) ? s : __int_as_float(0x7fc00000);
}

}  // namespace

size_t tc_static_scratch_bytes() { return kStaticScratchBytes; }

bool tc_tensor_maps_available() { return encode_fn() != nullptr; }

size_t tc_static_scratch_needed(int d_in, int d_out, int r, int B, int T) {
  const size_t slots = static_cast<size_t>(tc_partials_per_sample(r, d_out));
  return 256 + round256(static_cast<size_t>(d_in) * r * 2) +
         round256(static_cast<size_t>(B) * T * r * 2) + round256(static_cast<size_t>(B) * slots * 4);
}

cudaError_t tc_layer_sqnorms_static(const void* A, const void* G, int d_in, int d_out, int r, int B,
                                    int T, uint64_t seed, uint32_t layer, uint32_t step, float* out,
                                    cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* base_v = nullptr;
  {
    // First call on this device (which is current): take the array's device address.
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
      e = cudaGetSymbolAddress(&g_static_ptr[dev], g_static_scratch);
      if (e != cudaSuccess) {
        g_static_ptr[dev] = nullptr;
        return e;
      }
    }
    base_v = g_static_ptr[dev];
  }
  char* base = static_cast<char*>(base_v);
  int* err = reinterpret_cast<int*>(base);
  __nv_bfloat16* P16 = reinterpret_cast<__nv_bfloat16*>(base + 256);
  __nv_bfloat16* AP = reinterpret_cast<__nv_bfloat16*>(base + 256 + round256(static_cast<size_t>(d_in) * r * 2));
  float* partials = reinterpret_cast<float*>(reinterpret_cast<char*>(AP) +
                                             round256(static_cast<size_t>(B) * T * r * 2));
  const int slots = tc_partials_per_sample(r, d_out);
  const int64_t rows = static_cast<int64_t>(B) * T;

  // The error word is the only state that must start at zero; P, AP and every
  // partial slot are fully rewritten below.
  e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;

  int gx = cdiv(static_cast<int64_t>(d_in) * r / 4, 256);
  gx = gx < 1184 ? gx : 1184;
  gen_P_layer_static_kernel<<<gx, 256, 0, st>>>(P16, d_in, r, seed, layer, step);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  GroupParams gp;   // kernel parameters, staged on the host stack
  std::memset(&gp, 0, sizeof(gp));
  gp.err = err;
  gp.n_layers = 1;
  const int bnp = (r == 128) ? 128 : 256;
  // AP = A P
  if (!map_2d(&gp.mapA[0], A, rows, d_in, 64, kBM) || !map_2d(&gp.mapB[0], P16, d_in, r, 64, 64))
    return cudaErrorInvalidValue;
  GRAPE_EXT(gp.extA[0], d_in, rows, 1)
  GRAPE_EXT(gp.extB[0], r, d_in, 1)
  GroupLayer& L = gp.lay[0];
  L.tiles_begin = 0;
  L.mt = cdiv(rows, kBM);
  L.nt = r / bnp;
  L.ns = 1;
  L.kblocks = cdiv(d_in, kBK);
  L.M = static_cast<int>(rows);
  L.N = r;
  L.ldo = r;
  L.out = AP;
  e = (bnp == 128) ? launch_group<PROJECT, 128, kStagesProject128>(gp, L.mt * L.nt, st)
                   : launch_group<PROJECT, 256, kStagesProject256>(gp, L.mt * L.nt, st);
  if (e != cudaSuccess) return e;
  // ||(A_i P)^T Gout_i||^2 per sample, as partial slots
  std::memset(&gp, 0, sizeof(gp));
  gp.err = err;
  gp.n_layers = 1;
  gp.partials = partials;
  gp.part_stride = slots;
  if (!map_3d(&gp.mapA[0], AP, B, T, r) || !map_3d(&gp.mapB[0], G, B, T, d_out))
    return cudaErrorInvalidValue;
  GRAPE_EXT(gp.extA[0], r, T, B)
  GRAPE_EXT(gp.extB[0], d_out, T, B)
  L = GroupLayer{};
  L.mt = cdiv(r, kBM);
  L.nt = cdiv(d_out, kBnWide);
  L.ns = B;
  L.kblocks = cdiv(T, kBK);
  L.M = r;
  L.N = d_out;
  L.part_base = 0;
  e = launch_group<NORM, kBnWide, kStagesNorm>(gp, L.mt * L.nt * B, st);
  if (e != cudaSuccess) return e;
  sum_slots_static_kernel<<<cdiv(B, 128), 128, 0, st>>>(partials, slots, B, err, out);
  return cudaGetLastError();
}

}  // namespace grape
