/*
 * grape.h: C ABI of the B200 (sm_100a) DP-GRAPE projection step.
 *
 * The method ("Memory-Efficient Differentially Private Training with Gradient
 * Random Projection", gist.science/es/paper/2506.15588, Resumen Tecnico,
 * section "Metodologia: DP-GRAPE"): per linear layer l with weights
 * W_l (d_in x d_out), every sample's gradient G_i = A_i^T Gout_i is projected
 * onto a Gaussian matrix P_l (d_in x r) regenerated from a seed (design
 * choice 1), the projection comes before clipping and noise (design choice 2),
 * and Adam's moments live in the projected r x d_out space (design choice 3).
 * One step, as the closing paragraph of that section orders it:
 *
 *   P_l[k,j]  = z(seed, l, s, stream 0, e = k*r + j) / sqrt(r)
 *   R_{i,l}   = (A_{i,l} P_l)^T Gout_{i,l}              (G_i never formed)
 *   n_i       = sqrt(sum_l ||R_{i,l}||_F^2),  c_i = C/n_i if n_i > C else 1
 *   S_l       = sum_i c_i R_{i,l}
 *   g_l       = (S_l + sigma*C*xi_l) / B,  xi_l[j,n] = z(seed, l, s, stream 1, e = j*d_out + n)
 *   m, v      = Adam moments of g_l (r x d_out),  t = s + 1
 *   dR_l      = (m/(1-beta1^t)) / (sqrt(v/(1-beta2^t)) + eps)
 *   W_l      -= lr * P_l dR_l
 *
 * z(...) is a standard normal from Philox4x32-10 (Salmon et al., "Parallel
 * Random Numbers: As Easy as 1, 2, 3", SC'11) with key (seed lo, seed hi) and
 * counter (e/4, layer, step, stream), and Box-Muller: words (x0, x1) give
 * elements 4q, 4q+1 (cosine, sine), words (x2, x3) give 4q+2, 4q+3, with
 * u1 = (x_a + 1)/2^32 and u2 = x_b/2^32.  The normals are fp32, from the precise
 * logf, sqrtf and sincospif (grape_gaussian, the noise, the CUDA-core path's P),
 * except the tensor-core path's P, which is rounded to bf16 as it is written
 * and so takes the special-function unit's log and sine/cosine: at most about
 * 1e-3 from the exact transform where rho is that small, a few 1e-6 elsewhere.
 *
 * Conventions
 *  - Every device pointer is a CUDA device address on the context's device;
 *    host pointers are ordinary (preferably pinned) host memory.  A context is
 *    bound to the device current at grape_create: every call that launches,
 *    copies or synchronises returns GRAPE_EINVAL when another device is current.
 *  - Matrices are row-major.  A_l is B x T x d_in, Gout_l is B x T x d_out
 *    (samples contiguous, each sample's T token rows contiguous), in the
 *    context's input dtype (fp32, or bf16 as raw 16-bit patterns).  W_l is
 *    fp32 d_in x d_out.  Every device pointer must be 16-byte aligned.
 *  - The caller owns A, Gout, W and the stream; W is updated in place.  The
 *    library owns the Adam moments, the per-step projection scratch, the
 *    norms and the workspace, all allocated by grape_create and freed by
 *    grape_destroy.
 *  - All work is enqueued on the caller's stream; no call synchronises the
 *    device unless its comment says so.  Asynchronous faults surface as
 *    GRAPE_ECUDA from a later call.
 *  - Every function returns GRAPE_OK (0) or an error code; the reason is kept
 *    for grape_last_error(ctx).  A failed call leaves W, m and v unchanged
 *    unless it returns GRAPE_ECUDA.
 */
#ifndef GRAPE_H_
#define GRAPE_H_

#include <stdint.h>

#if defined(__GNUC__)
#define GRAPE_API __attribute__((visibility("default")))
#else
#define GRAPE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define GRAPE_OK 0
#define GRAPE_EINVAL 1        /* bad argument: null/misaligned pointer, bad size */
#define GRAPE_ENOMEM 2        /* device or host allocation failed */
#define GRAPE_ECUDA 3         /* a CUDA call failed (message in grape_last_error) */
#define GRAPE_ETIMEOUT 4      /* a bounded device-side wait gave up */
#define GRAPE_EUNSUPPORTED 5  /* the configuration has no kernel on this device */

#define GRAPE_MAX_LAYERS 64

enum grape_dtype { GRAPE_F32 = 0, GRAPE_BF16 = 1 };

/* Kernel family.  AUTO picks the tensor-core (tcgen05) path for bf16 inputs
 * and the fp32 CUDA-core path for fp32 inputs.  SIMT forces the fp32
 * CUDA-core kernels (exact fp32 arithmetic, any shape).  TC forces the
 * tcgen05 path and fails with GRAPE_EUNSUPPORTED where it does not apply. */
enum grape_path { GRAPE_PATH_AUTO = 0, GRAPE_PATH_SIMT = 1, GRAPE_PATH_TC = 2 };

typedef struct grape_ctx grape_ctx;                 /* opaque, library-owned */
typedef struct { int32_t d_in, d_out; } grape_layer;
typedef struct { double lr, beta1, beta2, eps; } grape_adam;

/* Create a context for a fixed stack of linear layers and a fixed batch shape.
 *  layers[n_layers]  layer shapes (1 <= n_layers <= GRAPE_MAX_LAYERS)
 *  r                 projection dimension, 1 <= r <= d_in of every layer
 *                    (reading: the pages only say r << d)
 *  C, sigma          clipping threshold (> 0) and noise multiplier (>= 0)
 *  seed              64-bit seed of the projection and noise streams
 *  adam              lr, beta1, beta2 in [0, 1), eps > 0
 *                    (scalars are taken in double; derived constants such as
 *                    1 - beta are formed in double before the kernels round
 *                    them to fp32)
 *  B, T              samples per batch and tokens per sample (>= 1)
 *  in_dtype          GRAPE_F32 or GRAPE_BF16 (A and Gout)
 *  path              enum grape_path
 * Allocates the Adam moments (zeroed) and the workspace on the current CUDA
 * device; synchronises that device once.  *out receives the handle.  The aggregation
 * method starts as GRAPE_AGG_AUTO resolves it (grape_set_aggregation). */
GRAPE_API int grape_create(const grape_layer* layers, int32_t n_layers, int32_t r, double C, double sigma,
                 uint64_t seed, const grape_adam* adam, int32_t B, int32_t T, int32_t in_dtype,
                 int32_t path, grape_ctx** out);

/* One full step s = step (>= 0; Adam uses t = s + 1) on `stream`
 * (a cudaStream_t, NULL = default stream).
 *  A[l], Gout[l]  device pointers of layer l's inputs (read only)
 *  W[l]           device pointer of layer l's fp32 weights (updated in place) */
GRAPE_API int grape_step(grape_ctx* ctx, const void* const* A, const void* const* Gout, float* const* W,
               int64_t step, void* stream);

/* The same step from HOST buffers: A and Gout are copied to library-owned
 * device staging on `stream` (allocated on first use), the step runs, and
 * the B per-sample norms n_i are copied to norms_host (may be NULL).  W
 * stays on the device.  Synchronises `stream` before returning, so the host
 * buffers may be reused and norms_host is valid on return. */
GRAPE_API int grape_step_host(grape_ctx* ctx, const void* const* A_host, const void* const* Gout_host,
                    float* const* W, int64_t step, float* norms_host, void* stream);

/* The data-parallel split of grape_step.  grape_accumulate runs the
 * projection, the per-sample norms, clipping and the aggregation, leaving
 * S_l = sum_i c_i R_{i,l} (fp32, r x d_out, row-major) in library memory,
 * whose device address grape_S_ptr returns.  A caller may all-reduce (sum)
 * every S_l across ranks, then grape_apply adds the noise, divides by
 * batch_total (the global batch; 0 means B), runs Adam and back-projects
 * onto W.  grape_step(ctx, ...) equals accumulate + apply(batch_total = B). */
GRAPE_API int grape_accumulate(grape_ctx* ctx, const void* const* A, const void* const* Gout, int64_t step,
                     void* stream);
GRAPE_API int grape_S_ptr(grape_ctx* ctx, int32_t layer, float** S_dev);
/* All S_l at once: they lie back to back in layer order (layer l at element offset
 * sum_{k<l} r * d_out_k, each r x d_out row-major, no padding), so one all-reduce of
 * *count fp32 elements from *S_dev sums every layer over the ranks.  Errors:
 * GRAPE_EINVAL for NULL arguments. */
GRAPE_API int grape_S_all(grape_ctx* ctx, float** S_dev, int64_t* count);
/* grape_apply(step) back-projects with the P of step's key (step / refresh period),
 * which must be the P the last grape_accumulate used and still the one in the scratch:
 * GRAPE_EINVAL when no accumulation ran, when the last one drew another key, or when
 * a later call (grape_sqnorms of another key, grape_set_refresh_period) replaced P. */
GRAPE_API int grape_apply(grape_ctx* ctx, float* const* W, int64_t step, int64_t batch_total, void* stream);

/* Live-token compaction for loss-masked inputs.  The pages are silent about
 * masks; a masked token contributes nothing to a sample's gradient (the
 * gradient of a linear layer is a sum over tokens), so dropping it before the
 * projection is an exact rewrite of the step of "Metodologia: DP-GRAPE"
 * (technical summary of "Memory-Efficient Differentially Private Training with
 * Gradient Random Projection") that removes the masked tokens' share of the
 * projection, norm and aggregation work.
 *
 * grape_enable_compaction: the context's T becomes the capacity (kept tokens per
 *   sample); steps given to grape_step_masked read inputs of T_full >= T tokens
 *   per sample.  Allocates B*T*(d_in + d_out) elements per layer of compact
 *   buffers (input dtype) and B*T + B + 1 int32 of bookkeeping, zeroed; call once.
 *   Errors: GRAPE_EINVAL (T_full < T, B > 65535, already enabled), GRAPE_ENOMEM.
 * grape_step_masked: as grape_step, with A[l], Gout[l] of shape B x T_full x d and
 *   mask_dev a device array of B x T_full bytes (row-major, nonzero = the token
 *   carries loss and is kept; one mask for all layers).  Each sample's kept tokens,
 *   in order, are gathered into T rows (zero padding after them) and the whole step
 *   runs on those.  The result equals grape_step on inputs whose masked tokens'
 *   Gout rows are zero.  A sample that keeps more than T tokens uses its first T
 *   and makes the next synchronising call (grape_live_counts, grape_debug,
 *   grape_step_host) return GRAPE_EINVAL.  Enqueued on `stream`.
 * grape_live_counts: synchronises the device and copies the kept-token count of
 *   each sample of the last masked step (at most T) to counts_host (B int32). */
GRAPE_API int grape_enable_compaction(grape_ctx* ctx, int32_t T_full);
GRAPE_API int grape_step_masked(grape_ctx* ctx, const void* const* A, const void* const* Gout,
                                float* const* W, const uint8_t* mask_dev, int64_t step, void* stream);
GRAPE_API int grape_live_counts(grape_ctx* ctx, int32_t* counts_host);

/* Self-test of the bounded waits every tensor-core kernel relies on; it faults and
 * hangs nothing.  One CTA waits on two mbarriers that nothing ever arrives on.  Warp 0
 * waits at most short_ns and must give up by itself, raising the CTA's abort flag.
 * Warp 1 waits at most long_ns and must give up early on that flag.  This is the
 * mechanism that turns a lost TMA load or MMA completion in a step into GRAPE_ETIMEOUT
 * with the context still usable.  *bits_out (may be NULL) receives 1 when warp 0 gave
 * up at its limit, plus 2 when warp 1 left on the abort flag (4 instead of 2 if it ran
 * to its own limit): 3 is the expected result.  Returns GRAPE_ETIMEOUT when warp 0 gave
 * up (the expected outcome) and GRAPE_OK otherwise.  Synchronises the current device.
 * Errors: GRAPE_EINVAL (need 0 <= short_ns <= 1e9 and short_ns <= long_ns <= 1e10),
 * GRAPE_ENOMEM, GRAPE_ECUDA. */
GRAPE_API int grape_selftest_wait_timeout(int64_t short_ns, int64_t long_ns, int32_t* bits_out);

/* CUDA-graph replay of grape_step (enable != 0; default off).  The step's launches
 * are captured once per set of A, Gout and W pointers (the first grape_step with a
 * set captures them on a library stream, then launches the graph), with
 * their programmatic dependencies, and replayed on the caller's stream (NULL
 * included); each replay rewrites the arguments that change with the step (P's
 * Philox key, Adam's step and bias corrections), so a replay computes exactly what
 * the ordinary launches compute, with one host call instead of one per kernel.  P is
 * regenerated on every replay (a refresh period then costs one P generation per step).
 * At most 8 pointer sets are kept (least recently used dropped).  Profiling
 * (grape_profile) runs the ordinary launches.  Disabling frees every graph.  Only
 * grape_step replays; the other entry points always launch directly. */
GRAPE_API int grape_set_graph(grape_ctx* ctx, int32_t enable);

/* How the per-sample squared norms ||R_i||^2 = ||(A_i P)^T Gout_i||_F^2 are formed.
 *  GRAPE_NORM_DIRECT  R_i tile by tile (r x 256 tiles, K = T), squares summed (default)
 *  GRAPE_NORM_GHOST   the ghost identity <(A_i P)(A_i P)^T, Gout_i Gout_i^T>_F from two
 *                     T x T Gram matrices per sample and layer, never forming R_i (Ghost
 *                     Clipping, which the technical summary of "Memory-Efficient
 *                     Differentially Private Training with Gradient Random Projection"
 *                     calls orthogonal to DP-GRAPE; the DP-SGD-RC summary costs it at
 *                     O(B T^2 (p + d)) per linear layer).  It costs 2 T^2 (r + d_out) flops
 *                     per sample and layer against 2 T r d_out, so it pays for short T.
 *                     The Grams are taken in 128 x 128 blocks of 128-token blocks a <= b
 *                     (off-diagonal blocks counted twice), so any T is accepted.
 * Both give the same value up to rounding; the step, grape_sqnorms and clipping use it.
 * The ghost norm forms no R_i, so its steps use the recomputed aggregation whatever
 * grape_set_aggregation says.
 * Errors: GRAPE_EINVAL (unknown method); GRAPE_EUNSUPPORTED (ghost needs the
 * tensor-core path). */
enum grape_norm_method { GRAPE_NORM_DIRECT = 0, GRAPE_NORM_GHOST = 1 };
GRAPE_API int grape_set_norm_method(grape_ctx* ctx, int32_t method);

/* How S_l = sum_i c_i R_{i,l} is formed (the aggregation of the clipped projected
 * per-sample gradients in the closing paragraph of "Metodologia: DP-GRAPE", technical
 * summary of "Memory-Efficient Differentially Private Training with Gradient Random
 * Projection").  Clipping needs every layer's ||R_i|| before any R_i can be weighted,
 * so R_i is either formed twice or kept:
 *  GRAPE_AGG_RECOMPUTE  S = (diag(c) A P)^T Gout over the B*T stacked token rows: a second
 *                       contraction of 2 B T r d_out flops per layer (AP is rescaled by
 *                       c in place first).  No extra memory.
 *  GRAPE_AGG_STORE      the norm kernel also writes every R_i as bf16 (B x r x d_out per
 *                       layer, 2 B r sum(d_out) bytes of device memory held by the
 *                       context); S is then the c-weighted sum of those B matrices, one
 *                       pass of 2 B r d_out bytes per layer.  R_i is rounded to bf16
 *                       before the weighted sum (relative 2^-9 per element).
 *  GRAPE_AGG_AUTO       STORE on the tensor-core path when T >= 256 tokens per sample,
 *                       where the contraction it saves (proportional to T) costs more than
 *                       moving R_i twice (independent of T); RECOMPUTE otherwise.  This is
 *                       what grape_create applies, with the stored R_i in its arena.
 * The ghost norm (GRAPE_NORM_GHOST) never forms R_i, so a context using it recomputes
 * whatever this says.  grape_set_aggregation allocates the R_i storage on first asking
 * for STORE when grape_create did not (GRAPE_ENOMEM if that fails) and keeps it until
 * grape_destroy.  Errors: GRAPE_EINVAL (unknown method), GRAPE_EUNSUPPORTED (STORE on the
 * CUDA-core path).  grape_aggregation_of reports the method the next step will use
 * (RECOMPUTE or STORE). */
enum grape_agg_method { GRAPE_AGG_AUTO = 0, GRAPE_AGG_RECOMPUTE = 1, GRAPE_AGG_STORE = 2 };
GRAPE_API int grape_set_aggregation(grape_ctx* ctx, int32_t method);
GRAPE_API int grape_aggregation_of(const grape_ctx* ctx, int32_t* method);

/* Projection-refresh period K >= 1 (default 1).  P_l of step s is drawn with
 * the step field of its Philox counter set to floor(s / K) instead of s, so one
 * random subspace serves K consecutive steps (the refresh schedule is left
 * open by design choice 1 of "Metodologia: DP-GRAPE" in the technical summary
 * of "Memory-Efficient Differentially Private Training with Gradient Random
 * Projection", which has P rebuilt from a seed).  The noise is still drawn per
 * step, and m and v carry over a refresh unchanged.  A step whose key equals
 * that of the P already in the library's scratch does not regenerate it.
 * Setting the period makes the next step draw P afresh.  The scratch is shared
 * by every call on the handle: a caller that alternates streams orders them.
 * Errors: GRAPE_EINVAL when K < 1 or ctx is NULL. */
GRAPE_API int grape_set_refresh_period(grape_ctx* ctx, int32_t period);

/* Per-sample squared norm estimates only: for every sample i,
 *   sqnorms_dev[i] = sum_l || (A_{i,l} P_l)^T Gout_{i,l} ||_F^2,
 * with P_l the step's projection (entries N(0, 1/r), key as for grape_step).
 * This is the Hutchinson estimate of the full per-sample gradient norm
 * sum_l ||A_{i,l}^T Gout_{i,l}||_F^2 with k = r Gaussian sketch columns
 * ("Metodologia: DP-SGD-RC" and step 3 of its "Flujo Algoritmico", technical
 * summary of DP-SGD-RC, gist.science 2605.24879): unbiased, with variance
 * 2 ||O||_F^2 / r per layer for O = (A^T G)(A^T G)^T.  No clip, aggregation,
 * noise or update runs, and m, v, W and the step's norms are untouched.
 *  A[l], Gout[l]  device inputs, same layouts as grape_step
 *  sqnorms_dev    device pointer to B floats (written)
 * Enqueued on `stream`; returns before the results are ready.
 * Errors: GRAPE_EINVAL for bad pointers or step; GRAPE_ECUDA for a launch error. */
GRAPE_API int grape_sqnorms(grape_ctx* ctx, const void* const* A, const void* const* Gout, int64_t step,
                            float* sqnorms_dev, void* stream);

/* Checkpoint / resume of the projected Adam moments of one layer (r x d_out
 * fp32 each, device pointers), enqueued on `stream`.  P is not state: it is
 * regenerated from (seed, layer, step). */
GRAPE_API int grape_get_state(grape_ctx* ctx, int32_t layer, float* m_dev, float* v_dev, void* stream);
GRAPE_API int grape_set_state(grape_ctx* ctx, int32_t layer, const float* m_dev, const float* v_dev,
                    void* stream);

/* Intermediates of the last step, copied to host memory (synchronises the
 * context's device).  what: */
enum grape_debug_what {
  GRAPE_DBG_NORMS = 0,   /* B floats: n_i */
  GRAPE_DBG_CLIP = 1,    /* B floats: c_i */
  GRAPE_DBG_S = 2,       /* r x d_out floats of `layer` */
  GRAPE_DBG_P = 3,       /* d_in x r floats of `layer`, as used by the last step */
  GRAPE_DBG_DR = 4,      /* r x d_out floats of `layer`: the Adam direction */
  GRAPE_DBG_M = 5,       /* r x d_out floats of `layer` */
  GRAPE_DBG_V = 6        /* r x d_out floats of `layer` */
};
GRAPE_API int grape_debug(grape_ctx* ctx, int32_t what, int32_t layer, void* host_out);

/* Measurement.  While profiling is on, every phase of every step is bracketed
 * by two CUDA events recorded on the step's stream; grape_profile_read
 * synchronises the device and returns, per phase, the summed milliseconds and
 * the number of bracketed calls since profiling was switched on (then starts
 * the sums again).  ms_out and count_out hold GRAPE_N_PHASES entries each
 * (either may be NULL).  grape_launch_count returns how many kernels the
 * context has launched since it was created. */
enum grape_phase {
  GRAPE_PHASE_GEN_P = 0,        /* regenerate P from (seed, layer, step) */
  GRAPE_PHASE_PROJECT = 1,      /* AP = A P over the stacked rows */
  GRAPE_PHASE_NORM = 2,         /* R_i = (A_i P)^T Gout_i and its squared norm */
  GRAPE_PHASE_CLIP = 3,         /* n_i and c_i */
  GRAPE_PHASE_AGGREGATE = 4,    /* S = sum_i c_i R_i */
  GRAPE_PHASE_ADAM = 5,         /* noise + projected Adam */
  GRAPE_PHASE_BACKPROJECT = 6,  /* W -= lr P dR */
  GRAPE_PHASE_COMPACT = 7,      /* live-token scan and gather (grape_step_masked) */
  GRAPE_PHASE_AGGREGATE_ADAM = 8, /* S = sum_i c_i R_i fused with noise + Adam: a step with
                                     the stored aggregation, in place of phases 4 and 5 */
  GRAPE_N_PHASES = 9
};
GRAPE_API int grape_profile(grape_ctx* ctx, int32_t enable);
GRAPE_API int grape_profile_read(grape_ctx* ctx, double* ms_out, int64_t* count_out);
GRAPE_API int grape_launch_count(const grape_ctx* ctx, uint64_t* launches);

/* Bytes of device memory the context holds (moments + workspace). */
GRAPE_API int grape_device_bytes(const grape_ctx* ctx, uint64_t* bytes);
/* The bytes grape_create would allocate for these arguments, computed on the host with no
 * device call: the Adam moments m and v (8 r d_out per layer), every S_l (4 r d_out), dR,
 * the projection scratch P (d_in r) and AP (B T r) per layer, the per-sample norm
 * buffers, the tensor-core workspace (an error word and, for r >= 256, the projection's
 * tile schedules, a few ints per 256-row tile), and the stored R_i (2 B r d_out per
 * layer) when GRAPE_AGG_AUTO chooses them, each block rounded up to 256 bytes.  grape_enable_compaction and the staging of
 * grape_step_host allocate separately.  Errors: as grape_create's argument checks
 * (GRAPE_EINVAL; GRAPE_EUNSUPPORTED for the tensor-core path with fp32 inputs).  It does
 * not check that the device supports the tensor-core path. */
GRAPE_API int grape_context_bytes(const grape_layer* layers, int32_t n_layers, int32_t r, int32_t B, int32_t T,
                                  int32_t in_dtype, int32_t path, uint64_t* bytes);

/* Which kernel family the context runs (enum grape_path, never AUTO). */
GRAPE_API int grape_path_of(const grape_ctx* ctx, int32_t* path);

/* Reason of the last failure on this context ("" if none).  Valid until the
 * next call on ctx. */
GRAPE_API const char* grape_last_error(const grape_ctx* ctx);

/* Reason of the last failure of a call without a context (grape_create,
 * the generator entry points).  Thread-local. */
GRAPE_API const char* grape_global_error(void);

GRAPE_API void grape_destroy(grape_ctx* ctx);

/* The method's generator on its own (Salmon et al. SC'11 Philox4x32-10 and
 * Box-Muller as above), for checking it against other implementations.
 *  grape_philox_words: out_dev[4q + w] = word w of counter (q, layer, step,
 *      stream) for q = 0 .. n_blocks-1 (uint32 device buffer, 4*n_blocks words).
 *  grape_gaussian: out_dev[e] = z(seed, layer, step, stream, e), e < n (fp32). */
GRAPE_API int grape_philox_words(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                       int64_t n_blocks, uint32_t* out_dev, void* stream);
GRAPE_API int grape_gaussian(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id, int64_t n,
                   float* out_dev, void* stream);

/* Per-sample squared projected norms ||(A_i P)^T Gout_i||_F^2 of ONE bf16 layer
 * (the quantity grape_step sums over layers before clipping), computed without
 * allocating anything.  The paper has no counterpart of this call: it exists
 * for callers that must not allocate device memory, e.g. code running under a
 * framework whose caching allocator has reserved the GPU's memory (a side
 * cudaMalloc can fail or fragment its pool) and latency-critical code that
 * cannot afford cudaMalloc/cudaFree, which may synchronise the device.
 *
 *  A, Gout        device pointers, bf16, B x T x d_in and B x T x d_out
 *  r              projection width; P = z(seed, layer, step, stream 0, .)/sqrt(r)
 *  layer, step    the layer and step fields of P's Philox counter.  `step` is the
 *                 projection KEY, not necessarily the training step: a context with
 *                 a refresh period K (grape_set_refresh_period) draws the P of
 *                 training step s with key s / K, so pass s / K to get its norms
 *  sqnorms_out    device pointer, B floats (written; NaN if a device-side wait
 *                 gave up)
 *  stream         cudaStream_t (NULL = default stream); nothing is synchronised
 * Limits: r % 128 == 0 (and % 256 above 256), d_in % 8 == 0, d_out % 256 == 0,
 * and d_in*r*2 + B*T*r*2 + B*ceil(r/128)*ceil(d_out/256)*4 + 256 bytes of
 * scratch within the library's static device array of 8 MiB; larger problems
 * are rejected with GRAPE_EINVAL before anything is launched.
 * All calls share that one array (every GPU that loads the library holds its
 * 8 MiB until the process exits), so calls whose work overlaps on the GPU, on
 * different streams or host threads, race on it; serialise them.  The array
 * keeps the last call's contents; each call clears the one word that must start
 * at zero (its error word) and rewrites the rest.  The first call on a device
 * looks the array's address up on that device (it must be the current device)
 * and keeps it for the life of the process; make that first call before any
 * stream capture.  A cudaDeviceReset invalidates the kept address: do not call
 * this entry point on a device after resetting it.  Several devices may each use
 * it from one process (each has its own array and address).  Errors are reported
 * through grape_global_error(): GRAPE_EINVAL (arguments, size), GRAPE_EUNSUPPORTED
 * (not an sm_100a device, or no tensor-map encoder in the driver), GRAPE_ECUDA. */
GRAPE_API int grape_layer_sqnorms_static(const void* A, const void* Gout, int32_t d_in, int32_t d_out,
                                         int32_t r, int32_t B, int32_t T, uint64_t seed,
                                         uint32_t layer, uint32_t step, float* sqnorms_out,
                                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GRAPE_H_ */
