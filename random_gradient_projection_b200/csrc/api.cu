// C ABI of the DP-GRAPE step: context, validation, workspace and the order of the
// phases (see include/grape.h for the contract of every entry point).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/grape.h"
#include "compact.h"
#include "kernels.h"
#include "tc.h"

namespace {

thread_local std::string g_global_error;

int set_global(int code, const std::string& msg) {
  g_global_error = msg;
  return code;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range over a scope: each public call and each phase of the step shows up by
// name in a timeline or under `ncu --nvtx`.  Without an attached tool the push and pop
// return at once.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Test hook: GRAPE_FAULT_ALLOC=n makes the n-th device allocation of a context fail.
int fault_alloc_index() {
  const char* s = std::getenv("GRAPE_FAULT_ALLOC");
  return s ? std::atoi(s) : 0;
}

}  // namespace

struct grape_ctx {
  grape::StepShape sh{};
  int path = GRAPE_PATH_SIMT;  // resolved (never AUTO)
  int device = 0;
  std::vector<grape_layer> layers;
  std::vector<grape::LayerWs> ws;
  void* arena = nullptr;
  size_t arena_bytes = 0;
  float* partials = nullptr;
  float* norms = nullptr;
  float* clip = nullptr;
  grape::TcWorkspace tc{};
  // staging for grape_step_host (allocated on first use)
  std::vector<void*> stage_A, stage_G;
  int64_t last_step = -1;
  int64_t S_count = 0;   // elements of all S_l together (they are contiguous)
  // projection refresh: P of step s is drawn with key s / refresh; p_key is the key of
  // the P now in the scratch (-1: none), so a step with the same key skips generating it
  uint32_t refresh = 1;
  int64_t p_key = -1;
  int norm_method = GRAPE_NORM_DIRECT;
  // aggregation (grape_set_aggregation): recompute (diag(c) AP)^T Gout, or sum the R_i the
  // norm kernel stored; agg is never AUTO.  The stored R_i live in the arena when AUTO
  // chose them at create, else in rst_buf, allocated when a caller asks for them.
  int agg = GRAPE_AGG_RECOMPUTE;
  void* rst_buf = nullptr;
  bool stores_R() const { return agg == GRAPE_AGG_STORE && norm_method == GRAPE_NORM_DIRECT; }
  // A one-process step with the stored aggregation sums the R_i inside the noise + Adam
  // kernel (tc_aggregate_adam); grape_accumulate / grape_apply keep them apart, since S
  // is all-reduced in between.  GRAPE_FUSE_ADAM=0 in the environment at grape_create
  // keeps them apart in every step too (a measurement knob: both give the same bits).
  bool fuse_adam = true;
  bool fuses_adam() const { return fuse_adam && path == GRAPE_PATH_TC && stores_R(); }
  // CUDA-graph replay of grape_step (grape_set_graph): one graph per set of A, Gout, W
  // pointers; the first step with a set captures it, later ones replay it
  struct StepGraph {
    std::vector<const void*> A, G;
    std::vector<float*> W;
    bool captured = false;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    cudaGraphNode_t gen_p = nullptr, adam = nullptr;
    bool adam_fused = false;   // the Adam node is tc_aggregate_adam's
    uint64_t launches = 0, used = 0;
  };
  bool graph_on = false;
  std::vector<StepGraph> graphs;
  uint64_t graph_tick = 0;
  cudaStream_t capture_stream = nullptr;

  void drop_graph(StepGraph& g) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    if (g.graph) cudaGraphDestroy(g.graph);
    g.exec = nullptr;
    g.graph = nullptr;
  }
  // live-token compaction (grape_enable_compaction): inputs of T_full tokens per sample,
  // compacted to the context's T rows; one allocation holds every buffer below
  int T_full = 0;
  void* compact_buf = nullptr;
  std::vector<void*> comp_A, comp_G;
  int32_t* comp_idx = nullptr;
  int32_t* comp_counts = nullptr;
  int* comp_overflow = nullptr;
  double beta1 = 0.9, beta2 = 0.999;   // as given (bias corrections are formed in double)
  std::string err;
  // measurement
  bool prof_on = false;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  struct Mark { int phase; cudaEvent_t a, b; };
  std::vector<Mark> marks;
  uint64_t launches = 0;

  cudaEvent_t next_event() {
    if (ev_used == ev_pool.size()) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      ev_pool.push_back(e);
    }
    return ev_pool[ev_used++];
  }

  int fail(int code, const std::string& msg) {
    err = msg;
    return code;
  }
  int cuda_fail(cudaError_t e, const char* where) {
    err = std::string(where) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return GRAPE_ECUDA;
  }
};

namespace {

struct Arena {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~static_cast<size_t>(255);
    return o;
  }
};

size_t in_elsize(int dtype) { return dtype == GRAPE_BF16 ? 2 : 4; }

// GRAPE_AGG_AUTO's choice.  Recomputing the aggregation costs a second contraction of
// 2 B T r d_out flops per layer (plus a re-read of Gout); storing R_i costs
// 2 B r d_out bytes written by the norm kernel and read once more.  At the measured
// tensor and HBM rates the two break even near T ~ kAggStoreMinT tokens per sample.
constexpr int kAggStoreMinT = 256;
bool auto_stores_R(int path, int T) { return path == GRAPE_PATH_TC && T >= kAggStoreMinT; }

// Bytes of every layer's stored R_i: B x r x d_out bf16 each.
size_t rstore_bytes(const grape_layer* layers, int n_layers, int r, int B) {
  size_t n = 0;
  for (int l = 0; l < n_layers; ++l) n += static_cast<size_t>(B) * r * layers[l].d_out * 2;
  return n;
}

int validate_io(grape_ctx* ctx, const void* const* A, const void* const* G, float* const* W,
                bool need_ag, bool need_w) {
  if (need_ag && (!A || !G)) return ctx->fail(GRAPE_EINVAL, "A and Gout arrays must not be null");
  if (need_w && !W) return ctx->fail(GRAPE_EINVAL, "W array must not be null");
  for (int l = 0; l < ctx->sh.L; ++l) {
    if (need_ag) {
      if (!A[l] || !G[l])
        return ctx->fail(GRAPE_EINVAL, "A[" + std::to_string(l) + "] or Gout[" + std::to_string(l) +
                                           "] is null");
      if (!aligned16(A[l]) || !aligned16(G[l]))
        return ctx->fail(GRAPE_EINVAL, "A/Gout of layer " + std::to_string(l) +
                                           " not 16-byte aligned");
    }
    if (need_w) {
      if (!W[l]) return ctx->fail(GRAPE_EINVAL, "W[" + std::to_string(l) + "] is null");
      if (!aligned16(W[l]))
        return ctx->fail(GRAPE_EINVAL, "W of layer " + std::to_string(l) + " not 16-byte aligned");
    }
  }
  return GRAPE_OK;
}

// The context's buffers live on the device it was created on: a call made while another
// device is current would launch there with this device's pointers.
int check_device(grape_ctx* ctx) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return ctx->fail(GRAPE_ECUDA, "cudaGetDevice failed");
  }
  if (cur != ctx->device)
    return ctx->fail(GRAPE_EINVAL, "the context was created on device " + std::to_string(ctx->device) +
                                       " but device " + std::to_string(cur) + " is current");
  return GRAPE_OK;
}

int check_step_index(grape_ctx* ctx, int64_t step) {
  if (int rc = check_device(ctx)) return rc;
  if (step < 0 || step > 0xFFFFFFFFll)
    return ctx->fail(GRAPE_EINVAL, "step must be in [0, 2^32)");
  return GRAPE_OK;
}

// Run one phase: launch it, count its kernels and, when profiling, bracket it
// with two events on the step's stream.
template <class F>
int phase(grape_ctx* ctx, int id, const char* what, cudaStream_t st, F&& launch) {
  const NvtxRange range(what);
  cudaEvent_t a = nullptr;
  if (ctx->prof_on) {
    a = ctx->next_event();
    if (!a) return ctx->fail(GRAPE_ECUDA, "cudaEventCreate failed");
    cudaEventRecord(a, st);
  }
  int n = 0;
  const cudaError_t e = launch(&n);
  if (e != cudaSuccess) return ctx->cuda_fail(e, what);
  ctx->launches += static_cast<uint64_t>(n);
  if (ctx->prof_on) {
    cudaEvent_t b = ctx->next_event();
    if (!b) return ctx->fail(GRAPE_ECUDA, "cudaEventCreate failed");
    cudaEventRecord(b, st);
    ctx->marks.push_back({id, a, b});
  }
  return GRAPE_OK;
}

// Generate P when its key changed, then AP = A P and the per-sample norm partials.
// store_R: the step's norm kernel also writes every R_i for the stored aggregation.
int run_project_norm(grape_ctx* ctx, const grape::LayerIo* io, int64_t step, cudaStream_t st,
                     bool store_R) {
  const grape::StepShape& sh = ctx->sh;
  const grape::LayerWs* ws = ctx->ws.data();
  const uint32_t key = static_cast<uint32_t>(step) / ctx->refresh;
  const bool gen = static_cast<int64_t>(key) != ctx->p_key;
  int rc;
  if (gen) {
    ctx->p_key = -1;   // the scratch is being rewritten
    rc = phase(ctx, GRAPE_PHASE_GEN_P, "generate P", st, [&](int* n) {
      if (ctx->path == GRAPE_PATH_TC) return grape::tc_generate_P(sh, ws, ctx->tc, key, st, n);
      *n = 1;
      return grape::simt_generate_P(sh, ws, key, st);
    });
    if (rc) return rc;
    ctx->p_key = key;
  }
  if (ctx->path == GRAPE_PATH_TC) {
    const grape::TcWorkspace& tc = ctx->tc;
    rc = phase(ctx, GRAPE_PHASE_PROJECT, "project", st,
               [&](int* n) { return grape::tc_project(sh, ws, io, tc, st, n, !gen); });
    if (rc) return rc;
    return phase(ctx, GRAPE_PHASE_NORM, "per-sample norms", st, [&](int* n) {
      if (ctx->norm_method == GRAPE_NORM_GHOST)
        return grape::tc_project_norm_ghost(sh, ws, io, tc, ctx->partials, st, n);
      return grape::tc_project_norm(sh, ws, io, tc, ctx->partials, store_R, st, n);
    });
  }
  rc = phase(ctx, GRAPE_PHASE_PROJECT, "project", st, [&](int* n) {
    *n = 1;
    return grape::simt_project_ap(sh, ws, io, st);
  });
  if (rc) return rc;
  return phase(ctx, GRAPE_PHASE_NORM, "per-sample norms", st, [&](int* n) {
    *n = 1;
    return grape::simt_project_norm(sh, ws, io, ctx->partials, st);
  });
}

// defer_stored: with the stored aggregation, leave the sum of the R_i to the fused noise +
// Adam kernel of run_apply (a one-process step).
int run_accumulate(grape_ctx* ctx, const void* const* A, const void* const* G, int64_t step,
                   cudaStream_t st, bool defer_stored = false) {
  std::vector<grape::LayerIo> io(ctx->sh.L);
  for (int l = 0; l < ctx->sh.L; ++l) io[l] = grape::LayerIo{A[l], G[l], nullptr};
  const grape::StepShape& sh = ctx->sh;
  const grape::LayerWs* ws = ctx->ws.data();
  const bool stored = ctx->path == GRAPE_PATH_TC && ctx->stores_R();
  int rc = run_project_norm(ctx, io.data(), step, st, stored);
  if (rc) return rc;
  rc = phase(ctx, GRAPE_PHASE_CLIP, "clip", st, [&](int* n) {
    if (ctx->path == GRAPE_PATH_TC)
      return grape::tc_clip_scale(sh, ws, ctx->tc, ctx->partials, ctx->norms, ctx->clip, !stored, st, n);
    *n = 1;
    return grape::finalize_clip(sh, ctx->partials, ctx->norms, ctx->clip, st);
  });
  if (rc) return rc;
  if (stored && defer_stored) {
    ctx->last_step = step;
    return GRAPE_OK;
  }
  if (ctx->path == GRAPE_PATH_TC) {
    rc = phase(ctx, GRAPE_PHASE_AGGREGATE, "aggregate", st, [&](int* n) {
      if (stored) return grape::tc_aggregate_stored(sh, ws, ctx->clip, st, n);
      return grape::tc_aggregate(sh, ws, io.data(), ctx->tc, ctx->clip, st, n);
    });
  } else {
    rc = phase(ctx, GRAPE_PHASE_AGGREGATE, "aggregate", st, [&](int* n) {
      *n = 1;
      return grape::simt_aggregate(sh, ws, io.data(), ctx->clip, st);
    });
  }
  if (rc) return rc;
  ctx->last_step = step;
  return GRAPE_OK;
}

grape::UpdateScalars update_scalars(const grape_ctx* ctx, int64_t step, int64_t batch_total) {
  const int64_t bt = batch_total > 0 ? batch_total : ctx->sh.B;
  const double t = static_cast<double>(step) + 1.0;
  grape::UpdateScalars u{};
  u.step = static_cast<uint32_t>(step);
  u.inv_batch = static_cast<float>(1.0 / static_cast<double>(bt));
  u.inv_bc1 = static_cast<float>(1.0 / (1.0 - std::pow(ctx->beta1, t)));
  u.inv_bc2 = static_cast<float>(1.0 / (1.0 - std::pow(ctx->beta2, t)));
  return u;
}

// fused: the aggregation was deferred (run_accumulate's defer_stored), and this step's
// noise + Adam kernel sums the stored R_i first.
int run_apply(grape_ctx* ctx, float* const* W, int64_t step, int64_t batch_total, cudaStream_t st,
              bool fused = false) {
  const grape::UpdateScalars u = update_scalars(ctx, step, batch_total);
  std::vector<grape::LayerIo> io(ctx->sh.L);
  for (int l = 0; l < ctx->sh.L; ++l) io[l] = grape::LayerIo{nullptr, nullptr, W[l]};
  const bool tc = ctx->path == GRAPE_PATH_TC;
  const grape::StepShape& sh = ctx->sh;
  const grape::LayerWs* ws = ctx->ws.data();
  int rc = fused ? phase(ctx, GRAPE_PHASE_AGGREGATE_ADAM, "aggregate + noise + adam", st,
                         [&](int* n) { return grape::tc_aggregate_adam(sh, ws, u, ctx->clip, st, n); })
                 : phase(ctx, GRAPE_PHASE_ADAM, "noise + adam", st, [&](int* n) {
                     *n = 1;
                     return grape::noise_adam(sh, ws, u, tc, tc, st);
                   });
  if (rc) return rc;
  return phase(ctx, GRAPE_PHASE_BACKPROJECT, "back-project", st, [&](int* n) {
    if (tc) return grape::tc_backproject(sh, ws, io.data(), ctx->tc, sh.lr, st, n);
    *n = 1;
    return grape::simt_backproject(sh, ws, io.data(), sh.lr, st);
  });
}

// One whole step in one process: accumulate, then apply, the stored aggregation fused
// into noise + Adam where the context does that.
int run_step(grape_ctx* ctx, const void* const* A, const void* const* G, float* const* W, int64_t step,
             cudaStream_t st) {
  const bool fuse = ctx->fuses_adam();
  int rc = run_accumulate(ctx, A, G, step, st, fuse);
  if (rc) return rc;
  return run_apply(ctx, W, step, 0, st, fuse);
}

// grape_step through a CUDA graph (see StepGraph).  Capture records the same launches as
// run_accumulate + run_apply, including their programmatic (PDL) dependencies, on a
// library stream; every replay rewrites the two step-dependent kernels' arguments (P's
// Philox key; the step and bias corrections of noise + Adam) and launches the graph on
// the caller's stream.  P is generated on every replay, so one graph serves any step.
int step_graph(grape_ctx* ctx, const void* const* A, const void* const* G, float* const* W, int64_t step,
               cudaStream_t st) {
  const int L = ctx->sh.L;
  grape_ctx::StepGraph* hit = nullptr;
  for (auto& g : ctx->graphs) {
    bool same = true;
    for (int l = 0; l < L && same; ++l) same = g.A[l] == A[l] && g.G[l] == G[l] && g.W[l] == W[l];
    if (same) {
      hit = &g;
      break;
    }
  }
  if (!hit) {   // first sight of this pointer set: captured below, then replayed
    if (ctx->graphs.size() >= 8) {
      size_t lru = 0;
      for (size_t k = 1; k < ctx->graphs.size(); ++k)
        if (ctx->graphs[k].used < ctx->graphs[lru].used) lru = k;
      ctx->drop_graph(ctx->graphs[lru]);
      ctx->graphs.erase(ctx->graphs.begin() + static_cast<long>(lru));
    }
    grape_ctx::StepGraph g;
    g.A.assign(A, A + L);
    g.G.assign(G, G + L);
    g.W.assign(W, W + L);
    ctx->graphs.push_back(g);
    hit = &ctx->graphs.back();
  }
  hit->used = ++ctx->graph_tick;
  if (!hit->captured) {
    if (!ctx->capture_stream) {
      cudaError_t e = cudaStreamCreateWithFlags(&ctx->capture_stream, cudaStreamNonBlocking);
      if (e != cudaSuccess) return ctx->cuda_fail(e, "cudaStreamCreate");
    }
    const int64_t saved_key = ctx->p_key;
    const uint64_t l0 = ctx->launches;
    ctx->p_key = -1;   // the graph always contains the generation of P
    cudaError_t e = cudaStreamBeginCapture(ctx->capture_stream, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return ctx->cuda_fail(e, "cudaStreamBeginCapture");
    int rc = run_step(ctx, A, G, W, step, ctx->capture_stream);
    cudaGraph_t graph = nullptr;
    e = cudaStreamEndCapture(ctx->capture_stream, &graph);
    hit->launches = ctx->launches - l0;
    ctx->launches = l0;           // nothing ran yet
    ctx->p_key = saved_key;       // nor was P generated
    if (rc || e != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      cudaGetLastError();
      return rc ? rc : ctx->cuda_fail(e, "cudaStreamEndCapture");
    }
    e = cudaGraphInstantiate(&hit->exec, graph, 0);
    if (e != cudaSuccess) {
      cudaGraphDestroy(graph);
      return ctx->cuda_fail(e, "cudaGraphInstantiate");
    }
    hit->graph = graph;
    size_t n = 0;
    cudaGraphGetNodes(graph, nullptr, &n);
    std::vector<cudaGraphNode_t> nodes(n);
    cudaGraphGetNodes(graph, nodes.data(), &n);
    const void* gen_fn = ctx->path == GRAPE_PATH_TC ? grape::tc_gen_P_func() : grape::simt_generate_P_func();
    for (cudaGraphNode_t nd : nodes) {
      cudaGraphNodeType ty;
      if (cudaGraphNodeGetType(nd, &ty) != cudaSuccess || ty != cudaGraphNodeTypeKernel) continue;
      cudaKernelNodeParams kp{};
      if (cudaGraphKernelNodeGetParams(nd, &kp) != cudaSuccess) continue;
      if (kp.func == gen_fn) hit->gen_p = nd;
      if (kp.func == grape::noise_adam_func() || kp.func == grape::tc_aggregate_adam_func()) {
        hit->adam = nd;
        hit->adam_fused = kp.func == grape::tc_aggregate_adam_func();
      }
    }
    if (!hit->gen_p || !hit->adam) {
      ctx->drop_graph(*hit);
      return ctx->fail(GRAPE_ECUDA, "captured step graph lacks its P-generation or Adam node");
    }
    hit->captured = true;
  }
  const uint32_t key = static_cast<uint32_t>(step) / ctx->refresh;
  const grape::StepShape& sh = ctx->sh;
  cudaError_t e = ctx->path == GRAPE_PATH_TC
                      ? grape::tc_generate_P_set_node(hit->exec, hit->gen_p, sh, ctx->ws.data(), key)
                      : grape::simt_generate_P_set_node(hit->exec, hit->gen_p, sh, ctx->ws.data(), key);
  if (e == cudaSuccess)
    e = hit->adam_fused ? grape::tc_aggregate_adam_set_node(hit->exec, hit->adam, sh, ctx->ws.data(),
                                                            update_scalars(ctx, step, 0), ctx->clip)
                        : grape::noise_adam_set_node(hit->exec, hit->adam, sh, ctx->ws.data(),
                                                     update_scalars(ctx, step, 0), ctx->path == GRAPE_PATH_TC);
  if (e == cudaSuccess) e = cudaGraphLaunch(hit->exec, st);
  if (e != cudaSuccess) return ctx->cuda_fail(e, "graph replay");
  ctx->launches += hit->launches;
  ctx->p_key = key;
  ctx->last_step = step;
  return GRAPE_OK;
}

// After a device synchronisation: a sample that kept more live tokens than the compact
// capacity, or a tensor-core wait that gave up, leaves a nonzero word.
int check_device_error(grape_ctx* ctx) {
  if (ctx->comp_overflow) {
    int v = 0;
    cudaError_t e = cudaMemcpy(&v, ctx->comp_overflow, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return ctx->cuda_fail(e, "read compaction flag");
    if (v != 0) {
      cudaMemset(ctx->comp_overflow, 0, sizeof(int));
      return ctx->fail(GRAPE_EINVAL, "a sample kept more live tokens than the compaction capacity T = " +
                                         std::to_string(ctx->sh.T) + " (only the first T were used)");
    }
  }
  if (ctx->path != GRAPE_PATH_TC) return GRAPE_OK;
  int* word = grape::tc_error_word(ctx->tc);
  if (!word) return GRAPE_OK;
  int v = 0;
  cudaError_t e = cudaMemcpy(&v, word, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return ctx->cuda_fail(e, "read error word");
  if (v != 0) {
    cudaMemset(word, 0, sizeof(int));
#ifdef GRAPE_CHECKED
    if (v & grape::kTcErrBounds)
      return ctx->fail(GRAPE_ECUDA, "checked build: a TMA box started outside its tensor or off the "
                                    "16-byte rule, and its copy was skipped (code " + std::to_string(v) + ")");
#endif
    return ctx->fail(GRAPE_ETIMEOUT, "a tensor-core kernel gave up waiting (code " +
                                         std::to_string(v) + ")");
  }
  return GRAPE_OK;
}

}  // namespace

extern "C" {

int grape_create(const grape_layer* layers, int32_t n_layers, int32_t r, double C, double sigma,
                 uint64_t seed, const grape_adam* adam, int32_t B, int32_t T, int32_t in_dtype,
                 int32_t path, grape_ctx** out) {
  if (!out) return set_global(GRAPE_EINVAL, "out must not be null");
  *out = nullptr;
  if (!layers) return set_global(GRAPE_EINVAL, "layers must not be null");
  if (!adam) return set_global(GRAPE_EINVAL, "adam must not be null");
  if (n_layers < 1 || n_layers > GRAPE_MAX_LAYERS)
    return set_global(GRAPE_EINVAL, "n_layers must be in [1, " + std::to_string(GRAPE_MAX_LAYERS) + "]");
  if (B < 1 || T < 1) return set_global(GRAPE_EINVAL, "B and T must be >= 1");
  if (r < 1) return set_global(GRAPE_EINVAL, "r must be >= 1");
  if (!(C > 0.0) || !std::isfinite(C)) return set_global(GRAPE_EINVAL, "C must be finite and > 0");
  if (!(sigma >= 0.0) || !std::isfinite(sigma)) return set_global(GRAPE_EINVAL, "sigma must be finite and >= 0");
  if (!(adam->lr >= 0.0) || !(adam->beta1 >= 0.0 && adam->beta1 < 1.0) ||
      !(adam->beta2 >= 0.0 && adam->beta2 < 1.0) || !(adam->eps > 0.0))
    return set_global(GRAPE_EINVAL, "adam: need lr >= 0, beta1 and beta2 in [0, 1), eps > 0");
  if (in_dtype != GRAPE_F32 && in_dtype != GRAPE_BF16)
    return set_global(GRAPE_EINVAL, "in_dtype must be GRAPE_F32 or GRAPE_BF16");
  if (path < GRAPE_PATH_AUTO || path > GRAPE_PATH_TC)
    return set_global(GRAPE_EINVAL, "path must be a grape_path value");
  for (int l = 0; l < n_layers; ++l) {
    if (layers[l].d_in < 1 || layers[l].d_out < 1)
      return set_global(GRAPE_EINVAL, "layer " + std::to_string(l) + ": d_in and d_out must be >= 1");
    if (r > layers[l].d_in)
      return set_global(GRAPE_EINVAL, "layer " + std::to_string(l) + ": r must be <= d_in");
  }
  if (static_cast<int64_t>(B) * T > (int64_t{1} << 31) / 4)
    return set_global(GRAPE_EINVAL, "B*T too large");

  int resolved = path;
  if (resolved == GRAPE_PATH_AUTO) resolved = (in_dtype == GRAPE_BF16) ? GRAPE_PATH_TC : GRAPE_PATH_SIMT;
  if (resolved == GRAPE_PATH_TC && in_dtype != GRAPE_BF16)
    return set_global(GRAPE_EUNSUPPORTED, "the tensor-core path takes bf16 inputs");

  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return set_global(GRAPE_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(ce));
  if (resolved == GRAPE_PATH_TC) {
    std::string why;
    if (!grape::tc_supported(dev, layers, n_layers, r, B, T, &why)) {
      if (path == GRAPE_PATH_TC) return set_global(GRAPE_EUNSUPPORTED, why);
      return set_global(GRAPE_EUNSUPPORTED, "bf16 inputs need the tensor-core path: " + why);
    }
  }

  grape_ctx* ctx = new grape_ctx();
  ctx->device = dev;
  ctx->path = resolved;
  ctx->layers.assign(layers, layers + n_layers);
  grape::StepShape& sh = ctx->sh;
  sh.L = n_layers;
  sh.r = r;
  sh.B = B;
  sh.T = T;
  sh.dtype = in_dtype;
  sh.seed = seed;
  sh.C = static_cast<float>(C);
  sh.sigma_C = static_cast<float>(sigma * C);
  sh.lr = static_cast<float>(adam->lr);
  sh.beta1 = static_cast<float>(adam->beta1);
  sh.beta2 = static_cast<float>(adam->beta2);
  sh.one_minus_beta1 = static_cast<float>(1.0 - adam->beta1);
  sh.one_minus_beta2 = static_cast<float>(1.0 - adam->beta2);
  sh.eps = static_cast<float>(adam->eps);
  ctx->beta1 = adam->beta1;
  ctx->beta2 = adam->beta2;

  const bool tc = resolved == GRAPE_PATH_TC;
  const size_t ap_el = tc ? 2 : 4;
  Arena ar;
  struct Offs { size_t P32, P16, AP, S, m, v, dR; };
  std::vector<Offs> offs(n_layers);
  int part = 0;
  ctx->ws.resize(n_layers);
  // every S_l back to back in one block (layer order, no padding), so a data-parallel
  // caller can sum them over ranks with a single all-reduce (grape_S_all)
  size_t s_total = 0;
  for (int l = 0; l < n_layers; ++l) s_total += static_cast<size_t>(r) * layers[l].d_out;
  const size_t off_s_all = ar.take(s_total * 4);
  ctx->S_count = static_cast<int64_t>(s_total);
  size_t s_at = off_s_all;
  for (int l = 0; l < n_layers; ++l) {
    const size_t di = layers[l].d_in, dout = layers[l].d_out;
    Offs& o = offs[l];
    o.P32 = tc ? SIZE_MAX : ar.take(di * r * 4);
    o.P16 = tc ? ar.take(di * r * 2) : SIZE_MAX;
    o.AP = ar.take(static_cast<size_t>(B) * T * r * ap_el);
    o.S = s_at;
    s_at += r * dout * 4;
    o.m = ar.take(r * dout * 4);
    o.v = ar.take(r * dout * 4);
    o.dR = ar.take(r * dout * (tc ? 2 : 4));
    grape::LayerWs& w = ctx->ws[l];
    w.d_in = layers[l].d_in;
    w.d_out = layers[l].d_out;
    w.part_base = part;
    w.part_count = tc ? grape::tc_partials_per_sample(r, layers[l].d_out)
                      : grape::simt_partials_per_sample(r, layers[l].d_out);
    part += w.part_count;
  }
  sh.part_stride = part;
  const size_t off_part = ar.take(static_cast<size_t>(B) * part * 4);
  const size_t off_norms = ar.take(static_cast<size_t>(B) * 4);
  const size_t off_clip = ar.take(static_cast<size_t>(B) * 4);
  size_t off_tc = 0;
  size_t tc_bytes = tc ? grape::tc_workspace_bytes(sh, ctx->ws.data()) : 0;
  if (tc) off_tc = ar.take(tc_bytes);
  // GRAPE_AGG_AUTO: every layer's stored R_i, when the aggregation sums them
  const bool store = auto_stores_R(resolved, T);
  ctx->agg = store ? GRAPE_AGG_STORE : GRAPE_AGG_RECOMPUTE;
  if (const char* v = std::getenv("GRAPE_FUSE_ADAM")) ctx->fuse_adam = std::strcmp(v, "0") != 0;
  std::vector<size_t> off_rst(n_layers, SIZE_MAX);
  if (store)
    for (int l = 0; l < n_layers; ++l) off_rst[l] = ar.take(static_cast<size_t>(B) * r * layers[l].d_out * 2);
  ctx->arena_bytes = ar.off;

  const int fault = fault_alloc_index();
  if (fault == 1) {
    delete ctx;
    return set_global(GRAPE_ENOMEM, "device allocation failed (GRAPE_FAULT_ALLOC)");
  }
  ce = cudaMalloc(&ctx->arena, ctx->arena_bytes);
  if (ce != cudaSuccess) {
    delete ctx;
    cudaGetLastError();
    return set_global(GRAPE_ENOMEM, "cudaMalloc of " + std::to_string(ar.off) + " bytes: " + cudaGetErrorString(ce));
  }
  char* base = static_cast<char*>(ctx->arena);
  auto at = [&](size_t o) -> char* { return o == SIZE_MAX ? nullptr : base + o; };
  for (int l = 0; l < n_layers; ++l) {
    grape::LayerWs& w = ctx->ws[l];
    const Offs& o = offs[l];
    w.P32 = reinterpret_cast<float*>(at(o.P32));
    w.P16 = reinterpret_cast<__nv_bfloat16*>(at(o.P16));
    w.AP = at(o.AP);
    w.S = reinterpret_cast<float*>(at(o.S));
    w.m = reinterpret_cast<float*>(at(o.m));
    w.v = reinterpret_cast<float*>(at(o.v));
    w.dR = at(o.dR);
    w.Rst = reinterpret_cast<__nv_bfloat16*>(at(off_rst[l]));
  }
  ctx->partials = reinterpret_cast<float*>(at(off_part));
  ctx->norms = reinterpret_cast<float*>(at(off_norms));
  ctx->clip = reinterpret_cast<float*>(at(off_clip));
  // Everything starts at zero: moments, S, norms, partial slots.
  ce = cudaMemset(ctx->arena, 0, ctx->arena_bytes);
  if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
  if (ce != cudaSuccess) {
    cudaFree(ctx->arena);
    delete ctx;
    return set_global(GRAPE_ECUDA, std::string("cudaMemset: ") + cudaGetErrorString(ce));
  }
  if (tc) {
    ce = grape::tc_init(sh, ctx->ws.data(), at(off_tc), tc_bytes, &ctx->tc);
    if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
    if (ce != cudaSuccess) {
      grape::tc_release(&ctx->tc);
      cudaFree(ctx->arena);
      delete ctx;
      return set_global(GRAPE_ECUDA, std::string("tensor-core set-up: ") + cudaGetErrorString(ce));
    }
  }
  *out = ctx;
  return GRAPE_OK;
}

int grape_step(grape_ctx* ctx, const void* const* A, const void* const* Gout, float* const* W,
               int64_t step, void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  int rc = check_step_index(ctx, step);
  if (rc) return rc;
  rc = validate_io(ctx, A, Gout, W, true, true);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ctx->graph_on && !ctx->prof_on) {
    const NvtxRange range("grape_step (graph replay)");
    return step_graph(ctx, A, Gout, W, step, st);
  }
  const NvtxRange range("grape_step");
  return run_step(ctx, A, Gout, W, step, st);
}

int grape_step_host(grape_ctx* ctx, const void* const* A_host, const void* const* Gout_host,
                    float* const* W, int64_t step, float* norms_host, void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  int rc = check_step_index(ctx, step);
  if (rc) return rc;
  if (!A_host || !Gout_host) return ctx->fail(GRAPE_EINVAL, "A_host and Gout_host must not be null");
  for (int l = 0; l < ctx->sh.L; ++l)
    if (!A_host[l] || !Gout_host[l]) return ctx->fail(GRAPE_EINVAL, "null host input pointer");
  rc = validate_io(ctx, nullptr, nullptr, W, false, true);
  if (rc) return rc;
  const NvtxRange range("grape_step_host");
  const size_t el = in_elsize(ctx->sh.dtype);
  const size_t rows = static_cast<size_t>(ctx->sh.B) * ctx->sh.T;
  if (ctx->stage_A.empty()) {
    std::vector<void*> sa(ctx->sh.L, nullptr), sg(ctx->sh.L, nullptr);
    for (int l = 0; l < ctx->sh.L; ++l) {
      if (cudaMalloc(&sa[l], rows * ctx->layers[l].d_in * el) != cudaSuccess ||
          cudaMalloc(&sg[l], rows * ctx->layers[l].d_out * el) != cudaSuccess) {
        cudaGetLastError();
        for (void* p : sa) cudaFree(p);   // cudaFree(nullptr) is a no-op
        for (void* p : sg) cudaFree(p);
        return ctx->fail(GRAPE_ENOMEM, "staging allocation for grape_step_host failed");
      }
    }
    ctx->stage_A = sa;   // kept only when every layer's staging exists
    ctx->stage_G = sg;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int l = 0; l < ctx->sh.L; ++l) {
    cudaError_t e = cudaMemcpyAsync(ctx->stage_A[l], A_host[l], rows * ctx->layers[l].d_in * el,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(ctx->stage_G[l], Gout_host[l], rows * ctx->layers[l].d_out * el,
                          cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return ctx->cuda_fail(e, "host-to-device copy");
  }
  rc = run_step(ctx, ctx->stage_A.data(), ctx->stage_G.data(), W, step, st);
  if (rc) return rc;
  if (norms_host) {
    cudaError_t e = cudaMemcpyAsync(norms_host, ctx->norms, ctx->sh.B * sizeof(float),
                                    cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return ctx->cuda_fail(e, "device-to-host copy");
  }
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return ctx->cuda_fail(e, "stream synchronize");
  return check_device_error(ctx);
}

int grape_accumulate(grape_ctx* ctx, const void* const* A, const void* const* Gout, int64_t step,
                     void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  int rc = check_step_index(ctx, step);
  if (rc) return rc;
  rc = validate_io(ctx, A, Gout, nullptr, true, false);
  if (rc) return rc;
  const NvtxRange range("grape_accumulate");
  return run_accumulate(ctx, A, Gout, step, static_cast<cudaStream_t>(stream));
}

int grape_S_ptr(grape_ctx* ctx, int32_t layer, float** S_dev) {
  if (!ctx || !S_dev) return set_global(GRAPE_EINVAL, "ctx and S_dev must not be null");
  if (layer < 0 || layer >= ctx->sh.L) return ctx->fail(GRAPE_EINVAL, "layer out of range");
  *S_dev = ctx->ws[layer].S;
  return GRAPE_OK;
}

int grape_S_all(grape_ctx* ctx, float** S_dev, int64_t* count) {
  if (!ctx || !S_dev || !count) return set_global(GRAPE_EINVAL, "ctx, S_dev and count must not be null");
  *S_dev = ctx->ws[0].S;
  *count = ctx->S_count;
  return GRAPE_OK;
}

int grape_apply(grape_ctx* ctx, float* const* W, int64_t step, int64_t batch_total, void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  int rc = check_step_index(ctx, step);
  if (rc) return rc;
  if (batch_total < 0) return ctx->fail(GRAPE_EINVAL, "batch_total must be >= 0");
  rc = validate_io(ctx, nullptr, nullptr, W, false, true);
  if (rc) return rc;
  // S lies in the span of the P its aggregation used, so the back-projection must use
  // that P: the last accumulation drew it with this step's key, and no later call
  // (grape_sqnorms, a refresh-period change) has replaced it in the scratch since.
  const int64_t key = static_cast<uint32_t>(step) / ctx->refresh;
  if (ctx->last_step < 0 || static_cast<uint32_t>(ctx->last_step) / ctx->refresh != key || ctx->p_key != key)
    return ctx->fail(GRAPE_EINVAL, "grape_apply(step " + std::to_string(step) +
                                       ") needs a grape_accumulate of a step with the same projection"
                                       " (key step / refresh period) as the last call that drew P");
  const NvtxRange range("grape_apply");
  return run_apply(ctx, W, step, batch_total, static_cast<cudaStream_t>(stream));
}

int grape_enable_compaction(grape_ctx* ctx, int32_t T_full) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  if (T_full < ctx->sh.T) return ctx->fail(GRAPE_EINVAL, "T_full must be >= the context's T (the capacity)");
  if (ctx->sh.B > 65535) return ctx->fail(GRAPE_EINVAL, "compaction supports B <= 65535");
  if (ctx->compact_buf) return ctx->fail(GRAPE_EINVAL, "compaction is already enabled");
  const size_t el = in_elsize(ctx->sh.dtype);
  const size_t rows = static_cast<size_t>(ctx->sh.B) * ctx->sh.T;
  Arena ar;
  std::vector<size_t> oa, og;
  for (const grape_layer& ly : ctx->layers) {
    oa.push_back(ar.take(rows * ly.d_in * el));
    og.push_back(ar.take(rows * ly.d_out * el));
  }
  const size_t o_idx = ar.take(rows * sizeof(int32_t));
  const size_t o_cnt = ar.take(static_cast<size_t>(ctx->sh.B) * sizeof(int32_t));
  const size_t o_flag = ar.take(sizeof(int));
  void* buf = nullptr;
  cudaError_t e = cudaMalloc(&buf, ar.off);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return ctx->fail(GRAPE_ENOMEM, "cudaMalloc of the compaction buffers failed");
  }
  e = cudaMemset(buf, 0, ar.off);
  if (e != cudaSuccess) {
    cudaFree(buf);
    return ctx->cuda_fail(e, "cudaMemset");
  }
  char* base = static_cast<char*>(buf);
  ctx->compact_buf = buf;
  ctx->T_full = T_full;
  for (size_t l = 0; l < oa.size(); ++l) {
    ctx->comp_A.push_back(base + oa[l]);
    ctx->comp_G.push_back(base + og[l]);
  }
  ctx->comp_idx = reinterpret_cast<int32_t*>(base + o_idx);
  ctx->comp_counts = reinterpret_cast<int32_t*>(base + o_cnt);
  ctx->comp_overflow = reinterpret_cast<int*>(base + o_flag);
  return GRAPE_OK;
}

int grape_step_masked(grape_ctx* ctx, const void* const* A, const void* const* Gout, float* const* W,
                      const uint8_t* mask_dev, int64_t step, void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (!ctx->compact_buf) return ctx->fail(GRAPE_EINVAL, "call grape_enable_compaction first");
  if (!mask_dev) return ctx->fail(GRAPE_EINVAL, "mask_dev must not be null");
  int rc = check_step_index(ctx, step);
  if (rc) return rc;
  rc = validate_io(ctx, A, Gout, W, true, true);
  if (rc) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const grape::StepShape& sh = ctx->sh;
  const NvtxRange range("grape_step_masked");
  rc = phase(ctx, GRAPE_PHASE_COMPACT, "compact live tokens", st, [&](int* n) {
    *n = 2;
    cudaError_t e = grape::compact_live_index(mask_dev, sh.B, ctx->T_full, sh.T, ctx->comp_idx,
                                              ctx->comp_counts, ctx->comp_overflow, st);
    if (e != cudaSuccess) return e;
    grape::CompactTable tb{};
    for (int l = 0; l < sh.L; ++l) {
      tb.A[l] = A[l];
      tb.G[l] = Gout[l];
      tb.Ac[l] = ctx->comp_A[l];
      tb.Gc[l] = ctx->comp_G[l];
      tb.d_in[l] = ctx->layers[l].d_in;
      tb.d_out[l] = ctx->layers[l].d_out;
    }
    return grape::compact_gather(tb, sh.L, sh.B, ctx->T_full, sh.T, static_cast<int>(in_elsize(sh.dtype)),
                                 ctx->comp_idx, st);
  });
  if (rc) return rc;
  return run_step(ctx, ctx->comp_A.data(), ctx->comp_G.data(), W, step, st);
}

int grape_live_counts(grape_ctx* ctx, int32_t* counts_host) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  if (!ctx->compact_buf) return ctx->fail(GRAPE_EINVAL, "compaction is not enabled");
  if (!counts_host) return ctx->fail(GRAPE_EINVAL, "counts_host must not be null");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return ctx->cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpy(counts_host, ctx->comp_counts, sizeof(int32_t) * ctx->sh.B, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return ctx->cuda_fail(e, "cudaMemcpy");
  return check_device_error(ctx);
}

int grape_set_graph(grape_ctx* ctx, int32_t enable) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (!enable) {
    for (auto& g : ctx->graphs) ctx->drop_graph(g);
    ctx->graphs.clear();
  }
  ctx->graph_on = enable != 0;
  return GRAPE_OK;
}

int grape_set_norm_method(grape_ctx* ctx, int32_t method) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (method != GRAPE_NORM_DIRECT && method != GRAPE_NORM_GHOST)
    return ctx->fail(GRAPE_EINVAL, "method must be GRAPE_NORM_DIRECT or GRAPE_NORM_GHOST");
  if (method == GRAPE_NORM_GHOST &&
      (ctx->path != GRAPE_PATH_TC || !grape::tc_ghost_supported(ctx->sh)))
    return ctx->fail(GRAPE_EUNSUPPORTED, "the ghost norm runs on the tensor-core path");
  if (method != ctx->norm_method) {   // captured graphs hold the other norm kernel
    for (auto& g : ctx->graphs) ctx->drop_graph(g);
    ctx->graphs.clear();
  }
  ctx->norm_method = method;
  return GRAPE_OK;
}

int grape_set_aggregation(grape_ctx* ctx, int32_t method) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (method != GRAPE_AGG_AUTO && method != GRAPE_AGG_RECOMPUTE && method != GRAPE_AGG_STORE)
    return ctx->fail(GRAPE_EINVAL, "method must be GRAPE_AGG_AUTO, GRAPE_AGG_RECOMPUTE or GRAPE_AGG_STORE");
  int resolved = method;
  if (resolved == GRAPE_AGG_AUTO)
    resolved = auto_stores_R(ctx->path, ctx->sh.T) ? GRAPE_AGG_STORE : GRAPE_AGG_RECOMPUTE;
  if (resolved == GRAPE_AGG_STORE) {
    if (ctx->path != GRAPE_PATH_TC)
      return ctx->fail(GRAPE_EUNSUPPORTED, "the stored aggregation runs on the tensor-core path");
    if (int rc = check_device(ctx)) return rc;
    if (!ctx->ws[0].Rst) {   // not in the arena: one allocation for every layer's R_i
      const size_t bytes = rstore_bytes(ctx->layers.data(), ctx->sh.L, ctx->sh.r, ctx->sh.B);
      void* buf = nullptr;
      if (fault_alloc_index() == 2 || cudaMalloc(&buf, bytes) != cudaSuccess) {
        cudaGetLastError();
        return ctx->fail(GRAPE_ENOMEM, "cudaMalloc of " + std::to_string(bytes) + " bytes for the stored R_i failed");
      }
      ctx->rst_buf = buf;
      char* at = static_cast<char*>(buf);
      for (int l = 0; l < ctx->sh.L; ++l) {
        ctx->ws[l].Rst = reinterpret_cast<__nv_bfloat16*>(at);
        at += static_cast<size_t>(ctx->sh.B) * ctx->sh.r * ctx->layers[l].d_out * 2;
      }
    }
  }
  if (resolved != ctx->agg) {   // captured graphs hold the other aggregation
    for (auto& g : ctx->graphs) ctx->drop_graph(g);
    ctx->graphs.clear();
  }
  ctx->agg = resolved;
  return GRAPE_OK;
}

int grape_aggregation_of(const grape_ctx* ctx, int32_t* method) {
  if (!ctx || !method) return set_global(GRAPE_EINVAL, "ctx and method must not be null");
  *method = ctx->stores_R() && ctx->path == GRAPE_PATH_TC ? GRAPE_AGG_STORE : GRAPE_AGG_RECOMPUTE;
  return GRAPE_OK;
}

int grape_set_refresh_period(grape_ctx* ctx, int32_t period) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (period < 1) return ctx->fail(GRAPE_EINVAL, "refresh period must be >= 1");
  ctx->refresh = static_cast<uint32_t>(period);
  ctx->p_key = -1;   // the next step draws P afresh
  return GRAPE_OK;
}

int grape_sqnorms(grape_ctx* ctx, const void* const* A, const void* const* Gout, int64_t step,
                  float* sqnorms_dev, void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  int rc = check_step_index(ctx, step);
  if (rc) return rc;
  rc = validate_io(ctx, A, Gout, nullptr, true, false);
  if (rc) return rc;
  if (!sqnorms_dev || (reinterpret_cast<uintptr_t>(sqnorms_dev) & 3u) != 0)
    return ctx->fail(GRAPE_EINVAL, "sqnorms_dev must be a non-null, 4-byte aligned device pointer");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const NvtxRange range("grape_sqnorms");
  std::vector<grape::LayerIo> io(ctx->sh.L);
  for (int l = 0; l < ctx->sh.L; ++l) io[l] = grape::LayerIo{A[l], Gout[l], nullptr};
  rc = run_project_norm(ctx, io.data(), step, st, false);
  if (rc) return rc;
  return phase(ctx, GRAPE_PHASE_CLIP, "sum norm partials", st, [&](int* n) {
    *n = 1;
    return grape::sum_partials(ctx->sh, ctx->partials, sqnorms_dev, st);
  });
}

int grape_get_state(grape_ctx* ctx, int32_t layer, float* m_dev, float* v_dev, void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  if (layer < 0 || layer >= ctx->sh.L) return ctx->fail(GRAPE_EINVAL, "layer out of range");
  if (!m_dev || !v_dev) return ctx->fail(GRAPE_EINVAL, "m_dev and v_dev must not be null");
  const size_t bytes = static_cast<size_t>(ctx->sh.r) * ctx->layers[layer].d_out * 4;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(m_dev, ctx->ws[layer].m, bytes, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(v_dev, ctx->ws[layer].v, bytes, cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? GRAPE_OK : ctx->cuda_fail(e, "get_state copy");
}

int grape_set_state(grape_ctx* ctx, int32_t layer, const float* m_dev, const float* v_dev,
                    void* stream) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  if (layer < 0 || layer >= ctx->sh.L) return ctx->fail(GRAPE_EINVAL, "layer out of range");
  if (!m_dev || !v_dev) return ctx->fail(GRAPE_EINVAL, "m_dev and v_dev must not be null");
  const size_t bytes = static_cast<size_t>(ctx->sh.r) * ctx->layers[layer].d_out * 4;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(ctx->ws[layer].m, m_dev, bytes, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(ctx->ws[layer].v, v_dev, bytes, cudaMemcpyDeviceToDevice, st);
  return e == cudaSuccess ? GRAPE_OK : ctx->cuda_fail(e, "set_state copy");
}

int grape_debug(grape_ctx* ctx, int32_t what, int32_t layer, void* host_out) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  if (!host_out) return ctx->fail(GRAPE_EINVAL, "host_out must not be null");
  const bool per_layer = what >= GRAPE_DBG_S;
  if (what < GRAPE_DBG_NORMS || what > GRAPE_DBG_V) return ctx->fail(GRAPE_EINVAL, "unknown debug item");
  if (per_layer && (layer < 0 || layer >= ctx->sh.L)) return ctx->fail(GRAPE_EINVAL, "layer out of range");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return ctx->cuda_fail(e, "synchronize");
  if (int rc = check_device_error(ctx)) return rc;
  const int r = ctx->sh.r;
  const bool tc = ctx->path == GRAPE_PATH_TC;
  const grape::LayerWs* w = per_layer ? &ctx->ws[layer] : nullptr;
  auto copy_bf16_as_f32 = [&](const void* src, size_t n) -> cudaError_t {
    std::vector<uint16_t> tmp(n);
    cudaError_t ce = cudaMemcpy(tmp.data(), src, n * 2, cudaMemcpyDeviceToHost);
    float* o = static_cast<float*>(host_out);
    for (size_t k = 0; k < n; ++k) {
      uint32_t u = static_cast<uint32_t>(tmp[k]) << 16;
      std::memcpy(&o[k], &u, 4);
    }
    return ce;
  };
  switch (what) {
    case GRAPE_DBG_NORMS:
      e = cudaMemcpy(host_out, ctx->norms, ctx->sh.B * 4, cudaMemcpyDeviceToHost);
      break;
    case GRAPE_DBG_CLIP:
      e = cudaMemcpy(host_out, ctx->clip, ctx->sh.B * 4, cudaMemcpyDeviceToHost);
      break;
    case GRAPE_DBG_S:
      e = cudaMemcpy(host_out, w->S, static_cast<size_t>(r) * w->d_out * 4, cudaMemcpyDeviceToHost);
      break;
    case GRAPE_DBG_M:
      e = cudaMemcpy(host_out, w->m, static_cast<size_t>(r) * w->d_out * 4, cudaMemcpyDeviceToHost);
      break;
    case GRAPE_DBG_V:
      e = cudaMemcpy(host_out, w->v, static_cast<size_t>(r) * w->d_out * 4, cudaMemcpyDeviceToHost);
      break;
    case GRAPE_DBG_P:
      e = tc ? copy_bf16_as_f32(w->P16, static_cast<size_t>(w->d_in) * r)
             : cudaMemcpy(host_out, w->P32, static_cast<size_t>(w->d_in) * r * 4, cudaMemcpyDeviceToHost);
      break;
    case GRAPE_DBG_DR:
      e = tc ? copy_bf16_as_f32(w->dR, static_cast<size_t>(r) * w->d_out)
             : cudaMemcpy(host_out, w->dR, static_cast<size_t>(r) * w->d_out * 4, cudaMemcpyDeviceToHost);
      break;
  }
  return e == cudaSuccess ? GRAPE_OK : ctx->cuda_fail(e, "debug copy");
}

int grape_profile(grape_ctx* ctx, int32_t enable) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return ctx->cuda_fail(e, "synchronize");
  ctx->marks.clear();
  ctx->ev_used = 0;
  ctx->prof_on = enable != 0;
  return GRAPE_OK;
}

int grape_profile_read(grape_ctx* ctx, double* ms_out, int64_t* count_out) {
  if (!ctx) return set_global(GRAPE_EINVAL, "ctx must not be null");
  if (int rc = check_device(ctx)) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return ctx->cuda_fail(e, "synchronize");
  double ms[GRAPE_N_PHASES] = {};
  int64_t cnt[GRAPE_N_PHASES] = {};
  for (const auto& mk : ctx->marks) {
    float t = 0.0f;
    e = cudaEventElapsedTime(&t, mk.a, mk.b);
    if (e != cudaSuccess) return ctx->cuda_fail(e, "cudaEventElapsedTime");
    ms[mk.phase] += t;
    cnt[mk.phase] += 1;
  }
  ctx->marks.clear();
  ctx->ev_used = 0;
  if (int rc = check_device_error(ctx)) return rc;
  for (int k = 0; k < GRAPE_N_PHASES; ++k) {
    if (ms_out) ms_out[k] = ms[k];
    if (count_out) count_out[k] = cnt[k];
  }
  return GRAPE_OK;
}

int grape_launch_count(const grape_ctx* ctx, uint64_t* launches) {
  if (!ctx || !launches) return set_global(GRAPE_EINVAL, "ctx and launches must not be null");
  *launches = ctx->launches;
  return GRAPE_OK;
}

int grape_device_bytes(const grape_ctx* ctx, uint64_t* bytes) {
  if (!ctx || !bytes) return set_global(GRAPE_EINVAL, "ctx and bytes must not be null");
  *bytes = ctx->arena_bytes;
  return GRAPE_OK;
}

int grape_path_of(const grape_ctx* ctx, int32_t* path) {
  if (!ctx || !path) return set_global(GRAPE_EINVAL, "ctx and path must not be null");
  *path = ctx->path;
  return GRAPE_OK;
}

const char* grape_last_error(const grape_ctx* ctx) { return ctx ? ctx->err.c_str() : ""; }

const char* grape_global_error(void) { return g_global_error.c_str(); }

int grape_context_bytes(const grape_layer* layers, int32_t n_layers, int32_t r, int32_t B, int32_t T,
                        int32_t in_dtype, int32_t path, uint64_t* bytes) {
  if (!bytes || !layers) return set_global(GRAPE_EINVAL, "layers and bytes must not be null");
  if (n_layers < 1 || n_layers > GRAPE_MAX_LAYERS)
    return set_global(GRAPE_EINVAL, "n_layers must be in [1, " + std::to_string(GRAPE_MAX_LAYERS) + "]");
  if (B < 1 || T < 1) return set_global(GRAPE_EINVAL, "B and T must be >= 1");
  if (r < 1) return set_global(GRAPE_EINVAL, "r must be >= 1");
  if (in_dtype != GRAPE_F32 && in_dtype != GRAPE_BF16)
    return set_global(GRAPE_EINVAL, "in_dtype must be GRAPE_F32 or GRAPE_BF16");
  if (path < GRAPE_PATH_AUTO || path > GRAPE_PATH_TC)
    return set_global(GRAPE_EINVAL, "path must be a grape_path value");
  for (int l = 0; l < n_layers; ++l) {
    if (layers[l].d_in < 1 || layers[l].d_out < 1)
      return set_global(GRAPE_EINVAL, "layer " + std::to_string(l) + ": d_in and d_out must be >= 1");
    if (r > layers[l].d_in)
      return set_global(GRAPE_EINVAL, "layer " + std::to_string(l) + ": r must be <= d_in");
  }
  if (static_cast<int64_t>(B) * T > (int64_t{1} << 31) / 4) return set_global(GRAPE_EINVAL, "B*T too large");
  const int resolved = path == GRAPE_PATH_AUTO ? (in_dtype == GRAPE_BF16 ? GRAPE_PATH_TC : GRAPE_PATH_SIMT) : path;
  if (resolved == GRAPE_PATH_TC && in_dtype != GRAPE_BF16)
    return set_global(GRAPE_EUNSUPPORTED, "the tensor-core path takes bf16 inputs");
  // the arena of grape_create, block by block in its order
  const bool tc = resolved == GRAPE_PATH_TC;
  Arena ar;
  size_t s_total = 0;
  for (int l = 0; l < n_layers; ++l) s_total += static_cast<size_t>(r) * layers[l].d_out;
  ar.take(s_total * 4);                                         // every S_l
  int part = 0;
  std::vector<grape::LayerWs> ws(n_layers);
  for (int l = 0; l < n_layers; ++l) {
    const size_t di = layers[l].d_in, dout = layers[l].d_out;
    ar.take(di * r * (tc ? 2 : 4));                             // P (bf16 or fp32)
    ar.take(static_cast<size_t>(B) * T * r * (tc ? 2 : 4));     // AP
    ar.take(r * dout * 4);                                      // m
    ar.take(r * dout * 4);                                      // v
    ar.take(r * dout * (tc ? 2 : 4));                           // dR
    ws[l].d_in = layers[l].d_in;
    ws[l].d_out = layers[l].d_out;
    ws[l].part_base = part;
    ws[l].part_count = tc ? grape::tc_partials_per_sample(r, layers[l].d_out)
                          : grape::simt_partials_per_sample(r, layers[l].d_out);
    part += ws[l].part_count;
  }
  ar.take(static_cast<size_t>(B) * part * 4);                   // norm partials
  ar.take(static_cast<size_t>(B) * 4);                          // norms
  ar.take(static_cast<size_t>(B) * 4);                          // clip factors
  if (tc) {
    grape::StepShape sh{};
    sh.L = n_layers;
    sh.r = r;
    sh.B = B;
    sh.T = T;
    sh.dtype = in_dtype;
    sh.part_stride = part;
    ar.take(grape::tc_workspace_bytes(sh, ws.data()));
  }
  if (auto_stores_R(resolved, T))                               // stored R_i (GRAPE_AGG_AUTO)
    for (int l = 0; l < n_layers; ++l) ar.take(static_cast<size_t>(B) * r * layers[l].d_out * 2);
  *bytes = ar.off;
  return GRAPE_OK;
}

void grape_destroy(grape_ctx* ctx) {
  if (!ctx) return;
  grape::tc_release(&ctx->tc);
  for (cudaEvent_t e : ctx->ev_pool) cudaEventDestroy(e);
  for (void* p : ctx->stage_A) cudaFree(p);
  for (void* p : ctx->stage_G) cudaFree(p);
  if (ctx->arena) cudaFree(ctx->arena);
  if (ctx->compact_buf) cudaFree(ctx->compact_buf);
  if (ctx->rst_buf) cudaFree(ctx->rst_buf);
  for (auto& g : ctx->graphs) ctx->drop_graph(g);
  if (ctx->capture_stream) cudaStreamDestroy(ctx->capture_stream);
  delete ctx;
}

int grape_philox_words(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id,
                       int64_t n_blocks, uint32_t* out_dev, void* stream) {
  if (n_blocks < 0 || n_blocks > 0xFFFFFFFFll) return set_global(GRAPE_EINVAL, "n_blocks out of range");
  if (n_blocks == 0) return GRAPE_OK;
  if (!out_dev || !aligned16(out_dev)) return set_global(GRAPE_EINVAL, "out_dev null or not 16-byte aligned");
  cudaError_t e = grape::launch_philox_words(seed, layer, step, stream_id, n_blocks, out_dev,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GRAPE_OK : set_global(GRAPE_ECUDA, cudaGetErrorString(e));
}

int grape_gaussian(uint64_t seed, uint32_t layer, uint32_t step, uint32_t stream_id, int64_t n,
                   float* out_dev, void* stream) {
  if (n < 0 || n > 4 * 0xFFFFFFFFll) return set_global(GRAPE_EINVAL, "n out of range");
  if (n == 0) return GRAPE_OK;
  if (!out_dev) return set_global(GRAPE_EINVAL, "out_dev must not be null");
  cudaError_t e = grape::launch_gaussian(seed, layer, step, stream_id, n, out_dev,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GRAPE_OK : set_global(GRAPE_ECUDA, cudaGetErrorString(e));
}

int grape_selftest_wait_timeout(int64_t short_ns, int64_t long_ns, int32_t* bits_out) {
  if (short_ns < 0 || short_ns > 1000000000ll || long_ns < short_ns || long_ns > 10000000000ll)
    return set_global(GRAPE_EINVAL, "need 0 <= short_ns <= 1e9 and short_ns <= long_ns <= 1e10");
  int* bits = nullptr;
  cudaError_t e = cudaMalloc(&bits, sizeof(int));
  if (e != cudaSuccess) return set_global(GRAPE_ENOMEM, cudaGetErrorString(e));
  e = cudaMemset(bits, 0, sizeof(int));
  if (e == cudaSuccess)
    e = grape::tc_selftest_wait(static_cast<uint64_t>(short_ns), static_cast<uint64_t>(long_ns), bits, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int v = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&v, bits, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(bits);
  if (e != cudaSuccess) return set_global(GRAPE_ECUDA, cudaGetErrorString(e));
  if (bits_out) *bits_out = v;
  if (v & 1) return set_global(GRAPE_ETIMEOUT, "a bounded device wait gave up (self-test)");
  return GRAPE_OK;
}

int grape_layer_sqnorms_static(const void* A, const void* Gout, int32_t d_in, int32_t d_out,
                               int32_t r, int32_t B, int32_t T, uint64_t seed, uint32_t layer,
                               uint32_t step, float* sqnorms_out, void* stream) {
  if (!A || !Gout || !sqnorms_out) return set_global(GRAPE_EINVAL, "A, Gout and sqnorms_out must not be null");
  if (!aligned16(A) || !aligned16(Gout)) return set_global(GRAPE_EINVAL, "A and Gout must be 16-byte aligned");
  if (B < 1 || T < 1 || d_in < 1 || d_out < 1 || r < 1 || r > d_in)
    return set_global(GRAPE_EINVAL, "need B, T, d_in, d_out >= 1 and 1 <= r <= d_in");
  if (r % 128 != 0 || (r > 256 && r % 256 != 0) || d_in % 8 != 0 || d_out % 256 != 0)
    return set_global(GRAPE_EINVAL, "need r % 128 == 0 (and % 256 above 256), d_in % 8 == 0, d_out % 256 == 0");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_global(GRAPE_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return set_global(GRAPE_EUNSUPPORTED, "needs an sm_100a device (B200)");
  if (!grape::tc_tensor_maps_available())
    return set_global(GRAPE_EUNSUPPORTED, "cuTensorMapEncodeTiled is not available from the driver");
  const size_t need = grape::tc_static_scratch_needed(d_in, d_out, r, B, T);
  if (need > grape::tc_static_scratch_bytes())
    return set_global(GRAPE_EINVAL, "problem needs " + std::to_string(need) + " bytes of scratch; the static scratch holds " +
                                        std::to_string(grape::tc_static_scratch_bytes()) +
                                        " (d_in*r*2 + B*T*r*2 + B*slots*4 + 256 bytes)");
  e = grape::tc_layer_sqnorms_static(A, Gout, d_in, d_out, r, B, T, seed, layer, step, sqnorms_out,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_global(GRAPE_ECUDA, std::string("layer sqnorms: ") + cudaGetErrorString(e));
  return GRAPE_OK;
}

}  // extern "C"
