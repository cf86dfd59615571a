// psispec.cu -- C ABI of libpsispec.so: argument checks, workspace layout and launches.
// The operations are specified in include/psispec.h.
#include "psispec.h"

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "cutrow.cuh"
#include "draw.cuh"
#include "finish.cuh"
#include "linear.cuh"
#include "sample.cuh"
#include "stats.cuh"
#include "topp.cuh"
#include "tree.cuh"
#include "trie.cuh"

namespace psi {
namespace {

constexpr int64_t kMaxRows = int64_t(1) << 26;
constexpr int64_t kMaxV = int64_t(1) << 24;
constexpr int64_t kMaxGrid = 0x7fffffff;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Carves a workspace into 256-byte aligned regions; with base == nullptr it only measures.
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename X>
  X* take(int64_t count) {
    X* p = base ? reinterpret_cast<X*>(base + used) : nullptr;
    used += align256(static_cast<size_t>(count) * sizeof(X));
    return p;
  }
};

struct StatsWs {
  Partial* parts;
  RowStat* stats;
};
StatsWs carve_stats(Carver& c, int64_t rows, int nch) {
  return StatsWs{c.take<Partial>(rows * nch), c.take<RowStat>(rows)};
}

struct SampleWs {
  StatsWs st;
};
SampleWs carve_sample(Carver& c, int64_t rows, int64_t V) {
  SampleWs w;
  w.st = carve_stats(c, rows, nchunks_for(V));
  return w;
}

struct LinearWs {
  StatsWs t, d;
  Job* jobs;
  int32_t* cnt;      // arrival counters, one per request
  double2* draw_tc;   // per (draw job, chunk) weight totals
  double2* draw_tg;   // per (draw job, chunk, group) weight totals
};
LinearWs carve_linear(Carver& c, int64_t B, int64_t K, int64_t V) {
  const int ns = nchunks_for(V);
  LinearWs w;
  w.t = carve_stats(c, B * (K + 1), ns);
  w.d = carve_stats(c, B * K, ns);
  w.jobs = c.take<Job>(B);
  w.cnt = c.take<int32_t>(B);
  w.draw_tc = c.take<double2>(B * ns);
  w.draw_tg = c.take<double2>(B * ns * kChunkGroups);
  return w;
}

// psispec_row_stats: the chunk partials (the records go to the caller's array).
Partial* carve_row_stats(Carver& c, int64_t rows, int64_t V) { return c.take<Partial>(rows * nchunks_for(V)); }

struct TreeWs {
  StatsWs st;  // rows [0, N) of the verifier tensor, then [N, 2N) of the draft tensor
};
TreeWs carve_tree(Carver& c, int64_t N, int64_t V) {
  TreeWs w;
  w.st = carve_stats(c, 2 * N, nchunks_for(V));
  return w;
}

psispec_status check_ws(const void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PSISPEC_ERR_WORKSPACE;
  return PSISPEC_OK;
}

inline bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// One kernel launch on the caller's stream; a launch error becomes PSISPEC_ERR_CUDA.
template <typename... KArgs, typename... Args>
psispec_status launch(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? PSISPEC_OK : PSISPEC_ERR_CUDA;
}

// Persistent grid for a warp-granular streaming kernel: one CTA per resident slot, fewer
// when there is less work than that.
template <typename Kern>
unsigned persistent_grid(Kern kernel, int64_t work_warps) {
  int dev = 0, sms = 148, occ = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, 0);
  const int64_t want = (work_warps + (kThreads / 32) - 1) / (kThreads / 32);
  const int64_t slots = static_cast<int64_t>(sms) * (occ > 0 ? occ : 1);
  return static_cast<unsigned>(want < 1 ? 1 : (want < slots ? want : slots));
}

// Persistent grid for a warp-granular kernel with `warps` warps per CTA and dynamic shared
// memory: one CTA per resident slot, fewer when there is less work than that.
template <typename Kern>
int64_t want_slots(int64_t work_warps, int warps, Kern kernel, int block, int smem) {
  int dev = 0, sms = 148, occ = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, block, smem);
  const int64_t want = (work_warps + warps - 1) / warps;
  const int64_t slots = static_cast<int64_t>(sms) * (occ > 0 ? occ : 1);
  return want < 1 ? 1 : (want < slots ? want : slots);
}

// Rows [0, rows) of one tensor, rows_per_req consecutive rows per request.
template <typename T>
RowSet<T> one_tensor(const T* base, int64_t rows, int rows_per_req, int nreq) {
  return RowSet<T>{base, nullptr, rows, rows_per_req, nullptr, nreq};
}

// The streaming pass over `rows` rows of a row set: one partial per chunk. Aligned tensors go
// through the bulk-copy ring kernel, others through plain 16-byte loads.
template <typename T>
psispec_status launch_stream(RowSet<T> set, int64_t rows, int V, const float* temperature, int nreq, Partial* parts,
                             cudaStream_t st, Skip skip = Skip{nullptr, nullptr, kSkipNone}, int32_t* zero = nullptr,
                             int nzero = 0) {
  const int64_t chunks = rows * nchunks_for(V);
  const bool aligned = (reinterpret_cast<uintptr_t>(set.a) & 15u) == 0 &&
                       (reinterpret_cast<uintptr_t>(set.b) & 15u) == 0 && (int64_t(V) * sizeof(T)) % 16 == 0;
  if (aligned) {
    const int smem = (kThreads / 32) * kRing * kStageBytes<T>;
    if (cudaFuncSetAttribute(stream_partials_tma_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return PSISPEC_ERR_CUDA;
    int dev = 0, sms = 148, occ = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, stream_partials_tma_kernel<T>, kThreads, smem);
    const int64_t want = (chunks + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t slots = static_cast<int64_t>(sms) * (occ > 0 ? occ : 1);
    const unsigned grid = static_cast<unsigned>(want < slots ? want : slots);
    return launch(stream_partials_tma_kernel<T>, grid, kThreads, smem, st, set, V, chunks, temperature, skip, nreq,
                  parts, zero, nzero);
  }
  return launch(stream_partials_kernel<T>, persistent_grid(stream_partials_kernel<T>, chunks), kThreads, 0, st, set, V,
                chunks, temperature, skip, parts, zero, nzero);
}

// Row statistics of `rows` rows of a row set (the tree's statistics pass, psispec_row_stats);
// the rows of the requests that `skip` selects are left out.
template <typename T>
psispec_status launch_stats(RowSet<T> set, int64_t rows, int V, const float* temperature, int nreq,
                            const float* top_p, const int32_t* top_k, Skip skip, StatsWs ws, cudaStream_t st) {
  psispec_status s = launch_stream<T>(set, rows, V, temperature, nreq, ws.parts, st, skip);
  if (s != PSISPEC_OK) return s;
  return launch(row_finalize_kernel<T>, static_cast<unsigned>((rows + kThreads / 32 - 1) / (kThreads / 32)), kThreads,
                0, st, set, rows, V, temperature, top_p, top_k, ws.parts, ws.stats, skip);
}

// bf16 rows of cut requests go through the one-pass cut-row path; the streaming pass leaves
// them alone. fp32 rows of such requests need the streaming pass's partials.
template <typename T>
Skip cut_skip(const float* top_p, const int32_t* top_k) {
  return Skip{top_p, top_k, sizeof(T) == 2 ? kSkipCut : kSkipNone};
}

// Launch configuration of `nclusters` clusters of CL CTAs of `threads` threads; returns
// PSISPEC_ERR_UNSUPPORTED when the device cannot schedule such a cluster. cfg.attrs points at
// attr.
template <typename Kern>
psispec_status cluster_config(Kern kernel, int64_t nclusters, int CL, int threads, int smem, cudaStream_t st,
                              cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&attr)[1]) {
  if (CL > 8 && cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return PSISPEC_ERR_UNSUPPORTED;
  }
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3(static_cast<unsigned>(nclusters * CL));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters < 1) {
    cudaGetLastError();
    return PSISPEC_ERR_UNSUPPORTED;
  }
  return PSISPEC_OK;
}

// The draw jobs of a verification call: one cluster per job (16 CTAs where the device can
// schedule such clusters, else 8), else a totals pass (bulk-copy ring when the rows allow it)
// and a pick pass.
template <typename T>
psispec_status launch_draws(const T* A, const T* Bt, int V, int njobs, const Partial* parts_a, const Job* jobs,
                            double2* tc, double2* tg, int32_t* out_tokens, cudaStream_t st) {
  {
    // clusters of 8 CTAs where each warp's part fits the step buffer, else of 16
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    psispec_status s = PSISPEC_ERR_UNSUPPORTED;
    if (draw_part(V, 8) <= kDrawMaxSteps * 256) {
      s = cluster_config(draw_cluster_kernel<T, 8>, njobs, 8, kDrawClusterWarps * 32, 0, st, cfg, attr);
      if (s == PSISPEC_OK)
        return cudaLaunchKernelEx(&cfg, draw_cluster_kernel<T, 8>, A, Bt, V, parts_a, jobs, out_tokens) == cudaSuccess
                   ? PSISPEC_OK
                   : PSISPEC_ERR_CUDA;
      if (s != PSISPEC_ERR_UNSUPPORTED) return s;
    }
    if (draw_part(V, 16) <= kDrawMaxSteps * 256) {
      s = cluster_config(draw_cluster_kernel<T, 16>, njobs, 16, kDrawClusterWarps * 32, 0, st, cfg, attr);
      if (s == PSISPEC_OK)
        return cudaLaunchKernelEx(&cfg, draw_cluster_kernel<T, 16>, A, Bt, V, parts_a, jobs, out_tokens) ==
                       cudaSuccess
                   ? PSISPEC_OK
                   : PSISPEC_ERR_CUDA;
      if (s != PSISPEC_ERR_UNSUPPORTED) return s;
    }
  }
  const int64_t items = int64_t(njobs) * nchunks_for(V);
  // the bulk-copy ring serves bf16 rows (fp32 stages would not fit enough warps per SM)
  const bool ring = sizeof(T) == 2 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0 &&
                    (reinterpret_cast<uintptr_t>(Bt) & 15u) == 0 && (int64_t(V) * sizeof(T)) % 16 == 0;
  const int smem = kDrawWarps * kDrawRing * kDrawStageBytes<T>;
  if (ring && cudaFuncSetAttribute(draw_totals_tma_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                  cudaSuccess)
    return PSISPEC_ERR_CUDA;
  psispec_status s;
  if (ring)
    s = launch(draw_totals_tma_kernel<T>, static_cast<unsigned>(want_slots(items, kDrawWarps, draw_totals_tma_kernel<T>,
                                                                           kDrawWarps * 32, smem)),
               kDrawWarps * 32, smem, st, A, Bt, V, njobs, jobs, tc, tg);
  else
    s = launch(draw_totals_kernel<T>, persistent_grid(draw_totals_kernel<T>, items), kThreads, 0, st, A, Bt, V, njobs,
               jobs, tc, tg);
  if (s != PSISPEC_OK) return s;
  return launch(draw_pick_kernel<T>, static_cast<unsigned>((njobs + kThreads / 32 - 1) / (kThreads / 32)), kThreads, 0,
                st, A, Bt, V, njobs, parts_a, jobs, tc, tg, out_tokens);
}

// The cut-row CTAs of a row kernel: persistent (one per resident slot) over the call's rows.
template <typename T, typename Kern>
psispec_status prepare_topp(Kern kernel, int64_t rows, unsigned* grid) {
  const int smem = static_cast<int>(sizeof(CutSmem<T>));
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return PSISPEC_ERR_CUDA;
  *grid = static_cast<unsigned>(want_slots(rows, 1, kernel, kTpThreads, smem));
  return PSISPEC_OK;
}

template <typename T>
psispec_status sample_draft_impl(const T* draft, int B, int K, int V, const float* temperature, const float* top_p,
                                 const int32_t* top_k, const float* u, int32_t* out_tokens, float* out_q, RowStat* out_stats, void* ws,
                                 cudaStream_t st) {
  const int64_t rows = int64_t(B) * K;
  Carver c(ws);
  SampleWs w = carve_sample(c, rows, V);
  RowStat* stats = out_stats ? out_stats : w.st.stats;
  // the rows of requests without a cut (and fp32 rows) through the streaming pass (maximum and
  // normaliser); the row kernel's warps finish them, its cut-row CTAs take the others
  psispec_status s = launch_stream<T>(one_tensor(draft, rows, K, B), rows, V, temperature, B, w.st.parts, st,
                                      cut_skip<T>(top_p, top_k));
  if (s != PSISPEC_OK) return s;
  unsigned tgrid = 1;
  if ((s = prepare_topp<T>(sample_rows_kernel<T>, rows, &tgrid)) != PSISPEC_OK) return s;
  const int warp_ctas = static_cast<int>((rows + kTpWarps - 1) / kTpWarps);
  CutArgs ca{};
  ca.mode = kCutSample;
  ca.V = V;
  ca.rows_a = static_cast<int>(rows);
  ca.per_a = K;
  ca.rows_b = 0;
  ca.per_b = 1;
  ca.temperature = temperature;
  ca.top_p = top_p;
  ca.top_k = top_k;
  ca.u = u;
  ca.out_tokens = out_tokens;
  ca.out_q = out_q;
  ca.stats_a = stats;
  return launch(sample_rows_kernel<T>, warp_ctas + tgrid, kTpThreads, sizeof(CutSmem<T>), st, draft, K, V,
                static_cast<int>(rows), temperature, top_p, top_k, u, w.st.parts, stats, out_tokens, out_q, warp_ctas,
                ca, VerifyArgs{});
}

template <typename T>
psispec_status verify_linear_impl(const T* tgt, const T* drf, int B, int K, int V, const int32_t* tokens,
                                  const RowStat* draft_stats, const float* u_acc, const float* u_res,
                                  const float* temperature, const float* top_p, const int32_t* top_k,
                                  int32_t* out_tokens, int32_t* out_len, float* out_p, float* out_q, void* ws,
                                  cudaStream_t st) {
  Carver c(ws);
  LinearWs w = carve_linear(c, B, K, V);
  const int64_t rows_t = int64_t(B) * (K + 1), rows_d = draft_stats ? 0 : int64_t(B) * K;
  VerifyArgs a;
  a.B = B;
  a.K = K;
  a.V = V;
  a.stream_draft = draft_stats ? 0 : 1;
  a.temperature = temperature;
  a.top_p = top_p;
  a.top_k = top_k;
  a.tokens = tokens;
  a.dstats_in = draft_stats;
  a.u_acc = u_acc;
  a.u_res = u_res;
  a.parts_t = w.t.parts;
  a.parts_d = w.d.parts;
  a.stats_t = w.t.stats;
  a.stats_d = w.d.stats;
  a.cnt = w.cnt;
  a.out_tokens = out_tokens;
  a.out_len = out_len;
  a.out_p = out_p;
  a.out_q = out_q;
  a.jobs = w.jobs;
  // the first streaming pass also clears the request arrival counters
  const Skip skip = cut_skip<T>(top_p, top_k);
  psispec_status s =
      launch_stream<T>(one_tensor(tgt, rows_t, K + 1, B), rows_t, V, temperature, B, w.t.parts, st, skip, w.cnt, B);
  if (s != PSISPEC_OK) return s;
  if (rows_d > 0 &&
      (s = launch_stream<T>(one_tensor(drf, rows_d, K, B), rows_d, V, temperature, B, w.d.parts, st, skip)) !=
          PSISPEC_OK)
    return s;
  // one row kernel: warps for the requests without a cut, whole CTAs for the others
  unsigned tgrid = 1;
  if ((s = prepare_topp<T>(verify_rows_kernel<T>, rows_t + rows_d, &tgrid)) != PSISPEC_OK) return s;
  const int warp_ctas = static_cast<int>((rows_t + rows_d + kTpWarps - 1) / kTpWarps);
  CutArgs ca{};
  ca.mode = kCutVerify;
  ca.V = V;
  ca.rows_a = static_cast<int>(rows_t);
  ca.per_a = K + 1;
  ca.rows_b = static_cast<int>(rows_d);
  ca.per_b = K;
  ca.temperature = temperature;
  ca.top_p = top_p;
  ca.top_k = top_k;
  ca.stats_a = a.stats_t;
  ca.stats_b = a.stats_d;
  s = launch(verify_rows_kernel<T>, warp_ctas + tgrid, kTpThreads, sizeof(CutSmem<T>), st, tgt, drf, a, ca, warp_ctas);
  if (s != PSISPEC_OK) return s;
  return launch_draws<T>(tgt, drf, V, B, w.t.parts, w.jobs, w.draw_tc, w.draw_tg, out_tokens, st);
}

// Launch configuration of the cluster tree walk with CL CTAs per trie; PSISPEC_ERR_UNSUPPORTED
// when V needs larger slices than shared memory holds or the device cannot schedule such a
// cluster. cfg.attrs points at attr; *dbuf tells whether a second r' buffer fits.
template <typename T, int CL>
psispec_status tree_cluster_config(int B, int V, cudaStream_t st, cudaLaunchConfig_t& cfg,
                                   cudaLaunchAttribute (&attr)[1], int* dbuf) {
  const size_t slice_bytes = static_cast<size_t>(tree_slice(V, CL)) * sizeof(float);
  auto kernel = tree_walk_cluster_kernel<T, CL>;
  int dev = 0, optin = 0;
  cudaFuncAttributes fa;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
    return PSISPEC_ERR_CUDA;
  const size_t room = static_cast<size_t>(optin) > fa.sharedSizeBytes ? optin - fa.sharedSizeBytes : 0;
  if (2 * slice_bytes > room) return PSISPEC_ERR_UNSUPPORTED;
  *dbuf = 3 * slice_bytes <= room;
  const int smem = static_cast<int>((*dbuf ? 3 : 2) * slice_bytes);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return PSISPEC_ERR_CUDA;
  return cluster_config(kernel, B, CL, kTreeWalkThreads, smem, st, cfg, attr);
}

template <typename T>
psispec_status verify_tree_impl(const T* tgt, const T* drf, int B, int N, int V, const int32_t* offs,
                                const int32_t* parent, const int32_t* tokens, const float* u_acc, const float* u_res,
                                const float* temperature, const float* top_p, const int32_t* top_k, int max_depth,
                                int32_t* out_path, int32_t* out_tokens, int32_t* out_len, void* ws, cudaStream_t st) {
  Carver c(ws);
  TreeWs w = carve_tree(c, N, V);
  // the walk: one cluster per trie, the node's rows staged across its CTAs' shared memory (16
  // CTAs where the device can schedule such clusters, else 8), else one CTA per trie
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  int CL = 16, dbuf = 0;
  psispec_status s = tree_cluster_config<T, 16>(B, V, st, cfg, attr, &dbuf);
  if (s == PSISPEC_ERR_UNSUPPORTED) {
    CL = 8;
    s = tree_cluster_config<T, 8>(B, V, st, cfg, attr, &dbuf);
  }
  if (s == PSISPEC_ERR_UNSUPPORTED) CL = 0;
  else if (s != PSISPEC_OK) return s;
  // the cluster walk finds the statistics of uncut requests' visited rows itself; with a top-k
  // array every row goes through the statistics pass (its records carry the top-k threshold)
  const int lazy = CL != 0 && top_k == nullptr;
  // one statistics pass over the rows of both tensors
  s = launch_stats<T>(RowSet<T>{tgt, drf, N, 1, offs, B}, 2 * int64_t(N), V, temperature, B, top_p, top_k,
                      Skip{top_p, top_k, lazy ? kSkipUncut : kSkipNone}, w.st, st);
  if (s != PSISPEC_OK) return s;
  const RowStat* ts = w.st.stats;
  const RowStat* ds = w.st.stats + N;
  cudaError_t e = cudaSuccess;
  if (CL == 16)
    e = cudaLaunchKernelEx(&cfg, tree_walk_cluster_kernel<T, 16>, tgt, drf, V, offs, parent, tokens,
                           ts, ds, u_acc,
                           u_res, temperature, top_p, lazy, dbuf, max_depth, out_path, out_tokens, out_len);
  else if (CL == 8)
    e = cudaLaunchKernelEx(&cfg, tree_walk_cluster_kernel<T, 8>, tgt, drf, V, offs, parent, tokens,
                           ts, ds, u_acc,
                           u_res, temperature, top_p, lazy, dbuf, max_depth, out_path, out_tokens, out_len);
  else
    return launch(tree_walk_kernel<T>, static_cast<unsigned>(B), kTreeThreads, 0, st, tgt, drf, V, offs, parent,
                  tokens, ts, ds, u_acc, u_res, max_depth, out_path, out_tokens, out_len);
  return e == cudaSuccess ? PSISPEC_OK : PSISPEC_ERR_CUDA;
}

template <typename T>
psispec_status row_stats_impl(const T* logits, int B, int K, int V, const float* temperature, const float* top_p,
                              const int32_t* top_k, RowStat* out, void* ws, cudaStream_t st) {
  const int64_t rows = int64_t(B) * K;
  Carver c(ws);
  Partial* parts = carve_row_stats(c, rows, V);
  const Skip skip = cut_skip<T>(top_p, top_k);
  psispec_status s =
      launch_stats<T>(one_tensor(logits, rows, K, B), rows, V, temperature, B, top_p, top_k, skip, StatsWs{parts, out}, st);
  if (s != PSISPEC_OK || skip.mode != kSkipCut) return s;
  // the cut requests' rows: one CTA per row at a time
  const int smem = static_cast<int>(sizeof(CutSmem<T>));
  if (cudaFuncSetAttribute(cut_rows_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return PSISPEC_ERR_CUDA;
  CutArgs a{};
  a.mode = kCutStats;
  a.V = V;
  a.rows_a = static_cast<int>(rows);
  a.per_a = K;
  a.rows_b = 0;
  a.per_b = 1;
  a.temperature = temperature;
  a.top_p = top_p;
  a.top_k = top_k;
  a.stats_a = out;
  return launch(cut_rows_kernel<T>, static_cast<unsigned>(want_slots(rows, 1, cut_rows_kernel<T>, kCrThreads, smem)),
                kCrThreads, smem, st, logits, a, VerifyArgs{}, static_cast<const Partial*>(parts));
}

struct TrieWs {
  StatsWs st;
  int32_t* cand_tok;
  double* cand_q;
  double* cand_l;
  int32_t* ncand;
};
TrieWs carve_trie(Carver& c, int64_t rows, int64_t V) {
  TrieWs w;
  w.st = carve_stats(c, rows, nchunks_for(V));
  w.cand_tok = c.take<int32_t>(rows * kTrieMaxCand);
  w.cand_q = c.take<double>(rows * kTrieMaxCand);
  w.cand_l = c.take<double>(rows * kTrieMaxCand);
  w.ncand = c.take<int32_t>(rows);
  return w;
}

// Candidate trie: row statistics of the B*K draft rows (with the sampling controls), the
// candidates of every row, then the best-first choice per request.
template <typename T>
psispec_status build_tree_impl(const T* draft, int B, int K, int V, const float* temperature, const float* top_p,
                               const int32_t* top_k, int cand_k, int n_prefixes, int32_t* out_parent,
                               int32_t* out_tokens, int32_t* out_depth, double* out_score, int32_t* out_nodes,
                               void* ws, cudaStream_t st) {
  const int64_t rows = int64_t(B) * K;
  Carver c(ws);
  TrieWs w = carve_trie(c, rows, V);
  // rows of requests with T > 0 and no cut: the candidate kernel finds their statistics itself
  psispec_status s = launch_stats<T>(one_tensor(draft, rows, K, B), rows, V, temperature, B, top_p, top_k,
                                     Skip{top_p, top_k, kSkipUncut}, w.st, st);
  if (s != PSISPEC_OK) return s;
  s = launch(trie_candidates_kernel<T>, static_cast<unsigned>(rows), kTrieThreads, 0, st, draft, K, V,
             static_cast<const RowStat*>(w.st.stats), 1, temperature, top_p, top_k, cand_k, w.cand_tok, w.cand_q,
             w.cand_l, w.ncand);
  if (s != PSISPEC_OK) return s;
  return launch(trie_select_kernel, static_cast<unsigned>(B), 32, 0, st, K, n_prefixes,
                static_cast<const int32_t*>(w.cand_tok), static_cast<const double*>(w.cand_q),
                static_cast<const double*>(w.cand_l), static_cast<const int32_t*>(w.ncand), out_parent, out_tokens,
                out_depth, out_score, out_nodes);
}

// Tree verification of a trie whose children were fixed in advance: statistics of the
// verifier rows, then one CTA per trie (no draft rows).
template <typename T>
psispec_status verify_tree_det_impl(const T* tgt, int B, int N, int V, const int32_t* offs, const int32_t* parent,
                                    const int32_t* tokens, const float* u_acc, const float* u_res,
                                    const float* temperature, const float* top_p, const int32_t* top_k,
                                    int max_depth, int32_t* out_path, int32_t* out_tokens, int32_t* out_len, void* ws,
                                    cudaStream_t st) {
  Carver c(ws);
  TreeWs w = carve_tree(c, N, V);
  psispec_status s = launch_stats<T>(RowSet<T>{tgt, tgt, N, 1, offs, B}, int64_t(N), V, temperature, B, top_p, top_k,
                                     Skip{top_p, top_k, kSkipNone}, w.st, st);
  if (s != PSISPEC_OK) return s;
  return launch(tree_walk_det_kernel<T>, static_cast<unsigned>(B), kTreeThreads, 0, st, tgt, V, offs, parent, tokens,
                static_cast<const RowStat*>(w.st.stats), u_acc, u_res, max_depth, out_path, out_tokens, out_len);
}

bool bad_dtype(int dtype) { return dtype != PSISPEC_F32 && dtype != PSISPEC_BF16; }
size_t esize(int dtype) { return dtype == PSISPEC_BF16 ? 2 : 4; }

}  // namespace
}  // namespace psi

// Scratch of psispec_verify_linear_static: one array per device, its address looked up once.
static __device__ __align__(256) unsigned char g_static_workspace[PSISPEC_STATIC_WORKSPACE_BYTES];

namespace psi {
namespace {
constexpr int kMaxDevices = 64;
std::atomic<void*> g_static_workspace_ptr[kMaxDevices];
}  // namespace
}  // namespace psi

using namespace psi;

extern "C" {

const char* psispec_status_string(int status) {
  switch (status) {
    case PSISPEC_OK: return "ok";
    case PSISPEC_ERR_INVALID_ARG: return "invalid argument";
    case PSISPEC_ERR_UNSUPPORTED: return "size beyond the supported limits";
    case PSISPEC_ERR_CUDA: return "CUDA launch failed";
    case PSISPEC_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    default: return "unknown status";
  }
}

int psispec_version(void) { return 100; }

size_t psispec_workspace_size(int op, int64_t a, int64_t b, int64_t c) {
  if (a <= 0 || b <= 0 || c <= 0 || c > kMaxV) return 0;
  Carver m(nullptr);
  switch (op) {
    case PSISPEC_OP_SAMPLE_DRAFT: carve_sample(m, a * b, c); break;
    case PSISPEC_OP_VERIFY_LINEAR: carve_linear(m, a, b, c); break;
    case PSISPEC_OP_VERIFY_TREE: carve_tree(m, b, c); break;
    case PSISPEC_OP_ROW_STATS: carve_row_stats(m, a * b, c); break;
    case PSISPEC_OP_BUILD_TREE: carve_trie(m, a * b, c); break;
    default: return 0;
  }
  return m.used;
}

psispec_status psispec_sample_draft_k(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                      const float* temperature, const float* top_p, const int32_t* top_k,
                                      const float* u, int32_t* out_tokens, float* out_q, void* out_row_stats,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!draft_logits || !temperature || !top_p || !u || !out_tokens || bad_dtype(dtype)) return PSISPEC_ERR_INVALID_ARG;
  if (B <= 0 || K <= 0 || V <= 0) return PSISPEC_ERR_INVALID_ARG;
  if (!aligned_to(draft_logits, esize(dtype)) || (out_row_stats && !aligned_to(out_row_stats, 16)))
    return PSISPEC_ERR_INVALID_ARG;
  const int64_t rows = int64_t(B) * K;
  if (rows > kMaxRows || V > kMaxV || rows * nslices_for(V) > kMaxGrid) return PSISPEC_ERR_UNSUPPORTED;
  psispec_status s = check_ws(workspace, workspace_bytes, psispec_workspace_size(PSISPEC_OP_SAMPLE_DRAFT, B, K, V));
  if (s != PSISPEC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RowStat* rs = static_cast<RowStat*>(out_row_stats);
  if (dtype == PSISPEC_BF16)
    return sample_draft_impl(static_cast<const __nv_bfloat16*>(draft_logits), B, K, V, temperature, top_p, top_k, u,
                             out_tokens, out_q, rs, workspace, st);
  return sample_draft_impl(static_cast<const float*>(draft_logits), B, K, V, temperature, top_p, top_k, u, out_tokens,
                           out_q, rs, workspace, st);
}

psispec_status psispec_sample_draft(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                    const float* temperature, const float* top_p, const float* u,
                                    int32_t* out_tokens, float* out_q, void* out_row_stats, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return psispec_sample_draft_k(draft_logits, dtype, B, K, V, temperature, top_p, nullptr, u, out_tokens, out_q,
                                out_row_stats, workspace, workspace_bytes, stream);
}

psispec_status psispec_verify_linear_k(const void* target_logits, const void* draft_logits, int dtype, int32_t B,
                                       int32_t K, int32_t V, const int32_t* draft_tokens, const void* draft_row_stats,
                                       const float* u_accept, const float* u_resid, const float* temperature,
                                       const float* top_p, const int32_t* top_k, int32_t* out_tokens,
                                       int32_t* out_accept_len, float* out_p, float* out_q, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!target_logits || !draft_logits || !draft_tokens || !u_accept || !u_resid || !temperature || !top_p ||
      !out_tokens || !out_accept_len || bad_dtype(dtype))
    return PSISPEC_ERR_INVALID_ARG;
  if (B <= 0 || K <= 0 || V <= 0) return PSISPEC_ERR_INVALID_ARG;
  if (!aligned_to(target_logits, esize(dtype)) || !aligned_to(draft_logits, esize(dtype)) ||
      (draft_row_stats && !aligned_to(draft_row_stats, 16)))
    return PSISPEC_ERR_INVALID_ARG;
  if (K > 64 || int64_t(B) * (K + 1) > kMaxRows || V > kMaxV ||
      int64_t(B) * (K + 1) * nslices_for(V) > kMaxGrid)
    return PSISPEC_ERR_UNSUPPORTED;
  psispec_status s = check_ws(workspace, workspace_bytes, psispec_workspace_size(PSISPEC_OP_VERIFY_LINEAR, B, K, V));
  if (s != PSISPEC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const RowStat* ds = static_cast<const RowStat*>(draft_row_stats);
  if (dtype == PSISPEC_BF16)
    return verify_linear_impl(static_cast<const __nv_bfloat16*>(target_logits),
                              static_cast<const __nv_bfloat16*>(draft_logits), B, K, V, draft_tokens, ds, u_accept,
                              u_resid, temperature, top_p, top_k, out_tokens, out_accept_len, out_p, out_q, workspace,
                              st);
  return verify_linear_impl(static_cast<const float*>(target_logits), static_cast<const float*>(draft_logits), B, K, V,
                            draft_tokens, ds, u_accept, u_resid, temperature, top_p, top_k, out_tokens,
                            out_accept_len, out_p, out_q, workspace, st);
}

psispec_status psispec_verify_linear(const void* target_logits, const void* draft_logits, int dtype, int32_t B,
                                     int32_t K, int32_t V, const int32_t* draft_tokens, const void* draft_row_stats,
                                     const float* u_accept, const float* u_resid, const float* temperature,
                                     const float* top_p, int32_t* out_tokens, int32_t* out_accept_len, float* out_p,
                                     float* out_q, void* workspace, size_t workspace_bytes, void* stream) {
  return psispec_verify_linear_k(target_logits, draft_logits, dtype, B, K, V, draft_tokens, draft_row_stats, u_accept,
                                 u_resid, temperature, top_p, nullptr, out_tokens, out_accept_len, out_p, out_q,
                                 workspace, workspace_bytes, stream);
}

psispec_status psispec_verify_tree_k(const void* target_logits, const void* draft_logits, int dtype, int32_t B,
                                     int32_t N, int32_t V, const int32_t* node_offsets, const int32_t* parent,
                                     const int32_t* tokens, const float* u_accept, const float* u_resid,
                                     const float* temperature, const float* top_p, const int32_t* top_k,
                                     int32_t max_depth, int32_t* out_path, int32_t* out_tokens,
                                     int32_t* out_accept_len, void* workspace, size_t workspace_bytes, void* stream) {
  if (!target_logits || !draft_logits || !node_offsets || !parent || !tokens || !u_accept || !u_resid ||
      !temperature || !top_p || !out_path || !out_tokens || !out_accept_len || bad_dtype(dtype))
    return PSISPEC_ERR_INVALID_ARG;
  if (B <= 0 || N < B || V <= 0 || max_depth < 1) return PSISPEC_ERR_INVALID_ARG;
  if (!aligned_to(target_logits, esize(dtype)) || !aligned_to(draft_logits, esize(dtype)))
    return PSISPEC_ERR_INVALID_ARG;
  if (max_depth > 64 || N > kMaxRows || V > kMaxV || int64_t(N) * nslices_for(V) > kMaxGrid)
    return PSISPEC_ERR_UNSUPPORTED;
  psispec_status s = check_ws(workspace, workspace_bytes, psispec_workspace_size(PSISPEC_OP_VERIFY_TREE, B, N, V));
  if (s != PSISPEC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PSISPEC_BF16)
    return verify_tree_impl(static_cast<const __nv_bfloat16*>(target_logits),
                            static_cast<const __nv_bfloat16*>(draft_logits), B, N, V, node_offsets, parent, tokens,
                            u_accept, u_resid, temperature, top_p, top_k, max_depth, out_path, out_tokens,
                            out_accept_len, workspace, st);
  return verify_tree_impl(static_cast<const float*>(target_logits), static_cast<const float*>(draft_logits), B, N, V,
                          node_offsets, parent, tokens, u_accept, u_resid, temperature, top_p, top_k, max_depth,
                          out_path, out_tokens, out_accept_len, workspace, st);
}

psispec_status psispec_verify_tree(const void* target_logits, const void* draft_logits, int dtype, int32_t B,
                                   int32_t N, int32_t V, const int32_t* node_offsets, const int32_t* parent,
                                   const int32_t* tokens, const float* u_accept, const float* u_resid,
                                   const float* temperature, const float* top_p, int32_t max_depth,
                                   int32_t* out_path, int32_t* out_tokens, int32_t* out_accept_len, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return psispec_verify_tree_k(target_logits, draft_logits, dtype, B, N, V, node_offsets, parent, tokens, u_accept,
                               u_resid, temperature, top_p, nullptr, max_depth, out_path, out_tokens, out_accept_len,
                               workspace, workspace_bytes, stream);
}

psispec_status psispec_row_stats_k(const void* logits, int dtype, int32_t B, int32_t K, int32_t V,
                                   const float* temperature, const float* top_p, const int32_t* top_k,
                                   void* out_row_stats, void* workspace, size_t workspace_bytes, void* stream) {
  if (!logits || !temperature || !top_p || !out_row_stats || bad_dtype(dtype)) return PSISPEC_ERR_INVALID_ARG;
  if (B <= 0 || K <= 0 || V <= 0) return PSISPEC_ERR_INVALID_ARG;
  if (!aligned_to(logits, esize(dtype)) || !aligned_to(out_row_stats, 16)) return PSISPEC_ERR_INVALID_ARG;
  const int64_t rows = int64_t(B) * K;
  if (rows > kMaxRows || V > kMaxV || rows * nslices_for(V) > kMaxGrid) return PSISPEC_ERR_UNSUPPORTED;
  psispec_status s = check_ws(workspace, workspace_bytes, psispec_workspace_size(PSISPEC_OP_ROW_STATS, B, K, V));
  if (s != PSISPEC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RowStat* rs = static_cast<RowStat*>(out_row_stats);
  if (dtype == PSISPEC_BF16)
    return row_stats_impl(static_cast<const __nv_bfloat16*>(logits), B, K, V, temperature, top_p, top_k, rs,
                          workspace, st);
  return row_stats_impl(static_cast<const float*>(logits), B, K, V, temperature, top_p, top_k, rs, workspace, st);
}

psispec_status psispec_row_stats(const void* logits, int dtype, int32_t B, int32_t K, int32_t V,
                                 const float* temperature, const float* top_p, void* out_row_stats,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return psispec_row_stats_k(logits, dtype, B, K, V, temperature, top_p, nullptr, out_row_stats, workspace,
                             workspace_bytes, stream);
}

psispec_status psispec_verify_linear_static(const void* target_logits, const void* draft_logits, int dtype,
                                            int32_t B, int32_t K, int32_t V, const int32_t* draft_tokens,
                                            const void* draft_row_stats, const float* u_accept,
                                            const float* u_resid, const float* temperature,
                                            const float* top_p, int32_t* out_tokens, int32_t* out_accept_len,
                                            float* out_p, float* out_q, void* stream) {
  if (B <= 0 || K <= 0 || V <= 0) return PSISPEC_ERR_INVALID_ARG;
  // the limits of psispec_verify_linear first, so that both calls report them alike
  if (K > 64 || int64_t(B) * (K + 1) > kMaxRows || V > kMaxV || int64_t(B) * (K + 1) * nslices_for(V) > kMaxGrid)
    return PSISPEC_ERR_UNSUPPORTED;
  const size_t need = psispec_workspace_size(PSISPEC_OP_VERIFY_LINEAR, B, K, V);
  if (need == 0) return PSISPEC_ERR_INVALID_ARG;
  if (need > static_cast<size_t>(PSISPEC_STATIC_WORKSPACE_BYTES)) return PSISPEC_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PSISPEC_ERR_CUDA;
  void* ws = g_static_workspace_ptr[dev].load(std::memory_order_acquire);
  if (ws == nullptr) {
    if (cudaGetSymbolAddress(&ws, g_static_workspace) != cudaSuccess || ws == nullptr) return PSISPEC_ERR_CUDA;
    g_static_workspace_ptr[dev].store(ws, std::memory_order_release);
  }
  return psispec_verify_linear(target_logits, draft_logits, dtype, B, K, V, draft_tokens, draft_row_stats, u_accept,
                               u_resid, temperature, top_p, out_tokens, out_accept_len, out_p, out_q, ws,
                               static_cast<size_t>(PSISPEC_STATIC_WORKSPACE_BYTES), stream);
}

psispec_status psispec_build_tree(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                  const float* temperature, const float* top_p, const int32_t* top_k, int32_t cand_k,
                                  int32_t n_prefixes, int32_t* out_parent, int32_t* out_tokens, int32_t* out_depth,
                                  double* out_score, int32_t* out_nodes, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!draft_logits || !temperature || !top_p || !out_parent || !out_tokens || !out_depth || !out_nodes ||
      bad_dtype(dtype))
    return PSISPEC_ERR_INVALID_ARG;
  if (B <= 0 || K <= 0 || V <= 0 || cand_k <= 0 || n_prefixes <= 0) return PSISPEC_ERR_INVALID_ARG;
  if (!aligned_to(draft_logits, esize(dtype))) return PSISPEC_ERR_INVALID_ARG;
  const int64_t rows = int64_t(B) * K;
  if (K > kTrieMaxK || cand_k > kTrieMaxCand || n_prefixes > kTrieMaxPrefixes || rows > kMaxRows || V > kMaxV ||
      rows * nslices_for(V) > kMaxGrid)
    return PSISPEC_ERR_UNSUPPORTED;
  psispec_status s = check_ws(workspace, workspace_bytes, psispec_workspace_size(PSISPEC_OP_BUILD_TREE, B, K, V));
  if (s != PSISPEC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PSISPEC_BF16)
    return build_tree_impl(static_cast<const __nv_bfloat16*>(draft_logits), B, K, V, temperature, top_p, top_k, cand_k,
                           n_prefixes, out_parent, out_tokens, out_depth, out_score, out_nodes, workspace, st);
  return build_tree_impl(static_cast<const float*>(draft_logits), B, K, V, temperature, top_p, top_k, cand_k,
                         n_prefixes, out_parent, out_tokens, out_depth, out_score, out_nodes, workspace, st);
}

psispec_status psispec_verify_tree_det(const void* target_logits, int dtype, int32_t B, int32_t N, int32_t V,
                                       const int32_t* node_offsets, const int32_t* parent, const int32_t* tokens,
                                       const float* u_accept, const float* u_resid, const float* temperature,
                                       const float* top_p, const int32_t* top_k, int32_t max_depth, int32_t* out_path,
                                       int32_t* out_tokens, int32_t* out_accept_len, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!target_logits || !node_offsets || !parent || !tokens || !u_accept || !u_resid || !temperature || !top_p ||
      !out_path || !out_tokens || !out_accept_len || bad_dtype(dtype))
    return PSISPEC_ERR_INVALID_ARG;
  if (B <= 0 || N < B || V <= 0 || max_depth < 1) return PSISPEC_ERR_INVALID_ARG;
  if (!aligned_to(target_logits, esize(dtype))) return PSISPEC_ERR_INVALID_ARG;
  if (max_depth > 64 || N > kMaxRows || V > kMaxV || int64_t(N) * nslices_for(V) > kMaxGrid)
    return PSISPEC_ERR_UNSUPPORTED;
  psispec_status s = check_ws(workspace, workspace_bytes, psispec_workspace_size(PSISPEC_OP_VERIFY_TREE, B, N, V));
  if (s != PSISPEC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PSISPEC_BF16)
    return verify_tree_det_impl(static_cast<const __nv_bfloat16*>(target_logits), B, N, V, node_offsets, parent,
                                tokens, u_accept, u_resid, temperature, top_p, top_k, max_depth, out_path, out_tokens,
                                out_accept_len, workspace, st);
  return verify_tree_det_impl(static_cast<const float*>(target_logits), B, N, V, node_offsets, parent, tokens, u_accept,
                              u_resid, temperature, top_p, top_k, max_depth, out_path, out_tokens, out_accept_len,
                              workspace, st);
}

}  // extern "C"
