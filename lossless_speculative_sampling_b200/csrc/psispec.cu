// psispec.cu -- C ABI of libpsispec.so: argument checks, workspace layout and launches.
// The operations are specified in include/psispec.h.
#include "psispec.h"

#include "common.cuh"
#include "linear.cuh"
#include "sample.cuh"
#include "stats.cuh"
#include "tree.cuh"

namespace psi {
namespace {

constexpr int64_t kMaxRows = int64_t(1) << 26;
constexpr int64_t kMaxV = int64_t(1) << 24;
constexpr int64_t kMaxGrid = 0x7fffffff;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int nslices_for(int64_t V) { return static_cast<int>((V + kSliceElems - 1) / kSliceElems); }

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
StatsWs carve_stats(Carver& c, int64_t rows, int ns) { return StatsWs{c.take<Partial>(rows * ns), c.take<RowStat>(rows)}; }

struct SampleWs {
  StatsWs st;
  Job* jobs;
  double2* cdf;
};
SampleWs carve_sample(Carver& c, int64_t rows, int ns) {
  SampleWs w;
  w.st = carve_stats(c, rows, ns);
  w.jobs = c.take<Job>(rows);
  w.cdf = c.take<double2>(rows * ns);
  return w;
}

struct LinearWs {
  StatsWs t, d;
  Job* jobs;
  double2* cdf;
};
LinearWs carve_linear(Carver& c, int64_t B, int64_t K, int ns) {
  LinearWs w;
  w.t = carve_stats(c, B * (K + 1), ns);
  w.d = carve_stats(c, B * K, ns);
  w.jobs = c.take<Job>(B);
  w.cdf = c.take<double2>(B * ns);
  return w;
}

struct TreeWs {
  StatsWs t, d;
  int32_t* row_req;
};
TreeWs carve_tree(Carver& c, int64_t N, int ns) {
  TreeWs w;
  w.t = carve_stats(c, N, ns);
  w.d = carve_stats(c, N, ns);
  w.row_req = c.take<int32_t>(N);
  return w;
}

psispec_status check_ws(const void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PSISPEC_ERR_WORKSPACE;
  return PSISPEC_OK;
}

inline bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline psispec_status launched() { return cudaGetLastError() == cudaSuccess ? PSISPEC_OK : PSISPEC_ERR_CUDA; }

// Request index of every node, from node_offsets (tree rows have no fixed count per request).
__global__ void node_request_kernel(const int32_t* __restrict__ offs, int B, int N, int32_t* __restrict__ row_req) {
  const int b = blockIdx.x;
  if (b >= B) return;
  const int lo = max(0, min(N, offs[b])), hi = max(lo, min(N, offs[b + 1]));
  for (int n = lo + threadIdx.x; n < hi; n += blockDim.x) row_req[n] = b;
}

// Row statistics of a [rows, V] tensor (and, for draft sampling, the draw jobs).
template <typename T>
psispec_status launch_stats(const T* base, int64_t rows, int rows_per_req, const int32_t* row_req, int V, int ns,
                            const float* temperature, const float* top_p, StatsWs ws, RowStat* stats_out,
                            const float* u, Job* jobs, int32_t* out_tokens, float* out_q, cudaStream_t st) {
  row_partial_kernel<T><<<static_cast<unsigned>(rows * ns), kThreads, 0, st>>>(base, rows_per_req, row_req, V, ns,
                                                                              temperature, ws.parts);
  psispec_status s = launched();
  if (s != PSISPEC_OK) return s;
  row_finalize_kernel<T><<<static_cast<unsigned>(rows), kThreads, 0, st>>>(
      base, rows_per_req, row_req, V, ns, temperature, top_p, ws.parts, stats_out, u, jobs, out_tokens, out_q);
  return launched();
}

template <typename T>
psispec_status sample_draft_impl(const T* draft, int B, int K, int V, const float* temperature, const float* top_p,
                                 const float* u, int32_t* out_tokens, float* out_q, RowStat* out_stats, void* ws,
                                 cudaStream_t st) {
  const int64_t rows = int64_t(B) * K;
  const int ns = nslices_for(V);
  Carver c(ws);
  SampleWs w = carve_sample(c, rows, ns);
  RowStat* stats = out_stats ? out_stats : w.st.stats;
  psispec_status s = launch_stats<T>(draft, rows, K, nullptr, V, ns, temperature, top_p, w.st, stats, u, w.jobs,
                                     out_tokens, out_q, st);
  if (s != PSISPEC_OK) return s;
  cdf_partial_kernel<T><<<static_cast<unsigned>(rows * ns), kThreads, 0, st>>>(draft, draft, stats, stats, w.jobs, V,
                                                                              ns, w.cdf);
  if ((s = launched()) != PSISPEC_OK) return s;
  cdf_pick_kernel<T><<<static_cast<unsigned>(rows), kThreads, 0, st>>>(draft, draft, stats, stats, w.jobs, V, ns,
                                                                       w.st.parts, w.cdf, out_tokens, out_q);
  return launched();
}

template <typename T>
psispec_status verify_linear_impl(const T* tgt, const T* drf, int B, int K, int V, const int32_t* tokens,
                                  const RowStat* draft_stats, const float* u_acc, const float* u_res,
                                  const float* temperature, const float* top_p, int32_t* out_tokens,
                                  int32_t* out_len, float* out_p, float* out_q, void* ws, cudaStream_t st) {
  const int ns = nslices_for(V);
  Carver c(ws);
  LinearWs w = carve_linear(c, B, K, ns);
  psispec_status s = launch_stats<T>(tgt, int64_t(B) * (K + 1), K + 1, nullptr, V, ns, temperature, top_p, w.t,
                                     w.t.stats, nullptr, nullptr, nullptr, nullptr, st);
  if (s != PSISPEC_OK) return s;
  const RowStat* ds = draft_stats;
  if (ds == nullptr) {
    s = launch_stats<T>(drf, int64_t(B) * K, K, nullptr, V, ns, temperature, top_p, w.d, w.d.stats, nullptr, nullptr,
                        nullptr, nullptr, st);
    if (s != PSISPEC_OK) return s;
    ds = w.d.stats;
  }
  constexpr int kWarps = 8;
  linear_decide_kernel<T><<<(B + kWarps - 1) / kWarps, 32 * kWarps, 0, st>>>(
      tgt, drf, B, K, V, tokens, w.t.stats, ds, u_acc, u_res, out_tokens, out_len, out_p, out_q, w.jobs);
  if ((s = launched()) != PSISPEC_OK) return s;
  cdf_partial_kernel<T><<<static_cast<unsigned>(int64_t(B) * ns), kThreads, 0, st>>>(tgt, drf, w.t.stats, ds, w.jobs,
                                                                                     V, ns, w.cdf);
  if ((s = launched()) != PSISPEC_OK) return s;
  cdf_pick_kernel<T><<<B, kThreads, 0, st>>>(tgt, drf, w.t.stats, ds, w.jobs, V, ns, w.t.parts, w.cdf, out_tokens,
                                              nullptr);
  return launched();
}

template <typename T>
psispec_status verify_tree_impl(const T* tgt, const T* drf, int B, int N, int V, const int32_t* offs,
                                const int32_t* parent, const int32_t* tokens, const float* u_acc, const float* u_res,
                                const float* temperature, const float* top_p, int max_depth, int32_t* out_path,
                                int32_t* out_tokens, int32_t* out_len, void* ws, cudaStream_t st) {
  const int ns = nslices_for(V);
  Carver c(ws);
  TreeWs w = carve_tree(c, N, ns);
  node_request_kernel<<<B, 128, 0, st>>>(offs, B, N, w.row_req);
  psispec_status s = launched();
  if (s != PSISPEC_OK) return s;
  s = launch_stats<T>(tgt, N, 1, w.row_req, V, ns, temperature, top_p, w.t, w.t.stats, nullptr, nullptr, nullptr,
                      nullptr, st);
  if (s != PSISPEC_OK) return s;
  s = launch_stats<T>(drf, N, 1, w.row_req, V, ns, temperature, top_p, w.d, w.d.stats, nullptr, nullptr, nullptr,
                      nullptr, st);
  if (s != PSISPEC_OK) return s;
  tree_walk_kernel<T><<<B, kTreeThreads, 0, st>>>(tgt, drf, V, offs, parent, tokens, w.t.stats, w.d.stats, u_acc,
                                                  u_res, max_depth, out_path, out_tokens, out_len);
  return launched();
}

bool bad_dtype(int dtype) { return dtype != PSISPEC_F32 && dtype != PSISPEC_BF16; }
size_t esize(int dtype) { return dtype == PSISPEC_BF16 ? 2 : 4; }

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
  const int ns = nslices_for(c);
  Carver m(nullptr);
  switch (op) {
    case PSISPEC_OP_SAMPLE_DRAFT: carve_sample(m, a * b, ns); break;
    case PSISPEC_OP_VERIFY_LINEAR: carve_linear(m, a, b, ns); break;
    case PSISPEC_OP_VERIFY_TREE: carve_tree(m, b, ns); break;
    default: return 0;
  }
  return m.used;
}

psispec_status psispec_sample_draft(const void* draft_logits, int dtype, int32_t B, int32_t K, int32_t V,
                                    const float* temperature, const float* top_p, const float* u,
                                    int32_t* out_tokens, float* out_q, void* out_row_stats, void* workspace,
                                    size_t workspace_bytes, void* stream) {
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
    return sample_draft_impl(static_cast<const __nv_bfloat16*>(draft_logits), B, K, V, temperature, top_p, u,
                             out_tokens, out_q, rs, workspace, st);
  return sample_draft_impl(static_cast<const float*>(draft_logits), B, K, V, temperature, top_p, u, out_tokens, out_q,
                           rs, workspace, st);
}

psispec_status psispec_verify_linear(const void* target_logits, const void* draft_logits, int dtype, int32_t B,
                                     int32_t K, int32_t V, const int32_t* draft_tokens, const void* draft_row_stats,
                                     const float* u_accept, const float* u_resid, const float* temperature,
                                     const float* top_p, int32_t* out_tokens, int32_t* out_accept_len, float* out_p,
                                     float* out_q, void* workspace, size_t workspace_bytes, void* stream) {
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
                              u_resid, temperature, top_p, out_tokens, out_accept_len, out_p, out_q, workspace, st);
  return verify_linear_impl(static_cast<const float*>(target_logits), static_cast<const float*>(draft_logits), B, K, V,
                            draft_tokens, ds, u_accept, u_resid, temperature, top_p, out_tokens, out_accept_len, out_p,
                            out_q, workspace, st);
}

psispec_status psispec_verify_tree(const void* target_logits, const void* draft_logits, int dtype, int32_t B,
                                   int32_t N, int32_t V, const int32_t* node_offsets, const int32_t* parent,
                                   const int32_t* tokens, const float* u_accept, const float* u_resid,
                                   const float* temperature, const float* top_p, int32_t max_depth,
                                   int32_t* out_path, int32_t* out_tokens, int32_t* out_accept_len, void* workspace,
                                   size_t workspace_bytes, void* stream) {
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
                            u_accept, u_resid, temperature, top_p, max_depth, out_path, out_tokens, out_accept_len,
                            workspace, st);
  return verify_tree_impl(static_cast<const float*>(target_logits), static_cast<const float*>(draft_logits), B, N, V,
                          node_offsets, parent, tokens, u_accept, u_resid, temperature, top_p, max_depth, out_path,
                          out_tokens, out_accept_len, workspace, st);
}

}  // extern "C"
