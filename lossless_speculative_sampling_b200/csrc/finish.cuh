// finish.cuh -- per-row and per-request completion of draft sampling and linear verification.
//
// The streaming pass (stream_partials_kernel) reads every logits row once and leaves one
// partial per kChunkElems-element chunk. The kernels here finish from those partials:
//   sample_finish_kernel   one warp per draft row: row statistics, then the inverse-CDF draw
//                          inside the one chunk that holds u * Z (chunk partials are the
//                          prefix totals);
//   sample_topp_kernel     one CTA per draft row with a top-p cut (returns at once for the
//                          others): threshold by radix select, then a draw over the row;
//   verify_finish_kernel   one CTA per request: statistics of its verifier (and draft) rows,
//                          then, for requests without top-p, the accept tests, the first
//                          rejection and the draw job;
//   verify_topp_kernel     one CTA per row of a top-p request: threshold; the CTA that
//                          completes the request decides it;
//   draw_jobs_kernel       one warp per (draw job, chunk): chunk totals of the residual (or
//                          kept) weights; the warp that completes a job picks the chunk that
//                          holds u * Z and walks it.
// Cross-warp handoffs use arrival counters (the last arrival continues); nothing waits.
#pragma once

#include "common.cuh"
#include "linear.cuh"
#include "sample.cuh"
#include "stats.cuh"

namespace psi {

// Arrival of a whole CTA (thread 0 arrives after a barrier); true in every thread of the CTA
// whose arrival makes the counter `count`.
__device__ __forceinline__ bool block_arrive_last(int* counter, int count, int* sh_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(counter, 1);
    *sh_flag = prev == count - 1;
    if (*sh_flag) __threadfence();
  }
  __syncthreads();
  return *sh_flag != 0;
}

// Arrival of one warp at `counter`; true (in every lane) for the warp whose arrival makes it
// `count`. Global writes made by lane 0 before the call are visible to that last warp.
__device__ __forceinline__ bool warp_arrive_last(int* counter, int count) {
  int last = 0;
  if ((threadIdx.x & 31) == 0) {
    __threadfence();
    last = atomicAdd(counter, 1) == count - 1;
    if (last) __threadfence();
  }
  return __shfl_sync(0xffffffffu, last, 0) != 0;
}

// Warp-level: locate the chunk holding u * Z given every lane's totals of its contiguous run
// of chunks [i0, i0 + q) in registers (q <= kCache). Returns the chunk to every lane (or -1
// when every total is zero), the weight before it in *base and u * Z in *target.
__device__ __forceinline__ int warp_pick_cached(const double (&t)[kCache], int q, int i0, int nchunks, float u,
                                                double* base, double* target) {
  const int lane = threadIdx.x & 31;
  double mine = 0.0;
#pragma unroll
  for (int k = 0; k < kCache; ++k) mine += t[k];
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  const double tg = static_cast<double>(u) * __shfl_sync(0xffffffffu, incl, 31);
  int sel = -1, last = -1;
  double b = 0.0, C = excl;
  bool open = excl <= tg && tg < incl;  // this lane's run holds u * Z
#pragma unroll
  for (int k = 0; k < kCache; ++k) {
    if (k < q && i0 + k < nchunks && t[k] > 0.0) {
      last = i0 + k;
      if (open) {  // the run's last positive chunk unless an earlier one already holds u * Z
        sel = i0 + k;
        b = C;
        open = !(C + t[k] > tg);
      }
    }
    C += t[k];
  }
  const unsigned who = __ballot_sync(0xffffffffu, sel >= 0);
  int chunk;
  if (who) {
    const int src = __ffs(who) - 1;
    chunk = __shfl_sync(0xffffffffu, sel, src);
    b = __shfl_sync(0xffffffffu, b, src);
  } else {  // rounding put u * Z past every chunk: the last chunk with positive weight
    chunk = __reduce_max_sync(0xffffffffu, last);
    const int owner = __reduce_max_sync(0xffffffffu, (chunk >= 0 && last == chunk) ? lane : -1);
    double bb = excl;
#pragma unroll
    for (int k = 0; k < kCache; ++k)
      if (i0 + k < chunk) bb += t[k];
    b = __shfl_sync(0xffffffffu, bb, owner < 0 ? 0 : owner);
  }
  *base = b;
  *target = tg;
  return chunk;
}

// Per-chunk totals (.x, or .y with use_y) written by an earlier kernel: same contract as
// warp_pick_cached; rows of more than 32 * kCache chunks are walked in two passes.
__device__ __forceinline__ int warp_pick_totals(const double2* tot, int nchunks, bool use_y, float u, double* base,
                                                double* target) {
  const int lane = threadIdx.x & 31;
  const int q = (nchunks + 31) / 32;
  const int i0 = min(nchunks, lane * q);
  if (q <= kCache) {
    double t[kCache];
#pragma unroll
    for (int k = 0; k < kCache; ++k)
      t[k] = (k < q && i0 + k < nchunks) ? (use_y ? __ldcg(&tot[i0 + k].y) : __ldcg(&tot[i0 + k].x)) : 0.0;
    return warp_pick_cached(t, q, i0, nchunks, u, base, target);
  }
  // long rows: totals in two passes (run totals, then the owning lane's walk)
  auto total = [&](int i) -> double { return use_y ? __ldcg(&tot[i].y) : __ldcg(&tot[i].x); };
  const int c1 = min(nchunks, i0 + q);
  double mine = 0.0;
  for (int i = i0; i < c1; ++i) mine += total(i);
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  const double tg = static_cast<double>(u) * __shfl_sync(0xffffffffu, incl, 31);
  int sel = -1, last = -1;
  double b = 0.0;
  if (excl <= tg && tg < incl) {
    double C = excl;
    for (int i = i0; i < c1; ++i) {
      const double w = total(i);
      if (w > 0.0) { sel = i; b = C; }
      if (C + w > tg && w > 0.0) break;
      C += w;
    }
  }
  for (int i = i0; i < c1; ++i)
    if (total(i) > 0.0) last = i;
  const unsigned who = __ballot_sync(0xffffffffu, sel >= 0);
  if (who) {
    const int src = __ffs(who) - 1;
    sel = __shfl_sync(0xffffffffu, sel, src);
    b = __shfl_sync(0xffffffffu, b, src);
  } else {
    sel = __reduce_max_sync(0xffffffffu, last);
    double before = 0.0;
    for (int i = lane; i < sel; i += 32) before += total(i);
    b = warp_sum(before);
  }
  *base = b;
  *target = tg;
  return sel;
}

// The chunk of a row's own (untruncated) distribution that holds u * Z, from the row's chunk
// partials (same contract as warp_pick_cached).
__device__ __forceinline__ int warp_pick_chunk(const Partial* pp, int nchunks, const RowStat& st, float u,
                                               double* base, double* target) {
  const int lane = threadIdx.x & 31;
  const int q = (nchunks + 31) / 32;
  const int i0 = min(nchunks, lane * q);
  auto total = [&](int i) -> double {
    const float m = __ldcg(&pp[i].m);
    return m > -INFINITY ? __ldcg(&pp[i].s) * static_cast<double>(ex2((m - st.m) * st.c)) : 0.0;
  };
  if (q <= kCache) {
    double t[kCache];
#pragma unroll
    for (int k = 0; k < kCache; ++k) t[k] = (k < q && i0 + k < nchunks) ? total(i0 + k) : 0.0;
    return warp_pick_cached(t, q, i0, nchunks, u, base, target);
  }
  const int c1 = min(nchunks, i0 + q);
  double mine = 0.0;
  int last = -1;
  for (int i = i0; i < c1; ++i) {
    const double w = total(i);
    mine += w;
    if (w > 0.0) last = i;
  }
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  const double tg = static_cast<double>(u) * __shfl_sync(0xffffffffu, incl, 31);
  int sel = -1;
  double b = 0.0;
  if (excl <= tg && tg < incl) {
    double C = excl;
    for (int i = i0; i < c1; ++i) {
      const double w = total(i);
      if (w > 0.0) { sel = i; b = C; }
      if (C + w > tg && w > 0.0) break;
      C += w;
    }
  }
  const unsigned who = __ballot_sync(0xffffffffu, sel >= 0);
  if (who) {
    const int src = __ffs(who) - 1;
    sel = __shfl_sync(0xffffffffu, sel, src);
    b = __shfl_sync(0xffffffffu, b, src);
  } else {
    sel = __reduce_max_sync(0xffffffffu, last);
    double before = 0.0;
    for (int i = lane; i < sel; i += 32) before += total(i);
    b = warp_sum(before);
  }
  *base = b;
  *target = tg;
  return sel;
}

// One warp per draft row: statistics, then the draw inside the chunk that holds u * Z. Rows
// with a top-p cut are left to sample_topp_kernel.
template <typename T>
__global__ void __launch_bounds__(kThreads) sample_finish_kernel(const T* __restrict__ draft, int K, int V, int rows,
                                                                 const float* __restrict__ temperature,
                                                                 const float* __restrict__ top_p,
                                                                 const float* __restrict__ u,
                                                                 const Partial* __restrict__ parts,
                                                                 RowStat* __restrict__ stats,
                                                                 int32_t* __restrict__ out_tokens,
                                                                 float* __restrict__ out_q) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int b = row / K;
  const int nch = nchunks_for(V);
  const T* rp = draft + static_cast<size_t>(row) * V;
  const Partial* pp = parts + static_cast<size_t>(row) * nch;
  const float tp = top_p[b];
  const bool no_cut = !(tp < 1.0f);
  RowPick rp_ = warp_finalize_pick(pp, nch, temperature[b], u[row], no_cut);
  const RowStat st = rp_.st;
  if (lane == 0) stats[row] = st;
  if (needs_topp(st, tp)) return;
  if (st.status != 0 || st.c == 0.0f) {
    if (lane == 0) {
      out_tokens[row] = st.status != 0 ? -1 : st.amax;
      if (out_q) out_q[row] = st.status != 0 ? -1.0f : 1.0f;
    }
    return;
  }
  JobRows<T, false> J;
  J.init(rp, st, nullptr, st);
  int ch = rp_.chunk;
  double base = rp_.base, target = rp_.target;
  if ((nch + 31) / 32 > kCache) ch = warp_pick_chunk(pp, nch, st, u[row], &base, &target);
  const int y = ch < 0 ? -1 : warp_draw_range<T, false, 8>(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems), base, target);
  if (lane == 0) {
    out_tokens[row] = y;
    if (out_q) out_q[row] = y >= 0 ? kept_weight(st, load_elem(rp + y)) / st.s_kept : -1.0f;
  }
}

// Draft rows with a top-p cut: one CTA per row finds the threshold and draws over the row.
template <typename T>
__global__ void __launch_bounds__(kThreads) sample_topp_kernel(const T* __restrict__ draft, int K, int V,
                                                               const float* __restrict__ top_p,
                                                               const float* __restrict__ u, RowStat* __restrict__ stats,
                                                               int32_t* __restrict__ out_tokens,
                                                               float* __restrict__ out_q) {
  __shared__ ToppSmem tsm;
  __shared__ DrawSmem dsm;
  const int row = blockIdx.x;
  const float tp = top_p[row / K];
  RowStat st = stats[row];
  if (!needs_topp(st, tp)) return;
  const T* rp = draft + static_cast<size_t>(row) * V;
  block_topp_select<T>(rp, V, tp, st, tsm);
  if (threadIdx.x == 0) stats[row] = st;
  JobRows<T, false> J;
  J.init(rp, st, nullptr, st);
  const int y = block_draw_range(J, 0, V, 0.0, -1.0, u[row], dsm);
  if (threadIdx.x == 0) {
    out_tokens[row] = y;
    if (out_q) out_q[row] = y >= 0 ? kept_weight(st, load_elem(rp + y)) / st.s_kept : -1.0f;
  }
}

// Arguments shared by the verification kernels.
struct VerifyArgs {
  int B, K, V, stream_draft;
  const float* temperature;
  const float* top_p;
  const int32_t* tokens;
  const RowStat* dstats_in;
  const float* u_acc;
  const float* u_res;
  Partial* parts_t;
  Partial* parts_d;
  RowStat* stats_t;
  RowStat* stats_d;
  int* cnt;  // one arrival counter per request (top-p requests)
  int32_t* out_tokens;
  int32_t* out_len;
  float* out_p;
  float* out_q;
  Job* jobs;
};

// Whether request b's rows carry a top-p cut (then verify_topp_kernel finishes it).
__device__ __forceinline__ bool request_topp(const VerifyArgs& a, int b) {
  return a.top_p[b] < 1.0f && temp_scale(a.temperature[b]) != 0.0f;
}

// One CTA per request: statistics of its rows (warps in parallel), then the decision.
template <typename T>
__global__ void __launch_bounds__(1024) verify_finish_kernel(const T* __restrict__ tgt, const T* __restrict__ drf,
                                                                 VerifyArgs a) {
  const int b = blockIdx.x;
  const int K = a.K, nch = nchunks_for(a.V);
  const int nrows = (K + 1) + (a.stream_draft ? K : 0);
  const float Tv = a.temperature[b];
  for (int i = threadIdx.x >> 5; i < nrows; i += blockDim.x >> 5) {
    const bool is_draft = i > K;
    const int row = is_draft ? b * K + (i - K - 1) : b * (K + 1) + i;
    const Partial* pp = (is_draft ? a.parts_d : a.parts_t) + static_cast<size_t>(row) * nch;
    const RowStat st = warp_finalize_pick(pp, nch, Tv, 0.0f, false).st;
    if ((threadIdx.x & 31) == 0) (is_draft ? a.stats_d : a.stats_t)[row] = st;
  }
  if (request_topp(a, b)) return;
  __syncthreads();
  __threadfence_block();
  if (threadIdx.x < 32)
    warp_decide_request<T>(b, tgt, drf, K, a.V, a.tokens, a.stats_t, a.stream_draft ? a.stats_d : a.dstats_in, a.u_acc,
                           a.u_res, a.out_tokens, a.out_len, a.out_p, a.out_q, a.jobs);
}

// One CTA per row of a top-p request: the threshold; the CTA that completes the request
// decides it.
template <typename T>
__global__ void __launch_bounds__(kThreads) verify_topp_kernel(const T* __restrict__ tgt, const T* __restrict__ drf,
                                                               VerifyArgs a) {
  __shared__ ToppSmem tsm;
  __shared__ int sh_flag;
  const int K = a.K, V = a.V;
  const int rows_t = a.B * (K + 1);
  const bool is_draft = static_cast<int>(blockIdx.x) >= rows_t;
  const int row = is_draft ? static_cast<int>(blockIdx.x) - rows_t : static_cast<int>(blockIdx.x);
  const int b = is_draft ? row / K : row / (K + 1);
  if (!request_topp(a, b)) return;
  const float tp = a.top_p[b];
  RowStat* sp = (is_draft ? a.stats_d : a.stats_t) + row;
  RowStat st = *sp;
  if (needs_topp(st, tp)) {
    block_topp_select<T>((is_draft ? drf : tgt) + static_cast<size_t>(row) * V, V, tp, st, tsm);
    if (threadIdx.x == 0) *sp = st;
  }
  if (!block_arrive_last(&a.cnt[b], (K + 1) + (a.stream_draft ? K : 0), &sh_flag)) return;
  if (threadIdx.x < 32)
    warp_decide_request<T>(b, tgt, drf, K, V, a.tokens, a.stats_t, a.stream_draft ? a.stats_d : a.dstats_in, a.u_acc,
                           a.u_res, a.out_tokens, a.out_len, a.out_p, a.out_q, a.jobs);
}

// Draw jobs (a residual draw at the first rejection, or the bonus draw from a row with a
// top-p cut) need per-chunk totals of their weights: draw_totals_kernel spreads the
// (job, chunk) items over every SM with persistent warps (two exponentials per element pair
// make this pass compute-heavy, so it must not sit on a few SMs). draw_pick_kernel then
// uses one warp per job: it finds the chunk that holds u * Z (from those totals, or from the
// row's own partials for a bonus draw without a cut) and walks it.
template <typename T>
__global__ void __launch_bounds__(kThreads) draw_totals_kernel(const T* __restrict__ A, const T* __restrict__ Bt,
                                                               int V, int njobs, const RowStat* __restrict__ sa,
                                                               const RowStat* __restrict__ sb,
                                                               const Job* __restrict__ jobs,
                                                               double2* __restrict__ tot) {
  const int lane = threadIdx.x & 31;
  const int nch = nchunks_for(V);
  const int64_t items = static_cast<int64_t>(njobs) * nch;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); g < items; g += nwarps) {
    const int jid = static_cast<int>(g / nch), chunk = static_cast<int>(g - static_cast<int64_t>(jid) * nch);
    const Job jb = jobs[jid];
    if (jb.mode < kSample) continue;
    const RowStat st_a = sa[jb.row_a];
    if (jb.mode == kSample && st_a.tau == 0u) continue;  // totals are the row's partials
    const T* ra = A + static_cast<size_t>(jb.row_a) * V;
    const int c0 = chunk * kChunkElems, c1 = min(V, c0 + kChunkElems);
    int last;
    double2 t;
    if (jb.mode == kSample) {
      JobRows<T, false> J;
      J.init(ra, st_a, nullptr, st_a);
      t = warp_range_totals(J, c0, c1, &last);
    } else {
      JobRows<T, true> J;
      J.init(ra, st_a, Bt + static_cast<size_t>(jb.row_b) * V, sb[jb.row_b]);
      t = warp_range_totals(J, c0, c1, &last);
    }
    if (lane == 0) tot[g] = t;
  }
}

template <typename T>
__global__ void __launch_bounds__(32) draw_pick_kernel(const T* __restrict__ A, const T* __restrict__ Bt, int V,
                                                             int njobs, const RowStat* __restrict__ sa,
                                                             const RowStat* __restrict__ sb,
                                                             const Partial* __restrict__ parts_a,
                                                             const Job* __restrict__ jobs,
                                                             const double2* __restrict__ tot,
                                                             int32_t* __restrict__ out_tokens) {
  const int lane = threadIdx.x & 31;
  const int jid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // one warp per job
  if (jid >= njobs) return;
  const Job jb = jobs[jid];
  if (jb.mode < kSample) return;
  const int nch = nchunks_for(V);
  const RowStat st_a = sa[jb.row_a];
  const T* ra = A + static_cast<size_t>(jb.row_a) * V;
  const double2* jt = tot + static_cast<size_t>(jid) * nch;
  double base, target;
  int y;
  if (jb.mode == kSample) {
    JobRows<T, false> J;
    J.init(ra, st_a, nullptr, st_a);
    const int ch = st_a.tau == 0u ? warp_pick_chunk(parts_a + static_cast<size_t>(jb.row_a) * nch, nch, st_a, jb.u, &base, &target)
                                  : warp_pick_totals(jt, nch, false, jb.u, &base, &target);
    y = ch < 0 ? -1 : warp_draw_range<T, false, 8>(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems), base, target);
  } else {
    JobRows<T, true> J;
    J.init(ra, st_a, Bt + static_cast<size_t>(jb.row_b) * V, sb[jb.row_b]);
    double z = 0.0;
#pragma unroll 4
    for (int i = lane; i < nch; i += 32) z += __ldcg(&jt[i].x);
    J.use_p = !(warp_sum(z) > 0.0);  // zero residual: draw from p instead
    const int ch = warp_pick_totals(jt, nch, J.use_p, jb.u, &base, &target);
    y = ch < 0 ? -1 : warp_draw_range<T, true, 8>(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems), base, target);
  }
  if (lane == 0) out_tokens[jb.out_index] = y;
}

}  // namespace psi
