// finish.cuh -- per-row and per-request completion of draft sampling and linear verification.
//
// The streaming pass (stream_partials_kernel) reads every logits row once and leaves one
// partial per kChunkElems-element chunk. The kernels here finish from those partials:
//   warp_sample_row     one warp per draft row (no cut): row statistics and the chunk
//                       holding u * Z (chunk partials are the prefix totals), then the draw
//                       inside that chunk;
//   warp_verify_row     one warp per verifier (and streamed draft) row (no cut):
//                       statistics, then an arrival on the request's counter; the warp
//                       completing a request runs the accept tests, finds the first rejection
//                       and writes the draw job (both run inside the row kernels of topp.cuh);
//   draw_totals_*       (fallback of the cluster draw in draw.cuh) one warp per (draw job,
//                       chunk) item over every SM: group and chunk totals of the residual (or
//                       kept) weights;
//   draw_pick_kernel    (same fallback) one warp per draw job: the chunk, then the 256-element
//                       group holding u * Z, and the walk of that group.
// Cross-CTA handoffs use arrival counters (the last arrival continues); nothing waits.
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

// Residual draw of a job: the chunk holding u * Z of max(0, p - q) (.x totals), or of p (.y
// totals) when the residual is zero everywhere (*use_p tells which). Same contract as
// warp_pick_cached.
__device__ __forceinline__ int warp_pick_resid(const double2* tot, int nchunks, float u, double* base, double* target,
                                               bool* use_p) {
  const int lane = threadIdx.x & 31;
  const int q = (nchunks + 31) / 32;
  const int i0 = min(nchunks, lane * q);
  if (q <= kCache) {
    double tx[kCache], ty[kCache], z = 0.0;
#pragma unroll
    for (int k = 0; k < kCache; ++k) {
      const bool ok = k < q && i0 + k < nchunks;
      tx[k] = ok ? __ldcg(&tot[i0 + k].x) : 0.0;
      ty[k] = ok ? __ldcg(&tot[i0 + k].y) : 0.0;
      z += tx[k];
    }
    *use_p = !(warp_sum(z) > 0.0);
    if (*use_p) {
#pragma unroll
      for (int k = 0; k < kCache; ++k) tx[k] = ty[k];
    }
    return warp_pick_cached(tx, q, i0, nchunks, u, base, target);
  }
  double z = 0.0;
  for (int i = lane; i < nchunks; i += 32) z += __ldcg(&tot[i].x);
  *use_p = !(warp_sum(z) > 0.0);
  return warp_pick_totals(tot, nchunks, *use_p, u, base, target);
}

// Warp-level finish of one draft row without a cut: statistics from the chunk
// partials, the chunk holding u * Z (chunk partials are the prefix totals), and the draw
// inside that chunk.
template <typename T>
__device__ void warp_sample_row(const T* __restrict__ draft, int row, int K, int V,
                                const float* __restrict__ temperature, const float* __restrict__ u,
                                const Partial* __restrict__ parts, RowStat* __restrict__ stats,
                                int32_t* __restrict__ out_tokens, float* __restrict__ out_q) {
  const int lane = threadIdx.x & 31;
  const int b = row / K;
  const int nch = nchunks_for(V);
  const T* rp = draft + static_cast<size_t>(row) * V;
  const Partial* pp = parts + static_cast<size_t>(row) * nch;
  const float ur = u[row];
  RowPick r = warp_finalize_pick(pp, nch, temperature[b], ur, true);
  const RowStat st = r.st;
  int y = -1;
  float q = -1.0f;
  if (st.status == 0 && st.c == 0.0f) {
    y = st.amax;
    q = 1.0f;
  } else if (st.status == 0) {
    if ((nch + 31) / 32 > kCache) r.chunk = warp_pick_chunk(pp, nch, st, ur, &r.base, &r.target);
    JobRows<T, false> J;
    J.init(rp, st, nullptr, st);
    float ly = 0.0f;
    if (r.chunk >= 0)
      y = warp_draw_chunk(J, r.chunk * kChunkElems, min(V, (r.chunk + 1) * kChunkElems), r.base, r.target, &ly);
    if (y >= 0) q = kept_weight(st, ly) / st.s_kept;
  }
  if (lane == 0) {
    stats[row] = st;
    out_tokens[row] = y;
    if (out_q) out_q[row] = q;
  }
}

// Arguments shared by the verification kernels.
struct VerifyArgs {
  int B, K, V, stream_draft;
  const float* temperature;
  const float* top_p;
  const int32_t* top_k;  // per request, or null (off)
  const int32_t* tokens;
  const RowStat* dstats_in;
  const float* u_acc;
  const float* u_res;
  Partial* parts_t;
  Partial* parts_d;
  RowStat* stats_t;
  RowStat* stats_d;
  int* cnt;  // arrival counters, one per request
  int32_t* out_tokens;
  int32_t* out_len;
  float* out_p;
  float* out_q;
  Job* jobs;
};

// Warp-level finish of one row g (verifier rows, then streamed draft rows) of a request
// without a cut: statistics from the chunk partials, then the arrival on the request's
// counter; the warp completing the request runs its accept tests, finds the first rejection
// and writes the draw job.
template <typename T>
__device__ void warp_verify_row(const T* __restrict__ tgt, const T* __restrict__ drf, int g, const VerifyArgs& a) {
  const int K = a.K;
  const int rows_t = a.B * (K + 1);
  const int per_req = (K + 1) + (a.stream_draft ? K : 0);
  const int nch = nchunks_for(a.V);
  const bool is_draft = g >= rows_t;
  const int row = is_draft ? g - rows_t : g;
  const int b = is_draft ? row / K : row / (K + 1);
  const Partial* pp = (is_draft ? a.parts_d : a.parts_t) + static_cast<size_t>(row) * nch;
  const RowStat st = warp_finalize_pick(pp, nch, a.temperature[b], 0.0f, false).st;
  if ((threadIdx.x & 31) == 0) (is_draft ? a.stats_d : a.stats_t)[row] = st;
  if (warp_arrive_last(&a.cnt[b], per_req))
    warp_decide_request<T>(b, tgt, drf, K, a.V, a.tokens, a.stats_t, a.stream_draft ? a.stats_d : a.dstats_in,
                           a.u_acc, a.u_res, a.out_tokens, a.out_len, a.out_p, a.out_q, a.jobs);
}

// Two-launch draw of the jobs (the residual draw at a first rejection, or the bonus draw after
// a fully accepted block), used where the one-launch cluster draw (draw.cuh) cannot run: no
// cluster of the needed size can be scheduled, or V is beyond its per-warp step buffer. The
// totals pass spreads (job, chunk) items over every SM: each warp reduces one chunk of the
// job's weights (.x the residual max(0, p - q) or the kept distribution, .y p) to its eight
// 256-element group totals and the chunk total. The pick pass gives each job a warp that
// locates the chunk holding u * Z, then the group inside it, and walks that group. A bonus
// draw without a top-p cut needs no totals: its chunk comes from the row's own partials and
// is walked whole.

// Whether a job's draw needs the totals pass.
__device__ __forceinline__ bool job_needs_totals(int32_t mode, uint32_t tau_a) {
  return mode == kResidual || (mode == kSample && tau_a != 0u);
}

// Per-lane group sums of one chunk held in shared memory (sa: row a, sb: row b; n elements).
template <typename T, bool RESID>
__device__ __forceinline__ void smem_chunk_sums(const JobRows<T, RESID>& J, const T* sa, const T* sb, int n,
                                                double (&sx)[kChunkGroups], double (&sy)[kChunkGroups]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int g = 0; g < kChunkGroups; ++g) {
    const int e = g * kGroup + lane * 8;
    Raw8<T, RESID> x;
    if (e + 8 <= n) {
      x.a.w[0] = *reinterpret_cast<const uint4*>(sa + e);
      if constexpr (sizeof(T) == 4) x.a.w[1] = *reinterpret_cast<const uint4*>(sa + e + 4);
      if constexpr (RESID) {
        x.b[0].w[0] = *reinterpret_cast<const uint4*>(sb + e);
        if constexpr (sizeof(T) == 4) x.b[0].w[1] = *reinterpret_cast<const uint4*>(sb + e + 4);
      }
    } else {
      float fa[8], fb[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        fa[k] = e + k < n ? load_elem_any(sa + e + k) : -INFINITY;
        fb[k] = (RESID && e + k < n) ? load_elem_any(sb + e + k) : -INFINITY;
      }
      x.a.pack(fa);
      if constexpr (RESID) x.b[0].pack(fb);
    }
    const double2 t = lane_group_sums(J, x);
    sx[g] = t.x;
    sy[g] = t.y;
  }
}

// Totals pass through a per-warp ring of bulk copies (rows 16-byte aligned, row bytes a
// multiple of 16): lane 0 keeps the next item's copies in flight, with the job record staged
// in shared memory for the warp, while the warp reduces the current item.
constexpr int kDrawRing = 2;
constexpr int kDrawWarps = 4;  // warps per CTA of the bulk-copy totals pass
template <typename T>
constexpr int kDrawStageBytes = 2 * kChunkElems * static_cast<int>(sizeof(T));  // rows a and b

template <typename T>
__global__ void __launch_bounds__(kDrawWarps * 32) draw_totals_tma_kernel(const T* __restrict__ A, const T* __restrict__ Bt,
                                                                  int V, int njobs, const Job* __restrict__ jobs,
                                                                  double2* __restrict__ tot_c,
                                                                  double2* __restrict__ tot_g) {
  extern __shared__ __align__(128) unsigned char dring_smem[];
  __shared__ uint64_t bars[kDrawWarps][kDrawRing];
  __shared__ Job sjob[kDrawWarps][kDrawRing];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char* ring = dring_smem + warp * kDrawRing * kDrawStageBytes<T>;
  uint64_t* bar = bars[warp];
  const int nch = nchunks_for(V);
  const int64_t items = static_cast<int64_t>(njobs) * nch;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kDrawWarps;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * kDrawWarps + warp;
  if (g0 >= items) return;
  if (lane == 0) {
    for (int s = 0; s < kDrawRing; ++s) mbar_init(&bar[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const int djob = static_cast<int>(nwarps / nch), dchunk = static_cast<int>(nwarps - static_cast<int64_t>(djob) * nch);
  int ijob = static_cast<int>(g0 / nch), ichunk = static_cast<int>(g0 - static_cast<int64_t>(ijob) * nch);
  int64_t gi = g0;
  // lane 0: stage the job record of this warp's i-th item and start its copies
  auto issue = [&](int i) {
    if (gi < items) {
      const int st = i % kDrawRing;
      const Job jb = load_job_cg(jobs + ijob);
      sjob[warp][st] = jb;
      if (job_needs_totals(jb.mode, jb.sa.tau)) {
        const int c0 = ichunk * kChunkElems, n = min(V - c0, kChunkElems);
        const uint32_t bytes = static_cast<uint32_t>(n) * sizeof(T);
        const bool resid = jb.mode == kResidual;
        unsigned char* dst = ring + st * kDrawStageBytes<T>;
        mbar_expect_tx(&bar[st], resid ? 2 * bytes : bytes);
        bulk_g2s(dst, A + static_cast<size_t>(jb.row_a) * V + c0, bytes, &bar[st]);
        if (resid) bulk_g2s(dst + kChunkElems * sizeof(T), Bt + static_cast<size_t>(jb.row_b) * V + c0, bytes, &bar[st]);
      }
    }
    gi += nwarps;
    ijob += djob;
    ichunk += dchunk;
    if (ichunk >= nch) {
      ichunk -= nch;
      ++ijob;
    }
  };
  if (lane == 0)
    for (int i = 0; i < kDrawRing - 1; ++i) issue(i);
  int jid = static_cast<int>(g0 / nch), chunk = static_cast<int>(g0 - static_cast<int64_t>(jid) * nch);
  uint32_t phase_bits = 0u;  // parity of the next wait, per stage
  int i = 0;
  for (int64_t g = g0; g < items; g += nwarps, ++i) {
    __syncwarp();  // every lane is done with the stage that the next copy overwrites
    if (lane == 0) issue(i + kDrawRing - 1);
    __syncwarp();
    const int st = i % kDrawRing;
    const Job& jb = sjob[warp][st];
    const int32_t mode = jb.mode;
    if (job_needs_totals(mode, jb.sa.tau)) {
      const bool landed = mbar_wait_bounded(&bar[st], (phase_bits >> st) & 1u);
      phase_bits ^= 1u << st;
      double2* tc = tot_c + static_cast<size_t>(jid) * nch + chunk;
      double2* tg = tot_g + (static_cast<size_t>(jid) * nch + chunk) * kChunkGroups;
      if (!__all_sync(0xffffffffu, landed)) {
        // a copy that never completed: poison the job's totals (its draw reports -1) and stop
        if (lane == 0) *tc = make_double2(NAN, NAN);
        return;
      }
      const int c0 = chunk * kChunkElems, n = min(V - c0, kChunkElems);
      const T* sa = reinterpret_cast<const T*>(ring + st * kDrawStageBytes<T>);
      const T* sb = sa + kChunkElems;
      double sx[kChunkGroups], sy[kChunkGroups];
      if (mode == kResidual) {
        JobRows<T, true> J;
        J.init(nullptr, jb.sa, nullptr, jb.sb);
        smem_chunk_sums(J, sa, sb, n, sx, sy);
      } else {
        JobRows<T, false> J;
        J.init(nullptr, jb.sa, nullptr, jb.sa);
        smem_chunk_sums(J, sa, sa, n, sx, sy);
      }
      (void)c0;
      emit_chunk_totals(sx, sy, tc, tg);
    }
    chunk += dchunk;
    jid += djob;
    if (chunk >= nch) {
      chunk -= nch;
      ++jid;
    }
  }
}

// Totals pass with plain vector loads (any alignment), one warp per (job, chunk) item.
template <typename T>
__global__ void __launch_bounds__(kThreads) draw_totals_kernel(const T* __restrict__ A, const T* __restrict__ Bt, int V,
                                                              int njobs, const Job* __restrict__ jobs,
                                                              double2* __restrict__ tot_c,
                                                              double2* __restrict__ tot_g) {
  const int lane = threadIdx.x & 31;
  const int nch = nchunks_for(V);
  const int64_t items = static_cast<int64_t>(njobs) * nch;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items;
       it += nwarps) {
    const int jid = static_cast<int>(it / nch), chunk = static_cast<int>(it - static_cast<int64_t>(jid) * nch);
    const Job jb = load_job_cg(jobs + jid);
    if (!job_needs_totals(jb.mode, jb.sa.tau)) continue;
    const int c0 = chunk * kChunkElems, c1 = min(V, c0 + kChunkElems);
    double sx[kChunkGroups], sy[kChunkGroups];
    if (jb.mode == kResidual) {
      JobRows<T, true> J;
      J.init(A + static_cast<size_t>(jb.row_a) * V, jb.sa, Bt + static_cast<size_t>(jb.row_b) * V, jb.sb);
#pragma unroll
      for (int g = 0; g < kChunkGroups; ++g) {
        Raw8<T, true> x;
        J.load(c0 + g * kGroup + lane * 8, c1, x);
        const double2 t = lane_group_sums(J, x);
        sx[g] = t.x;
        sy[g] = t.y;
      }
    } else {
      JobRows<T, false> J;
      J.init(A + static_cast<size_t>(jb.row_a) * V, jb.sa, nullptr, jb.sa);
#pragma unroll
      for (int g = 0; g < kChunkGroups; ++g) {
        Raw8<T, false> x;
        J.load(c0 + g * kGroup + lane * 8, c1, x);
        const double2 t = lane_group_sums(J, x);
        sx[g] = t.x;
        sy[g] = t.y;
      }
    }
    emit_chunk_totals(sx, sy, tot_c + static_cast<size_t>(jid) * nch + chunk,
                      tot_g + (static_cast<size_t>(jid) * nch + chunk) * kChunkGroups);
  }
}

// Pick pass: one warp per job.
template <typename T>
__global__ void __launch_bounds__(kThreads, 1) draw_pick_kernel(const T* __restrict__ A, const T* __restrict__ Bt, int V,
                                                            int njobs, const Partial* __restrict__ parts_a,
                                                            const Job* __restrict__ jobs,
                                                            const double2* __restrict__ tot_c,
                                                            const double2* __restrict__ tot_g,
                                                            int32_t* __restrict__ out_tokens) {
  const int lane = threadIdx.x & 31;
  const int jid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (jid >= njobs) return;
  const Job jb = load_job_cg(jobs + jid);
  if (jb.mode < kSample) return;
  const int nch = nchunks_for(V);
  const T* ra = A + static_cast<size_t>(jb.row_a) * V;
  const T* rb = Bt + static_cast<size_t>(jb.row_b) * V;
  float ly;
  int y = -1;
  if (!job_needs_totals(jb.mode, jb.sa.tau)) {  // bonus draw without a cut: the row's partials
    double base, target;
    const int ch = warp_pick_chunk(parts_a + static_cast<size_t>(jb.row_a) * nch, nch, jb.sa, jb.u, &base, &target);
    JobRows<T, false> J;
    J.init(ra, jb.sa, nullptr, jb.sa);
    if (ch >= 0) y = warp_draw_chunk(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems), base, target, &ly);
  } else {
    const double2* jc = tot_c + static_cast<size_t>(jid) * nch;
    double base = 0.0, target = 0.0;
    bool use_p = false;
    const int ch = jb.mode == kSample ? warp_pick_totals(jc, nch, false, jb.u, &base, &target)
                                      : warp_pick_resid(jc, nch, jb.u, &base, &target, &use_p);
    if (ch >= 0) {
      // the group of the chunk holding target: lanes 0..7 hold the group totals
      const double2* jg = tot_g + (static_cast<size_t>(jid) * nch + ch) * kChunkGroups;
      const double t = lane < kChunkGroups ? (use_p ? __ldcg(&jg[lane].y) : __ldcg(&jg[lane].x)) : 0.0;
      double incl = t;
#pragma unroll
      for (int o = 1; o < kChunkGroups; o <<= 1) {
        const double v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      double excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.0;
      const bool in = lane < kChunkGroups && t > 0.0;
      const unsigned hit = __ballot_sync(0xffffffffu, in && base + incl > target);
      const unsigned pos = __ballot_sync(0xffffffffu, in);
      if (pos) {
        // rounding can leave no group crossing: the chunk's last positive group then
        const int G = hit ? __ffs(hit) - 1 : 31 - __clz(pos);
        const double gb = base + __shfl_sync(0xffffffffu, excl, G);
        const int c1 = min(V, (ch + 1) * kChunkElems);
        if (jb.mode == kSample) {
          JobRows<T, false> J;
          J.init(ra, jb.sa, nullptr, jb.sa);
          y = warp_draw_group(J, ch * kChunkElems + G * kGroup, c1, gb, target, &ly);
        } else {
          JobRows<T, true> J;
          J.init(ra, jb.sa, rb, jb.sb);
          J.use_p = use_p;
          y = warp_draw_group(J, ch * kChunkElems + G * kGroup, c1, gb, target, &ly);
        }
      }
    }
  }
  if (lane == 0) out_tokens[jb.out_index] = y;
}

}  // namespace psi
