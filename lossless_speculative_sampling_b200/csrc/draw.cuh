// draw.cuh -- the draw jobs of a verification call (the residual draw max(0, p - q) at a
// first rejection, or the bonus draw from p after a fully accepted block; Psi-Spec review page
// of arXiv 2609.04010, section 3.3) in one launch: a cluster of CL CTAs per job.
//
// CTA `rank` owns the vocabulary slice [rank * slice, (rank + 1) * slice) and each of its warps
// a contiguous part of that slice, read in steps of 256 elements (8 per lane). One pass over
// both rows reduces every part to its total, once for the job's weights (x) and once for p
// (y, the fallback when the residual is zero everywhere), keeping each lane's 8-element group
// weights in shared memory. The CTAs push their parts' totals to every
// rank through distributed shared memory; after one cluster barrier every thread forms the
// same running sums over (rank, warp), i.e. in vocabulary order, and the one part whose
// interval [start, next start) holds u * Z scans its kept group weights to the group, which one
// lane reads again (from L1/L2) to the first index whose inclusive prefix exceeds u * Z.
// Rounding inside a part falls back to the part's last index with positive weight, as the
// two-pass draw does.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "finish.cuh"
#include "sample.cuh"

namespace psi {

namespace cgd = cooperative_groups;

constexpr int kDrawClusterWarps = 8;
constexpr int kMaxDrawCluster = 16;
constexpr int kDrawClusterBatch = 3;  // steps of both rows in flight per lane
constexpr int kDrawMaxSteps = 16;     // 256-element steps per warp part (the host checks V)

struct DrawClusterShared {
  double gt[kDrawClusterWarps][kDrawMaxSteps][32];   // per (warp, step, lane): the group's weight
  double wt[kDrawClusterWarps][2];                   // this CTA's part totals (x, y)
  double xw[kMaxDrawCluster][kDrawClusterWarps][2];  // every rank's part totals (pushed)
  int pick;                                          // rank 0: the drawn index (atomic minimum)
};

__host__ __device__ inline int draw_slice(int V, int cl) { return (((V + cl - 1) / cl) + 7) & ~7; }
__host__ __device__ inline int draw_part(int V, int cl) {
  return ((draw_slice(V, cl) + kDrawClusterWarps - 1) / kDrawClusterWarps + 7) & ~7;
}

// Bonus draw without a top-p cut (the verifier row's own chunk partials locate the chunk,
// which one warp walks); returns the index or -1.
template <typename T>
__device__ int warp_bonus_draw(const Job& jb, const T* ra, int V, const Partial* parts_a) {
  const int nch = nchunks_for(V);
  double base, target;
  const int ch = warp_pick_chunk(parts_a + static_cast<size_t>(jb.row_a) * nch, nch, jb.sa, jb.u, &base, &target);
  JobRows<T, false> J;
  J.init(ra, jb.sa, nullptr, jb.sa);
  float ly;
  return ch >= 0 ? warp_draw_chunk(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems), base, target, &ly) : -1;
}

// Inclusive scan of a double over the lanes.
__device__ __forceinline__ double lane_incl_scan(double v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// The element of one 8-element group at e whose inclusive prefix (from C) exceeds target,
// else the group's last positive element (-1 if none): one lane's walk.
template <typename T, bool RESID>
__device__ __forceinline__ int group_walk(const JobRows<T, RESID>& J, int e, int end, double C, double target) {
  Raw8<T, RESID> xg;
  J.load(e, end, xg);
  float w[8], pw[8];
  J.weights(xg, w, pw);
  int y = -1, lp = -1;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    C += static_cast<double>(w[k]);
    if (w[k] > 0.0f) lp = e + k;
    if (y < 0 && w[k] > 0.0f && C > target) y = e + k;
  }
  return y >= 0 ? y : lp;
}

template <typename T, bool RESID, int CL>
__device__ void draw_cluster_job(cgd::cluster_group& cl, DrawClusterShared& sh, const Job& jb, const T* ra,
                                 const T* rb, int V) {
  constexpr int W = kDrawClusterWarps, NB = kDrawClusterBatch, kStepElems = 256;
  const int rank = static_cast<int>(cl.block_rank());
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slice = draw_slice(V, CL), part = draw_part(V, CL);
  const int v0 = min(V, rank * slice), v1 = min(V, v0 + slice);
  const int w0 = min(v1, v0 + warp * part), w1 = min(v1, w0 + part);
  JobRows<T, RESID> J;
  J.init(ra, jb.sa, RESID ? rb : ra, RESID ? jb.sb : jb.sa);

  // pass 1: each lane's group weights (8-term fp32 sums, kept as fp64 for the walk) and the
  // part's totals
  double ax = 0.0, ay = 0.0;
  int step = 0;
  for (int s0 = w0; s0 < w1; s0 += NB * kStepElems) {
    Raw8<T, RESID> x[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (s0 + b * kStepElems < w1) J.load(s0 + b * kStepElems + lane * 8, w1, x[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (s0 + b * kStepElems >= w1) break;
      float w[8], pw[8];
      J.weights(x[b], w, pw);
      const double mx = static_cast<double>(sum8(w));
      sh.gt[warp][step++][lane] = mx;
      ax += mx;
      ay += static_cast<double>(sum8(pw));
    }
  }
  const double Wx = warp_sum(ax), Wy = warp_sum(ay);
  if (lane == 0) {
    sh.wt[warp][0] = Wx;
    sh.wt[warp][1] = Wy;
  }
  if (threadIdx.x == 0) sh.pick = 0x7fffffff;
  __syncthreads();
  if (threadIdx.x < CL) {  // this CTA's totals to rank threadIdx.x
    double* xw = cl.map_shared_rank(&sh.xw[rank][0][0], static_cast<int>(threadIdx.x));
#pragma unroll
    for (int i = 0; i < W; ++i) {
      xw[2 * i] = sh.wt[i][0];
      xw[2 * i + 1] = sh.wt[i][1];
    }
  }
  cl.sync();

  // running sums over the parts (rank, warp) in vocabulary order: lane l holds parts
  // kPer * l .. kPer * l + kPer - 1; the same procedure in every warp of every CTA
  constexpr int kParts = CL * W, kPer = (kParts + 31) / 32;
  static_assert(kPer <= 4, "parts per lane");
  double px[kPer], py[kPer], sx = 0.0, sy = 0.0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int k = lane * kPer + i;
    px[i] = k < kParts ? sh.xw[k / W][k % W][0] : 0.0;
    py[i] = k < kParts ? sh.xw[k / W][k % W][1] : 0.0;
    sx += px[i];
    sy += py[i];
  }
  const double ix = lane_incl_scan(sx), iy = lane_incl_scan(sy);
  const double gx = __shfl_sync(0xffffffffu, ix, 31), gy = __shfl_sync(0xffffffffu, iy, 31);
  const bool use_p = RESID && !(gx > 0.0);  // residual zero everywhere: p itself
  const double grand = use_p ? gy : gx;
  const double target = static_cast<double>(jb.u) * grand;
  // part starts: a lane's first part starts at the previous lane's inclusive sum, and every
  // part ends where the next one starts (the lane's sum closes its last part), so the
  // intervals tile [0, grand) up to one-ulp overlaps, which the minimum below resolves
  const double incl = use_p ? iy : ix;
  double st[kPer + 1];
  st[0] = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) st[0] = 0.0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) st[i + 1] = i + 1 < kPer ? st[i] + (use_p ? py[i] : px[i]) : incl;
  const int me = rank * W + warp;  // this warp's part
  const int holder = me / kPer, slot = me % kPer;
  double my_start = 0.0, my_end = 0.0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const double s0 = __shfl_sync(0xffffffffu, st[i], holder);
    const double s1 = __shfl_sync(0xffffffffu, st[i + 1], holder);
    if (i == slot) {
      my_start = s0;
      my_end = s1;
    }
  }

  if (my_start <= target && target < my_end) {
    // this part holds u * Z: its steps' group weights locate the group, one lane walks it
    J.use_p = use_p;
    double C = my_start;
    int y = -1, last_e = -1;  // last_e: the last group with positive weight
    for (int s = 0; s < step && y < 0; ++s) {
      const int e = w0 + s * kStepElems + lane * 8;
      double mine;
      if (use_p) {  // the kept group weights are the residual's: recompute p's (rare)
        Raw8<T, RESID> xg;
        J.load(e, w1, xg);
        float w[8], pw[8];
        J.weights(xg, w, pw);
        mine = static_cast<double>(sum8(w));
      } else {
        mine = sh.gt[warp][s][lane];
      }
      const double gi = lane_incl_scan(mine);
      const unsigned pos = __ballot_sync(0xffffffffu, mine > 0.0);
      if (pos) last_e = w0 + s * kStepElems + (31 - __clz(pos)) * 8;
      const unsigned hit = __ballot_sync(0xffffffffu, mine > 0.0 && C + gi > target);
      if (hit) {
        const int src = __ffs(hit) - 1;
        const double Cs = C + __shfl_sync(0xffffffffu, gi - mine, src);
        if (lane == 0) y = group_walk(J, w0 + s * kStepElems + src * 8, w1, Cs, target);
        y = __shfl_sync(0xffffffffu, y, 0);
        if (y < 0) y = 0x7fffffff;  // (cannot happen: the group has positive weight)
      }
      C += __shfl_sync(0xffffffffu, gi, 31);
    }
    // rounding past the part's end: its last positive element
    if (y < 0 && last_e >= 0 && lane == 0) y = group_walk(J, last_e, w1, 0.0, INFINITY);
    if (lane == 0 && y >= 0 && y != 0x7fffffff) atomicMin(cl.map_shared_rank(&sh.pick, 0), y);
  }
  cl.sync();  // the pick has landed in rank 0; no CTA leaves while another may write to it
}

template <typename T, int CL>
__global__ void __launch_bounds__(kDrawClusterWarps * 32, sizeof(T) == 2 ? 4 : 2) draw_cluster_kernel(
    const T* __restrict__ A, const T* __restrict__ Bt, int V, const Partial* __restrict__ parts_a,
    const Job* __restrict__ jobs, int32_t* __restrict__ out_tokens) {
  static_assert(CL <= kMaxDrawCluster, "push slots per rank");
  cgd::cluster_group cl = cgd::this_cluster();
  __shared__ DrawClusterShared sh;
  const int rank = static_cast<int>(cl.block_rank());
  const Job jb = load_job_cg(jobs + blockIdx.x / CL);  // the grid holds exactly njobs clusters
  if (jb.mode < kSample) return;                     // the same job in every CTA of the cluster
  const T* ra = A + static_cast<size_t>(jb.row_a) * V;
  const T* rb = Bt + static_cast<size_t>(jb.row_b) * V;
  if (!job_needs_totals(jb.mode, jb.sa.tau)) {  // no cluster barrier on this path
    if (rank == 0 && threadIdx.x < 32) {
      const int y = warp_bonus_draw<T>(jb, ra, V, parts_a);
      if (threadIdx.x == 0) out_tokens[jb.out_index] = y;
    }
    return;
  }
  if (jb.mode == kResidual)
    draw_cluster_job<T, true, CL>(cl, sh, jb, ra, rb, V);
  else
    draw_cluster_job<T, false, CL>(cl, sh, jb, ra, rb, V);
  if (rank == 0 && threadIdx.x == 0) out_tokens[jb.out_index] = sh.pick != 0x7fffffff ? sh.pick : -1;
}

}  // namespace psi
