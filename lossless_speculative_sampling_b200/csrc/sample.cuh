// sample.cuh -- inverse-CDF draws in vocabulary order.
//
// A draw with uniform u over non-negative weights r returns the first index v with
// C(v) > u * Z, C the inclusive prefix sum and Z the total (so a zero-weight token is never
// drawn). Two weight families are needed by the method (review page of arXiv 2609.04010,
// section 3.3): a row's own distribution (drafting, and the bonus token after a fully
// accepted block) and the residual max(0, p - q) of a rejected position.
//
// The draw is hierarchical. Slice totals (kSliceElems elements each) locate the slice that
// holds u * Z; they come from the row-statistics partials when the row's own distribution
// has no top-p cut, and from cdf_partial_kernel otherwise (a residual, or a kept set). Then
// one CTA scans that slice: each warp totals a contiguous kWarpSpan sub-range with coalesced
// 16-byte loads, a block scan picks the owning warp, which walks its sub-range 256 elements
// at a time with warp scans; the owning lane walks its 8 elements. All prefix sums are fp64.
#pragma once

#include "common.cuh"

namespace psi {

constexpr int kWarpSpan = kSliceElems / (kThreads / 32);  // elements per warp in a slice scan

struct ResidCtx {
  RowStat a, b;
  float ia, ib;  // 1 / s_kept of rows a and b
};

// residual weight max(0, p_a(v) - q_b(v)) and p_a(v)
__device__ __forceinline__ void resid_weight(const ResidCtx& r, float xa, float xb, float& res, float& pa) {
  pa = kept_weight(r.a, xa) * r.ia;
  float qb = kept_weight(r.b, xb) * r.ib;
  res = fmaxf(pa - qb, 0.0f);
}

// 8 consecutive elements starting at e (elements at or past `end` read as -inf)
template <typename T>
__device__ __forceinline__ void load8(const T* __restrict__ row, int e, int end, bool aligned, float (&x)[8]) {
  if (aligned && e + 8 <= end) {
    if (sizeof(T) == 2) {
      Vec<T>::load(row + e, x);
    } else {
      float lo[8], hi[8];
      Vec<T>::load(row + e, lo);
      Vec<T>::load(row + e + 4, hi);
#pragma unroll
      for (int k = 0; k < 4; ++k) { x[k] = lo[k]; x[k + 4] = hi[k]; }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = e + k < end ? load_elem(row + e + k) : -INFINITY;
  }
}

template <typename T>
struct JobRows {
  int mode;
  bool use_p;
  ResidCtx r;
  const T* ra;
  const T* rb;
  bool al_a, al_b;
  int end;

  // weights of elements e .. e+7; returns their fp32 sum
  __device__ __forceinline__ float weights8(int e, float (&w)[8]) const {
    float xa[8];
    load8(ra, e, end, al_a, xa);
    float sum = 0.0f;
    if (mode == kSample) {
#pragma unroll
      for (int k = 0; k < 8; ++k) { w[k] = kept_weight(r.a, xa[k]); sum += w[k]; }
    } else {
      float xb[8];
      load8(rb, e, end, al_b, xb);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float res, pa;
        resid_weight(r, xa[k], xb[k], res, pa);
        w[k] = use_p ? pa : res;
        sum += w[k];
      }
    }
    return sum;
  }
};

template <typename T>
__global__ void __launch_bounds__(kThreads) cdf_partial_kernel(const T* __restrict__ A, const T* __restrict__ Bt,
                                                               const RowStat* __restrict__ sa,
                                                               const RowStat* __restrict__ sb,
                                                               const Job* __restrict__ jobs, int V, int nslices,
                                                               double2* __restrict__ out) {
  __shared__ double red[33];
  const int unit = blockIdx.x;
  const int job = unit / nslices, slice = unit - job * nslices;
  const Job jb = jobs[job];
  if (jb.mode < kSample) return;
  ResidCtx r;
  r.a = sa[jb.row_a];
  if (jb.mode == kSample && r.a.tau == 0u) return;  // slice totals come from the row statistics
  const int v0 = slice * kSliceElems, v1 = min(V, v0 + kSliceElems);
  r.ia = 1.0f / r.a.s_kept;
  const T* ra = A + static_cast<size_t>(jb.row_a) * V;
  double sr = 0.0, sp = 0.0;
  constexpr int N = Vec<T>::N;
  if (jb.mode == kSample) {
    int a0, a1;
    vec_range(ra, v0, v1, a0, a1);
    for (int v = v0 + threadIdx.x; v < a0; v += blockDim.x) sr += kept_weight(r.a, load_elem(ra + v));
    for (int v = a1 + threadIdx.x; v < v1; v += blockDim.x) sr += kept_weight(r.a, load_elem(ra + v));
    for (int v = a0 + threadIdx.x * N; v < a1; v += blockDim.x * N) {
      float x[8], acc = 0.0f;
      Vec<T>::load(ra + v, x);
#pragma unroll
      for (int k = 0; k < N; ++k) acc += kept_weight(r.a, x[k]);
      sr += static_cast<double>(acc);
    }
  } else {
    r.b = sb[jb.row_b];
    r.ib = 1.0f / r.b.s_kept;
    const T* rb = Bt + static_cast<size_t>(jb.row_b) * V;
    int a0, a1, b0, b1;
    vec_range(ra, v0, v1, a0, a1);
    vec_range(rb, v0, v1, b0, b1);
    if (a0 != b0) { a0 = v1; a1 = v1; }  // rows aligned differently: scalar path
    auto one = [&](float xa, float xb, float& ar, float& ap) {
      float res, pa;
      resid_weight(r, xa, xb, res, pa);
      ar += res;
      ap += pa;
    };
    float ar = 0.0f, ap = 0.0f;
    for (int v = v0 + threadIdx.x; v < a0; v += blockDim.x) one(load_elem(ra + v), load_elem(rb + v), ar, ap);
    for (int v = a1 + threadIdx.x; v < v1; v += blockDim.x) one(load_elem(ra + v), load_elem(rb + v), ar, ap);
    sr += ar;
    sp += ap;
    for (int v = a0 + threadIdx.x * N; v < a1; v += blockDim.x * N) {
      float xa[8], xb[8];
      Vec<T>::load(ra + v, xa);
      Vec<T>::load(rb + v, xb);
      ar = 0.0f;
      ap = 0.0f;
#pragma unroll
      for (int k = 0; k < N; ++k) one(xa[k], xb[k], ar, ap);
      sr += static_cast<double>(ar);
      sp += static_cast<double>(ap);
    }
  }
  double tr = block_sum(sr, red);
  double tp = block_sum(sp, red);
  if (threadIdx.x == 0) out[unit] = make_double2(tr, tp);
}

// parts_a: row-statistics partials of tensor A (used for sample jobs without a top-p cut)
template <typename T>
__global__ void __launch_bounds__(kThreads) cdf_pick_kernel(const T* __restrict__ A, const T* __restrict__ Bt,
                                                            const RowStat* __restrict__ sa,
                                                            const RowStat* __restrict__ sb, const Job* __restrict__ jobs,
                                                            int V, int nslices, const Partial* __restrict__ parts_a,
                                                            const double2* __restrict__ parts, int32_t* __restrict__ out_tokens,
                                                            float* __restrict__ out_q) {
  __shared__ double wtot[kThreads / 32];
  __shared__ int sh_slice, sh_use_p, sh_y, sh_last, sh_owner;
  __shared__ double sh_base, sh_target, sh_c0;
  const Job jb = jobs[blockIdx.x];
  if (jb.mode < kSample) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const RowStat sta = sa[jb.row_a];
  const bool from_stats = jb.mode == kSample && sta.tau == 0u;
  if (threadIdx.x == 0) {
    const double2* pp = parts + static_cast<size_t>(blockIdx.x) * nslices;
    const Partial* ps = parts_a + static_cast<size_t>(jb.row_a) * nslices;
    auto total = [&](int s, int use_p) -> double {
      if (from_stats) return ps[s].m > -INFINITY ? ps[s].s * static_cast<double>(ex2((ps[s].m - sta.m) * sta.c)) : 0.0;
      return use_p ? pp[s].y : pp[s].x;
    };
    double Z = 0.0;
    for (int s = 0; s < nslices; ++s) Z += total(s, 0);
    int use_p = 0;
    if (jb.mode == kResidual && !(Z > 0.0)) {  // zero residual: draw from p instead
      use_p = 1;
      Z = 0.0;
      for (int s = 0; s < nslices; ++s) Z += total(s, 1);
    }
    const double target = static_cast<double>(jb.u) * Z;
    double C = 0.0, base = 0.0;
    int sel = -1;
    for (int s = 0; s < nslices; ++s) {
      const double w = total(s, use_p);
      if (w > 0.0) { sel = s; base = C; }
      if (C + w > target && w > 0.0) break;
      C += w;
    }
    sh_slice = sel;
    sh_use_p = use_p;
    sh_base = base;
    sh_target = target;
    sh_y = 0x7fffffff;
    sh_last = -1;
    sh_owner = -1;
  }
  __syncthreads();
  const int sel = sh_slice;
  if (sel < 0) {  // no mass anywhere (cannot happen for a valid row): report a data error
    if (threadIdx.x == 0) {
      out_tokens[jb.out_index] = -1;
      if (out_q && jb.aux >= 0) out_q[jb.aux] = -1.0f;
    }
    return;
  }
  JobRows<T> J;
  J.mode = jb.mode;
  J.use_p = sh_use_p != 0;
  J.r.a = sta;
  J.r.ia = 1.0f / sta.s_kept;
  J.ra = A + static_cast<size_t>(jb.row_a) * V;
  J.rb = nullptr;
  J.al_a = (reinterpret_cast<uintptr_t>(J.ra) & 15u) == 0;
  J.al_b = false;
  if (jb.mode == kResidual) {
    J.r.b = sb[jb.row_b];
    J.r.ib = 1.0f / J.r.b.s_kept;
    J.rb = Bt + static_cast<size_t>(jb.row_b) * V;
    J.al_b = (reinterpret_cast<uintptr_t>(J.rb) & 15u) == 0;
  }
  const int v0 = sel * kSliceElems, v1 = min(V, v0 + kSliceElems);
  const int w0 = v0 + warp * kWarpSpan, w1 = min(v1, w0 + kWarpSpan);
  J.end = w1;
  const double target = sh_target;

  // phase 1: per-warp totals of contiguous sub-ranges
  double mine = 0.0;
  int last = -1;
  for (int e = w0 + lane * 8; e < w1; e += 256) {
    float w[8];
    mine += static_cast<double>(J.weights8(e, w));
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (w[k] > 0.0f) last = e + k;
  }
  mine = warp_sum(mine);
  last = __reduce_max_sync(0xffffffffu, last);
  if (lane == 0) {
    wtot[warp] = mine;
    if (last >= 0) atomicMax(&sh_last, last);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double C = sh_base;
    for (int i = 0; i < kThreads / 32; ++i) {
      if (C <= target && target < C + wtot[i]) { sh_owner = i; sh_c0 = C; break; }
      C += wtot[i];
    }
  }
  __syncthreads();

  // phase 2: the owning warp walks its sub-range, 256 elements per step (vector sums in fp64
  // so that the lane walk below retraces the scanned totals)
  if (warp == sh_owner) {
    double Cb = sh_c0;
    int wlast = -1;
    for (int e = w0 + lane * 8; e - lane * 8 < w1; e += 256) {
      float w[8];
      J.weights8(e, w);
      double vs = 0.0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        vs += static_cast<double>(w[k]);
        if (w[k] > 0.0f) wlast = e + k;
      }
      double incl = vs;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      double excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.0;
      const unsigned hit = __ballot_sync(0xffffffffu, Cb + incl > target);
      if (hit) {
        if (lane == __ffs(hit) - 1) {
          double C = Cb + excl;
          int y = -1, lastpos = -1;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            C += static_cast<double>(w[k]);
            if (w[k] > 0.0f) lastpos = e + k;
            if (y < 0 && C > target) y = e + k;
          }
          sh_y = y >= 0 ? y : lastpos;  // rounding at the group's end: its last positive entry
        }
        break;
      }
      Cb += __shfl_sync(0xffffffffu, incl, 31);
    }
    // no crossing found (rounding against the phase-1 total): the warp's last positive entry
    wlast = __reduce_max_sync(0xffffffffu, wlast);
    if (lane == 0 && sh_y == 0x7fffffff && wlast >= 0) sh_y = wlast;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int y = sh_y != 0x7fffffff ? sh_y : sh_last;  // rounding at a sub-range edge: last positive entry
    out_tokens[jb.out_index] = y;
    if (out_q && jb.aux >= 0) out_q[jb.aux] = kept_weight(sta, load_elem(J.ra + y)) / sta.s_kept;
  }
}

}  // namespace psi
