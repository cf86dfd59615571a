// sample.cuh -- inverse-CDF draws in vocabulary order.
//
// A draw with uniform u over non-negative weights r returns the first index v with
// C(v) > u * Z, C the inclusive prefix sum and Z the total (so a zero-weight token is never
// drawn). Two weight families are needed by the method (review page of arXiv 2609.04010,
// section 3.3): a row's own distribution (drafting, and the bonus token after a fully
// accepted block) and the residual max(0, p - q) of a rejected position.
//
//   cdf_partial_kernel  one CTA per (job, slice): the slice's total weight (fp64), plus the
//                       total of p for the fallback when the residual is zero everywhere;
//   cdf_pick_kernel     one CTA per job: locates the slice holding u * Z from the slice
//                       totals, splits it into one contiguous run per thread, scans the run
//                       totals (fp64, thread order) and lets the owning thread walk its run.
#pragma once

#include "common.cuh"

namespace psi {

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

// Weight of element v for a job; `use_p` selects p_a for a residual job whose residual is 0.
template <typename T>
__device__ __forceinline__ float job_weight(int mode, bool use_p, const ResidCtx& r, const T* ra, const T* rb, int v) {
  float xa = load_elem(ra + v);
  if (mode == kSample) return kept_weight(r.a, xa);
  float res, pa;
  resid_weight(r, xa, load_elem(rb + v), res, pa);
  return use_p ? pa : res;
}

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
  const int v0 = slice * kSliceElems, v1 = min(V, v0 + kSliceElems);
  ResidCtx r;
  r.a = sa[jb.row_a];
  r.ia = 1.0f / r.a.s_kept;
  const T* ra = A + static_cast<size_t>(jb.row_a) * V;
  float sr = 0.0f, sp = 0.0f;
  constexpr int N = Vec<T>::N;
  if (jb.mode == kSample) {
    int a0, a1;
    vec_range(ra, v0, v1, a0, a1);
    for (int v = v0 + threadIdx.x; v < a0; v += blockDim.x) sr += kept_weight(r.a, load_elem(ra + v));
    for (int v = a1 + threadIdx.x; v < v1; v += blockDim.x) sr += kept_weight(r.a, load_elem(ra + v));
    for (int v = a0 + threadIdx.x * N; v < a1; v += blockDim.x * N) {
      float x[8];
      Vec<T>::load(ra + v, x);
#pragma unroll
      for (int k = 0; k < N; ++k) sr += kept_weight(r.a, x[k]);
    }
  } else {
    r.b = sb[jb.row_b];
    r.ib = 1.0f / r.b.s_kept;
    const T* rb = Bt + static_cast<size_t>(jb.row_b) * V;
    int a0, a1, b0, b1;
    vec_range(ra, v0, v1, a0, a1);
    vec_range(rb, v0, v1, b0, b1);
    if (a0 != b0) { a0 = v1; a1 = v1; }  // rows aligned differently: scalar path
    auto one = [&](float xa, float xb) {
      float res, pa;
      resid_weight(r, xa, xb, res, pa);
      sr += res;
      sp += pa;
    };
    for (int v = v0 + threadIdx.x; v < a0; v += blockDim.x) one(load_elem(ra + v), load_elem(rb + v));
    for (int v = a1 + threadIdx.x; v < v1; v += blockDim.x) one(load_elem(ra + v), load_elem(rb + v));
    for (int v = a0 + threadIdx.x * N; v < a1; v += blockDim.x * N) {
      float xa[8], xb[8];
      Vec<T>::load(ra + v, xa);
      Vec<T>::load(rb + v, xb);
#pragma unroll
      for (int k = 0; k < N; ++k) one(xa[k], xb[k]);
    }
  }
  double tr = block_sum(static_cast<double>(sr), red);
  double tp = block_sum(static_cast<double>(sp), red);
  if (threadIdx.x == 0) out[unit] = make_double2(tr, tp);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) cdf_pick_kernel(const T* __restrict__ A, const T* __restrict__ Bt,
                                                            const RowStat* __restrict__ sa,
                                                            const RowStat* __restrict__ sb, const Job* __restrict__ jobs,
                                                            int V, int nslices, const double2* __restrict__ parts,
                                                            int32_t* __restrict__ out_tokens, float* __restrict__ out_q) {
  __shared__ double red[33];
  __shared__ int sh_slice, sh_use_p, sh_y, sh_last;
  __shared__ double sh_base, sh_target;
  const Job jb = jobs[blockIdx.x];
  if (jb.mode < kSample) return;
  const double2* pp = parts + static_cast<size_t>(blockIdx.x) * nslices;
  if (threadIdx.x == 0) {
    double Z = 0.0;
    for (int s = 0; s < nslices; ++s) Z += pp[s].x;
    int use_p = 0;
    if (jb.mode == kResidual && !(Z > 0.0)) {  // zero residual: draw from p instead
      use_p = 1;
      Z = 0.0;
      for (int s = 0; s < nslices; ++s) Z += pp[s].y;
    }
    const double target = static_cast<double>(jb.u) * Z;
    double C = 0.0;
    int sel = -1;
    double base = 0.0;
    for (int s = 0; s < nslices; ++s) {
      double w = use_p ? pp[s].y : pp[s].x;
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
  ResidCtx r;
  r.a = sa[jb.row_a];
  r.ia = 1.0f / r.a.s_kept;
  const T* ra = A + static_cast<size_t>(jb.row_a) * V;
  const T* rb = nullptr;
  if (jb.mode == kResidual) {
    r.b = sb[jb.row_b];
    r.ib = 1.0f / r.b.s_kept;
    rb = Bt + static_cast<size_t>(jb.row_b) * V;
  }
  const bool use_p = sh_use_p != 0;
  const int v0 = sel * kSliceElems, v1 = min(V, v0 + kSliceElems);
  const int run = (v1 - v0 + blockDim.x - 1) / blockDim.x;
  const int r0 = min(v1, v0 + threadIdx.x * run), r1 = min(v1, r0 + run);
  double mine = 0.0;
  int last = -1;
  for (int v = r0; v < r1; ++v) {
    float w = job_weight<T>(jb.mode, use_p, r, ra, rb, v);
    mine += static_cast<double>(w);
    if (w > 0.0f) last = v;
  }
  double total;
  const double C0 = sh_base + block_exclusive_scan(mine, red, &total);
  if (last >= 0) atomicMax(&sh_last, last);
  const double target = sh_target;
  if (C0 <= target && target < C0 + mine) {
    double C = C0;
    for (int v = r0; v < r1; ++v) {
      C += static_cast<double>(job_weight<T>(jb.mode, use_p, r, ra, rb, v));
      if (C > target) {
        atomicMin(&sh_y, v);
        break;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int y = sh_y != 0x7fffffff ? sh_y : sh_last;  // rounding at a run edge: last positive entry
    out_tokens[jb.out_index] = y;
    if (out_q && jb.aux >= 0) out_q[jb.aux] = kept_weight(r.a, load_elem(ra + y)) / r.a.s_kept;
  }
}

}  // namespace psi
