// sample.cuh -- inverse-CDF draws in vocabulary order (warp- and block-level building blocks).
//
// A draw with uniform u over non-negative weights r returns the first index v with
// C(v) > u * Z, C the inclusive prefix sum and Z the total (so a zero-weight token is never
// drawn). Two weight families are needed by the method (review page of arXiv 2609.04010,
// section 3.3): a row's own distribution (drafting, and the bonus token after a fully
// accepted block) and the residual max(0, p - q) of a rejected position.
//
// Ranges are walked by warps in groups of 256 elements (8 consecutive elements per lane,
// coalesced), with kBatch groups loaded before any is used. warp_draw_range scans a range
// with warp-wide fp64 prefix sums and lets the lane that crosses u * Z walk its 8 elements;
// block_draw_range first totals one contiguous sub-range per warp and hands the crossing to
// the owning warp. Per-element weights are fp32, every prefix sum is fp64.
#pragma once

#include "common.cuh"

namespace psi {

constexpr int kGroup = 256;     // elements per warp step (8 per lane)
template <bool RESID>
constexpr int kDrawBatch = 4;  // groups in flight per lane

struct ResidCtx {
  RowStat a, b;
  float ia, ib;  // 1 / s_kept of rows a and b
};

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

// The raw bits of 8 consecutive elements (one 16-byte word for bf16, two for fp32), kept
// packed while loads are in flight. Elements at or past `end` read as -inf.
template <typename T>
struct Raw8x {
  uint4 w[sizeof(T) == 2 ? 1 : 2];
  __device__ __forceinline__ void load(const T* __restrict__ row, int e, int end, bool aligned) {
    if (aligned && e + 8 <= end) {
      w[0] = __ldg(reinterpret_cast<const uint4*>(row + e));
      if constexpr (sizeof(T) == 4) w[1] = __ldg(reinterpret_cast<const uint4*>(row + e + 4));
    } else {
      float x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = e + k < end ? load_elem(row + e + k) : -INFINITY;
      pack(x);
    }
  }
  __device__ __forceinline__ void pack(const float (&x)[8]) {
    if constexpr (sizeof(T) == 2) {  // every value here is an exact bf16 (or -inf)
      w[0] = make_uint4((__float_as_uint(x[0]) >> 16) | (__float_as_uint(x[1]) & 0xFFFF0000u),
                        (__float_as_uint(x[2]) >> 16) | (__float_as_uint(x[3]) & 0xFFFF0000u),
                        (__float_as_uint(x[4]) >> 16) | (__float_as_uint(x[5]) & 0xFFFF0000u),
                        (__float_as_uint(x[6]) >> 16) | (__float_as_uint(x[7]) & 0xFFFF0000u));
    } else {
      w[0] = make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
      w[1] = make_uint4(__float_as_uint(x[4]), __float_as_uint(x[5]), __float_as_uint(x[6]), __float_as_uint(x[7]));
    }
  }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    if constexpr (sizeof(T) == 2) {
      Vec<T>::unpack(w[0], x);
    } else {
      float lo[8], hi[8];
      Vec<T>::unpack(w[0], lo);
      Vec<T>::unpack(w[1], hi);
#pragma unroll
      for (int k = 0; k < 4; ++k) { x[k] = lo[k]; x[k + 4] = hi[k]; }
    }
  }
};

// Raw logits of one 8-element group (row a, and row b for a residual).
template <typename T, bool RESID>
struct Raw8 {
  Raw8x<T> a;
  Raw8x<T> b[RESID ? 1 : 0 + 1];
};

// The weights a draw runs over: row a's kept distribution (RESID = false), or the residual
// max(0, p_a - q_b) (RESID = true), or, with use_p, p_a normalised (the fallback when the
// residual is zero everywhere).
template <typename T, bool RESID>
struct JobRows {
  static constexpr bool kResid = RESID;
  bool use_p;
  ResidCtx r;
  const T* ra;
  const T* rb;
  bool al_a, al_b;

  __device__ __forceinline__ void init(const T* rowa, const RowStat& sa, const T* rowb, const RowStat& sb) {
    use_p = false;
    r.a = sa;
    r.ia = 1.0f / sa.s_kept;
    ra = rowa;
    al_a = (reinterpret_cast<uintptr_t>(rowa) & 15u) == 0;
    rb = rowb;
    r.b = sb;
    r.ib = RESID ? 1.0f / sb.s_kept : 0.0f;
    al_b = RESID && (reinterpret_cast<uintptr_t>(rowb) & 15u) == 0;
  }
  __device__ __forceinline__ void load(int e, int end, Raw8<T, RESID>& x) const {
    x.a.load(ra, e, end, al_a);
    if constexpr (RESID) x.b[0].load(rb, e, end, al_b);
  }
  // weights (and p_a, for residual totals) of a loaded group
  __device__ __forceinline__ void weights(const Raw8<T, RESID>& x, float (&w)[8], float (&pw)[8]) const {
    float xa[8];
    x.a.unpack(xa);
    exp8(xa, r.a.m, r.a.c, pw);
    if (r.a.tau != 0u) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (fkey(xa[k]) < r.a.tau) pw[k] = 0.0f;
    }
    if constexpr (RESID) {
      float xb[8], qw[8];
      x.b[0].unpack(xb);
      exp8(xb, r.b.m, r.b.c, qw);
      if (r.b.tau != 0u) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (fkey(xb[k]) < r.b.tau) qw[k] = 0.0f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        pw[k] *= r.ia;
        w[k] = use_p ? pw[k] : fmaxf(pw[k] - qw[k] * r.ib, 0.0f);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = pw[k];
    }
  }
};

// Warp-level totals over [lo, hi) of the job weights (.x) and of p_a (.y), and the last
// index with positive weight; every lane gets them.
template <typename T, bool RESID>
__device__ double2 warp_range_totals(const JobRows<T, RESID>& J, int lo, int hi, int* last_pos) {
  const int lane = threadIdx.x & 31;
  double sr = 0.0, sp = 0.0;
  int last = -1;
  for (int g = lo; g < hi; g += kDrawBatch<RESID> * kGroup) {
    Raw8<T, RESID> x[kDrawBatch<RESID>];
#pragma unroll
    for (int b = 0; b < kDrawBatch<RESID>; ++b) J.load(g + b * kGroup + lane * 8, hi, x[b]);
#pragma unroll
    for (int b = 0; b < kDrawBatch<RESID>; ++b) {
      float w[8], pw[8];
      J.weights(x[b], w, pw);
      float ar = 0.0f, ap = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        ar += w[k];
        ap += pw[k];
        if (w[k] > 0.0f) last = g + b * kGroup + lane * 8 + k;
      }
      sr += static_cast<double>(ar);
      sp += static_cast<double>(ap);
    }
  }
  *last_pos = __reduce_max_sync(0xffffffffu, last);
  return make_double2(warp_sum(sr), warp_sum(sp));
}

// Warp-level draw inside [lo, hi): `base` is the weight before lo, `target` = u * Z.
// Returns the first index whose inclusive prefix exceeds target, or the last index with
// positive weight when rounding leaves none (-1 if the range has no positive weight).
template <typename T, bool RESID, int NB = kDrawBatch<RESID>>
__device__ int warp_draw_range(const JobRows<T, RESID>& J, int lo, int hi, double base, double target) {
  const int lane = threadIdx.x & 31;
  double Cb = base;
  int wlast = -1;
  for (int g = lo; g < hi; g += NB * kGroup) {
    Raw8<T, RESID> x[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) J.load(g + b * kGroup + lane * 8, hi, x[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int e = g + b * kGroup + lane * 8;
      float w[8], pw[8];
      J.weights(x[b], w, pw);
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
        const int src = __ffs(hit) - 1;
        int y = -1, lastpos = -1;
        if (lane == src) {
          double C = Cb + excl;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            C += static_cast<double>(w[k]);
            if (w[k] > 0.0f) lastpos = e + k;
            if (y < 0 && C > target) y = e + k;
          }
          if (y < 0) y = lastpos;  // rounding at the group's end: its last positive entry
        }
        return __shfl_sync(0xffffffffu, y, src);
      }
      Cb += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  return __reduce_max_sync(0xffffffffu, wlast);
}

// Block-level totals over [lo, hi) (.x job weights, .y p_a); every thread gets them.
template <typename T, bool RESID>
__device__ double2 block_range_totals(const JobRows<T, RESID>& J, int lo, int hi, double* red) {
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int span = (((hi - lo + nw - 1) / nw) + 7) & ~7;
  const int w0 = min(hi, lo + warp * span), w1 = min(hi, w0 + span);
  int last;
  const double2 t = warp_range_totals(J, w0, w1, &last);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) { red[warp] = t.x; red[32 + warp] = t.y; }
  __syncthreads();
  double x = 0.0, y = 0.0;
  for (int i = 0; i < nw; ++i) { x += red[i]; y += red[32 + i]; }
  __syncthreads();
  return make_double2(x, y);
}

struct DrawSmem {
  double wtot[32];
  double c0, target;
  int owner, y, last;
};

// Block-level draw inside [lo, hi) (lo a multiple of 8). With target >= 0 the draw is
// absolute: `base` is the weight before lo and `target` = u * Z of the whole distribution.
// With target < 0 the range is the whole distribution: target = u * (range total). Returns
// the drawn index to every thread (-1 if the range has no positive weight).
template <typename T, bool RESID>
__device__ int block_draw_range(const JobRows<T, RESID>& J, int lo, int hi, double base, double target, float u,
                                DrawSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int span = (((hi - lo + nw - 1) / nw) + 7) & ~7;
  const int w0 = min(hi, lo + warp * span), w1 = min(hi, w0 + span);
  int last;
  const double2 t = warp_range_totals(J, w0, w1, &last);
  __syncthreads();
  if (threadIdx.x == 0) { sm.y = -1; sm.last = -1; sm.owner = -1; }
  __syncthreads();
  if (lane == 0) {
    sm.wtot[warp] = t.x;
    if (last >= 0) atomicMax(&sm.last, last);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double C = base, tg = target;
    if (tg < 0.0) {
      double Z = 0.0;
      for (int i = 0; i < nw; ++i) Z += sm.wtot[i];
      tg = static_cast<double>(u) * Z;
      C = 0.0;
    }
    sm.target = tg;
    for (int i = 0; i < nw; ++i) {
      if (C <= tg && tg < C + sm.wtot[i]) { sm.owner = i; sm.c0 = C; break; }
      C += sm.wtot[i];
    }
  }
  __syncthreads();
  if (warp == sm.owner) {
    const int y = warp_draw_range(J, w0, w1, sm.c0, sm.target);
    if (lane == 0) sm.y = y;
  }
  __syncthreads();
  const int y = sm.y >= 0 ? sm.y : sm.last;  // past every sub-range (rounding): last positive entry
  __syncthreads();
  return y;
}

}  // namespace psi
