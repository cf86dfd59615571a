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
  float ta, tb;  // smallest kept logit of rows a and b (cut_value of their thresholds)
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
  // 8 elements known to be in range, from a 16-byte aligned address
  __device__ __forceinline__ void load_full(const T* __restrict__ row, int e) {
    w[0] = __ldg(reinterpret_cast<const uint4*>(row + e));
    if constexpr (sizeof(T) == 4) w[1] = __ldg(reinterpret_cast<const uint4*>(row + e + 4));
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
    r.ta = cut_value(sa.tau);
    r.tb = cut_value(sb.tau);
    al_b = RESID && (reinterpret_cast<uintptr_t>(rowb) & 15u) == 0;
  }
  __device__ __forceinline__ float logit_a(int v) const { return load_elem(ra + v); }
  // whether [lo, lo + n) can be read with unconditional aligned vector loads
  __device__ __forceinline__ bool vector_ok(int lo, int hi, int n) const {
    return hi - lo == n && al_a && (!RESID || al_b);
  }
  __device__ __forceinline__ void load_full(int e, Raw8<T, RESID>& x) const {
    x.a.load_full(ra, e);
    if constexpr (RESID) x.b[0].load_full(rb, e);
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
        if (xa[k] < r.ta) pw[k] = 0.0f;
    }
    if constexpr (RESID) {
      float xb[8], qw[8];
      x.b[0].unpack(xb);
      exp8(xb, r.b.m, r.b.c, qw);
      if (r.b.tau != 0u) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (xb[k] < r.tb) qw[k] = 0.0f;
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

// Groups of one chunk, and how many of them warp_chunk_totals and warp_draw_chunk keep in
// flight at once (the whole chunk, except for residual fp32 rows: half of it).
constexpr int kChunkGroups = kChunkElems / kGroup;
template <typename T, bool RESID>
constexpr int kChunkBatch = (sizeof(T) == 4 && RESID) ? kChunkGroups / 2 : kChunkGroups;

// This lane's weight in one loaded group (8 elements: an fp32 sum, returned as fp64), and its
// last positive index.
template <typename T, bool RESID>
__device__ __forceinline__ double lane_group_weight(const JobRows<T, RESID>& J, const Raw8<T, RESID>& x, int e,
                                                    int* last) {
  float w[8], pw[8];
  J.weights(x, w, pw);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (w[k] > 0.0f) *last = e + k;
  return static_cast<double>(sum8(w));
}

// This lane's sums of the job weights (.x) and of p_a (.y) over one loaded group (8-term fp32
// sums, returned as fp64).
template <typename T, bool RESID>
__device__ __forceinline__ double2 lane_group_sums(const JobRows<T, RESID>& J, const Raw8<T, RESID>& x) {
  float w[8], pw[8];
  J.weights(x, w, pw);
  return make_double2(static_cast<double>(sum8(w)), RESID ? static_cast<double>(sum8(pw)) : 0.0);
}

// Warp-level totals of one chunk [lo, hi) (hi - lo <= kChunkElems, lo a multiple of 8): the
// job weights (.x) and p_a (.y), summed in fp64 per lane and across lanes, with a whole batch
// of groups in flight at once. Every lane gets them.
template <typename T, bool RESID>
__device__ double2 warp_chunk_totals(const JobRows<T, RESID>& J, int lo, int hi) {
  constexpr int NB = kChunkBatch<T, RESID>;
  const int lane = threadIdx.x & 31;
  const bool full = J.vector_ok(lo, hi, kChunkElems);
  double sr = 0.0, sp = 0.0;
#pragma unroll
  for (int g0 = 0; g0 < kChunkGroups; g0 += NB) {
    Raw8<T, RESID> x[NB];
    if (full) {
#pragma unroll
      for (int g = 0; g < NB; ++g) J.load_full(lo + (g0 + g) * kGroup + lane * 8, x[g]);
    } else {
#pragma unroll
      for (int g = 0; g < NB; ++g) J.load(lo + (g0 + g) * kGroup + lane * 8, hi, x[g]);
    }
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      const double2 t = lane_group_sums(J, x[g]);
      sr += t.x;
      sp += t.y;
    }
  }
  return make_double2(warp_sum(sr), warp_sum(sp));
}

// Warp-level total of the job weights of one chunk [lo, hi) (8-term fp32 sums per lane, fp64
// beyond), with a whole batch of groups in flight at once. Every lane gets it.
template <typename T, bool RESID>
__device__ double warp_chunk_weight(const JobRows<T, RESID>& J, int lo, int hi) {
  constexpr int NB = kChunkBatch<T, RESID>;
  const int lane = threadIdx.x & 31;
  const bool full = J.vector_ok(lo, hi, kChunkElems);
  double s = 0.0;
#pragma unroll
  for (int g0 = 0; g0 < kChunkGroups; g0 += NB) {
    Raw8<T, RESID> x[NB];
    if (full) {
#pragma unroll
      for (int g = 0; g < NB; ++g) J.load_full(lo + (g0 + g) * kGroup + lane * 8, x[g]);
    } else {
#pragma unroll
      for (int g = 0; g < NB; ++g) J.load(lo + (g0 + g) * kGroup + lane * 8, hi, x[g]);
    }
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      float w[8], pw[8];
      J.weights(x[g], w, pw);
      s += static_cast<double>(sum8(w));
    }
  }
  return warp_sum(s);
}

// Reduce-scatter of eight per-lane values: lane l ends with the warp total of value
// (l >> 2) & 7 (halves exchanged over lane bits 4, 3, 2, then summed over bits 1, 0).
__device__ __forceinline__ double warp_reduce_scatter8(const double (&v)[8]) {
  const int lane = threadIdx.x & 31;
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  double h[4], q[2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const double send = b4 ? v[k] : v[k + 4], keep = b4 ? v[k + 4] : v[k];
    h[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const double send = b3 ? h[k] : h[k + 2], keep = b3 ? h[k + 2] : h[k];
    q[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const double send = b2 ? q[0] : q[1], keep = b2 ? q[1] : q[0];
  double r = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  r += __shfl_xor_sync(0xffffffffu, r, 2);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r;
}

// Totals of one chunk from per-lane group sums (sx the job weights, sy p_a): writes the eight
// group totals to tg[0..7] and the chunk total to *tc (fp64 throughout).
__device__ __forceinline__ void emit_chunk_totals(const double (&sx)[kChunkGroups], const double (&sy)[kChunkGroups],
                                                  double2* tc, double2* tg) {
  static_assert(kChunkGroups == 8, "eight groups per chunk");
  const int lane = threadIdx.x & 31;
  double gx = warp_reduce_scatter8(sx), gy = warp_reduce_scatter8(sy);
  if ((lane & 3) == 0) tg[lane >> 2] = make_double2(gx, gy);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    gx += __shfl_xor_sync(0xffffffffu, gx, o);
    gy += __shfl_xor_sync(0xffffffffu, gy, o);
  }
  if (lane == 0) *tc = make_double2(gx, gy);
}

// Warp-level draw inside one group [e0, e0 + kGroup) (clipped at hi): `base` is the weight
// before e0 and `target` = u * Z. Returns the first index whose inclusive prefix exceeds
// target, else (rounding) the group's last index with positive weight, or -1 if it has none;
// *la receives row a's logit at that index.
template <typename T, bool RESID>
__device__ int warp_draw_group(const JobRows<T, RESID>& J, int e0, int hi, double base, double target, float* la) {
  const int lane = threadIdx.x & 31;
  const int e = e0 + lane * 8;
  Raw8<T, RESID> xg;
  if (J.vector_ok(e0, min(hi, e0 + kGroup), kGroup))
    J.load_full(e, xg);
  else
    J.load(e, hi, xg);
  float w[8], pw[8], xa[8];
  J.weights(xg, w, pw);
  xg.a.unpack(xa);
  double mine = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) mine += static_cast<double>(w[k]);
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  const unsigned hit = __ballot_sync(0xffffffffu, base + incl > target);
  const unsigned pos = __ballot_sync(0xffffffffu, mine > 0.0);
  if (pos == 0u) {
    *la = 0.0f;
    return -1;
  }
  // rounding can leave no lane crossing: the group's last positive element then
  const int src = hit ? __ffs(hit) - 1 : 31 - __clz(pos);
  int yl = -1, lp = -1;
  float lyl = 0.0f, llp = 0.0f;
  double Cl = base + excl;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    Cl += static_cast<double>(w[k]);
    if (w[k] > 0.0f) { lp = k; llp = xa[k]; }
    if (yl < 0 && w[k] > 0.0f && Cl > target) { yl = k; lyl = xa[k]; }
  }
  if (yl < 0) { yl = lp; lyl = llp; }
  *la = __shfl_sync(0xffffffffu, lyl, src);
  return __shfl_sync(0xffffffffu, e + yl, src);
}

// Warp-level draw inside one chunk [lo, hi) (hi - lo <= kChunkElems, lo a multiple of 8):
// `base` is the weight before lo and `target` = u * Z. A whole batch of groups is in flight
// at once; the group totals locate the 256-element group whose prefix crosses target, which
// warp_draw_group then walks (its data comes again from L1/L2). Returns the first index
// whose inclusive prefix exceeds target, else (rounding) the last index with positive
// weight, or -1 if the chunk has no positive weight; *la receives row a's logit there.
template <typename T, bool RESID>
__device__ int warp_draw_chunk(const JobRows<T, RESID>& J, int lo, int hi, double base, double target, float* la) {
  constexpr int NB = kChunkBatch<T, RESID>;
  const int lane = threadIdx.x & 31;
  const bool full = J.vector_ok(lo, hi, kChunkElems);
  double C = base, cG = 0.0;
  int last = -1, G = -1;
#pragma unroll 1
  for (int g0 = 0; g0 < kChunkGroups && G < 0; g0 += NB) {
    double gs[NB];
    {
      Raw8<T, RESID> x[NB];
      if (full) {
#pragma unroll
        for (int g = 0; g < NB; ++g) J.load_full(lo + (g0 + g) * kGroup + lane * 8, x[g]);
      } else {
#pragma unroll
        for (int g = 0; g < NB; ++g) J.load(lo + (g0 + g) * kGroup + lane * 8, hi, x[g]);
      }
#pragma unroll
      for (int g = 0; g < NB; ++g) gs[g] = lane_group_weight(J, x[g], lo + (g0 + g) * kGroup + lane * 8, &last);
    }
#pragma unroll
    for (int g = 0; g < NB; ++g) gs[g] = warp_sum(gs[g]);
    // the group whose prefix crosses target (every lane computes the same)
#pragma unroll
    for (int g = 0; g < NB; ++g) {
      if (G < 0 && gs[g] > 0.0 && C + gs[g] > target) {
        G = g0 + g;
        cG = C;
      }
      C += gs[g];
    }
  }
  if (G < 0) {
    // rounding put target past the chunk's total: its last positive element
    const int y = __reduce_max_sync(0xffffffffu, last);
    *la = y >= 0 ? J.logit_a(y) : 0.0f;
    return y;
  }
  return warp_draw_group(J, lo + G * kGroup, hi, cG, target, la);
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
