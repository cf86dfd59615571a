// topp.cuh -- rows of requests with a cut (top-p below 1 or an active top-k, at T > 0):
// statistics, threshold and (draft rows) draw, one CTA per row.
//
// The cut keeps every token whose logit is at least tau, the largest logit value t of the row
// with mass(l >= t) >= top_p (review page of arXiv 2609.04010: the samplers take --top-p
// with --temperature; ties are kept together), and renormalises over the kept set. With a
// top-k (the README's --top-k), the mass and the tail are those of the tokens at or above the
// k-th largest logit, ties included.
//
// A CTA reads its row once from HBM and then, while the row is still in L2:
//   A  maximum m (NaN-propagating; bf16 pairs compared packed);
//   B  value histogram: bin b holds the logits with (x - m) c within 1/4 of -b/2; every element
//      adds its weight relative to the bin's reference weight 2^(-b/2), a number in
//      [2^(-1/4), 2^(1/4)], as a fixed-point integer with 20 fractional bits to a
//      thread-private 32-bit counter (conflict-free shared-memory reductions, exact and
//      order-independent). The bin totals give the normaliser s and the bin holding tau;
//   C  most-significant-digit select on the order-preserving keys of that bin's elements
//      only (6 bits per pass, the same thread-private counters and fixed-point masses): tau
//      exactly, and the kept mass;
//   D  (draft rows) per-chunk totals of the kept weights, then the inverse-CDF draw inside the
//      chunk holding u * Z.
// Rows too long for exact 32-bit counters, or whose threshold lies below the histogram's
// range, take the general radix select (block_topp_radix).
#pragma once

#include "common.cuh"
#include "finish.cuh"
#include "linear.cuh"
#include "sample.cuh"
#include "stats.cuh"

namespace psi {

// One to the shared-memory counter p[o] when o < n, as a predicated reduction (no branch;
// p + o is not formed into an access otherwise). It declares no memory effect, so that the
// compiler can schedule loads and arithmetic around it: callers order every other access to
// the counters with a barrier (__syncthreads or __syncwarp) between them and the reductions.
__device__ __forceinline__ void count_if_below(uint32_t* p, uint32_t o, uint32_t n) {
  asm volatile(
      "{\n"
      " .reg .pred q;\n"
      " setp.lt.u32 q, %1, %2;\n"
      " @q red.shared.add.u32 [%0], 1;\n"
      "}" ::"r"(smem_u32(p) + 4u * o),
      "r"(o), "r"(n));
}

constexpr int kTpThreads = 256;
constexpr int kTpWarps = kTpThreads / 32;
constexpr int kTpBins = 64;                                  // half log2 units below the maximum
constexpr int kTpMaxV = kTpThreads * 2048;                   // counters stay below 2^32 up to this V
constexpr int kTpMaxChunks = (kTpMaxV + kChunkElems - 1) / kChunkElems;

struct TpSmem {
  uint32_t priv[kTpBins][kTpThreads];             // thread-private bin (pass B) or digit (pass C) counters
  double mass[kTpBins];                           // bin or digit masses
  double ctot[kTpMaxChunks];                      // kept weight per chunk (pass D)
  float fred[kTpWarps];
  float stage[kTpWarps][256];  // per-warp compaction buffer of pass C
  RowStat st;
  double above, total, target;
  uint32_t prefix;
  int bin, fallback;
  int y, flag;
  double base, tgt;
  int chunk;
  RadixSmem radix;  // the general select
  DrawSmem draw;    // the general draw
};

// Bins and fixed-point masses of a logit pair, packed (identical arithmetic in passes B and
// C). r = -2 (x - m) c + 1.5 * 2^23 rounds to the bin index in its low mantissa bits; values
// too far below the maximum (and -inf) land in the last bin with a zero or negligible mass.
constexpr float kTpMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ f32x2 tp_r2(float x0, float x1, f32x2 mm, f32x2 cc, f32x2& d) {
  d = mul2(sub2(pack2(x0, x1), mm), cc);  // log2 weights, <= 0
  return fma2(d, pack2(-2.0f, -2.0f), pack2(kTpMagic, kTpMagic));
}

__device__ __forceinline__ void tp_bin2(float x0, float x1, f32x2 mm, f32x2 cc, int& b0, int& b1, uint32_t& u0,
                                        uint32_t& u1) {
  f32x2 d;
  const f32x2 r = tp_r2(x0, x1, mm, cc, d);
  float r0, r1, f0, f1, a0, a1, y0, y1;
  unpack2(r, r0, r1);
  b0 = min(__float_as_int(r0) - __float_as_int(kTpMagic), kTpBins - 1);
  b1 = min(__float_as_int(r1) - __float_as_int(kTpMagic), kTpBins - 1);
  unpack2(sub2(r, pack2(kTpMagic, kTpMagic)), f0, f1);
  f0 = fminf(f0, static_cast<float>(kTpBins - 1));
  f1 = fminf(f1, static_cast<float>(kTpBins - 1));
  unpack2(fma2(pack2(f0, f1), pack2(0.5f, 0.5f), d), a0, a1);            // d + b/2
  unpack2(add2(pack2(ex2(a0), ex2(a1)), pack2(8.0f, 8.0f)), y0, y1);      // 8 + 2^(d + b/2)
  u0 = __float_as_uint(y0) - __float_as_uint(8.0f);                       // 2^(d + b/2) * 2^20, rounded
  u1 = __float_as_uint(y1) - __float_as_uint(8.0f);
}

// Visit this thread's elements of row [0, V): f8(x) for every 8-element vector of the aligned
// body (kLoads 16-byte loads in flight), f8 with -inf padding for the scalar edges.
template <typename T, int kLoads, typename F>
__device__ __forceinline__ void tp_for_each8(const T* __restrict__ row, int V, F&& f8) {
  constexpr int N = Vec<T>::N;
  int a0, a1;
  vec_range(row, 0, V, a0, a1);
  for (int v = threadIdx.x; v < a0; v += blockDim.x) {
    float x[8] = {load_elem(row + v), -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
    f8(x);
  }
  for (int v = a1 + threadIdx.x; v < V; v += blockDim.x) {
    float x[8] = {load_elem(row + v), -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
    f8(x);
  }
  const int step = blockDim.x * N;
  for (int v = a0 + threadIdx.x * N; v < a1; v += kLoads * step) {
    uint4 raw[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i)
      if (v + i * step < a1) raw[i] = __ldcg(reinterpret_cast<const uint4*>(row + v + i * step));
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      if (v + i * step < a1) {
        float x[8];
        Vec<T>::unpack(raw[i], x);
        if constexpr (N == 4) {
#pragma unroll
          for (int k = 4; k < 8; ++k) x[k] = -INFINITY;
        }
        f8(x);
      }
    }
  }
}

// 2^(-b/2) * 2^-20 in fp64: the weight of one fixed-point unit of bin b.
__device__ __forceinline__ double tp_unit(int b) {
  return ldexp((b & 1) ? 0.70710678118654752440 : 1.0, -(b >> 1) - 20);
}

// Visit the elements of row [0, V) of this thread: f(x) per element; 16-byte vector loads,
// kLoads of them in flight.
template <typename T, int kLoads, typename F>
__device__ __forceinline__ void tp_for_each(const T* __restrict__ row, int V, F&& f) {
  constexpr int N = Vec<T>::N;
  int a0, a1;
  vec_range(row, 0, V, a0, a1);
  for (int v = threadIdx.x; v < a0; v += blockDim.x) f(load_elem(row + v));
  for (int v = a1 + threadIdx.x; v < V; v += blockDim.x) f(load_elem(row + v));
  const int step = blockDim.x * N;
  for (int v = a0 + threadIdx.x * N; v < a1; v += kLoads * step) {
    uint4 raw[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i)
      if (v + i * step < a1) raw[i] = __ldcg(reinterpret_cast<const uint4*>(row + v + i * step));
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      if (v + i * step < a1) {
        float x[8];
        Vec<T>::unpack(raw[i], x);
#pragma unroll
        for (int k = 0; k < N; ++k) f(x[k]);
      }
    }
  }
}

// Pass A: NaN-propagating maximum of the row (every thread gets it).
template <typename T>
__device__ float tp_row_max(const T* __restrict__ row, int V, TpSmem& sm) {
  constexpr int N = Vec<T>::N;
  constexpr int kLoads = 4;
  int a0, a1;
  vec_range(row, 0, V, a0, a1);
  float m = -INFINITY;
  for (int v = threadIdx.x; v < a0; v += blockDim.x) m = fmax_nan(m, load_elem(row + v));
  for (int v = a1 + threadIdx.x; v < V; v += blockDim.x) m = fmax_nan(m, load_elem(row + v));
  const int step = blockDim.x * N;
  uint32_t pm = 0xFF80FF80u;  // packed bf16 pair (-inf, -inf)
  for (int v = a0 + threadIdx.x * N; v < a1; v += kLoads * step) {
    uint4 raw[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i)
      if (v + i * step < a1) raw[i] = __ldg(reinterpret_cast<const uint4*>(row + v + i * step));
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      if (v + i * step < a1) {
        if constexpr (sizeof(T) == 2) {
          pm = bmax2(pm, bmax2(bmax2(raw[i].x, raw[i].y), bmax2(raw[i].z, raw[i].w)));
        } else {
          m = fmax_nan(m, fmax_nan(fmax_nan(__uint_as_float(raw[i].x), __uint_as_float(raw[i].y)),
                                   fmax_nan(__uint_as_float(raw[i].z), __uint_as_float(raw[i].w))));
        }
      }
    }
  }
  if constexpr (sizeof(T) == 2) m = fmax_nan(m, fmax_nan(__uint_as_float(pm << 16), __uint_as_float(pm & 0xFFFF0000u)));
  m = warp_max(m);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sm.fred[threadIdx.x >> 5] = m;
  __syncthreads();
  float r = sm.fred[0];
  for (int w = 1; w < kTpWarps; ++w) r = fmax_nan(r, sm.fred[w]);
  return r;
}

// Passes A-C for one row: its statistics with the top-p threshold (every thread gets them).
template <typename T>
__device__ RowStat tp_row_stats(const T* __restrict__ row, int V, float Tv, float tp, TpSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  RowStat st;
  st.c = temp_scale(Tv);
  st.m = tp_row_max(row, V, sm);
  st.s = 1.0f;
  st.s_kept = 1.0f;
  st.tau = 0u;
  st.amax = -1;
  st.pad = 0;
  st.status = (st.m > -INFINITY && st.m < INFINITY && Tv >= 0.0f && Tv < INFINITY) ? 0 : 1;
  if (st.status != 0) return st;
  const float m = st.m, c = st.c;
  if (V > kTpMaxV) {
    // general path: normaliser by a block reduction, then the general select
    double s = 0.0;
    tp_for_each8<T, 4>(row, V, [&](const float (&x)[8]) {
      float g = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) g += ex2((x[k] - m) * c);
      s += static_cast<double>(g);
    });
    __syncthreads();
    s = block_sum(s, reinterpret_cast<double*>(&sm.mass[0]));
    st.s = static_cast<float>(s);
    block_topp_radix<T>(row, V, tp, st, sm.radix);
    return st;
  }
  // pass B: thread-private fixed-point bin masses
#pragma unroll
  for (int b = 0; b < kTpBins; ++b) sm.priv[b][threadIdx.x] = 0u;
  const f32x2 mm = pack2(m, m), cc = pack2(c, c);
  tp_for_each8<T, 4>(row, V, [&](const float (&x)[8]) {
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      int b0, b1;
      uint32_t u0, u1;
      tp_bin2(x[k], x[k + 1], mm, cc, b0, b1, u0, u1);
      // reductions (no return value): no dependence chain through shared memory
      if (u0 != 0u) atomicAdd(&sm.priv[b0][threadIdx.x], u0);
      if (u1 != 0u) atomicAdd(&sm.priv[b1][threadIdx.x], u1);
    }
  });
  __syncthreads();
  // bin totals: warp w reduces bins w, w + kTpWarps, ...
  for (int b = warp; b < kTpBins; b += kTpWarps) {
    unsigned long long t = 0ull;
    for (int j = lane; j < kTpThreads; j += 32) t += sm.priv[b][j];
#pragma unroll
    for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) sm.mass[b] = static_cast<double>(t) * tp_unit(b);
  }
  __syncthreads();
  if (warp == 0) {
    static_assert(kTpBins == 64, "two bins per lane");
    const double m0 = sm.mass[2 * lane], m1 = sm.mass[2 * lane + 1];
    const double mine = m0 + m1;
    double incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const double total = __shfl_sync(0xffffffffu, incl, 31);
    const double target = static_cast<double>(tp) * total;
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= target && mine > 0.0);
    const unsigned pos = __ballot_sync(0xffffffffu, mine > 0.0);
    const int src = hit ? __ffs(hit) - 1 : 31 - __clz(pos);
    if (lane == src) {
      int pick;
      double before;
      if (m0 > 0.0 && (excl + m0 >= target || m1 <= 0.0)) {
        pick = 2 * lane;
        before = excl;
      } else {
        pick = 2 * lane + 1;
        before = excl + m0;
      }
      sm.bin = pick;
      sm.above = before;
      sm.total = total;
      sm.target = target;
      sm.prefix = 0u;
      sm.fallback = pick == kTpBins - 1;
    }
  }
  __syncthreads();
  st.s = static_cast<float>(sm.total);
  if (sm.fallback) {
    block_topp_radix<T>(row, V, tp, st, sm.radix);
    return st;
  }
  // pass C: inside bin b*, most-significant-digit select on the element keys, 6 bits of
  // (key - klo) per pass, with the thread-private counters of pass B. [klo, khi] covers the
  // bin's value range widened by a few representable values; an element of the bin outside
  // it (which the widening rules out) sends the row to the general select.
  const int bstar = sm.bin;
  const double unit = tp_unit(bstar);
  constexpr int kKeyShift = sizeof(T) == 2 ? 16 : 0;  // bf16 logits differ in the top 16 key bits only
  const float xlo = m - (static_cast<float>(bstar) + 0.51f) / (2.0f * c);
  const float xhi = bstar == 0 ? m : m - (static_cast<float>(bstar) - 0.51f) / (2.0f * c);
  const uint32_t klo0 = fkey(xlo) >> kKeyShift, khi0 = fkey(xhi) >> kKeyShift;
  const uint32_t klo = klo0 > 2u ? klo0 - 2u : 0u;
  const uint32_t kmax = sizeof(T) == 2 ? 0xFFFFu : 0xFFFFFFFFu;
  const uint32_t khi = khi0 < kmax - 2u ? khi0 + 2u : kmax;
  const uint32_t span = khi - klo;  // largest offset
  int levels = 1;
  while (levels < 6 && (span >> (6 * levels)) != 0u) ++levels;
  uint32_t prefix = 0u;  // digits chosen so far (offset >> (6 * remaining levels))
  bool outside = false;
  for (int lv = 0; lv < levels; ++lv) {
    const int shift = 6 * (levels - 1 - lv);
#pragma unroll
    for (int d = 0; d < 64; ++d) sm.priv[d][threadIdx.x] = 0u;
    const float rstar = kTpMagic + static_cast<float>(bstar);  // r of the elements of bin b*
    // an element of bin b*: its fixed-point mass goes to the counter of its digit
    auto add = [&](float x) {
      const uint32_t kk = fkey(x) >> kKeyShift;
      if (kk < klo || kk > khi) {
        outside = true;
        return;
      }
      const uint32_t off = kk - klo;
      if (shift + 6 < 32 && (off >> (shift + 6)) != prefix) return;
      int b0, b1;
      uint32_t u0, u1;
      tp_bin2(x, -INFINITY, mm, cc, b0, b1, u0, u1);
      atomicAdd(&sm.priv[(off >> shift) & 63u][threadIdx.x], u0);
    };
    {
      constexpr int N = Vec<T>::N;
      constexpr int kLoads = 4;
      int a0, a1;
      vec_range(row, 0, V, a0, a1);
      for (int v = threadIdx.x; v < a0; v += blockDim.x) {  // scalar edges: few elements
        const float x = load_elem(row + v);
        f32x2 d;
        float r0, r1;
        unpack2(tp_r2(x, -INFINITY, mm, cc, d), r0, r1);
        if (r0 == rstar) add(x);
      }
      for (int v = a1 + threadIdx.x; v < V; v += blockDim.x) {
        const float x = load_elem(row + v);
        f32x2 d;
        float r0, r1;
        unpack2(tp_r2(x, -INFINITY, mm, cc, d), r0, r1);
        if (r0 == rstar) add(x);
      }
      // vector body in rounds every lane takes part in: the lanes flag the elements of bin b*,
      // the warp compacts them into its staging buffer and shares the work on them evenly
      const int nvec = (a1 - a0) / N;
      const int rounds = (nvec + kTpThreads - 1) / kTpThreads;
      float* stage = sm.stage[warp];
      for (int r0i = 0; r0i < rounds; r0i += kLoads) {
        uint4 raw[kLoads];
#pragma unroll
        for (int i = 0; i < kLoads; ++i) {
          const int vi = (r0i + i) * kTpThreads + threadIdx.x;
          if (r0i + i < rounds && vi < nvec) raw[i] = __ldcg(reinterpret_cast<const uint4*>(row + a0 + vi * N));
        }
#pragma unroll
        for (int i = 0; i < kLoads; ++i) {
          if (r0i + i >= rounds) break;  // uniform: every thread runs the same rounds
          const int vi = (r0i + i) * kTpThreads + threadIdx.x;
          float x[8];
          uint32_t mask = 0u;
          if (vi < nvec) {
            Vec<T>::unpack(raw[i], x);
#pragma unroll
            for (int k = 0; k < N; k += 2) {
              f32x2 d;
              float ra, rb;
              unpack2(tp_r2(x[k], x[k + 1], mm, cc, d), ra, rb);
              mask |= (ra == rstar ? 1u : 0u) << k;
              mask |= (rb == rstar ? 1u : 0u) << (k + 1);
            }
          }
          const int cnt = __popc(mask);
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const int total = __shfl_sync(0xffffffffu, incl, 31);
          if (total == 0) continue;
          int pos = incl - cnt;
#pragma unroll
          for (int k = 0; k < N; ++k)
            if (mask & (1u << k)) stage[pos++] = x[k];
          __syncwarp();
          for (int j = lane; j < total; j += 32) add(stage[j]);
          __syncwarp();
        }
      }
    }
    if (__syncthreads_or(outside)) {
      if (threadIdx.x == 0) sm.fallback = 1;
      break;
    }
    for (int d = warp; d < 64; d += kTpWarps) {
      unsigned long long t = 0ull;
      for (int j = lane; j < kTpThreads; j += 32) t += sm.priv[d][j];
#pragma unroll
      for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) sm.mass[d] = static_cast<double>(t) * unit;
    }
    __syncthreads();
    if (warp == 0) {
      // digits from the largest key down: lane l holds digits 63 - 2l and 62 - 2l
      const double m0 = sm.mass[63 - 2 * lane], m1 = sm.mass[62 - 2 * lane];
      const double mine = m0 + m1;
      double incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      double excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.0;
      const double above = sm.above, target = sm.target;
      const unsigned hit = __ballot_sync(0xffffffffu, above + incl >= target && mine > 0.0);
      const unsigned pos = __ballot_sync(0xffffffffu, mine > 0.0);
      // rounding can leave the target unreached: the bin's smallest key with mass then
      const int src = hit ? __ffs(hit) - 1 : 31 - __clz(pos);
      if (lane == src) {
        int pick;
        double before;
        if (m0 > 0.0 && (above + excl + m0 >= target || m1 <= 0.0)) {
          pick = 63 - 2 * lane;
          before = above + excl;
        } else {
          pick = 62 - 2 * lane;
          before = above + excl + m0;
        }
        sm.bin = pick;  // the chosen digit
        sm.above = before;
        sm.base = before + (pick == 63 - 2 * lane ? m0 : m1);
      }
    }
    __syncthreads();
    prefix = (prefix << 6) | static_cast<uint32_t>(sm.bin);
  }
  if (sm.fallback) {
    __syncthreads();
    block_topp_radix<T>(row, V, tp, st, sm.radix);
    return st;
  }
  st.tau = (klo + prefix) << kKeyShift;
  st.s_kept = static_cast<float>(sm.base);
  __syncthreads();
  return st;
}

// The value window of a bf16 row: every element with the same logit has the same weight, so
// counting the elements of each of the kTpWindow representable values just below the row
// maximum m gives their masses exactly (count times one weight), and the cut is the first value,
// from m down, at which the cumulative mass reaches top_p * s (window_pick).
constexpr int kTpWindow = 2048;

// The logit value of a 16-bit order key of a bf16 number (the inverse of fkey(x) >> 16 on
// bf16 values: positive keys carry the bits with the sign set, negative keys their complement).
__device__ __forceinline__ float key16_value(uint32_t k16) {
  const uint32_t b16 = (k16 & 0x8000u) ? (k16 & 0x7FFFu) : (~k16 & 0xFFFFu);
  return __uint_as_float(b16 << 16);
}

// The cut from the counts of the kTpWindow values just below the row maximum (key16 km): the
// value of offset o is the bf16 whose 16-bit order key is km - o, and count(o) how many
// elements of the row carry it. Every element with one value has one weight, so the masses
// are count x weight, exact up to the weight's rounding. Top-k: the first offset whose
// cumulative count reaches k bounds the kept set (ties kept together) and its cumulative mass
// is the top-k total s_k; top-p: the first offset (up to that bound) whose cumulative mass
// reaches top_p x s_k (s_k = st.s without top-k). Sets st.tau and st.s_kept and returns true;
// returns false (st untouched) when the window holds less than the goal. Called by every
// thread of an NT-thread block: count(o) is evaluated for offsets [kPer t, kPer t + kPer) by
// thread t (and by thread 0 for the rounding fallback); scan holds 33 doubles of scratch;
// *bin, *tgt and *base are shared scalars.
template <int NT, typename CountAt>
__device__ bool window_pick(uint32_t km, float tp, int k, RowStat& st, CountAt&& count_at, double* scan, int* bin,
                            double* tgt, double* base) {
  constexpr int kPer = kTpWindow / NT;
  static_assert(kPer * NT == kTpWindow, "the window splits evenly over the block");
  double mass[kPer];
  uint32_t cnt8[kPer];
  double tsum = 0.0, tcnt = 0.0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int o = threadIdx.x * kPer + j;
    const uint32_t c = km >= static_cast<uint32_t>(o) ? count_at(o) : 0u;
    cnt8[j] = c;
    mass[j] = 0.0;
    if (c != 0u) mass[j] = static_cast<double>(c) * static_cast<double>(ex2((key16_value(km - o) - st.m) * st.c));
    tsum += mass[j];
    tcnt += static_cast<double>(c);
  }
  double total;
  const double C0 = block_exclusive_scan(tsum, scan, &total);
  // top-k: the offset of the k-th largest element (ties kept together) bounds the kept set;
  // the top-p target is then top_p of the mass at or above it
  int o_lim = kTpWindow - 1;
  double s_k = static_cast<double>(st.s);
  if (k > 0) {
    double count_total;
    const double K0 = block_exclusive_scan(tcnt, scan, &count_total);
    if (!(count_total >= static_cast<double>(k))) return false;  // the k-th value lies below the window
    if (threadIdx.x == 0) *bin = -1;
    __syncthreads();
    if (K0 < static_cast<double>(k) && K0 + tcnt >= static_cast<double>(k)) {
      double run = K0, runm = C0;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        run += static_cast<double>(cnt8[j]);
        runm += mass[j];
        if (run >= static_cast<double>(k)) {
          *bin = threadIdx.x * kPer + j;
          *tgt = runm;
          break;
        }
      }
    }
    __syncthreads();
    o_lim = *bin;
    s_k = *tgt;
    __syncthreads();
    if (o_lim < 0) return false;  // uniform
    if (!(tp < 1.0f)) {  // top-k alone
      st.tau = (km - static_cast<uint32_t>(o_lim)) << 16;
      st.s_kept = static_cast<float>(s_k);
      return true;
    }
  }
  const double target = static_cast<double>(tp) * s_k;
  if (!(total >= target)) return false;  // the threshold lies below the window (uniform)
  if (threadIdx.x == 0) *bin = -1;
  __syncthreads();
  if (C0 < target && C0 + tsum >= target) {  // the thread whose offsets cross the target
    double run = C0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (mass[j] > 0.0 && run + mass[j] >= target) {
        *bin = threadIdx.x * kPer + j;
        *base = run + mass[j];
        break;
      }
      run += mass[j];
    }
  }
  __syncthreads();
  int ostar = *bin;
  if (ostar < 0) {
    // a target of zero (the maximum's value alone), or rounding at a thread boundary: the
    // first offset whose cumulative mass reaches the target, by thread 0
    if (threadIdx.x == 0) {
      double run = 0.0;
      int pick = -1;
      for (int o = 0; o <= o_lim && pick < 0; ++o) {
        const uint32_t c = km >= static_cast<uint32_t>(o) ? count_at(o) : 0u;
        if (c == 0u) continue;
        run += static_cast<double>(c) * static_cast<double>(ex2((key16_value(km - o) - st.m) * st.c));
        if (run >= target) pick = o;
      }
      if (pick < 0 && k > 0) pick = o_lim;  // rounding: the whole top-k set
      *bin = pick;
      *base = run;
    }
    __syncthreads();
    ostar = *bin;
    if (ostar < 0) return false;  // uniform
  }
  if (ostar > o_lim) {  // rounding past the top-k bound: the whole top-k set
    ostar = o_lim;
    if (threadIdx.x == 0) *base = s_k;
    __syncthreads();
  }
  st.tau = (km - static_cast<uint32_t>(ostar)) << 16;
  st.s_kept = static_cast<float>(*base);
  __syncthreads();
  return true;
}

// Statistics of a row of a request with a top-p or top-k cut from the row's chunk partials
// (the fp32 rows; bf16 rows take the one-pass path of cutrow.cuh): the general top-k then top-p
// radix select from the partials' maximum and normaliser, or passes A-C over the row (top-p
// alone). k is the request's top-k (0: off).
template <typename T>
__device__ RowStat tp_row_stats_partials(const T* __restrict__ row, int V, float Tv, float tp, int k,
                                         const Partial* __restrict__ pp, TpSmem& sm) {
  if (threadIdx.x < 32) {
    const RowStat s0 = warp_finalize_pick(pp, nchunks_for(V), Tv, 0.0f, false).st;
    if (threadIdx.x == 0) sm.st = s0;
  }
  __syncthreads();
  RowStat st = sm.st;
  __syncthreads();
  if (st.status != 0) return st;
  if (k > 0) {
    block_topk_topp_radix<T>(row, V, tp, k, st, sm.radix);
    return st;
  }
  return tp_row_stats(row, V, Tv, tp, sm);
}

// Pass D: inverse-CDF draw with uniform u over the kept weights of the row, in vocabulary
// order (the first index whose inclusive prefix exceeds u * Z). Returns the token to every
// thread and, in *q, its kept probability.
template <typename T>
__device__ int tp_row_draw(const T* __restrict__ row, int V, const RowStat& st, float u, TpSmem& sm, float* q) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nch = nchunks_for(V);
  JobRows<T, false> J;
  J.init(row, st, nullptr, st);
  if (V > kTpMaxV) {  // rows beyond the chunk table: the general block draw
    const int y = block_draw_range(J, 0, V, 0.0, -1.0, u, sm.draw);
    *q = y >= 0 ? kept_weight(st, load_elem(row + y)) / st.s_kept : -1.0f;
    return y;
  }
  for (int ch = warp; ch < nch; ch += kTpWarps) {
    const double t = warp_chunk_weight(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems));
    if (lane == 0) sm.ctot[ch] = t;
  }
  __syncthreads();
  if (warp == 0) {
    // lane l owns the contiguous chunks [l q, l q + q)
    const int qn = (nch + 31) / 32;
    const int i0 = min(nch, lane * qn), i1 = min(nch, i0 + qn);
    double mine = 0.0;
    for (int i = i0; i < i1; ++i) mine += sm.ctot[i];
    double incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const double target = static_cast<double>(u) * __shfl_sync(0xffffffffu, incl, 31);
    int sel = -1, last = -1;
    double b = 0.0, C = excl, blast = 0.0;
    bool open = excl <= target && target < incl;
    for (int i = i0; i < i1; ++i) {
      const double w = sm.ctot[i];
      if (w > 0.0) {
        last = i;
        blast = C;
        if (open) {
          sel = i;
          b = C;
          open = !(C + w > target);
        }
      }
      C += w;
    }
    const unsigned who = __ballot_sync(0xffffffffu, sel >= 0);
    int ch;
    if (who) {
      const int src = __ffs(who) - 1;
      ch = __shfl_sync(0xffffffffu, sel, src);
      b = __shfl_sync(0xffffffffu, b, src);
    } else {  // rounding put u * Z past every chunk: the last chunk with positive weight
      ch = __reduce_max_sync(0xffffffffu, last);
      const int owner = __reduce_max_sync(0xffffffffu, (ch >= 0 && last == ch) ? lane : -1);
      b = __shfl_sync(0xffffffffu, blast, owner < 0 ? 0 : owner);
    }
    float ly = 0.0f;
    int y = -1;
    if (ch >= 0) y = warp_draw_chunk(J, ch * kChunkElems, min(V, (ch + 1) * kChunkElems), b, target, &ly);
    if (lane == 0) {
      sm.y = y;
      sm.base = y >= 0 ? static_cast<double>(kept_weight(st, ly) / st.s_kept) : -1.0;
    }
  }
  __syncthreads();
  const int y = sm.y;
  *q = static_cast<float>(sm.base);
  __syncthreads();
  return y;
}

// Whether request r's rows carry a cut (top-p below 1 or an active top-k, at T > 0).
__device__ __forceinline__ bool request_cut(const float* __restrict__ temperature, const float* __restrict__ top_p,
                                            const int32_t* __restrict__ top_k, int r, int V) {
  return temp_scale(temperature[r]) != 0.0f && (top_p[r] < 1.0f || request_k(top_k, r, V) > 0);
}

}  // namespace psi
