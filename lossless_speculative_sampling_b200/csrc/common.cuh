// common.cuh -- device helpers shared by the Psi-Spec kernels (sm_100a).
//
// Arithmetic conventions of the CUDA path:
//   * a logit l of a row with statistics (m, c) has weight w = 2^((l - m) * c), c = log2(e)/T,
//     evaluated with the hardware ex2.approx instruction (ftz); m is the row maximum, so
//     every weight is in [0, 1];
//   * weights are summed in fp32 over one 16-byte vector (at most 8 terms) and accumulated in
//     fp64 from there on (per thread, across threads, across slices, in top-p histograms), so
//     normalisers and CDF totals carry about the ex2 error (~1e-7 relative), not the
//     accumulation error of long fp32 sums;
//   * top-p thresholds are compared on order-preserving 32-bit keys of the logit values, so
//     ties are kept or dropped together.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace psi {

constexpr int kThreads = 256;                               // threads per CTA of the streaming kernels
constexpr int kChunkElems = 2048;                           // contiguous elements per warp (one partial)
constexpr int kSliceElems = kChunkElems * (kThreads / 32);  // elements per CTA work unit

__host__ __device__ inline int nchunks_for(int64_t V) { return static_cast<int>((V + kChunkElems - 1) / kChunkElems); }
__host__ __device__ inline int nslices_for(int64_t V) { return static_cast<int>((V + kSliceElems - 1) / kSliceElems); }

// Per-row statistics record (32 bytes; also the public row-stats record).
struct RowStat {
  float m;         // row maximum
  float c;         // log2(e) / T; 0 means greedy
  float s;         // sum over the row of 2^((l - m) c)
  float s_kept;    // the same sum restricted to the top-p kept set
  uint32_t tau;    // kept <=> key(l) >= tau (0 keeps every token)
  int32_t amax;    // lowest index of the maximum (greedy rows)
  int32_t status;  // 0 ok, 1 data error in this row
  int32_t pad;
};
static_assert(sizeof(RowStat) == 32, "row stats record is 32 bytes");

// Partial statistics of one (row, chunk): a warp's contiguous kChunkElems elements.
struct Partial {
  double s;  // sum of 2^((l - m) c) over the chunk, relative to the chunk's own maximum m
  float m;
  int32_t amax;
  int32_t bad;
  int32_t pad;
};
static_assert(sizeof(Partial) == 24 && offsetof(Partial, m) == 8 && offsetof(Partial, bad) == 16, "partial layout");

// Inverse-CDF job: draw from row a of tensor A (mode kSample) or from max(0, pA - qB)
// (mode kResidual), with uniform u; the result goes to out_tokens[out_index]. The job carries
// the statistics of both rows so that a worker needs one load to start.
enum JobMode : int32_t { kNone = 0, kSample = 2, kResidual = 3 };
struct __align__(16) Job {
  int32_t mode;
  int32_t row_a;
  int32_t row_b;
  int32_t out_index;
  float u;
  int32_t pad[3];
  RowStat sa;  // statistics of row a
  RowStat sb;  // statistics of row b (residual jobs)
};
static_assert(sizeof(Job) == 96 && offsetof(Job, sa) == 32 && offsetof(Job, sb) == 64, "job record layout");

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// maximum that propagates NaN (so a NaN logit poisons the row statistics)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float y;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
  return y;
}

// Two fp32 values in one 64-bit register, for the packed sm_100 fp32x2 arithmetic. The
// packed operations round every lane exactly like their scalar counterparts.
using f32x2 = unsigned long long;
__device__ __forceinline__ f32x2 pack2(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack2(f32x2 r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^((x_k - m) c) for the 8 values of x, in the same arithmetic as kept_weight (x - m
// rounded, then the product rounded, then ex2).
__device__ __forceinline__ void exp8(const float (&x)[8], float m, float c, float (&w)[8]) {
  const f32x2 mm = pack2(m, m), cc = pack2(c, c);
#pragma unroll
  for (int k = 0; k < 8; k += 2) {
    float a, b;
    unpack2(mul2(sub2(pack2(x[k], x[k + 1]), mm), cc), a, b);
    w[k] = ex2(a);
    w[k + 1] = ex2(b);
  }
}

// Sum of 8 values as four packed pair sums then two scalar adds (a fixed association).
__device__ __forceinline__ float sum8(const float (&w)[8]) {
  const f32x2 s = add2(add2(pack2(w[0], w[1]), pack2(w[2], w[3])), add2(pack2(w[4], w[5]), pack2(w[6], w[7])));
  float a, b;
  unpack2(s, a, b);
  return a + b;
}

// A row-statistics record from its two 16-byte words.
__device__ __forceinline__ RowStat stat_from(const int4& a, const int4& b) {
  RowStat s;
  s.m = __int_as_float(a.x);
  s.c = __int_as_float(a.y);
  s.s = __int_as_float(a.z);
  s.s_kept = __int_as_float(a.w);
  s.tau = static_cast<uint32_t>(b.x);
  s.amax = b.y;
  s.status = b.z;
  s.pad = b.w;
  return s;
}

// A row-statistics record written by another CTA of the running kernel (read through L2).
__device__ __forceinline__ RowStat load_stat_cg(const RowStat* p) {
  const int4* q = reinterpret_cast<const int4*>(p);
  return stat_from(__ldcg(q), __ldcg(q + 1));
}

// A job record written by another CTA or an earlier kernel (read through L2).
__device__ __forceinline__ Job load_job_cg(const Job* p) {
  const int4* q = reinterpret_cast<const int4*>(p);
  const int4 h = __ldcg(q), g = __ldcg(q + 1), a0 = __ldcg(q + 2), a1 = __ldcg(q + 3), b0 = __ldcg(q + 4),
             b1 = __ldcg(q + 5);
  Job j;
  j.mode = h.x;
  j.row_a = h.y;
  j.row_b = h.z;
  j.out_index = h.w;
  j.u = __int_as_float(g.x);
  j.pad[0] = g.y;
  j.pad[1] = g.z;
  j.pad[2] = g.w;
  j.sa = stat_from(a0, a1);
  j.sb = stat_from(b0, b1);
  return j;
}

// Row statistics held by lane `src` of the warp, to every lane.
__device__ __forceinline__ RowStat shfl_stat(const RowStat& s, int src) {
  RowStat r;
  r.m = __shfl_sync(0xffffffffu, s.m, src);
  r.c = __shfl_sync(0xffffffffu, s.c, src);
  r.s = __shfl_sync(0xffffffffu, s.s, src);
  r.s_kept = __shfl_sync(0xffffffffu, s.s_kept, src);
  r.tau = __shfl_sync(0xffffffffu, s.tau, src);
  r.amax = __shfl_sync(0xffffffffu, s.amax, src);
  r.status = __shfl_sync(0xffffffffu, s.status, src);
  r.pad = __shfl_sync(0xffffffffu, s.pad, src);
  return r;
}

// order-preserving key of a float; -0 and +0 share one key
__device__ __forceinline__ uint32_t fkey(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ bool is_finite(float x) { return fabsf(x) <= 3.402823466e38f; }

__device__ __forceinline__ float load_elem(const float* p) { return __ldg(p); }
// element load through a generic pointer (global or shared memory)
__device__ __forceinline__ float load_elem_any(const float* p) { return *p; }
__device__ __forceinline__ float load_elem_any(const __nv_bfloat16* p) {
  return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(p)) << 16);
}
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p) {
  unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(p));
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// 16-byte vector of elements
template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static void load(const float* p, float (&f)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), f);
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xFFFF0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xFFFF0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xFFFF0000u);
  }
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), f);
  }
};

// The aligned vector range of [v0, v1) within a row: [a0, a1) with a0 - v0 < N elements.
template <typename T>
__device__ __forceinline__ void vec_range(const T* row, int v0, int v1, int& a0, int& a1) {
  constexpr int N = Vec<T>::N;
  uintptr_t addr = reinterpret_cast<uintptr_t>(row + v0);
  int head = static_cast<int>(((16u - (addr & 15u)) & 15u) / sizeof(T));
  a0 = min(v1, v0 + head);
  a1 = a0 + ((v1 - a0) / N) * N;
}

// The float whose order key is `key` (the inverse of fkey on keys of actual values).
__device__ __forceinline__ float key_value(uint32_t key) {
  return (key & 0x80000000u) ? __uint_as_float(key & 0x7FFFFFFFu) : __uint_as_float(~key);
}

// Smallest kept logit value of a threshold key as a float bound: l is kept iff
// l >= cut_value(tau), which equals fkey(l) >= tau for every non-NaN l. A key at or below the
// key of -inf (0 included, and the 16-bit prefix 0x007F0000 a bf16 select leaves for -inf,
// whose inverse bits would be a NaN) keeps every value.
__device__ __forceinline__ float cut_value(uint32_t tau) { return tau <= 0x007FFFFFu ? -INFINITY : key_value(tau); }

// Weight of logit l under row statistics st (kept set applied); greedy rows are handled by
// the callers.
__device__ __forceinline__ float kept_weight(const RowStat& st, float l) {
  const float w = ex2((l - st.m) * st.c);
  return l >= cut_value(st.tau) ? w : 0.0f;
}

// Probability of token v with logit l under st.
__device__ __forceinline__ float prob_of(const RowStat& st, float l, int v) {
  if (st.c == 0.0f) return v == st.amax ? 1.0f : 0.0f;
  return kept_weight(st, l) / st.s_kept;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x = fmax_nan(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Block-wide reductions (blockDim.x a multiple of 32, at most 1024); the result is returned
// to every thread. `scratch` holds at least 32 elements and is reused after a barrier.
__device__ __forceinline__ float block_max(float x, float* scratch) {
  int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  x = warp_max(x);
  __syncthreads();
  if (lane == 0) scratch[warp] = x;
  __syncthreads();
  x = lane < nw ? scratch[lane] : -INFINITY;
  return warp_max(x);
}
__device__ __forceinline__ float block_sum(float x, float* scratch) {
  int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  x = warp_sum(x);
  __syncthreads();
  if (lane == 0) scratch[warp] = x;
  __syncthreads();
  x = lane < nw ? scratch[lane] : 0.0f;
  return warp_sum(x);
}
__device__ __forceinline__ double block_sum(double x, double* scratch) {
  int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  x = warp_sum(x);
  __syncthreads();
  if (lane == 0) scratch[warp] = x;
  __syncthreads();
  x = lane < nw ? scratch[lane] : 0.0;
  return warp_sum(x);
}

// Exclusive prefix sum of one double per thread, in thread order (deterministic).
// `scratch` holds at least 33 doubles; *total receives the block total.
__device__ __forceinline__ double block_exclusive_scan(double x, double* scratch, double* total) {
  int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  double incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  __syncthreads();
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    double w = lane < nw ? scratch[lane] : 0.0;
    double wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      double y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    double we = __shfl_up_sync(0xffffffffu, wi, 1);
    if (lane == 0) we = 0.0;
    if (lane < nw) scratch[lane] = we;
    if (lane == nw - 1) scratch[32] = wi;
  }
  __syncthreads();
  double r = scratch[warp] + excl;
  *total = scratch[32];
  return r;
}

}  // namespace psi
