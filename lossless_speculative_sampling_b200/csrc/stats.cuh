// stats.cuh -- per-row distribution statistics: maximum, softmax normaliser, top-p threshold.
//
// A row's distribution after temperature T and top-p (review page of arXiv 2609.04010,
// section 3.3: p_AR and p_draft are full-vocabulary next-token distributions; README
// inference flags --temperature/--top-p) is summarised by RowStat: the maximum m, c =
// log2(e)/T, the normaliser s = sum 2^((l - m) c), the top-p threshold key tau and the kept
// normaliser s_kept. Any probability of the row is then one ex2 away.
//
// Two kernels:
//   row_partial_kernel  one CTA per (row, slice of kSliceElems): streaming online max/sum
//                       with 16-byte vector loads (greedy rows: max and lowest argmax);
//   row_finalize_kernel one CTA per row: combines the slice partials and, when top-p is on,
//                       finds tau by a most-significant-digit radix select over the keys,
//                       accumulating probability mass per digit.
#pragma once

#include "common.cuh"

namespace psi {

// Online max/sum over [v0, v1) of one row, per thread. The vector body batches kBatch
// 16-byte loads before using them (memory-level parallelism) and sums weights per vector in
// fp32, accumulating vector sums with a compensated (Kahan) fp32 sum: ~1 ulp overall without
// fp64 work in the loop.
constexpr int kBatch = 4;

template <typename T, bool GREEDY>
__device__ __forceinline__ void thread_slice_stats(const T* __restrict__ row, int v0, int v1, float c, float& m,
                                                   double& s_out, int& amax, bool& bad) {
  constexpr int N = Vec<T>::N;
  int a0, a1;
  vec_range(row, v0, v1, a0, a1);
  float s = 0.0f, comp = 0.0f;
  auto add = [&](float y) {  // compensated s += y
    y -= comp;
    const float t = s + y;
    comp = (t - s) - y;
    s = t;
  };
  auto rescale = [&](float nm) {
    const float f = ex2((m - nm) * c);
    s *= f;
    comp *= f;
    m = nm;
  };
  auto scalar = [&](int v) {
    float x = load_elem(row + v);
    bad |= !(x < INFINITY);
    if (GREEDY) {
      if (x > m) { m = x; amax = v; }
    } else {
      if (x > m) rescale(x);
      if (m > -INFINITY) add(ex2((x - m) * c));
    }
  };
  // head and tail elements (fewer than N each), then the aligned body
  for (int v = v0 + threadIdx.x; v < a0; v += blockDim.x) scalar(v);
  for (int v = a1 + threadIdx.x; v < v1; v += blockDim.x) scalar(v);
  const int stride = blockDim.x * N;
  for (int vb = a0 + threadIdx.x * N; vb < a1; vb += kBatch * stride) {
    float f[kBatch][8];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (vb + u * stride < a1) Vec<T>::load(row + vb + u * stride, f[u]);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = vb + u * stride;
      if (v >= a1) break;
      float vmax = f[u][0];
#pragma unroll
      for (int k = 1; k < N; ++k) vmax = fmax_nan(vmax, f[u][k]);
      bad |= !(vmax < INFINITY);
      if (GREEDY) {
        if (vmax > m) {
#pragma unroll
          for (int k = N - 1; k >= 0; --k)
            if (f[u][k] == vmax) amax = v + k;
          m = vmax;
        }
      } else {
        if (vmax > m) rescale(vmax);
        if (m > -INFINITY) {
          float acc = 0.0f;
#pragma unroll
          for (int k = 0; k < N; ++k) acc += ex2((f[u][k] - m) * c);
          add(acc);
        }
      }
    }
  }
  s_out = static_cast<double>(s) - static_cast<double>(comp);
}

__device__ __forceinline__ float temp_scale(float T) {
  return T > 0.0f && T < INFINITY ? static_cast<float>(1.4426950408889634 / static_cast<double>(T)) : 0.0f;
}

// Request of a row: rows_per_req consecutive rows per request, or an explicit table.
__device__ __forceinline__ int row_request(int row, int rows_per_req, const int32_t* __restrict__ row_req) {
  return row_req ? row_req[row] : row / rows_per_req;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) row_partial_kernel(const T* __restrict__ base, int rows_per_req,
                                                                const int32_t* __restrict__ row_req, int V,
                                                                int nslices, const float* __restrict__ temperature,
                                                                Partial* __restrict__ out) {
  __shared__ float red[32];
  __shared__ double dred[33];
  __shared__ int ired[32];
  const int unit = blockIdx.x;
  const int row = unit / nslices, slice = unit - row * nslices;
  const float c = temp_scale(temperature[row_request(row, rows_per_req, row_req)]);
  const T* rp = base + static_cast<size_t>(row) * V;
  const int v0 = slice * kSliceElems, v1 = min(V, v0 + kSliceElems);
  float m = -INFINITY;
  double s = 0.0;
  int amax = 0x7fffffff;
  bool bad = false;
  if (c == 0.0f) {
    thread_slice_stats<T, true>(rp, v0, v1, c, m, s, amax, bad);
    float M = block_max(m, red);
    int cand = (m == M) ? amax : 0x7fffffff;
    // lowest index attaining the maximum
    cand = __reduce_min_sync(0xffffffffu, cand);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) ired[threadIdx.x >> 5] = cand;
    __syncthreads();
    if (threadIdx.x < 32) {
      int x = threadIdx.x < (blockDim.x >> 5) ? ired[threadIdx.x] : 0x7fffffff;
      x = __reduce_min_sync(0xffffffffu, x);
      if (threadIdx.x == 0) ired[0] = x;
    }
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) out[unit] = Partial{0.0, M, ired[0], bad ? 1 : 0, 0};
  } else {
    thread_slice_stats<T, false>(rp, v0, v1, c, m, s, amax, bad);
    float M = block_max(m, red);
    double mine = (m > -INFINITY) ? s * static_cast<double>(ex2((m - M) * c)) : 0.0;
    double S = block_sum(mine, dred);
    bad = __syncthreads_or(bad);
    if (threadIdx.x == 0) out[unit] = Partial{S, M, 0, bad ? 1 : 0, 0};
  }
}

// Visit every element of row [0, V) with f(x); vectorised body, scalar edges.
template <typename T, typename F>
__device__ __forceinline__ void for_each_elem(const T* __restrict__ row, int V, F&& f) {
  constexpr int N = Vec<T>::N;
  int a0, a1;
  vec_range(row, 0, V, a0, a1);
  for (int v = threadIdx.x; v < a0; v += blockDim.x) f(load_elem(row + v));
  for (int v = a1 + threadIdx.x; v < V; v += blockDim.x) f(load_elem(row + v));
  for (int v = a0 + threadIdx.x * N; v < a1; v += blockDim.x * N) {
    float x[8];
    Vec<T>::load(row + v, x);
#pragma unroll
    for (int k = 0; k < N; ++k) f(x[k]);
  }
}

// One CTA per row. When `jobs` is given (draft sampling), also emits this row's draw job, or
// writes the token directly for greedy and bad rows.
template <typename T>
__global__ void __launch_bounds__(kThreads) row_finalize_kernel(
    const T* __restrict__ base, int rows_per_req, const int32_t* __restrict__ row_req, int V, int nslices,
    const float* __restrict__ temperature, const float* __restrict__ top_p, const Partial* __restrict__ parts,
    RowStat* __restrict__ stats,
    const float* __restrict__ u, Job* __restrict__ jobs, int32_t* __restrict__ out_tokens,
    float* __restrict__ out_q) {
  __shared__ double hmass[256];
  __shared__ int hcnt[256];
  __shared__ RowStat st;
  __shared__ uint32_t sh_prefix;
  __shared__ double sh_above, sh_bucket;
  const int row = blockIdx.x, req = row_request(row, rows_per_req, row_req);
  const float Tv = temperature[req];
  const float c = temp_scale(Tv);
  const Partial* pp = parts + static_cast<size_t>(row) * nslices;

  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float M = -INFINITY;
    bool bad = !(Tv >= 0.0f && Tv < INFINITY);
    for (int i = lane; i < nslices; i += 32) {
      M = fmax_nan(M, pp[i].m);
      bad |= pp[i].bad != 0;
    }
    M = warp_max(M);
    double S = 0.0;
    int amax = 0x7fffffff;
    for (int i = lane; i < nslices; i += 32) {
      Partial q = pp[i];
      if (c != 0.0f) {
        if (q.m > -INFINITY) S += q.s * static_cast<double>(ex2((q.m - M) * c));
      } else if (q.m == M) {
        amax = min(amax, q.amax);
      }
    }
    S = warp_sum(S);
    amax = __reduce_min_sync(0xffffffffu, amax);
    bad = __any_sync(0xffffffffu, bad) || !(M > -INFINITY) || !(M < INFINITY);
    if (lane == 0) {
      st.m = M;
      st.c = c;
      st.s = c != 0.0f ? static_cast<float>(S) : 1.0f;
      st.s_kept = st.s;
      st.tau = 0u;
      st.amax = c != 0.0f ? -1 : amax;
      st.status = bad ? 1 : 0;
      st.pad = 0;
    }
  }
  __syncthreads();

  const float tp = top_p[req];
  if (st.status == 0 && st.c != 0.0f && tp < 1.0f) {
    // Top-p threshold: radix select on the 32-bit keys, most significant digit first. For
    // bf16 rows the two top digits already separate every distinct value.
    const T* rp = base + static_cast<size_t>(row) * V;
    const float M = st.m;
    const double target = static_cast<double>(tp) * static_cast<double>(st.s);
    const int levels = sizeof(T) == 2 ? 2 : 4;
    if (threadIdx.x == 0) { sh_prefix = 0u; sh_above = 0.0; sh_bucket = 0.0; }
    for (int lv = 0; lv < levels; ++lv) {
      const int shift = 24 - 8 * lv;
      for (int d = threadIdx.x; d < 256; d += blockDim.x) { hmass[d] = 0.0; hcnt[d] = 0; }
      __syncthreads();
      const uint32_t prefix = sh_prefix;
      for_each_elem(rp, V, [&](float x) {
        uint32_t k = fkey(x);
        if (lv == 0 || (k >> (shift + 8)) == (prefix >> (shift + 8))) {
          int d = (k >> shift) & 255;
          atomicAdd(&hmass[d], static_cast<double>(ex2((x - M) * c)));
          atomicAdd(&hcnt[d], 1);
        }
      });
      __syncthreads();
      if (threadIdx.x == 0) {
        double running = sh_above;
        int pick = -1;
        for (int d = 255; d >= 0; --d) {
          if (hcnt[d] == 0) continue;
          if (running + hmass[d] >= target) { pick = d; break; }
          running += hmass[d];
        }
        if (pick < 0) {  // rounding left the target unreached: keep the whole candidate range
          running = sh_above;
          for (int d = 255; d >= 0; --d)
            if (hcnt[d] != 0) { pick = d; running += hmass[d]; }
          running -= hmass[pick];
        }
        sh_prefix = prefix | (static_cast<uint32_t>(pick) << shift);
        sh_above = running;
        sh_bucket = hmass[pick];
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) {
      st.tau = sh_prefix;
      st.s_kept = static_cast<float>(sh_above + sh_bucket);
    }
    __syncthreads();
  }

  if (threadIdx.x == 0) {
    stats[row] = st;
    if (jobs != nullptr) {
      Job jb{kNone, row, -1, row, u[row], row, {0, 0}};
      if (st.status != 0) {
        out_tokens[row] = -1;
        if (out_q) out_q[row] = -1.0f;
      } else if (st.c == 0.0f) {
        out_tokens[row] = st.amax;
        if (out_q) out_q[row] = 1.0f;
      } else {
        jb.mode = kSample;
      }
      jobs[row] = jb;
    }
  }
}

}  // namespace psi
