// stats.cuh -- per-row distribution statistics: maximum, softmax normaliser, top-p threshold.
//
// A row's distribution after temperature T and top-p (review page of arXiv 2609.04010,
// section 3.3: p_AR and p_draft are full-vocabulary next-token distributions; README
// inference flags --temperature/--top-p) is summarised by RowStat: the maximum m, c =
// log2(e)/T, the normaliser s = sum 2^((l - m) c), the top-p threshold key tau and the kept
// normaliser s_kept. Any probability of the row is then one ex2 away.
//
// Streaming: a warp covers one contiguous chunk of kChunkElems elements of a row with
// coalesced 16-byte loads (lanes take consecutive vectors, kBatch loads in flight per lane)
// and leaves that chunk's partial (maximum and normaliser relative to it, or the lowest
// argmax for greedy rows). Chunk partials are also the prefix totals that a draw uses to find
// the chunk holding u * Z. warp_finalize_row combines a row's chunk partials;
// block_topp_select finds the top-p threshold by a most-significant-digit radix select over
// the keys with the fp64 mass of every digit.
#pragma once

#include "common.cuh"

namespace psi {

constexpr int kBatch = 4;  // 16-byte loads in flight per lane

__device__ __forceinline__ float temp_scale(float T) {
  return T > 0.0f && T < INFINITY ? static_cast<float>(1.4426950408889634 / static_cast<double>(T)) : 0.0f;
}

// Whether a request samples at a positive temperature with no top-p cut: its row statistics
// are then the maximum and the sum alone, which the cluster tree walk computes itself on the
// rows it visits. (Calls with a top-k array do not use this: every row is finalized.)
__device__ __forceinline__ bool uncut_request(const float* __restrict__ temperature, const float* __restrict__ top_p,
                                              int req) {
  return temp_scale(temperature[req]) != 0.0f && !(top_p[req] < 1.0f);
}

// Request r's top-k (0 when off: no array, k <= 0 or k >= V).
__device__ __forceinline__ int request_k(const int32_t* __restrict__ top_k, int r, int V) {
  const int k = top_k ? top_k[r] : 0;
  return k > 0 && k < V ? k : 0;
}

// Which requests' rows a statistics pass leaves to another kernel: none; those sampling at a
// positive temperature without a cut (the cluster tree walk finds their statistics itself); or
// those with a cut, top-p below 1 or an active top-k at a positive temperature (the one-pass
// cut-row kernel of cutrow.cuh takes them).
enum SkipMode : int { kSkipNone = 0, kSkipUncut = 1, kSkipCut = 2 };
struct Skip {
  const float* top_p;    // per request (read unless mode is kSkipNone)
  const int32_t* top_k;  // per request, or null (off)
  int mode;
};

// Scale c of a request's rows for the streaming pass, or -1 for the rows it leaves alone.
__device__ __forceinline__ float stream_scale(const float* __restrict__ temperature, const Skip& sk, int req, int V) {
  const float c = temp_scale(temperature[req]);
  if (sk.mode == kSkipNone || c == 0.0f) return c;
  const bool cut = sk.top_p[req] < 1.0f || request_k(sk.top_k, req, V) > 0;
  return (sk.mode == kSkipUncut ? !cut : cut) ? -1.0f : c;
}

// The rows a statistics pass reads: rows [0, rows_a) of tensor a, then the rows of tensor b
// (same V). The request of row k of either tensor is k / rows_per_req, or, with offs (the
// node offsets of nreq tries), the j with offs[j] <= k < offs[j + 1] (a binary search that
// stays in [0, nreq) whatever offs holds).
template <typename T>
struct RowSet {
  const T* a;
  const T* b;
  int64_t rows_a;
  int rows_per_req;
  const int32_t* offs;
  int nreq;
  __device__ __forceinline__ const T* row(int64_t r, int V) const {
    return r < rows_a ? a + static_cast<size_t>(r) * V : b + static_cast<size_t>(r - rows_a) * V;
  }
  __device__ __forceinline__ int request(int64_t r) const {
    const int64_t k = r < rows_a ? r : r - rows_a;
    if (offs == nullptr) return static_cast<int>(k / rows_per_req);
    int lo = 0, hi = nreq;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(offs + mid) <= k) lo = mid;
      else hi = mid;
    }
    return lo;
  }
};

// Running statistics of one lane over a chunk: maximum m and the fp32 sum s of
// 2^((x - m) c), or (greedy rows) the maximum and its lowest index. A NaN or +inf logit
// makes s NaN (non-greedy) or sets `bad` (greedy), which marks the row as a data error.
struct LaneStat {
  float m, s;
  int amax;
  bool bad;
};

template <bool GREEDY>
__device__ __forceinline__ void lane_scalar(LaneStat& L, float x, int v, float c) {
  if (GREEDY) {
    L.bad |= !(x < INFINITY);
    if (x > L.m) { L.m = x; L.amax = v; }
  } else {
    if (x > L.m) {
      L.s *= ex2((L.m - x) * c);
      L.m = x;
    }
    L.s += ex2((x - L.m) * c);
  }
}

template <typename T, bool GREEDY>
__device__ __forceinline__ void lane_vector(LaneStat& L, const uint4& raw, int v, float c) {
  constexpr int N = Vec<T>::N;
  float f[8];
  Vec<T>::unpack(raw, f);
  if (GREEDY) {
    float vmax = f[0];
#pragma unroll
    for (int k = 1; k < N; ++k) vmax = fmax_nan(vmax, f[k]);
    L.bad |= !(vmax < INFINITY);
    if (vmax > L.m) {
#pragma unroll
      for (int k = N - 1; k >= 0; --k)
        if (f[k] == vmax) L.amax = v + k;
      L.m = vmax;
    }
  } else {
    float vmax;
    if (N == 8) {
      vmax = fmaxf(fmaxf(fmaxf(f[0], f[1]), fmaxf(f[2], f[3])), fmaxf(fmaxf(f[4], f[5]), fmaxf(f[6], f[7])));
    } else {
      vmax = fmaxf(fmaxf(f[0], f[1]), fmaxf(f[2], f[3]));
    }
    if (vmax > L.m) {
      L.s *= ex2((L.m - vmax) * c);
      L.m = vmax;
    }
    if (N == 8) {
      float w[8];
      exp8(f, L.m, c, w);
      L.s += sum8(w);
    } else {
      float acc = 0.0f;
#pragma unroll
      for (int k = 0; k < N; ++k) acc += ex2((f[k] - L.m) * c);
      L.s += acc;
    }
  }
}

// Warp-level partial of the chunk [c0, c1) of one row: per lane online statistics over
// coalesced 16-byte vectors (kBatch loads in flight), across lanes fp64. All lanes get it.
// The lane maximum starts at the lowest finite float so that -inf logits add exact zeros;
// a lane that saw no finite logit ends with s == 0 and reports -inf.
template <typename T, bool GREEDY>
__device__ __forceinline__ Partial warp_chunk_partial(const T* __restrict__ row, int c0, int c1, float c) {
  constexpr int N = Vec<T>::N;
  constexpr int stride = 32 * N;
  constexpr int kFull = kChunkElems / stride;  // vectors per lane in a full chunk
  const int lane = threadIdx.x & 31;
  LaneStat L{GREEDY ? -INFINITY : -3.402823466e38f, 0.0f, 0x7fffffff, false};
  const bool full = c1 - c0 == kChunkElems && (reinterpret_cast<uintptr_t>(row + c0) & 15u) == 0;
  if (full) {
    static_assert(kFull % kBatch == 0, "full chunks are whole batches");
#pragma unroll
    for (int b = 0; b < kFull; b += kBatch) {
      uint4 raw[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        raw[u] = __ldg(reinterpret_cast<const uint4*>(row + c0 + (b + u) * stride + lane * N));
#pragma unroll
      for (int u = 0; u < kBatch; ++u) lane_vector<T, GREEDY>(L, raw[u], c0 + (b + u) * stride + lane * N, c);
    }
  } else {
    int a0, a1;
    vec_range(row, c0, c1, a0, a1);
    for (int v = c0 + lane; v < a0; v += 32) lane_scalar<GREEDY>(L, load_elem(row + v), v, c);
    for (int v = a1 + lane; v < c1; v += 32) lane_scalar<GREEDY>(L, load_elem(row + v), v, c);
#pragma unroll 1
    for (int vb = a0 + lane * N; vb < a1; vb += kBatch * stride) {
      uint4 raw[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (vb + u * stride < a1) raw[u] = __ldg(reinterpret_cast<const uint4*>(row + vb + u * stride));
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (vb + u * stride < a1) lane_vector<T, GREEDY>(L, raw[u], vb + u * stride, c);
    }
  }
  if (!GREEDY && L.s == 0.0f) L.m = -INFINITY;  // no finite logit in this lane
  const float M = warp_max(L.m);
  Partial p{0.0, M, 0, __any_sync(0xffffffffu, L.bad) ? 1 : 0, 0};
  if (GREEDY) {
    p.amax = __reduce_min_sync(0xffffffffu, L.m == M ? L.amax : 0x7fffffff);
  } else {
    const double mine = L.m > -INFINITY ? static_cast<double>(L.s) * static_cast<double>(ex2((L.m - M) * c)) : 0.0;
    p.s = warp_sum(mine);  // NaN when the chunk holds a NaN or +inf logit
  }
  return p;
}

// The streaming pass: persistent warps over every chunk of a [rows, V] tensor, each chunk
// read once, one partial per chunk (parts[row * nchunks + chunk]), except the rows that
// stream_scale marks. CTA 0
// also clears the nzero arrival counters at `zero` that the call's later kernels use.
template <typename T>
__global__ void __launch_bounds__(kThreads, 4) stream_partials_kernel(RowSet<T> rows, int V,
                                                                    int64_t total_chunks,
                                                                    const float* __restrict__ temperature, Skip skip,
                                                                    Partial* __restrict__ parts,
                                                                    int32_t* __restrict__ zero, int nzero) {
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0;
  const int nch = nchunks_for(V);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= total_chunks) return;
  // (row, chunk) of g, advanced by nwarps chunks per step without a division in the loop
  int row = static_cast<int>(g / nch), chunk = static_cast<int>(g - static_cast<int64_t>(row) * nch);
  const int drow = static_cast<int>(nwarps / nch), dchunk = static_cast<int>(nwarps - static_cast<int64_t>(drow) * nch);
#pragma unroll 1
  for (; g < total_chunks; g += nwarps) {
    const float c = stream_scale(temperature, skip, rows.request(row), V);
    if (c >= 0.0f) {
      const T* rp = rows.row(row, V);
      const int c0 = chunk * kChunkElems, c1 = min(V, c0 + kChunkElems);
      const Partial p =
          c == 0.0f ? warp_chunk_partial<T, true>(rp, c0, c1, c) : warp_chunk_partial<T, false>(rp, c0, c1, c);
      if ((threadIdx.x & 31) == 0) parts[g] = p;
    }
    row += drow;
    chunk += dchunk;
    if (chunk >= nch) {
      chunk -= nch;
      ++row;
    }
  }
}

// ---------------------------------------------------------------------------------------
// Bulk-copy (TMA, non-tensor) streaming pass. Every warp owns a private ring of kRing
// shared-memory stages of one chunk each; its lane 0 keeps kRing - 1 chunks in flight with
// cp.async.bulk (completion counted on one mbarrier per stage) while the warp reduces the
// oldest one from shared memory. Requires 16-byte aligned rows whose byte length is a
// multiple of 16 (then every chunk copy is aligned); other tensors use the LDG pass.
constexpr int kRing = 2;
template <typename T>
constexpr int kStageBytes = kChunkElems * static_cast<int>(sizeof(T));  // one chunk

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for a stage: false if the copy has not landed after about a second.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 1000000000ull) return false;
  return true;
}

// NaN-propagating maximum of two packed bf16 pairs.
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// NaN-propagating maximum of the elements of NV 16-byte vectors (bf16 pairs are compared
// packed, before any conversion).
template <typename T, int NV>
__device__ __forceinline__ float lane_max_raw(const uint4 (&raw)[NV]) {
  if constexpr (sizeof(T) == 2) {
    uint32_t m0 = bmax2(raw[0].x, raw[0].y), m1 = bmax2(raw[0].z, raw[0].w);
#pragma unroll
    for (int j = 1; j < NV; ++j) {
      m0 = bmax2(m0, bmax2(raw[j].x, raw[j].y));
      m1 = bmax2(m1, bmax2(raw[j].z, raw[j].w));
    }
    const uint32_t m = bmax2(m0, m1);
    return fmax_nan(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
  } else {
    float m0 = fmax_nan(__uint_as_float(raw[0].x), __uint_as_float(raw[0].y));
    float m1 = fmax_nan(__uint_as_float(raw[0].z), __uint_as_float(raw[0].w));
#pragma unroll
    for (int j = 1; j < NV; ++j) {
      m0 = fmax_nan(m0, fmax_nan(__uint_as_float(raw[j].x), __uint_as_float(raw[j].y)));
      m1 = fmax_nan(m1, fmax_nan(__uint_as_float(raw[j].z), __uint_as_float(raw[j].w)));
    }
    return fmax_nan(m0, m1);
  }
}

// Warp-level partial of one full chunk held in registers (NV vectors per lane), in two
// steps: the chunk maximum M first (NaN-propagating, so a NaN or +inf logit leaves s NaN),
// then the weights 2^((x - M) c) relative to it, summed in packed fp32 pairs per lane and in
// fp64 across lanes. A chunk of -inf logits only reports s = 0, m = -inf.
template <typename T, int NV>
__device__ __forceinline__ Partial warp_chunk_partial_full(const uint4 (&raw)[NV], float c) {
  const float M = warp_max(lane_max_raw<T, NV>(raw));
  Partial p{0.0, M, 0, 0, 0};
  if (M == -INFINITY) return p;
  const f32x2 mm = pack2(M, M), cc = pack2(c, c);
  f32x2 acc0 = pack2(0.0f, 0.0f), acc1 = acc0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    float f[8];
    Vec<T>::unpack(raw[j], f);
#pragma unroll
    for (int k = 0; k < Vec<T>::N; k += 4) {
      float a, b, d, e;
      unpack2(mul2(sub2(pack2(f[k], f[k + 1]), mm), cc), a, b);
      unpack2(mul2(sub2(pack2(f[k + 2], f[k + 3]), mm), cc), d, e);
      acc0 = add2(acc0, pack2(ex2(a), ex2(b)));
      acc1 = add2(acc1, pack2(ex2(d), ex2(e)));
    }
  }
  float a, b, d, e;
  unpack2(acc0, a, b);
  unpack2(acc1, d, e);
  p.s = warp_sum((static_cast<double>(a) + static_cast<double>(b)) + (static_cast<double>(d) + static_cast<double>(e)));
  return p;
}

// Warp-level partial of one chunk held in shared memory (n elements, 16-byte vectors).
template <typename T, bool GREEDY>
__device__ __forceinline__ Partial warp_chunk_partial_smem(const T* __restrict__ sp, int c0, int n, float c) {
  constexpr int N = Vec<T>::N;
  constexpr int kFull = kChunkElems / (32 * N);  // vectors per lane in a full chunk
  const int lane = threadIdx.x & 31;
  const uint4* v4 = reinterpret_cast<const uint4*>(sp);
  if (!GREEDY && n == kChunkElems) {
    uint4 raw[kFull];
#pragma unroll
    for (int j = 0; j < kFull; ++j) raw[j] = v4[lane + 32 * j];
    return warp_chunk_partial_full<T, kFull>(raw, c);
  }
  LaneStat L{GREEDY ? -INFINITY : -3.402823466e38f, 0.0f, 0x7fffffff, false};
  if (n == kChunkElems) {
    uint4 raw[kFull];
#pragma unroll
    for (int j = 0; j < kFull; ++j) raw[j] = v4[lane + 32 * j];
#pragma unroll
    for (int j = 0; j < kFull; ++j) lane_vector<T, GREEDY>(L, raw[j], c0 + (lane + 32 * j) * N, c);
  } else {
    const int nv = n / N;
    for (int j = lane; j < nv; j += 32) lane_vector<T, GREEDY>(L, v4[j], c0 + j * N, c);
  }
  if (!GREEDY && L.s == 0.0f) L.m = -INFINITY;  // no finite logit in this lane
  const float M = warp_max(L.m);
  Partial p{0.0, M, 0, __any_sync(0xffffffffu, L.bad) ? 1 : 0, 0};
  if (GREEDY) {
    p.amax = __reduce_min_sync(0xffffffffu, L.m == M ? L.amax : 0x7fffffff);
  } else {
    const double mine = L.m > -INFINITY ? static_cast<double>(L.s) * static_cast<double>(ex2((L.m - M) * c)) : 0.0;
    p.s = warp_sum(mine);
  }
  return p;
}

// log2(e)/T of up to kScaleTable requests, computed once per CTA into shared memory (the
// fp64 division per chunk would otherwise cost a few percent of the streaming pass).
constexpr int kScaleTable = 1024;

template <typename T>
__global__ void __launch_bounds__(kThreads) stream_partials_tma_kernel(RowSet<T> rows, int V,
                                                                        int64_t total_chunks,
                                                                        const float* __restrict__ temperature, Skip skip,
                                                                        int nreq,
                                                                        Partial* __restrict__ parts,
                                                                        int32_t* __restrict__ zero, int nzero) {
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0;
  extern __shared__ __align__(128) unsigned char ring_smem[];
  __shared__ uint64_t bars[kThreads / 32][kRing];
  __shared__ float scale[kScaleTable];
  const bool table = nreq <= kScaleTable;
  bool some = !table;  // whether any request's rows are read
  if (table)
    for (int i = threadIdx.x; i < nreq; i += kThreads) {
      scale[i] = stream_scale(temperature, skip, i, V);
      some |= scale[i] >= 0.0f;
    }
  if (!__syncthreads_or(some)) return;  // every row left alone
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char* ring = ring_smem + warp * kRing * kStageBytes<T>;
  uint64_t* bar = bars[warp];
  const int nch = nchunks_for(V);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + warp;
  if (g0 >= total_chunks) return;
  if (lane == 0) {
    for (int s = 0; s < kRing; ++s) mbar_init(&bar[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  // (row, chunk) cursors advanced by nwarps chunks per step, for the copies and the reduction
  const int drow = static_cast<int>(nwarps / nch), dchunk = static_cast<int>(nwarps - static_cast<int64_t>(drow) * nch);
  auto advance = [&](int& row, int& chunk) {
    row += drow;
    chunk += dchunk;
    if (chunk >= nch) {
      chunk -= nch;
      ++row;
    }
  };
  int row = static_cast<int>(g0 / nch), chunk = static_cast<int>(g0 - static_cast<int64_t>(row) * nch);
  int irow = row, ichunk = chunk;  // cursor of the next copy to issue
  int64_t gi = g0;
  auto scale_of = [&](int r) {
    const int req = rows.request(r);
    return table ? scale[req] : stream_scale(temperature, skip, req, V);
  };
  uint32_t pending = 0u;  // (lane 0) stages with a copy in flight
  auto issue = [&](int i) {  // copy of this warp's i-th chunk into stage i % kRing (lane 0)
    if (gi < total_chunks && scale_of(irow) >= 0.0f) {
      const int c0 = ichunk * kChunkElems, n = min(V - c0, kChunkElems);
      const uint32_t bytes = static_cast<uint32_t>(n) * sizeof(T);
      uint64_t* b = &bar[i % kRing];
      mbar_expect_tx(b, bytes);
      bulk_g2s(ring + (i % kRing) * kStageBytes<T>, rows.row(irow, V) + c0, bytes, b);
      pending |= 1u << (i % kRing);
    }
    gi += nwarps;
    advance(irow, ichunk);
  };
  if (lane == 0)
    for (int i = 0; i < kRing - 1; ++i) issue(i);
  int i = 0;
  uint32_t phase_bits = 0u;  // parity of each stage's next completion (stages of skipped rows do not flip)
  for (int64_t g = g0; g < total_chunks; g += nwarps, ++i) {
    __syncwarp();  // every lane is done with the stage that the next copy overwrites
    if (lane == 0) issue(i + kRing - 1);
    const int c0 = chunk * kChunkElems, n = min(V - c0, kChunkElems);
    const float c = scale_of(row);
    if (c < 0.0f) {  // a row this pass leaves alone
      advance(row, chunk);
      continue;
    }
    const int st = i % kRing;
    const uint32_t parity = (phase_bits >> st) & 1u;
    const bool landed = mbar_wait_bounded(&bar[st], parity);
    if (!__all_sync(0xffffffffu, landed)) {
      // a copy that never completed: this chunk and every later chunk of this warp are reported
      // as data errors (their rows end with status 1), nothing more is issued, and the copies
      // still in flight get a bounded wait before the warp leaves (they write this CTA's
      // shared memory)
      if (lane == 0) {
        for (int64_t h = g; h < total_chunks; h += nwarps) {
          if (scale_of(row) >= 0.0f) parts[h] = Partial{0.0, NAN, 0, 1, 0};
          advance(row, chunk);
        }
        for (int s = 0; s < kRing; ++s)
          if ((pending >> s) & 1u) mbar_wait_bounded(&bar[s], s == st ? parity : (phase_bits >> s) & 1u);
      }
      return;
    }
    phase_bits ^= 1u << st;
    pending &= ~(1u << st);
    const T* sp = reinterpret_cast<const T*>(ring + st * kStageBytes<T>);
    const Partial p = c == 0.0f ? warp_chunk_partial_smem<T, true>(sp, c0, n, c)
                                : warp_chunk_partial_smem<T, false>(sp, c0, n, c);
    if (lane == 0) parts[g] = p;
    advance(row, chunk);
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

// A partial written by another warp of the running kernel, read through L2.
__device__ __forceinline__ Partial load_partial_cg(const Partial* p) {
  Partial q;
  q.s = __ldcg(&p->s);
  const int2 a = __ldcg(reinterpret_cast<const int2*>(&p->m));
  const int2 b = __ldcg(reinterpret_cast<const int2*>(&p->bad));
  q.m = __int_as_float(a.x);
  q.amax = a.y;
  q.bad = b.x;
  q.pad = b.y;
  return q;
}

// Warp-level: combine the chunk partials of one row in one pass (read through L2: they may
// come from other warps of the running kernel). Every lane gets the statistics; top-p is not
// applied.
__device__ __forceinline__ RowStat warp_finalize_row(const Partial* __restrict__ pp, int nchunks, float Tv) {
  const int lane = threadIdx.x & 31;
  const float c = temp_scale(Tv);
  float M = -INFINITY;
  double S = 0.0;
  int amax = 0x7fffffff;
  bool bad = !(Tv >= 0.0f && Tv < INFINITY);
  for (int i = lane; i < nchunks; i += 32) {
    const Partial q = load_partial_cg(pp + i);
    bad |= q.bad != 0 || q.m != q.m;
    if (c != 0.0f) {
      if (q.m > M) {
        if (M > -INFINITY) S *= static_cast<double>(ex2((M - q.m) * c));
        M = q.m;
      }
      if (q.m > -INFINITY) S += q.s * static_cast<double>(ex2((q.m - M) * c));
    } else if (q.m > M || (q.m == M && q.amax < amax)) {
      M = q.m;
      amax = q.amax;
    }
  }
  const float Mw = warp_max(M);
  if (c != 0.0f) {
    S = M > -INFINITY ? S * static_cast<double>(ex2((M - Mw) * c)) : 0.0;
    S = warp_sum(S);
  }
  amax = __reduce_min_sync(0xffffffffu, M == Mw ? amax : 0x7fffffff);
  bad = __any_sync(0xffffffffu, bad) || !(Mw > -INFINITY) || !(Mw < INFINITY) || (c != 0.0f && !(S == S));
  RowStat st;
  st.m = Mw;
  st.c = c;
  st.s = c != 0.0f ? static_cast<float>(S) : 1.0f;
  st.s_kept = st.s;
  st.tau = 0u;
  st.amax = c != 0.0f ? -1 : amax;
  st.status = bad ? 1 : 0;
  st.pad = 0;
  return st;
}

constexpr int kCache = 4;  // chunk partials per lane held in registers by warp_finalize_pick

// Result of warp_finalize_pick.
struct RowPick {
  RowStat st;
  int chunk;           // chunk holding u * Z (-1 if none / not requested)
  double base, target;  // weight before that chunk, and u * Z
};

// Warp-level finish of one row from its chunk partials in one round trip: statistics (as
// warp_finalize_row) and, when `pick` is set, the chunk holding u * Z of the row's own
// distribution (no top-p cut). Lane l owns the contiguous chunks [l*q, l*q + q); for rows
// of more than 32 * kCache chunks it falls back to two passes.
__device__ __forceinline__ RowPick warp_finalize_pick(const Partial* __restrict__ pp, int nchunks, float Tv, float u,
                                                      bool pick) {
  const int lane = threadIdx.x & 31;
  RowPick r;
  r.chunk = -1;
  r.base = 0.0;
  r.target = 0.0;
  const int q = (nchunks + 31) / 32;
  if (q > kCache) {
    r.st = warp_finalize_row(pp, nchunks, Tv);
    return r;  // callers use warp_pick_chunk on this path
  }
  const float c = temp_scale(Tv);
  const int i0 = min(nchunks, lane * q);
  Partial part[kCache];
#pragma unroll
  for (int k = 0; k < kCache; ++k)
    if (k < q && i0 + k < nchunks) part[k] = load_partial_cg(pp + i0 + k);
  float M = -INFINITY;
  int amax = 0x7fffffff;
  bool bad = !(Tv >= 0.0f && Tv < INFINITY);
#pragma unroll
  for (int k = 0; k < kCache; ++k) {
    if (!(k < q && i0 + k < nchunks)) continue;
    bad |= part[k].bad != 0 || part[k].m != part[k].m;
    if (part[k].m > M || (c == 0.0f && part[k].m == M && part[k].amax < amax)) {
      M = part[k].m;
      amax = part[k].amax;
    }
  }
  const float Mw = warp_max(M);
  double t[kCache];
  double mine = 0.0;
#pragma unroll
  for (int k = 0; k < kCache; ++k) {
    t[k] = (k < q && i0 + k < nchunks && c != 0.0f && part[k].m > -INFINITY)
               ? part[k].s * static_cast<double>(ex2((part[k].m - Mw) * c))
               : 0.0;
    mine += t[k];
  }
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const double S = __shfl_sync(0xffffffffu, incl, 31);
  amax = __reduce_min_sync(0xffffffffu, M == Mw ? amax : 0x7fffffff);
  bad = __any_sync(0xffffffffu, bad) || !(Mw > -INFINITY) || !(Mw < INFINITY) || (c != 0.0f && !(S == S));
  r.st.m = Mw;
  r.st.c = c;
  r.st.s = c != 0.0f ? static_cast<float>(S) : 1.0f;
  r.st.s_kept = r.st.s;
  r.st.tau = 0u;
  r.st.amax = c != 0.0f ? -1 : amax;
  r.st.status = bad ? 1 : 0;
  r.st.pad = 0;
  if (pick && !bad && c != 0.0f) {
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const double tg = static_cast<double>(u) * S;
    int sel = -1, last = -1;
    double b = 0.0, C = excl;
#pragma unroll
    for (int k = 0; k < kCache; ++k) {
      if (t[k] > 0.0) {
        last = i0 + k;
        if (sel < 0 && excl <= tg && tg < incl) {
          if (C + t[k] > tg) { sel = i0 + k; b = C; }
        }
      }
      C += t[k];
    }
    const unsigned who = __ballot_sync(0xffffffffu, sel >= 0);
    if (who) {
      const int src = __ffs(who) - 1;
      r.chunk = __shfl_sync(0xffffffffu, sel, src);
      r.base = __shfl_sync(0xffffffffu, b, src);
    } else {  // rounding put u * Z past every chunk: the last chunk with positive weight
      const int lastc = __reduce_max_sync(0xffffffffu, last);
      const int owner = __reduce_max_sync(0xffffffffu, last == lastc ? lane : -1);
      double bb = excl;
#pragma unroll
      for (int k = 0; k < kCache; ++k)
        if (i0 + k < lastc) bb += t[k];
      r.chunk = lastc;
      r.base = __shfl_sync(0xffffffffu, bb, owner < 0 ? 0 : owner);
    }
    r.target = tg;
  }
  return r;
}

// Whether a row's statistics still need the top-p threshold.
__device__ __forceinline__ bool needs_topp(const RowStat& st, float tp) {
  return st.status == 0 && st.c != 0.0f && tp < 1.0f;
}

// Top-p threshold (value-threshold reading: keep every token whose logit is at least the
// largest logit value t with mass(l >= t) >= top_p, ties kept together).
//
// First pass: every element of the row falls into one of kToppBins value bins, bin b holding
// the logits whose log2 weight (x - m) c lies within 1/16 of -b/8 (the last bin collects all
// smaller values). An element adds its weight relative to the bin's reference weight 2^(-b/8),
// 2^((x - m) c + b/8) in [2^(-1/16), 2^(1/16)], as a fixed-point integer with 22 fractional
// bits, to per-warp 64-bit histograms: sums are exact and independent of the order. The bin
// holding the threshold is the first, scanning from the maximum, whose cumulative mass
// reaches top_p of the total. Second, the bin's elements alone (no other element needs an
// exponential) go through a most-significant-digit radix select on their order-preserving
// keys, 8 bits per pass, with the same fixed-point masses; the key of the threshold value is
// exact after two passes for bf16 rows (four for fp32).
constexpr int kToppBins = 256;
constexpr int kToppWarps = 8;  // histograms per CTA (blockDim.x <= 32 * kToppWarps)

// Shared memory of the general radix select (block_topp_radix).
struct RadixSmem {
  double hmass[256];
  int hcnt[256];
  uint32_t prefix;
  double above, bucket, cabove;
};

struct ToppSmem {
  unsigned long long h[kToppWarps][kToppBins];
  double mass[kToppBins];
  double above, total, target;
  uint32_t prefix;
  int bin, fallback;
  RadixSmem radix;
};

// Value bin of logit x under (m, c) and its fixed-point mass relative to the bin's reference
// weight; identical arithmetic in every pass.
__device__ __forceinline__ void topp_bin(float x, float m, float c, int& b, uint32_t& u) {
  const float d = (x - m) * c;                                // log2 weight, <= 0
  const float t = fminf(d * -8.0f, 4096.0f);                  // -8 d, capped (also for -inf)
  const float r = t + 12582912.0f;                            // round to an integer (1.5 * 2^23 trick)
  b = min(__float_as_int(r) - __float_as_int(12582912.0f), kToppBins - 1);
  const float bf = fminf(r - 12582912.0f, static_cast<float>(kToppBins - 1));
  const float y = ex2(fmaf(bf, 0.125f, d));                   // 2^(d + b/8)
  u = __float_as_uint(y + 2.0f) - 0x40000000u;                // y * 2^22, rounded to nearest
}

// Bin of x only (no exponential).
__device__ __forceinline__ int topp_bin_only(float x, float m, float c) {
  const float t = fminf((x - m) * c * -8.0f, 4096.0f);
  return min(__float_as_int(t + 12582912.0f) - __float_as_int(12582912.0f), kToppBins - 1);
}

// 2^(-b/8) in fp64.
__device__ __forceinline__ double topp_ref(int b) { return ldexp(exp2(-static_cast<double>(b & 7) * 0.125), -(b >> 3)); }

// Visit every element of row [0, V) with f(x, v); vectorised body with kLoads 16-byte loads in
// flight per thread, scalar edges.
template <typename T, int kLoads, typename F>
__device__ __forceinline__ void for_each_elem_batched(const T* __restrict__ row, int V, F&& f) {
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
      if (v + i * step < a1) raw[i] = __ldg(reinterpret_cast<const uint4*>(row + v + i * step));
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

// General top-p select (fallback when the threshold lies below the first pass's value range):
// radix select on the 32-bit keys with fp64 atomics.
// One most-significant-digit radix select over the order keys of row rp (8 bits a level; 2
// levels cover a bf16 value, 4 an fp32 one), with the count and the fp64 weight of every
// digit. BY_COUNT: the key of the goal-th largest element (ties kept together); otherwise the
// largest key whose tie-inclusive tail weight reaches goal. Elements with a key below
// floor_key take no part. Returns the key; *above gets the weight of the elements strictly
// above its final digit bucket and *bucket that bucket's weight, so *above + *bucket is the
// weight of every element with a key >= the returned one. The result is in every thread.
template <typename T, bool BY_COUNT>
__device__ uint32_t block_radix_pick(const T* __restrict__ rp, int V, const RowStat& st, double goal,
                                     uint32_t floor_key, RadixSmem& sm, double* above, double* bucket) {
  const float M = st.m, c = st.c;
  const int levels = sizeof(T) == 2 ? 2 : 4;
  if (threadIdx.x == 0) { sm.prefix = 0u; sm.above = 0.0; sm.bucket = 0.0; sm.cabove = 0.0; }
  for (int lv = 0; lv < levels; ++lv) {
    const int shift = 24 - 8 * lv;
    for (int d = threadIdx.x; d < 256; d += blockDim.x) { sm.hmass[d] = 0.0; sm.hcnt[d] = 0; }
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for_each_elem(rp, V, [&](float x) {
      const uint32_t k = fkey(x);
      if (k >= floor_key && (lv == 0 || (k >> (shift + 8)) == (prefix >> (shift + 8)))) {
        const int d = (k >> shift) & 255;
        atomicAdd(&sm.hmass[d], static_cast<double>(ex2((x - M) * c)));
        atomicAdd(&sm.hcnt[d], 1);
      }
    });
    __syncthreads();
    if (threadIdx.x == 0) {
      double running = sm.above, counted = sm.cabove;
      int pick = -1;
      for (int d = 255; d >= 0; --d) {
        if (sm.hcnt[d] == 0) continue;
        if (BY_COUNT ? counted + sm.hcnt[d] >= goal : running + sm.hmass[d] >= goal) { pick = d; break; }
        running += sm.hmass[d];
        counted += sm.hcnt[d];
      }
      if (pick < 0) {  // the goal is not reached (rounding, or fewer elements): the lowest bucket
        running = sm.above;
        counted = sm.cabove;
        for (int d = 255; d >= 0; --d)
          if (sm.hcnt[d] != 0) { pick = d; running += sm.hmass[d]; counted += sm.hcnt[d]; }
        if (pick < 0) pick = 0;
        running -= sm.hmass[pick];
        counted -= sm.hcnt[pick];
      }
      sm.prefix = prefix | (static_cast<uint32_t>(pick) << shift);
      sm.above = running;
      sm.cabove = counted;
      sm.bucket = sm.hmass[pick];
    }
    __syncthreads();
  }
  const uint32_t key = sm.prefix;
  *above = sm.above;
  *bucket = sm.bucket;
  __syncthreads();
  return key;
}

// General top-p select (any dtype and V): the largest key whose tail weight reaches top_p of
// the row's total. Sets st.tau and st.s_kept in every thread.
template <typename T>
__device__ void block_topp_radix(const T* __restrict__ rp, int V, float tp, RowStat& st, RadixSmem& sm) {
  double above, bucket;
  st.tau = block_radix_pick<T, false>(rp, V, st, static_cast<double>(tp) * static_cast<double>(st.s), 0u, sm, &above,
                                      &bucket);
  st.s_kept = static_cast<float>(above + bucket);
}

// General top-k then top-p select (any dtype and V): the k-th largest key first (every
// element at or above it kept), then, among those, the largest key whose tail weight reaches
// top_p of their total. Sets st.tau and st.s_kept in every thread.
template <typename T>
__device__ void block_topk_topp_radix(const T* __restrict__ rp, int V, float tp, int k, RowStat& st, RadixSmem& sm) {
  double above, bucket;
  const uint32_t tau_k = block_radix_pick<T, true>(rp, V, st, static_cast<double>(k), 0u, sm, &above, &bucket);
  const double s_k = above + bucket;
  st.tau = tau_k;
  st.s_kept = static_cast<float>(s_k);
  if (tp < 1.0f) {
    st.tau = block_radix_pick<T, false>(rp, V, st, static_cast<double>(tp) * s_k, tau_k, sm, &above, &bucket);
    st.s_kept = static_cast<float>(above + bucket);
  }
}

// Block-level top-p threshold of row rp under statistics st (m, c, s set); sets st.tau and
// st.s_kept in every thread. Any block size up to 32 * kToppWarps threads.
template <typename T>
__device__ void block_topp_select(const T* __restrict__ rp, int V, float tp, RowStat& st, ToppSmem& sm) {
  const float m = st.m, c = st.c;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long* hw = sm.h[warp];
  for (int i = threadIdx.x; i < kToppWarps * kToppBins; i += blockDim.x) (&sm.h[0][0])[i] = 0ull;
  __syncthreads();
  for_each_elem_batched<T, 4>(rp, V, [&](float x) {
    int b;
    uint32_t u;
    topp_bin(x, m, c, b, u);
    if (u != 0u) atomicAdd(&hw[b], static_cast<unsigned long long>(u));
  });
  __syncthreads();
  for (int b = threadIdx.x; b < kToppBins; b += blockDim.x) {
    unsigned long long t = 0ull;
    for (int w = 0; w < nw; ++w) t += sm.h[w][b];
    sm.mass[b] = static_cast<double>(t) * topp_ref(b);
  }
  __syncthreads();
  if (warp == 0) {
    // bins of lane l: [8l, 8l + 8) (kToppBins == 256)
    double mine = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) mine += sm.mass[lane * 8 + k];
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
    const int src = hit ? __ffs(hit) - 1 : 31 - __clz(__ballot_sync(0xffffffffu, mine > 0.0));
    if (lane == src) {
      double run = excl;
      int pick = -1;
      double before = excl;
      for (int k = 0; k < 8; ++k) {
        const double mk = sm.mass[lane * 8 + k];
        if (mk > 0.0) {
          pick = lane * 8 + k;
          before = run;
          if (run + mk >= target) break;
        }
        run += mk;
      }
      sm.bin = pick;
      sm.above = before;
      sm.total = total;
      sm.target = target;
      sm.prefix = 0u;
      sm.fallback = pick == kToppBins - 1;
    }
  }
  __syncthreads();
  if (sm.fallback) {
    block_topp_radix<T>(rp, V, tp, st, sm.radix);
    return;
  }
  // radix select on the keys of bin sm.bin's elements, 8 bits per pass
  const int bstar = sm.bin;
  const double ref = topp_ref(bstar);
  const int levels = sizeof(T) == 2 ? 2 : 4;
  for (int lv = 0; lv < levels; ++lv) {
    const int shift = 24 - 8 * lv;
    for (int i = threadIdx.x; i < nw * 256; i += blockDim.x) (&sm.h[0][0])[(i / 256) * kToppBins + (i % 256)] = 0ull;
    __syncthreads();
    const uint32_t prefix = sm.prefix;
    for_each_elem_batched<T, 4>(rp, V, [&](float x) {
      if (topp_bin_only(x, m, c) != bstar) return;
      const uint32_t k = fkey(x);
      if (lv != 0 && (k >> (shift + 8)) != (prefix >> (shift + 8))) return;
      int b;
      uint32_t u;
      topp_bin(x, m, c, b, u);
      if (u != 0u) atomicAdd(&hw[(k >> shift) & 255], static_cast<unsigned long long>(u));
    });
    __syncthreads();
    for (int d = threadIdx.x; d < 256; d += blockDim.x) {
      unsigned long long t = 0ull;
      for (int w = 0; w < nw; ++w) t += sm.h[w][d];
      sm.mass[d] = static_cast<double>(t) * ref;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      // digits from the largest key down: the first whose cumulative mass reaches the target
      double run = sm.above;
      int pick = -1, last = -1;
      double before = run;
      for (int d = 255; d >= 0; --d) {
        const double md = sm.mass[d];
        if (md <= 0.0) continue;
        last = d;
        before = run;
        if (run + md >= sm.target) { pick = d; break; }
        run += md;
      }
      if (pick < 0) pick = last;  // rounding: the bin's smallest digit with mass
      sm.prefix = prefix | (static_cast<uint32_t>(pick < 0 ? 0 : pick) << shift);
      sm.above = before;
      if (lv == levels - 1) sm.mass[0] = before + (pick < 0 ? 0.0 : sm.mass[pick]);
    }
    __syncthreads();
  }
  st.tau = sm.prefix;
  st.s_kept = static_cast<float>(static_cast<double>(st.s) * (sm.mass[0] / sm.total));
  __syncthreads();
}

// Row statistics from the chunk partials (the tree's statistics pass and psispec_row_stats):
// kThreads / 32 rows per CTA, one warp finalizing each row; the CTA then runs the top-p
// select (or, for a request with a top-k, the top-k then top-p select) for those of its rows
// that need one. Rows that stream_scale marks are skipped. top_k may be null (off).
template <typename T>
__global__ void __launch_bounds__(kThreads) row_finalize_kernel(RowSet<T> rows, int64_t nrows, int V,
                                                                 const float* __restrict__ temperature,
                                                                 const float* __restrict__ top_p,
                                                                 const int32_t* __restrict__ top_k,
                                                                 const Partial* __restrict__ parts,
                                                                 RowStat* __restrict__ stats, Skip skip) {
  constexpr int kRows = kThreads / 32;
  __shared__ ToppSmem sm;
  __shared__ RowStat sh_st[kRows];
  __shared__ int sh_topp[kRows];
  __shared__ int sh_k[kRows];
  const int warp = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRows + warp;
  const int nch = nchunks_for(V);
  if (row < nrows) {
    const int req = rows.request(row);
    int topp = 0, k = 0;
    if (stream_scale(temperature, skip, req, V) >= 0.0f) {
      const RowStat st = warp_finalize_row(parts + static_cast<size_t>(row) * nch, nch, temperature[req]);
      k = st.status == 0 && st.c != 0.0f ? request_k(top_k, req, V) : 0;
      topp = needs_topp(st, top_p[req]) || k > 0;
      if ((threadIdx.x & 31) == 0) {
        sh_st[warp] = st;
        if (!topp) stats[row] = st;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      sh_topp[warp] = topp;
      sh_k[warp] = k;
    }
  } else if ((threadIdx.x & 31) == 0) {
    sh_topp[warp] = 0;
    sh_k[warp] = 0;
  }
  __syncthreads();
  for (int w = 0; w < kRows; ++w) {
    if (!sh_topp[w]) continue;  // the same branch in every thread
    const int64_t r = static_cast<int64_t>(blockIdx.x) * kRows + w;
    RowStat st = sh_st[w];
    if (sh_k[w] > 0)  // the same branch in every thread
      block_topk_topp_radix<T>(rows.row(r, V), V, top_p[rows.request(r)], sh_k[w], st, sm.radix);
    else
      block_topp_select<T>(rows.row(r, V), V, top_p[rows.request(r)], st, sm);
    if (threadIdx.x == 0) stats[r] = st;
  }
}

}  // namespace psi
