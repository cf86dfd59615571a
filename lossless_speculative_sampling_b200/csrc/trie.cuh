// trie.cuh -- candidate trie of the tree sampler (review page of arXiv 2609.04010, section 3.4,
// "Tree Sampler": at every position of the drafted block take the top-K tokens, then keep the
// V most probable prefixes, verified together; the README's tree example sets the two sizes).
//
// Readings: a position's distribution is its draft row's q after the sampling controls; the
// candidates are the cand_k kept tokens of largest q (ties to the lower index, q > 0); a
// prefix's probability is the product of its tokens' q; the n_prefixes most probable prefixes
// are kept, ties to the shorter prefix and then to the smaller sequence of candidate ranks,
// and numbered in the order kept (node 0 is the empty prefix). Prefixes of one length share
// their normalisers, so they compare exactly by their logit sums (fp64 sums of the input
// values); prefixes of different lengths compare by their fp64 probabilities.
//
// Two kernels after the row statistics of the B*K draft rows (rows of requests with a cut;
// the others get theirs in the first kernel's pass):
//   trie_candidates_kernel  one CTA per row: one coalesced pass keeps the maximum of every lane
//                           block (a lane's elements of a few steps) in shared memory (and,
//                           for a row without a cut, each lane's running maximum and sum of
//                           weights); the cand_k-th largest block maximum (an exact radix
//                           select over the block keys) is a pivot at or below the cand_k-th
//                           largest element; only the blocks at or above it are read again,
//                           their elements at or above it are ranked exactly (key, then the
//                           lower index) and the first cand_k kept. Rows with more elements at
//                           the pivot than the ranking holds (long runs of equal values) take a
//                           general radix select instead;
//   trie_select_kernel      one warp per request: best-first choice of the prefixes, one
//                           offer per kept node (its best child not kept yet) held in lane
//                           registers, the products in fp64.
// Then tree_walk_det_kernel verifies such a trie (the deterministic-candidate rule).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "stats.cuh"
#include "tree.cuh"

namespace psi {

constexpr int kTrieMaxCand = 32;      // cand_k limit (one lane per candidate when ranking)
constexpr int kTrieMaxPrefixes = 64;  // n_prefixes limit
constexpr int kTrieMaxK = 16;         // positions limit (rank paths are kept per node)
constexpr int kTrieThreads = 512;
constexpr int kTrieVec = 8;            // 16-byte loads per lane per step
constexpr int kTrieMaxBlocks = 8192;   // lane blocks whose maxima shared memory holds
constexpr int kTrieCap = 1024;         // elements at or above the pivot that are ranked exactly

struct TrieFastSmem {
  uint32_t bkey[kTrieMaxBlocks + 1];  // order key of each lane block's maximum (+ the edge block)
  unsigned long long cand[kTrieCap];  // (key << 32) | ~index of the elements at or above the pivot
  unsigned long long top[kTrieMaxCand];
  uint32_t hist[256];
  uint32_t prefix;
  int need, ncand;
};

struct TrieGenSmem {
  RadixSmem radix;
  double scan[33];
  int gt_idx[kTrieMaxCand];
  int eq_idx[kTrieMaxCand];
  int ngt;
};

union TrieCandSmem {
  TrieFastSmem fast;
  TrieGenSmem gen;
};

// Lane blocks of a row: the aligned interior [a0, a1) holds nv 16-byte vectors; a step of a
// warp is 32 * kTrieVec vectors (vector j * 32 + lane of the step to each lane); warp w takes
// steps [w spw, (w + 1) spw); a lane block is r consecutive steps of one lane; bpl blocks per
// lane; block (w bpl + i) * 32 + lane; block nb holds the unaligned edges [0, a0) and [a1, V).
struct TrieGeom {
  int a0, a1, nv, spw, r, bpl, nb;
};

template <typename T>
__device__ __forceinline__ TrieGeom trie_geom(const T* rp, int V) {
  constexpr int N = Vec<T>::N;
  TrieGeom g;
  vec_range(rp, 0, V, g.a0, g.a1);
  g.nv = (g.a1 - g.a0) / N;
  const int nw = blockDim.x >> 5;
  const int steps = (g.nv + 32 * kTrieVec - 1) / (32 * kTrieVec);
  g.spw = (steps + nw - 1) / nw;
  const int cap = kTrieMaxBlocks / (nw * 32);
  g.r = max(1, (g.spw + cap - 1) / cap);
  g.bpl = (g.spw + g.r - 1) / g.r;
  g.nb = nw * g.bpl * 32;
  return g;
}

// Maximum of the 8 (bf16) or 4 (fp32) values of one 16-byte vector, folded into m. NaN
// propagates (a row that reaches this pass with one is a data error: rows with statistics
// from the statistics pass have none, and the rows found here check).
__device__ __forceinline__ void vmax_fold(const uint4& v, __nv_bfloat162& m, const __nv_bfloat16*) {
  m = __hmax2_nan(m, *reinterpret_cast<const __nv_bfloat162*>(&v.x));
  m = __hmax2_nan(m, *reinterpret_cast<const __nv_bfloat162*>(&v.y));
  m = __hmax2_nan(m, *reinterpret_cast<const __nv_bfloat162*>(&v.z));
  m = __hmax2_nan(m, *reinterpret_cast<const __nv_bfloat162*>(&v.w));
}
__device__ __forceinline__ void vmax_fold(const uint4& v, float& m, const float*) {
  m = fmax_nan(m, fmax_nan(fmax_nan(__uint_as_float(v.x), __uint_as_float(v.y)),
                           fmax_nan(__uint_as_float(v.z), __uint_as_float(v.w))));
}
__device__ __forceinline__ float vmax_value(const __nv_bfloat162& m) {
  return fmax_nan(__low2float(m), __high2float(m));
}
__device__ __forceinline__ float vmax_value(float m) { return m; }
__device__ __forceinline__ void vmax_merge(__nv_bfloat162& m, const __nv_bfloat162& x) { m = __hmax2_nan(m, x); }
__device__ __forceinline__ void vmax_merge(float& m, float x) { m = fmax_nan(m, x); }

// Sum of the weights 2^((x - M) c) of one 16-byte vector (8 bf16 or 4 fp32 values), each the
// arithmetic of kept_weight, summed in fp32.
__device__ __forceinline__ float vweight_sum(const uint4& v, float M, float c, const __nv_bfloat16*) {
  float x[8], w[8];
  Vec<__nv_bfloat16>::unpack(v, x);
  exp8(x, M, c, w);
  return sum8(w);
}
__device__ __forceinline__ float vweight_sum(const uint4& v, float M, float c, const float*) {
  return ex2((__uint_as_float(v.x) - M) * c) + ex2((__uint_as_float(v.y) - M) * c) +
         (ex2((__uint_as_float(v.z) - M) * c) + ex2((__uint_as_float(v.w) - M) * c));
}

// A lane's running maximum M of the values it has seen and its fp64 sum of 2^((x - M) c),
// rescaled when M grows.
struct TrieLaneSum {
  float M;
  double s;
  bool bad;  // a NaN or +inf seen
  __device__ __forceinline__ void grow(float mx, float c) {
    bad |= !(mx < INFINITY) && !(mx == -INFINITY);
    if (mx > M && mx < INFINITY) {
      if (M > -INFINITY) s *= static_cast<double>(ex2((M - mx) * c));
      M = mx;
    }
  }
};

template <typename T>
struct VmaxAcc;
template <>
struct VmaxAcc<__nv_bfloat16> {
  using type = __nv_bfloat162;
  __device__ __forceinline__ static type init() { return __floats2bfloat162_rn(-INFINITY, -INFINITY); }
  static constexpr uint32_t kNegInfWord = 0xFF80FF80u;
};
template <>
struct VmaxAcc<float> {
  using type = float;
  __device__ __forceinline__ static type init() { return -INFINITY; }
  static constexpr uint32_t kNegInfWord = 0xFF800000u;
};

// The k-th largest of keys[0, n) (duplicates counted), n >= k >= 1, to its top 8 * levels
// bits (the lower bits 0): an 8-bit most-significant-digit radix select over the shared
// array. Result in every thread.
__device__ uint32_t smem_kth_largest(const uint32_t* keys, int n, int k, int levels, TrieFastSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t prefix = 0u;
  int need = k;
  for (int lv = 0; lv < levels; ++lv) {
    const int shift = 24 - 8 * lv;
    for (int d = threadIdx.x; d < 256; d += blockDim.x) sm.hist[d] = 0u;
    __syncthreads();
    for (int b = threadIdx.x; b < n; b += blockDim.x) {
      const uint32_t key = keys[b];
      if (lv == 0 || (key >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8 l down to 248 - 8 l
      uint32_t c[8], s = 0u;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = sm.hist[255 - 8 * lane - q];
        s += c[q];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - s;
      const unsigned hit = __ballot_sync(0xffffffffu, excl < static_cast<uint32_t>(need) &&
                                                         static_cast<uint32_t>(need) <= incl);
      if (lane == __ffs(hit) - 1) {
        uint32_t acc = excl;
        int digit = 255 - 8 * lane - 7;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (acc + c[q] >= static_cast<uint32_t>(need)) { digit = 255 - 8 * lane - q; break; }
          acc += c[q];
        }
        sm.prefix = prefix | (static_cast<uint32_t>(digit) << shift);
        sm.need = need - static_cast<int>(acc);
      }
    }
    __syncthreads();
    prefix = sm.prefix;
    need = sm.need;
  }
  __syncthreads();
  return prefix;
}

// Packed candidate: larger means a larger key, then the lower index.
__device__ __forceinline__ unsigned long long trie_pack(uint32_t key, int idx) {
  return (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ void trie_push(TrieFastSmem& sm, uint32_t key, int idx) {
  const int slot = atomicAdd(&sm.ncand, 1);
  if (slot < kTrieCap) sm.cand[slot] = trie_pack(key, idx);
}

// Candidates of one row by the general radix select (the first cand_k kept elements by key,
// ties to the lower index); *nsel their number and sm.gt_idx / sm.eq_idx their indices.
template <typename T>
__device__ int trie_general_select(const T* __restrict__ rp, int V, const RowStat& st, int cand_k, uint32_t floor_key,
                                   TrieGenSmem& sm, int* out_idx) {
  double above, bucket;
  const uint32_t kc = block_radix_pick<T, true>(rp, V, st, static_cast<double>(cand_k), floor_key, sm.radix, &above,
                                                &bucket);
  constexpr int kShift = sizeof(T) == 2 ? 16 : 0;  // a bf16 select fixes the top 16 key bits
  const uint32_t kcs = kc >> kShift;
  if (threadIdx.x == 0) sm.ngt = 0;
  __syncthreads();
  const int per = (V + blockDim.x - 1) / blockDim.x;
  const int v0 = min(V, static_cast<int>(threadIdx.x) * per), v1 = min(V, v0 + per);
  int n_eq = 0;
  for (int v = v0; v < v1; ++v) {
    const uint32_t key = fkey(load_elem(rp + v));
    if (key < floor_key) continue;
    const uint32_t ks = key >> kShift;
    if (ks > kcs) {
      const int slot = atomicAdd(&sm.ngt, 1);
      if (slot < kTrieMaxCand) sm.gt_idx[slot] = v;
    } else if (ks == kcs) {
      ++n_eq;
    }
  }
  double n_eq_total;
  const int eq_base = static_cast<int>(block_exclusive_scan(static_cast<double>(n_eq), sm.scan, &n_eq_total));
  const int ngt = min(sm.ngt, kTrieMaxCand);
  const int need = max(0, cand_k - ngt);
  if (eq_base < need) {
    int rank = eq_base;
    for (int v = v0; v < v1 && rank < need; ++v) {
      const uint32_t key = fkey(load_elem(rp + v));
      if (key >= floor_key && (key >> kShift) == kcs) sm.eq_idx[rank++] = v;
    }
  }
  __syncthreads();
  const int neq = min(need, static_cast<int>(n_eq_total));
  const int nc = min(cand_k, ngt + neq);
  for (int i = threadIdx.x; i < nc; i += blockDim.x) out_idx[i] = i < ngt ? sm.gt_idx[i] : sm.eq_idx[i - ngt];
  __syncthreads();
  return nc;
}

// Candidates of draft row `row`: cand_tok[row, r], cand_q[row, r] and their logits cand_l[row,
// r] for r < ncand[row] in rank order; ncand = -1 for a row with a data error. With `lazy`,
// the rows of requests with T > 0 and no cut (no top-p, no top-k) take their statistics from
// the kernel's own pass: every lane keeps its running maximum and sum of weights while it
// finds its block maxima, and the block combines them (a NaN or +inf anywhere, or no finite
// value, is a data error; every element is kept). The other rows read `stats`.
template <typename T>
__global__ void __launch_bounds__(kTrieThreads, 2) trie_candidates_kernel(
    const T* __restrict__ draft, int K, int V, const RowStat* __restrict__ stats, int lazy,
    const float* __restrict__ temperature, const float* __restrict__ top_p, const int32_t* __restrict__ top_k,
    int cand_k, int32_t* __restrict__ cand_tok, double* __restrict__ cand_q, double* __restrict__ cand_l,
    int32_t* __restrict__ ncand) {
  constexpr int N = Vec<T>::N;
  using Acc = VmaxAcc<T>;
  __shared__ TrieCandSmem smu;
  __shared__ int sel_idx[kTrieMaxCand];
  __shared__ double red_s[32];
  __shared__ float red_m[32];
  TrieFastSmem& sm = smu.fast;
  const int64_t row = blockIdx.x;
  const int req = static_cast<int>(row / K);
  const T* rp = draft + row * static_cast<int64_t>(V);
  const bool own = lazy && uncut_request(temperature, top_p, req) && request_k(top_k, req, V) == 0;
  RowStat st = own ? RowStat{} : stats[row];
  int32_t* tok = cand_tok + row * kTrieMaxCand;
  double* qo = cand_q + row * kTrieMaxCand;
  double* lo = cand_l + row * kTrieMaxCand;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (!own && st.status != 0) {
    if (threadIdx.x == 0) ncand[row] = -1;
    return;
  }
  if (!own && st.c == 0.0f) {  // greedy: a point mass on the argmax
    if (threadIdx.x == 0) {
      tok[0] = st.amax;
      qo[0] = 1.0;
      lo[0] = static_cast<double>(load_elem(rp + st.amax));
      ncand[row] = 1;
    }
    return;
  }
  const TrieGeom g = trie_geom(rp, V);
  const uint4 ninf = make_uint4(Acc::kNegInfWord, Acc::kNegInfWord, Acc::kNegInfWord, Acc::kNegInfWord);

  // pass 1: the maximum of every lane block (and, for a row whose statistics are found here,
  // the lane's running maximum and sum of weights)
  const float c_own = own ? temp_scale(temperature[req]) : 0.0f;
  TrieLaneSum ls{-INFINITY, 0.0, false};
  for (int i = 0; i < g.bpl; ++i) {
    typename Acc::type m = Acc::init();
    const int s0 = warp * g.spw + i * g.r, s1 = warp * g.spw + min((i + 1) * g.r, g.spw);
    for (int s = s0; s < s1; ++s) {
      uint4 w[kTrieVec];
#pragma unroll
      for (int j = 0; j < kTrieVec; ++j) {
        const int vi = (s * kTrieVec + j) * 32 + lane;
        w[j] = vi < g.nv ? __ldg(reinterpret_cast<const uint4*>(rp + g.a0 + vi * N)) : ninf;
      }
      typename Acc::type ms = Acc::init();
#pragma unroll
      for (int j = 0; j < kTrieVec; ++j) vmax_fold(w[j], ms, rp);
      vmax_merge(m, ms);
      if (own) {  // uniform
        ls.grow(vmax_value(ms), c_own);
        if (ls.M > -INFINITY) {
          float acc = 0.0f;
#pragma unroll
          for (int j = 0; j < kTrieVec; ++j) acc += vweight_sum(w[j], ls.M, c_own, rp);
          ls.s += static_cast<double>(acc);
        }
      }
    }
    sm.bkey[(warp * g.bpl + i) * 32 + lane] = fkey(vmax_value(m));
  }
  if (warp == 0) {  // the edge block: [0, a0) to lanes 0..15, [a1, V) to lanes 16..31
    const int v = lane < 16 ? lane : g.a1 + lane - 16;
    const bool in = lane < 16 ? v < g.a0 : v < V;
    const float xe = in ? load_elem(rp + v) : -INFINITY;
    if (own && in) {
      ls.grow(xe, c_own);
      if (ls.M > -INFINITY) ls.s += static_cast<double>(ex2((xe - ls.M) * c_own));
    }
    float x = xe;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmax_nan(x, __shfl_xor_sync(0xffffffffu, x, o));
    if (lane == 0) sm.bkey[g.nb] = fkey(x);
  }
  if (own) {  // the row's statistics from the lanes' (the same order in every thread)
    const float mw = warp_max(ls.M);
    const double sw = warp_sum(ls.M > -INFINITY ? ls.s * static_cast<double>(ex2((ls.M - mw) * c_own)) : 0.0);
    const bool bw = __any_sync(0xffffffffu, ls.bad);
    if (lane == 0) {
      red_m[warp] = bw ? NAN : mw;
      red_s[warp] = sw;
    }
  }
  if (threadIdx.x == 0) sm.ncand = 0;
  __syncthreads();
  if (own) {
    const int nw = blockDim.x >> 5;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmax_nan(M, red_m[w]);
    double S = 0.0;
    if (M > -INFINITY && M < INFINITY)
      for (int w = 0; w < nw; ++w)
        if (red_m[w] > -INFINITY) S += red_s[w] * static_cast<double>(ex2((red_m[w] - M) * c_own));
    st = RowStat{M, c_own, static_cast<float>(S), static_cast<float>(S), 0u, -1,
                 (M > -INFINITY && M < INFINITY && S > 0.0 && S < INFINITY) ? 0 : 1, 0};
    if (st.status != 0) {
      if (threadIdx.x == 0) ncand[row] = -1;
      return;
    }
  }
  // eligible: kept by the row's threshold and above -inf
  const uint32_t floor_key = max(st.tau, 0x00800000u);

  // the pivot: at most the cand_k-th largest eligible element (a bf16 value fixes the top 16
  // bits of its key, so two digits find it)
  uint32_t pivot = floor_key;
  if (g.nb + 1 > cand_k)
    pivot = max(pivot, smem_kth_largest(sm.bkey, g.nb + 1, cand_k, sizeof(T) == 2 ? 2 : 4, sm));

  // pass 2: every element at or above the pivot, from the blocks that hold one
  for (int b = threadIdx.x; b <= g.nb; b += blockDim.x) {
    if (sm.bkey[b] < pivot) continue;
    if (b == g.nb) {
      for (int v = 0; v < g.a0; ++v) {
        const uint32_t key = fkey(load_elem(rp + v));
        if (key >= pivot) trie_push(sm, key, v);
      }
      for (int v = g.a1; v < V; ++v) {
        const uint32_t key = fkey(load_elem(rp + v));
        if (key >= pivot) trie_push(sm, key, v);
      }
      continue;
    }
    const int bl = b & 31, wi = b >> 5, bw = wi / g.bpl, bi = wi - bw * g.bpl;
    const int s0 = bw * g.spw + bi * g.r, s1 = bw * g.spw + min((bi + 1) * g.r, g.spw);
    for (int s = s0; s < s1; ++s) {
      for (int j = 0; j < kTrieVec; ++j) {
        const int vi = (s * kTrieVec + j) * 32 + bl;
        if (vi >= g.nv) continue;
        const int e0 = g.a0 + vi * N;
        float x[8];
        Vec<T>::load(rp + e0, x);
#pragma unroll
        for (int e = 0; e < N; ++e) {
          const uint32_t key = fkey(x[e]);
          if (key >= pivot) trie_push(sm, key, e0 + e);
        }
      }
    }
  }
  __syncthreads();
  const int total = sm.ncand;
  int nsel;
  if (total <= kTrieCap) {
    // exact ranks among the collected elements (all distinct)
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
      const unsigned long long pk = sm.cand[i];
      int r = 0;
      for (int j = 0; j < total; ++j) r += sm.cand[j] > pk;
      if (r < cand_k) sm.top[r] = pk;
    }
    __syncthreads();
    nsel = min(cand_k, total);
    for (int i = threadIdx.x; i < nsel; i += blockDim.x) sel_idx[i] = static_cast<int>(~static_cast<uint32_t>(sm.top[i]));
    __syncthreads();
  } else {
    __syncthreads();
    nsel = trie_general_select(rp, V, st, cand_k, floor_key, smu.gen, sel_idx);
  }
  if (warp == 0) {
    double q = 0.0, lx = 0.0;
    int idx = -1;
    uint32_t key = 0u;
    if (lane < nsel) {
      idx = sel_idx[lane];
      const float x = load_elem(rp + idx);
      lx = static_cast<double>(x);
      key = fkey(x);
      q = exp2((static_cast<double>(x) - static_cast<double>(st.m)) * static_cast<double>(st.c)) /
          static_cast<double>(st.s_kept);
    }
    // rank: larger key first, then the lower index (the general select leaves them unordered)
    int rank = 0;
    for (int j = 0; j < nsel; ++j) {
      const int ij = __shfl_sync(0xffffffffu, idx, j);
      const uint32_t kj = __shfl_sync(0xffffffffu, key, j);
      if (lane < nsel && (kj > key || (kj == key && ij < idx))) ++rank;
    }
    // candidates whose q underflows to zero carry no probability: drop them (they rank last)
    const int nz = __popc(__ballot_sync(0xffffffffu, lane < nsel && q > 0.0));
    if (lane < nsel && rank < nz) {
      tok[rank] = idx;
      qo[rank] = q;
      lo[rank] = lx;
    }
    if (lane == 0) ncand[row] = nz;
  }
}

struct TrieSelSmem {
  double cq[kTrieMaxK][kTrieMaxCand];  // the request's candidates, position by position
  double cl[kTrieMaxK][kTrieMaxCand];
  int ct[kTrieMaxK][kTrieMaxCand];
  int nc[kTrieMaxK];
  int node_par[kTrieMaxPrefixes + 1];
  int node_dep[kTrieMaxPrefixes + 1];
  int node_tok[kTrieMaxPrefixes + 1];
  double node_score[kTrieMaxPrefixes + 1];
  uint8_t node_rank[kTrieMaxPrefixes + 1][kTrieMaxK];
};

// An offer: the best child not kept yet of node n, at depth d (0: no offer), candidate rank
// r, probability s and logit sum l.
struct TrieOffer {
  double s, l;
  int d, r, n;
};

__device__ __forceinline__ TrieOffer trie_shfl_xor(const TrieOffer& o, int m) {
  TrieOffer x;
  x.s = __shfl_xor_sync(0xffffffffu, o.s, m);
  x.l = __shfl_xor_sync(0xffffffffu, o.l, m);
  const int packed = __shfl_xor_sync(0xffffffffu, o.d | (o.r << 8) | (o.n << 16), m);
  x.d = packed & 0xFF;
  x.r = (packed >> 8) & 0xFF;
  x.n = packed >> 16;
  return x;
}

// Whether offer a precedes offer b: an offer precedes no offer; of different lengths, the
// higher fp64 probability, then the shorter; of one length, the larger logit sum (exact), then
// the smaller rank path (the parents' paths, then the offers' own ranks).
__device__ __forceinline__ bool trie_before(const TrieSelSmem& sm, const TrieOffer& a, const TrieOffer& b) {
  if (a.d == 0 || b.d == 0) return a.d != 0;
  if (a.d != b.d) return a.s > b.s || (a.s == b.s && a.d < b.d);
  if (a.l != b.l) return a.l > b.l;
  for (int j = 0; j + 1 < a.d; ++j) {
    const int ra = sm.node_rank[a.n][j], rb = sm.node_rank[b.n][j];
    if (ra != rb) return ra < rb;
  }
  return a.r < b.r;
}

// Node n's offer of its child of rank r (node n at depth dn, probability ns, logit sum nl).
__device__ __forceinline__ TrieOffer trie_offer(const TrieSelSmem& sm, int K, int n, int dn, double ns, double nl,
                                                int r) {
  TrieOffer o;
  o.n = n;
  o.r = r;
  if (dn < K && r < sm.nc[dn]) {
    o.d = dn + 1;
    o.s = ns * sm.cq[dn][r];
    o.l = nl + sm.cl[dn][r];
  } else {
    o.d = 0;
    o.s = o.l = 0.0;
  }
  return o;
}

constexpr int kTrieSlots = (kTrieMaxPrefixes + 1 + 31) / 32;  // nodes per lane

// Best-first choice of the n_prefixes most probable prefixes of request b (one warp). A
// node's children are offered in candidate-rank order, which is their order in the choice
// (a lower rank has a larger q, or an equal one and the smaller rank), so the frontier holds
// one offer per kept node. Lane l keeps the offers (and probabilities and logit sums) of
// nodes l, l + 32, l + 64 in registers; a butterfly over the lanes finds the best offer.
// Outputs [B, n_prefixes + 1]: parent, tokens, depth, score; unused slots -1 (score 0);
// out_nodes[b] the node count, or -1 when a draft row of the request has a data error.
__global__ void __launch_bounds__(32) trie_select_kernel(int K, int n_prefixes, const int32_t* __restrict__ cand_tok,
                                                         const double* __restrict__ cand_q,
                                                         const double* __restrict__ cand_l,
                                                         const int32_t* __restrict__ ncand,
                                                         int32_t* __restrict__ out_parent,
                                                         int32_t* __restrict__ out_tokens,
                                                         int32_t* __restrict__ out_depth,
                                                         double* __restrict__ out_score,
                                                         int32_t* __restrict__ out_nodes) {
  __shared__ TrieSelSmem sm;
  const int b = blockIdx.x, lane = threadIdx.x;
  const int cap = n_prefixes + 1;
  const int64_t r0 = static_cast<int64_t>(b) * K;
  int32_t* par = out_parent + static_cast<int64_t>(b) * cap;
  int32_t* tk = out_tokens + static_cast<int64_t>(b) * cap;
  int32_t* dp = out_depth + static_cast<int64_t>(b) * cap;
  double* sc = out_score ? out_score + static_cast<int64_t>(b) * cap : nullptr;
  bool bad = false;
  for (int i = lane; i < K; i += 32) {
    const int n = ncand[r0 + i];
    sm.nc[i] = n;
    bad |= n < 0;
  }
  bad = __any_sync(0xffffffffu, bad);
  for (int i = lane; i < cap; i += 32) {
    par[i] = -1;
    tk[i] = -1;
    dp[i] = -1;
    if (sc) sc[i] = 0.0;
  }
  if (bad) {
    if (lane == 0) out_nodes[b] = -1;
    return;
  }
#pragma unroll 4
  for (int d = 0; d < K; ++d) {
    const int64_t base = (r0 + d) * kTrieMaxCand;
    sm.cq[d][lane] = cand_q[base + lane];
    sm.cl[d][lane] = cand_l[base + lane];
    sm.ct[d][lane] = cand_tok[base + lane];
  }
  if (lane == 0) {
    sm.node_par[0] = -1;
    sm.node_dep[0] = 0;
    sm.node_tok[0] = -1;
    sm.node_score[0] = 1.0;
  }
  __syncwarp();
  // this lane's nodes: probability, logit sum, and offer
  double ns[kTrieSlots], nl[kTrieSlots];
  TrieOffer of[kTrieSlots];
#pragma unroll
  for (int k = 0; k < kTrieSlots; ++k) {
    ns[k] = nl[k] = 0.0;
    of[k].d = 0;
    of[k].r = of[k].n = 0;
    of[k].s = of[k].l = 0.0;
  }
  if (lane == 0) {
    ns[0] = 1.0;
    of[0] = trie_offer(sm, K, 0, 0, 1.0, 0.0, 0);
  }
  int nn = 1;
  while (nn < cap) {
    TrieOffer best = of[0];
#pragma unroll
    for (int k = 1; k < kTrieSlots; ++k)
      if (trie_before(sm, of[k], best)) best = of[k];
    // the lanes' best offers by the top 32 bits of their probabilities (positive doubles order
    // as their bits): a lead of two or more in those bits is a relative gap of at least 2^-20,
    // far above rounding, so it decides in the order trie_before gives (of one length,
    // probability and logit-sum order agree then: the prefixes share their normalisers);
    // offers within one of the lead go to the full comparison
    const uint32_t key =
        best.d == 0 ? 0u : max(1u, static_cast<uint32_t>(__double_as_longlong(best.s) >> 32));
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
    if (kmax == 0u) break;  // no offer left
    const unsigned tied = __ballot_sync(0xffffffffu, key != 0u && key + 1u >= kmax);
    if (__popc(tied) == 1) {
      const int src = __ffs(tied) - 1;
      best.s = __shfl_sync(0xffffffffu, best.s, src);
      best.l = __shfl_sync(0xffffffffu, best.l, src);
      const int packed = __shfl_sync(0xffffffffu, best.d | (best.r << 8) | (best.n << 16), src);
      best.d = packed & 0xFF;
      best.r = (packed >> 8) & 0xFF;
      best.n = packed >> 16;
    } else {
      if (!(key != 0u && key + 1u >= kmax)) best.d = 0;
#pragma unroll
      for (int m = 16; m > 0; m >>= 1) {
        const TrieOffer other = trie_shfl_xor(best, m);
        if (trie_before(sm, other, best)) best = other;
      }
    }
    const int p = best.n, d = best.d, r = best.r;
    // the new node nn: its rank path, record, and first offer
    if (lane + 1 < d) sm.node_rank[nn][lane] = sm.node_rank[p][lane];
    if (lane == d - 1) sm.node_rank[nn][lane] = static_cast<uint8_t>(r);
    if (lane == 0) {
      sm.node_par[nn] = p;
      sm.node_dep[nn] = d;
      sm.node_tok[nn] = sm.ct[d - 1][r];
      sm.node_score[nn] = best.s;
    }
#pragma unroll
    for (int k = 0; k < kTrieSlots; ++k) {
      if (lane + 32 * k == p) of[k] = trie_offer(sm, K, p, d - 1, ns[k], nl[k], r + 1);  // p's next child
      if (lane + 32 * k == nn) {
        ns[k] = best.s;
        nl[k] = best.l;
        of[k] = trie_offer(sm, K, nn, d, best.s, best.l, 0);
      }
    }
    __syncwarp();
    ++nn;
  }
  for (int i = lane; i < nn; i += 32) {
    par[i] = sm.node_par[i];
    tk[i] = sm.node_tok[i];
    dp[i] = sm.node_dep[i];
    if (sc) sc[i] = sm.node_score[i];
  }
  if (lane == 0) out_nodes[b] = nn;
}

// Weights of one loaded group of 8 (element e upward) with the removed tokens zeroed; rem is
// sorted ascending and *j the first entry not below e (advanced past the group).
template <typename T>
__device__ __forceinline__ void masked_weights(const JobRows<T, false>& J, const Raw8<T, false>& x, int e,
                                               const int* rem, int nrem, int* j, float (&w)[8]) {
  float pw[8];
  J.weights(x, w, pw);
  while (*j < nrem && rem[*j] < e + 8) {
    const int d = rem[*j] - e;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k == d) w[k] = 0.0f;
    ++*j;
  }
}

// Groups of 8 a lane keeps in flight in the draw without removed tokens.
template <typename T>
constexpr int kDetBatch = sizeof(T) == 2 ? 8 : 4;

// Warp total over [lo, hi) (lo a multiple of 8) of the kept weights without the tokens
// rem[0, nrem) (sorted ascending), and the last index with positive weight; every lane gets
// them.
template <typename T>
__device__ double warp_total_without(const JobRows<T, false>& J, int lo, int hi, const int* rem, int nrem,
                                     int* last_pos) {
  constexpr int NB = kDetBatch<T>;
  const int lane = threadIdx.x & 31;
  double tot = 0.0;
  int last = -1;
  int j = 0;
  while (j < nrem && rem[j] < lo + lane * 8) ++j;
  for (int g = lo; g < hi; g += NB * kGroup) {
    Raw8<T, false> x[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) J.load(g + b * kGroup + lane * 8, hi, x[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int e = g + b * kGroup + lane * 8;
      float w[8];
      masked_weights(J, x[b], e, rem, nrem, &j, w);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        tot += static_cast<double>(w[k]);
        if (w[k] > 0.0f) last = e + k;
      }
      while (j < nrem && rem[j] < e + kGroup) ++j;  // the lane's next group starts there
    }
  }
  *last_pos = __reduce_max_sync(0xffffffffu, last);
  return warp_sum(tot);
}

// Warp-level draw inside [lo, hi) (lo a multiple of 8) without the removed tokens: `base` is
// the weight before lo and `target` = u * Z. The first index whose inclusive prefix exceeds
// target, or -1 if none does.
template <typename T>
__device__ int warp_draw_without(const JobRows<T, false>& J, int lo, int hi, const int* rem, int nrem, double base,
                                 double target) {
  constexpr int NB = kDetBatch<T>;
  const int lane = threadIdx.x & 31;
  double Cb = base;
  for (int g = lo; g < hi; g += NB * kGroup) {
    Raw8<T, false> x[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) J.load(g + b * kGroup + lane * 8, hi, x[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int e = g + b * kGroup + lane * 8;
      int j = 0;
      while (j < nrem && rem[j] < e) ++j;
      float w[8];
      masked_weights(J, x[b], e, rem, nrem, &j, w);
      double vs = 0.0;
#pragma unroll
      for (int k = 0; k < 8; ++k) vs += static_cast<double>(w[k]);
      double incl = vs;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, Cb + incl > target);
      if (hit) {
        const int src = __ffs(hit) - 1;
        int y = -1, lastpos = -1;
        if (lane == src) {
          double C = Cb + (incl - vs);
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
  return -1;
}

// The sub-range of [lo, hi) that warp w of nw takes (spans a multiple of 8).
__device__ __forceinline__ void warp_span(int lo, int hi, int w, int nw, int& w0, int& w1) {
  const int span = (((hi - lo + nw - 1) / nw) + 7) & ~7;
  w0 = min(hi, lo + w * span);
  w1 = min(hi, w0 + span);
}

// Draw with uniform u from the kept weights of row J without the tokens rem[0, nrem) (sorted
// ascending): the first index, in vocabulary order, whose inclusive prefix exceeds u times the
// total. The warps total contiguous sub-ranges (coalesced groups of 8 per lane, fp64 sums);
// the sub-range holding the target is split among the warps again, and the warp whose part
// holds it scans that part. Returns the index to every thread, the last positive entry when
// rounding leaves none, -1 when no weight is left.
template <typename T>
__device__ int block_draw_without(const JobRows<T, false>& J, int V, const int* rem, int nrem, float u,
                                  DrawSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int w0, w1, last;
  warp_span(0, V, warp, nw, w0, w1);
  const double tot = warp_total_without(J, w0, w1, rem, nrem, &last);
  if (threadIdx.x == 0) { sm.y = -1; sm.last = -1; sm.owner = -1; }
  __syncthreads();
  if (lane == 0) {
    sm.wtot[warp] = tot;
    if (last >= 0) atomicMax(&sm.last, last);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double Z = 0.0;
    for (int i = 0; i < nw; ++i) Z += sm.wtot[i];
    const double tg = static_cast<double>(u) * Z;
    double C = 0.0;
    sm.target = tg;
    for (int i = 0; i < nw; ++i) {
      if (C <= tg && tg < C + sm.wtot[i]) { sm.owner = i; sm.c0 = C; break; }
      C += sm.wtot[i];
    }
  }
  __syncthreads();
  const int owner = sm.owner;
  if (owner >= 0) {
    // the owner's sub-range, split again among the warps
    int o0, o1, p0, p1, plast;
    warp_span(0, V, owner, nw, o0, o1);
    warp_span(o0, o1, warp, nw, p0, p1);
    const double pt = warp_total_without(J, p0, p1, rem, nrem, &plast);
    __syncthreads();
    if (lane == 0) sm.wtot[warp] = pt;
    __syncthreads();
    if (threadIdx.x == 0) {
      const double tg = sm.target;
      double C = sm.c0;
      int sub = -1;
      for (int i = 0; i < nw; ++i) {
        if (C <= tg && tg < C + sm.wtot[i]) { sub = i; break; }
        C += sm.wtot[i];
      }
      sm.owner = sub;
      sm.c0 = C;
    }
    __syncthreads();
    if (warp == sm.owner) {
      const int y = warp_draw_without(J, p0, p1, rem, nrem, sm.c0, sm.target);
      if (lane == 0) sm.y = y;
    }
  }
  __syncthreads();
  const int y = sm.y >= 0 ? sm.y : sm.last;  // past every sub-range (rounding): last positive entry
  __syncthreads();
  return y;
}

// Tree walk under the deterministic-candidate rule (children fixed in advance, as the
// candidate trie's are): at a node with verifier distribution p, child t is accepted iff
// u < p(t) / R, R the mass of p left after removing the siblings rejected before it; a
// rejection removes t (r = p without the removed tokens, renormalised). Where the walk stops,
// the final token is drawn from that r with u_resid of the node. No draft row is read, and a
// rejection needs no pass over the vocabulary. One CTA per trie; ts = statistics records of
// the verifier rows (every row's, found in parallel beforehand: a walk can be as deep as the
// block, so no per-node pass sits on its chain). Every node's p(token) under its parent's row
// and its uniform are read by the whole CTA before the walk; the walk itself is one warp
// (children listed by ballots, the accept tests in child order on one lane, all from shared
// memory); the final draw is one coalesced block draw.
template <typename T>
__global__ void __launch_bounds__(kTreeThreads, 1) tree_walk_det_kernel(
    const T* __restrict__ tgt, int V, const int32_t* __restrict__ offs, const int32_t* __restrict__ parent,
    const int32_t* __restrict__ tokens, const RowStat* __restrict__ ts, const float* __restrict__ u_acc,
    const float* __restrict__ u_res, int max_depth, int32_t* __restrict__ out_path, int32_t* __restrict__ out_tokens,
    int32_t* __restrict__ out_len) {
  __shared__ int depth[kMaxNodes];
  __shared__ int spar[kMaxNodes];
  __shared__ int stok[kMaxNodes];
  __shared__ double pn[kMaxNodes];  // node c's p(token) under its parent's verifier row
  __shared__ float un[kMaxNodes];   // node c's u_accept
  __shared__ int rowf[kMaxNodes];   // node c's own row: -2 data error, -1 sampling, else the greedy argmax
  __shared__ int ch[kMaxChildren];
  __shared__ int removed[kMaxChildren];
  __shared__ DrawSmem dsm;
  __shared__ int sh_bad, sh_cur, sh_len, sh_draw, sh_y, sh_nrem;
  const int b = blockIdx.x;
  const int n0 = offs[b], n = offs[b + 1] - n0;
  int32_t* path = out_path + static_cast<size_t>(b) * max_depth;
  int32_t* toks = out_tokens + static_cast<size_t>(b) * (max_depth + 1);

  const bool size_ok = n > 0 && n <= kMaxNodes;
  if (size_ok)
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
      spar[c] = parent[n0 + c];
      stok[c] = tokens[n0 + c];
    }
  __syncthreads();
  if (threadIdx.x == 0) {
    int bad = size_ok ? (spar[0] != -1) : 1;
    if (!bad) depth[0] = 0;
    for (int c = 1; c < n && !bad; ++c) {
      const int pa = spar[c], t = stok[c];
      if (pa < 0 || pa >= c || t < 0 || t >= V) { bad = 1; break; }
      depth[c] = depth[pa] + 1;
      if (depth[c] > max_depth) bad = 1;
    }
    sh_bad = bad;
  }
  __syncthreads();
  if (!sh_bad)
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
      const RowStat own = ts[n0 + c];
      rowf[c] = own.status != 0 ? -2 : (own.c == 0.0f ? own.amax : -1);
      if (c > 0) {
        const int pa = spar[c];
        const RowStat sp = ts[n0 + pa];
        pn[c] = sp.status == 0 && sp.c != 0.0f
                    ? static_cast<double>(kept_weight(sp, load_elem(tgt + static_cast<size_t>(n0 + pa) * V + stok[c]))) /
                          static_cast<double>(sp.s_kept)
                    : 0.0;
        un[c] = u_acc[n0 + c];
      }
    }
  __syncthreads();

  if (threadIdx.x < 32 && !sh_bad) {  // the walk: one warp
    const int lane = threadIdx.x;
    int cur = 0, len = 0, bad = 0, draw = 0, y = -1, nrem = 0;
    while (true) {
      const int f = rowf[cur];
      if (f == -2) { bad = 1; break; }
      int nch = 0;
      for (int c0 = cur + 1; c0 < n; c0 += 32) {
        const int c = c0 + lane;
        const bool is = c < n && spar[c] == cur;
        const unsigned m = __ballot_sync(0xffffffffu, is);
        const int pos = nch + __popc(m & ((1u << lane) - 1u));
        if (is && pos < kMaxChildren) ch[pos] = c;
        nch += __popc(m);
      }
      if (nch > kMaxChildren) { bad = 1; break; }
      __syncwarp();
      int next = -1;
      if (lane == 0) {
        if (f >= 0) {  // greedy: follow the child carrying the verifier argmax
          for (int k = 0; k < nch; ++k)
            if (stok[ch[k]] == f) { next = ch[k]; break; }
          y = f;
        } else {
          double R = 1.0;  // mass of p left
          nrem = 0;
          for (int k = 0; k < nch; ++k) {
            const int c = ch[k], t = stok[c];
            bool gone = false;
            for (int i = 0; i < nrem; ++i) gone |= removed[i] == t;
            const double pt = gone ? 0.0 : pn[c];
            if (R > 0.0 && static_cast<double>(un[c]) * R < pt) { next = c; break; }
            if (!gone) {
              removed[nrem++] = t;
              R -= pt;
            }
          }
        }
        if (next >= 0) {
          path[len] = next;
          toks[len] = stok[next];
        }
      }
      next = __shfl_sync(0xffffffffu, next, 0);
      if (next < 0) {
        draw = f == -1;
        break;
      }
      cur = next;
      ++len;
    }
    if (lane == 0) {
      if (draw)  // ascending order for the draw
        for (int i = 1; i < nrem; ++i) {
          const int t = removed[i];
          int k = i - 1;
          while (k >= 0 && removed[k] > t) { removed[k + 1] = removed[k]; --k; }
          removed[k + 1] = t;
        }
      sh_bad = bad;
      sh_cur = cur;
      sh_len = len;
      sh_draw = draw;
      sh_y = y;
      sh_nrem = nrem;
    }
  }
  __syncthreads();
  if (!sh_bad && sh_draw) {  // final draw from p without the removed tokens
    const int cur = sh_cur;
    const T* rp = tgt + static_cast<size_t>(n0 + cur) * V;
    const RowStat sp = ts[n0 + cur];
    JobRows<T, false> J;
    J.init(rp, sp, nullptr, sp);
    const int y = block_draw_without(J, V, removed, sh_nrem, u_res[n0 + cur], dsm);
    if (threadIdx.x == 0) sh_y = y;
  }
  __syncthreads();

  if (threadIdx.x == 0) {
    if (sh_bad) {
      for (int i = 0; i < max_depth; ++i) path[i] = -1;
      for (int i = 0; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = -1;
    } else {
      const int len = sh_len;
      for (int i = len; i < max_depth; ++i) path[i] = -1;
      toks[len] = sh_y;
      for (int i = len + 1; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = len;
    }
  }
}

}  // namespace psi
