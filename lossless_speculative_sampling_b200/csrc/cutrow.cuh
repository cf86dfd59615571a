// cutrow.cuh -- rows of requests with a cut (top-p below 1 or an active top-k, at T > 0),
// bf16, in one pass over HBM.
//
// The cut keeps every token whose logit is at least tau, the largest logit value t of the row
// with mass(l >= t) >= top_p (review page of arXiv 2609.04010: the samplers take --top-p with
// --temperature; ties are kept together), and renormalises over the kept set; with a top-k
// (the README's --top-k), mass and tail are those of the tokens at or above the k-th largest
// logit. Every element with one bf16 value has one weight, so counting the elements of each
// value just below the row maximum gives the masses the cut is decided on (window_pick,
// topp.cuh). The two-pass select counts them after a statistics pass has found the maximum;
// here the counts are taken in the same pass that finds it.
//
// One CTA per row at a time, persistent over the rows, three CTAs per SM. Warp w of the CTA
// streams a contiguous range of the row once from HBM (five 16-byte loads per lane per step;
// the 24 warps of an SM keep the loads in flight) and keeps, over its range:
//   - the running maximum M (NaN-propagating, bf16 pairs compared packed) and, per lane, the
//     fp64 sum of 2^((x - M) c), rescaled whenever M grows;
//   - a ring of kCrRing counters in shared memory, counter d counting the elements whose
//     16-bit order key is lower + d. The ring's top key, lower + kCrRing - 1, is set kCrHead
//     keys above the warp's maximum at its first finite value and moved up (counters shifted)
//     only when the maximum passes it, so the counters cover the kTpWindow keys below the
//     warp's maximum at every moment, hence also the kTpWindow keys below the row's maximum at
//     the end.
// The CTA then combines its warps: the maximum m, the normaliser s (fp64), and the counts of
// the window below m, from which window_pick finds tau and the kept mass. A draft row draws
// its token at once: the warps' kept masses (counts x weights) give the warp whose range holds
// u * Z, and only that range is read again (from L2) to find the token. A verifier row (or a
// draft row that a verification reads) writes its record and arrives on its request's
// counter; the last arrival runs the accept tests. A row whose cut lies outside the window is
// finished in place by the general selects of topp.cuh and stats.cuh (the row is read again).
// The same CTAs take fp32 rows with the general selects throughout.
#pragma once

#include "common.cuh"
#include "finish.cuh"
#include "linear.cuh"
#include "sample.cuh"
#include "stats.cuh"
#include "topp.cuh"

namespace psi {

constexpr int kCrWarps = 8;                   // warps per CTA, each one contiguous range of the row
constexpr int kCrThreads = kCrWarps * 32;
constexpr int kCrHead = 224;                  // keys of headroom above a warp's maximum at its ring's top
constexpr int kCrRing = kTpWindow + kCrHead;  // counters per warp
constexpr int kCrVec = 5;                     // 16-byte vectors per lane per step
static_assert(kCrRing % 32 == 0, "ring shifts move 32 counters per step");

enum CutMode : int { kCutSample = 0, kCutVerify = 1, kCutStats = 2 };

// Rows of one cut-row launch: rows [0, rows_a) of tensor a (per_a rows per request), then
// rows [0, rows_b) of tensor b (per_b rows per request). Sampling: a = the draft rows [B, K].
// Verification: a = the verifier rows [B, K+1], b = the draft rows [B, K] when the call reads
// them. Row statistics: a = the rows [B, K].
struct CutArgs {
  int mode;
  int V;
  int rows_a, per_a, rows_b, per_b;
  const float* temperature;
  const float* top_p;
  const int32_t* top_k;  // per request, or null (off)
  const float* u;        // kCutSample: one uniform per row
  int32_t* out_tokens;   // kCutSample: the drawn token per row
  float* out_q;          // kCutSample: its kept probability (nullable)
  RowStat* stats_a;      // records of tensor a's rows
  RowStat* stats_b;      // records of tensor b's rows
};

struct CrSmem {
  uint32_t ring[kCrWarps][kCrRing + 32];  // the counters, then one discard counter per lane
  float wm[kCrWarps];     // the warps' maxima (-inf: no finite value in the range)
  double ws[kCrWarps];    // the warps' sums, relative to their own maxima
  uint32_t wl[kCrWarps];  // the warps' ring lower keys (0: no finite value)
  int wbad[kCrWarps];     // a NaN or +inf logit in the warp's range
  double wk[kCrWarps];    // the warps' kept masses (draft rows)
  double scan[40];
  double tgt, base, dtarget, dbase;
  int bin, flag, dwarp;
  DrawSmem draw;
};

// One warp's running state over its range. Per lane: the running maximum M of the lane's own
// values and the fp64 sum of 2^((x - M) c) over them (rescaled when M grows), and whether a NaN
// or +inf logit was seen. Uniform across the warp: the ring's keys.
struct CrLane {
  float M;         // this lane's running maximum; -inf before its first finite value
  float mref;      // M, or 0 while M is -inf (so that -inf values weigh exp2(-inf) = 0)
  double s;        // this lane's sum of 2^((x - M) c)
  bool bad;        // this lane saw a NaN or +inf logit
  uint32_t top;    // the ring's top key (uniform); 0 before the warp's first finite value
  uint32_t lower;  // its lowest key, top - kCrRing + 1
  uint32_t nl16;   // -((lower - 0x8000) << 16): the positive-only path's offset of raw value bits
  bool fast;       // every key the ring covers belongs to a positive value
  uint32_t dl;     // (kCrRing + lane) << 16: this lane's discard counter, as a clamp
  uint32_t ra;     // shared address of the warp's ring
};

// The 16-bit order key of a bf16 bit pattern (fkey(x) >> 16 of the widened value; -0 and +0
// share the key of +0).
__device__ __forceinline__ uint32_t key16_bits(uint32_t h) {
  return (h & 0x8000u) ? (h == 0x8000u ? 0x8000u : (~h & 0xFFFFu)) : (h | 0x8000u);
}

// Some lane's maximum passed the ring's top key (or the warp's first finite value arrived): the
// top moves kCrHead keys above the warp's maximum key kmax; returns the new top. With the top
// (and the lower key) up by delta, counter d counts key lower + delta + d: it takes old counter
// d + delta, or zero. Warp-uniform; rare, but inlined: a call inside the streaming loop would
// make the loop keep its values in memory across it.
__device__ __forceinline__ uint32_t cr_rebase(uint32_t top, uint32_t kmax, uint32_t* ring) {
  const int lane = threadIdx.x & 31;
  const uint32_t nt = min(kmax + static_cast<uint32_t>(kCrHead), 0xFFFFu);
  const uint32_t delta = top == 0u ? static_cast<uint32_t>(kCrRing) : nt - top;
  __syncwarp();  // the reductions of earlier steps are visible to every lane
  if (delta >= static_cast<uint32_t>(kCrRing)) {
    for (int d = lane; d < kCrRing; d += 32) ring[d] = 0u;
  } else {
    // bottom up, 32 counters per step: a step reads above what earlier steps wrote
    for (int b = 0; b < kCrRing; b += 32) {
      const int d = b + lane;
      const uint32_t v = d + static_cast<int>(delta) < kCrRing ? ring[d + static_cast<int>(delta)] : 0u;
      __syncwarp();
      ring[d] = v;
      __syncwarp();
    }
  }
  __syncwarp();
  return nt;
}

// One to ring counter d = h - lb of a positive bf16 value h (the ring holds positive values
// only; lb = lower - 0x8000 is the raw bits of its lowest value), taken from the value's bits
// xf = h << 16 as a float's upper half: t = xf - (lb << 16) = d << 16, one add of nl16 =
// -(lb << 16). A value below the ring wraps to a large t; a negative value (xf >= 2^31) gives
// t >= 2^31 - (lb << 16) >= kCrRing << 16, as lb <= 0xFFFF - (kCrRing - 1) - 0x8000.
// Either lands on a discard counter: t is clamped to this lane's dl =
// (kCrRing + lane) << 16, so that every value takes one unconditional reduction (a predicated
// one costs a branch around it). The counter's shared address is ra + 4 d = ra + (t >> 14).
// No memory effect is declared (see count_if_below).
__device__ __forceinline__ void cr_count_pos(uint32_t xf, uint32_t nl16, uint32_t dl, uint32_t ra) {
  asm volatile(
      "{\n"
      " .reg .u32 t;\n"
      " add.u32 t, %0, %1;\n"
      " min.u32 t, t, %2;\n"
      " shr.u32 t, t, 14;\n"
      " add.u32 t, t, %3;\n"
      " red.shared.add.u32 [t], 1;\n"
      "}" ::"r"(xf),
      "r"(nl16), "r"(dl), "r"(ra));
}

// One step of a warp's range: kCrVec 16-byte vectors per lane (a range's last step and its
// scalar edges padded with -inf, which weighs nothing and, on the positive-only path, lands on a
// discard counter; rows whose window could reach -inf's key take the general select).
struct CrStep {
  uint4 v[kCrVec];
};

// Sums and counts of one step. FAST: the ring holds positive values only (counted from the raw
// bits); otherwise every value is mapped to its 16-bit order key first.
template <bool FAST>
__device__ __forceinline__ void cr_absorb_sum(CrLane& L, const CrStep& raw, float c, uint32_t* ring) {
  const uint32_t nl16 = L.nl16, dl = L.dl, ra = L.ra;
  // weights 2^((x - M) c) with the difference and the product each rounded, the arithmetic of
  // every other weight in the library (x c - M c in one fused step would round M c once, off by
  // up to half an ulp of M c for every weight alike, and overflow for |M| near the float range)
  const f32x2 mm = pack2(L.mref, L.mref), cc = pack2(c, c);
  f32x2 p0 = pack2(0.0f, 0.0f), p1 = p0;
#pragma unroll
  for (int j = 0; j < kCrVec; ++j) {
    const uint32_t w[4] = {raw.v[j].x, raw.v[j].y, raw.v[j].z, raw.v[j].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t lo = w[q] << 16, hi = w[q] & 0xFFFF0000u;  // the two values as float bits
      float d0, d1;
      unpack2(mul2(sub2(pack2(__uint_as_float(lo), __uint_as_float(hi)), mm), cc), d0, d1);
      if (q & 1) p1 = add2(p1, pack2(ex2(d0), ex2(d1)));
      else p0 = add2(p0, pack2(ex2(d0), ex2(d1)));
      if (FAST) {
        cr_count_pos(lo, nl16, dl, ra);
        cr_count_pos(hi, nl16, dl, ra);
      } else {
        count_if_below(ring, key16_bits(lo >> 16) - L.lower, kCrRing);
        count_if_below(ring, key16_bits(hi >> 16) - L.lower, kCrRing);
      }
    }
  }
  float a0, a1, a2, a3;
  unpack2(p0, a0, a1);
  unpack2(p1, a2, a3);
  L.s += (static_cast<double>(a0) + static_cast<double>(a1)) + (static_cast<double>(a2) + static_cast<double>(a3));
}

// The per-step bookkeeping: this lane's maximum of the step (NaN and +inf flagged), the ring's
// top following the warp's maximum (a vote per step; the move itself is rare), the lane's sum
// rescaled when its maximum grows.
__device__ __forceinline__ void cr_step_max(CrLane& L, const CrStep& raw, float c, uint32_t* ring) {
  uint32_t pm = 0xFF80FF80u;  // packed bf16 pair (-inf, -inf)
#pragma unroll
  for (int j = 0; j < kCrVec; ++j)
    pm = bmax2(pm, bmax2(bmax2(raw.v[j].x, raw.v[j].y), bmax2(raw.v[j].z, raw.v[j].w)));
  const float lm = fmax_nan(__uint_as_float(pm << 16), __uint_as_float(pm & 0xFFFF0000u));
  const bool finite = lm > -INFINITY && lm < INFINITY;
  L.bad |= !(lm < INFINITY);  // NaN or +inf
  const uint32_t lk = finite ? fkey(lm) >> 16 : 0u;
  if (__any_sync(0xffffffffu, lk > L.top)) {
    uint32_t wk = lk;
#pragma unroll
    for (int o = 16; o; o >>= 1) wk = max(wk, __shfl_xor_sync(0xffffffffu, wk, o));
    L.top = cr_rebase(L.top, wk, ring);
    L.lower = L.top - static_cast<uint32_t>(kCrRing - 1);
    L.fast = L.lower > 0x8000u;
    L.nl16 = (0x8000u - L.lower) << 16;
  }
  if (finite && lm > L.M) {  // this lane's maximum grows
    if (L.M > -INFINITY) L.s *= static_cast<double>(ex2((L.M - lm) * c));
    L.M = lm;
    L.mref = lm;
  }
}

// One step: bookkeeping, then sums and counts on the path the ring's keys allow (uniform).
// Everything is inlined: a call inside the streaming loop would make the loop keep its values
// in memory across it.
__device__ __forceinline__ void cr_absorb(CrLane& L, const CrStep& raw, float c, uint32_t* ring) {
  cr_step_max(L, raw, c, ring);
  if (L.fast) cr_absorb_sum<true>(L, raw, c, ring);
  else cr_absorb_sum<false>(L, raw, c, ring);
}

// This warp's range of row rp: the aligned body [a0, a1) split into kCrWarps runs of whole
// 16-byte vectors, warp 0 also owning the head [0, a0) and the last warp the tail [a1, V).
struct CrRange {
  int lo, hi;      // elements of the row this warp owns (in index order)
  int v0, v1;      // its body vectors [v0, v1) (vector i = elements a0 + 8i .. a0 + 8i + 7)
  int e0, e1;      // its scalar edge elements [e0, e1) (empty for middle warps)
};

template <typename T>
__device__ __forceinline__ CrRange cr_range(const T* rp, int V, int w) {
  int a0, a1;
  vec_range(rp, 0, V, a0, a1);
  const int nvec = (a1 - a0) / 8;
  const int qv = (nvec + kCrWarps - 1) / kCrWarps;
  CrRange r;
  r.v0 = min(nvec, w * qv);
  r.v1 = min(nvec, (w + 1) * qv);
  r.lo = w == 0 ? 0 : a0 + 8 * r.v0;
  r.hi = w == kCrWarps - 1 ? V : a0 + 8 * r.v1;
  r.e0 = w == 0 ? 0 : (w == kCrWarps - 1 ? a1 : 0);
  r.e1 = w == 0 ? a0 : (w == kCrWarps - 1 ? V : 0);
  return r;
}

// Warp w streams its range of row rp (bf16) into L and its ring. Not inlined: the streaming
// loop gets the registers to itself, apart from the row-end work of the caller.
__device__ __noinline__ CrLane cr_stream(const __nv_bfloat16* __restrict__ rp, int V, const CrRange r, float c,
                                         uint32_t* ring) {
  const int lane = threadIdx.x & 31;
  CrLane L{-INFINITY, 0.0f, 0.0, false, 0u, 0u, 0u, false, 0u, 0u};
  L.dl = static_cast<uint32_t>(kCrRing + lane) << 16;
  L.ra = smem_u32(ring);
  constexpr uint32_t kNegInf2 = 0xFF80FF80u;  // packed bf16 pair (-inf, -inf)
  int a0, a1;
  vec_range(rp, 0, V, a0, a1);
  const uint4* body = reinterpret_cast<const uint4*>(rp + a0);
  // scalar edges first (at most 7 elements): one element per lane, the rest -inf
  if (r.e1 > r.e0) {
    CrStep raw;
    const int e = r.e0 + lane;
    const uint32_t h = e < r.e1 ? static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(rp)[e]) : 0xFF80u;
    raw.v[0] = make_uint4(h | 0xFF800000u, kNegInf2, kNegInf2, kNegInf2);
#pragma unroll
    for (int j = 1; j < kCrVec; ++j) raw.v[j] = make_uint4(kNegInf2, kNegInf2, kNegInf2, kNegInf2);
    cr_absorb(L, raw, c, ring);
  }
  constexpr int kStep = 32 * kCrVec;  // vectors per warp step
  const int n = r.v1 - r.v0;
  const int steps = (n + kStep - 1) / kStep;
  auto load = [&](CrStep& buf, int s) {
    const uint4* p = body + r.v0 + s * kStep + lane;
    if ((s + 1) * kStep <= n) {  // a full step (warp-uniform)
#pragma unroll
      for (int j = 0; j < kCrVec; ++j) buf.v[j] = __ldg(p + j * 32);
    } else {  // the range's last step: -inf past its end
#pragma unroll
      for (int j = 0; j < kCrVec; ++j)
        buf.v[j] = s * kStep + j * 32 + lane < n ? __ldg(p + j * 32) : make_uint4(kNegInf2, kNegInf2, kNegInf2, kNegInf2);
    }
  };
  CrStep A;
  for (int s = 0; s < steps; ++s) {
    load(A, s);
    // the warp's next step (2.5 KB contiguous) brought into L2 while this one is reduced: its
    // loads then wait on L2 rather than HBM (measured: 2.03 against 2.10 ms per step of
    // B=512, K=16, top-p 0.95)
    if (lane == 0 && s + 1 < steps) {
      const uint4* pf = body + r.v0 + (s + 1) * kStep;
      const uint32_t bytes = static_cast<uint32_t>(min(kStep, n - (s + 1) * kStep)) * 16u;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(pf), "r"(bytes) : "memory");
    }
    cr_absorb(L, A, c, ring);
  }
  __syncwarp();  // the ring's reductions are complete before the caller's barrier
  return L;
}

// The count of window key `key` in the warps' rings (warps without a finite value add nothing;
// a key above a warp's base has no element in its range).
__device__ __forceinline__ uint32_t cr_count(const CrSmem& sm, uint32_t key) {
  uint32_t c = 0u;
#pragma unroll
  for (int w = 0; w < kCrWarps; ++w) {
    const uint32_t d = key - sm.wl[w];
    if (sm.wm[w] > -INFINITY && d < static_cast<uint32_t>(kCrRing)) c += sm.ring[w][d];
  }
  return c;
}

// Shared memory of the general selects of a bf16 row whose cut lies outside the window: the
// block histogram select (and the radix selects inside it), the block draw.
struct GenSmem {
  ToppSmem topp;
  DrawSmem draw;
  int flag;
};

// Shared memory of a CTA of the row kernels: bf16, the one-pass cut rows or the general
// selects; fp32, the general selects from the streaming pass's partials.
template <typename T>
union CutSmem;
template <>
union CutSmem<__nv_bfloat16> {
  CrSmem cr;
  GenSmem gen;
};
template <>
union CutSmem<float> {
  TpSmem tp;
};

// CTAs per SM of the row kernels. bf16: three (24 warps; 80 registers a thread, which the
// single-buffered streaming loop fits without spilling, and 74.6 KB of shared memory each);
// more warps hide the loads better than a second register buffer per warp did (measured:
// 2.10 against 2.25 ms per step of B=512, K=16, top-p 0.95). fp32: two.
template <typename T>
constexpr int kRowCtas = sizeof(T) == 2 ? 3 : 2;

// Finish a row once its record st is known: the draw (sampling), the arrival and, for the last
// arrival of a request, the accept tests (verification), or the record alone (statistics).
// For a draft row whose draw the caller has made, y and q are its token and probability.
template <typename T>
__device__ __forceinline__ void cut_row_finish(const T* __restrict__ A, const T* __restrict__ Bt, const CutArgs& a,
                                               const VerifyArgs& va, RowStat* rec, const RowStat& st, int row,
                                               int req, int y, float q, int* flag) {
  if (a.mode == kCutSample) {
    if (threadIdx.x == 0) {
      *rec = st;
      a.out_tokens[row] = y;
      if (a.out_q) a.out_q[row] = q;
    }
  } else if (a.mode == kCutVerify) {
    if (threadIdx.x == 0) *rec = st;
    const int per_req = (va.K + 1) + (va.stream_draft ? va.K : 0);
    if (block_arrive_last(&va.cnt[req], per_req, flag) && threadIdx.x < 32)
      warp_decide_request<T>(req, A, Bt, va.K, a.V, va.tokens, va.stats_t, va.stream_draft ? va.stats_d : va.dstats_in,
                             va.u_acc, va.u_res, va.out_tokens, va.out_len, va.out_p, va.out_q, va.jobs);
  } else if (threadIdx.x == 0) {
    *rec = st;
  }
}

// A row's cut by the general selects: top-k by the count-then-mass radix select (m and c from
// the one-pass statistics in st, or from the partials), top-p by tp_row_stats (which finds m and
// s itself for bf16 rows; fp32 rows take them from the partials); then the draw, the arrival or
// the record. Not inlined: a rare path, kept out of the streaming loop's registers.
template <typename T>
__device__ __noinline__ void cut_row_general(const T* __restrict__ A, const T* __restrict__ Bt, const CutArgs& a,
                                             const VerifyArgs& va, const Partial* __restrict__ parts_a,
                                             const Partial* __restrict__ parts_b, CutSmem<T>& smu, const T* rp,
                                             RowStat* rec, RowStat st, bool in_b, int row, int req, float Tv,
                                             float tp, int k, float u) {
  const int V = a.V;
  int y = -1;
  float q = -1.0f;
  if constexpr (sizeof(T) == 2) {
    // m, c and s from the one pass; the threshold by the block selects, the draw over the row
    GenSmem& sm = smu.gen;
    if (k > 0) block_topk_topp_radix<T>(rp, V, tp, k, st, sm.topp.radix);
    else block_topp_select<T>(rp, V, tp, st, sm.topp);
    if (a.mode == kCutSample && st.status == 0) {
      JobRows<T, false> J;
      J.init(rp, st, nullptr, st);
      y = block_draw_range(J, 0, V, 0.0, -1.0, u, sm.draw);
      if (y >= 0) q = kept_weight(st, load_elem(rp + y)) / st.s_kept;
    }
    cut_row_finish<T>(A, Bt, a, va, rec, st, row, req, y, q, &sm.flag);
  } else {
    (void)Tv;
    TpSmem& sm = smu.tp;
    const Partial* pp = (in_b ? parts_b : parts_a) + static_cast<size_t>(row) * nchunks_for(V);
    st = tp_row_stats_partials(rp, V, Tv, tp, k, pp, sm);
    if (a.mode == kCutSample && st.status == 0) y = tp_row_draw(rp, V, st, u, sm, &q);
    cut_row_finish<T>(A, Bt, a, va, rec, st, row, req, y, q, &sm.flag);
  }
  __syncthreads();
}

// The rows of cut requests of a launch, one CTA per row at a time: CTA `cta` of `nctas` takes
// rows cta, cta + nctas, ... (rows of other requests are skipped). bf16 rows take the
// one-pass path, with the general selects (tp_row_stats, block_topk_topp_radix) for a cut
// outside the window; fp32 rows take the general selects throughout (their maximum and
// normaliser come from the streaming pass's partials, parts_a / parts_b).
template <typename T>
__device__ void cut_rows_cta(const T* __restrict__ A, const T* __restrict__ Bt, const CutArgs& a,
                             const VerifyArgs& va, const Partial* __restrict__ parts_a,
                             const Partial* __restrict__ parts_b, int cta, int nctas, CutSmem<T>& smu) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int V = a.V;
  const int total = a.rows_a + a.rows_b;
  for (int g = cta; g < total; g += nctas) {
    const bool in_b = g >= a.rows_a;
    const int row = in_b ? g - a.rows_a : g;
    const int req = in_b ? row / a.per_b : row / a.per_a;
    if (!request_cut(a.temperature, a.top_p, a.top_k, req, V)) continue;  // uniform
    const T* rp = (in_b ? Bt : A) + static_cast<size_t>(row) * V;
    RowStat* rec = (in_b ? a.stats_b : a.stats_a) + row;
    const float Tv = a.temperature[req];
    const float c = temp_scale(Tv);
    const float tp = a.top_p[req];
    const int k = request_k(a.top_k, req, V);
    const float u = a.mode == kCutSample ? a.u[row] : 0.0f;
    RowStat st{};
    if constexpr (sizeof(T) == 2) {
      CrSmem& sm = smu.cr;
      uint32_t* ring = sm.ring[warp];
      // every warp streams its range
      const CrRange r = cr_range(rp, V, warp);
      const CrLane L = cr_stream(reinterpret_cast<const __nv_bfloat16*>(rp), V, r, c, ring);
      // the warp: its maximum, and the lanes' sums brought to it
      const float mw = warp_max(L.M);
      const double sw = warp_sum(L.M > -INFINITY ? L.s * static_cast<double>(ex2((L.M - mw) * c)) : 0.0);
      const bool badw = __any_sync(0xffffffffu, L.bad);
      if (lane == 0) {
        sm.wm[warp] = mw;
        sm.ws[warp] = sw;
        sm.wl[warp] = L.top != 0u ? L.lower : 0u;
        sm.wbad[warp] = badw ? 1 : 0;
      }
      __syncthreads();
      // the row: maximum, normaliser, status (the same arithmetic in every thread)
      float m = -INFINITY;
      bool bad = !(Tv >= 0.0f && Tv < INFINITY);
#pragma unroll
      for (int w = 0; w < kCrWarps; ++w) {
        bad |= sm.wbad[w] != 0;
        m = fmax_nan(m, sm.wm[w]);
      }
      bad |= !(m > -INFINITY) || !(m < INFINITY);
      double S = 0.0;
      if (!bad) {
#pragma unroll
        for (int w = 0; w < kCrWarps; ++w)
          if (sm.wm[w] > -INFINITY) S += sm.ws[w] * static_cast<double>(ex2((sm.wm[w] - m) * c));
      }
      st = RowStat{m, c, static_cast<float>(S), static_cast<float>(S), 0u, -1, bad ? 1 : 0, 0};
      const uint32_t km = bad ? 0u : fkey(m) >> 16;
      // a window reaching the keys of -inf (rows of huge negative logits) takes the general select
      bool general = !bad && km < static_cast<uint32_t>(kTpWindow) + 0x80u;
      if (!bad && !general)
        general = !window_pick<kCrThreads>(
            km, tp, k, st, [&](int o) { return cr_count(sm, km - static_cast<uint32_t>(o)); }, sm.scan, &sm.bin,
            &sm.tgt, &sm.base);
      if (!general) {
        int y = -1;
        float q = -1.0f;
        if (a.mode == kCutSample && !bad) {
          // kept mass of each warp's range from its counts (keys ktau .. km of the window)
          const uint32_t ktau = st.tau >> 16;
          double acc = 0.0;
          if (sm.wm[warp] > -INFINITY) {
            for (uint32_t key = km - static_cast<uint32_t>(lane); key >= ktau && key <= km; key -= 32u) {
              const uint32_t d = key - sm.wl[warp];
              if (d < static_cast<uint32_t>(kCrRing) && ring[d] != 0u)
                acc += static_cast<double>(ring[d]) * static_cast<double>(ex2((key16_value(key) - m) * c));
              if (key < 32u) break;
            }
          }
          acc = warp_sum(acc);
          if (lane == 0) sm.wk[warp] = acc;
          __syncthreads();
          if (threadIdx.x == 0) {
            // the warp whose range holds u * Z (else, by rounding, the last one with kept mass)
            double Z = 0.0;
            for (int w = 0; w < kCrWarps; ++w) Z += sm.wk[w];
            const double target = static_cast<double>(u) * Z;
            double C = 0.0, lastC = 0.0;
            int pick = -1, last = -1;
            for (int w = 0; w < kCrWarps; ++w) {
              if (sm.wk[w] > 0.0) {
                last = w;
                lastC = C;
                if (pick < 0 && C + sm.wk[w] > target) {
                  pick = w;
                  sm.dbase = C;
                }
              }
              C += sm.wk[w];
            }
            if (pick < 0) {
              pick = last;
              sm.dbase = lastC;
            }
            sm.dwarp = pick;
            sm.dtarget = target;
          }
          __syncthreads();
          const int pw = sm.dwarp;
          if (pw >= 0) {  // uniform
            const CrRange pr = cr_range(rp, V, pw);
            JobRows<T, false> J;
            J.init(rp, st, nullptr, st);
            y = block_draw_range(J, pr.lo, pr.hi, sm.dbase, sm.dtarget, u, sm.draw);
            if (y >= 0) q = kept_weight(st, load_elem(rp + y)) / st.s_kept;
          }
        }
        cut_row_finish<T>(A, Bt, a, va, rec, st, row, req, y, q, &sm.flag);
        __syncthreads();
        continue;
      }
      __syncthreads();  // the general select below reuses the shared memory
      if (bad) {
        cut_row_finish<T>(A, Bt, a, va, rec, st, row, req, -1, -1.0f, &smu.gen.flag);
        __syncthreads();
        continue;
      }
    }
    cut_row_general<T>(A, Bt, a, va, parts_a, parts_b, smu, rp, rec, st, in_b, row, req, Tv, tp, k, u);
  }
}

// Row statistics of the cut requests' rows alone (psispec_row_stats): one CTA per row at a
// time.
// (The argument structs are grid constants: the helpers take them by reference without a
// per-thread copy in local memory.)
template <typename T>
__global__ void __launch_bounds__(kCrThreads, kRowCtas<T>) cut_rows_kernel(const T* __restrict__ A,
                                                                const __grid_constant__ CutArgs a,
                                                                const __grid_constant__ VerifyArgs va,
                                                                const Partial* __restrict__ parts) {
  extern __shared__ __align__(16) unsigned char cut_smem_raw[];
  cut_rows_cta<T>(A, nullptr, a, va, parts, nullptr, blockIdx.x, gridDim.x, *reinterpret_cast<CutSmem<T>*>(cut_smem_raw));
}

// The row kernel of sample_draft. CTAs [0, warp_ctas) finish the rows without a cut, one
// warp per row; the remaining CTAs take the rows of requests with a cut (cut_rows_cta). One
// launch serves both kinds of rows.
template <typename T>
__global__ void __launch_bounds__(kTpThreads, kRowCtas<T>) sample_rows_kernel(const T* __restrict__ draft, int K, int V,
                                                                   int rows, const float* __restrict__ temperature,
                                                                   const float* __restrict__ top_p,
                                                                   const int32_t* __restrict__ top_k,
                                                                   const float* __restrict__ u,
                                                                   const Partial* __restrict__ parts,
                                                                   RowStat* __restrict__ stats,
                                                                   int32_t* __restrict__ out_tokens,
                                                                   float* __restrict__ out_q, int warp_ctas,
                                                                   const __grid_constant__ CutArgs a,
                                                                   const __grid_constant__ VerifyArgs va) {
  if (static_cast<int>(blockIdx.x) < warp_ctas) {
    const int row = blockIdx.x * kTpWarps + (threadIdx.x >> 5);
    if (row < rows && !request_cut(temperature, top_p, top_k, row / K, V))
      warp_sample_row(draft, row, K, V, temperature, u, parts, stats, out_tokens, out_q);
    return;
  }
  extern __shared__ __align__(16) unsigned char cut_smem_raw[];
  cut_rows_cta<T>(draft, nullptr, a, va, parts, nullptr, static_cast<int>(blockIdx.x) - warp_ctas,
                  static_cast<int>(gridDim.x) - warp_ctas, *reinterpret_cast<CutSmem<T>*>(cut_smem_raw));
}

// The row kernel of verify_linear. CTAs [0, warp_ctas) finish the rows of requests without a
// cut, one warp per row; the remaining CTAs take the rows of requests with a cut
// (cut_rows_cta). Every row then arrives on its request's counter, and whoever completes a
// request runs its accept tests and writes the draw job.
template <typename T>
__global__ void __launch_bounds__(kTpThreads, kRowCtas<T>) verify_rows_kernel(const T* __restrict__ tgt,
                                                                   const T* __restrict__ drf,
                                                                   const __grid_constant__ VerifyArgs va,
                                                                   const __grid_constant__ CutArgs a, int warp_ctas) {
  const int K = va.K, V = va.V;
  const int rows_t = va.B * (K + 1);
  const int rows = rows_t + (va.stream_draft ? va.B * K : 0);
  if (static_cast<int>(blockIdx.x) < warp_ctas) {
    const int g = blockIdx.x * kTpWarps + (threadIdx.x >> 5);
    if (g < rows && !request_cut(va.temperature, va.top_p, va.top_k, g < rows_t ? g / (K + 1) : (g - rows_t) / K, V))
      warp_verify_row(tgt, drf, g, va);
    return;
  }
  extern __shared__ __align__(16) unsigned char cut_smem_raw[];
  cut_rows_cta<T>(tgt, drf, a, va, va.parts_t, va.parts_d, static_cast<int>(blockIdx.x) - warp_ctas,
                  static_cast<int>(gridDim.x) - warp_ctas, *reinterpret_cast<CutSmem<T>*>(cut_smem_raw));
}

}  // namespace psi
