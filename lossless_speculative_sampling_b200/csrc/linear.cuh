// linear.cuh -- accept test, first-rejection scan and output assembly of the linear sampler.
//
// Review page of arXiv 2609.04010, section 3.3: draft token x_i is accepted with probability
// min(1, p(x_i)/q(x_i)), the longest prefix before the first rejection is kept, the rejected
// position is resampled from the normalised residual [p - q]_+, and a fully accepted block
// earns a bonus token from the last verifier row. Section 3.4: the linear sampler proposes
// one candidate per position.
//
// One warp per request: lane i tests position i (and i + 32), a ballot gives the first
// rejection j, and lane 0 writes the residual (or bonus) draw job. Greedy requests (T == 0)
// need no draw: the verifier argmax is written directly.
#pragma once

#include "common.cuh"

namespace psi {

// u * q(x) < p(x), evaluated as u < 2^(((lp - lq) + (mq - mp)) c) * sq / sp so that tiny
// probabilities do not underflow before the comparison.
__device__ __forceinline__ bool accept_test(float u, const RowStat& sp, float lp, const RowStat& sq, float lq, int x) {
  if (sp.c == 0.0f) return x == sp.amax;
  const bool p_pos = lp >= cut_value(sp.tau) && lp > -INFINITY;
  const bool q_pos = lq >= cut_value(sq.tau) && lq > -INFINITY;
  if (!p_pos) return false;
  if (!q_pos) return true;
  const float e = ((lp - lq) + (sq.m - sp.m)) * sp.c;
  const float ratio = ex2(e) * (sq.s_kept / sp.s_kept);
  return u < ratio;
}

// Called by one full warp for request b. ts: verifier rows [B*(K+1)], ds: draft rows [B*K].
template <typename T>
__device__ void warp_decide_request(int b, const T* __restrict__ tgt, const T* __restrict__ drf, int K, int V,
                                    const int32_t* __restrict__ tokens, const RowStat* ts, const RowStat* ds,
                                    const float* __restrict__ u_acc, const float* __restrict__ u_res,
                                    int32_t* __restrict__ out_tokens, int32_t* __restrict__ out_len,
                                    float* __restrict__ out_p, float* __restrict__ out_q, Job* __restrict__ jobs) {
  const int lane = threadIdx.x & 31;
  const size_t trow0 = static_cast<size_t>(b) * (K + 1), drow0 = static_cast<size_t>(b) * K;
  bool bad = false;
  uint32_t rej_lo = 0u, rej_hi = 0u;
  int x_mine[3] = {-1, -1, -1};
  float p_mine[2] = {-1.0f, -1.0f}, q_mine[2] = {-1.0f, -1.0f};
  RowStat sq_mine[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = lane + 32 * h;
    sq_mine[h] = RowStat{0.0f, 0.0f, 1.0f, 1.0f, 0u, -1, 1, 0};
    if (i >= K) continue;
    const int x = tokens[drow0 + i];
    const RowStat sp = load_stat_cg(ts + trow0 + i), sq = load_stat_cg(ds + drow0 + i);
    sq_mine[h] = sq;
    const bool rowbad = sp.status != 0 || sq.status != 0 || x < 0 || x >= V;
    bool acc = false;
    if (!rowbad) {
      const float lp = load_elem(tgt + (trow0 + i) * V + x);
      const float lq = load_elem(drf + (drow0 + i) * V + x);
      p_mine[h] = prob_of(sp, lp, x);
      q_mine[h] = prob_of(sq, lq, x);
      acc = accept_test(u_acc[drow0 + i], sp, lp, sq, lq, x);
    }
    x_mine[h] = x;
    bad |= rowbad;
    if (!acc) (h ? rej_hi : rej_lo) |= 1u << lane;
  }
  const RowStat bonus = load_stat_cg(ts + trow0 + K);
  bad = __any_sync(0xffffffffu, bad) || bonus.status != 0;
  rej_lo = __reduce_or_sync(0xffffffffu, rej_lo);
  rej_hi = __reduce_or_sync(0xffffffffu, rej_hi);
  const int j = rej_lo ? __ffs(rej_lo) - 1 : (rej_hi ? 32 + __ffs(rej_hi) - 1 : K);
  const RowStat sj = load_stat_cg(ts + trow0 + j);  // verifier row of the draw (row K for the bonus)
  // draft row of a residual draw (held by lane j % 32 of half j / 32)
  const RowStat sqj = shfl_stat(j >= 32 ? sq_mine[1] : sq_mine[0], j & 31);

#pragma unroll
  for (int h = 0; h < 3; ++h) {  // K + 1 <= 65 token slots
    const int i = lane + 32 * h;
    if (i < K && h < 2) {
      if (out_p) out_p[drow0 + i] = bad ? -1.0f : p_mine[h];
      if (out_q) out_q[drow0 + i] = bad ? -1.0f : q_mine[h];
    }
    if (i <= K) {
      int t = -1;
      if (!bad) {
        if (i < j) t = x_mine[h];
        else if (i == j && sj.c == 0.0f) t = sj.amax;  // greedy: the verifier argmax
      }
      out_tokens[trow0 + i] = t;
    }
  }
  if (lane == 0) {
    out_len[b] = bad ? -1 : j;
    Job jb;
    jb.mode = (!bad && sj.c != 0.0f) ? (j < K ? kResidual : kSample) : kNone;
    jb.row_a = static_cast<int32_t>(trow0 + j);
    jb.row_b = static_cast<int32_t>(drow0 + j);
    jb.out_index = static_cast<int32_t>(trow0 + j);
    jb.u = u_res[trow0 + j];
    jb.pad[0] = jb.pad[1] = jb.pad[2] = 0;
    jb.sa = sj;
    jb.sb = sqj;
    jobs[b] = jb;
  }
}

}  // namespace psi
