// tree.cuh -- tree verification: recursive rejection without replacement over the children
// of each node (the tree sampler of the review page of arXiv 2609.04010, section 3.4, names
// the method but prints no acceptance rule; this is the plainest lossless reading).
//
// At the current node, r starts as the verifier distribution p and q~ as the draft
// distribution q. Child k with token t_k is accepted iff u * q~_k(t_k) < r_{k-1}(t_k). On a
// rejection r_k = max(0, r_{k-1} - q~_k) / Z_k (unchanged when Z_k = 0) and t_k leaves the
// draft: q~_{k+1}(v) = q(v) / Q_{k+1} for the tokens not yet removed, Q_{k+1} = Q_k - q(t_k).
// Every r_k(v) is therefore a short chain of max/scale steps applied to p(v) and q(v), so the
// kernel stores only the scalars (t_i, Q_i, Z_i) and re-evaluates the chain per element in
// each pass over the vocabulary: one pass per rejected child (for Z_k) and one final
// prefix-scan draw at the node where the walk stops.
//
// One CTA of kTreeThreads per request. Row statistics come from the stats kernels.
#pragma once

#include "common.cuh"

namespace psi {

constexpr int kTreeThreads = 512;
constexpr int kMaxNodes = 1024;    // nodes per request
constexpr int kMaxChildren = 64;   // children of one node

struct ChainStep {
  int t;       // token removed at this step
  float Q;     // draft mass divisor at this step
  float invZ;  // 1 / Z (residual normaliser), 0 when the step left r unchanged
};

struct ChainCtx {
  RowStat p, q;
  float ip, iq;
  int nsteps;
};

// r_k(v) for the first ctx.nsteps steps
__device__ __forceinline__ float chain_eval(const ChainCtx& c, const ChainStep* steps, float lp, float lq, int v) {
  float r = kept_weight(c.p, lp) * c.ip;
  if (c.nsteps == 0) return r;
  const float qv = kept_weight(c.q, lq) * c.iq;
  for (int i = 0; i < c.nsteps; ++i) {
    bool removed = false;
    for (int k = 0; k < i; ++k) removed |= steps[k].t == v;
    if (steps[i].invZ > 0.0f) r = fmaxf(r - (removed ? 0.0f : qv / steps[i].Q), 0.0f) * steps[i].invZ;
  }
  return r;
}

template <typename T>
__global__ void __launch_bounds__(kTreeThreads) tree_walk_kernel(
    const T* __restrict__ tgt, const T* __restrict__ drf, int V, const int32_t* __restrict__ offs,
    const int32_t* __restrict__ parent, const int32_t* __restrict__ tokens, const RowStat* __restrict__ ts,
    const RowStat* __restrict__ ds, const float* __restrict__ u_acc, const float* __restrict__ u_res, int max_depth,
    int32_t* __restrict__ out_path, int32_t* __restrict__ out_tokens, int32_t* __restrict__ out_len) {
  __shared__ int depth[kMaxNodes];
  __shared__ int ch[kMaxChildren];
  __shared__ ChainStep steps[kMaxChildren];
  __shared__ double red[33];
  __shared__ int sh_bad, sh_nch, sh_next, sh_y;
  __shared__ float sh_Q;
  __shared__ ChainCtx ctx;
  const int b = blockIdx.x;
  const int n0 = offs[b], n = offs[b + 1] - n0;
  int32_t* path = out_path + static_cast<size_t>(b) * max_depth;
  int32_t* toks = out_tokens + static_cast<size_t>(b) * (max_depth + 1);

  if (threadIdx.x == 0) {
    int bad = (n <= 0 || n > kMaxNodes) ? 1 : (parent[n0] != -1);
    if (!bad) depth[0] = 0;
    for (int c = 1; c < n && !bad; ++c) {
      const int pa = parent[n0 + c], t = tokens[n0 + c];
      if (pa < 0 || pa >= c || t < 0 || t >= V) { bad = 1; break; }
      depth[c] = depth[pa] + 1;
      if (depth[c] > max_depth) bad = 1;
    }
    sh_bad = bad;
  }
  __syncthreads();

  int cur = 0, len = 0;
  while (!sh_bad) {
    const RowStat sp = ts[n0 + cur];
    if (threadIdx.x == 0) {
      int nch = 0;
      for (int c = cur + 1; c < n; ++c)
        if (parent[n0 + c] == cur) {
          if (nch == kMaxChildren) { sh_bad = 1; break; }
          ch[nch++] = c;
        }
      sh_nch = nch;
      sh_next = -1;
      if (sp.status != 0) sh_bad = 1;
    }
    __syncthreads();
    if (sh_bad) break;
    const int nch = sh_nch;
    if (sp.c == 0.0f) {  // greedy: follow the child carrying the verifier argmax
      if (threadIdx.x == 0) {
        for (int k = 0; k < nch; ++k)
          if (tokens[n0 + ch[k]] == sp.amax) { sh_next = ch[k]; break; }
        sh_y = sp.amax;
      }
      __syncthreads();
      if (sh_next >= 0) {
        if (threadIdx.x == 0) { path[len] = sh_next; toks[len] = tokens[n0 + sh_next]; }
        cur = sh_next;
        ++len;
        __syncthreads();
        continue;
      }
      break;  // final token sh_y
    }

    const T* rp = tgt + static_cast<size_t>(n0 + cur) * V;
    const T* rq = drf + static_cast<size_t>(n0 + cur) * V;
    if (threadIdx.x == 0) {
      ctx.p = sp;
      ctx.ip = 1.0f / sp.s_kept;
      ctx.nsteps = 0;
      sh_Q = 1.0f;
      if (nch > 0) {
        ctx.q = ds[n0 + cur];
        ctx.iq = 1.0f / ctx.q.s_kept;
        if (ctx.q.status != 0) sh_bad = 1;
      } else {
        ctx.q = sp;
        ctx.iq = 0.0f;
      }
    }
    __syncthreads();
    if (sh_bad) break;

    for (int k = 0; k < nch; ++k) {
      // accept test for child k (one thread), then a residual pass when it is rejected
      if (threadIdx.x == 0) {
        const int c = ch[k], t = tokens[n0 + c];
        const float Q = sh_Q;
        if (!(Q > 0.0f)) {
          sh_nch = -1;  // draft mass exhausted: the remaining children are skipped
        } else {
          const float lp = load_elem(rp + t), lq = load_elem(rq + t);
          const float rt = chain_eval(ctx, steps, lp, lq, t);
          bool removed = false;
          for (int i = 0; i < ctx.nsteps; ++i) removed |= steps[i].t == t;
          const float qt = removed ? 0.0f : kept_weight(ctx.q, lq) * ctx.iq / Q;
          if (u_acc[n0 + c] * qt < rt) sh_next = c;
        }
      }
      __syncthreads();
      if (sh_next >= 0 || sh_nch < 0) break;
      // Z_k = sum_v max(0, r_{k-1}(v) - q~_k(v)), and the draft mass left once t_k is removed
      const int t = tokens[n0 + ch[k]];
      const float Q = sh_Q;
      double z = 0.0, qrem = 0.0;
      for (int v = threadIdx.x; v < V; v += blockDim.x) {
        const float lp = load_elem(rp + v), lq = load_elem(rq + v);
        const float r = chain_eval(ctx, steps, lp, lq, v);
        bool removed = false;
        for (int i = 0; i < ctx.nsteps; ++i) removed |= steps[i].t == v;
        const float qraw = removed ? 0.0f : kept_weight(ctx.q, lq) * ctx.iq;
        z += static_cast<double>(fmaxf(r - qraw / Q, 0.0f));
        if (v != t) qrem += static_cast<double>(qraw);
      }
      z = block_sum(z, red);
      qrem = block_sum(qrem, red);
      if (threadIdx.x == 0) {
        steps[ctx.nsteps] = ChainStep{t, Q, z > 0.0 ? static_cast<float>(1.0 / z) : 0.0f};
        ctx.nsteps += 1;
        sh_Q = static_cast<float>(qrem);  // 0 exactly when no draft mass is left
      }
      __syncthreads();
    }
    if (sh_next >= 0) {
      if (threadIdx.x == 0) { path[len] = sh_next; toks[len] = tokens[n0 + sh_next]; }
      cur = sh_next;
      ++len;
      __syncthreads();
      continue;
    }

    // final draw from r at this node: contiguous runs, scanned in thread order
    const int run = (V + blockDim.x - 1) / blockDim.x;
    const int r0 = min(V, static_cast<int>(threadIdx.x) * run), r1 = min(V, r0 + run);
    double mine = 0.0;
    int last = -1;
    for (int v = r0; v < r1; ++v) {
      const float w = chain_eval(ctx, steps, load_elem(rp + v), load_elem(rq + v), v);
      mine += static_cast<double>(w);
      if (w > 0.0f) last = v;
    }
    if (threadIdx.x == 0) sh_y = 0x7fffffff;
    double total;
    const double C0 = block_exclusive_scan(mine, red, &total);
    const double target = static_cast<double>(u_res[n0 + cur]) * total;
    int* lastp = &sh_nch;  // reuse: last index with positive weight
    if (threadIdx.x == 0) *lastp = -1;
    __syncthreads();
    if (last >= 0) atomicMax(lastp, last);
    if (C0 <= target && target < C0 + mine) {
      double C = C0;
      for (int v = r0; v < r1; ++v) {
        C += static_cast<double>(chain_eval(ctx, steps, load_elem(rp + v), load_elem(rq + v), v));
        if (C > target) { atomicMin(&sh_y, v); break; }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && sh_y == 0x7fffffff) sh_y = *lastp;
    __syncthreads();
    break;
  }

  if (threadIdx.x == 0) {
    if (sh_bad) {
      for (int i = 0; i < max_depth; ++i) path[i] = -1;
      for (int i = 0; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = -1;
    } else {
      for (int i = len; i < max_depth; ++i) path[i] = -1;
      toks[len] = sh_y;
      for (int i = len + 1; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = len;
    }
  }
}

}  // namespace psi
