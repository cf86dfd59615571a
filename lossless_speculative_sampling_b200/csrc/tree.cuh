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

#include <cooperative_groups.h>

#include "common.cuh"
#include "sample.cuh"

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

// ---------------------------------------------------------------------------------------
// Cluster walk. A cluster of CL CTAs (16 where the device can schedule it, else 8) verifies
// one trie; CTA `rank` owns the
// vocabulary slice [rank * slice, (rank + 1) * slice). At every visited node the slices of
// r (unnormalised, r = r' / S) and q (normalised) are staged in shared memory as fp32, so the
// passes a rejection needs run on chip:
//   accept child k with token t  iff  u * q(t) * S < r'(t) * Q   (q~ = q / Q, r = r' / S);
//   on rejection                      r' <- max(r' - (S / Q) q, 0),  S <- sum r',
//                                     q(t) <- 0,  Q <- sum q       (r' unchanged when S = 0).
// Sums are fp64: per CTA by a block reduction, across the cluster in rank order through
// distributed shared memory, so every CTA computes the same value and takes the same branch
// (the cluster barriers below are therefore reached in the same order by every CTA).
namespace cg = cooperative_groups;

constexpr int kTreeWalkThreads = 256;
constexpr int kTreeMaxSlice = 26624;  // elements per CTA: r and q slices as fp32 fit in 208 KB

__host__ __device__ inline int tree_slice(int V, int cl) {
  return (((V + cl - 1) / cl) + 7) & ~7;  // a multiple of 8 elements
}

struct TreeWalkShared {
  int depth[kMaxNodes];
  int ch[kMaxChildren];
  double red[33];
  double slot[4];  // this CTA's contribution to a cluster reduction
  int islot[2];
  int bad, nch, next, y, acc;
};

// Sums of a and b over the cluster, in rank order (the same doubles in every CTA).
template <int CL>
__device__ __forceinline__ double2 cluster_sum2(cg::cluster_group& cl, double a, double b, TreeWalkShared& sh) {
  if (threadIdx.x == 0) {
    sh.slot[0] = a;
    sh.slot[1] = b;
  }
  cl.sync();
  double sa = 0.0, sb = 0.0;
  for (int r = 0; r < CL; ++r) {
    const double* rs = cl.map_shared_rank(sh.slot, r);
    sa += rs[0];
    sb += rs[1];
  }
  cl.sync();
  return make_double2(sa, sb);
}

template <typename T, int CL>
__global__ void __launch_bounds__(kTreeWalkThreads, 1) tree_walk_cluster_kernel(
    const T* __restrict__ tgt, const T* __restrict__ drf, int V, const int32_t* __restrict__ offs,
    const int32_t* __restrict__ parent, const int32_t* __restrict__ tokens, const RowStat* __restrict__ ts,
    const RowStat* __restrict__ ds, const float* __restrict__ u_acc, const float* __restrict__ u_res, int max_depth,
    int32_t* __restrict__ out_path, int32_t* __restrict__ out_tokens, int32_t* __restrict__ out_len) {
  cg::cluster_group cl = cg::this_cluster();
  __shared__ TreeWalkShared sh;
  extern __shared__ __align__(16) float tw_smem[];
  const int rank = static_cast<int>(cl.block_rank());
  const int slice = tree_slice(V, CL);
  float* rs = tw_smem;          // r' of this CTA's slice
  float* qs = tw_smem + slice;  // q of this CTA's slice
  const int v0 = min(V, rank * slice), v1 = min(V, v0 + slice), ns = v1 - v0;
  const int b = blockIdx.x / CL;
  const int n0 = offs[b], n = offs[b + 1] - n0;
  int32_t* path = out_path + static_cast<size_t>(b) * max_depth;
  int32_t* toks = out_tokens + static_cast<size_t>(b) * (max_depth + 1);
  const bool writer = rank == 0 && threadIdx.x == 0;

  if (threadIdx.x == 0) {  // structure checks (every CTA, same data, same answer)
    int bad = (n <= 0 || n > kMaxNodes) ? 1 : (parent[n0] != -1);
    if (!bad) sh.depth[0] = 0;
    for (int c = 1; c < n && !bad; ++c) {
      const int pa = parent[n0 + c], t = tokens[n0 + c];
      if (pa < 0 || pa >= c || t < 0 || t >= V) {
        bad = 1;
        break;
      }
      sh.depth[c] = sh.depth[pa] + 1;
      if (sh.depth[c] > max_depth) bad = 1;
    }
    sh.bad = bad;
    sh.y = -1;
  }
  __syncthreads();

  int cur = 0, len = 0;
  while (!sh.bad) {
    const RowStat sp = ts[n0 + cur];
    if (threadIdx.x == 0) {
      int nch = 0;
      for (int c = cur + 1; c < n; ++c)
        if (parent[n0 + c] == cur) {
          if (nch == kMaxChildren) {
            sh.bad = 1;
            break;
          }
          sh.ch[nch++] = c;
        }
      sh.nch = nch;
      sh.next = -1;
      if (sp.status != 0) sh.bad = 1;
    }
    __syncthreads();
    if (sh.bad) break;
    const int nch = sh.nch;
    if (sp.c == 0.0f) {  // greedy: follow the child carrying the verifier argmax
      if (threadIdx.x == 0) {
        for (int k = 0; k < nch; ++k)
          if (tokens[n0 + sh.ch[k]] == sp.amax) {
            sh.next = sh.ch[k];
            break;
          }
        sh.y = sp.amax;
      }
      __syncthreads();
      const int next = sh.next;
      if (next >= 0) {
        if (writer) {
          path[len] = next;
          toks[len] = tokens[n0 + next];
        }
        cur = next;
        ++len;
        __syncthreads();
        continue;
      }
      break;  // final token sh.y
    }
    RowStat sq = sp;
    if (nch > 0) {
      sq = ds[n0 + cur];
      if (sq.status != 0) {
        if (threadIdx.x == 0) sh.bad = 1;
        __syncthreads();
        break;
      }
    }
    // stage the node's slices: r' = kept weight of p (relative to its maximum), q normalised
    {
      const T* rp = tgt + static_cast<size_t>(n0 + cur) * V;
      const T* rq = drf + static_cast<size_t>(n0 + cur) * V;
      JobRows<T, true> J;
      J.init(rp, sp, rq, sq);
      const float iq = nch > 0 ? 1.0f / sq.s_kept : 0.0f;
      double sr = 0.0, sqm = 0.0;
      constexpr int kStageBatch = 4;  // 8-element groups of both rows in flight per thread
      constexpr int kStep = kTreeWalkThreads * 8;
      for (int e0 = v0 + threadIdx.x * 8; e0 < v1; e0 += kStageBatch * kStep) {
        Raw8<T, true> x[kStageBatch];
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j)
          if (e0 + j * kStep < v1) J.load(e0 + j * kStep, v1, x[j]);
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
          const int e = e0 + j * kStep;
          if (e >= v1) continue;
          float lp[8], lq[8];
          x[j].a.unpack(lp);
          x[j].b[0].unpack(lq);
          float gr = 0.0f, gq = 0.0f;  // 8-term fp32 sums, then fp64
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (e + k < v1) {
              const float r = kept_weight(sp, lp[k]);
              const float q = nch > 0 ? kept_weight(sq, lq[k]) * iq : 0.0f;
              rs[e + k - v0] = r;
              qs[e + k - v0] = q;
              gr += r;
              gq += q;
            }
          }
          sr += static_cast<double>(gr);
          sqm += static_cast<double>(gq);
        }
      }
      // the walk continues at one of the children: bring their slices towards L2 meanwhile
      for (int k = 0; k < nch; ++k) {
        const size_t row = static_cast<size_t>(n0 + sh.ch[k]) * V;
        for (int e = v0 + threadIdx.x * 64; e < v1; e += kTreeWalkThreads * 64) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(tgt + row + e));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(drf + row + e));
        }
      }
      sr = block_sum(sr, sh.red);
      sqm = block_sum(sqm, sh.red);
      __syncthreads();
      const double2 t = cluster_sum2<CL>(cl, sr, sqm, sh);  // also publishes the staged slices
      double S = t.x, Q = t.y;
      for (int k = 0; k < nch; ++k) {
        if (!(Q > 0.0)) break;  // draft mass exhausted: the remaining children are skipped
        const int c = sh.ch[k], tok = tokens[n0 + c];
        const int owner = tok / slice, off = tok - owner * slice;
        if (threadIdx.x == 0) {
          const float rt = cl.map_shared_rank(rs, owner)[off];
          const float qt = cl.map_shared_rank(qs, owner)[off];
          sh.acc = static_cast<double>(u_acc[n0 + c]) * static_cast<double>(qt) * S <
                   static_cast<double>(rt) * Q;
        }
        cl.sync();  // every CTA has read r'(t) and q(t) before any slice changes
        if (sh.acc) {
          if (threadIdx.x == 0) sh.next = c;
          __syncthreads();
          break;
        }
        // rejected: totals of the residual and of the draft mass without t (4-term fp32 sums,
        // then fp64), over float4 vectors of the slices
        const float scale = static_cast<float>(S / Q);
        const int tl = tok - v0;  // t's offset in this slice (outside [0, ns) elsewhere)
        const int n4 = ns >> 2;
        float4* r4 = reinterpret_cast<float4*>(rs);
        const float4* q4 = reinterpret_cast<const float4*>(qs);
        double zr = 0.0, zq = 0.0;
        for (int i = threadIdx.x; i < n4; i += kTreeWalkThreads) {
          const float4 r = r4[i], q = q4[i];
          zr += static_cast<double>((fmaxf(r.x - scale * q.x, 0.0f) + fmaxf(r.y - scale * q.y, 0.0f)) +
                                    (fmaxf(r.z - scale * q.z, 0.0f) + fmaxf(r.w - scale * q.w, 0.0f)));
          const int j = tl - 4 * i;  // the removed token's lane within this vector, if any
          zq += static_cast<double>(((j == 0 ? 0.0f : q.x) + (j == 1 ? 0.0f : q.y)) +
                                    ((j == 2 ? 0.0f : q.z) + (j == 3 ? 0.0f : q.w)));
        }
        for (int i = 4 * n4 + threadIdx.x; i < ns; i += kTreeWalkThreads) {
          zr += static_cast<double>(fmaxf(rs[i] - scale * qs[i], 0.0f));
          if (i != tl) zq += static_cast<double>(qs[i]);
        }
        zr = block_sum(zr, sh.red);
        zq = block_sum(zq, sh.red);
        __syncthreads();
        const double2 z = cluster_sum2<CL>(cl, zr, zq, sh);
        if (z.x > 0.0) {
          for (int i = threadIdx.x; i < n4; i += kTreeWalkThreads) {
            float4 r = r4[i];
            const float4 q = q4[i];
            r.x = fmaxf(r.x - scale * q.x, 0.0f);
            r.y = fmaxf(r.y - scale * q.y, 0.0f);
            r.z = fmaxf(r.z - scale * q.z, 0.0f);
            r.w = fmaxf(r.w - scale * q.w, 0.0f);
            r4[i] = r;
          }
          for (int i = 4 * n4 + threadIdx.x; i < ns; i += kTreeWalkThreads) rs[i] = fmaxf(rs[i] - scale * qs[i], 0.0f);
          S = z.x;
        }
        if (rank == owner && threadIdx.x == 0) qs[off] = 0.0f;
        Q = z.y;
        __syncthreads();
        cl.sync();  // the updated slices are visible before the next child's test
      }
    }
    const int next = sh.next;
    if (next >= 0) {
      if (writer) {
        path[len] = next;
        toks[len] = tokens[n0 + next];
      }
      cur = next;
      ++len;
      __syncthreads();
      continue;
    }
    // final draw from r at this node: contiguous runs per thread, scanned in thread order
    // inside each slice, slices in rank order
    const int run = (ns + kTreeWalkThreads - 1) / kTreeWalkThreads;
    const int r0 = min(ns, static_cast<int>(threadIdx.x) * run), r1 = min(ns, r0 + run);
    double mine = 0.0;
    int last = -1;
    for (int i = r0; i < r1; ++i) {
      const float w = rs[i];
      mine += static_cast<double>(w);
      if (w > 0.0f) last = v0 + i;
    }
    double total;
    const double C0 = block_exclusive_scan(mine, sh.red, &total);
    if (threadIdx.x == 0) {
      sh.slot[0] = total;
      sh.islot[0] = 0x7fffffff;  // drawn index, if it falls in this slice
      sh.islot[1] = -1;          // last index with positive weight in this slice
    }
    cl.sync();
    double base = 0.0, grand = 0.0;
    for (int r = 0; r < CL; ++r) {
      const double tr = cl.map_shared_rank(sh.slot, r)[0];
      if (r < rank) base += tr;
      grand += tr;
    }
    const double target = static_cast<double>(u_res[n0 + cur]) * grand;
    if (last >= 0) atomicMax(&sh.islot[1], last);
    if (base + C0 <= target && target < base + C0 + mine) {
      double C = base + C0;
      for (int i = r0; i < r1; ++i) {
        C += static_cast<double>(rs[i]);
        if (C > target && rs[i] > 0.0f) {
          atomicMin(&sh.islot[0], v0 + i);
          break;
        }
      }
    }
    __syncthreads();
    cl.sync();
    if (writer) {
      int y = 0x7fffffff, lastpos = -1;
      for (int r = 0; r < CL; ++r) {
        const int* is = cl.map_shared_rank(sh.islot, r);
        y = min(y, is[0]);
        lastpos = max(lastpos, is[1]);
      }
      sh.y = y != 0x7fffffff ? y : lastpos;  // rounding past every slice: the last positive index
    }
    break;
  }
  cl.sync();  // no CTA leaves while another may still read its shared memory
  if (writer) {
    if (sh.bad) {
      for (int i = 0; i < max_depth; ++i) path[i] = -1;
      for (int i = 0; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = -1;
    } else {
      for (int i = len; i < max_depth; ++i) path[i] = -1;
      toks[len] = sh.y;
      for (int i = len + 1; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = len;
    }
  }
}

}  // namespace psi
