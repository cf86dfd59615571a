// tree.cuh -- tree verification: recursive rejection without replacement over the children
// of each node (the tree sampler of the review page of arXiv 2609.04010, section 3.4, names
// the method but prints no acceptance rule; this is the plainest lossless reading).
//
// At the current node, r starts as the verifier distribution p and q~ as the draft
// distribution q. Child k with token t_k is accepted iff u * q~_k(t_k) < r_{k-1}(t_k). On a
// rejection r_k = max(0, r_{k-1} - q~_k) / Z_k (unchanged when Z_k = 0) and t_k leaves the
// draft: q~_{k+1}(v) = q(v) / Q_{k+1} for the tokens not yet removed, Q_{k+1} = Q_k - q(t_k).
//
// Two kernels implement it. The cluster walk (tree_walk_cluster_kernel, below) spreads each
// trie over a cluster of CTAs that stage the node's rows in shared memory. The fallback
// (tree_walk_kernel, one CTA of kTreeThreads per trie, for devices that cannot schedule such
// clusters) uses that every r_k(v) is a short chain of max/scale steps applied to p(v) and
// q(v): it stores only the scalars (t_i, Q_i, Z_i) and re-evaluates the chain per element in
// each pass over the vocabulary, one pass per rejected child (for Z_k) and one final
// prefix-scan draw at the node where the walk stops. Its row statistics come from the stats
// kernels.
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
// one trie; CTA `rank` owns the vocabulary slice [rank * slice, (rank + 1) * slice). At every
// visited node the slices of r' and q' (kept weights, so r = r' / S and q~ = q' / Q) are
// staged in shared memory as fp32 and the passes a rejection needs run on chip:
//   accept child k with token t  iff  u * q'(t) * S < r'(t) * Q;
//   on rejection                      r' <- max(r' - (S / Q) q', 0),  S <- sum r',
//                                     q'(t) <- 0,  Q <- sum q'      (r' unchanged when S = 0).
// Row statistics come from ts / ds, except for requests with T > 0 and no top-p cut when
// `lazy` is set (the statistics pass skipped those rows): their weights are staged relative
// to each slice's own maxima, and every CTA scales its slice to the rows' maxima on the fly
// (factors fr, fq) once the maxima are exchanged, until the first residual update rewrites it.
// Values cross the cluster by exchanges through distributed shared memory; their sums are
// formed in the same order in every CTA, so all CTAs take the same branches and reach the
// cluster barriers in the same order.
namespace cg = cooperative_groups;

constexpr int kTreeWalkThreads = 512;
constexpr int kMaxCluster = 16;
constexpr int kXVals = 6;  // values a CTA posts in one cluster exchange

__host__ __device__ inline int tree_slice(int V, int cl) {
  return (((V + cl - 1) / cl) + 7) & ~7;  // a multiple of 8 elements
}

struct TreeWalkShared {
  int depth[kMaxNodes];
  int par[kMaxNodes];  // the trie's parent indices and tokens, read once
  int tok[kMaxNodes];
  int ch[kMaxChildren];
  float cu[kMaxChildren];  // u_accept of the current node's children
  double red[33];
  double red2[2][32];
  double x[2][kMaxCluster][kXVals];  // exchange slots: x[parity][rank] holds what rank posted
  double xt[kMaxCluster];            // final draw: the slices' totals
  int xi[kMaxCluster][2];            // final draw: each slice's pick (read by rank 0)
  int islot[2];
  int bad, nch, next, y;
};

// Block sums of two doubles (the same values in every thread; the order is fixed).
__device__ __forceinline__ void block_sum2(double& a, double& b, double (&s)[2][32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  a = warp_sum(a);
  b = warp_sum(b);
  __syncthreads();  // earlier readers of s are done
  if (lane == 0) {
    s[0][warp] = a;
    s[1][warp] = b;
  }
  __syncthreads();
  a = warp_sum(lane < kTreeWalkThreads / 32 ? s[0][lane] : 0.0);
  b = warp_sum(lane < kTreeWalkThreads / 32 ? s[1][lane] : 0.0);
}

// NaN-propagating block maxima of two floats.
__device__ __forceinline__ void block_max2(float& a, float& b, double (&s)[2][32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  a = warp_max(a);
  b = warp_max(b);
  __syncthreads();
  if (lane == 0) {
    s[0][warp] = a;
    s[1][warp] = b;
  }
  __syncthreads();
  a = warp_max(lane < kTreeWalkThreads / 32 ? static_cast<float>(s[0][lane]) : -INFINITY);
  b = warp_max(lane < kTreeWalkThreads / 32 ? static_cast<float>(s[1][lane]) : -INFINITY);
}

// One cluster exchange: thread r of every CTA writes the CTA's kXVals values into rank r's
// slot array, then one cluster barrier makes them visible; afterwards every CTA reads all
// ranks' values from its own shared memory. Consecutive exchanges use alternate parities: a
// slot is written again only after the next barrier, which every CTA reaches after its reads
// of this exchange.
template <int CL>
__device__ __forceinline__ void cluster_post(cg::cluster_group& cl, TreeWalkShared& sh, int ph, int rank,
                                             const double (&v)[kXVals]) {
  if (threadIdx.x < CL) {
    double* dst = cl.map_shared_rank(&sh.x[ph][rank][0], static_cast<int>(threadIdx.x));
#pragma unroll
    for (int i = 0; i < kXVals; ++i) dst[i] = v[i];
  }
  cl.sync();
}

// Sum over the ranks of value i of an exchange, each scaled by the lane's weight w, in the
// same lane order in every warp of every CTA (so every thread obtains the same double).
template <int CL>
__device__ __forceinline__ double xsum(const TreeWalkShared& sh, int ph, int i, float w = 1.0f) {
  const int lane = threadIdx.x & 31;
  return warp_sum(lane < CL ? sh.x[ph][lane][i] * static_cast<double>(w) : 0.0);
}

// Scale taking weights relative to a slice's own maximum m to weights relative to the row's
// maximum M: 2^((m - M) c), and 0 for a slice without a finite logit.
__device__ __forceinline__ float frame_factor(float m, float M, float c) { return m > -INFINITY ? ex2((m - M) * c) : 0.0f; }

// 8 consecutive floats to shared memory at a 32-byte aligned address (n < 8: the first n).
__device__ __forceinline__ void store8(float* dst, const float (&v)[8], int n) {
  if (n >= 8) {
    reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < n) dst[k] = v[k];
  }
}
__device__ __forceinline__ void load8(const float* src, float (&v)[8], int n) {
  if (n >= 8) {
    const float4 a = reinterpret_cast<const float4*>(src)[0], c = reinterpret_cast<const float4*>(src)[1];
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = c.x, v[5] = c.y, v[6] = c.z, v[7] = c.w;
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = k < n ? src[k] : -INFINITY;
  }
}

// The rejection update of one residual weight in the rows' frame: max(fr r - s fq q, 0).
__device__ __forceinline__ float resid_update(float rg, float s, float qg) { return fmaxf(__fmaf_rn(-s, qg, rg), 0.0f); }

// Kept weights of 8 logits (values past the row's end are -inf: weight 0).
__device__ __forceinline__ void kept8(const float (&l)[8], const RowStat& st, float cut, float (&w)[8]) {
  exp8(l, st.m, st.c, w);
#pragma unroll
  for (int k = 0; k < 8; ++k) w[k] = l[k] >= cut ? w[k] : 0.0f;
}

template <typename T, int CL>
__global__ void __launch_bounds__(kTreeWalkThreads, 1) tree_walk_cluster_kernel(
    const T* __restrict__ tgt, const T* __restrict__ drf, int V, const int32_t* __restrict__ offs,
    const int32_t* __restrict__ parent, const int32_t* __restrict__ tokens, const RowStat* __restrict__ ts,
    const RowStat* __restrict__ ds, const float* __restrict__ u_acc, const float* __restrict__ u_res,
    const float* __restrict__ temperature, const float* __restrict__ top_p, int lazy, int dbuf, int max_depth,
    int32_t* __restrict__ out_path, int32_t* __restrict__ out_tokens, int32_t* __restrict__ out_len) {
  static_assert(CL <= kMaxCluster, "exchange slots per rank");
  constexpr int kStageBatch = sizeof(T) == 2 ? 3 : 2;  // 8-element groups of both rows in flight
  constexpr int kStep = kTreeWalkThreads * 8;
  cg::cluster_group cl = cg::this_cluster();
  __shared__ TreeWalkShared sh;
  extern __shared__ __align__(16) float tw_smem[];
  const int rank = static_cast<int>(cl.block_rank());
  const int lane = threadIdx.x & 31;
  const int slice = tree_slice(V, CL);
  // r' of this CTA's slice (with dbuf, two buffers: a rejection pass writes the updated r'
  // into the other one), and q'
  auto rbuf = [&](int i) { return i ? tw_smem + 2 * slice : tw_smem; };
  float* qs = tw_smem + slice;
  const int v0 = min(V, rank * slice), v1 = min(V, v0 + slice), ns = v1 - v0;
  const int b = blockIdx.x / CL;
  const int n0 = offs[b], n = offs[b + 1] - n0;
  int32_t* path = out_path + static_cast<size_t>(b) * max_depth;
  int32_t* toks = out_tokens + static_cast<size_t>(b) * (max_depth + 1);
  const bool writer = rank == 0 && threadIdx.x == 0;
  const bool uncut = lazy && uncut_request(temperature, top_p, b);  // statistics found here
  const bool regs = uncut && ns <= kStageBatch * kStep;             // whole slice in registers
  RowStat own;  // row statistics of an uncut request's visited rows (maxima set per slice)
  own.m = 0.0f;
  own.c = temp_scale(temperature[b]);
  own.s = own.s_kept = 1.0f;
  own.tau = 0u;
  own.amax = -1;
  own.status = 0;
  own.pad = 0;
  int ph = 0;  // exchange parity

  if (n > 0 && n <= kMaxNodes)
    for (int i = threadIdx.x; i < n; i += kTreeWalkThreads) {
      sh.par[i] = parent[n0 + i];
      sh.tok[i] = tokens[n0 + i];
    }
  __syncthreads();
  if (threadIdx.x == 0) {  // structure checks (every CTA, same data, same answer)
    int bad = (n <= 0 || n > kMaxNodes) ? 1 : (sh.par[0] != -1);
    if (!bad) sh.depth[0] = 0;
    for (int c = 1; c < n && !bad; ++c) {
      const int pa = sh.par[c], t = sh.tok[c];
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

  auto owner_of = [&](int t) { return t < 0 ? -1 : t / slice; };

  int cur = 0, len = 0;
  bool drew = false;  // the walk ended with the cluster's residual draw
  while (!sh.bad) {
    const T* rp = tgt + static_cast<size_t>(n0 + cur) * V;
    const T* rq = drf + static_cast<size_t>(n0 + cur) * V;
    const bool al_p = (reinterpret_cast<uintptr_t>(rp) & 15u) == 0;
    const bool al_q = (reinterpret_cast<uintptr_t>(rq) & 15u) == 0;
    Raw8x<T> xp[kStageBatch], xq[kStageBatch];
    auto load_batch = [&](int e0) {
#pragma unroll
      for (int j = 0; j < kStageBatch; ++j) {
        const int e = e0 + j * kStep;
        if (e < v1) {
          xp[j].load(rp, e, v1, al_p);
          xq[j].load(rq, e, v1, al_q);
        }
      }
    };
    if (regs) load_batch(v0 + threadIdx.x * 8);  // in flight while the children are listed
    RowStat sp = uncut ? own : ts[n0 + cur];
    if (threadIdx.x < 32) {  // children of cur in index order (warp ballots)
      int nch = 0;
      for (int c0 = cur + 1; c0 < n; c0 += 32) {
        const int c = c0 + lane;
        const bool is = c < n && sh.par[c] == cur;
        const unsigned m = __ballot_sync(0xffffffffu, is);
        const int pos = nch + __popc(m & ((1u << lane) - 1u));
        if (is && pos < kMaxChildren) sh.ch[pos] = c;
        nch += __popc(m);
      }
      if (lane == 0) {
        sh.nch = min(nch, kMaxChildren);
        sh.next = -1;
        if (nch > kMaxChildren || sp.status != 0) sh.bad = 1;
      }
    }
    __syncthreads();
    if (sh.bad) break;
    const int nch = sh.nch;
    if (sp.c == 0.0f) {  // greedy: follow the child carrying the verifier argmax
      if (threadIdx.x == 0) {
        for (int k = 0; k < nch; ++k)
          if (sh.tok[sh.ch[k]] == sp.amax) {
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
          toks[len] = sh.tok[next];
        }
        cur = next;
        ++len;
        __syncthreads();
        continue;
      }
      break;  // final token sh.y
    }
    const float ucu = threadIdx.x < nch ? u_acc[n0 + sh.ch[threadIdx.x]] : 0.0f;  // stored after the staging
    RowStat sq = sp;
    if (nch > 0 && !uncut) {
      sq = ds[n0 + cur];
      if (sq.status != 0) {
        if (threadIdx.x == 0) sh.bad = 1;
        __syncthreads();
        break;
      }
    }
    // stage the node's slices (q' only when the node has children); each thread owns the same
    // 8-element groups throughout
    const bool with_q = nch > 0;
    int rb = 0;  // current r' buffer
    float* rs = rbuf(0);
    double sr = 0.0, sqm = 0.0;
    float mp_me = 0.0f, mq_me = 0.0f;  // this slice's maxima (uncut requests)
    {
      const float cut_p = cut_value(sp.tau), cut_q = cut_value(sq.tau);
      // weights of the group at e into the slices, with their 8-term fp32 sums (then fp64)
      auto put = [&](int e, const float(&lp)[8], const float(&lq)[8]) {
        float w[8];
        kept8(lp, sp, cut_p, w);
        store8(rs + (e - v0), w, v1 - e);
        sr += static_cast<double>(sum8(w));
        if (with_q) {
          kept8(lq, sq, cut_q, w);
          store8(qs + (e - v0), w, v1 - e);
          sqm += static_cast<double>(sum8(w));
        }
      };
      // this slice's maxima set the frame of an uncut request's weights
      auto set_frame = [&](float mp, float mq) {
        block_max2(mp, mq, sh.red2);
        mp_me = mp;
        mq_me = mq;
        sp.m = mp > -INFINITY ? mp : 0.0f;  // a slice of -inf: weights 0
        sq.m = mq > -INFINITY ? mq : 0.0f;
      };
      if (regs) {
        // the whole slice in registers: maxima, then weights
        const int e0 = v0 + threadIdx.x * 8;
        float mp = -INFINITY, mq = -INFINITY;
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
          if (e0 + j * kStep >= v1) continue;
          float lp[8], lq[8];
          xp[j].unpack(lp);
          xq[j].unpack(lq);
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // values past the end were filled with -inf
            mp = fmax_nan(mp, lp[k]);
            if (with_q) mq = fmax_nan(mq, lq[k]);
          }
        }
        set_frame(mp, mq);
#pragma unroll
        for (int j = 0; j < kStageBatch; ++j) {
          const int e = e0 + j * kStep;
          if (e >= v1) continue;
          float lp[8], lq[8];
          xp[j].unpack(lp);
          xq[j].unpack(lq);
          put(e, lp, lq);
        }
      } else {
        // batches: raw logits into the slices first when the frame is not known yet
        float mp = -INFINITY, mq = -INFINITY;
        for (int e0 = v0 + threadIdx.x * 8; e0 < v1; e0 += kStageBatch * kStep) {
          load_batch(e0);
#pragma unroll
          for (int j = 0; j < kStageBatch; ++j) {
            const int e = e0 + j * kStep;
            if (e >= v1) continue;
            float lp[8], lq[8];
            xp[j].unpack(lp);
            xq[j].unpack(lq);
            if (uncut) {
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                mp = fmax_nan(mp, lp[k]);
                if (with_q) mq = fmax_nan(mq, lq[k]);
              }
              store8(rs + (e - v0), lp, v1 - e);
              if (with_q) store8(qs + (e - v0), lq, v1 - e);
            } else {
              put(e, lp, lq);
            }
          }
        }
        if (uncut) {
          set_frame(mp, mq);
          for (int e = v0 + threadIdx.x * 8; e < v1; e += kStep) {  // the groups this thread wrote
            float lp[8], lq[8];
            load8(rs + (e - v0), lp, v1 - e);
            if (with_q) load8(qs + (e - v0), lq, v1 - e);
            put(e, lp, lq);
          }
        }
      }
    }
    if (threadIdx.x < nch) sh.cu[threadIdx.x] = ucu;
    block_sum2(sr, sqm, sh.red2);  // also makes the staged slice visible to the whole CTA
    // exchange: slice totals, slice maxima, and r'(t), q'(t) of the first child's token
    int tnext = nch > 0 ? sh.tok[sh.ch[0]] : -1;
    int pick = owner_of(tnext);
    {
      const bool mine = pick == rank;
      const double v[kXVals] = {sr, sqm, mp_me, mq_me, mine ? rs[tnext - v0] : 0.0, mine ? qs[tnext - v0] : 0.0};
      cluster_post<CL>(cl, sh, ph, rank, v);
    }
    double S, Q;
    float rt = 0.0f, qt = 0.0f;
    float fr = 1.0f, fq = 1.0f;  // this slice's factors to the rows' frames
    if (uncut) {
      // the rows' maxima; a NaN or +inf logit, or a row of -inf, is a data error (the same
      // maxima in every CTA)
      const float ml_p = lane < CL ? static_cast<float>(sh.x[ph][lane][2]) : -INFINITY;
      const float ml_q = lane < CL ? static_cast<float>(sh.x[ph][lane][3]) : -INFINITY;
      const float Mp = warp_max(ml_p), Mq = warp_max(ml_q);
      if (!(Mp > -INFINITY && Mp < INFINITY) || (with_q && !(Mq > -INFINITY && Mq < INFINITY))) {
        if (threadIdx.x == 0) sh.bad = 1;
        __syncthreads();
        break;
      }
      const float c = own.c;
      S = xsum<CL>(sh, ph, 0, frame_factor(ml_p, Mp, c));
      Q = with_q ? xsum<CL>(sh, ph, 1, frame_factor(ml_q, Mq, c)) : 0.0;
      if (pick >= 0) {
        rt = static_cast<float>(sh.x[ph][pick][4]) * frame_factor(static_cast<float>(sh.x[ph][pick][2]), Mp, c);
        qt = static_cast<float>(sh.x[ph][pick][5]) * frame_factor(static_cast<float>(sh.x[ph][pick][3]), Mq, c);
      }
      fr = frame_factor(mp_me, Mp, c);
      fq = with_q ? frame_factor(mq_me, Mq, c) : 0.0f;
    } else {
      S = xsum<CL>(sh, ph, 0);
      Q = xsum<CL>(sh, ph, 1);
      if (pick >= 0) {
        rt = static_cast<float>(sh.x[ph][pick][4]);
        qt = static_cast<float>(sh.x[ph][pick][5]);
      }
    }
    ph ^= 1;
    int next = -1;
    for (int k = 0; k < nch; ++k) {
      if (!(Q > 0.0)) break;  // draft mass exhausted: the remaining children are skipped
      const int c = sh.ch[k], tok = sh.tok[c];
      // accept iff u * q~(t) < r(t), with q~ = q' / Q and r = r' / S (every thread decides alike)
      if (static_cast<double>(sh.cu[k]) * static_cast<double>(qt) * S < static_cast<double>(rt) * Q) {
        next = c;
        break;
      }
      // rejected: totals of the residual and of the draft mass without t over float4 vectors
      // of the slice (4-term fp32 sums, then fp64); with dbuf the updated r' goes to the other
      // buffer in the same pass, and the thread holding q'(t) removes t once it has used q'(t)
      const float scale = static_cast<float>(S / Q);
      const int tl = tok - v0;  // t's offset in this slice (outside [0, ns) elsewhere)
      const int n4 = ns >> 2;
      const float4* r4 = reinterpret_cast<const float4*>(rs);
      float4* q4 = reinterpret_cast<float4*>(qs);
      float* os = rbuf(rb ^ 1);
      float4* o4 = reinterpret_cast<float4*>(os);
      double zr = 0.0, zq = 0.0;
      for (int i = threadIdx.x; i < n4; i += kTreeWalkThreads) {
        const float4 r = r4[i];
        float4 q = q4[i];
        float4 o;
        o.x = resid_update(fr * r.x, scale, fq * q.x);
        o.y = resid_update(fr * r.y, scale, fq * q.y);
        o.z = resid_update(fr * r.z, scale, fq * q.z);
        o.w = resid_update(fr * r.w, scale, fq * q.w);
        zr += static_cast<double>((o.x + o.y) + (o.z + o.w));
        const int j = tl - 4 * i;  // the removed token's lane within this vector, if any
        zq += static_cast<double>(((j == 0 ? 0.0f : fq * q.x) + (j == 1 ? 0.0f : fq * q.y)) +
                                  ((j == 2 ? 0.0f : fq * q.z) + (j == 3 ? 0.0f : fq * q.w)));
        if (dbuf) {
          o4[i] = o;
          if (j >= 0 && j < 4) {
            if (j == 0) q.x = 0.0f;
            else if (j == 1) q.y = 0.0f;
            else if (j == 2) q.z = 0.0f;
            else q.w = 0.0f;
            q4[i] = q;
          }
        }
      }
      for (int i = 4 * n4 + threadIdx.x; i < ns; i += kTreeWalkThreads) {
        const float o = resid_update(fr * rs[i], scale, fq * qs[i]);
        zr += static_cast<double>(o);
        if (i != tl) zq += static_cast<double>(fq * qs[i]);
        if (dbuf) {
          os[i] = o;
          if (i == tl) qs[i] = 0.0f;
        }
      }
      block_sum2(zr, zq, sh.red2);
      // the next child's r'(t2), q'(t2) in the rows' frame before this update ride along
      tnext = k + 1 < nch ? sh.tok[sh.ch[k + 1]] : -1;
      pick = owner_of(tnext);
      {
        const bool mine = pick == rank && tnext != tok;
        const double v[kXVals] = {zr, zq, 0.0, 0.0, mine ? fr * rs[tnext - v0] : 0.0, mine ? fq * qs[tnext - v0] : 0.0};
        cluster_post<CL>(cl, sh, ph, rank, v);
      }
      const double zS = xsum<CL>(sh, ph, 0), zQ = xsum<CL>(sh, ph, 1);
      // t2 == t (a repeated sibling token): its values are the ones just tested
      const float r2 = tnext == tok ? rt : pick >= 0 ? static_cast<float>(sh.x[ph][pick][4]) : 0.0f;
      const float q2 = tnext == tok ? qt : pick >= 0 ? static_cast<float>(sh.x[ph][pick][5]) : 0.0f;
      ph ^= 1;
      if (zS > 0.0) {
        if (dbuf) {
          rb ^= 1;
          rs = rbuf(rb);
        } else {
          float4* w4 = reinterpret_cast<float4*>(rs);
          for (int i = threadIdx.x; i < n4; i += kTreeWalkThreads) {
            float4 r = w4[i];
            const float4 q = q4[i];
            r.x = resid_update(fr * r.x, scale, fq * q.x);
            r.y = resid_update(fr * r.y, scale, fq * q.y);
            r.z = resid_update(fr * r.z, scale, fq * q.z);
            r.w = resid_update(fr * r.w, scale, fq * q.w);
            w4[i] = r;
          }
          for (int i = 4 * n4 + threadIdx.x; i < ns; i += kTreeWalkThreads)
            rs[i] = resid_update(fr * rs[i], scale, fq * qs[i]);
        }
        fr = 1.0f;  // the slice now holds r' in the rows' frame
        S = zS;
        rt = resid_update(r2, scale, q2);
      } else {
        rt = r2;
      }
      if (!dbuf && rank == owner_of(tok)) {  // t leaves the draft once every thread has used q'(t)
        __syncthreads();
        if (threadIdx.x == 0) qs[tl] = 0.0f;
      }
      Q = zQ;
      qt = tnext == tok ? 0.0f : q2;
      if (!dbuf) __syncthreads();  // the updated slice is complete before the next pass reads it
    }
    if (next >= 0) {
      if (writer) {
        path[len] = next;
        toks[len] = sh.tok[next];
      }
      cur = next;
      ++len;
      __syncthreads();
      continue;
    }
    // final draw from r at this node: contiguous runs per thread, scanned in thread order
    // inside each slice, slices in rank order
    __syncthreads();  // the slice's last writes are visible to every thread
    const int run = (ns + kTreeWalkThreads - 1) / kTreeWalkThreads;
    const int r0 = min(ns, static_cast<int>(threadIdx.x) * run), r1 = min(ns, r0 + run);
    double mine = 0.0;
    int last = -1;
    for (int i = r0; i < r1; ++i) {
      const float w = fr * rs[i];
      mine += static_cast<double>(w);
      if (w > 0.0f) last = v0 + i;
    }
    double total;
    const double C0 = block_exclusive_scan(mine, sh.red, &total);
    if (threadIdx.x < CL) *cl.map_shared_rank(&sh.xt[rank], static_cast<int>(threadIdx.x)) = total;
    if (threadIdx.x == 0) {
      sh.islot[0] = 0x7fffffff;  // drawn index, if it falls in this slice
      sh.islot[1] = -1;          // last index with positive weight in this slice
    }
    cl.sync();
    // the slices' totals in rank order: the same running sums in every CTA
    const double lane_total = lane < CL ? sh.xt[lane] : 0.0;
    double base = 0.0, grand = 0.0;
#pragma unroll
    for (int r = 0; r < CL; ++r) {
      const double tr = __shfl_sync(0xffffffffu, lane_total, r);
      if (r < rank) base += tr;
      grand += tr;
    }
    const double target = static_cast<double>(u_res[n0 + cur]) * grand;
    if (last >= 0) atomicMax(&sh.islot[1], last);
    if (base + C0 <= target && target < base + C0 + mine) {
      double C = base + C0;
      for (int i = r0; i < r1; ++i) {
        const float w = fr * rs[i];
        C += static_cast<double>(w);
        if (C > target && w > 0.0f) {
          atomicMin(&sh.islot[0], v0 + i);
          break;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // this slice's pick to rank 0 (visible after the final barrier)
      int* dst = cl.map_shared_rank(&sh.xi[rank][0], 0);
      dst[0] = sh.islot[0];
      dst[1] = sh.islot[1];
    }
    drew = true;
    break;
  }
  cl.sync();  // the picks have landed; no CTA leaves while another may still read its memory
  if (writer) {
    if (sh.bad) {
      for (int i = 0; i < max_depth; ++i) path[i] = -1;
      for (int i = 0; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = -1;
    } else {
      int y = sh.y;
      if (drew) {
        int pick = 0x7fffffff, lastpos = -1;
        for (int r = 0; r < CL; ++r) {
          pick = min(pick, sh.xi[r][0]);
          lastpos = max(lastpos, sh.xi[r][1]);
        }
        y = pick != 0x7fffffff ? pick : lastpos;  // rounding past every slice: the last positive index
      }
      for (int i = len; i < max_depth; ++i) path[i] = -1;
      toks[len] = y;
      for (int i = len + 1; i <= max_depth; ++i) toks[i] = -1;
      out_len[b] = len;
    }
  }
}

}  // namespace psi
