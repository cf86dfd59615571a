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
// Two kernels after the row statistics of the B*K draft rows:
//   trie_candidates_kernel  one CTA per row: a count radix select gives the key of the
//                           cand_k-th largest kept logit; one pass over contiguous per-thread
//                           ranges collects every larger element and, in vocabulary order, the
//                           first of the tied ones; one warp ranks them and computes their q in
//                           fp64 from the row record;
//   trie_select_kernel      one warp per request: best-first choice of the prefixes over a
//                           frontier in shared memory, the products in fp64.
#pragma once

#include "common.cuh"
#include "stats.cuh"
#include "tree.cuh"

namespace psi {

constexpr int kTrieMaxCand = 32;      // cand_k limit (one lane per candidate when ranking)
constexpr int kTrieMaxPrefixes = 64;  // n_prefixes limit
constexpr int kTrieMaxK = 16;         // positions limit (rank paths are kept per node)
constexpr int kTrieThreads = 256;
constexpr int kTrieFrontier = kTrieMaxCand * (kTrieMaxPrefixes + 1) + 1;

struct TrieCandSmem {
  RadixSmem radix;
  double scan[33];
  int gt_idx[kTrieMaxCand];
  int eq_idx[kTrieMaxCand];
  int ngt;
};

// Candidates of draft row `row`: cand_tok[row, r], cand_q[row, r] and their logits cand_l[row,
// r] for r < ncand[row] in rank order; ncand = -1 for a row with a data error.
template <typename T>
__global__ void __launch_bounds__(kTrieThreads) trie_candidates_kernel(const T* __restrict__ draft, int V,
                                                                       const RowStat* __restrict__ stats, int cand_k,
                                                                       int32_t* __restrict__ cand_tok,
                                                                       double* __restrict__ cand_q,
                                                                       double* __restrict__ cand_l,
                                                                       int32_t* __restrict__ ncand) {
  __shared__ TrieCandSmem sm;
  const int64_t row = blockIdx.x;
  const T* rp = draft + row * static_cast<int64_t>(V);
  const RowStat st = stats[row];
  int32_t* tok = cand_tok + row * kTrieMaxCand;
  double* qo = cand_q + row * kTrieMaxCand;
  double* lo = cand_l + row * kTrieMaxCand;
  if (st.status != 0) {
    if (threadIdx.x == 0) ncand[row] = -1;
    return;
  }
  if (st.c == 0.0f) {  // greedy: a point mass on the argmax
    if (threadIdx.x == 0) {
      tok[0] = st.amax;
      qo[0] = 1.0;
      lo[0] = static_cast<double>(load_elem(rp + st.amax));
      ncand[row] = 1;
    }
    return;
  }
  // eligible: kept by the row's threshold and above -inf
  const uint32_t floor_key = max(st.tau, 0x00800000u);
  double above, bucket;
  const uint32_t kc = block_radix_pick<T, true>(rp, V, st, static_cast<double>(cand_k), floor_key, sm.radix, &above,
                                                &bucket);
  constexpr int kShift = sizeof(T) == 2 ? 16 : 0;  // a bf16 select fixes the top 16 key bits
  const uint32_t kcs = kc >> kShift;
  if (threadIdx.x == 0) sm.ngt = 0;
  __syncthreads();
  const int per = (V + kTrieThreads - 1) / kTrieThreads;
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
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int idx = -1;
    uint32_t ks = 0u;
    double q = 0.0, lx = 0.0;
    if (lane < nc) {
      idx = lane < ngt ? sm.gt_idx[lane] : sm.eq_idx[lane - ngt];
      const float x = load_elem(rp + idx);
      lx = static_cast<double>(x);
      ks = fkey(x) >> kShift;
      q = exp2((static_cast<double>(x) - static_cast<double>(st.m)) * static_cast<double>(st.c)) /
          static_cast<double>(st.s_kept);
    }
    // rank: larger key first, then the lower index
    int rank = 0;
    for (int j = 0; j < nc; ++j) {
      const int ij = __shfl_sync(0xffffffffu, idx, j);
      const uint32_t kj = __shfl_sync(0xffffffffu, ks, j);
      if (lane < nc && (kj > ks || (kj == ks && ij < idx))) ++rank;
    }
    // candidates whose q underflows to zero carry no probability: drop them (they rank last)
    const int nz = __popc(__ballot_sync(0xffffffffu, lane < nc && q > 0.0));
    if (lane < nc && rank < nz) {
      tok[rank] = idx;
      qo[rank] = q;
      lo[rank] = lx;
    }
    if (lane == 0) ncand[row] = nz;
  }
}

struct TrieSelSmem {
  double node_score[kTrieMaxPrefixes + 1];
  double node_lsum[kTrieMaxPrefixes + 1];
  int node_par[kTrieMaxPrefixes + 1];
  int node_dep[kTrieMaxPrefixes + 1];
  int node_tok[kTrieMaxPrefixes + 1];
  uint8_t node_rank[kTrieMaxPrefixes + 1][kTrieMaxK];
  double f_score[kTrieFrontier];
  double f_lsum[kTrieFrontier];
  int16_t f_par[kTrieFrontier];
  uint8_t f_rank[kTrieFrontier];
};

// Whether frontier entry a precedes entry b: of different lengths, the higher fp64 probability,
// then the shorter; of one length, the larger logit sum (exact), then the smaller rank path
// (the parents' paths, then the entries' own ranks).
__device__ __forceinline__ bool trie_before(const TrieSelSmem& sm, int a, int b) {
  const int pa = sm.f_par[a], pb = sm.f_par[b];
  const int da = sm.node_dep[pa], db = sm.node_dep[pb];
  if (da != db) {
    const double sa = sm.f_score[a], sb = sm.f_score[b];
    return sa > sb || (sa == sb && da < db);
  }
  const double la = sm.f_lsum[a], lb = sm.f_lsum[b];
  if (la != lb) return la > lb;
  for (int j = 0; j < da; ++j) {
    const int ra = sm.node_rank[pa][j], rb = sm.node_rank[pb][j];
    if (ra != rb) return ra < rb;
  }
  return sm.f_rank[a] < sm.f_rank[b];
}

// Best-first choice of the n_prefixes most probable prefixes of request b (one warp). Outputs
// [B, n_prefixes + 1]: parent, tokens, depth, score; unused slots -1 (score 0); out_nodes[b]
// the node count, or -1 when a draft row of the request has a data error.
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
  for (int i = lane; i < K; i += 32) bad |= ncand[r0 + i] < 0;
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
  if (lane == 0) {
    sm.node_par[0] = -1;
    sm.node_dep[0] = 0;
    sm.node_tok[0] = -1;
    sm.node_score[0] = 1.0;
    sm.node_lsum[0] = 0.0;
  }
  int nf = K > 0 ? ncand[r0] : 0;
  if (lane < nf) {
    sm.f_par[lane] = 0;
    sm.f_rank[lane] = static_cast<uint8_t>(lane);
    sm.f_score[lane] = 1.0 * cand_q[r0 * kTrieMaxCand + lane];
    sm.f_lsum[lane] = 0.0 + cand_l[r0 * kTrieMaxCand + lane];
  }
  __syncwarp();
  int nn = 1;
  while (nn < cap && nf > 0) {
    int best = -1;
    for (int e = lane; e < nf; e += 32)
      if (best < 0 || trie_before(sm, e, best)) best = e;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const int other = __shfl_down_sync(0xffffffffu, best, off);
      if (other >= 0 && (best < 0 || trie_before(sm, other, best))) best = other;
    }
    best = __shfl_sync(0xffffffffu, best, 0);
    const int pa = sm.f_par[best], ra = sm.f_rank[best];
    const int d = sm.node_dep[pa];
    const double s = sm.f_score[best], ls = sm.f_lsum[best];
    __syncwarp();
    if (lane == 0) {
      sm.f_par[best] = sm.f_par[nf - 1];
      sm.f_rank[best] = sm.f_rank[nf - 1];
      sm.f_score[best] = sm.f_score[nf - 1];
      sm.f_lsum[best] = sm.f_lsum[nf - 1];
      sm.node_par[nn] = pa;
      sm.node_dep[nn] = d + 1;
      sm.node_tok[nn] = cand_tok[(r0 + d) * kTrieMaxCand + ra];
      sm.node_score[nn] = s;
      sm.node_lsum[nn] = ls;
      for (int j = 0; j < d; ++j) sm.node_rank[nn][j] = sm.node_rank[pa][j];
      sm.node_rank[nn][d] = static_cast<uint8_t>(ra);
    }
    __syncwarp();
    --nf;
    if (d + 1 < K) {
      const int nkids = ncand[r0 + d + 1];
      if (lane < nkids) {
        sm.f_par[nf + lane] = static_cast<int16_t>(nn);
        sm.f_rank[nf + lane] = static_cast<uint8_t>(lane);
        sm.f_score[nf + lane] = s * cand_q[(r0 + d + 1) * kTrieMaxCand + lane];
        sm.f_lsum[nf + lane] = ls + cand_l[(r0 + d + 1) * kTrieMaxCand + lane];
      }
      nf += nkids;
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

// Tree walk under the deterministic-candidate rule (children fixed in advance, as the
// candidate trie's are): at a node with verifier distribution p, child t is accepted iff
// u < p(t) / R, R the mass of p left after removing the siblings rejected before it; a
// rejection removes t (r = p without the removed tokens, renormalised). Where the walk stops,
// the final token is drawn from that r with u_resid of the node. No draft row is read, and a
// rejection needs no pass over the vocabulary. One CTA per trie; ts = statistics records of
// the verifier rows.
template <typename T>
__global__ void __launch_bounds__(kTreeThreads) tree_walk_det_kernel(
    const T* __restrict__ tgt, int V, const int32_t* __restrict__ offs, const int32_t* __restrict__ parent,
    const int32_t* __restrict__ tokens, const RowStat* __restrict__ ts, const float* __restrict__ u_acc,
    const float* __restrict__ u_res, int max_depth, int32_t* __restrict__ out_path, int32_t* __restrict__ out_tokens,
    int32_t* __restrict__ out_len) {
  __shared__ int depth[kMaxNodes];
  __shared__ int ch[kMaxChildren];
  __shared__ int removed[kMaxChildren];
  __shared__ double red[33];
  __shared__ int sh_bad, sh_nch, sh_next, sh_y, sh_nrem, sh_last;
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
    sh_y = -1;
  }
  __syncthreads();

  int cur = 0, len = 0;
  while (!sh_bad) {
    const RowStat sp = ts[n0 + cur];
    const T* rp = tgt + static_cast<size_t>(n0 + cur) * V;
    if (threadIdx.x == 0) {
      int nch = 0;
      for (int c = cur + 1; c < n; ++c)
        if (parent[n0 + c] == cur) {
          if (nch == kMaxChildren) { sh_bad = 1; break; }
          ch[nch++] = c;
        }
      sh_nch = nch;
      sh_next = -1;
      sh_nrem = 0;
      if (sp.status != 0) sh_bad = 1;
      if (!sh_bad && sp.c == 0.0f) {  // greedy: follow the child carrying the verifier argmax
        for (int k = 0; k < nch; ++k)
          if (tokens[n0 + ch[k]] == sp.amax) { sh_next = ch[k]; break; }
        sh_y = sp.amax;
      } else if (!sh_bad) {
        double R = 1.0;  // mass of p left
        for (int k = 0; k < nch; ++k) {
          const int c = ch[k], t = tokens[n0 + c];
          bool gone = false;
          for (int i = 0; i < sh_nrem; ++i) gone |= removed[i] == t;
          const double pt = gone ? 0.0 : static_cast<double>(kept_weight(sp, load_elem(rp + t))) /
                                             static_cast<double>(sp.s_kept);
          if (R > 0.0 && static_cast<double>(u_acc[n0 + c]) * R < pt) { sh_next = c; break; }
          if (!gone) {
            removed[sh_nrem++] = t;
            R -= pt;
          }
        }
      }
    }
    __syncthreads();
    if (sh_bad) break;
    if (sh_next >= 0) {
      if (threadIdx.x == 0) { path[len] = sh_next; toks[len] = tokens[n0 + sh_next]; }
      cur = sh_next;
      ++len;
      __syncthreads();
      continue;
    }
    if (sp.c == 0.0f) break;  // greedy: final token sh_y

    // final draw from p without the removed tokens: contiguous runs, scanned in thread order
    const int nrem = sh_nrem;
    const int run = (V + blockDim.x - 1) / blockDim.x;
    const int r0 = min(V, static_cast<int>(threadIdx.x) * run), r1 = min(V, r0 + run);
    auto weight = [&](int v) {
      for (int i = 0; i < nrem; ++i)
        if (removed[i] == v) return 0.0f;
      return kept_weight(sp, load_elem(rp + v));
    };
    double mine = 0.0;
    int last = -1;
    for (int v = r0; v < r1; ++v) {
      const float w = weight(v);
      mine += static_cast<double>(w);
      if (w > 0.0f) last = v;
    }
    if (threadIdx.x == 0) {
      sh_y = 0x7fffffff;
      sh_last = -1;
    }
    double total;
    const double C0 = block_exclusive_scan(mine, red, &total);
    const double target = static_cast<double>(u_res[n0 + cur]) * total;
    if (last >= 0) atomicMax(&sh_last, last);
    if (C0 <= target && target < C0 + mine) {
      double C = C0;
      for (int v = r0; v < r1; ++v) {
        C += static_cast<double>(weight(v));
        if (C > target) { atomicMin(&sh_y, v); break; }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && sh_y == 0x7fffffff) sh_y = sh_last;  // rounding, or no mass left (-1)
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
