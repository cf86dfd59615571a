"""Seeded synthetic inputs for the verification step: logits, uniforms, trie topologies.

This module holds none of the method's arithmetic (no softmax, no top-p, no acceptance
rule). It is the one piece shared by the CUDA path's callers and the oracle's tests: both
consume exactly the tensors produced here.

Shapes and value distributions follow the five workloads the build is measured on (the pages
measure end-to-end decoding with 1K random input / 8K output tokens on real models, review page
section 5.1; these synthetic rows stand in for the verifier and drafter heads):

  tiny     B=1,   K=4,  V=1024,   fp32, target N(0, 2^2), draft = target + N(0, 0.5^2), T=1
  mid      B=64,  K=8,  V=151936, bf16, target N(0, 3^2) + 8 * rank^-1.1 (a seeded permutation
                                  ranks the vocabulary per request), draft = target + N(0, 1), T=1
  max      B=512, K=16, V=151936, bf16, target N(0, 2^2), draft noise std ~ U(0.25, 2) per
                                  request, T=1, top-p 0.95
  tree     B=4 tries x 64 nodes, depth <= 8, branching <= 4, bf16, rows as "tiny" (target
                                  N(0, 2^2), draft noise 0.5), child tokens drawn without
                                  replacement from the parent's draft distribution; tree_deep the
                                  same with draft = target (walks to full depth)
  sweep    B in {1, 32, 256}, K=32, V=151936, bf16, draft std 0.5, T in {0, 0.7, 1}, top-p 0.9
  trie     the tree sampler's candidate trie: B=16 requests (trie_32_b1: one, the operating
           point's own batch), K=15 drafted positions (a block of 16 whose first token is the
           verifier's), V=151936, bf16, draft rows N(0, 1) plus 14 * r^-1.1 on the token of rank r
           of a seeded per-row ranking (peaked: the rank-1 token holds about 0.8 of a row's
           mass), T=1; cand_k=32 candidates per position, 32 kept prefixes (review page section
           3.4's single-request optimum) or 60 (the README's tree example); the verifier row of
           a node at depth d is the draft row of position d plus N(0, 0.5^2)

Uniforms are fp32 values k * 2^-24 (k a uniform 24-bit integer from numpy's PCG64), so fp32
and fp64 consumers see the same numbers.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

V_QWEN = 151936


@dataclass
class LinearCase:
    name: str
    B: int
    K: int
    V: int
    dtype: torch.dtype
    target_std: float
    draft_std: float | tuple  # scalar, or (lo, hi) for a per-request U(lo, hi) std
    temperature: float
    top_p: float
    zipf_bias: float = 0.0  # amplitude of the rank bias; 0 disables it
    zipf_exponent: float = 1.1
    seed: int = 0
    top_k: int = 0  # per-request top-k of every request (0: off)


@dataclass
class TreeCase:
    name: str
    B: int
    nodes: int
    max_depth: int
    max_branch: int
    V: int
    dtype: torch.dtype
    target_std: float
    draft_std: float
    temperature: float
    top_p: float
    seed: int = 0


def linear_cases():
    """The linear workloads by name (parity sizes and the benchmarked sizes)."""
    bf = torch.bfloat16
    c = {
        "tiny": LinearCase("tiny", 1, 4, 1024, torch.float32, 2.0, 0.5, 1.0, 1.0, seed=0),
        "mid": LinearCase("mid", 64, 8, V_QWEN, bf, 3.0, 1.0, 1.0, 1.0, zipf_bias=8.0, seed=1001),
        "max": LinearCase("max", 512, 16, V_QWEN, bf, 2.0, (0.25, 2.0), 1.0, 0.95, seed=1002),
        # the default workload's sizes and logits under top-k 50 and top-p 0.95
        "mid_topk": LinearCase("mid_topk", 64, 8, V_QWEN, bf, 3.0, 1.0, 1.0, 0.95, zipf_bias=8.0, seed=1001, top_k=50),
    }
    for B in (1, 32, 256):
        for T in (0.0, 0.7, 1.0):
            key = "sweep_b%d_t%g" % (B, T)
            c[key] = LinearCase(key, B, 32, V_QWEN, bf, 2.0, 0.5, T, 0.9, seed=1004)
    return c


def tree_cases():
    return {
        "tree": TreeCase("tree", 4, 64, 8, 4, V_QWEN, torch.bfloat16, 2.0, 0.5, 1.0, 1.0, seed=1003),
        # the drafter equal to the verifier: every first child is accepted, walks reach full depth
        "tree_deep": TreeCase("tree_deep", 4, 64, 8, 4, V_QWEN, torch.bfloat16, 2.0, 0.0, 1.0, 1.0, seed=1007),
    }


def uniforms(shape, seed: int) -> torch.Tensor:
    """fp32 uniforms in [0, 1) on the 2^-24 grid, from numpy PCG64 (host tensor)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    k = rng.integers(0, 1 << 24, size=shape, dtype=np.int64)
    return torch.from_numpy((k.astype(np.float64) * 2.0**-24).astype(np.float32))


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draft_std(case, B, seed):
    if isinstance(case.draft_std, tuple):
        lo, hi = case.draft_std
        rng = np.random.Generator(np.random.PCG64(seed + 7))
        return torch.from_numpy(rng.uniform(lo, hi, size=B).astype(np.float32))
    return torch.full((B,), float(case.draft_std))


@dataclass
class TrieCase:
    name: str
    B: int
    K: int
    V: int
    dtype: torch.dtype
    draft_std: float
    target_noise: float
    temperature: float
    top_p: float
    cand_k: int
    n_prefixes: int
    seed: int = 0
    zipf_bias: float = 0.0  # amplitude of a per-row rank bias; 0 disables it
    zipf_exponent: float = 1.1


def trie_cases():
    bf = torch.bfloat16
    # peaked rows: the rank-1 token of a row holds about 0.8 of its mass (bias 14 over
    # N(0, 1) logits of 151936 tokens), the next ranks fall off as r^-1.1
    return {
        "trie_32": TrieCase("trie_32", 16, 15, V_QWEN, bf, 1.0, 0.5, 1.0, 1.0, 32, 32, seed=1005, zipf_bias=14.0),
        "trie_60": TrieCase("trie_60", 16, 15, V_QWEN, bf, 1.0, 0.5, 1.0, 1.0, 32, 60, seed=1006, zipf_bias=14.0),
        # the single-request operating point itself (batch 1)
        "trie_32_b1": TrieCase("trie_32_b1", 1, 15, V_QWEN, bf, 1.0, 0.5, 1.0, 1.0, 32, 32, seed=1008, zipf_bias=14.0),
    }


def trie_draft(case: TrieCase, device="cpu"):
    """Draft rows [B, K, V] of the candidate-trie workload: N(0, draft_std^2) logits plus, with
    zipf_bias, bias * r^-exponent on the token of rank r of a seeded per-row ranking."""
    dev = torch.device(device)
    g = _gen(dev, case.seed)
    d = torch.randn((case.B, case.K, case.V), generator=g, device=dev, dtype=torch.float32) * case.draft_std
    if case.zipf_bias:
        bias = case.zipf_bias * torch.arange(1, case.V + 1, device=dev, dtype=torch.float32).pow(-case.zipf_exponent)
        for b in range(case.B):
            for k in range(case.K):
                perm = torch.randperm(case.V, generator=g, device=dev)
                d[b, k, perm] += bias
    return d.to(case.dtype)


def trie_verifier_rows(case: TrieCase, draft: torch.Tensor, depth: torch.Tensor):
    """Verifier rows of the trie's nodes: [B * (n_prefixes + 1), V] for depth [B, n_prefixes + 1]
    (a node at depth d < K gets draft row d plus noise; depth K or an unused slot, noise alone)."""
    B, K, V = draft.shape
    dev = draft.device
    g = _gen(dev, case.seed + 1)
    dep = depth.to(dev).long()
    base = torch.zeros((B, dep.shape[1], V), dtype=torch.float32, device=dev)
    has = (dep >= 0) & (dep < K)
    dep = dep.clamp(min=0)
    idx = dep.clamp(max=K - 1)
    rows = torch.gather(draft.float(), 1, idx.unsqueeze(-1).expand(-1, -1, V))
    base = torch.where(has.unsqueeze(-1), rows, base)
    noise = torch.randn(base.shape, generator=g, device=dev, dtype=torch.float32) * case.target_noise
    return (base + noise).to(case.dtype).reshape(-1, V)


def trie_uniforms(case: TrieCase):
    n = case.B * (case.n_prefixes + 1)
    s = case.seed * 16
    return uniforms((n,), s + 2), uniforms((n,), s + 3)


def linear_logits(case: LinearCase, device="cpu", B: int | None = None, chunk_rows: int = 2048):
    """Returns (target [B, K+1, V], draft [B, K, V]) in case.dtype on `device`.

    Values are drawn in fp32 with a seeded torch generator on `device`, in chunks of requests
    so that peak memory stays near the output size, then rounded to the case dtype.
    """
    B = case.B if B is None else B
    K, V = case.K, case.V
    dev = torch.device(device)
    g = _gen(dev, case.seed)
    target = torch.empty((B, K + 1, V), dtype=case.dtype, device=dev)
    draft = torch.empty((B, K, V), dtype=case.dtype, device=dev)
    stds = _draft_std(case, B, case.seed).to(dev)
    per = max(1, chunk_rows // (K + 1))
    for b0 in range(0, B, per):
        b1 = min(B, b0 + per)
        n = b1 - b0
        t = torch.randn((n, K + 1, V), generator=g, device=dev, dtype=torch.float32) * case.target_std
        if case.zipf_bias:
            # a per-request seeded ranking of the vocabulary; rank r gets bias * r^-exponent
            for i in range(n):
                perm = torch.randperm(V, generator=g, device=dev)
                bias = case.zipf_bias * torch.arange(1, V + 1, device=dev, dtype=torch.float32).pow(-case.zipf_exponent)
                t[i, :, perm] += bias
        noise = torch.randn((n, K, V), generator=g, device=dev, dtype=torch.float32)
        d = t[:, :K, :] + noise * stds[b0:b1].view(n, 1, 1)
        target[b0:b1] = t.to(case.dtype)
        draft[b0:b1] = d.to(case.dtype)
        del t, noise, d
    return target, draft


def linear_uniforms(case: LinearCase, B: int | None = None):
    """(u_draft [B, K], u_accept [B, K], u_resid [B, K+1]) host fp32 tensors."""
    B = case.B if B is None else B
    s = case.seed * 16
    return (uniforms((B, case.K), s + 1), uniforms((B, case.K), s + 2), uniforms((B, case.K + 1), s + 3))


def gumbel_tokens(draft: torch.Tensor, temperature: float, seed: int, k: int = 1) -> torch.Tensor:
    """k distinct tokens per row via the Gumbel-top-k trick on logits / T (argmax for T == 0).

    Used only to synthesise plausible draft tokens where no sampler output is wanted (for
    example the rows a parity test does not compare); [rows, V] -> [rows, k] int32.
    """
    x = draft.float()
    if temperature > 0:
        g = _gen(x.device, seed)
        u = torch.rand(x.shape, generator=g, device=x.device, dtype=torch.float32).clamp_(1e-12, 1.0)
        x = x / temperature - torch.log(-torch.log(u))
    return torch.topk(x, k, dim=-1).indices.to(torch.int32)


@dataclass
class Trie:
    node_offsets: torch.Tensor  # [B+1] int32
    parent: torch.Tensor  # [N] int32, request-local parent index, -1 at roots
    depth: torch.Tensor  # [N] int32
    N: int = 0
    children: list = field(default_factory=list)  # per global node: list of global child ids


def trie_topology(B: int, nodes: int, max_depth: int, max_branch: int, seed: int) -> Trie:
    """Random tries: node i > 0 picks a uniformly random earlier node whose depth is below
    max_depth and whose child count is below max_branch."""
    rng = np.random.Generator(np.random.PCG64(seed))
    parent = np.full(B * nodes, -1, np.int32)
    depth = np.zeros(B * nodes, np.int32)
    children = [[] for _ in range(B * nodes)]
    for b in range(B):
        base = b * nodes
        nchild = np.zeros(nodes, np.int32)
        for i in range(1, nodes):
            ok = [j for j in range(i) if depth[base + j] < max_depth and nchild[j] < max_branch]
            j = int(ok[rng.integers(0, len(ok))])
            parent[base + i] = j
            depth[base + i] = depth[base + j] + 1
            nchild[j] += 1
            children[base + j].append(base + i)
    off = np.arange(0, B * nodes + 1, nodes, dtype=np.int32)
    return Trie(torch.from_numpy(off), torch.from_numpy(parent), torch.from_numpy(depth), B * nodes, children)


def tree_inputs(case: TreeCase, device="cpu"):
    """Trie, per-node target/draft rows [N, V], child tokens [N] and uniforms [N].

    Child tokens of a node are distinct and drawn without replacement from softmax(q / T) of
    that node's draft row (Gumbel-top-k), so acceptance rates are realistic."""
    trie = trie_topology(case.B, case.nodes, case.max_depth, case.max_branch, case.seed)
    N, V = trie.N, case.V
    dev = torch.device(device)
    g = _gen(dev, case.seed)
    t = torch.randn((N, V), generator=g, device=dev, dtype=torch.float32) * case.target_std
    d = t + torch.randn((N, V), generator=g, device=dev, dtype=torch.float32) * case.draft_std
    target, draft = t.to(case.dtype), d.to(case.dtype)
    tokens = torch.zeros(N, dtype=torch.int32)
    parents_with_children = [n for n in range(N) if trie.children[n]]
    if parents_with_children:
        kmax = case.max_branch
        idx = torch.tensor(parents_with_children, device=dev)
        picks = gumbel_tokens(draft[idx], case.temperature, case.seed + 11, k=kmax).cpu()
        for row, n in enumerate(parents_with_children):
            for k, c in enumerate(trie.children[n]):
                tokens[c] = int(picks[row, k])
    s = case.seed * 16
    return trie, target, draft, tokens, uniforms((N,), s + 2), uniforms((N,), s + 3)
