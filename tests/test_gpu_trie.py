"""Parity of the candidate-trie kernels (psispec_build_tree) with the oracle, on a B200.

Prefixes of one length are compared by their exact logit sums on both sides. Prefixes of
different lengths are compared by fp64 probabilities, which the kernels form from fp32 row
statistics and the oracle in fp64 throughout. So a request whose oracle order holds a
near-tie between prefixes of different lengths (a relative gap within 1e-5), or a top-p
threshold within its band, is counted, not compared. Every other request must give the
identical trie, and its probabilities must agree to a relative 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import band_limit, compare_tree, tree_recheck
from lossless_speculative_sampling_b200 import psispec, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
REL = 1e-5


def _in_band(d, T, top_p, top_k, cand_k, n):
    for row in d:
        if oracle.row_dist(row, T, top_p, top_k)[1] < 1e-6:
            return True
    more = oracle.build_tree(d, T, top_p, cand_k, n + 1, top_k=top_k)
    s, dep = more["score"][1:], more["depth"][1:]
    for i in range(len(s) - 1):
        for j in range(i + 1, len(s)):
            if dep[i] != dep[j] and s[i] != s[j] and abs(s[i] - s[j]) <= REL * max(s[i], s[j]):
                return True
    return False


@pytest.mark.parametrize("K,V,dtype,T,top_p,cand_k,n", [
    (3, 5000, torch.float32, 1.0, 1.0, 4, 20),
    (4, 20011, torch.bfloat16, 0.8, 0.9, 8, 60),
    (2, 151936, torch.bfloat16, 1.0, 0.95, 32, 60),
    (3, 3000, torch.bfloat16, 0.0, 1.0, 4, 10),
    (5, 40000, torch.bfloat16, 1.0, 1.0, 1, 8),
])
def test_build_tree_parity(K, V, dtype, T, top_p, cand_k, n):
    B = 4
    g = torch.Generator().manual_seed(V + K)
    d = (torch.randn((B, K, V), generator=g) * 3.0).to(dtype)
    d[1, 1] = d[1, 0]  # a repeated row: exact ties between prefixes
    Ts, Ps = torch.full((B,), T), torch.full((B,), top_p)
    out = psispec.build_tree(d.to(DEV), Ts.to(DEV), Ps.to(DEV), cand_k, n)
    got = {k: v.cpu().numpy() for k, v in out.items()}
    host = d.float().numpy().astype(np.float64)
    banded = 0
    for b in range(B):
        ora = oracle.build_tree(host[b], T, top_p, cand_k, n)
        if _in_band(host[b], T, top_p, 0, cand_k, n):
            banded += 1
            continue
        m = len(ora["parent"])
        assert got["nodes"][b] == m
        assert np.array_equal(got["parent"][b, :m], ora["parent"])
        assert np.array_equal(got["tokens"][b, :m], ora["tokens"])
        assert np.array_equal(got["depth"][b, :m], ora["depth"])
        assert np.allclose(got["score"][b, :m], ora["score"], rtol=REL, atol=0.0)
        assert (got["parent"][b, m:] == -1).all()
    assert banded < B


def test_build_tree_top_k_and_data_errors():
    B, K, V, n = 3, 3, 9001, 30
    g = torch.Generator().manual_seed(5)
    d = (torch.randn((B, K, V), generator=g) * 2.0).to(torch.bfloat16)
    d[2, 1, 17] = float("nan")  # request 2: a data error
    Ts, Ps = torch.tensor([1.0, 0.7, 1.0]), torch.tensor([1.0, 0.9, 1.0])
    Ks = torch.tensor([3, 50, 0], dtype=torch.int32)
    out = psispec.build_tree(d.to(DEV), Ts.to(DEV), Ps.to(DEV), 6, n, top_k=Ks.to(DEV))
    got = {k: v.cpu().numpy() for k, v in out.items()}
    host = d.float().numpy().astype(np.float64)
    assert got["nodes"][2] == -1 and (got["parent"][2] == -1).all()
    for b in range(2):
        ora = oracle.build_tree(host[b], float(Ts[b]), float(Ps[b]), 6, n, top_k=int(Ks[b]))
        if _in_band(host[b], float(Ts[b]), float(Ps[b]), int(Ks[b]), 6, n):
            continue
        m = len(ora["parent"])
        assert got["nodes"][b] == m
        assert np.array_equal(got["tokens"][b, :m], ora["tokens"])
        assert np.array_equal(got["parent"][b, :m], ora["parent"])


@pytest.mark.parametrize("V,dtype,T,top_p", [(3000, torch.float32, 1.0, 1.0), (20011, torch.bfloat16, 0.8, 0.9),
                                             (151936, torch.bfloat16, 1.0, 0.95), (4000, torch.bfloat16, 0.0, 1.0)])
def test_verify_tree_det_parity(V, dtype, T, top_p):
    """Candidate tries (built by the oracle) verified with the deterministic-candidate rule:
    every node's verifier row is its position's draft row plus noise, so children are accepted
    as well as rejected; results identical to the oracle's outside the bands."""
    B, K, ck, n = 4, 3, 4, 12
    g = torch.Generator().manual_seed(V + 9)
    drafts = (torch.randn((B, K, V), generator=g) * 4.0).to(dtype)
    offs, par, tok, rows = [0], [], [], []
    for b in range(B):
        t = oracle.build_tree(drafts[b].float().numpy().astype(np.float64), T, top_p, ck, n)
        tk = t["tokens"].copy()
        tk[0] = 0  # the root's token is not read
        par.append(t["parent"])
        tok.append(tk)
        offs.append(offs[-1] + len(tk))
        for dep in t["depth"]:
            base = drafts[b, dep].float() if dep < K else torch.zeros(V)
            rows.append(base + torch.randn(V, generator=g) * 0.5)
    N = offs[-1]
    tgt = torch.stack(rows).to(dtype)
    par, tok = np.concatenate(par).astype(np.int32), np.concatenate(tok).astype(np.int32)
    ua, ur = synth.uniforms((N,), V + 1), synth.uniforms((N,), V + 2)
    Ts, Ps = torch.full((B,), T), torch.full((B,), top_p)
    out = psispec.verify_tree_det(tgt.to(DEV), torch.tensor(offs, dtype=torch.int32, device=DEV),
                                  torch.from_numpy(par).to(DEV), torch.from_numpy(tok).to(DEV), ua.to(DEV), ur.to(DEV),
                                  Ts.to(DEV), Ps.to(DEV), K)
    ora = oracle.verify_tree(tgt, tgt, np.array(offs), par, tok, ua, ur, Ts.numpy(), Ps.numpy(), K,
                             rule=oracle.TREE_DETERMINISTIC)
    rc = tree_recheck(tgt, tgt, np.array(offs), par, tok, ua, ur, Ts, Ps, K, rule=oracle.TREE_DETERMINISTIC)
    compare_tree(out, ora, recheck=rc, limit=band_limit(B, V, 1.0, 2 * N / B if top_p < 1 else 0),
                 label="deterministic tree %s" % ((V, T, top_p),))
