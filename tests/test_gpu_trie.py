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


@pytest.mark.parametrize("V,dtype,T,top_p,ck,n", [(3000, torch.float32, 1.0, 1.0, 4, 12),
                                                  (20011, torch.bfloat16, 0.8, 0.9, 4, 12),
                                                  (151936, torch.bfloat16, 1.0, 0.95, 4, 12),
                                                  (4000, torch.bfloat16, 0.0, 1.0, 4, 12),
                                                  (20011, torch.bfloat16, 1.0, 1.0, 32, 48),
                                                  (5003, torch.float32, 1.3, 1.0, 32, 40)])
def test_verify_tree_det_parity(V, dtype, T, top_p, ck, n):
    """Candidate tries (built by the oracle) verified with the deterministic-candidate rule:
    every node's verifier row is its position's draft row plus noise, so children are accepted
    as well as rejected; results identical to the oracle's outside the bands. With 32
    candidates a node's final draw skips up to 32 removed tokens."""
    B, K = 4, 3
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


def _check_build(d, Ts, Ps, cand_k, n, top_k=None):
    """build_tree on the GPU against the oracle, request by request (requests in a band skipped);
    returns the GPU trie and the number compared."""
    B = d.shape[0]
    Ks = top_k if top_k is not None else torch.zeros(B, dtype=torch.int32)
    out = psispec.build_tree(d.to(DEV), Ts.to(DEV), Ps.to(DEV), cand_k, n, top_k=Ks.to(DEV))
    got = {k: v.cpu().numpy() for k, v in out.items()}
    host = d.float().numpy().astype(np.float64)
    compared = 0
    for b in range(B):
        T, tp, tk = float(Ts[b]), float(Ps[b]), int(Ks[b])
        if _in_band(host[b], T, tp, tk, cand_k, n):
            continue
        ora = oracle.build_tree(host[b], T, tp, cand_k, n, top_k=tk)
        m = len(ora["parent"])
        assert got["nodes"][b] == m, (b, got["nodes"][b], m)
        assert np.array_equal(got["parent"][b, :m], ora["parent"]), b
        assert np.array_equal(got["tokens"][b, :m], ora["tokens"]), b
        assert np.array_equal(got["depth"][b, :m], ora["depth"]), b
        assert np.allclose(got["score"][b, :m], ora["score"], rtol=REL, atol=0.0), b
        assert (got["parent"][b, m:] == -1).all()
        compared += 1
    return got, compared


@pytest.mark.parametrize("V", [7, 33, 1000, 20011])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_build_tree_edge_rows(V, dtype):
    """Rows of equal values (every element ties: past the exact ranking's capacity the general
    select takes over), rows with fewer finite values than candidates, one-hot rows, and rows
    quantised to a few values (ties at the pivot resolved by index); unaligned rows for odd V."""
    B, K, cand_k, n = 4, 3, 8, 24
    g = torch.Generator().manual_seed(V * 3 + 1)
    d = torch.randn((B, K, V), generator=g)
    d[0] = 1.5
    d[1] = -float("inf")
    for k in range(K):
        idx = torch.randperm(V, generator=g)[:min(V, 5 + k * 3)]
        d[1, k, idx] = torch.randn(len(idx), generator=g)
    d[2, :, min(V - 1, 3)] = 40.0
    d[3] = torch.round(d[3] * 2.0) / 2.0
    d = d.to(dtype)
    Ts, Ps = torch.ones(B), torch.ones(B)
    _, compared = _check_build(d, Ts, Ps, cand_k, n)
    assert compared >= 2


def test_build_tree_long_rows():
    """V = 600000 (a lane block spans two steps: the block table's capacity decides)."""
    B, K, V = 2, 2, 600000
    g = torch.Generator().manual_seed(77)
    d = (torch.randn((B, K, V), generator=g) * 2.0).to(torch.bfloat16)
    _, compared = _check_build(d, torch.ones(B), torch.tensor([1.0, 0.9]), 32, 40)
    assert compared >= 1


@pytest.mark.parametrize("name", ["trie_32", "trie_60", "trie_32_b1"])
def test_full_size_trie(name):
    """The candidate-trie workloads at full size: every request's trie against the oracle's,
    then the deterministic-rule verification of those tries against the oracle."""
    case = synth.trie_cases()[name]
    B, K, V, n = case.B, case.K, case.V, case.n_prefixes
    d = synth.trie_draft(case, device="cpu")
    Ts, Ps = torch.full((B,), case.temperature), torch.full((B,), case.top_p)
    got, compared = _check_build(d, Ts, Ps, case.cand_k, n)
    assert compared >= B - 2
    assert (got["nodes"] == n + 1).all()
    dep = torch.from_numpy(got["depth"])
    tgt = synth.trie_verifier_rows(case, d, dep)
    ua, ur = synth.trie_uniforms(case)
    cap = n + 1
    offs = np.arange(0, B * cap + 1, cap)
    par = got["parent"].reshape(-1).astype(np.int32)
    tok = got["tokens"].reshape(-1).astype(np.int32)
    out = psispec.verify_tree_det(tgt.to(DEV), torch.from_numpy(offs.astype(np.int32)).to(DEV),
                                  torch.from_numpy(par).to(DEV), torch.from_numpy(tok).to(DEV), ua.to(DEV), ur.to(DEV),
                                  Ts.to(DEV), Ps.to(DEV), K)
    ora = oracle.verify_tree(tgt, tgt, offs, par, tok, ua, ur, Ts.numpy(), Ps.numpy(), K,
                             rule=oracle.TREE_DETERMINISTIC)
    rc = tree_recheck(tgt, tgt, offs, par, tok, ua, ur, Ts, Ps, K, rule=oracle.TREE_DETERMINISTIC)
    compare_tree(out, ora, recheck=rc, limit=band_limit(B, V, 1.0, 0), label="%s deterministic walk" % name)
    if B >= 8:
        assert float(np.mean(ora["accept_len"])) >= 1.0  # peaked rows: the walks go past the root


@pytest.mark.parametrize("V,dtype", [(20011, torch.bfloat16), (3001, torch.float32), (151936, torch.bfloat16)])
def test_verify_tree_det_mixed_requests_and_data_errors(V, dtype):
    """Per-trie temperature/top-p under the deterministic rule: uncut tries (T > 0, no top-p)
    take the walk's own statistics of the rows they visit, the others the statistics pass;
    -inf logits, unaligned rows (odd V), and data errors confined to their trie (NaN, +inf, no
    finite logit in a visited row; a NaN in a row the walk does not visit is no error)."""
    B, nodes = 8, 24
    trie = synth.trie_topology(B, nodes, 6, 3, 93)
    g = torch.Generator().manual_seed(93)
    tgt = torch.randn((trie.N, V), generator=g) * 3.0
    tgt[torch.rand((trie.N, V), generator=g) < 0.1] = -float("inf")
    Ts = torch.tensor([1.0, 0.8, 0.0, 1.0, 1.0, 1.0, 0.9, 1.2])
    Ps = torch.tensor([1.0, 1.0, 1.0, 0.9, 1.0, 1.0, 0.95, 1.0])
    off = trie.node_offsets
    toks = torch.zeros(trie.N, dtype=torch.int32)
    for n in range(trie.N):
        if trie.children[n]:
            # children among the row's most probable tokens, so walks also accept
            top = torch.topk(tgt[n].nan_to_num(0.0), len(trie.children[n]) + 2).indices
            for k, c in enumerate(trie.children[n]):
                toks[c] = int(top[k + 1])
    tgt[int(off[4]), 5] = float("nan")  # visited root row with a NaN: trie 4
    tgt[int(off[5]), 7] = float("inf")  # root row with +inf: trie 5
    tgt[int(off[6]), :] = -float("inf")  # root row without a finite logit: trie 6
    tgt[int(off[7 + 1]) - 1, 3] = float("nan")  # a late node of trie 7: an error only if visited
    tgt = tgt.to(dtype)
    ua, ur = synth.uniforms((trie.N,), 94), synth.uniforms((trie.N,), 95)
    out = psispec.verify_tree_det(tgt.to(DEV), off.to(DEV), trie.parent.to(DEV), toks.to(DEV), ua.to(DEV),
                                  ur.to(DEV), Ts.to(DEV), Ps.to(DEV), 6)
    ora = oracle.verify_tree(tgt, tgt, off.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur, Ts.numpy(),
                             Ps.numpy(), 6, rule=oracle.TREE_DETERMINISTIC)
    assert ora["accept_len"][4] == ora["accept_len"][5] == ora["accept_len"][6] == -1
    assert (ora["accept_len"][[0, 1, 2, 3]] >= 0).all()
    rc = tree_recheck(tgt, tgt, off.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur, Ts, Ps, 6,
                      rule=oracle.TREE_DETERMINISTIC)
    compare_tree(out, ora, recheck=rc, limit=band_limit(B, V, 1.0, 2 * trie.N / B),
                 label="deterministic mixed tries V=%d" % V)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_build_tree_uncut_data_errors(dtype):
    """Requests sampling with no cut take their row statistics from the candidate kernel's own
    pass: a NaN, a +inf, or a row without a finite value is a data error of its request only."""
    B, K, V, n = 4, 3, 5003, 12
    g = torch.Generator().manual_seed(17)
    d = torch.randn((B, K, V), generator=g) * 2.0
    d[0, 1, 4000] = float("nan")
    d[1, 2, 17] = float("inf")
    d[2, 0] = -float("inf")
    d = d.to(dtype)
    Ts, Ps = torch.ones(B), torch.ones(B)
    out = psispec.build_tree(d.to(DEV), Ts.to(DEV), Ps.to(DEV), 4, n)
    got = {k: v.cpu().numpy() for k, v in out.items()}
    assert list(got["nodes"][:3]) == [-1, -1, -1]
    assert (got["parent"][:3] == -1).all()
    ora = oracle.build_tree(d[3].float().numpy().astype(np.float64), 1.0, 1.0, 4, n)
    m = len(ora["parent"])
    assert got["nodes"][3] == m
    assert np.array_equal(got["tokens"][3, :m], ora["tokens"])
    assert np.array_equal(got["parent"][3, :m], ora["parent"])
