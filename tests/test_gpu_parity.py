"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Integer results must be identical except on requests the oracle marks in-band (see
tests/parity.py); probabilities agree to 1e-5. Draft tokens fed to verification come from the
oracle's own sampler (or from the input generator for rows the oracle does not check), never
from the CUDA path. Small cases span several 16384-element slices and a ragged tail; the
full-size workloads run in the benchmark's launch configuration and are checked on sampled
requests.
"""
import numpy as np
import pytest
import torch

import oracle
from goldens import load, nums, rows
from parity import (band_limit, compare_linear, compare_sample, compare_tree, linear_recheck, sample_recheck,
                    tree_recheck)
from lossless_speculative_sampling_b200 import psispec, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _cuda(x, dtype=None):
    t = torch.as_tensor(np.asarray(x)) if not isinstance(x, torch.Tensor) else x
    return t.to(DEV, dtype=dtype).contiguous()


def _rand_logits(g, shape, dtype, std=2.0, neg_inf_frac=0.0):
    x = torch.randn(shape, generator=g) * std
    if neg_inf_frac:
        x[torch.rand(shape, generator=g) < neg_inf_frac] = -float("inf")
    return x.to(dtype)


def check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, Ks=None, label="", check_pq=True):
    """compare_linear with the oracle recheck of in-band requests and the in-band bound."""
    B, K1, V = tgt.shape
    cut = bool((np.asarray(Ps) < 1).any()) or Ks is not None
    return compare_linear(out, ora, check_pq=check_pq, recheck=linear_recheck(tgt, drf, x, ua, ur, Ts, Ps, Ks),
                          limit=band_limit(B, V, 1.0, 2 * K1 - 1 if cut else 0), label=label)


def check_sample(tok, q, ora, drf_rows, Ts, Ps, u, row_req, Ks=None, label=""):
    n, V = drf_rows.shape
    cut = bool((np.asarray(Ps) < 1).any()) or Ks is not None
    return compare_sample(tok, q, ora, recheck=sample_recheck(drf_rows, Ts, Ps, u, row_req, Ks),
                          limit=band_limit(n, V, 1.0, 1 if cut else 0), label=label)


def check_tree(out, ora, tgt, drf, offs, parent, toks, ua, ur, Ts, Ps, D, Ks=None, label=""):
    N, V = tgt.shape
    B = len(offs) - 1
    cut = bool((np.asarray(Ps) < 1).any()) or Ks is not None
    return compare_tree(out, ora, recheck=tree_recheck(tgt, drf, offs, parent, toks, ua, ur, Ts, Ps, D, Ks),
                        limit=band_limit(B, V, 1.0, 2 * N / B if cut else 0), label=label)


# ------------------------------------------------------------------ worked examples


@pytest.mark.parametrize("case", load("linear.txt"), ids=lambda c: c["name"])
def test_golden_linear_gpu(case):
    tgt, drf = rows(case["target"]), rows(case["draft"])
    K, V = drf.shape
    out = psispec.verify_linear(_cuda(tgt[None], torch.float32), _cuda(drf[None], torch.float32),
                                _cuda(np.array(nums(case["tokens"]), np.int32)[None]),
                                _cuda(nums(case["u_accept"]), torch.float32), _cuda(nums(case["u_resid"]), torch.float32),
                                _cuda([nums(case["T"])[0]], torch.float32), _cuda([nums(case["top_p"])[0]], torch.float32))
    assert int(out["accept_len"][0]) == int(nums(case["expect_len"])[0])
    assert out["tokens"][0].tolist() == [int(x) for x in nums(case["expect_tokens"])]
    np.testing.assert_allclose(out["p"][0].cpu().numpy(), nums(case["expect_p"]), atol=1e-6)
    np.testing.assert_allclose(out["q"][0].cpu().numpy(), nums(case["expect_q"]), atol=1e-6)


@pytest.mark.parametrize("case", load("tree.txt"), ids=lambda c: c["name"])
def test_golden_tree_gpu(case):
    tgt, drf = rows(case["target"]), rows(case["draft"])
    n = tgt.shape[0]
    md = int(case["max_depth"])
    out = psispec.verify_tree(_cuda(tgt, torch.float32), _cuda(drf, torch.float32), _cuda(np.array([0, n], np.int32)),
                              _cuda(np.array(nums(case["parent"]), np.int32)), _cuda(np.array(nums(case["tokens"]), np.int32)),
                              _cuda(nums(case["u_accept"]), torch.float32), _cuda(nums(case["u_resid"]), torch.float32),
                              _cuda([nums(case["T"])[0]], torch.float32), _cuda([nums(case["top_p"])[0]], torch.float32), md)
    assert int(out["accept_len"][0]) == int(nums(case["expect_len"])[0])
    assert out["path"][0].tolist() == [int(x) for x in nums(case["expect_path"])]
    assert out["tokens"][0].tolist() == [int(x) for x in nums(case["expect_tokens"])]


# ------------------------------------------------------------------ random small cases

GRID = [
    # B, K, V, dtype, T, top_p, draft noise
    (3, 4, 1, torch.float32, 1.0, 1.0, 0.5),
    (4, 3, 7, torch.float32, 0.7, 1.0, 0.5),
    (5, 4, 1024, torch.float32, 1.0, 1.0, 0.5),
    (4, 5, 16384 * 2 + 37, torch.bfloat16, 1.0, 1.0, 1.0),
    (4, 5, 16384 * 2 + 37, torch.bfloat16, 0.7, 0.9, 0.5),
    (3, 6, 50001, torch.bfloat16, 1.0, 0.5, 2.0),
    (3, 4, 40000, torch.float32, 1.3, 0.95, 1.0),
    (4, 4, 20000, torch.bfloat16, 0.0, 0.9, 0.5),
    (2, 64, 3000, torch.bfloat16, 1.0, 1.0, 0.05),
    (1, 1, 151936, torch.bfloat16, 1.0, 0.95, 1.0),
]


def _linear_inputs(B, K, V, dtype, T, top_p, noise, seed, neg_inf_frac=0.0):
    g = torch.Generator().manual_seed(seed)
    tgt = _rand_logits(g, (B, K + 1, V), torch.float32, 2.0, neg_inf_frac)
    drf = (tgt[:, :K].float() + torch.randn((B, K, V), generator=g) * noise).to(dtype)
    tgt = tgt.to(dtype)
    ud, ua, ur = synth.uniforms((B, K), seed + 1), synth.uniforms((B, K), seed + 2), synth.uniforms((B, K + 1), seed + 3)
    Ts, Ps = torch.full((B,), T), torch.full((B,), top_p)
    return tgt, drf, ud, ua, ur, Ts, Ps


@pytest.mark.parametrize("B,K,V,dtype,T,top_p,noise", GRID)
def test_sample_draft_parity(B, K, V, dtype, T, top_p, noise):
    tgt, drf, ud, ua, ur, Ts, Ps = _linear_inputs(B, K, V, dtype, T, top_p, noise, seed=V + K)
    tok, q, _ = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud))
    ora = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1), row_req=np.arange(B * K) // K)
    check_sample(tok, q, ora, drf.reshape(B * K, V), Ts, Ps, ud, np.arange(B * K) // K,
                 label="sample %s" % ((B, K, V, T, top_p),))


def _decode_stats(rec):
    """Host view of [rows, 32] uint8 row-statistics records: m, c, s, s_kept (fp32), tau (u32),
    amax, status (int32)."""
    r = np.ascontiguousarray(rec.reshape(-1, 32).cpu().numpy())
    f, u, i = r.view(np.float32), r.view(np.uint32), r.view(np.int32)
    return {"m": f[:, 0], "c": f[:, 1], "s": f[:, 2], "s_kept": f[:, 3], "tau": u[:, 4], "amax": i[:, 5],
            "status": i[:, 6]}


def _fkey(x):
    """Order-preserving uint32 key of fp32 values (the threshold record's encoding)."""
    u = np.asarray(x, np.float32).view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


@pytest.mark.parametrize("B,K,V,dtype,T,top_p", [(3, 4, 40000, torch.bfloat16, 1.0, 1.0),
                                                 (3, 4, 40000, torch.bfloat16, 0.7, 0.9),
                                                 (2, 5, 16384 * 2 + 37, torch.float32, 1.3, 0.5),
                                                 (4, 3, 3001, torch.float32, 0.0, 1.0)])
def test_row_stats_parity(B, K, V, dtype, T, top_p):
    """psispec_row_stats records against the oracle's row distributions: the probability every
    record implies for every token (kept set from the threshold key) within 1e-5, the greedy
    argmax exactly, data errors flagged; and the records serve verification."""
    tgt, drf, ud, ua, ur, Ts, Ps = _linear_inputs(B, K, V, dtype, T, top_p, 0.6, seed=V + 11, neg_inf_frac=0.05)
    drf[1, 2, 9] = float("nan")  # one row with a data error
    rec = psispec.row_stats(_cuda(drf), _cuda(Ts), _cuda(Ps))
    st = _decode_stats(rec)
    rows = drf.reshape(B * K, V).float().numpy().astype(np.float64)
    for r in range(B * K):
        if r == 1 * K + 2:
            assert st["status"][r] != 0
            continue
        assert st["status"][r] == 0
        probs, band = oracle.row_dist(rows[r], T, top_p)
        if T == 0.0:
            assert st["amax"][r] == int(np.argmax(rows[r]))
            continue
        if band < 1e-6:
            continue  # a threshold tie within the band: the kept set is not unique
        l = rows[r].astype(np.float32)
        kept = (_fkey(l) >= st["tau"][r]) if st["tau"][r] != 0 else np.ones(V, bool)
        p = np.where(kept, np.exp2((l.astype(np.float64) - st["m"][r]) * st["c"][r]) / st["s_kept"][r], 0.0)
        assert np.abs(p - probs).max() <= 1e-5, (r, np.abs(p - probs).max())
    # the records stand in for the draft statistics of verification
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1),
                              row_req=np.arange(B * K) // K)
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    x[x < 0] = 0
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                                draft_row_stats=rec)
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy())
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, label="row-stats records %s" % ((B, K, V, T, top_p),))


@pytest.mark.parametrize("use_stats", [False, True])
@pytest.mark.parametrize("B,K,V,dtype,T,top_p,noise", GRID)
def test_verify_linear_parity(B, K, V, dtype, T, top_p, noise, use_stats):
    tgt, drf, ud, ua, ur, Ts, Ps = _linear_inputs(B, K, V, dtype, T, top_p, noise, seed=V + 3 * K)
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1), row_req=np.arange(B * K) // K)
    x = torch.from_numpy(o_s["tokens"].reshape(B, K).astype(np.int32))
    stats = None
    if use_stats:
        _, _, stats = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud))
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                                draft_row_stats=stats)
    ora = oracle.verify_linear(tgt, drf, x.numpy(), ua, ur, Ts.numpy(), Ps.numpy())
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, label="verify %s" % ((B, K, V, T, top_p, use_stats),))


def test_verify_linear_mixed_requests_and_data_errors():
    """Per-request temperature/top-p, -inf logits, and data errors confined to their request."""
    B, K, V = 8, 5, 9000
    tgt, drf, ud, ua, ur, _, _ = _linear_inputs(B, K, V, torch.bfloat16, 1.0, 1.0, 0.7, seed=77, neg_inf_frac=0.2)
    Ts = torch.tensor([1.0, 0.0, 0.5, 2.0, 1.0, 1.0, 0.8, 1.0])
    Ps = torch.tensor([1.0, 0.9, 0.8, 0.3, 1.0, 0.99, 1.0, 1e-6])
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1), row_req=np.arange(B * K) // K)
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    x[4, 2] = V  # out-of-range token: request 4 is a data error
    tgt[5, 3, 17] = float("nan")  # NaN logit: request 5 is a data error
    drf[6, 1, :] = -float("inf")  # draft row without a finite logit: request 6
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps))
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy())
    assert ora["accept_len"][4] == ora["accept_len"][5] == ora["accept_len"][6] == -1
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, label="mixed requests")


@pytest.mark.parametrize("V,T,top_p", [(40000, 100.0, 0.9), (40000, 30.0, 0.5), ((1 << 19) + 1000, 1.0, 0.9)])
def test_topp_fallback_paths(V, T, top_p):
    """bf16 top-p rows whose threshold lies below the 2048-value window under the row maximum
    (a far outlier and a high temperature put most of the mass far below it), and rows longer
    than the top-p counters' range (2^19): the histogram / digit select and the general radix
    select and block draw, for sampling and verification."""
    B, K = 2, 3
    g = torch.Generator().manual_seed(V + int(T))
    tgt = torch.randn((B, K + 1, V), generator=g) * 2.0
    drf = tgt[:, :K] + torch.randn((B, K, V), generator=g) * 0.5
    if T > 1.0:
        tgt[..., 7] = 120.0  # an outlier far above the rest: the window covers only [~0.002, 120]
        drf[..., 7] = 120.0
    tgt, drf = tgt.to(torch.bfloat16), drf.to(torch.bfloat16)
    Ts, Ps = torch.full((B,), T), torch.full((B,), top_p)
    ud, ua, ur = synth.uniforms((B, K), 5), synth.uniforms((B, K), 6), synth.uniforms((B, K + 1), 7)
    tok, q, _ = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud))
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1),
                              row_req=np.arange(B * K) // K)
    check_sample(tok, q, o_s, drf.reshape(B * K, V), Ts, Ps, ud, np.arange(B * K) // K,
                 label="fallback sample %s" % ((V, T, top_p),))
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps))
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy())
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, label="fallback verify %s" % ((V, T, top_p),))


TOPK_GRID = [
    # B, K, V, dtype, T, top_p, top_k
    (3, 4, 40000, torch.bfloat16, 1.0, 1.0, 50),       # value window, top-k alone
    (3, 4, 50001, torch.bfloat16, 0.7, 0.9, 200),      # value window, top-k then top-p
    (3, 4, 40000, torch.bfloat16, 1.0, 0.95, 30000),   # k-th value below the window: radix select
    (3, 4, 40000, torch.float32, 1.3, 0.8, 1000),      # fp32: radix select, count then mass
    (2, 3, 40000, torch.float32, 1.0, 1.0, 1),         # k = 1 (the maximum and its ties)
    (4, 3, 7, torch.float32, 1.0, 0.9, 3),
    (1, 2, 151936, torch.bfloat16, 1.0, 0.95, 20),
]


@pytest.mark.parametrize("use_stats", [False, True])
@pytest.mark.parametrize("B,K,V,dtype,T,top_p,top_k", TOPK_GRID)
def test_topk_parity(B, K, V, dtype, T, top_p, top_k, use_stats):
    """Top-k (then top-p) in sampling and in verification against the oracle's reading: the
    value-window select (bf16), the general radix select (fp32, or a k-th value below the
    window), ties at the k-th value (bf16 rows hold many equal values), and the sampler's
    records reused by verification."""
    tgt, drf, ud, ua, ur, Ts, Ps = _linear_inputs(B, K, V, dtype, T, top_p, 0.6, seed=V + top_k)
    Ks = torch.full((B,), top_k, dtype=torch.int32)
    tok, q, rec = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud), top_k=_cuda(Ks))
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1),
                              row_req=np.arange(B * K) // K, top_k=Ks.numpy())
    check_sample(tok, q, o_s, drf.reshape(B * K, V), Ts, Ps, ud, np.arange(B * K) // K, Ks,
                 label="top-k sample %s" % ((B, K, V, T, top_p, top_k),))
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                                top_k=_cuda(Ks), draft_row_stats=rec if use_stats else None)
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy(), top_k=Ks.numpy())
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, Ks, label="top-k verify %s" % ((B, K, V, T, top_p, top_k),))


def test_q_equals_p_accepts_all_on_gpu():
    B, K, V = 16, 8, 30000
    g = torch.Generator().manual_seed(5)
    tgt = _rand_logits(g, (B, K + 1, V), torch.bfloat16)
    drf = tgt[:, :K].clone()
    x = torch.randint(0, V, (B, K), generator=g, dtype=torch.int32)
    ua = synth.uniforms((B, K), 9)
    ur = synth.uniforms((B, K + 1), 10)
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(torch.ones(B)),
                                _cuda(torch.ones(B)))
    assert (out["accept_len"] == K).all()
    assert torch.equal(out["p"], out["q"])  # the p and q pipelines are bit-identical


def _tree_inputs(B, nodes, V, dtype, T, top_p, seed):
    trie = synth.trie_topology(B, nodes, 6, 3, seed)
    g = torch.Generator().manual_seed(seed)
    tgt = _rand_logits(g, (trie.N, V), torch.float32, 2.0)
    drf = (tgt + torch.randn((trie.N, V), generator=g) * 0.7).to(dtype)
    tgt = tgt.to(dtype)
    toks = torch.zeros(trie.N, dtype=torch.int32)
    for n in range(trie.N):
        if trie.children[n]:
            picks = synth.gumbel_tokens(drf[n:n + 1], max(T, 1e-3), seed + n, k=len(trie.children[n]))[0]
            for k, c in enumerate(trie.children[n]):
                toks[c] = int(picks[k])
    ua, ur = synth.uniforms((trie.N,), seed + 1), synth.uniforms((trie.N,), seed + 2)
    return trie, tgt, drf, toks, ua, ur


@pytest.mark.parametrize("V,dtype,T,top_p", [(5, torch.float32, 1.0, 1.0), (1000, torch.float32, 0.8, 0.9),
                                             (20000, torch.bfloat16, 1.0, 1.0), (33000, torch.bfloat16, 0.7, 0.8),
                                             (4000, torch.bfloat16, 0.0, 1.0)])
def test_verify_tree_parity(V, dtype, T, top_p):
    B, nodes = 6, 24
    trie, tgt, drf, toks, ua, ur = _tree_inputs(B, nodes, V, dtype, T, top_p, seed=V)
    Ts, Ps = torch.full((B,), T), torch.full((B,), top_p)
    out = psispec.verify_tree(_cuda(tgt), _cuda(drf), _cuda(trie.node_offsets), _cuda(trie.parent), _cuda(toks),
                              _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps), 6)
    ora = oracle.verify_tree(tgt, drf, trie.node_offsets.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur,
                             Ts.numpy(), Ps.numpy(), 6)
    check_tree(out, ora, tgt, drf, trie.node_offsets, trie.parent, toks, ua, ur, Ts, Ps, 6,
               label="tree %s" % ((V, T, top_p),))


@pytest.mark.parametrize("V,dtype", [(20011, torch.bfloat16), (3001, torch.float32), (151936, torch.bfloat16)])
def test_verify_tree_mixed_requests_and_data_errors(V, dtype):
    """Per-trie temperature/top-p (uncut tries take the walk's own row maxima), -inf logits,
    unaligned rows (odd V), and data errors confined to their trie."""
    B, nodes = 8, 24
    trie = synth.trie_topology(B, nodes, 6, 3, 91)
    g = torch.Generator().manual_seed(91)
    tgt = _rand_logits(g, (trie.N, V), torch.float32, 2.0, neg_inf_frac=0.1)
    drf = tgt + torch.randn((trie.N, V), generator=g) * 0.7
    Ts = torch.tensor([1.0, 0.8, 0.0, 1.0, 1.0, 1.0, 0.9, 1.2])
    Ps = torch.tensor([1.0, 1.0, 1.0, 0.9, 1.0, 1.0, 0.95, 1.0])
    off = trie.node_offsets
    tgt[int(off[4]), 5] = float("nan")  # visited root row with a NaN: trie 4 is a data error
    drf[int(off[5]), 7] = float("inf")  # root draft row with +inf (the root has children): trie 5
    tgt[int(off[6]), :] = -float("inf")  # root target row without a finite logit: trie 6
    tgt[int(off[7 + 1]) - 1, 3] = float("nan")  # a late node of trie 7: an error only if visited
    tgt, drf = tgt.to(dtype), drf.to(dtype)
    toks = torch.zeros(trie.N, dtype=torch.int32)
    for n in range(trie.N):
        if trie.children[n]:
            picks = synth.gumbel_tokens(drf[n:n + 1].float().nan_to_num(0.0, 0.0), 1.0, 91 + n,
                                        k=len(trie.children[n]))[0]
            for k, c in enumerate(trie.children[n]):
                toks[c] = int(picks[k])
    ua, ur = synth.uniforms((trie.N,), 92), synth.uniforms((trie.N,), 93)
    out = psispec.verify_tree(_cuda(tgt), _cuda(drf), _cuda(off), _cuda(trie.parent), _cuda(toks), _cuda(ua),
                              _cuda(ur), _cuda(Ts), _cuda(Ps), 6)
    ora = oracle.verify_tree(tgt, drf, off.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur, Ts.numpy(),
                             Ps.numpy(), 6)
    assert ora["accept_len"][4] == ora["accept_len"][5] == ora["accept_len"][6] == -1
    assert (ora["accept_len"][[0, 1, 2, 3]] >= 0).all()
    check_tree(out, ora, tgt, drf, off, trie.parent, toks, ua, ur, Ts, Ps, 6, label="mixed tries V=%d" % V)


def test_verify_tree_structure_errors():
    """Malformed tries are data errors confined to their request: a parent that is not
    earlier, a token outside [0, V), a path deeper than max_depth, a root with a parent, an
    empty request; the well-formed tries around them (one greedy) match the oracle. A node with
    more than 64 children exceeds the walk's documented limit and is a data error there."""
    V, D = 3000, 6
    rng = np.random.default_rng(5)
    parents, toks = [], []

    def add(par, tk):
        parents.append(np.asarray(par, np.int32))
        toks.append(np.asarray(tk, np.int32))

    def good(n):
        par = [-1] + [int(rng.integers(0, i)) for i in range(1, n)]
        depth = [0] * n
        for i in range(1, n):  # keep the path length within D
            if depth[par[i]] >= D:
                par[i] = 0
            depth[i] = depth[par[i]] + 1
        return par, rng.choice(V, n, replace=False)

    add(*good(16))                                        # 0: well formed
    p1, t1 = good(12); p1[3] = 5; add(p1, t1)              # 1: parent after the node
    p2, t2 = good(12); t2[2] = V; add(p2, t2)              # 2: token out of range
    add(list(range(-1, 8)), rng.choice(V, 9, replace=False))  # 3: a chain of depth 8 > D
    p4, t4 = good(10); p4[0] = 0; add(p4, t4)              # 4: the root has a parent
    add([-1] + [0] * 70, rng.choice(V, 71, replace=False))   # 5: 70 children under the root
    add([], [])                                           # 6: an empty request
    add(*good(14))                                        # 7: well formed, greedy
    B = len(parents)
    offs = np.concatenate([[0], np.cumsum([len(x) for x in parents])]).astype(np.int32)
    parent, tokens = np.concatenate(parents), np.concatenate(toks)
    N = int(offs[-1])
    g = torch.Generator().manual_seed(17)
    tgt = _rand_logits(g, (N, V), torch.float32, 2.0)
    drf = tgt + torch.randn((N, V), generator=g) * 0.5
    Ts = torch.tensor([1.0] * (B - 1) + [0.0])
    Ps = torch.ones(B)
    ua, ur = synth.uniforms((N,), 18), synth.uniforms((N,), 19)
    out = psispec.verify_tree(_cuda(tgt), _cuda(drf), _cuda(offs), _cuda(parent), _cuda(tokens), _cuda(ua),
                              _cuda(ur), _cuda(Ts), _cuda(Ps), D)
    ora = oracle.verify_tree(tgt, drf, offs, parent, tokens, ua, ur, Ts.numpy(), Ps.numpy(), D)
    g_len = out["accept_len"].cpu().numpy()
    assert (g_len[[1, 2, 3, 4, 5, 6]] == -1).all(), g_len
    assert (ora["accept_len"][[1, 2, 3, 4, 6]] == -1).all(), ora["accept_len"]
    assert (g_len[[0, 7]] >= 0).all()
    keep = [0, 1, 2, 3, 4, 6, 7]  # request 5 is beyond the walk's limit only
    rep = compare_tree({k: v[keep] for k, v in out.items()}, {k: np.asarray(v)[keep] for k, v in ora.items()},
                       label="malformed tries")
    assert rep["differ_in_band"] == 0


def test_branching_one_tree_equals_linear_gpu():
    B, K, V = 6, 5, 12000
    tgt, drf, ud, ua, ur, Ts, Ps = _linear_inputs(B, K, V, torch.bfloat16, 0.9, 0.95, 0.6, seed=31)
    x, _, _ = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud))
    lin = psispec.verify_linear(_cuda(tgt), _cuda(drf), x, _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps))
    N = B * (K + 1)
    d_rows = torch.cat([drf, torch.zeros((B, 1, V), dtype=drf.dtype)], dim=1).reshape(N, V)
    parent = torch.arange(-1, K, dtype=torch.int32).repeat(B)
    tok = torch.zeros((B, K + 1), dtype=torch.int32)
    tok[:, 1:] = x.cpu()
    uacc = torch.zeros((B, K + 1))
    uacc[:, 1:] = ua
    tr = psispec.verify_tree(_cuda(tgt.reshape(N, V)), _cuda(d_rows), _cuda(torch.arange(0, N + 1, K + 1, dtype=torch.int32)),
                             _cuda(parent), _cuda(tok.reshape(-1)), _cuda(uacc.reshape(-1)), _cuda(ur.reshape(-1)),
                             _cuda(Ts), _cuda(Ps), K)
    assert torch.equal(lin["accept_len"], tr["accept_len"])
    assert torch.equal(lin["tokens"], tr["tokens"])


# ------------------------------------------------------------------ full-size workloads


def _sampled(B, n):
    return np.unique(np.linspace(0, B - 1, n).astype(int))


@pytest.mark.parametrize("name", ["mid", "max", "sweep_b32_t0", "sweep_b32_t0.7", "sweep_b32_t1", "sweep_b1_t0",
                                  "sweep_b1_t0.7", "sweep_b1_t1", "sweep_b256_t0", "sweep_b256_t0.7", "sweep_b256_t1",
                                  "mid_topk"])
def test_full_size_linear_sampled(name):
    case = synth.linear_cases()[name]
    B, K, V = case.B, case.K, case.V
    tgt, drf = synth.linear_logits(case, device=DEV)
    ud, ua, ur = synth.linear_uniforms(case)
    Ts, Ps = torch.full((B,), case.temperature), torch.full((B,), case.top_p)
    Ks = torch.full((B,), case.top_k, dtype=torch.int32) if case.top_k else None
    Kd = _cuda(Ks) if case.top_k else None
    x, q, stats = psispec.sample_draft(drf, _cuda(Ts), _cuda(Ps), _cuda(ud), top_k=Kd)
    pick = _sampled(B, 4 if B >= 256 else 6)
    idx = torch.as_tensor(pick, device=DEV)
    d_host = drf[idx].cpu()
    Kp = Ks[pick].numpy() if case.top_k else None
    o_s = oracle.sample_draft(d_host.reshape(-1, V), Ts[pick].numpy(), Ps[pick].numpy(), ud[pick].reshape(-1),
                              row_req=np.arange(len(pick) * K) // K, top_k=Kp)
    rows_req = np.arange(len(pick) * K) // K
    check_sample(x[idx], q[idx], o_s, d_host.reshape(-1, V), Ts[pick], Ps[pick], ud[pick], rows_req, Kp,
                 label="full-size sample %s" % name)
    # the oracle's draft tokens replace the sampled requests' rows
    x_in = x.clone()
    x_in[idx] = torch.from_numpy(o_s["tokens"].reshape(len(pick), K)).to(DEV)
    out = psispec.verify_linear(tgt, drf, x_in, _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps), top_k=Kd,
                                draft_row_stats=stats)
    ora = oracle.verify_linear(tgt[idx].cpu(), d_host, o_s["tokens"].reshape(len(pick), K), ua[pick], ur[pick],
                               Ts[pick].numpy(), Ps[pick].numpy(), top_k=Kp)
    sub = {k: v[idx] for k, v in out.items()}
    stats_report = check_linear(sub, ora, tgt[idx].cpu(), d_host, o_s["tokens"].reshape(len(pick), K), ua[pick],
                                ur[pick], Ts[pick], Ps[pick], Kp, label="full-size verify %s" % name)
    lens = out["accept_len"].cpu().numpy()
    assert (lens >= 0).all() and (lens <= K).all()
    print(name, stats_report, "gpu mean accept", lens.mean())


@pytest.mark.parametrize("name", ["tree", "tree_deep"])
def test_full_size_tree(name):
    case = synth.tree_cases()[name]
    trie, tgt, drf, toks, ua, ur = synth.tree_inputs(case, device=DEV)
    B = case.B
    Ts, Ps = torch.full((B,), case.temperature), torch.full((B,), case.top_p)
    out = psispec.verify_tree(tgt, drf, _cuda(trie.node_offsets), _cuda(trie.parent), _cuda(toks), _cuda(ua), _cuda(ur),
                              _cuda(Ts), _cuda(Ps), case.max_depth)
    ora = oracle.verify_tree(tgt.cpu(), drf.cpu(), trie.node_offsets.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur,
                             Ts.numpy(), Ps.numpy(), case.max_depth)
    rep = check_tree(out, ora, tgt.cpu(), drf.cpu(), trie.node_offsets, trie.parent, toks, ua, ur, Ts, Ps,
                     case.max_depth, label="full-size tree")
    print(name, rep, "accept", out["accept_len"].tolist())
    if name == "tree_deep":  # q == p: every first child is accepted down to a leaf
        assert (out["accept_len"].cpu() >= 1).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_tree_walk_single_cta_fallback(dtype):
    """V too large for the cluster walk's shared-memory slices (16 or 8 CTAs): the walk runs
    one CTA per trie (tree_walk_kernel) on the statistics pass's records."""
    B, nodes, V = 2, 8, 500_000
    trie, tgt, drf, toks, ua, ur = _tree_inputs(B, nodes, V, dtype, 1.0, 1.0, seed=77)
    for T, P in ((1.0, 1.0), (0.8, 0.9)):
        Ts, Ps = torch.full((B,), T), torch.full((B,), P)
        out = psispec.verify_tree(_cuda(tgt), _cuda(drf), _cuda(trie.node_offsets), _cuda(trie.parent), _cuda(toks),
                                  _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps), 6)
        ora = oracle.verify_tree(tgt, drf, trie.node_offsets.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur,
                                 Ts.numpy(), Ps.numpy(), 6)
        check_tree(out, ora, tgt, drf, trie.node_offsets, trie.parent, toks, ua, ur, Ts, Ps, 6,
                   label="single-CTA walk V=%d %s T=%g P=%g" % (V, dtype, T, P))


# ------------------------------------------------------------------ top-k: mixed requests and negative rows


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_topk_mixed_requests(dtype):
    """Per-request top-k, off by k <= 0 and k >= V, beside greedy rows, top-p alone and both."""
    B, K, V = 8, 4, 20011
    tgt, drf, ud, ua, ur, _, _ = _linear_inputs(B, K, V, dtype, 1.0, 1.0, 0.7, seed=91, neg_inf_frac=0.1)
    Ts = torch.tensor([1.0, 0.0, 0.8, 1.0, 1.5, 1.0, 0.7, 1.0])
    Ps = torch.tensor([1.0, 1.0, 0.9, 0.5, 1.0, 1.0, 0.95, 0.9])
    Ks = torch.tensor([0, 5, 100, 7, V, V - 1, -3, 2500], dtype=torch.int32)
    tok, q, _ = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud), top_k=_cuda(Ks))
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1),
                              row_req=np.arange(B * K) // K, top_k=Ks.numpy())
    check_sample(tok, q, o_s, drf.reshape(B * K, V), Ts, Ps, ud, np.arange(B * K) // K, Ks,
                 label="top-k mixed sample %s" % dtype)
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                                top_k=_cuda(Ks))
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy(), top_k=Ks.numpy())
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, Ks, label="top-k mixed verify %s" % dtype)
    # a null top-k array and an all-off one agree with the entry points without top-k
    off = torch.zeros(B, dtype=torch.int32)
    a = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                              top_k=_cuda(off))
    b = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps))
    assert torch.equal(a["tokens"], b["tokens"]) and torch.equal(a["accept_len"], b["accept_len"])
    assert torch.equal(a["p"], b["p"]) and torch.equal(a["q"], b["q"])


@pytest.mark.parametrize("top_p,top_k", [(0.9, 0), (1.0, 100), (0.8, 500)])
def test_negative_logit_rows(top_p, top_k):
    """bf16 rows of log-probabilities (every logit negative): the top-p/top-k value window then
    lies among negative values, whose weights come from the inverse of their 16-bit order keys."""
    B, K, V = 3, 4, 40000
    tgt, drf, ud, ua, ur, Ts, Ps = _linear_inputs(B, K, V, torch.float32, 1.0, top_p, 0.6, seed=404 + top_k)
    tgt = torch.log_softmax(tgt, dim=-1).to(torch.bfloat16)
    drf = torch.log_softmax(drf, dim=-1).to(torch.bfloat16)
    Ks = torch.full((B,), top_k, dtype=torch.int32)
    tok, q, _ = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud), top_k=_cuda(Ks))
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1),
                              row_req=np.arange(B * K) // K, top_k=Ks.numpy())
    check_sample(tok, q, o_s, drf.reshape(B * K, V), Ts, Ps, ud, np.arange(B * K) // K, Ks,
                 label="negative rows sample %s" % ((top_p, top_k),))
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                                top_k=_cuda(Ks))
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy(), top_k=Ks.numpy())
    check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, Ks, label="negative rows verify %s" % ((top_p, top_k),))


# ------------------------------------------------------------------ top-k: tree and row statistics


@pytest.mark.parametrize("V,dtype,T,top_p", [(1000, torch.float32, 0.8, 1.0), (20011, torch.bfloat16, 1.0, 0.9),
                                             (151936, torch.bfloat16, 1.0, 0.95)])
def test_verify_tree_topk_parity(V, dtype, T, top_p):
    """Per-request top-k in tree verification (off, k = 1, small and large k, k >= V)."""
    B, nodes = 6, 24
    trie, tgt, drf, toks, ua, ur = _tree_inputs(B, nodes, V, dtype, T, top_p, seed=V + 5)
    Ts, Ps = torch.full((B,), T), torch.full((B,), top_p)
    Ks = torch.tensor([5, 0, 100, V - 1, 1, V], dtype=torch.int32)
    out = psispec.verify_tree(_cuda(tgt), _cuda(drf), _cuda(trie.node_offsets), _cuda(trie.parent), _cuda(toks),
                              _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps), 6, top_k=_cuda(Ks))
    ora = oracle.verify_tree(tgt, drf, trie.node_offsets.numpy(), trie.parent.numpy(), toks.numpy(), ua, ur,
                             Ts.numpy(), Ps.numpy(), 6, top_k=Ks.numpy())
    check_tree(out, ora, tgt, drf, trie.node_offsets, trie.parent, toks, ua, ur, Ts, Ps, 6, Ks,
               label="top-k tree %s" % ((V, T, top_p),))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_row_stats_topk_parity(dtype):
    """psispec_row_stats_k records: the probability each record implies for every token within
    1e-5 of the oracle's top-k (then top-p) distribution."""
    B, K, V = 4, 3, 30011
    tgt, drf, ud, ua, ur, _, _ = _linear_inputs(B, K, V, dtype, 1.0, 1.0, 0.6, seed=313, neg_inf_frac=0.05)
    Ts = torch.tensor([1.0, 0.7, 1.3, 1.0])
    Ps = torch.tensor([1.0, 0.9, 0.8, 1.0])
    Ks = torch.tensor([40, 300, 5000, 0], dtype=torch.int32)
    rec = psispec.row_stats(_cuda(drf), _cuda(Ts), _cuda(Ps), top_k=_cuda(Ks))
    st = _decode_stats(rec)
    rows = drf.reshape(B * K, V).float().numpy().astype(np.float64)
    for r in range(B * K):
        b = r // K
        assert st["status"][r] == 0
        probs, band = oracle.row_dist(rows[r], float(Ts[b]), float(Ps[b]), int(Ks[b]))
        if band < 1e-6:
            continue  # a threshold tie within the band: the kept set is not unique
        l = rows[r].astype(np.float32)
        kept = (_fkey(l) >= st["tau"][r]) if st["tau"][r] != 0 else np.ones(V, bool)
        p = np.where(kept, np.exp2((l.astype(np.float64) - st["m"][r]) * st["c"][r]) / st["s_kept"][r], 0.0)
        assert np.abs(p - probs).max() <= 1e-5, (r, np.abs(p - probs).max())


# ------------------------------------------------------------------ one-pass cut rows: edge rows


def _edge_rows(V, n_rows, g):
    """bf16 draft-like rows that stress the one-pass cut path: the row maximum arriving last
    (far above, and just above, what the first values set), spikes in several warps' ranges,
    rows of huge negative logits (the window reaches the keys of -inf) and of huge positive ones,
    a row of -inf with one finite value, a NaN row, and a row whose first half is -inf."""
    x = torch.randn((n_rows, V), generator=g) * 2.0
    x[0, V - 3] = 60.0                    # the maximum last, many binades above the rest
    x[1, V - 1] = 9.0                     # just above the usual maximum, at the very end
    x[2, ::V // 7 + 1] = torch.linspace(5.0, 40.0, len(range(0, V, V // 7 + 1)))  # rising spikes
    x[3] = -3.0e38 + x[3].abs() * 1.0e36  # huge negative logits
    x[4] = -float("inf")
    x[4, V // 2] = 1.0                    # one finite value
    x[5, min(17, V - 1)] = float("nan")   # a data error
    x[6, :V // 2] = -float("inf")         # the first half -inf: the first warps see no finite value
    x[7] = 3.0e38 - x[7].abs() * 1.0e36   # huge positive logits (their products with log2(e)/T overflow)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("V", [7, 300, 16384 * 2 + 37, 151936])
@pytest.mark.parametrize("top_p,top_k", [(0.9, 0), (1.0, 40), (0.95, 500)])
def test_cut_rows_edge_rows(V, top_p, top_k):
    """The one-pass cut-row path on edge rows, for sampling, verification (streaming the draft
    rows, and reusing the sampler's records) and row statistics, against the oracle."""
    B, K = 4, 2
    g = torch.Generator().manual_seed(V + 7 * top_k)
    drf = _edge_rows(V, B * K, g).reshape(B, K, V)
    tgt = torch.cat([_edge_rows(V, B * K, g).reshape(B, K, V)[:, torch.randperm(K, generator=g)],
                     (torch.randn((B, 1, V), generator=g) * 2.0).to(torch.bfloat16)], dim=1)
    Ts = torch.tensor([1.0, 0.7, 1.3, 1.0])
    Ps = torch.full((B,), top_p)
    Ks = torch.full((B,), top_k, dtype=torch.int32) if top_k else None
    Kd = _cuda(Ks) if top_k else None
    ud, ua, ur = synth.uniforms((B, K), V + 1), synth.uniforms((B, K), V + 2), synth.uniforms((B, K + 1), V + 3)
    tok, q, rec = psispec.sample_draft(_cuda(drf), _cuda(Ts), _cuda(Ps), _cuda(ud), top_k=Kd)
    rr = np.arange(B * K) // K
    o_s = oracle.sample_draft(drf.reshape(B * K, V), Ts.numpy(), Ps.numpy(), ud.reshape(-1), row_req=rr,
                              top_k=None if Ks is None else Ks.numpy())
    assert (o_s["tokens"].reshape(B, K)[:, :] >= -1).all()
    check_sample(tok, q, o_s, drf.reshape(B * K, V), Ts, Ps, ud, rr, Ks, label="edge rows sample V=%d" % V)
    x = o_s["tokens"].reshape(B, K).astype(np.int32)
    x[x < 0] = 0
    ora = oracle.verify_linear(tgt, drf, x, ua, ur, Ts.numpy(), Ps.numpy(), top_k=None if Ks is None else Ks.numpy())
    for stats in (None, rec):
        out = psispec.verify_linear(_cuda(tgt), _cuda(drf), _cuda(x), _cuda(ua), _cuda(ur), _cuda(Ts), _cuda(Ps),
                                    top_k=Kd, draft_row_stats=stats)
        check_linear(out, ora, tgt, drf, x, ua, ur, Ts, Ps, Ks, label="edge rows verify V=%d" % V)
    # the records the statistics entry writes imply the oracle's distributions
    recs = _decode_stats(psispec.row_stats(_cuda(drf), _cuda(Ts), _cuda(Ps), top_k=Kd))
    rows = drf.reshape(B * K, V).float().numpy().astype(np.float64)
    for r in range(B * K):
        b = r // K
        probs, band = oracle.row_dist(rows[r], float(Ts[b]), float(Ps[b]), top_k)
        if probs is None:
            assert recs["status"][r] != 0, r
            continue
        assert recs["status"][r] == 0, r
        if band < 1e-6:
            continue
        l = rows[r].astype(np.float32)
        kept = (_fkey(l) >= recs["tau"][r]) if recs["tau"][r] != 0 else np.ones(V, bool)
        p = np.where(kept, np.exp2((l.astype(np.float64) - recs["m"][r]) * recs["c"][r]) / recs["s_kept"][r], 0.0)
        assert np.abs(p - probs).max() <= 1e-5, (r, np.abs(p - probs).max())
