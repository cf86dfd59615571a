"""The seeded input generators (synth.py) against the recipes they state: shapes and dtypes,
determinism, the uniforms' 2^-24 grid, the linear draft-around-target structure, the peaked
candidate-trie rows, the verifier rows of a trie's nodes, and valid tree topologies. CPU only,
at reduced sizes where the recipe allows."""
import dataclasses

import numpy as np
import pytest
import torch

from lossless_speculative_sampling_b200 import synth


def test_uniforms_grid_and_determinism():
    a, b = synth.uniforms((1000,), 7), synth.uniforms((1000,), 7)
    assert torch.equal(a, b) and a.dtype == torch.float32
    k = a.double() * 2.0**24
    assert torch.equal(k, torch.round(k)) and float(a.min()) >= 0.0 and float(a.max()) < 1.0
    assert not torch.equal(a, synth.uniforms((1000,), 8))


def test_linear_logits_recipe():
    case = dataclasses.replace(synth.linear_cases()["max"], B=3, V=4096)
    tgt, drf = synth.linear_logits(case)
    assert tgt.shape == (3, case.K + 1, 4096) and drf.shape == (3, case.K, 4096)
    assert tgt.dtype == drf.dtype == torch.bfloat16
    t2, d2 = synth.linear_logits(case)
    assert torch.equal(tgt, t2) and torch.equal(drf, d2)
    # target N(0, 2^2); draft = target + per-request noise of std in [0.25, 2]
    assert abs(float(tgt.float().std()) - 2.0) < 0.1
    noise = (drf.float() - tgt[:, :case.K].float()).std(dim=(1, 2))
    assert bool(((noise > 0.2) & (noise < 2.1)).all())


def test_mid_rows_carry_the_rank_bias():
    case = dataclasses.replace(synth.linear_cases()["mid"], B=2, V=8192)
    tgt, _ = synth.linear_logits(case)
    top = tgt.float().max(dim=-1).values
    # 8 * rank^-1.1 on top of N(0, 3^2): the maxima sit well above a plain N(0, 9) row's
    assert float(top.mean()) > 11.0


def test_trie_rows_are_peaked():
    case = dataclasses.replace(synth.trie_cases()["trie_32"], B=2, K=3)
    d = synth.trie_draft(case)
    assert d.shape == (2, 3, case.V) and d.dtype == torch.bfloat16
    p = torch.softmax(d.double(), dim=-1)
    top1 = p.max(dim=-1).values
    assert bool(((top1 > 0.6) & (top1 < 0.95)).all()), top1  # about 0.8 of a row's mass
    assert torch.equal(d, synth.trie_draft(case))


def test_trie_verifier_rows_follow_the_depths():
    case = dataclasses.replace(synth.trie_cases()["trie_32"], B=2, K=3, V=2048, zipf_bias=0.0)
    d = synth.trie_draft(case)
    depth = torch.tensor([[0, 1, 2, 3, -1], [0, 1, 1, 2, 3]], dtype=torch.int32)
    rows = synth.trie_verifier_rows(case, d, depth).float().view(2, 5, case.V)
    for b in range(2):
        for n in range(5):
            dep = int(depth[b, n])
            base = d[b, dep].float() if 0 <= dep < case.K else torch.zeros(case.V)
            resid = rows[b, n] - base
            assert abs(float(resid.std()) - case.target_noise) < 0.1, (b, n)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_tree_topology_is_a_valid_trie(seed):
    t = synth.trie_topology(4, 64, 8, 4, seed)
    offs = t.node_offsets.numpy()
    par = t.parent.numpy()
    assert offs[0] == 0 and (np.diff(offs) == 64).all()
    for b in range(4):
        p = par[offs[b]:offs[b + 1]]
        assert p[0] == -1 and all(0 <= p[i] < i for i in range(1, len(p)))
        depth = [0] * len(p)
        kids = [0] * len(p)
        for i in range(1, len(p)):
            depth[i] = depth[p[i]] + 1
            kids[p[i]] += 1
        assert max(depth) <= 8 and max(kids) <= 4
