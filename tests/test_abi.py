"""The C ABI library loads and exports every declared entry point; host-side argument checks
return their status codes before anything reaches a GPU (no device needed)."""
import ctypes

import pytest

from lossless_speculative_sampling_b200 import build as libbuild
from lossless_speculative_sampling_b200 import psispec


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return psispec.lib()


def test_exports_every_declared_symbol(L):
    names = psispec.declared_symbols()
    assert {"psispec_sample_draft", "psispec_verify_linear", "psispec_verify_tree", "psispec_workspace_size",
            "psispec_status_string", "psispec_version"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    for s in range(5):
        assert psispec.status_string(s) and psispec.status_string(s) != "unknown status"
    assert psispec.status_string(99) == "unknown status"
    assert L.psispec_version() >= 100


def test_workspace_size(L):
    V = 151936
    for op, a, b in ((psispec.OP_SAMPLE_DRAFT, 64, 8), (psispec.OP_VERIFY_LINEAR, 64, 8), (psispec.OP_VERIFY_TREE, 4, 256),
                     (psispec.OP_ROW_STATS, 64, 9)):
        n = psispec.workspace_size(op, a, b, V)
        assert n > 0 and n % 256 == 0
        assert psispec.workspace_size(op, a * 2, b, V) >= n
    assert psispec.workspace_size(7, 1, 1, 1) == 0
    assert psispec.workspace_size(psispec.OP_VERIFY_LINEAR, 0, 8, V) == 0
    assert psispec.workspace_size(psispec.OP_VERIFY_LINEAR, 1, 8, (1 << 24) + 1) == 0


FAKE = ctypes.c_void_p(4096)  # aligned, never dereferenced: every call below fails validation


def _sample(L, **kw):
    a = dict(d=FAKE, dtype=psispec.BF16, B=2, K=3, V=100, T=FAKE, P=FAKE, u=FAKE, tok=FAKE, q=None, st=None, ws=FAKE,
             wsb=1 << 30)
    a.update(kw)
    return L.psispec_sample_draft(a["d"], a["dtype"], a["B"], a["K"], a["V"], a["T"], a["P"], a["u"], a["tok"], a["q"],
                                  a["st"], a["ws"], a["wsb"], None)


def test_sample_draft_host_checks(L):
    assert _sample(L, d=None) == psispec.ERR_INVALID_ARG
    assert _sample(L, u=None) == psispec.ERR_INVALID_ARG
    assert _sample(L, dtype=5) == psispec.ERR_INVALID_ARG
    assert _sample(L, B=0) == psispec.ERR_INVALID_ARG
    assert _sample(L, V=-1) == psispec.ERR_INVALID_ARG
    assert _sample(L, d=ctypes.c_void_p(4097)) == psispec.ERR_INVALID_ARG  # misaligned bf16
    assert _sample(L, V=(1 << 24) + 1) == psispec.ERR_UNSUPPORTED
    assert _sample(L, ws=None) == psispec.ERR_WORKSPACE
    assert _sample(L, ws=ctypes.c_void_p(4096 + 128)) == psispec.ERR_WORKSPACE
    assert _sample(L, wsb=16) == psispec.ERR_WORKSPACE


def _row_stats(L, **kw):
    a = dict(l=FAKE, dtype=psispec.BF16, B=2, K=3, V=100, T=FAKE, P=FAKE, out=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return L.psispec_row_stats(a["l"], a["dtype"], a["B"], a["K"], a["V"], a["T"], a["P"], a["out"], a["ws"], a["wsb"],
                               None)


def test_row_stats_host_checks(L):
    assert _row_stats(L, l=None) == psispec.ERR_INVALID_ARG
    assert _row_stats(L, P=None) == psispec.ERR_INVALID_ARG
    assert _row_stats(L, out=None) == psispec.ERR_INVALID_ARG
    assert _row_stats(L, dtype=5) == psispec.ERR_INVALID_ARG
    assert _row_stats(L, K=0) == psispec.ERR_INVALID_ARG
    assert _row_stats(L, out=ctypes.c_void_p(4096 + 8)) == psispec.ERR_INVALID_ARG  # records are 16-byte aligned
    assert _row_stats(L, V=(1 << 24) + 1) == psispec.ERR_UNSUPPORTED
    assert _row_stats(L, ws=None) == psispec.ERR_WORKSPACE
    assert _row_stats(L, wsb=16) == psispec.ERR_WORKSPACE


def _linear(L, **kw):
    a = dict(t=FAKE, d=FAKE, dtype=psispec.F32, B=2, K=4, V=64, x=FAKE, st=None, ua=FAKE, ur=FAKE, T=FAKE, P=FAKE,
             ot=FAKE, ol=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return L.psispec_verify_linear(a["t"], a["d"], a["dtype"], a["B"], a["K"], a["V"], a["x"], a["st"], a["ua"],
                                   a["ur"], a["T"], a["P"], a["ot"], a["ol"], None, None, a["ws"], a["wsb"], None)


def test_verify_linear_host_checks(L):
    assert _linear(L, t=None) == psispec.ERR_INVALID_ARG
    assert _linear(L, ol=None) == psispec.ERR_INVALID_ARG
    assert _linear(L, K=0) == psispec.ERR_INVALID_ARG
    assert _linear(L, K=65) == psispec.ERR_UNSUPPORTED
    assert _linear(L, t=ctypes.c_void_p(4098)) == psispec.ERR_INVALID_ARG  # misaligned fp32
    assert _linear(L, st=ctypes.c_void_p(4100)) == psispec.ERR_INVALID_ARG  # misaligned stats
    assert _linear(L, wsb=0) == psispec.ERR_WORKSPACE


def test_topk_entries_host_checks(L):
    """The top-k entry points validate like the plain ones (the top-k array itself may be null)."""
    def sample_k(**kw):
        a = dict(d=FAKE, B=2, K=3, V=100, u=FAKE, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.psispec_sample_draft_k(a["d"], psispec.BF16, a["B"], a["K"], a["V"], FAKE, FAKE, FAKE, a["u"], FAKE,
                                        None, None, a["ws"], a["wsb"], None)

    def linear_k(**kw):
        a = dict(t=FAKE, K=4, V=64, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.psispec_verify_linear_k(a["t"], FAKE, psispec.F32, 2, a["K"], a["V"], FAKE, None, FAKE, FAKE, FAKE,
                                         FAKE, None, FAKE, FAKE, None, None, a["ws"], a["wsb"], None)

    assert sample_k(d=None) == psispec.ERR_INVALID_ARG
    assert sample_k(u=None) == psispec.ERR_INVALID_ARG
    assert sample_k(B=0) == psispec.ERR_INVALID_ARG
    assert sample_k(V=(1 << 24) + 1) == psispec.ERR_UNSUPPORTED
    assert sample_k(wsb=16) == psispec.ERR_WORKSPACE
    assert linear_k(t=None) == psispec.ERR_INVALID_ARG
    assert linear_k(K=65) == psispec.ERR_UNSUPPORTED
    assert linear_k(t=ctypes.c_void_p(4098)) == psispec.ERR_INVALID_ARG
    assert linear_k(ws=None) == psispec.ERR_WORKSPACE

    def tree_k(**kw):
        a = dict(par=FAKE, N=10, md=4, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.psispec_verify_tree_k(FAKE, FAKE, psispec.BF16, 2, a["N"], 64, FAKE, a["par"], FAKE, FAKE, FAKE, FAKE,
                                       FAKE, None, a["md"], FAKE, FAKE, FAKE, a["ws"], a["wsb"], None)

    def row_stats_k(**kw):
        a = dict(l=FAKE, out=FAKE, K=3, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.psispec_row_stats_k(a["l"], psispec.BF16, 2, a["K"], 100, FAKE, FAKE, None, a["out"], a["ws"], a["wsb"],
                                     None)

    assert tree_k(par=None) == psispec.ERR_INVALID_ARG
    assert tree_k(N=1) == psispec.ERR_INVALID_ARG
    assert tree_k(md=65) == psispec.ERR_UNSUPPORTED
    assert tree_k(ws=None) == psispec.ERR_WORKSPACE
    assert row_stats_k(l=None) == psispec.ERR_INVALID_ARG
    assert row_stats_k(K=0) == psispec.ERR_INVALID_ARG
    assert row_stats_k(out=ctypes.c_void_p(4096 + 8)) == psispec.ERR_INVALID_ARG
    assert row_stats_k(wsb=16) == psispec.ERR_WORKSPACE


def test_build_tree_host_checks(L):
    def bt(**kw):
        a = dict(d=FAKE, B=2, K=3, V=100, ck=4, n=10, par=FAKE, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.psispec_build_tree(a["d"], psispec.BF16, a["B"], a["K"], a["V"], FAKE, FAKE, None, a["ck"], a["n"],
                                    a["par"], FAKE, FAKE, None, FAKE, a["ws"], a["wsb"], None)

    assert bt(d=None) == psispec.ERR_INVALID_ARG
    assert bt(par=None) == psispec.ERR_INVALID_ARG
    assert bt(ck=0) == psispec.ERR_INVALID_ARG
    assert bt(n=0) == psispec.ERR_INVALID_ARG
    assert bt(K=17) == psispec.ERR_UNSUPPORTED
    assert bt(ck=33) == psispec.ERR_UNSUPPORTED
    assert bt(n=65) == psispec.ERR_UNSUPPORTED
    assert bt(ws=None) == psispec.ERR_WORKSPACE
    assert psispec.workspace_size(psispec.OP_BUILD_TREE, 4, 16, 151936) > 0


def _tree(L, **kw):
    a = dict(t=FAKE, d=FAKE, dtype=psispec.BF16, B=2, N=10, V=64, off=FAKE, par=FAKE, tok=FAKE, ua=FAKE, ur=FAKE,
             T=FAKE, P=FAKE, md=4, op=FAKE, ot=FAKE, ol=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return L.psispec_verify_tree(a["t"], a["d"], a["dtype"], a["B"], a["N"], a["V"], a["off"], a["par"], a["tok"],
                                 a["ua"], a["ur"], a["T"], a["P"], a["md"], a["op"], a["ot"], a["ol"], a["ws"],
                                 a["wsb"], None)


def test_verify_tree_host_checks(L):
    assert _tree(L, par=None) == psispec.ERR_INVALID_ARG
    assert _tree(L, N=1) == psispec.ERR_INVALID_ARG  # fewer nodes than requests
    assert _tree(L, md=0) == psispec.ERR_INVALID_ARG
    assert _tree(L, md=65) == psispec.ERR_UNSUPPORTED
    assert _tree(L, ws=None) == psispec.ERR_WORKSPACE


def test_binding_refuses_cpu_tensors(L):
    import torch

    x = torch.zeros(1, 2, 8)
    with pytest.raises(TypeError):
        psispec.sample_draft(x, torch.ones(1), torch.ones(1), torch.zeros(2))
