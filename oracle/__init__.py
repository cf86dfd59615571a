"""Plain fp64 CPU oracle of the Psi-Spec verification step.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / reference leg may import this package. It shares no code with the CUDA
library in ``lossless_speculative_sampling_b200`` and neither imports the other.

The arithmetic lives in ``psispec_oracle.c`` (straight fp64 loops, compiled ``-O2`` without
fast-math). This module only marshals numpy arrays into it. Source of the method:
"Unlocking Lossless Speedups in LLMs via Discrete Diffusion" (arXiv 2609.04010), long-form
review page, section 3.3 "Psi-Spec" (accept with min(1, p_AR/p_draft), longest prefix before
the first rejection, residual [p_AR - p_draft]_+ resample, bonus token on full acceptance) and
section 3.4 (linear and tree samplers).

Pins (see tests/test_oracle_*.py): closed forms on hand-made rows, q == p accepts every
position, disjoint one-hot drafts reject at position 0, temperature 0 is exact argmax
matching, exhaustive uniform grids reproduce the exact rejection-sampling law, and
Monte-Carlo chi-squared tests show the emitted tokens follow the verifier's law (linear and
tree, under each tree rule); the candidate trie equals a full enumeration of the candidate
prefixes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "psispec_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpsispec_oracle.so")
_lib = None

E_BAND = 1e-6  # decisions whose margin is below this may differ between correct implementations

# candidate rules of tree verification (psispec_oracle.h)
TREE_SAMPLED_WOR, TREE_DETERMINISTIC, TREE_SAMPLED_WR = 0, 1, 2
# kinds of decision behind a band ("band_kind" outputs): none, accept test, draw edge, top-p tail
BAND_NONE, BAND_E1, BAND_E2, BAND_E3 = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math). Returns the library path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIB points the tests' mutation check at a deliberately broken build of the
        # same source; it is never set otherwise.
        lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        D, I = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)
        lib.oracle_row_dist.argtypes = [D, ctypes.c_int, ctypes.c_double, ctypes.c_double, D, D]
        lib.oracle_row_dist_k.argtypes = [D, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int, D, D]
        lib.oracle_inverse_cdf.argtypes = [D, ctypes.c_int, ctypes.c_double, D]
        lib.oracle_sample_draft.argtypes = [D, ctypes.c_int, ctypes.c_int, I, D, D, I, D, I, D, D, I]
        lib.oracle_verify_linear.argtypes = [D, D, ctypes.c_int, ctypes.c_int, ctypes.c_int, I, D, D, D, D, I,
                                             I, I, D, D, D, D, I]
        lib.oracle_verify_tree.argtypes = [D, D, ctypes.c_int, ctypes.c_int, I, I, I, D, D, D, D, I,
                                           ctypes.c_int, I, I, I, D, I]
        lib.oracle_verify_tree_rule.argtypes = [D, D, ctypes.c_int, ctypes.c_int, I, I, I, D, D, D, D, I,
                                                ctypes.c_int, ctypes.c_int, I, I, I, D, I]
        lib.oracle_build_tree.argtypes = [D, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, I, I, I, D, I]
        _lib = lib
    return _lib


def _f64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _i32(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int32))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _as_f64(x):
    """Accept numpy arrays or torch CPU tensors (bf16/fp32 convert to fp64 exactly)."""
    if hasattr(x, "detach"):
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def row_dist(logits, temperature: float, top_p: float = 1.0, top_k: int = 0):
    """Distribution of one row after temperature, top-k (0: off) and top-p. Returns
    (probs, e3_band) or (None, inf) for a bad row."""
    l, lp = _f64(_as_f64(logits).reshape(-1))
    out, op = _f64(np.zeros_like(l))
    band, bp = _f64(np.zeros(1))
    if top_k:
        rc = _load().oracle_row_dist_k(lp, l.size, float(temperature), float(top_p), int(top_k), op, bp)
    else:
        rc = _load().oracle_row_dist(lp, l.size, float(temperature), float(top_p), op, bp)
    return (None, float("inf")) if rc != 0 else (out, float(band[0]))


def _top_k(top_k, B):
    """Per-request top-k as an int32 array and its pointer, or (None, None) when off."""
    if top_k is None:
        return None, None
    return _i32(np.broadcast_to(np.asarray(top_k, dtype=np.int32), (B,)))


def inverse_cdf(r, u: float):
    """y = min{v : C(v) > u Z} in vocabulary order. Returns (y, e2_band)."""
    r, rp = _f64(np.asarray(r).reshape(-1))
    band, bp = _f64(np.zeros(1))
    y = _load().oracle_inverse_cdf(rp, r.size, float(u), bp)
    return int(y), float(band[0])


def sample_draft(draft_logits, temperature, top_p, u, row_req=None, top_k=None):
    """draft_logits [rows, V]; temperature/top_p (and top_k, None: off) per request; u [rows];
    row_req maps rows to requests (default: row i -> request i). Returns dict(tokens, q, band,
    band_kind)."""
    d = _as_f64(draft_logits)
    rows, V = d.shape
    rr = np.arange(rows) if row_req is None else np.asarray(row_req)
    d, dp = _f64(d)
    rr, rrp = _i32(rr)
    T, Tp = _f64(np.atleast_1d(temperature))
    P, Pp = _f64(np.atleast_1d(top_p))
    u, up = _f64(_as_f64(u).reshape(-1))
    tok, tokp = _i32(np.zeros(rows))
    q, qp = _f64(np.zeros(rows))
    band, bp = _f64(np.zeros(rows))
    kind, kp = _i32(np.zeros(rows))
    Kk, Kkp = _top_k(top_k, P.size)
    _load().oracle_sample_draft(dp, rows, V, rrp, Tp, Pp, Kkp, up, tokp, qp, bp, kp)
    return {"tokens": tok, "q": q, "band": band, "band_kind": kind}


def verify_linear(target, draft, draft_tokens, u_accept, u_resid, temperature, top_p, top_k=None):
    """target [B, K+1, V], draft [B, K, V], draft_tokens [B, K], u_accept [B, K],
    u_resid [B, K+1], temperature [B], top_p [B], top_k [B] (None: off). Returns dict(tokens [B, K+1],
    accept_len [B], p [B, K], q [B, K], band [B], pq_band [B, K], band_kind [B])."""
    t = _as_f64(target)
    B, K1, V = t.shape
    K = K1 - 1
    t, tp = _f64(t)
    d, dp = _f64(_as_f64(draft).reshape(B, K, V) if K > 0 else np.zeros((B, 0, V)))
    x, xp = _i32(np.asarray(draft_tokens).reshape(B, K))
    ua, uap = _f64(_as_f64(u_accept).reshape(B, K))
    ur, urp = _f64(_as_f64(u_resid).reshape(B, K + 1))
    T, Tp = _f64(np.broadcast_to(np.asarray(temperature, dtype=np.float64), (B,)))
    P, Pp = _f64(np.broadcast_to(np.asarray(top_p, dtype=np.float64), (B,)))
    tok, tokp = _i32(np.zeros((B, K + 1)))
    ln, lnp = _i32(np.zeros(B))
    p, pp = _f64(np.zeros((B, K)))
    q, qp = _f64(np.zeros((B, K)))
    band, bp = _f64(np.zeros(B))
    pqb, pqbp = _f64(np.zeros((B, K)))
    kind, kp = _i32(np.zeros(B))
    Kk, Kkp = _top_k(top_k, B)
    _load().oracle_verify_linear(tp, dp, B, K, V, xp, uap, urp, Tp, Pp, Kkp, tokp, lnp, pp, qp, bp, pqbp, kp)
    return {"tokens": tok, "accept_len": ln, "p": p, "q": q, "band": band, "pq_band": pqb, "band_kind": kind}


def verify_tree(target, draft, node_offsets, parent, tokens, u_accept, u_resid, temperature, top_p,
                max_depth: int, top_k=None, rule: int = TREE_SAMPLED_WOR):
    """target/draft [N, V]; node_offsets [B+1]; parent/tokens/u_accept/u_resid [N] (parent is
    the request-local index, -1 at the root); rule: how the children were produced
    (TREE_SAMPLED_WOR, TREE_DETERMINISTIC, TREE_SAMPLED_WR). Returns dict(path [B, max_depth],
    tokens [B, max_depth+1], accept_len [B], band [B], band_kind [B])."""
    t = _as_f64(target)
    N, V = t.shape
    off = np.asarray(node_offsets)
    B = off.size - 1
    t, tp = _f64(t)
    d, dp = _f64(_as_f64(draft).reshape(N, V))
    off, offp = _i32(off)
    par, parp = _i32(parent)
    tk, tkp = _i32(tokens)
    ua, uap = _f64(_as_f64(u_accept).reshape(N))
    ur, urp = _f64(_as_f64(u_resid).reshape(N))
    T, Tp = _f64(np.broadcast_to(np.asarray(temperature, dtype=np.float64), (B,)))
    P, Pp = _f64(np.broadcast_to(np.asarray(top_p, dtype=np.float64), (B,)))
    path, pathp = _i32(np.zeros((B, max(max_depth, 0))))
    otk, otkp = _i32(np.zeros((B, max_depth + 1)))
    ln, lnp = _i32(np.zeros(B))
    band, bp = _f64(np.zeros(B))
    kind, kp = _i32(np.zeros(B))
    Kk, Kkp = _top_k(top_k, B)
    if rule == TREE_SAMPLED_WOR:
        rc = _load().oracle_verify_tree(tp, dp, B, V, offp, parp, tkp, uap, urp, Tp, Pp, Kkp, int(max_depth), pathp,
                                        otkp, lnp, bp, kp)
    else:
        rc = _load().oracle_verify_tree_rule(tp, dp, B, V, offp, parp, tkp, uap, urp, Tp, Pp, Kkp, int(max_depth),
                                             int(rule), pathp, otkp, lnp, bp, kp)
    if rc != 0:
        raise ValueError("oracle_verify_tree: bad arguments (rule %r)" % (rule,))
    return {"path": path, "tokens": otk, "accept_len": ln, "band": band, "band_kind": kind}


def build_tree(draft_rows, temperature: float, top_p: float, cand_k: int, n_prefixes: int, top_k: int = 0):
    """Candidate trie from the draft rows of K positions ([K, V] logits): the cand_k most probable
    tokens per position, then the n_prefixes most probable prefixes. Returns dict(parent,
    tokens, depth, score) over the trie's nodes (node 0 the empty prefix), or None when a
    draft row is bad."""
    d = _as_f64(draft_rows)
    K, V = d.shape
    d, dp = _f64(d)
    cap = int(n_prefixes) + 1
    par, parp = _i32(np.zeros(cap))
    tok, tokp = _i32(np.zeros(cap))
    dep, depp = _i32(np.zeros(cap))
    sc, scp = _f64(np.zeros(cap))
    nn, nnp = _i32(np.zeros(1))
    rc = _load().oracle_build_tree(dp, K, V, float(temperature), float(top_p), int(top_k), int(cand_k),
                                   int(n_prefixes), parp, tokp, depp, scp, nnp)
    if rc == -1:
        return None
    if rc != 0:
        raise ValueError("oracle_build_tree: bad arguments")
    n = int(nn[0])
    return {"parent": par[:n].copy(), "tokens": tok[:n].copy(), "depth": dep[:n].copy(), "score": sc[:n].copy()}
