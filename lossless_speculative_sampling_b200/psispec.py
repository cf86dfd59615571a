"""ctypes binding of libpsispec.so (the C ABI in include/psispec.h).

Argument marshalling only: torch CUDA tensors in, device pointers and sizes to the library,
torch tensors out. Outputs and workspaces that the caller does not pass are allocated with
torch (device memory is plumbing here); the library itself allocates nothing. Calls are
enqueued on the current torch stream of the tensors' device (or the `stream` argument).

Loading fails loudly when the library has not been built (`python -m
lossless_speculative_sampling_b200.build`); there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsispec.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "psispec.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE = 0, 1, 2, 3, 4
STATIC_WORKSPACE_BYTES = 16 << 20  # PSISPEC_STATIC_WORKSPACE_BYTES
F32, BF16 = 0, 1
OP_SAMPLE_DRAFT, OP_VERIFY_LINEAR, OP_VERIFY_TREE, OP_ROW_STATS, OP_BUILD_TREE = 0, 1, 2, 3, 4
ROW_STATS_BYTES = 32

_lib = None


class PsispecError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


def lib():
    """The loaded library (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libpsispec.so is not built (%s); run `python -m lossless_speculative_sampling_b200.build`"
                               % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.psispec_status_string.argtypes, L.psispec_status_string.restype = [ctypes.c_int], ctypes.c_char_p
        L.psispec_version.argtypes, L.psispec_version.restype = [], ctypes.c_int
        L.psispec_workspace_size.argtypes, L.psispec_workspace_size.restype = [ctypes.c_int, I64, I64, I64], SZ
        L.psispec_sample_draft.argtypes = [P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, SZ, P]
        L.psispec_row_stats.argtypes = [P, ctypes.c_int, I32, I32, I32, P, P, P, P, SZ, P]
        L.psispec_verify_linear.argtypes = [P, P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.psispec_sample_draft_k.argtypes = [P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, P, SZ, P]
        L.psispec_verify_linear_k.argtypes = [P, P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P, P, SZ,
                                              P]
        L.psispec_verify_tree.argtypes = [P, P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, I32, P, P, P, P, SZ,
                                          P]
        L.psispec_verify_tree_k.argtypes = [P, P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, P, I32, P, P, P, P,
                                            SZ, P]
        L.psispec_row_stats_k.argtypes = [P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, SZ, P]
        L.psispec_build_tree.argtypes = [P, ctypes.c_int, I32, I32, I32, P, P, P, I32, I32, P, P, P, P, P, P, SZ, P]
        L.psispec_verify_tree_det.argtypes = [P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, P, I32, P, P, P, P,
                                              SZ, P]
        L.psispec_verify_linear_static.argtypes = [P, P, ctypes.c_int, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P]
        for f in ("psispec_sample_draft", "psispec_sample_draft_k", "psispec_row_stats", "psispec_row_stats_k",
                  "psispec_verify_linear", "psispec_verify_linear_k", "psispec_verify_tree", "psispec_verify_tree_k",
                  "psispec_verify_linear_static", "psispec_build_tree", "psispec_verify_tree_det"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def declared_symbols():
    """Function names declared in include/psispec.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(psispec_[a-z_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().psispec_status_string(int(status)).decode()


def workspace_size(op: int, a: int, b: int, c: int) -> int:
    return int(lib().psispec_workspace_size(int(op), int(a), int(b), int(c)))


_ws_cache: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A cached device scratch buffer of at least nbytes (256-byte aligned by torch's allocator).
    Calls on different streams must not share it; pass an explicit workspace in that case."""
    dev = torch.device(device)
    buf = _ws_cache.get(dev)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _ws_cache[dev] = buf
    return buf


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError("logits must be bfloat16 or float32, got %s" % t.dtype)


def _req(t: torch.Tensor, name: str, dtype=None, numel=None, device=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if numel is not None and t.numel() != numel:
        raise ValueError("%s must have %d elements, got %d" % (name, numel, t.numel()))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    return t


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, what: str):
    if status != OK:
        raise PsispecError(status, what)


def sample_draft(draft, temperature, top_p, u, *, top_k=None, out_tokens=None, out_q=None, row_stats=None, ws=None,
                 stream=None):
    """Draw one token per drafted position from q = softmax(draft / T) after top-k and top-p.

    draft [B, K, V] bf16/fp32; temperature, top_p [B] fp32; u [B, K] fp32 in [0, 1); top_k
    [B] int32 or None (off; k <= 0 or k >= V is off too).
    Returns (tokens [B, K] int32, q(token) [B, K] fp32, row_stats [B, K, 32] uint8), the last
    reusable by verify_linear(draft_row_stats=...) with the same top_k."""
    B, K, V = draft.shape
    dev = draft.device
    _req(draft, "draft")
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    _req(u, "u", torch.float32, B * K, dev)
    if top_k is not None:
        _req(top_k, "top_k", torch.int32, B, dev)
    out_tokens = torch.empty((B, K), dtype=torch.int32, device=dev) if out_tokens is None else out_tokens
    out_q = torch.empty((B, K), dtype=torch.float32, device=dev) if out_q is None else out_q
    row_stats = torch.empty((B, K, ROW_STATS_BYTES), dtype=torch.uint8, device=dev) if row_stats is None else row_stats
    _req(out_tokens, "out_tokens", torch.int32, B * K, dev)
    _req(out_q, "out_q", torch.float32, B * K, dev)
    _req(row_stats, "row_stats", torch.uint8, B * K * ROW_STATS_BYTES, dev)
    need = workspace_size(OP_SAMPLE_DRAFT, B, K, V)
    ws = workspace(need, dev) if ws is None else ws
    if top_k is None:
        st = lib().psispec_sample_draft(_p(draft), _dtype(draft), B, K, V, _p(temperature), _p(top_p), _p(u),
                                        _p(out_tokens), _p(out_q), _p(row_stats), _p(ws), ws.numel(),
                                        _stream(dev, stream))
    else:
        st = lib().psispec_sample_draft_k(_p(draft), _dtype(draft), B, K, V, _p(temperature), _p(top_p), _p(top_k),
                                          _p(u), _p(out_tokens), _p(out_q), _p(row_stats), _p(ws), ws.numel(),
                                          _stream(dev, stream))
    _check(st, "psispec_sample_draft")
    return out_tokens, out_q, row_stats


def row_stats(logits, temperature, top_p, *, top_k=None, out=None, ws=None, stream=None):
    """Per-row statistics records of softmax(logits / T) after top-k and top-p.

    logits [B, K, V] bf16/fp32; temperature, top_p [B] fp32; top_k [B] int32 or None (off).
    Returns [B, K, 32] uint8 records, usable as verify_linear(draft_row_stats=...) for the same
    logits and controls."""
    B, K, V = logits.shape
    dev = logits.device
    _req(logits, "logits")
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    if top_k is not None:
        _req(top_k, "top_k", torch.int32, B, dev)
    out = torch.empty((B, K, ROW_STATS_BYTES), dtype=torch.uint8, device=dev) if out is None else out
    _req(out, "out", torch.uint8, B * K * ROW_STATS_BYTES, dev)
    need = workspace_size(OP_ROW_STATS, B, K, V)
    ws = workspace(need, dev) if ws is None else ws
    if top_k is None:
        st = lib().psispec_row_stats(_p(logits), _dtype(logits), B, K, V, _p(temperature), _p(top_p), _p(out),
                                     _p(ws), ws.numel(), _stream(dev, stream))
    else:
        st = lib().psispec_row_stats_k(_p(logits), _dtype(logits), B, K, V, _p(temperature), _p(top_p), _p(top_k),
                                       _p(out), _p(ws), ws.numel(), _stream(dev, stream))
    _check(st, "psispec_row_stats")
    return out


def verify_linear(target, draft, draft_tokens, u_accept, u_resid, temperature, top_p, *, top_k=None,
                  draft_row_stats=None, out_tokens=None, out_accept_len=None, out_p=None, out_q=None, want_pq=True,
                  ws=None, stream=None):
    """Psi-Spec linear verification. target [B, K+1, V], draft [B, K, V] (same dtype),
    draft_tokens [B, K] int32, u_accept [B, K], u_resid [B, K+1], temperature/top_p [B],
    top_k [B] int32 or None (off).
    Returns dict(tokens [B, K+1], accept_len [B], p [B, K], q [B, K]) (p/q None if not wanted)."""
    B, K1, V = target.shape
    K = K1 - 1
    dev = target.device
    _req(target, "target")
    _req(draft, "draft", target.dtype, B * K * V, dev)
    _req(draft_tokens, "draft_tokens", torch.int32, B * K, dev)
    _req(u_accept, "u_accept", torch.float32, B * K, dev)
    _req(u_resid, "u_resid", torch.float32, B * (K + 1), dev)
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    if top_k is not None:
        _req(top_k, "top_k", torch.int32, B, dev)
    if draft_row_stats is not None:
        _req(draft_row_stats, "draft_row_stats", torch.uint8, B * K * ROW_STATS_BYTES, dev)
    out_tokens = torch.empty((B, K + 1), dtype=torch.int32, device=dev) if out_tokens is None else out_tokens
    out_accept_len = torch.empty(B, dtype=torch.int32, device=dev) if out_accept_len is None else out_accept_len
    if want_pq:
        out_p = torch.empty((B, K), dtype=torch.float32, device=dev) if out_p is None else out_p
        out_q = torch.empty((B, K), dtype=torch.float32, device=dev) if out_q is None else out_q
    need = workspace_size(OP_VERIFY_LINEAR, B, K, V)
    ws = workspace(need, dev) if ws is None else ws
    if top_k is None:
        st = lib().psispec_verify_linear(_p(target), _p(draft), _dtype(target), B, K, V, _p(draft_tokens),
                                         _p(draft_row_stats), _p(u_accept), _p(u_resid), _p(temperature), _p(top_p),
                                         _p(out_tokens), _p(out_accept_len), _p(out_p), _p(out_q), _p(ws), ws.numel(),
                                         _stream(dev, stream))
    else:
        st = lib().psispec_verify_linear_k(_p(target), _p(draft), _dtype(target), B, K, V, _p(draft_tokens),
                                           _p(draft_row_stats), _p(u_accept), _p(u_resid), _p(temperature),
                                           _p(top_p), _p(top_k), _p(out_tokens), _p(out_accept_len), _p(out_p),
                                           _p(out_q), _p(ws), ws.numel(), _stream(dev, stream))
    _check(st, "psispec_verify_linear")
    return {"tokens": out_tokens, "accept_len": out_accept_len, "p": out_p, "q": out_q}


def verify_tree(target, draft, node_offsets, parent, tokens, u_accept, u_resid, temperature, top_p, max_depth: int,
                *, top_k=None, out_path=None, out_tokens=None, out_accept_len=None, ws=None, stream=None):
    """Psi-Spec tree verification. target/draft [N, V]; node_offsets [B+1] int32; parent,
    tokens [N] int32 (request-local parents, -1 at roots); u_accept, u_resid [N] fp32;
    temperature/top_p [B]; top_k [B] int32 or None (off). Returns dict(path [B, max_depth],
    tokens [B, max_depth+1], accept_len [B])."""
    N, V = target.shape
    B = node_offsets.numel() - 1
    dev = target.device
    _req(target, "target")
    _req(draft, "draft", target.dtype, N * V, dev)
    _req(node_offsets, "node_offsets", torch.int32, B + 1, dev)
    for name, t in (("parent", parent), ("tokens", tokens)):
        _req(t, name, torch.int32, N, dev)
    for name, t in (("u_accept", u_accept), ("u_resid", u_resid)):
        _req(t, name, torch.float32, N, dev)
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    if top_k is not None:
        _req(top_k, "top_k", torch.int32, B, dev)
    out_path = torch.empty((B, max_depth), dtype=torch.int32, device=dev) if out_path is None else out_path
    out_tokens = torch.empty((B, max_depth + 1), dtype=torch.int32, device=dev) if out_tokens is None else out_tokens
    out_accept_len = torch.empty(B, dtype=torch.int32, device=dev) if out_accept_len is None else out_accept_len
    need = workspace_size(OP_VERIFY_TREE, B, N, V)
    ws = workspace(need, dev) if ws is None else ws
    if top_k is None:
        st = lib().psispec_verify_tree(_p(target), _p(draft), _dtype(target), B, N, V, _p(node_offsets), _p(parent),
                                       _p(tokens), _p(u_accept), _p(u_resid), _p(temperature), _p(top_p),
                                       int(max_depth), _p(out_path), _p(out_tokens), _p(out_accept_len), _p(ws),
                                       ws.numel(), _stream(dev, stream))
    else:
        st = lib().psispec_verify_tree_k(_p(target), _p(draft), _dtype(target), B, N, V, _p(node_offsets),
                                         _p(parent), _p(tokens), _p(u_accept), _p(u_resid), _p(temperature),
                                         _p(top_p), _p(top_k), int(max_depth), _p(out_path), _p(out_tokens),
                                         _p(out_accept_len), _p(ws), ws.numel(), _stream(dev, stream))
    _check(st, "psispec_verify_tree")
    return {"path": out_path, "tokens": out_tokens, "accept_len": out_accept_len}


def verify_linear_static(target, draft, draft_tokens, u_accept, u_resid, temperature, top_p, *, draft_row_stats=None,
                         out_tokens=None, out_accept_len=None, out_p=None, out_q=None, want_pq=True, stream=None):
    """verify_linear with the library-owned scratch array (psispec_verify_linear_static): no
    workspace argument. Outputs not passed in are allocated here; pass them all to keep the
    call free of allocations."""
    B, K1, V = target.shape
    K = K1 - 1
    dev = target.device
    _req(target, "target")
    _req(draft, "draft", target.dtype, B * K * V, dev)
    _req(draft_tokens, "draft_tokens", torch.int32, B * K, dev)
    _req(u_accept, "u_accept", torch.float32, B * K, dev)
    _req(u_resid, "u_resid", torch.float32, B * (K + 1), dev)
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    if draft_row_stats is not None:
        _req(draft_row_stats, "draft_row_stats", torch.uint8, B * K * ROW_STATS_BYTES, dev)
    out_tokens = torch.empty((B, K + 1), dtype=torch.int32, device=dev) if out_tokens is None else out_tokens
    out_accept_len = torch.empty(B, dtype=torch.int32, device=dev) if out_accept_len is None else out_accept_len
    if want_pq:
        out_p = torch.empty((B, K), dtype=torch.float32, device=dev) if out_p is None else out_p
        out_q = torch.empty((B, K), dtype=torch.float32, device=dev) if out_q is None else out_q
    st = lib().psispec_verify_linear_static(_p(target), _p(draft), _dtype(target), B, K, V, _p(draft_tokens),
                                            _p(draft_row_stats), _p(u_accept), _p(u_resid), _p(temperature),
                                            _p(top_p), _p(out_tokens), _p(out_accept_len), _p(out_p), _p(out_q),
                                            _stream(dev, stream))
    _check(st, "psispec_verify_linear_static")
    return {"tokens": out_tokens, "accept_len": out_accept_len, "p": out_p, "q": out_q}

def build_tree(draft, temperature, top_p, cand_k: int, n_prefixes: int, *, top_k=None, out=None, ws=None,
               stream=None):
    """Candidate trie of the tree sampler from draft rows [B, K, V] (bf16/fp32): the cand_k
    most probable tokens per position, then the n_prefixes most probable prefixes.
    Returns dict(parent, tokens, depth [B, n_prefixes+1] int32, score [B, n_prefixes+1] fp64,
    nodes [B] int32); `out` may hold those tensors to write into."""
    B, K, V = draft.shape
    dev = draft.device
    _req(draft, "draft")
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    if top_k is not None:
        _req(top_k, "top_k", torch.int32, B, dev)
    cap = int(n_prefixes) + 1
    out = {} if out is None else out
    par = out.get("parent") if out.get("parent") is not None else torch.empty((B, cap), dtype=torch.int32, device=dev)
    tok = out.get("tokens") if out.get("tokens") is not None else torch.empty((B, cap), dtype=torch.int32, device=dev)
    dep = out.get("depth") if out.get("depth") is not None else torch.empty((B, cap), dtype=torch.int32, device=dev)
    score = out.get("score") if out.get("score") is not None else torch.empty((B, cap), dtype=torch.float64,
                                                                              device=dev)
    nodes = out.get("nodes") if out.get("nodes") is not None else torch.empty(B, dtype=torch.int32, device=dev)
    for name, t, dt in (("parent", par, torch.int32), ("tokens", tok, torch.int32), ("depth", dep, torch.int32),
                        ("score", score, torch.float64)):
        _req(t, name, dt, B * cap, dev)
    _req(nodes, "nodes", torch.int32, B, dev)
    need = workspace_size(OP_BUILD_TREE, B, K, V)
    ws = workspace(need, dev) if ws is None else ws
    st = lib().psispec_build_tree(_p(draft), _dtype(draft), B, K, V, _p(temperature), _p(top_p), _p(top_k),
                                  int(cand_k), int(n_prefixes), _p(par), _p(tok), _p(dep), _p(score), _p(nodes),
                                  _p(ws), ws.numel(), _stream(dev, stream))
    _check(st, "psispec_build_tree")
    return {"parent": par, "tokens": tok, "depth": dep, "score": score, "nodes": nodes}


def verify_tree_det(target, node_offsets, parent, tokens, u_accept, u_resid, temperature, top_p, max_depth: int, *,
                    top_k=None, out_path=None, out_tokens=None, out_accept_len=None, ws=None, stream=None):
    """Tree verification of a trie whose children were fixed in advance (the candidate trie):
    target [N, V]; node_offsets [B+1]; parent, tokens [N] int32; u_accept, u_resid [N] fp32;
    temperature/top_p [B]; top_k [B] int32 or None. Returns dict(path, tokens, accept_len)."""
    N, V = target.shape
    B = node_offsets.numel() - 1
    dev = target.device
    _req(target, "target")
    _req(node_offsets, "node_offsets", torch.int32, B + 1, dev)
    for name, t in (("parent", parent), ("tokens", tokens)):
        _req(t, name, torch.int32, N, dev)
    for name, t in (("u_accept", u_accept), ("u_resid", u_resid)):
        _req(t, name, torch.float32, N, dev)
    _req(temperature, "temperature", torch.float32, B, dev)
    _req(top_p, "top_p", torch.float32, B, dev)
    if top_k is not None:
        _req(top_k, "top_k", torch.int32, B, dev)
    out_path = torch.empty((B, max_depth), dtype=torch.int32, device=dev) if out_path is None else out_path
    out_tokens = torch.empty((B, max_depth + 1), dtype=torch.int32, device=dev) if out_tokens is None else out_tokens
    out_len = torch.empty(B, dtype=torch.int32, device=dev) if out_accept_len is None else out_accept_len
    _req(out_path, "out_path", torch.int32, B * max_depth, dev)
    _req(out_tokens, "out_tokens", torch.int32, B * (max_depth + 1), dev)
    _req(out_len, "out_accept_len", torch.int32, B, dev)
    need = workspace_size(OP_VERIFY_TREE, B, N, V)
    ws = workspace(need, dev) if ws is None else ws
    st = lib().psispec_verify_tree_det(_p(target), _dtype(target), B, N, V, _p(node_offsets), _p(parent), _p(tokens),
                                       _p(u_accept), _p(u_resid), _p(temperature), _p(top_p), _p(top_k),
                                       int(max_depth), _p(out_path), _p(out_tokens), _p(out_len), _p(ws), ws.numel(),
                                       _stream(dev, stream))
    _check(st, "psispec_verify_tree_det")
    return {"path": out_path, "tokens": out_tokens, "accept_len": out_len}
