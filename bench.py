"""Benchmark of the Psi-Spec verification step on B200.

One step = the whole hot path over one batch: psispec_sample_draft over the [B, K, V] draft
logits (token draw, q(x), per-row statistics), then psispec_verify_linear over the
[B, K+1, V] verifier logits reusing those statistics (accept tests, first rejection,
residual or bonus draw). Default workload "max", the largest linear configuration: B=512
requests, K=16 drafted positions, V=151936, bf16, T=1, top-p 0.95 on both distributions. Inputs
are synthetic (seeded) and already resident in HBM; together they are 5.1 GB, far larger than
the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload max] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun), every rank verifies its own batch; no
collective touches the data path (only the max-over-ranks timing reduction).
"""
import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified draft positions/sec and logits HBM GB/s vs B200 peak (Ψ-Spec verify)"
UNIT = "positions/s"
# kernel launches per step of the default workload (see csrc/psispec.cu): sample_draft =
# streaming pass + row finisher; verify_linear = streaming pass + row finisher + draw totals +
# draw pick


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _kernel_source_hash(files=None):
    """Hash of the kernel sources (all of them, or the named files that define one kernel)
    with their comments removed: a comment edit leaves the captured traffic valid; any code
    change invalidates it."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "lossless_speculative_sampling_b200", "csrc")
    for f in sorted(files or os.listdir(d)):
        with open(os.path.join(d, f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = "\n".join(line.split("//")[0].rstrip() for line in src.splitlines() if line.split("//")[0].strip())
        h.update(f.encode() + src.encode())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per launch of the dominant call, from the committed ncu summary, if it was
    taken on the current kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("source_hash") == _kernel_source_hash(e.get("source_files")):
            return e.get("bytes_per_call")
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        # nvidia-smi numbers GPUs differently from CUDA when CUDA_VISIBLE_DEVICES is set; the
        # UUID names the same device in both
        try:
            self.gpu = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.gpu = str(device.index or 0)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = [r.split(",") for r in self.out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


def _dist(backend: str = "nccl"):
    """(process group module or None, rank, world size, local rank) from the torchrun
    environment. Ranks are independent replicas; the only collectives are the timing barrier
    and the max over ranks. The GPU bench uses NCCL; the host-side tests use gloo."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        local = int(os.environ.get("LOCAL_RANK", "0"))
        timeout = datetime.timedelta(seconds=120)
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
        return dist, dist.get_rank(), ws, local
    return None, 0, 1, 0


def _barrier(dist):
    if dist is not None:
        dist.barrier()


def _max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    on_gpu = dist.get_backend() == "nccl"
    t = torch.tensor([x], device="cuda" if on_gpu else "cpu", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _rank_seed(seed: int, rank: int) -> int:
    """Each rank verifies its own batch (weak scaling): a seed per rank."""
    return seed + 97 * rank


def _oracle_sample(case, tgt_h, drf_h, ud, ua, ur, reqs):
    """The oracle (fp64 C, one thread) on requests `reqs` of the workload: draft draws then
    verification, exactly the step the GPU runs. Returns (draws, verification)."""
    import oracle

    K, V = case.K, case.V
    n = len(reqs)
    T, P = np.full(n, case.temperature), np.full(n, case.top_p)
    Kk = np.full(n, case.top_k, dtype=np.int32) if case.top_k else None
    d = drf_h[reqs].to(torch.float64).numpy()
    s = oracle.sample_draft(d.reshape(n * K, V), T, P, ud[reqs].reshape(-1), row_req=np.arange(n * K) // K, top_k=Kk)
    r = oracle.verify_linear(tgt_h[reqs].to(torch.float64).numpy(), d, s["tokens"].reshape(n, K), ua[reqs], ur[reqs],
                             T, P, top_k=Kk)
    return s, r


def _host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _oracle_parallel(case, tgt_h, drf_h, ud, ua, ur, reqs, threads):
    """The same oracle calls, one request per task on `threads` host threads (the C oracle
    runs outside the interpreter lock). Returns per-request (draws, verification) pairs."""
    from concurrent.futures import ThreadPoolExecutor

    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(lambda b: _oracle_sample(case, tgt_h, drf_h, ud, ua, ur, np.array([b])), reqs))


def _exceptions(case, results, reqs, gpu_x, gpu_tok, gpu_len):
    """Counted exceptions of the GPU results against the oracle on the sampled requests: draws
    and verifications whose path holds a decision within 1e-6 of its boundary, by kind (E1
    accept test, E2 draw edge, E3 top-p tail), how many of those differ, and any difference
    outside the bands (none is allowed)."""
    import oracle

    kinds = {oracle.BAND_E1: "e1", oracle.BAND_E2: "e2", oracle.BAND_E3: "e3"}
    out = {"requests_checked": 0, "rows_checked": 0, "e1": 0, "e2": 0, "e3": 0, "differ_in_band": 0,
           "differ_outside_band": 0, "verify_skipped_draft_differs": 0}
    K = case.K
    for b, (s, r) in zip(reqs, results):
        out["rows_checked"] += K
        same_x = True
        for i in range(K):
            band, kind = float(s["band"][i]), int(s["band_kind"][i])
            differs = int(gpu_x[b, i]) != int(s["tokens"][i])
            same_x &= not differs
            if band < oracle.E_BAND:
                out[kinds.get(kind, "e2")] += 1
                out["differ_in_band"] += int(differs)
            elif differs:
                out["differ_outside_band"] += 1
        if not same_x:
            out["verify_skipped_draft_differs"] += 1
            continue
        out["requests_checked"] += 1
        band, kind = float(r["band"][0]), int(r["band_kind"][0])
        differs = int(gpu_len[b]) != int(r["accept_len"][0]) or list(map(int, gpu_tok[b])) != list(
            map(int, r["tokens"][0]))
        if band < oracle.E_BAND:
            out[kinds.get(kind, "e2")] += 1
            out["differ_in_band"] += int(differs)
        elif differs:
            out["differ_outside_band"] += 1
    return out


def run_reference(args):
    """The reference arm: the oracle timed on the host cores (rank 0 only), one request per
    host thread."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from lossless_speculative_sampling_b200 import synth

    if args.workload in synth.tree_cases():
        return _run_reference_tree(args)
    if args.workload in synth.trie_cases():
        return _run_reference_trie(args)
    case = synth.linear_cases()[args.workload]
    threads = _host_threads()
    # one request per host thread per step, bounded so that the whole run stays near two
    # minutes (a request of the top-p workloads takes about a second on one thread)
    per_req = 1.0 if case.top_p < 1.0 or case.top_k else 0.1
    n_req = max(1, min(case.B, threads * args.ref_requests,
                       int(threads * 120.0 / (per_req * (args.steps + args.warmup)))))
    tgt, drf = synth.linear_logits(case, device="cpu", B=n_req)
    ud, ua, ur = synth.linear_uniforms(case, B=n_req)
    reqs = np.arange(n_req)
    for _ in range(args.warmup):
        _oracle_parallel(case, tgt, drf, ud, ua, ur, reqs[:threads], threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_parallel(case, tgt, drf, ud, ua, ur, reqs, threads)
    dt = (time.perf_counter() - t0) / args.steps
    value = n_req * case.K / dt
    sample = "%d of %d requests of workload %s per step (fp64 C oracle, one request per host thread, %d threads)" % (
        n_req, case.B, args.workload, threads)
    _print_reference(args, value, dt, "f64", {"workload": args.workload, "requests_per_step": n_req, "block": case.K,
                                              "vocab": case.V}, sample, cores=threads)


def _run_reference_tree(args):
    import oracle
    from lossless_speculative_sampling_b200 import synth

    case = synth.tree_cases()[args.workload]
    trie, tgt, drf, tokens, ua, ur = synth.tree_inputs(case, device="cpu")
    n_req = max(1, min(case.B, args.ref_requests))
    n = int(trie.node_offsets[n_req])
    t, d = tgt[:n].to(torch.float64).numpy(), drf[:n].to(torch.float64).numpy()
    off, par, tok = trie.node_offsets[: n_req + 1].numpy(), trie.parent[:n].numpy(), tokens[:n].numpy()
    a, r = ua[:n].numpy(), ur[:n].numpy()
    T, P = np.full(n_req, case.temperature), np.full(n_req, case.top_p)

    def one():
        oracle.verify_tree(t, d, off, par, tok, a, r, T, P, case.max_depth)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / args.steps
    sample = "%d of %d tries (%d nodes) of workload %s per step (fp64 C oracle, 1 thread)" % (n_req, case.B, n,
                                                                                              args.workload)
    _print_reference(args, n / dt, dt, "f64", {"workload": args.workload, "tries_per_step": n_req, "nodes": n,
                                               "vocab": case.V}, sample)


def _run_reference_trie(args):
    """The oracle's candidate trie and its deterministic-rule verification, one request per host
    thread, on a bounded number of the workload's requests."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from lossless_speculative_sampling_b200 import synth

    case = synth.trie_cases()[args.workload]
    K, V, n = case.K, case.V, case.n_prefixes
    threads = _host_threads()
    n_req = max(1, min(case.B, threads))
    drf = synth.trie_draft(case, device="cpu")[:n_req].to(torch.float64)
    ua, ur = synth.trie_uniforms(case)

    def one(b):
        t = oracle.build_tree(drf[b].numpy(), case.temperature, case.top_p, case.cand_k, n)
        dep = torch.from_numpy(t["depth"]).view(1, -1)
        rows = synth.trie_verifier_rows(case, drf[b:b + 1].to(case.dtype), dep).to(torch.float64).numpy()
        tk = t["tokens"].copy()
        tk[0] = 0
        m = len(tk)
        s0 = b * (n + 1)
        return oracle.verify_tree(rows, rows, [0, m], t["parent"], tk, ua[s0:s0 + m], ur[s0:s0 + m],
                                  [case.temperature], [case.top_p], K, rule=oracle.TREE_DETERMINISTIC)

    def step():
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(n_req)))

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    sample = "%d of %d requests of workload %s per step (fp64 C oracle, one request per host thread, %d threads)" % (
        n_req, case.B, args.workload, threads)
    _print_reference(args, n_req * n / dt, dt, "f64", {"workload": args.workload, "requests_per_step": n_req,
                                                       "block": K, "vocab": V, "cand_k": case.cand_k,
                                                       "n_prefixes": n}, sample, cores=threads)


def _print_reference(args, value, dt, dtype, config, sample, cores=1):
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                             "host_cores": os.cpu_count()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _prepare_linear(case, dev):
    """Device inputs, outputs and the two calls of one linear step."""
    from lossless_speculative_sampling_b200 import psispec, synth

    B, K, V = case.B, case.K, case.V
    tgt, drf = synth.linear_logits(case, device=dev)
    ud, ua, ur = synth.linear_uniforms(case)
    ud, ua, ur = ud.to(dev), ua.to(dev), ur.to(dev)
    Ts = torch.full((B,), case.temperature, device=dev)
    Ps = torch.full((B,), case.top_p, device=dev)
    Ks = torch.full((B,), case.top_k, dtype=torch.int32, device=dev) if case.top_k else None
    x = torch.empty((B, K), dtype=torch.int32, device=dev)
    q = torch.empty((B, K), dtype=torch.float32, device=dev)
    stats = torch.empty((B, K, psispec.ROW_STATS_BYTES), dtype=torch.uint8, device=dev)
    o_tok = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    o_len = torch.empty(B, dtype=torch.int32, device=dev)
    o_p = torch.empty((B, K), dtype=torch.float32, device=dev)
    o_q = torch.empty((B, K), dtype=torch.float32, device=dev)
    ws_s = torch.empty(psispec.workspace_size(psispec.OP_SAMPLE_DRAFT, B, K, V), dtype=torch.uint8, device=dev)
    ws_v = torch.empty(psispec.workspace_size(psispec.OP_VERIFY_LINEAR, B, K, V), dtype=torch.uint8, device=dev)
    ws_r = torch.empty(psispec.workspace_size(psispec.OP_ROW_STATS, B, K + 1, V), dtype=torch.uint8, device=dev)
    rec = torch.empty((B, K + 1, psispec.ROW_STATS_BYTES), dtype=torch.uint8, device=dev)
    esz = tgt.element_size()

    def sample(t_in=tgt, d_in=drf):
        psispec.sample_draft(d_in, Ts, Ps, ud, top_k=Ks, out_tokens=x, out_q=q, row_stats=stats, ws=ws_s)

    def verify(t_in=tgt, d_in=drf):
        psispec.verify_linear(t_in, d_in, x, ua, ur, Ts, Ps, top_k=Ks, draft_row_stats=stats, out_tokens=o_tok,
                              out_accept_len=o_len, out_p=o_p, out_q=o_q, ws=ws_v)

    def stream_leg():  # the streaming pass over the verifier tensor alone (plus its row finalize)
        psispec.row_stats(tgt, Ts, Ps, out=rec, ws=ws_r)

    return {
        "inputs": (tgt, drf), "calls": [("sample_draft", sample), ("verify_linear", verify)],
        "outputs": (o_tok, o_len), "draft_tokens": x, "positions": B * K, "esz": esz,
        # algorithmic bytes: sample_draft reads the draft tensor once; verify_linear reads the
        # verifier tensor once plus, per request, the one draft row of the residual draw
        "bytes": {"sample_draft": B * K * V * esz, "verify_linear": B * (K + 1) * V * esz + B * V * esz},
        "bytes_step": (B * (K + 1) + B * K) * V * esz,
        # stream + sample rows; stream + verify rows + cluster draw
        "launches": 2 + 3,
        # the dominant kernel: with a cut (top-p / top-k, bf16), the one-pass cut-row CTAs
        # (cut_rows_kernel, the launch psispec_row_stats makes for them; the streaming pass and
        # the finalize there find no rows and return at once); without one, the streaming pass
        "kernel_leg": (("cut_rows_kernel" if (case.top_p < 1.0 or case.top_k) and esz == 2 else
                        "stream_partials_tma_kernel") + " (psispec_row_stats over the verifier tensor)", stream_leg,
                       B * (K + 1) * V * esz),
        "describe": "linear verify B=%d K=%d V=%d %s, T=%g, top-p %g%s" % (
            B, K, V, "bf16" if esz == 2 else "fp32", case.temperature, case.top_p,
            ", top-k %d" % case.top_k if case.top_k else ""),
        "config": {"global_batch": B, "block": K, "vocab": V},
        "accept": lambda: float(o_len.float().mean()),
    }


def _prepare_tree(case, dev):
    """Device inputs, outputs and the one call of a tree step."""
    from lossless_speculative_sampling_b200 import psispec, synth

    trie, tgt, drf, tokens, ua, ur = synth.tree_inputs(case, device=dev)
    B, N, V = case.B, trie.N, case.V
    offs, parent, tok = trie.node_offsets.to(dev), trie.parent.to(dev), tokens.to(dev)
    ua, ur = ua.to(dev), ur.to(dev)
    Ts = torch.full((B,), case.temperature, device=dev)
    Ps = torch.full((B,), case.top_p, device=dev)
    D = case.max_depth
    o_path = torch.empty((B, D), dtype=torch.int32, device=dev)
    o_tok = torch.empty((B, D + 1), dtype=torch.int32, device=dev)
    o_len = torch.empty(B, dtype=torch.int32, device=dev)
    ws = torch.empty(psispec.workspace_size(psispec.OP_VERIFY_TREE, B, N, V), dtype=torch.uint8, device=dev)
    esz = tgt.element_size()

    def verify(t_in=tgt, d_in=drf):
        psispec.verify_tree(t_in, d_in, offs, parent, tok, ua, ur, Ts, Ps, D, out_path=o_path, out_tokens=o_tok,
                            out_accept_len=o_len, ws=ws)

    def visited_bytes():
        # what the walk actually reads: the verifier and draft rows of the nodes it visits (the
        # accepted path and the node where it stops), len + 1 nodes per trie
        n = int((o_len.clamp(min=-1) + 1).sum())
        return 2 * n * V * esz

    return {
        "inputs": (tgt, drf), "calls": [("verify_tree", verify)], "outputs": (o_tok, o_len), "positions": N,
        # algorithmic bytes as the metric defines them: both logit tensors once
        "esz": esz, "bytes": {"verify_tree": 2 * N * V * esz}, "bytes_step": 2 * N * V * esz,
        "read_bytes": visited_bytes, "launches": 3,
        "describe": "tree verify B=%d tries x %d nodes (depth <= %d, branching <= %d) V=%d %s, T=%g, top-p %g" % (
            B, case.nodes, case.max_depth, case.max_branch, V, "bf16" if esz == 2 else "fp32", case.temperature,
            case.top_p),
        "config": {"global_batch": B, "nodes": N, "vocab": V},
        "accept": lambda: float(o_len.float().mean()),
    }


def _prepare_trie(case, dev):
    """The tree sampler's step: the candidate trie from the draft rows (psispec_build_tree),
    then its verification with the deterministic-candidate rule (psispec_verify_tree_det) on
    the verifier rows of its nodes."""
    from lossless_speculative_sampling_b200 import psispec, synth

    B, K, V, n = case.B, case.K, case.V, case.n_prefixes
    cap = n + 1
    drf = synth.trie_draft(case, device=dev)
    Ts = torch.full((B,), case.temperature, device=dev)
    Ps = torch.full((B,), case.top_p, device=dev)
    trie = {"parent": torch.empty((B, cap), dtype=torch.int32, device=dev),
            "tokens": torch.empty((B, cap), dtype=torch.int32, device=dev),
            "depth": torch.empty((B, cap), dtype=torch.int32, device=dev),
            "score": torch.empty((B, cap), dtype=torch.float64, device=dev),
            "nodes": torch.empty(B, dtype=torch.int32, device=dev)}
    ws_b = torch.empty(psispec.workspace_size(psispec.OP_BUILD_TREE, B, K, V), dtype=torch.uint8, device=dev)
    psispec.build_tree(drf, Ts, Ps, case.cand_k, n, out=trie, ws=ws_b)
    assert bool((trie["nodes"] == cap).all()), "every request keeps n_prefixes prefixes"
    tgt = synth.trie_verifier_rows(case, drf, trie["depth"])  # the verifier rows of the built trie's nodes
    ua, ur = (t.to(dev) for t in synth.trie_uniforms(case))
    offs = torch.arange(0, B * cap + 1, cap, dtype=torch.int32, device=dev)
    o_path = torch.empty((B, K), dtype=torch.int32, device=dev)
    o_tok = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    o_len = torch.empty(B, dtype=torch.int32, device=dev)
    ws_v = torch.empty(psispec.workspace_size(psispec.OP_VERIFY_TREE, B, B * cap, V), dtype=torch.uint8, device=dev)
    esz = tgt.element_size()

    def build(t_in=tgt, d_in=drf):
        psispec.build_tree(d_in, Ts, Ps, case.cand_k, n, out=trie, ws=ws_b)

    def verify(t_in=tgt, d_in=drf):
        psispec.verify_tree_det(t_in, offs, trie["parent"].view(-1), trie["tokens"].view(-1), ua, ur, Ts, Ps, K,
                                out_path=o_path, out_tokens=o_tok, out_accept_len=o_len, ws=ws_v)

    return {
        "inputs": (tgt, drf), "calls": [("build_tree", build), ("verify_tree_det", verify)],
        "outputs": (o_tok, o_len), "positions": B * n, "esz": esz,
        "bytes": {"build_tree": B * K * V * esz, "verify_tree_det": B * cap * V * esz},
        "bytes_step": (B * K + B * cap) * V * esz, "launches": 4 + 3,
        "describe": "candidate trie B=%d K=%d V=%d %s, %d candidates per position, %d prefixes, T=%g, top-p %g" % (
            B, K, V, "bf16" if esz == 2 else "fp32", case.cand_k, n, case.temperature, case.top_p),
        "config": {"global_batch": B, "block": K, "vocab": V, "cand_k": case.cand_k, "n_prefixes": n},
        "accept": lambda: float(o_len.float().mean()),
    }


def _prepare(name, dev, rank=0):
    from lossless_speculative_sampling_b200 import synth

    lin, tre, tri = synth.linear_cases(), synth.tree_cases(), synth.trie_cases()
    if name in lin:
        case = lin[name]
        case.seed = _rank_seed(case.seed, rank)
        return _prepare_linear(case, dev), case
    if name in tri:
        case = tri[name]
        case.seed = _rank_seed(case.seed, rank)
        return _prepare_trie(case, dev), case
    case = tre[name]
    case.seed = _rank_seed(case.seed, rank)
    return _prepare_tree(case, dev), case


def _graphs(calls, dev, warmup):
    """Each call captured once into a CUDA graph and replayed: the launch sequence a serving
    loop would use."""
    for _ in range(warmup):
        for _, f in calls:
            f()
    torch.cuda.synchronize()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _, f in calls:
            f()
    torch.cuda.current_stream(dev).wait_stream(side)
    out = []
    for name, f in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            f()
        out.append((name, g.replay, g))
    for _ in range(warmup):
        for _, r, _g in out:
            r()
    torch.cuda.synchronize()
    return out


def _time_leg(fn, dev, steps, warmup):
    """Mean device time (ms) of one launch sequence, captured in a CUDA graph."""
    ((_, replay, g),) = _graphs([("leg", fn)], dev, warmup)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / steps


def _time_steps(calls, steps, dist=None):
    """Device time of `steps` steps (CUDA events on the launching stream): (ms per step,
    {call: mean ms})."""
    n = len(calls)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range((n + 1) * steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    _barrier(dist)
    start.record()
    for k in range(steps):
        for i, c in enumerate(calls):
            ev[(n + 1) * k + i].record()
            c[1]()
        ev[(n + 1) * k + n].record()
    end.record()
    torch.cuda.synchronize()
    _barrier(dist)
    ms = _max_over_ranks(dist, start.elapsed_time(end)) / steps
    per = {c[0]: statistics.mean(ev[(n + 1) * k + i].elapsed_time(ev[(n + 1) * k + i + 1]) for k in range(steps))
           for i, c in enumerate(calls)}
    return ms, per


def _all_workloads(args, dev):
    """One JSON line per workload (the parity configurations at full size), for the tables."""
    from lossless_speculative_sampling_b200 import synth

    peak, peak_kind = _peaks()
    names = [n for n in synth.linear_cases() if n != "tiny"] + list(synth.tree_cases()) + list(synth.trie_cases())
    for name in names:
        P, case = _prepare(name, dev)
        calls = _graphs(P["calls"], dev, 3) if not args.no_graph else P["calls"]
        steps = max(5, min(args.steps, int(2e5 / max(1.0, P["bytes_step"] / 1e6))))
        ms, per = _time_steps(calls, steps)
        line = {"workload": name, "describe": P["describe"], "value": P["positions"] / (ms * 1e-3), "unit": UNIT,
                "ms_per_step": ms, "steps": steps, "step_gbs": P["bytes_step"] / (ms * 1e-3) / 1e9,
                "calls_ms": per, "calls_gbs": {k: P["bytes"][k] / (per[k] * 1e-3) / 1e9 for k in per},
                "peak_gbs": peak, "peak_kind": peak_kind, "mean_accept_len": P["accept"]()}
        line["step_frac"] = line["step_gbs"] / peak
        print(json.dumps(line), flush=True)
        del P, calls
        torch.cuda.empty_cache()


def run_ours(args):
    dist, rank, world, local = _dist()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.all:
        _all_workloads(args, dev)
        if dist is not None:
            dist.destroy_process_group()
        return
    P, case = _prepare(args.workload, dev, rank)
    calls = P["calls"] if args.no_graph else _graphs(P["calls"], dev, args.warmup)
    if args.no_graph:
        for _ in range(args.warmup):
            for _, f in calls:
                f()
    _barrier(dist)
    with ClockSampler(dev) as clk:
        ms_step, per = _time_steps(calls, args.steps, dist)
        # the dominant kernel alone, for the roofline (same inputs, launched right after)
        leg_ms = None
        if "kernel_leg" in P:
            leg_ms = _max_over_ranks(dist, _time_leg(P["kernel_leg"][1], dev, max(args.steps, 10), args.warmup))
    mean_accept = P["accept"]()

    # end to end through the public API with host buffers: pinned H2D of the step's inputs,
    # the step, D2H of its result, every step inside the timed region
    e2e_steps = max(3, min(args.steps, 20))
    hosts = [t.cpu().pin_memory() for t in P["inputs"]]
    devs = [torch.empty_like(t) for t in P["inputs"]]
    outs_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in P["outputs"]]
    for _, f in P["calls"]:
        f(*devs)
    torch.cuda.synchronize()
    _barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        for d, h in zip(devs, hosts):
            d.copy_(h, non_blocking=True)
        for _, f in P["calls"]:
            f(*devs)
        for h, o in zip(outs_h, P["outputs"]):
            h.copy_(o, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(dist, e0.elapsed_time(e1)) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for t in P["inputs"])
    d2h = sum(o.numel() * o.element_size() for o in P["outputs"])
    del hosts, devs

    cpu, exc = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload in _linear_names():
        cpu, exc = _cpu_baseline(args, case, P)

    peak, peak_kind = _peaks()
    main_call = P["calls"][-1][0]
    if leg_ms is not None:
        kname, kbytes = P["kernel_leg"][0], P["kernel_leg"][2]
        gbs_main = kbytes / (leg_ms * 1e-3) / 1e9
    else:  # the call itself (the tree, where the walk dominates)
        kname, kbytes = "psispec_" + main_call, P["bytes"][main_call]
        gbs_main = kbytes / (per[main_call] * 1e-3) / 1e9
    value = world * P["positions"] / (ms_step * 1e-3)
    esz = P["esz"]
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if esz == 2 else "f32", "data": "synthetic",
            "config": dict({"workload": "%s: %s" % (args.workload, P["describe"]), "parallelism": "replicas x%d" % world,
                            "l2": "inputs %.0f MB > 126 MB L2, no flush" % (P["bytes_step"] / 1e6),
                            "cuda_graph": not args.no_graph}, **P["config"]),
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": gbs_main, "peak": peak,
                         "unit": "GB/s", "frac": gbs_main / peak, "peak_kind": peak_kind,
                         "traffic": _traffic(args.workload), "bytes_per_launch": kbytes,
                         "ms_per_launch": leg_ms if leg_ms is not None else per[main_call]},
            # bytes the step's kernels read from the logits where that is less than the metric's
            # both-tensors-once (the tree walk reads only the rows of the nodes it visits)
            "logit_bytes_read_per_step": P["read_bytes"]() if "read_bytes" in P else None,
            "step_gbs": P["bytes_step"] / (ms_step * 1e-3) / 1e9,
            "step_frac": P["bytes_step"] / (ms_step * 1e-3) / 1e9 / peak,
            "calls": dict({k + "_ms": v for k, v in per.items()},
                          **{k + "_gbs": P["bytes"][k] / (v * 1e-3) / 1e9 for k, v in per.items()}),
            "mean_accept_len": mean_accept,
            # the GPU's results on the requests the oracle leg computed (1e-6 bands by kind)
            "exceptions": exc,
            "e2e": {"value": world * P["positions"] / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": P["launches"] * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def _linear_names():
    from lossless_speculative_sampling_b200 import synth

    return set(synth.linear_cases())


def _cpu_baseline(args, case, P):
    """The oracle as it stands, on a bounded sample of the same workload (host cores): one
    thread, then one request per host thread; its results on the sampled requests are also the
    exception counts of the GPU's results (returned separately)."""
    from lossless_speculative_sampling_b200 import synth

    B, K = case.B, case.K
    tgt_c, drf_c = (t.cpu() for t in P["inputs"])
    udc, uac, urc = synth.linear_uniforms(synth.linear_cases()[args.workload])
    threads = _host_threads()
    # single thread: requests spread over the batch until about half the time budget is spent
    order = np.unique(np.linspace(0, B - 1, B).astype(int))[::max(1, B // 64)]
    done, results = [], []
    t0 = time.perf_counter()
    for b in order:
        if time.perf_counter() - t0 >= args.cpu_seconds / 2:
            break
        results.append(_oracle_sample(case, tgt_c, drf_c, udc, uac, urc, np.array([b])))
        done.append(int(b))
    dt1 = time.perf_counter() - t0
    one = len(done) * K / dt1
    # one request per host thread: as many requests as one thread did per thread, bounded by B
    n_par = int(min(B, max(threads, len(done) * threads)))
    par = np.linspace(0, B - 1, n_par).astype(int)
    t0 = time.perf_counter()
    res_par = _oracle_parallel(case, tgt_c, drf_c, udc, uac, urc, par, threads)
    dtp = time.perf_counter() - t0
    many = n_par * K / dtp
    x = P["draft_tokens"].cpu().numpy()
    tok, ln = (o.cpu().numpy() for o in P["outputs"])
    seen = set(done)
    all_reqs = done + [int(b) for b in par if int(b) not in seen]
    all_res = results + [r for b, r in zip(par, res_par) if int(b) not in seen]
    exc = _exceptions(case, all_res, all_reqs, x, tok, ln)
    cpu = {"value": many, "unit": UNIT, "cores": threads, "kind": "oracle", "host_cores": os.cpu_count(),
           "single_thread_value": one,
           "sample": "workload %s (sample_draft + verify_linear, fp64 C oracle): %d requests on 1 thread in %.1f s, "
                     "then %d requests spread over the batch, one per host thread on %d threads, in %.1f s" % (
                         args.workload, len(done), dt1, n_par, threads, dtp)}
    return cpu, exc


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="max")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch calls directly instead of replaying CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--ref-requests", type=int, default=2, help="requests per host thread in a reference step")
    ap.add_argument("--all", action="store_true", help="one line per full-size workload instead of the bench line")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
