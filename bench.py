"""Benchmark of the Psi-Spec verification step on B200.

One step = the whole hot path over one batch: psispec_sample_draft over the [B, K, V] draft
logits (token draw, q(x), per-row statistics), then psispec_verify_linear over the
[B, K+1, V] verifier logits reusing those statistics (accept tests, first rejection,
residual or bonus draw). Default workload "mid": B=64 requests, K=8 drafted positions,
V=151936, bf16, T=1, no top-p. Inputs are synthetic (seeded) and already resident in HBM;
together they are 330 MB, larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mid] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun), every rank verifies its own batch; no
collective touches the data path (only the max-over-ranks timing reduction).
"""
import argparse
import hashlib
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
# kernel launches per call (see csrc/psispec.cu): sample_draft = stream + finish + top-p;
# verify_linear = stream + finish + top-p + draw totals + draw pick (the per-request
# arrival counters are cleared with a memset, which is not a kernel of this library)
LAUNCHES_PER_STEP = 2 + 4  # sample: stream, sample_row; verify: stream, verify_row, draw totals, draw pick


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _kernel_source_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "lossless_speculative_sampling_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per launch of the dominant call, from the committed ncu summary, if it was
    taken on the current kernel sources."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("source_hash") == _kernel_source_hash():
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


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), ws, local
    return None, 0, 1, 0


def _barrier(dist):
    if dist is not None:
        dist.barrier()


def _max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], device="cuda", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _oracle_sample(case, tgt_h, drf_h, ud, ua, ur, reqs):
    """The oracle (fp64 C, one thread) on requests `reqs` of the workload: draft draws then
    verification, exactly the step the GPU runs."""
    import oracle

    K, V = case.K, case.V
    n = len(reqs)
    T, P = np.full(n, case.temperature), np.full(n, case.top_p)
    d = drf_h[reqs].to(torch.float64).numpy()
    s = oracle.sample_draft(d.reshape(n * K, V), T, P, ud[reqs].reshape(-1), row_req=np.arange(n * K) // K)
    r = oracle.verify_linear(tgt_h[reqs].to(torch.float64).numpy(), d, s["tokens"].reshape(n, K), ua[reqs], ur[reqs],
                             T, P)
    return r


def run_reference(args):
    """The reference arm: the oracle timed on the host cores (rank 0 only)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from lossless_speculative_sampling_b200 import synth

    case = synth.linear_cases()[args.workload]
    # about 80 ms of oracle work per request at V = 151936: keep the whole run near two minutes
    n_req = max(1, min(args.ref_requests, int(120.0 / (0.08 * (args.steps + args.warmup)))))
    tgt, drf = synth.linear_logits(case, device="cpu", B=n_req)
    ud, ua, ur = synth.linear_uniforms(case, B=n_req)
    reqs = np.arange(n_req)
    for _ in range(args.warmup):
        _oracle_sample(case, tgt, drf, ud, ua, ur, reqs[:1])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_sample(case, tgt, drf, ud, ua, ur, reqs)
    dt = (time.perf_counter() - t0) / args.steps
    value = n_req * case.K / dt
    sample = "%d of %d requests of workload %s per step (fp64 C oracle, 1 thread)" % (n_req, case.B, args.workload)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "requests_per_step": n_req, "block": case.K, "vocab": case.V},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    from lossless_speculative_sampling_b200 import psispec, synth

    dist, rank, world, local = _dist()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    case = synth.linear_cases()[args.workload]
    B, K, V = case.B, case.K, case.V
    case.seed += 97 * rank  # each rank verifies its own batch
    tgt, drf = synth.linear_logits(case, device=dev)
    ud, ua, ur = synth.linear_uniforms(case)
    ud, ua, ur = ud.to(dev), ua.to(dev), ur.to(dev)
    Ts = torch.full((B,), case.temperature, device=dev)
    Ps = torch.full((B,), case.top_p, device=dev)
    esz = tgt.element_size()

    x = torch.empty((B, K), dtype=torch.int32, device=dev)
    q = torch.empty((B, K), dtype=torch.float32, device=dev)
    stats = torch.empty((B, K, psispec.ROW_STATS_BYTES), dtype=torch.uint8, device=dev)
    o_tok = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    o_len = torch.empty(B, dtype=torch.int32, device=dev)
    o_p = torch.empty((B, K), dtype=torch.float32, device=dev)
    o_q = torch.empty((B, K), dtype=torch.float32, device=dev)
    ws_s = torch.empty(psispec.workspace_size(psispec.OP_SAMPLE_DRAFT, B, K, V), dtype=torch.uint8, device=dev)
    ws_v = torch.empty(psispec.workspace_size(psispec.OP_VERIFY_LINEAR, B, K, V), dtype=torch.uint8, device=dev)

    def step(t_in, d_in):
        psispec.sample_draft(d_in, Ts, Ps, ud, out_tokens=x, out_q=q, row_stats=stats, ws=ws_s)
        psispec.verify_linear(t_in, d_in, x, ua, ur, Ts, Ps, draft_row_stats=stats, out_tokens=o_tok,
                              out_accept_len=o_len, out_p=o_p, out_q=o_q, ws=ws_v)

    def call_sample():
        psispec.sample_draft(drf, Ts, Ps, ud, out_tokens=x, out_q=q, row_stats=stats, ws=ws_s)

    def call_verify():
        psispec.verify_linear(tgt, drf, x, ua, ur, Ts, Ps, draft_row_stats=stats, out_tokens=o_tok,
                              out_accept_len=o_len, out_p=o_p, out_q=o_q, ws=ws_v)

    for _ in range(args.warmup):
        step(tgt, drf)
    torch.cuda.synchronize()
    if not args.no_graph:
        # each call is captured once and replayed: the launch sequence a serving loop would use
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            call_sample()
            call_verify()
        torch.cuda.current_stream(dev).wait_stream(side)
        g_s, g_v = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_s):
            call_sample()
        with torch.cuda.graph(g_v):
            call_verify()
        call_sample, call_verify = g_s.replay, g_v.replay
        for _ in range(args.warmup):
            call_sample()
            call_verify()
        torch.cuda.synchronize()
    _barrier(dist)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        torch.cuda.synchronize()
        _barrier(dist)
        start.record()
        for k in range(args.steps):
            ev[3 * k].record()
            call_sample()
            ev[3 * k + 1].record()
            call_verify()
            ev[3 * k + 2].record()
        end.record()
        torch.cuda.synchronize()
        _barrier(dist)
    ms_total = _max_over_ranks(dist, start.elapsed_time(end))
    ms_step = ms_total / args.steps
    t_sample = statistics.mean(ev[3 * k].elapsed_time(ev[3 * k + 1]) for k in range(args.steps))
    t_verify = statistics.mean(ev[3 * k + 1].elapsed_time(ev[3 * k + 2]) for k in range(args.steps))
    mean_accept = float(o_len.float().mean())

    # end to end through the public API with host buffers: pinned H2D of the step's inputs,
    # the step, D2H of its result, every step inside the timed region
    e2e_steps = max(3, min(args.steps, 20))
    tgt_h = tgt.cpu().pin_memory()
    drf_h = drf.cpu().pin_memory()
    tok_h = torch.empty((B, K + 1), dtype=torch.int32).pin_memory()
    len_h = torch.empty(B, dtype=torch.int32).pin_memory()
    t_dev, d_dev = torch.empty_like(tgt), torch.empty_like(drf)
    step(tgt, drf)
    torch.cuda.synchronize()
    _barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        t_dev.copy_(tgt_h, non_blocking=True)
        d_dev.copy_(drf_h, non_blocking=True)
        step(t_dev, d_dev)
        tok_h.copy_(o_tok, non_blocking=True)
        len_h.copy_(o_len, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(dist, e0.elapsed_time(e1)) / e2e_steps
    h2d = (tgt.numel() + drf.numel()) * esz
    d2h = tok_h.numel() * 4 + len_h.numel() * 4

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tgt_c, drf_c = tgt.cpu(), drf.cpu()
        udc, uac, urc = synth.linear_uniforms(synth.linear_cases()[args.workload])
        n = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds and n < B:
            _oracle_sample(case, tgt_c, drf_c, udc, uac, urc, np.arange(n, min(B, n + 4)))
            n = min(B, n + 4)
        dt = time.perf_counter() - t0
        cpu = {"value": n * K / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": "%d of %d requests of workload %s (sample_draft + verify_linear, fp64 C oracle, "
                         "single thread, %.1f s)" % (n, B, args.workload, dt)}

    peak, peak_kind = _peaks()
    # algorithmic bytes: sample_draft reads the draft tensor once; verify_linear reads the
    # verifier tensor once plus, per request, the one draft row of the residual draw
    bytes_sample = B * K * V * esz
    bytes_verify = B * (K + 1) * V * esz + B * V * esz
    gbs_verify = bytes_verify / (t_verify * 1e-3) / 1e9
    gbs_sample = bytes_sample / (t_sample * 1e-3) / 1e9
    bytes_step = (B * (K + 1) + B * K) * V * esz
    value = world * B * K / (ms_step * 1e-3)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if esz == 2 else "f32", "data": "synthetic",
            "config": {"workload": "%s: linear verify B=%d K=%d V=%d %s, T=%g, top-p %g" % (
                args.workload, B, K, V, "bf16" if esz == 2 else "fp32", case.temperature, case.top_p),
                "global_batch": B * world, "block": K, "vocab": V, "parallelism": "replicas x%d" % world,
                "l2": "inputs %.0f MB > 126 MB L2, no flush" % (bytes_step / 1e6),
                "cuda_graph": not args.no_graph},
            "roofline": {"bound": "hbm", "kernel": "psispec_verify_linear", "achieved": gbs_verify, "peak": peak,
                         "unit": "GB/s", "frac": gbs_verify / peak, "peak_kind": peak_kind,
                         "traffic": _traffic(args.workload)},
            "step_gbs": bytes_step / (ms_step * 1e-3) / 1e9,
            "calls": {"sample_draft_ms": t_sample, "sample_draft_gbs": gbs_sample, "verify_linear_ms": t_verify,
                      "verify_linear_gbs": gbs_verify},
            "mean_accept_len": mean_accept,
            "e2e": {"value": world * B * K / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="mid")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch calls directly instead of replaying CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-requests", type=int, default=2)
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
