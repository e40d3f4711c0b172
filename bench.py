#!/usr/bin/env python
"""Benchmark: chunkwise causal linear attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl la|reference]
                    [--workload NAME]

One step = one la_fwd_chunk call (the whole hot path: phi, intra-chunk
products, inter-chunk state carry, normaliser, epilogue) over one batch of the
workload, inputs resident in HBM.  Default workload: B=8, H=16, d_k=d_v=128,
T=16384, bf16, gamma_h evenly spaced in [0.9, 0.999], phi=identity, chunk=64,
unnormalised.  The inputs (2.15 GB per step) are larger than L2, so no flush
is needed between steps.

Prints ONE JSON line on rank 0.  Multi-GPU (torchrun, one rank per GPU): every
rank runs its own batch (independent sequences -> weak scaling, no collective
on the data path); the time is the maximum over ranks of the device time.

--impl reference times the float64 CPU oracle (the only reference that
exists) on a bounded prefix sample of the same workload per step, on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "causal linear-attn fwd tokens/s and % of roofline (bf16, B200)"
METRIC_BWD = "causal linear-attn bwd (dq, dk, dv) tokens/s and % of roofline (bf16, B200)"
METRIC_NG = "causal linear-attn fwd + output RMSNorm/Swish gate tokens/s and % of roofline (bf16, B200)"
METRIC_GD = "gated delta rule fwd tokens/s and % of roofline (bf16, B200)"

# forward workloads timed and checked beside the main one in the default run
EXTRA_FWD = ("sweep_T16384", "sweep_T4096", "sweep_T8192", "retnet_d256", "varlen", "long_1m")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clocks / throttle reasons, sampled every 50 ms in a thread."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.samples = []  # (t, sm, smmax, [reason flags])
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            flags = [p.lower().startswith("active") for p in parts[3:7]]
            self.samples.append((time.time(), sm, smax, flags))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        win = [s for s in self.samples if t0 - 0.05 <= s[0] <= t1 + 0.05]
        if not win and self.samples:  # region shorter than the sampling period: nearest samples
            win = sorted(self.samples, key=lambda s: abs(s[0] - 0.5 * (t0 + t1)))[:3]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({n for s in win for n, f in zip(self.NAMES, s[3]) if f})
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": max(s[2] for s in win),
                "reasons": reasons, "samples": len(win)}


def max_over_ranks(values, device, dist_mod=None):
    """Element-wise maximum of a list of floats over all ranks (identity on one rank)."""
    import torch

    if dist_mod is None or not dist_mod.is_initialized() or dist_mod.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate_rate(units_per_rank_per_step, steps, world, max_ms):
    """Whole-job throughput: units every rank processed over the slowest rank's time."""
    return units_per_rank_per_step * steps * world / (max_ms / 1e3)


def rank_seed(rank):
    """Each rank draws its own batch (independent sequences: weak scaling)."""
    return rank


def _algorithmic(w, n_seqs, tokens):
    """Bytes and flops one launch must move / perform (per rank)."""
    e = 2 if w.dtype == "bf16" else 4
    bytes_ = tokens * w.H * e * (2 * w.d_k + 2 * w.d_v) + n_seqs * w.H * w.d_k * w.d_v * 4
    if w.gate is not None:  # the data-dependent log decay, fp32 per token and head
        bytes_ += tokens * w.H * 4
    C = w.chunk
    flops = tokens * w.H * ((C + 1) * (w.d_k + w.d_v) + 4 * w.d_k * w.d_v)
    return bytes_, flops


def _kernel_sources_sha():
    h = hashlib.sha256()
    for fn in ("la_tc.cu", "la_tc_sync.cuh", "la_sm100.cuh", "la_common.cuh"):
        with open(os.path.join(ROOT, "chunkwise_causal_linear_la_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(workload_name, units_scale):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        ent = t["chunk_tc_kernel"]
        if ent.get("source_sha") != _kernel_sources_sha():
            return None
        if ent.get("workload") == workload_name:
            return float(ent["dram_bytes_per_launch"])
        if "dram_bytes_per_unit" in ent:
            return float(ent["dram_bytes_per_unit"]) * units_scale
    except Exception:
        return None
    return None


def _oracle_run(oracle, w, q, k, v, gamma, g=None, bwd=False, beta=None):
    """The oracle's recurrence for workload w (per-head gamma, or the per-token log decay g;
    with beta, the gated delta rule); bwd: its adjoint for an all-ones output gradient."""
    if beta is not None:
        return oracle.gated_delta(q, k, v, g, beta)
    if bwd:
        import torch

        if g is not None:
            return oracle.backward_gated(q, k, v, torch.ones_like(v), g, phi=w.phi)
        if w.normalize:
            return oracle.backward_norm(q, k, v, torch.ones_like(v), gamma, phi=w.phi)
        return oracle.backward(q, k, v, torch.ones_like(v), gamma, phi=w.phi)
    if g is not None:
        return oracle.recurrent_gated(q, k, v, g, phi=w.phi, normalize=w.normalize)[:2]
    return oracle.recurrent(q, k, v, gamma, phi=w.phi, normalize=w.normalize)


def _norm_bwd_terms(oracle, q, k, v, dout, gamma, phi):
    """|numerator| and |denominator| terms of the normalised dq and dk for one (sequence, head):
    the unnormalised adjoints for (v, dout / den) and for (1, e), e_t = -(dout_t . o_t) / den_t."""
    import numpy as np
    import torch

    q, k, v = q.double(), k.double(), v.double()
    ones = torch.ones(v.shape[:3] + (1,), dtype=torch.float64)
    den = torch.from_numpy(oracle.recurrent(q, k, ones, [gamma], phi=phi, normalize=False)[0])
    o = torch.from_numpy(oracle.recurrent(q, k, v, [gamma], phi=phi, normalize=True)[0])
    a = oracle.backward(q, k, v, dout.double() / den, [gamma], phi=phi)
    b = oracle.backward(q, k, ones, -(dout.double() * o).sum(-1, keepdim=True) / den, [gamma], phi=phi)
    return [np.maximum(np.abs(a[0]), np.abs(b[0])), np.maximum(np.abs(a[1]), np.abs(b[1])), None]


def _oracle_rate(w, x, budget_s, max_tokens=None, nseq=1, bwd=False):
    """Time the float64 oracle on a prefix of the first nseq sequences (all heads).

    Returns (tokens/s, tokens per sequence, secs, threads)."""
    import oracle

    oracle.build()
    T = int(x["q"].shape[1]) if w.varlen is None else int(x["cu_seqlens"][1])
    if w.varlen is not None:
        nseq = 1
    q, k, v = (t[:nseq] for t in (x["q"], x["k"], x["v"]))
    gd = x["g"][:nseq] if "g" in x else None
    bd = x["beta"][:nseq] if "beta" in x else None
    g = x["gamma"].double().cpu().numpy()

    def sample(n):
        qs, ks, vs = (t[:, :n].cpu().contiguous() for t in (q, k, v))
        return qs, ks, vs, None if gd is None else gd[:, :n].double().cpu().numpy()

    def run(qs, ks, vs, gs, n):
        b_ = None if bd is None else bd[:, :n].double().cpu().numpy()
        _oracle_run(oracle, w, qs, ks, vs, g, gs, bwd, beta=b_)

    # calibrate on short prefixes (the second sized to about a second), then size the sample to the budget
    n = min(T, 64)
    for target in (1.0, budget_s):
        qs, ks, vs, gs = sample(n)
        t0 = time.perf_counter()
        run(qs, ks, vs, gs, n)
        dt = max(time.perf_counter() - t0, 1e-4)
        n = int(min(T, max(n, n * target / dt)))
    if max_tokens:
        n = min(n, max_tokens)
    qs, ks, vs, gs = sample(n)
    t0 = time.perf_counter()
    run(qs, ks, vs, gs, n)
    secs = time.perf_counter() - t0
    return nseq * n / secs, n, secs, oracle.max_threads()


def run_reference(args):
    """The reference arm: the float64 oracle timed on host cores, rank 0 only."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import torch

    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS[args.workload]
    x = make_inputs(w, seed=0, device="cpu", B=1, T=min(w.T, 4096) if w.varlen is None else None)
    # per step: a prefix sample sized so that all steps fit in about two minutes
    per_step = max(0.02, 120.0 / max(1, args.steps + args.warmup))
    import oracle

    oracle.build()
    _, n, _, threads = _oracle_rate(w, x, per_step)
    q, k, v = (t[:1, :n].contiguous() for t in (x["q"], x["k"], x["v"]))
    g = x["gamma"].double().numpy()
    gs = x["g"][:1, :n].double().numpy() if "g" in x else None
    for _ in range(args.warmup):
        _oracle_run(oracle, w, q, k, v, g, gs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_run(oracle, w, q, k, v, g, gs)
    secs = time.perf_counter() - t0
    value = n * args.steps / secs
    sample = "sequence 0 of %s, all %d heads, first %d tokens per step (float64 recurrence)" % (w.name, w.H, n)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(w, ws),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(w, ws):
    return {
        "workload": w.name, "global_batch": w.B * ws, "seq_len": w.T, "B_per_gpu": w.B, "H": w.H,
        "d_k": w.d_k, "d_v": w.d_v, "chunk": w.chunk, "phi": w.phi, "normalize": w.normalize,
        "gamma": w.gamma_rule or ("per head: %s" % ", ".join("%.6g" % x for x in w.gamma)),
        "parallelism": "dp%d" % ws, "l2": "inputs larger than L2 (no flush needed)",
    }


def _roofline(alg_bytes, alg_flops, launch_ms, hbm_peak, tc_peak):
    """Roofline of one launch: the larger of the HBM time (bytes at the copy peak) and the
    tensor time (flops at the bf16 peak) is the bound; frac = that time / the launch time."""
    t_hbm = alg_bytes / (hbm_peak * 1e9)
    t_tc = alg_flops / (tc_peak * 1e12)
    s = launch_ms / 1e3
    if t_hbm >= t_tc:
        return {"bound": "hbm", "achieved": alg_bytes / s / 1e9, "peak": hbm_peak, "unit": "GB/s",
                "frac": t_hbm / s, "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6}
    return {"bound": "tensor", "achieved": alg_flops / s / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
            "frac": t_tc / s, "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6}


def _slice_err(got, ref):
    import numpy as np

    d = float(np.max(np.abs(ref)))
    e = float(np.max(np.abs(got - ref)))
    return e / d if d > 0 else e


def _fwd_leg(la, w, dev, stream, hbm_peak, tc_peak, nrep=30, warm=5, parity=True):
    """One forward workload other than the timed one: per-launch CUDA events over nrep
    launches of la_fwd_chunk (all its kernels), the roofline, and parity of two full-length
    (sequence, head) slices against the float64 oracle."""
    import torch

    from chunkwise_causal_linear_la_b200.workloads import make_inputs

    x = make_inputs(w, seed=0, device=dev)
    q, k, v, g, cu = x["q"], x["k"], x["v"], x["gamma"], x["cu_seqlens"]
    B, T = q.shape[:2]
    n_seqs = B if cu is None else cu.numel() - 1
    tokens = B * T if cu is None else int(cu[-1])
    out = torch.empty((B, T, w.H, w.d_v), dtype=q.dtype, device=dev)
    fs = torch.empty((n_seqs, w.H, w.d_k, w.d_v), dtype=torch.float32, device=dev)
    nws = la.workspace_size(B, T, w.H, w.d_k, w.d_v, n_seqs, cu is not None, w.chunk, q.dtype)
    wsbuf = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)

    def call():
        la.la_fwd_chunk(q, k, v, g, cu_seqlens=cu, chunk=w.chunk, phi=w.phi, normalize=w.normalize, out=out,
                        final_state=fs, workspace=wsbuf, stream=stream)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nrep)]
    for a_, b_ in ev:
        a_.record(stream)
        call()
        b_.record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a_.elapsed_time(b_) for a_, b_ in ev)
    alg_bytes, alg_flops = _algorithmic(w, n_seqs, tokens)
    res = {"workload": w.name, "ms_per_launch": ms, "tokens_per_s": tokens / (ms / 1e3), "tokens": tokens,
           "launches_per_call": (2 if cu is not None else 3) if nws > 0 else 1, "timed_calls": nrep,
           "roofline": dict(_roofline(alg_bytes, alg_flops, ms, hbm_peak, tc_peak),
                            alg_bytes_per_launch=alg_bytes, alg_flops_per_launch=alg_flops),
           "config": _config(w, 1)}
    if parity:
        import oracle

        oracle.build()
        if cu is None:
            sl = [(0, 0, T, 0), (B - 1, 0, T, w.H - 1)]
            fidx = lambda b: b  # noqa: E731
        else:
            lens = (cu[1:] - cu[:-1]).tolist()
            nl = max(range(n_seqs), key=lambda m: lens[m])
            sl = [(0, int(cu[0]), int(cu[1]), 0), (0, int(cu[nl]), int(cu[nl + 1]), w.H - 1)]
            seqs = [0, nl]
        worst, names = 0.0, []
        for m, (b, s0, e0, h) in enumerate(sl):
            cut = lambda t: t[b:b + 1, s0:e0, h:h + 1].cpu()  # noqa: E731
            ref, fref = oracle.recurrent(cut(q), cut(k), cut(v), [float(g[h])], phi=w.phi, normalize=w.normalize)
            n_ = fidx(b) if cu is None else seqs[m]
            worst = max(worst, _slice_err(cut(out).double().numpy(), ref),
                        _slice_err(fs[n_:n_ + 1, h:h + 1].double().cpu().numpy(), fref))
            names.append("(sequence %d, head %d, %d tokens)" % (n_, h, e0 - s0))
        res["parity"] = {"max_rel_err": worst, "tolerance": 2e-2 if w.dtype == "bf16" else 1e-4,
                         "slices": ", ".join(names) + " vs float64 oracle, outputs and final states"}
    del x, q, k, v, out, fs, wsbuf
    torch.cuda.empty_cache()
    return res


def _decode_leg(la, dev, stream, hbm_peak, rank, nrep=400, norm=False, delta=False, check=False):
    """Times la_step (norm: la_step_norm, which also carries z; delta: one token of
    the gated delta rule, la_fwd_gated_delta with the state updated in place) on the
    decode workload: per-launch CUDA events, four state batches used in turn so that
    each step's 67 MB state was last touched three steps (~200 MB of traffic)
    earlier and is not served from the 126 MB L2."""
    import torch

    from chunkwise_causal_linear_la_b200.workloads import DECODE, make_decode_inputs

    d = make_decode_inputs(DECODE["N"], DECODE["H"], DECODE["d_k"], DECODE["d_v"], DECODE["scale"],
                           DECODE["state_std"], DECODE["gamma"], seed=rank, device=dev)
    states = [d["state"]] + [d["state"].clone() for _ in range(3)]
    st = states[0]
    dq, dk_, dv_, dg = d["q"], d["k"], d["v"], d["gamma"]
    do = torch.empty_like(dv_)
    phi = "elu1" if norm else DECODE["phi"]
    zs = [torch.ones(st.shape[:3], dtype=torch.float32, device=dev) for _ in range(4)] if norm else None

    if delta:  # [N, 1, H, d] views, per-(sequence, head) log decay and write strength
        q4, k4, v4, o4 = dq.unsqueeze(1), dk_.unsqueeze(1), dv_.unsqueeze(1), do.unsqueeze(1)
        lg = torch.log(dg).reshape(1, 1, -1).expand(dq.shape[0], 1, -1).contiguous()
        bt = torch.full_like(lg, 0.5)

    def call(i):
        if delta:
            la.la_fwd_gated_delta(q4, k4, v4, lg, bt, initial_state=states[i % 4], out=o4,
                                  final_state=states[i % 4], stream=stream)
        elif norm:
            la.la_step_norm(dq, dk_, dv_, dg, states[i % 4], zs[i % 4], out=do, phi=phi, stream=stream)
        else:
            la.la_step(dq, dk_, dv_, dg, states[i % 4], out=do, phi=phi, stream=stream)

    # parity first: one call on state batch 0 against the oracle's step from the same state
    parity = None
    if check:
        import numpy as np

        import oracle

        oracle.build()
        st0 = states[0].double().cpu().numpy()
        z0 = zs[0].double().cpu().numpy() if norm else None
        call(0)
        torch.cuda.synchronize()
        if delta:
            ref, fref = oracle.gated_delta(dq.unsqueeze(1).cpu(), dk_.unsqueeze(1).cpu(), dv_.unsqueeze(1).cpu(),
                                           lg.double().cpu().numpy(), bt.double().cpu().numpy(), init=st0)
            ref = ref[:, 0]
        elif norm:
            ref, fref, _ = oracle.step_norm(dq.cpu(), dk_.cpu(), dv_.cpu(), dg.double().cpu().numpy(), st0, z0,
                                            phi=phi)
        else:
            ref, fref = oracle.step(dq.cpu(), dk_.cpu(), dv_.cpu(), dg.double().cpu().numpy(), st0, phi=phi)
        got_o = do.double().cpu().numpy()
        got_s = states[0].double().cpu().numpy()
        e_o = max(_slice_err(got_o[n_, h_], ref[n_, h_]) for n_ in range(ref.shape[0]) for h_ in range(ref.shape[1]))
        e_s = max(_slice_err(got_s[n_, h_], fref[n_, h_]) for n_ in range(ref.shape[0])
                  for h_ in range(ref.shape[1]))
        parity = {"max_rel_err_out": e_o, "max_rel_err_state": e_s, "tolerance": 1e-4,
                  "slices": "every (sequence, head) of one call, fp32, vs the float64 oracle's step"}
        del st0, got_s, fref
    for i in range(12):
        call(i)
    torch.cuda.synchronize()
    evd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nrep)]
    for i in range(nrep):
        evd[i][0].record(stream)
        call(i)
        evd[i][1].record(stream)
    torch.cuda.synchronize()
    us = statistics.mean(a.elapsed_time(b) for a, b in evd) * 1e3
    dbytes = 2 * st.numel() * 4 + (dq.numel() + dk_.numel() + dv_.numel() + do.numel()) * 4
    if norm:
        dbytes += 2 * zs[0].numel() * 4
    if delta:
        dbytes += 2 * lg.numel() * 4
    name = DECODE["name"] + ("_normalised" if norm else "") + ("_gated_delta" if delta else "")
    return {"workload": name, "us_per_step": us, "alg_bytes": dbytes,
            "achieved_gbs": dbytes / (us / 1e6) / 1e9, "peak_gbs": hbm_peak,
            "frac": dbytes / (us / 1e6) / 1e9 / hbm_peak, "kernel": "delta_kernel" if delta else "step_kernel",
            "launches": nrep, "parity": parity,
            "note": "per-launch CUDA events; four state batches in rotation (L2-cold)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="la", choices=["la", "reference"])
    ap.add_argument("--workload", default="sweep_T16384")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--normgate", action="store_true",
                    help="forward with the output RMSNorm and Swish gate (la_fwd_chunk_normgate)")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward (la_bwd_chunk) on the workload instead of the forward")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode step (la_step) and print its JSON object")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import chunkwise_causal_linear_la_b200 as la
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    ws, rank, local = _dist()
    if ws != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, ws))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    hbm_peak, tc_peak, peak_kind = _peaks()
    stream = torch.cuda.current_stream()
    if args.decode_only:
        res = _decode_leg(la, dev, stream, hbm_peak, rank, nrep=max(args.steps, 1))
        resn = _decode_leg(la, dev, stream, hbm_peak, rank, nrep=max(args.steps, 1), norm=True)
        resd = _decode_leg(la, dev, stream, hbm_peak, rank, nrep=max(args.steps, 1), delta=True)
        if rank == 0:
            print(json.dumps({"impl": "la", "decode": res, "decode_norm": resn, "decode_gated_delta": resd,
                              "peak_kind": peak_kind}), flush=True)
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    w = WORKLOADS[args.workload]
    x = make_inputs(w, seed=rank_seed(rank), device=dev)
    q, k, v, g, cu = x["q"], x["k"], x["v"], x["gamma"], x["cu_seqlens"]
    B, T = q.shape[:2]
    n_seqs = B if cu is None else cu.numel() - 1
    tokens = B * T if cu is None else int(cu[-1])
    out = torch.empty((B, T, w.H, w.d_v), dtype=q.dtype, device=dev)
    fs = torch.empty((n_seqs, w.H, w.d_k, w.d_v), dtype=torch.float32, device=dev)
    nws = la.workspace_size(B, T, w.H, w.d_k, w.d_v, n_seqs, cu is not None, w.chunk, q.dtype)
    wsbuf = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)

    gd = x.get("g")  # data-dependent log decay (gated workloads)
    if args.bwd:
        if x.get("beta") is not None or (w.normalize and gd is not None) or w.dtype != "bf16" and w.normalize:
            raise SystemExit("--bwd covers the per-head-decay forwards (normalised in bf16) and the "
                             "unnormalised per-token decay")
        from chunkwise_causal_linear_la_b200.workloads import make_dout

        dout = make_dout(v, seed=rank_seed(rank))
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        if gd is not None:  # the per-token decay's backward also returns dg
            grads = grads + (torch.empty_like(gd),)
        if w.normalize:  # the normalised backward keeps [v, 1, 1], [u, e_hi, e_lo] and phi(k) in its workspace
            nws = la.bwd_norm_workspace_size(B, T, w.H, w.d_k, w.d_v, w.chunk, q.dtype)
            wsbuf = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)

    if args.normgate:
        if gd is not None or args.bwd:
            raise SystemExit("--normgate covers the per-head-decay forward")
        from chunkwise_causal_linear_la_b200.workloads import make_norm_gate

        ng_gate, ng_w = make_norm_gate(v, seed=rank_seed(rank))

    gbeta = x.get("beta")  # gated delta rule workloads
    if gbeta is not None:  # the chunked (WY) path keeps W and T diag(beta) V in its workspace
        nws = la.gated_delta_workspace_size(B, T, w.H, w.d_k, w.d_v, n_seqs, cu is not None, q.dtype)
        wsbuf = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)

    def step():
        if gbeta is not None:
            la.la_fwd_gated_delta_chunk(q, k, v, gd, gbeta, cu_seqlens=cu, out=out, final_state=fs,
                                        workspace=wsbuf, stream=stream)
        elif args.normgate:
            la.la_fwd_chunk_normgate(q, k, v, g, ng_gate, ng_w, eps=1e-5, cu_seqlens=cu, chunk=w.chunk, phi=w.phi,
                                     normalize=w.normalize, out=out, final_state=fs, workspace=wsbuf, stream=stream)
        elif args.bwd and gd is not None:
            la.la_bwd_chunk_gated(q, k, v, dout, gd, cu_seqlens=cu, chunk=w.chunk, phi=w.phi, dq=grads[0],
                                  dk=grads[1], dv=grads[2], dg=grads[3], stream=stream)
        elif args.bwd and w.normalize:
            la.la_bwd_chunk_norm(q, k, v, dout, g, cu_seqlens=cu, chunk=w.chunk, phi=w.phi, dq=grads[0],
                                 dk=grads[1], dv=grads[2], workspace=wsbuf, stream=stream)
        elif args.bwd:
            la.la_bwd_chunk(q, k, v, dout, g, cu_seqlens=cu, chunk=w.chunk, phi=w.phi, dq=grads[0], dk=grads[1],
                            dv=grads[2], stream=stream)
        elif gd is not None:
            la.la_fwd_chunk_gated(q, k, v, gd, cu_seqlens=cu, chunk=w.chunk, phi=w.phi, normalize=w.normalize,
                                  out=out, final_state=fs, workspace=wsbuf, stream=stream)
        else:
            la.la_fwd_chunk(q, k, v, g, cu_seqlens=cu, chunk=w.chunk, phi=w.phi, normalize=w.normalize,
                            out=out, final_state=fs, workspace=wsbuf, stream=stream)

    def barrier():
        if ws > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.get_device_properties(dev).uuid and
                           "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)).start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_wall0 = time.time()
    e_all0, e_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_all0.record(stream)
    for i in range(args.steps):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    e_all1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    torch.cuda.synchronize()
    time.sleep(0.1)
    sampler.stop()
    elapsed_ms, launch_ms = max_over_ranks(
        [e_all0.elapsed_time(e_all1), statistics.mean(a.elapsed_time(b) for a, b in evs)], dev, dist)
    value = aggregate_rate(tokens, args.steps, ws, elapsed_ms)
    alg_bytes, alg_flops = _algorithmic(w, n_seqs, tokens)
    if gbeta is not None:  # beta is read too
        alg_bytes += tokens * w.H * 4
    if args.normgate:  # the gate is read too
        alg_bytes += tokens * w.H * (2 if w.dtype == "bf16" else 4) * w.d_v
    if args.bwd:  # read q, k, v, dout; write dq, dk, dv (no final state); three forward-shaped passes of flops
        e_ = 2 if w.dtype == "bf16" else 4
        alg_bytes = tokens * w.H * e_ * (4 * w.d_k + 3 * w.d_v)
        if gd is not None:  # read g, write dg (fp32 per token and head)
            alg_bytes += tokens * w.H * 8
        alg_flops = 3 * alg_flops
    roof = _roofline(alg_bytes, alg_flops, launch_ms, hbm_peak, tc_peak)
    # kernels launched per step: segmented sequences take a state pass, a scan and the output pass
    # (a packed batch with a workspace has its longest-first order computed first: 2 launches)
    # (backward: three tensor-core passes, two phi copies with elu + 1, and with a per-token decay the
    # reverse cumulative sum of dg, whose row terms the passes' epilogues add; the normalised backward
    # adds [v, 1, 1], the forward of the widened values and the [u, e] row pass)
    launches_per_step = (5 if w.phi == "elu1" else 3) if args.bwd else (
        (2 if cu is not None else 3) if nws > 0 else 1)
    if args.bwd and gd is not None:
        launches_per_step += 1
    if args.bwd and w.normalize:
        launches_per_step += 3
    if gbeta is not None:  # chunk offsets (packed batches), the per-chunk WY pass, the sequential pass
        launches_per_step = (3 if cu is not None else 2) if nws > 0 else 1
    clocks = sampler.summary(t_wall0, t_wall1)

    # ---- parity on sampled (sequence, head) slices, float64 oracle (rank 0)
    parity = None
    if rank == 0 and not args.no_extra:
        import numpy as np

        import oracle

        oracle.build()
        torch.cuda.synchronize()
        sl = [(0, 0), (B - 1, w.H - 1)] if cu is None else [(0, 0)]
        worst = 0.0
        for b, h in sl if args.bwd else []:  # backward: dq, dk, dv against the oracle's adjoint
            s0, e0_ = (0, T) if cu is None else (int(cu[0]), int(cu[1]))
            bb = b if cu is None else 0
            cut = lambda t: t[bb:bb + 1, s0:e0_, h:h + 1].cpu()  # noqa: E731
            if gd is not None:
                refs = oracle.backward_gated(cut(q), cut(k), cut(v), cut(dout),
                                             gd[bb:bb + 1, s0:e0_, h:h + 1].double().cpu().numpy(), phi=w.phi)
            elif w.normalize:
                refs = oracle.backward_norm(cut(q), cut(k), cut(v), cut(dout), [float(g[h])], phi=w.phi)
            else:
                refs = oracle.backward(cut(q), cut(k), cut(v), cut(dout), [float(g[h])], phi=w.phi)
            # the normalised dq, dk are differences of a numerator and a denominator term that
            # cancel: their error is measured against the larger of the two as well
            terms = (_norm_bwd_terms(oracle, cut(q), cut(k), cut(v), cut(dout), float(g[h]), w.phi)
                     if w.normalize else [None, None, None])
            for got, ref, sc in zip(grads, refs, terms):
                o = (cut(got) if got.dim() == 4 else got[bb:bb + 1, s0:e0_, h:h + 1].cpu()).double().numpy()
                den = np.max(np.abs(ref)) if sc is None else max(np.max(np.abs(ref)), np.max(sc))
                worst = max(worst, float(np.max(np.abs(o - ref)) / den))
        for b, h in [] if args.bwd else sl:
            if cu is None:
                qs, ks, vs = (t[b:b + 1, :, h:h + 1].cpu() for t in (q, k, v))
                gs = None if gd is None else gd[b:b + 1, :, h:h + 1].double().cpu().numpy()
                bs = None if gbeta is None else gbeta[b:b + 1, :, h:h + 1].double().cpu().numpy()
                ref, fref = _oracle_run(oracle, w, qs, ks, vs, [float(g[h])], gs, beta=bs)
                if args.normgate:
                    ref = oracle.norm_gate(ref, ng_gate[b:b + 1, :, h:h + 1].cpu(), ng_w.double().cpu().numpy())
                o = out[b:b + 1, :, h:h + 1].float().cpu().numpy()
                f = fs[b:b + 1, h:h + 1].cpu().numpy()
            else:
                s, e = int(cu[0]), int(cu[1])
                qs, ks, vs = (t[:, s:e, h:h + 1].cpu() for t in (q, k, v))
                gs = None if gd is None else gd[:, s:e, h:h + 1].double().cpu().numpy()
                bs = None if gbeta is None else gbeta[:, s:e, h:h + 1].double().cpu().numpy()
                ref, fref = _oracle_run(oracle, w, qs, ks, vs, [float(g[h])], gs, beta=bs)
                o = out[:, s:e, h:h + 1].float().cpu().numpy()
                f = fs[0:1, h:h + 1].cpu().numpy()
            worst = max(worst, float(np.max(np.abs(o - ref)) / np.max(np.abs(ref))),
                        float(np.max(np.abs(f - fref)) / np.max(np.abs(fref))))
        parity = {"max_rel_err": worst, "tolerance": 2e-2 if w.dtype == "bf16" else 1e-4,
                  "slices": "(sequence, head) = %s vs float64 oracle, full length" % sl}

    # ---- end to end: pinned host buffers, copies inside the timed region.  The plain forward
    # goes through the C-ABI call that takes host buffers (la_fwd_chunk_host: copies in, forward,
    # copies out, one stream); the other legs copy through torch around their device call.
    plain = not (args.bwd or args.normgate or gbeta is not None or gd is not None)
    inputs = (q, k, v) if gd is None else (q, k, v, gd)
    if gbeta is not None:
        inputs = (q, k, v, gd, gbeta)
    if args.normgate:
        inputs = (q, k, v, ng_gate)
    if args.bwd:
        inputs = (q, k, v, dout) if gd is None else (q, k, v, dout, gd)
    if plain:
        inputs = (q, k, v, g) + (() if cu is None else (cu,))
    outputs = grads if args.bwd else (out, fs)
    hosts = [t.cpu().pin_memory() for t in inputs]
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outputs]
    if plain:
        arena = torch.empty(la.host_arena_size(B, T, w.H, w.d_k, w.d_v, n_seqs, cu is not None, w.chunk, q.dtype),
                            dtype=torch.uint8, device=dev)

    def e2e_step():
        if plain:
            la.la_fwd_chunk_host(hosts[0], hosts[1], hosts[2], hosts[3], cu_seqlens=hosts[4] if cu is not None else None,
                                 chunk=w.chunk, phi=w.phi, normalize=w.normalize, out=host_out[0],
                                 final_state=host_out[1], arena=arena, stream=stream)
            return
        for dst, src in zip(inputs, hosts):
            dst.copy_(src, non_blocking=True)
        step()
        for dst, src in zip(host_out, outputs):
            dst.copy_(src, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], dev, dist)
    h2d = sum(t.numel() * t.element_size() for t in inputs)
    d2h = sum(t.numel() * t.element_size() for t in outputs)
    e2e = {"value": aggregate_rate(tokens, args.e2e_steps, ws, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
           "call": "la_fwd_chunk_host (C ABI, host buffers)" if plain else "torch copies around the device call"}

    # ---- CPU baseline: the float64 oracle on host cores, rank 0 at N=1 only
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        nseq = 1 if cu is not None else B
        rate, n, secs, threads = _oracle_rate(w, x, budget_s=15.0, nseq=nseq, bwd=args.bwd)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": "%d sequence(s) of %s, all %d heads, first %d tokens each (float64 %s, %.1f s)"
                         % (nseq, w.name, w.H, n, "adjoint of the recurrence" if args.bwd else "recurrence", secs)}

    # ---- decode step (la_step), HBM-bound: achieved GB/s
    extra = {}
    if not args.no_extra:
        chk = rank == 0
        extra["decode"] = _decode_leg(la, dev, stream, hbm_peak, rank, check=chk)
        extra["decode_norm"] = _decode_leg(la, dev, stream, hbm_peak, rank, norm=True, check=chk)
        extra["decode_gated_delta"] = _decode_leg(la, dev, stream, hbm_peak, rank, delta=True, check=chk)
        # the other forward workloads, each timed and checked on its own (one GPU only: the
        # multi-GPU run times the main workload alone)
        if ws == 1 and not (args.bwd or args.normgate or gbeta is not None or gd is not None):
            del out, fs, wsbuf, hosts, host_out, arena
            del x, q, k, v
            torch.cuda.empty_cache()
            for name in EXTRA_FWD:
                if WORKLOADS[name].name == w.name:
                    continue
                extra[name] = _fwd_leg(la, WORKLOADS[name], dev, stream, hbm_peak, tc_peak,
                                       nrep=20 if name == "long_1m" else 30)

    if rank == 0:
        line = {
            "metric": METRIC_BWD if args.bwd else (METRIC_NG if args.normgate else (
                METRIC_GD if gbeta is not None else METRIC)), "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": str(w.dtype), "data": "synthetic",
            "config": _config(w, ws),
            "roofline": {"bound": roof["bound"], "achieved": roof["achieved"], "peak": roof["peak"],
                         "unit": roof["unit"], "frac": roof["frac"],
                         "t_hbm_us": roof["t_hbm_us"], "t_tensor_us": roof["t_tensor_us"],
                         "traffic": None if (args.bwd or args.normgate or gbeta is not None) else
                         _traffic(w.name, 1.0),
                         "peak_kind": "%s (burst: %s)" % (peak_kind, "copy bandwidth" if roof["bound"] == "hbm"
                                                          else "cuBLAS bf16 GEMM"),
                         "alg_bytes_per_launch": alg_bytes, "alg_flops_per_launch": alg_flops,
                         "launch_ms": launch_ms,
                         # the launch time scaled to the maximum SM clock by the median sampled clock, so that
                         # settling under the power cap shows (time x median MHz / max MHz)
                         "launch_ms_at_max_clock": (launch_ms * clocks["sm_mhz"] / clocks["sm_max_mhz"]
                                                    if clocks.get("sm_mhz") and clocks.get("sm_max_mhz") else None),
                         "kernel": ("chunk_tc_kernel (4 passes: forward of [v, 1, 1], forward + 2 in reverse time)"
                                    if w.normalize else "chunk_tc_kernel (3 passes: forward + 2 in reverse time)")
                         if args.bwd
                         else ("gdn_prep_kernel + gdn_tc_kernel (whole step)" if gbeta is not None
                               else "chunk_tc_kernel")},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps * launches_per_step, "clocks": clocks,
            "parity": parity, "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
