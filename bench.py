#!/usr/bin/env python
"""Benchmark of the blockwise attention hot path on B200.

One step = one pass of the whole path over one synthetic batch of the
Llama-3-V-like GQA cross-attention workload (B=1, H=32, H_kv=8, d=128,
S_Q=2048, S_KV=65536, n=8 KV blocks, bf16):
  K, V = y W_k, y W_v        (K/V recomputation from the shared visual features)
  partials (O_i, L_i) over the 8 KV blocks, then their merge   (forward)
  D = rowsum(dO o O), dQ, dK, dV from the stored LSE            (backward)

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lvx|reference]

Prints one JSON line (rank 0).  ``value`` is whole-job attention TFLOP/s
over all ranks: the attention FLOPs (forward 4*B*H*S_Q*S_KV*d, backward 2.5x
that) divided by the device time of the attention stages (block partials +
merge, and the backward), summed over the K timed steps and maxed over
ranks.  The K/V recomputation (2*2*B*S_KV*d_embed*H_kv*d) runs in every step
and is reported as its own stage; ``step_tflops`` divides all counted FLOPs
by the whole step.  With N > 1 every rank runs its own batch of the same
shape (weak scaling, no data-path collective).  ``--impl reference`` times
the fp64 CPU oracle on a bounded sample of the same workload.

Peaks: the measured cuBLAS bf16 burst figure for a timed region shorter than
two seconds (the kernels then run near the maximum clock, as the burst GEMM
did), the sustained figure (measured under the power cap) for longer ones.
"""

from __future__ import annotations

import argparse
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

METRIC = "attention fwd+bwd TFLOP/s and % of B200 dense BF16 peak, 1 GPU"
WORKLOAD = "C2"

# ncu DRAM traffic of the dominant kernel per launch, by (workload, stage), with
# the hash of the source file it was taken from (reported only for that
# workload at its full size, and only while the source is unchanged).
TRAFFIC = {
    # bwd_tc_kernel, one full C2 launch under ncu (median of 8): 336.4 MB read + 254.8 MB written
    ("C2", "bwd"): {"bytes": 591.2e6, "source": "blockwise_long_context_b200/csrc/lvx_bwd_tc.cu",
            "sha": "d7ece40cc0620fe0"},
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        mhz = (d.get("clocks_under_load") or {}).get("sm_mhz_median")
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d["bf16_tflops_sustained"],
                    sust_mhz=mhz, src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, sust_mhz=1300.0, src="fallback")


# A timed region at least this long holds the power cap (as the sustained GEMM
# measurement did); a shorter one runs near the maximum clock (as the burst did).
SUSTAINED_AFTER_S = 2.0


def bf16_peak(peaks, timed_s: float):
    """(peak TFLOP/s, description) for a tensor-bound stage timed over ``timed_s`` seconds."""
    if timed_s >= SUSTAINED_AFTER_S:
        return peaks["bf16_sust"], (f"{peaks['src']} sustained cuBLAS bf16 (timed region "
                                    f"{timed_s:.2f} s >= {SUSTAINED_AFTER_S} s; that peak was "
                                    f"measured at a median {peaks['sust_mhz']} MHz)")
    return peaks["bf16"], (f"{peaks['src']} burst cuBLAS bf16 (timed region {timed_s:.2f} s < "
                           f"{SUSTAINED_AFTER_S} s)")


def stats(xs):
    """mean, median, min and max of a list of stage times (ms)."""
    return {"mean": statistics.mean(xs), "median": statistics.median(xs), "min": min(xs),
            "max": max(xs)}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0])); smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[2:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU oracle baseline

def oracle_sample(w, kv_grads: bool = False):
    """Times the fp64 oracle on a bounded sample of the workload's step.

    Sample: the same heads, head width and S_KV, with S_Q cut to ``rows``
    query rows (forward + full textbook backward), plus K/V recomputation of
    ``rows`` rows of y (and, with ``kv_grads``, its gradients over those rows).
    Returns (TFLOP/s of counted work, seconds, description).
    """
    import numpy as np
    import oracle
    from blockwise_long_context_b200 import inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    rows = 32
    keys = w.S_KV if w.S_KV <= 262144 else 65536   # cap for the 15M-key shape
    sw = w.scaled(S_Q=rows, S_KV=keys)
    host = inputs.make(sw, tensors=("q", "k", "v", "do"))
    q, k, v, do = (host[t].double().numpy() for t in ("q", "k", "v", "do"))
    kvw = inputs.make(w, tensors=("w_k", "w_v")) if w.d_embed else None
    t0 = time.perf_counter()
    oracle.attention_fwd(q, k, v, causal=sw.causal)
    flops = sw.fwd_flops()
    if w.backward:
        oracle.attention_bwd(q, k, v, do, causal=sw.causal)
        flops += 2.5 * sw.fwd_flops()
    t_attn = time.perf_counter() - t0
    attn_flops = flops
    if kvw is not None:
        y = np.random.default_rng(0).standard_normal((rows, w.d_embed))
        oracle.kv_recompute(y, kvw["w_k"].double().numpy(), kvw["w_v"].double().numpy())
        flops += 2 * 2 * rows * w.d_embed * w.H_kv * w.d
        if kv_grads:
            g = np.random.default_rng(1).standard_normal((2, rows, w.H_kv * w.d))
            oracle.kv_recompute_bwd(y, kvw["w_k"].double().numpy(), kvw["w_v"].double().numpy(),
                                    g[0], g[1])
            flops += 2 * 2 * 2 * rows * w.d_embed * w.H_kv * w.d
    dt = time.perf_counter() - t0
    desc = (f"fp64 oracle, forward{' + backward' if w.backward else ''} for {rows} of {w.S_Q} "
            f"query rows over all {w.H} heads and "
            f"{'all ' + str(w.S_KV) if keys == w.S_KV else f'the first {keys} of {w.S_KV}'} keys"
            f"{f' (plus K/V recompute of {rows} rows of y' if kvw is not None else ''}"
            f"{' and its gradients' if kv_grads and kvw is not None else ''}"
            f"{', timed apart' if kvw is not None else ''}); attention FLOPs / attention time")
    return attn_flops / t_attn / 1e12, dt, cores, desc


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from blockwise_long_context_b200 import inputs
    w = inputs.WORKLOADS[a.workload]
    kv_grads = a.kv_grads and w.d_embed > 0 and w.backward
    for _ in range(a.warmup):
        oracle_sample(w, kv_grads)
    vals, secs = [], []
    cores, desc = 1, ""
    for _ in range(a.steps):
        v, s, cores, desc = oracle_sample(w, kv_grads)
        vals.append(v); secs.append(s)
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": _config(w, a.gpus, kv_grads),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _input_bytes(w):
    """Bytes of the per-step inputs (bf16 / fp32 as the workload computes)."""
    es = 4 if w.dtype == "f32" else 2
    qo = w.B * w.S_Q * w.H * w.d * es * (2 if w.backward else 1)
    if w.d_embed:
        return qo + (w.B * w.S_KV + 2 * w.H_kv * w.d) * w.d_embed * es
    return qo + 2 * w.B * w.S_KV * w.H_kv * w.d * es


def _config(w, n, kv_grads=False):
    c = {"workload": f"{w.name}: {w.desc}", "B": w.B, "H": w.H, "H_kv": w.H_kv, "d": w.d,
         "S_Q": w.S_Q, "S_KV": w.S_KV, "n_blocks": w.n_blocks, "causal": w.causal,
         "d_embed": w.d_embed, "parallelism": f"replicas{n}" if n > 1 else "single",
         "l2": (f"inputs larger than L2 (126 MB): {_input_bytes(w) / 2**20:.0f} MiB read every step"
                + (", K/V 256 MiB rewritten" if w.d_embed else "")) if _input_bytes(w) > 126e6
               else f"inputs ({_input_bytes(w) / 2**20:.1f} MiB) fit in L2: not a timing workload",
         "flops_counted": "value: attention fwd 4*B*H*S_Q*S_KV*d + bwd 2.5x fwd; step_tflops "
                          "adds the K/V recompute 2*2*B*S_KV*d_embed*H_kv*d"}
    if kv_grads:
        c["kv_grads"] = True
        c["flops_counted"] += " and its gradients dW_k, dW_v, dy (2x the recompute)"
    return c


# ---------------------------------------------------------------- multi-rank helpers

def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank device time over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, steps: int, world: int, ms: float) -> float:
    """Weak scaling: every rank does the same work; the slowest rank sets the time."""
    return world * flops_per_rank_step * steps / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------- GPU arm

def _file_sha(rel):
    p = os.path.join(ROOT, rel)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16] if os.path.exists(p) else None


def run_gpu(a):
    import torch
    import torch.distributed as dist
    from blockwise_long_context_b200 import inputs
    from blockwise_long_context_b200 import binding as lvx

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = inputs.WORKLOADS[a.workload]
    if a.s_kv:
        w = w.scaled(S_KV=a.s_kv)
    peaks = _peaks()

    recompute = w.d_embed > 0   # K, V regenerated from y every step (else they are inputs)
    kv_grads = recompute and w.backward and a.kv_grads   # + dW_k, dW_v, dy of the recomputation
    names = (("q", "do") if w.backward else ("q",)) + (("y", "w_k", "w_v") if recompute else ("k", "v"))
    if _input_bytes(w) > (8 << 30):
        # tens of GB (the VMME shape): drawn on the device, copied once to pinned host memory
        d = inputs.make_device(w, tensors=names, device=dev)
        pinned = {k_: torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t)
                  for k_, t in d.items()}
    else:
        host = inputs.make(w, tensors=names)
        pinned = {k_: t.pin_memory() for k_, t in host.items()}
        d = {k_: t.to(dev) for k_, t in pinned.items()}
    B, S_Q, H, hd = d["q"].shape
    if recompute:
        k = torch.empty(w.B, w.S_KV, w.H_kv, w.d, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
    else:
        k, v = d["k"], d["v"]
    out = torch.empty_like(d["q"])
    lse = torch.empty(B, H, S_Q, dtype=torch.float32, device=dev)
    dq = dk = dv = None
    if w.backward:
        dq = torch.empty_like(d["q"]); dk = torch.empty_like(k); dv = torch.empty_like(k)
    if kv_grads:
        dy = torch.empty_like(d["y"]); dwk = torch.empty_like(d["w_k"]); dwv = torch.empty_like(d["w_v"])
    fws = lvx.fwd_workspace(d["q"], k, w.n_blocks, w.causal)
    bws = lvx.bwd_workspace(d["q"], k, w.causal) if w.backward else None
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev: ev[0].record(stream)
        if recompute:
            lvx.lvx_kv_recompute(d["y"], d["w_k"], d["w_v"], k, v, w.H_kv, w.d)
        if ev: ev[1].record(stream)
        lvx.lvx_attn_fwd(d["q"], k, v, out, lse, w.n_blocks, w.causal, 0.0, fws)
        if ev: ev[2].record(stream)
        if w.backward:
            lvx.lvx_attn_bwd(d["q"], k, v, out, lse, d["do"], dq, dk, dv, w.causal, 0.0, bws)
        if ev: ev[3].record(stream)
        if kv_grads:
            lvx.lvx_kv_recompute_bwd(d["y"], d["w_k"], d["w_v"], dk, dv, dy, dwk, dwv)
        if ev: ev[4].record(stream)

    warm = max(a.warmup, 3)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()

    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(a.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0.record(stream)
    for i in range(a.steps):
        step(stage_ev[i])
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms_total = e0.elapsed_time(e1)
    per = {name: [ev[i].elapsed_time(ev[i + 1]) for ev in stage_ev]
           for i, name in enumerate(("kv", "fwd", "bwd", "kv_bwd"))}
    t_kv, t_fwd, t_bwd, t_kvb = (statistics.mean(per[s_]) for s_ in ("kv", "fwd", "bwd", "kv_bwd"))
    lvx.lvx_last_device_error()

    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / a.steps
    kvb_flops = 2.0 * w.kv_flops() if kv_grads else 0.0
    attn_flops = w.fwd_flops() + w.bwd_flops()
    step_flops = attn_flops + w.kv_flops() + kvb_flops
    # attention stages only (block partials + merge, backward), summed over the
    # timed steps, slowest rank
    ms_attn = max_over_ranks(sum(per["fwd"]) + sum(per["bwd"]), dev)
    value = whole_job_tflops(attn_flops, a.steps, world, ms_attn)
    step_value = whole_job_tflops(step_flops, a.steps, world, ms_total)
    peak_tf, peak_desc = bf16_peak(peaks, ms_total * 1e-3)

    # merge kernel alone (HBM-bound) through the merge entry point: ten back-to-back
    # launches per timing after an L2 flush; the partials they stream (288 MB at C1's
    # shape) are larger than L2, so each launch reads them from HBM again
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    O_p, L_p = lvx.fwd_partials_view(fws, w.n_blocks, w.B, w.H, w.S_Q, w.d)
    mt = []
    for _ in range(5):
        flush.zero_()
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for _ in range(10):
            lvx.lvx_merge_partials(O_p, L_p, out, lse)
        m1.record(stream)
        torch.cuda.synchronize()
        mt.append(m0.elapsed_time(m1) / 10)
    t_merge = statistics.median(mt)
    merge_bytes = w.B * w.H * w.S_Q * (w.n_blocks * (4 * w.d + 4) + (2 * w.d + 4))
    merge_gbs = merge_bytes / (t_merge * 1e-3) / 1e9

    # End to end through the public API with host buffers.  Every step uploads its
    # inputs from pinned host memory and downloads its gradients; the upload of step
    # i+1 (copy stream) and the download of step i-1 (d2h stream) overlap the compute
    # of step i, with two device sets of inputs and outputs.  When a second set of
    # inputs would not fit comfortably (the 62.6 GB VMME shape), one set is used and
    # each upload waits for the previous step's compute.  The timed region spans
    # the first upload through the last download.
    res_names = ("dq", "dk", "dv") if w.backward else ("out",)
    res_dev = {"dq": dq, "dk": dk, "dv": dv, "out": out}
    res_dev_all = dict(res_dev, lse=lse)
    if kv_grads:   # the gradients reaching y and the weights replace dK, dV as results
        res_names = ("dq", "dy", "dwk", "dwv")
        res_dev.update(dy=dy, dwk=dwk, dwv=dwv)
    res_host = {n_: torch.empty(res_dev[n_].shape, dtype=res_dev[n_].dtype).pin_memory()
                for n_ in res_names}
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in res_host.values())
    # enough steps that the first upload and the last download, which nothing overlaps,
    # are a small share of the timed region
    n_e2e = max(3, min(a.steps, 30))
    single = 2 * h2d > 0.4 * torch.cuda.get_device_properties(dev).total_memory
    in_sets = [d, d] if single else [d, {k2: torch.empty_like(t) for k2, t in d.items()}]
    res_keys = ("dq", "dk", "dv", "out", "lse") if w.backward else ("out", "lse")
    out_sets = [{n_: res_dev_all[n_] for n_ in res_keys},
                {n_: torch.empty_like(res_dev_all[n_]) for n_ in res_keys}]
    if kv_grads:
        out_sets[0].update(dy=dy, dwk=dwk, dwv=dwv)
        out_sets[1].update(dy=torch.empty_like(dy), dwk=torch.empty_like(dwk),
                           dwv=torch.empty_like(dwv))

    def run_step(inp, o):
        kk, vv = k, v
        if recompute:
            lvx.lvx_kv_recompute(inp["y"], inp["w_k"], inp["w_v"], k, v, w.H_kv, w.d)
        else:
            kk, vv = inp["k"], inp["v"]
        lvx.lvx_attn_fwd(inp["q"], kk, vv, o["out"], o["lse"], w.n_blocks, w.causal, 0.0, fws)
        if w.backward:
            lvx.lvx_attn_bwd(inp["q"], kk, vv, o["out"], o["lse"], inp["do"], o["dq"], o["dk"],
                             o["dv"], w.causal, 0.0, bws)
        if kv_grads:
            lvx.lvx_kv_recompute_bwd(inp["y"], inp["w_k"], inp["w_v"], o["dk"], o["dv"], o["dy"],
                                     o["dwk"], o["dwv"])

    copy_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, in_free, out_done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def upload(slot):
        with torch.cuda.stream(copy_s):
            for name, t in pinned.items():
                in_sets[slot][name].copy_(t, non_blocking=True)
            in_ready[slot].record(copy_s)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    copy_s.wait_event(x0)
    upload(0)
    for i in range(n_e2e):
        cur = i % 2
        icur = 0 if single else cur
        if not single and i + 1 < n_e2e:
            if i >= 1:
                copy_s.wait_event(in_free[1 - cur])     # step i-1 is done reading that set
            upload(1 - cur)
        stream.wait_event(in_ready[icur])
        if i >= 2:
            stream.wait_event(out_free[cur])            # step i-2's download is done
        run_step(in_sets[icur], out_sets[cur])
        in_free[icur].record(stream)
        out_done[cur].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(out_done[cur])
            for name in res_names:
                res_host[name].copy_(out_sets[cur][name], non_blocking=True)
            out_free[cur].record(d2h_s)
        if single and i + 1 < n_e2e:
            copy_s.wait_event(in_free[0])               # step i is done reading the one set
            upload(0)
    stream.wait_stream(d2h_s)
    stream.wait_stream(copy_s)
    x1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = x0.elapsed_time(x1)
    ms_e2e = max_over_ranks(ms_e2e, dev)
    # the same metric (attention FLOPs) over the whole end-to-end step: copies, K/V
    # recomputation and attention
    e2e_value = whole_job_tflops(attn_flops, n_e2e, world, ms_e2e)

    # roofline of the dominant kernel group, against the peak the timed region's length calls for
    stages = {"bwd": (t_bwd, w.bwd_flops(), "lvx_attn_bwd (preprocess + main + dQ finalize)"),
              "fwd": (t_fwd, w.fwd_flops(), "lvx_attn_fwd (block partials + merge)"),
              "kv": (t_kv, w.kv_flops(), "lvx_kv_recompute"),
              "kv_bwd": (t_kvb, kvb_flops, "lvx_kv_recompute_bwd")}
    stages = {k_: v_ for k_, v_ in stages.items() if v_[1] > 0}
    dom = max(stages, key=lambda s: stages[s][0])
    t_dom, f_dom, dom_desc = stages[dom]
    achieved = f_dom / (t_dom * 1e-3) / 1e12
    tr = None if a.s_kv else TRAFFIC.get((w.name, dom))
    traffic = tr["bytes"] if tr and _file_sha(tr["source"]) == tr["sha"] else None
    # tensor-core dispatch: K/V recompute (1), fwd partials (1) + merge (n_blocks > 1),
    # bwd preprocess + main + dQ finalize (3)
    launches_per_step = (1 if recompute else 0) + 1 + (1 if w.n_blocks > 1 else 0) + \
        (3 if w.backward else 0) + (2 if kv_grads else 0)
    stage_names = {"kv": "kv_recompute", "fwd": "fwd", "bwd": "bwd", "kv_bwd": "kv_recompute_bwd"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": warm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian, shapes of the "
        "pages' Llama-3-V cross-attention workload)",
        "config": _config(w, world, kv_grads),
        "pct_of_peak": 100.0 * value / peak_tf,
        "value_counts": "attention forward (partials + merge) + backward FLOPs over their own "
                        "stage times; the K/V recomputation is the kv_recompute stage",
        "attn_ms_per_step": ms_attn / a.steps,
        "step_tflops": step_value,
        "stages_ms": {stage_names[s_]: stats(per[s_]) for s_ in stages},
        "stage_tflops": {stage_names[s_]: (stages[s_][1] / (stages[s_][0] * 1e-3) / 1e12
                                           if stages[s_][0] else None) for s_ in stages},
        "roofline": {"bound": "tensor", "kernel": dom_desc, "achieved": achieved,
                     "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved / peak_tf, "traffic": traffic,
                     "achieved_from": "algorithmic FLOPs / mean CUDA-event time of the stage over "
                                      "the timed steps",
                     "peak_source": peak_desc + ", MEASURED_PEAKS.json"},
        "merge": {"ms": t_merge, "achieved_gbs": merge_gbs, "peak_gbs": peaks["hbm"],
                  "frac": merge_gbs / peaks["hbm"], "bytes": merge_bytes},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e, "ms_per_step": ms_e2e / n_e2e,
                "counts": "attention FLOPs over the whole step: uploads, K/V recompute, "
                          "attention, downloads",
                "note": ("one input set: each upload follows the previous step's compute" if single
                         else "uploads of step i+1 and downloads of step i-1 overlap step i's compute")},
        "gpu_launches": launches_per_step * a.steps,
        "clocks": clk,
    }
    if world == 1 and rank == 0 and not a.no_cpu_baseline:
        cv, cs, cores, desc = oracle_sample(w, kv_grads)
        line["cpu_baseline"] = {"value": cv, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": cs}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_split(a):
    """LV-XAttn's method across the ranks of the launch (``--split kv``).

    Weak scaling: every rank holds one key/value shard of the workload's size
    (the visual sequence is W * S_KV long) and S_Q / W of the query rows; K and
    V of the shard are recomputed from the rank's shard of y each step.  The
    forward is the ring form (query blocks travel, partials return to their
    owner and merge there, ``distributed.xattn_forward_ring``), the backward
    its gradient (``distributed.xattn_backward_ring``: dQ accumulators travel
    with their blocks, dK/dV stay with the shard).  NCCL carries the
    transfers.  ``value`` is the attention FLOPs of the whole problem
    (4 * B * H * S_Q * W * S_KV * d forward, 2.5x that backward) over the
    max-over-ranks device time of the attention stages."""
    import datetime
    import torch
    import torch.distributed as dist
    from blockwise_long_context_b200 import inputs
    from blockwise_long_context_b200 import binding as lvx
    from blockwise_long_context_b200.distributed import (shard_bounds, xattn_backward_ring,
                                                         xattn_forward_ring)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = inputs.WORKLOADS[a.workload].scaled(backward=True)
    if a.s_kv:
        w = w.scaled(S_KV=a.s_kv)
    qlo, qhi = shard_bounds(w.S_Q, world, rank)
    # this rank's inputs: its query rows and its own key/value shard (seeds offset by rank)
    wr = w.scaled(S_Q=qhi - qlo, index=w.index + 100 * rank)
    recompute = w.d_embed > 0
    d = inputs.make_device(wr, tensors=("q", "do") + (("y", "w_k", "w_v") if recompute
                                                     else ("k", "v")), device=dev)
    if recompute:
        k = torch.empty(w.B, w.S_KV, w.H_kv, w.d, dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
    else:
        k, v = d["k"], d["v"]
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev: ev[0].record(stream)
        if recompute:
            lvx.lvx_kv_recompute(d["y"], d["w_k"], d["w_v"], k, v, w.H_kv, w.d)
        if ev: ev[1].record(stream)
        out, lse = xattn_forward_ring(d["q"], k, v, n_local_blocks=w.n_blocks)
        if ev: ev[2].record(stream)
        grads = xattn_backward_ring(d["q"], k, v, out, lse, d["do"])
        if ev: ev[3].record(stream)
        return grads

    warm = max(a.warmup, 3)
    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(a.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(a.steps):
        step(evs[i])
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    lvx.lvx_last_device_error()
    per = {n_: [ev[i].elapsed_time(ev[i + 1]) for ev in evs] for i, n_ in enumerate(("kv", "fwd", "bwd"))}
    ms_total = max_over_ranks(e0.elapsed_time(e1), dev)
    ms_attn = max_over_ranks(sum(per["fwd"]) + sum(per["bwd"]), dev)
    whole = w.scaled(S_KV=world * w.S_KV)
    attn_flops = whole.fwd_flops() + whole.bwd_flops()
    value = attn_flops * a.steps / (ms_attn * 1e-3) / 1e12
    peaks = _peaks()
    peak_tf, peak_desc = bf16_peak(peaks, ms_total * 1e-3)
    line = {
        "metric": "LV-XAttn attention fwd+bwd TFLOP/s across the ranks (key/value sharded)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps, "warmup": warm,
        "ms_per_step": ms_total / a.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian)",
        "config": {"workload": f"{w.name} per rank: a key/value shard of {w.S_KV} keys, "
                               f"{w.S_Q} query rows over all ranks (ring form)",
                   "B": w.B, "H": w.H, "H_kv": w.H_kv, "d": w.d, "S_Q": w.S_Q,
                   "S_KV_total": world * w.S_KV, "n_local_blocks": w.n_blocks,
                   "d_embed": w.d_embed, "parallelism": f"kv{world}",
                   "l2": "inputs larger than L2 (K/V of the shard recomputed every step)"},
        "pct_of_peak": 100.0 * value / (world * peak_tf),
        "peak_source": peak_desc,
        "stages_ms": {"kv_recompute": stats(per["kv"]), "fwd": stats(per["fwd"]),
                      "bwd": stats(per["bwd"])},
        # per step: K/V GEMM (1), per round the partials (1) and the backward's
        # preprocess, main kernel and dQ finalize (3), and one merge
        "gpu_launches": a.steps * ((1 if recompute else 0) + 4 * world + 1),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_recompute_compare(a):
    """``--recompute-compare``: one training step of the cross-attention layer
    with K, V regenerated from y (LV-XAttn review page, Figure 6), two ways:

      materialised: K, V = y W (whole), forward, backward (dK, dV whole), then
                    dy, dW_k, dW_v from dK, dV (lvx_kv_recompute, lvx_attn_fwd,
                    lvx_attn_bwd, lvx_kv_recompute_bwd);
      block-wise:   lvx_attn_fwd_recompute and lvx_attn_bwd_recompute, which
                    regenerate one key block's K, V at a time in each pass.

    Both produce out, lse, dq, dy and the weight gradients.  Prints the time per
    step of each (CUDA events) and the device bytes each holds beyond the
    inputs and outputs (K, V, dK, dV and workspaces)."""
    import torch
    from blockwise_long_context_b200 import inputs
    from blockwise_long_context_b200 import binding as lvx
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = inputs.WORKLOADS[a.workload].scaled(backward=True)
    if a.s_kv:
        w = w.scaled(S_KV=a.s_kv)
    d = inputs.make_device(w, tensors=("q", "do", "y", "w_k", "w_v"), device=dev)
    q, do, y, wk, wv = d["q"], d["do"], d["y"], d["w_k"], d["w_v"]
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.S_Q, dtype=torch.float32, device=dev)
    dq = torch.empty_like(q)
    dy = torch.empty_like(y)
    # materialised
    k = torch.empty(w.B, w.S_KV, w.H_kv, w.d, dtype=torch.bfloat16, device=dev)
    v, dk, dv = torch.empty_like(k), torch.empty_like(k), torch.empty_like(k)
    dwk, dwv = torch.empty_like(wk), torch.empty_like(wv)
    fws, bws = lvx.fwd_workspace(q, k, w.n_blocks), lvx.bwd_workspace(q, k)
    mat_bytes = 4 * k.numel() * 2 + (fws.numel() if fws is not None else 0) + bws.numel()

    def materialised():
        lvx.lvx_kv_recompute(y, wk, wv, k, v, w.H_kv, w.d)
        lvx.lvx_attn_fwd(q, k, v, out, lse, w.n_blocks, False, 0.0, fws)
        lvx.lvx_attn_bwd(q, k, v, out, lse, do, dq, dk, dv, False, 0.0, bws)
        lvx.lvx_kv_recompute_bwd(y, wk, wv, dk, dv, dy, dwk, dwv)

    rfws, rbws = lvx.recompute_workspaces(q, y, w.H_kv, w.n_blocks)
    dwk32 = torch.empty(wk.shape, dtype=torch.float32, device=dev)
    dwv32 = torch.empty_like(dwk32)
    blk_bytes = rfws.numel() + rbws.numel()

    def blockwise():
        lvx.lvx_attn_fwd_recompute(q, y, wk, wv, out, lse, w.H_kv, w.n_blocks, workspace=rfws)
        lvx.lvx_attn_bwd_recompute(q, y, wk, wv, out, lse, do, dq, dy, dwk32, dwv32, w.H_kv,
                                   w.n_blocks, workspace=rbws)

    res = {}
    clocks = ClockSampler(0)
    clocks.start()
    for name, f in (("materialised", materialised), ("blockwise", blockwise)) * 2:
        for _ in range(max(a.warmup, 3)):
            f()
        torch.cuda.synchronize()
        ts = []
        for _ in range(a.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        res.setdefault(name, []).extend(ts)
    clk = clocks.stop()
    lvx.lvx_last_device_error()
    flops = w.fwd_flops() + w.bwd_flops() + 3 * w.kv_flops()   # K/V once, dy and dW
    flops_blk = flops + w.kv_flops()                            # K/V regenerated in both passes
    line = {
        "metric": "cross-attention training step with K, V recomputed from y: materialised vs "
                  "block-wise regeneration",
        "unit": "ms per step", "higher_is_better": False, "n_gpus": 1, "steps": a.steps,
        "dtype": "bf16", "data": "synthetic (seeded Gaussian)",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} H_kv={w.H_kv} d={w.d} S_Q={w.S_Q} "
                               f"S_KV={w.S_KV} d_embed={w.d_embed} n_blocks={w.n_blocks}"},
        "materialised": {"ms": stats(res["materialised"]), "transient_bytes": mat_bytes,
                         "tflops": flops / (statistics.median(res["materialised"]) * 1e-3) / 1e12,
                         "note": "K, V, dK, dV whole (bf16) + forward and backward workspaces"},
        "blockwise": {"ms": stats(res["blockwise"]), "transient_bytes": blk_bytes,
                      "tflops": flops_blk / (statistics.median(res["blockwise"]) * 1e-3) / 1e12,
                      "note": "one block's K, V, dK, dV (bf16) + partials and dQ accumulator; "
                              "K, V are computed twice (forward and backward)"},
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def run_ring(a):
    """Ring Attention (pass-KV), the busiest rank of a ``--ring W`` ring on one GPU.

    The rank whose chunk pairs hold the most work (with the contiguous layout
    under the causal mask: rank W-1, which computes W-1 full blocks and the
    diagonal; with ``--ring-layout zigzag`` every rank does the same work):
    its chunk-pair partials, their merge and its chunk-pair gradients, with the
    library's kernels, timed with CUDA events.  ``value`` is that rank's
    measured TFLOP/s.  ``projection`` divides the whole problem's FLOPs by the
    busiest rank's time: what W GPUs would reach if the key/value transfers are
    hidden, which ``comm`` checks against the measured 770 GB/s NVLink
    peer-copy bandwidth.  Nothing crosses a GPU boundary in this run."""
    import torch
    from blockwise_long_context_b200 import inputs
    from blockwise_long_context_b200 import binding as lvx
    from blockwise_long_context_b200.ring import (DIAG, SKIP, chunks_of, kernel_block_grad,
                                                  kernel_merge, kernel_partial, pair_mode,
                                                  shard_bounds)
    W, layout = a.ring, a.ring_layout
    w = inputs.WORKLOADS[a.workload].scaled(backward=True, d_embed=0)
    if a.s_kv:
        w = w.scaled(S_KV=a.s_kv, S_Q=a.s_kv if w.causal else w.S_Q)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nC = W if layout == "contiguous" else 2 * W
    qb = [shard_bounds(w.S_Q, nC, c) for c in range(nC)]
    kb = [shard_bounds(w.S_KV, nC, c) for c in range(nC)]
    pair_flops = lambda cq, ck, mode: 3.5 * 4.0 * w.B * w.H * w.d * (
        (qb[cq][1] - qb[cq][0]) * (qb[cq][1] - qb[cq][0] + 1) / 2 if mode == DIAG
        else (qb[cq][1] - qb[cq][0]) * (kb[ck][1] - kb[ck][0]))
    sched = {r: [(st, cq, ck, pair_mode(cq, ck, w.causal)) for st in range(W)
                 for cq in chunks_of(r, W, layout) for ck in chunks_of((r - st) % W, W, layout)]
             for r in range(W)}
    work = {r: sum(pair_flops(cq, ck, m) for _, cq, ck, m in sched[r] if m != SKIP) for r in range(W)}
    r = max(range(W), key=lambda x: work[x])
    pairs = [(st, cq, ck, m) for st, cq, ck, m in sched[r] if m != SKIP]
    d = inputs.make_device(w, tensors=("q", "k", "v", "do"), device=dev)
    cut = lambda t, b: t[:, b[0]:b[1]].contiguous()
    mine = chunks_of(r, W, layout)
    q_c = {c: cut(d["q"], qb[c]) for c in mine}
    do_c = {c: cut(d["do"], qb[c]) for c in mine}
    kv_c = {ck: (cut(d["k"], kb[ck]), cut(d["v"], kb[ck])) for _, _, ck, _ in pairs}
    del d
    partial, grad = kernel_partial(), kernel_block_grad()
    B, H, hd = w.B, w.H, w.d
    slots = {c: W * len(mine) for c in mine}
    o_parts = {c: torch.zeros((slots[c], B, H, q_c[c].shape[1], hd), dtype=torch.float32, device=dev)
               for c in mine}
    l_parts = {c: torch.full((slots[c], B, H, q_c[c].shape[1]), float("-inf"), dtype=torch.float32,
                             device=dev) for c in mine}
    dq = {c: torch.zeros(q_c[c].shape, dtype=torch.float32, device=dev) for c in mine}
    acc = {ck: (torch.zeros(kv[0].shape, dtype=torch.float32, device=dev),
                torch.zeros(kv[1].shape, dtype=torch.float32, device=dev)) for ck, kv in kv_c.items()}

    def rank_step():
        for st, cq, ck, m in pairs:
            slot = st * len(mine) + chunks_of((r - st) % W, W, layout).index(ck)
            partial(q_c[cq], *kv_c[ck], o_parts[cq][slot:slot + 1], l_parts[cq][slot:slot + 1],
                    m == DIAG)
        merged = {c: kernel_merge(q_c[c])(o_parts[c], l_parts[c]) for c in mine}
        for st, cq, ck, m in pairs:
            grad(q_c[cq], *kv_c[ck], merged[cq][0], merged[cq][1], do_c[cq], m == DIAG,
                 dq[cq], acc[ck][0], acc[ck][1])

    for _ in range(max(a.warmup, 3)):
        rank_step()
    torch.cuda.synchronize()
    lvx.lvx_last_device_error()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    e0.record()
    for _ in range(a.steps):
        rank_step()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    lvx.lvx_last_device_error()
    ms = e0.elapsed_time(e1) / a.steps
    total = w.fwd_flops() + w.bwd_flops()
    kv_step_bytes = 2 * B * (w.S_KV // W) * w.H_kv * w.d * 2
    line = {
        "metric": f"Ring Attention fwd+bwd, busiest rank of a {W}-rank ring, on one GPU",
        "value": work[r] / ms / 1e9, "unit": "TFLOP/s", "n_gpus": 1, "steps": a.steps,
        "warmup": max(a.warmup, 3), "ms_per_rank_step": ms, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded Gaussian)",
        "config": {"workload": f"{w.name}: ring of {W} ranks, {layout} layout, rank {r} (the busiest)",
                   "B": w.B, "H": w.H, "H_kv": w.H_kv, "d": w.d, "S_Q": w.S_Q, "S_KV": w.S_KV,
                   "causal": w.causal, "chunk_pairs_computed": len(pairs),
                   "work_balance": min(work.values()) / work[r]},
        "rank_flops": work[r],
        "projection": {"ring_tflops": total / ms / 1e9, "per_gpu_tflops": total / ms / 1e9 / W,
                       "assumes": f"{W} GPUs, key/value transfers hidden behind the compute"},
        "comm": {"kv_bytes_per_step": kv_step_bytes,
                 "ms_per_step_at_770_GBps": kv_step_bytes / 770e9 * 1e3,
                 "compute_ms_per_step": ms / W},
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lvx", choices=["lvx", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-grads", action="store_true",
                    help="also run the gradients of the K/V recomputation (dW_k, dW_v, dy) each step")
    ap.add_argument("--s-kv", type=int, default=0,
                    help="override S_KV (smaller case of the same workload, for profiler captures)")
    ap.add_argument("--ring", type=int, default=0,
                    help="time the busiest rank of a Ring Attention ring of this many ranks (one GPU)")
    ap.add_argument("--ring-layout", default="contiguous", choices=["contiguous", "zigzag"],
                    help="rows per rank: one contiguous shard, or chunks r and 2W-1-r of 2W")
    ap.add_argument("--recompute-compare", action="store_true",
                    help="time a training step with K, V materialised vs regenerated block by block")
    ap.add_argument("--split", default="replicas", choices=["replicas", "kv"],
                    help="replicas: every rank runs its own batch (default); kv: LV-XAttn across "
                         "the ranks, one key/value shard per rank (weak scaling), NCCL exchange")
    a = ap.parse_args()
    if a.impl == "reference":
        run_reference(a)
    elif a.ring:
        run_ring(a)
    elif a.recompute_compare:
        run_recompute_compare(a)
    elif a.split == "kv":
        run_split(a)
    else:
        run_gpu(a)


if __name__ == "__main__":
    main()
