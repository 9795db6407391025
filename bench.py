#!/usr/bin/env python
"""Benchmark of the SATA attention hot path (prefill + decode, d_K = d_V = 64, P = 4).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  ``value`` is prefill throughput in tokens/s summed
over all ranks on the long bf16 prefill (B=1, H=8, N=16384): one step is one
``sata_prefill`` call (basis tables, feature expansion, chunk states, readout,
normalisation, final state).  The ``decode`` object reports the batched
decode workload (B=32, H=8, state of an N=8192 bf16 prefill): one step is one
``sata_decode_step`` call for all 32 sequences.  Inputs are seeded synthetic
N(0,1) (``sata_inputs``).  Timing: CUDA events on the launching stream; prefill
steps are separated by an L2 flush (a 256 MiB write) outside the events; the
decode state (3.19 GB) is larger than L2.  Multi-GPU runs are weak scaling:
every rank processes its own independent batch of heads, no collective on the
data path; times are the max over ranks.
``--impl reference`` times the fp64 CPU oracle on the host cores instead (a
bounded sample of the same workloads, reported in the same unit).
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

METRIC = "tokens/sec/GPU (prefill & decode) at d_K=64,P=4; % tensor / HBM roofline"
PREFILL = dict(B=1, H=8, N=16384, dK=64, dV=64, P=4)
PREFILL_DK32 = dict(B=4, H=8, N=4096, dK=32, dV=32, P=4)
DECODE = dict(B=32, H=8, N=8192, dK=64, dV=64, P=4)
WORKLOAD = ("prefill B=1,H=8,N=16384,dK=dV=64,P=4 bf16 (one sata_prefill per step); "
            "decode B=32,H=8,dK=dV=64,P=4 fp32 state of an N=8192 bf16 prefill "
            "(one sata_decode_step per step)")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


def basis_m(dK, P):
    return math.comb(dK + P - 1, P - 1)


def alg_one(w, m):
    """Algorithmic flops of one of the two state contractions for workload w:
    B*H*N tokens x 2 (dV+1) m."""
    return w["B"] * w["H"] * w["N"] * 2 * (w["dV"] + 1) * m


# --------------------------------------------------------------- clocks sampler
class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        mhz, mx, reasons = [], [], set()
        for r in self.rows:
            try:
                mhz.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [x for x in mhz if x > 0.5 * max(mhz)] or mhz
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------- traffic record
def traffic_record(kernel: str):
    """Per-launch DRAM bytes of ``kernel`` from the committed ncu summary, or
    None when the kernel's source files changed since the counters were taken
    (the record lists them; the hash covers their names and contents)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    r = rec.get(kernel)
    if not r or r.get("source_sha") != source_sha(r.get("sources")):
        return None
    return r.get("bytes_per_launch")


def source_sha(files=None) -> str:
    """sha256 prefix over the named files of the CUDA sources (all of them
    when ``files`` is None), in sorted order."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_cost_attention_b200", "csrc")
    for name in sorted(files if files else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------- oracle timing
def oracle_prefill_sample(n: int, seed: int = 0):
    """The fp64 oracle on a bounded sample of the prefill workload: its
    quadratic form (``oracle.quadratic_form``) over the first ``n`` tokens of
    one head, then the final state (``oracle.final_state``) of those tokens.
    Returns (seconds, tokens of the whole workload the same work is worth):
    the quadratic form's cost grows with the number of (query, key) pairs, so
    n tokens of one head are worth n(n+1)/2 of the H*N(N+1)/2 pairs; the
    state's cost grows with the tokens (n of H*N)."""
    import oracle
    from sata_inputs import make_qkv

    w = PREFILL
    q, k, v = make_qkv(1, 1, n, w["dK"], w["dV"], seed=seed, dtype="bf16")
    t0 = time.perf_counter()
    oracle.quadratic_form(q, k, v, w["P"])
    t1 = time.perf_counter()
    oracle.final_state(k, v, w["P"])
    t2 = time.perf_counter()
    full_pairs = w["H"] * w["N"] * (w["N"] + 1) / 2
    full_tokens = w["B"] * w["H"] * w["N"]
    t_full = (t1 - t0) * full_pairs / (n * (n + 1) / 2) + (t2 - t1) * full_tokens / n
    return t2 - t0, w["B"] * w["N"] * (t2 - t0) / t_full


def oracle_decode_sample(heads: int, seed: int = 1):
    """``oracle.decode_step`` on `heads` heads from a random state.  Returns
    (seconds, equivalent tokens of the B=32,H=8 step)."""
    import numpy as np

    import oracle

    w = DECODE
    r = np.random.default_rng(seed)
    m = basis_m(w["dK"], w["P"])
    S = r.standard_normal((1, heads, m, w["dV"] + 1))
    qv = r.standard_normal((1, heads, w["dK"]))
    kv = r.standard_normal((1, heads, w["dK"]))
    vv = r.standard_normal((1, heads, w["dV"]))
    t0 = time.perf_counter()
    oracle.decode_step(qv, kv, vv, S, w["P"])
    dt = time.perf_counter() - t0
    return dt, heads / w["H"]


def host_threads() -> dict:
    """Host cores available to this process, and the threads numpy's BLAS
    pool uses (the oracle's matrix products run there)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    blas = 1
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        blas = max(int(i.get("num_threads", 1)) for i in info) if info else 1
    except Exception:
        pass
    return {"cores": cores, "numpy_threads": blas}


def cpu_baseline(budget_s: float = 20.0):
    oracle_prefill_sample(256)  # first-call set-up (thread pools, tables) untimed
    n = 2048
    dt, tok = oracle_prefill_sample(n)
    while dt < budget_s * 0.25 and n < PREFILL["N"]:
        n = min(PREFILL["N"], n * 2)
        dt, tok = oracle_prefill_sample(n)
    ddt, dtok = oracle_decode_sample(2)
    th = host_threads()
    return {"value": tok / dt, "unit": "tokens/s", "cores": th["cores"],
            "numpy_threads": th["numpy_threads"], "kind": "oracle",
            "sample": f"prefill: oracle.quadratic_form + oracle.final_state on the first {n} "
                      f"tokens of 1 of the 8 heads (fp64 numpy, {dt:.1f} s), scaled to the "
                      f"workload by (query, key) pairs and by tokens respectively",
            "decode": {"value": dtok / ddt, "unit": "tokens/s",
                       "sample": f"oracle.decode_step on 2 of the 256 heads from a random "
                                 f"state, {ddt:.2f} s"}}


# --------------------------------------------------------------- ranks
def dist_barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def dist_max(x: float, world: int, device=None) -> float:
    """Max of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, steps: int, units_per_step_per_rank: float,
                       max_total_ms: float) -> float:
    """Whole-job throughput: every rank processes its own units each step."""
    return world * steps * units_per_step_per_rank / (max_total_ms / 1e3)


# --------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import linear_cost_attention_b200 as sata
    from sata_inputs import DecodeStream, make_qkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pk = peaks()
    stream = torch.cuda.current_stream()

    def barrier():
        dist_barrier(world)

    def max_over_ranks(x: float) -> float:
        return dist_max(x, world, dev)

    vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    phys = vis[local_rank] if local_rank < len(vis) else str(local_rank)
    sampler = ClockSampler(int(phys) if phys.strip().isdigit() else local_rank)

    # ---------------- prefill
    w = PREFILL
    m = basis_m(w["dK"], w["P"])
    q, k, v = make_qkv(w["B"], w["H"], w["N"], w["dK"], w["dV"], seed=20261204 + 1000 * rank,
                       dtype="bf16")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty(w["B"], w["H"], w["N"], w["dV"], device=dev)
    state = torch.empty(w["B"], w["H"], m, w["dV"] + 1, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def prefill():
        sata.sata_prefill(qd, kd, vd, out, state, w["B"], w["H"], w["N"], w["dK"], w["dV"],
                          w["P"], torch.bfloat16, stream)

    for _ in range(args.warmup):
        prefill()
    torch.cuda.synchronize()
    sata.sata_profile_enable(True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    kern = {}
    launches = 0
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        prefill()
        ev[i][1].record(stream)
        prof = sata.sata_profile_read()  # syncs on this step's kernel events
        launches += len(prof)
        for name, ms in prof:
            kern.setdefault(name, []).append(ms)
    torch.cuda.synchronize()
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms))
    prefill_tokens = w["B"] * w["N"]
    value = weak_scaling_value(world, args.steps, prefill_tokens, total_ms)
    assert sata.sata_get_error() == sata.SATA_OK

    # dominant kernel of the prefill step
    share = {n: sum(x) for n, x in kern.items()}
    top = max(share, key=share.get)
    top_ms = statistics.mean(kern[top])
    per_tok_head = 2 * (w["dV"] + 1) * m  # one of the two state contractions
    if top in ("tc_readout", "tc_chunk_states", "simt_readout", "simt_chunk_states"):
        alg = w["B"] * w["H"] * w["N"] * per_tok_head
    else:
        alg = w["B"] * w["H"] * w["N"] * 2 * per_tok_head
    if top.startswith("tc_"):
        bound, peak, unit = "tensor", pk["bf16_tflops"], "TFLOP/s"
    else:
        # fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 flop x max SM clock
        bound, peak, unit = "alu", 148 * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12, "TFLOP/s"
    achieved = alg / (top_ms / 1e3) / 1e12
    # both state contractions over the whole step, per GPU
    step_tflops = 2 * alg_one(w, m) / (total_ms / args.steps / 1e3) / 1e12
    roof = {"bound": bound, "kernel": top, "achieved": achieved, "peak": peak, "unit": unit,
            "step_tensor_tflops": step_tflops, "step_frac": step_tflops / pk["bf16_tflops"],
            "frac": achieved / peak, "traffic": traffic_record(top),
            "peak_source": pk["source"] if bound == "tensor" else "derived: 148x128x2 flop x sm_max_mhz",
            "kernel_ms": top_ms, "algorithmic_flop_per_launch": alg,
            "kernel_share": {n: s / sum(share.values()) for n, s in share.items()}}

    # e2e prefill: pinned host inputs, H2D + call + D2H of out and state per step
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    st_h = torch.empty(state.shape, dtype=state.dtype, pin_memory=True)
    e2e_ms = []
    sata.sata_profile_enable(False)
    for i in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        prefill()
        out_h.copy_(out, non_blocking=True)
        st_h.copy_(state, non_blocking=True)
        b.record(stream)
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_total = max_over_ranks(sum(e2e_ms))
    e2e = {"value": weak_scaling_value(world, args.steps, prefill_tokens, e2e_total),
           "unit": "tokens/s",
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (q, k, v)),
           "d2h_bytes_per_step": out.numel() * 4 + state.numel() * 4}
    del qd, kd, vd, out, state, q, k, v, qh, kh, vh, out_h, st_h

    # ---------------- the bf16 dK = dV = 32 prefill workload ([4,8,4096,32])
    pw3 = PREFILL_DK32
    m3 = basis_m(pw3["dK"], pw3["P"])
    q3, k3, v3 = (t.to(dev) for t in make_qkv(pw3["B"], pw3["H"], pw3["N"], pw3["dK"], pw3["dV"],
                                              seed=20261203 + 1000 * rank, dtype="bf16"))
    out3 = torch.empty(pw3["B"], pw3["H"], pw3["N"], pw3["dV"], device=dev)
    st3 = torch.empty(pw3["B"], pw3["H"], m3, pw3["dV"] + 1, device=dev)

    def prefill3():
        sata.sata_prefill(q3, k3, v3, out3, st3, pw3["B"], pw3["H"], pw3["N"], pw3["dK"],
                          pw3["dV"], pw3["P"], torch.bfloat16, stream)

    for _ in range(args.warmup):
        prefill3()
    torch.cuda.synchronize()
    sata.sata_profile_enable(True)
    k3ms, t3 = {}, []
    barrier()
    for i in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        prefill3()
        b.record(stream)
        for name, ms in sata.sata_profile_read():
            k3ms.setdefault(name, []).append(ms)
            launches += 1
        t3.append(a.elapsed_time(b))
    torch.cuda.synchronize()
    barrier()
    sata.sata_profile_enable(False)
    tot3 = max_over_ranks(sum(t3))
    share3 = {n: sum(x) for n, x in k3ms.items()}
    top3 = max(share3, key=share3.get)
    top3_ms = statistics.mean(k3ms[top3])
    alg3 = pw3["B"] * pw3["H"] * pw3["N"] * 2 * (pw3["dV"] + 1) * m3
    ach3 = alg3 / (top3_ms / 1e3) / 1e12
    prefill_dk32 = {
        "workload": "prefill B=4,H=8,N=4096,dK=dV=32,P=4 bf16 (one sata_prefill per step)",
        "value": weak_scaling_value(world, args.steps, pw3["B"] * pw3["N"], tot3),
        "unit": "tokens/s", "ms_per_step": tot3 / args.steps,
        "step_tensor_tflops": 2 * alg3 / (tot3 / args.steps / 1e3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": top3, "achieved": ach3, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": ach3 / pk["bf16_tflops"],
                     "peak_source": pk["source"], "kernel_ms": top3_ms,
                     "algorithmic_flop_per_launch": alg3,
                     "kernel_share": {n: x / sum(share3.values()) for n, x in share3.items()}},
    }
    del q3, k3, v3, out3, st3

    # ---------------- decode: fp32 state and mixed-precision state
    dw = DECODE
    dm = basis_m(dw["dK"], dw["P"])
    q, k, v = make_qkv(dw["B"], dw["H"], dw["N"], dw["dK"], dw["dV"],
                       seed=20261205 + 100 + 1000 * rank, dtype="bf16")
    dstate = torch.empty(dw["B"], dw["H"], dm, dw["dV"] + 1, device=dev)
    dout = torch.empty(dw["B"], dw["H"], w["dV"], device=dev)
    sata.sata_prefill(q.to(dev), k.to(dev), v.to(dev),
                      torch.empty(dw["B"], dw["H"], dw["N"], dw["dV"], device=dev),
                      dstate, dw["B"], dw["H"], dw["N"], dw["dK"], dw["dV"], dw["P"],
                      torch.bfloat16, stream)
    m_lo = sata.sata_state_fp32_rows(dw["dK"], dw["P"])
    lo = torch.empty(dw["B"], dw["H"], m_lo, dw["dV"] + 1, device=dev)
    hi = torch.empty(dw["B"], dw["H"], dm - m_lo, dw["dV"] + 1, device=dev, dtype=torch.float16)
    sata.sata_state_split(dstate, lo, hi, dw["B"], dw["H"], dw["dK"], dw["dV"], dw["P"], stream)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    nsteps = args.decode_steps
    ds = DecodeStream(5)
    toks = [tuple(t.to(dev) for t in ds.next()) for _ in range(args.warmup + nsteps)]
    hq = [tuple(t.pin_memory() for t in ds.next()) for _ in range(min(nsteps, 64))]

    def fp32_step(qt, kt, vt):
        sata.sata_decode_step(qt, kt, vt, dstate, dout, dw["B"], dw["H"], dw["dK"], dw["dV"],
                              dw["P"], torch.bfloat16, stream)

    def mixed_step(qt, kt, vt):
        sata.sata_decode_step_mixed(qt, kt, vt, lo, hi, dout, dw["B"], dw["H"], dw["dK"],
                                    dw["dV"], dw["P"], torch.bfloat16, stream)

    def time_decode(step, state_bytes, label):
        """All decode steps timed one by one (context grows by one token per
        step), the library's kernels timed by its event hook."""
        nonlocal launches
        for i in range(args.warmup):
            step(*toks[i])
        torch.cuda.synchronize()
        sata.sata_profile_enable(True)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(nsteps)]
        kk = {}
        barrier()
        torch.cuda.synchronize()
        for i in range(nsteps):
            ev[i][0].record(stream)
            step(*toks[args.warmup + i])
            ev[i][1].record(stream)
            for name, ms in sata.sata_profile_read():
                kk.setdefault(name, []).append(ms)
                launches += 1
        torch.cuda.synchronize()
        barrier()
        sata.sata_profile_enable(False)
        dms = [a.elapsed_time(b) for a, b in ev]
        total = max_over_ranks(sum(dms))
        dbytes = 2 * dw["B"] * dw["H"] * state_bytes
        kname = max(kk, key=lambda n: sum(kk[n]))
        kms = statistics.mean(kk[kname])
        ach = dbytes / (kms / 1e3) / 1e9
        qn = max(1, nsteps // 4)
        quarters = [statistics.median(dms[j * qn:(j + 1) * qn]) for j in range(4)
                    if dms[j * qn:(j + 1) * qn]]
        res = {
            "state": label, "value": weak_scaling_value(world, nsteps, dw["B"], total),
            "unit": "tokens/s", "ms_per_step": total / nsteps, "steps": nsteps,
            "context": [dw["N"] + args.warmup + 1, dw["N"] + args.warmup + nsteps],
            "latency_ms_quarter_medians": quarters,
            "latency_ms_min": min(dms), "latency_ms_max": max(dms),
            "latency_flatness": max(quarters) / min(quarters) - 1.0,
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": ach,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                         "traffic": traffic_record(kname if label == "fp32" else kname + ":mixed"),
                         "peak_source": pk["source"], "kernel_ms": kms,
                         "algorithmic_bytes_per_launch": dbytes},
        }
        # e2e: H2D of the step's q,k,v from pinned host memory, D2H of out
        dout_h = torch.empty(dout.shape, pin_memory=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        qt, kt, vt = toks[0]
        a.record(stream)
        for qh_, kh_, vh_ in hq:
            qt.copy_(qh_, non_blocking=True)
            kt.copy_(kh_, non_blocking=True)
            vt.copy_(vh_, non_blocking=True)
            step(qt, kt, vt)
            dout_h.copy_(dout, non_blocking=True)
        b.record(stream)
        b.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b))
        res["e2e"] = {"value": world * len(hq) * dw["B"] / (e2e_ms / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hq[0]),
                      "d2h_bytes_per_step": dout.numel() * 4}
        return res

    decode = time_decode(fp32_step, dm * (dw["dV"] + 1) * 4, "fp32")
    decode["mixed_state"] = time_decode(
        mixed_step, m_lo * (dw["dV"] + 1) * 4 + (dm - m_lo) * (dw["dV"] + 1) * 2,
        f"rows of degree <= 2 fp32 ({m_lo}/head), degree 3 fp16 ({dm - m_lo}/head)")
    variants = time_variants(sata, stream, dev, flush, pk, rank)
    clocks = sampler.stop()
    assert sata.sata_get_error() == sata.SATA_OK

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded i.i.d. N(0,1) q,k,v cast to bf16",
        "config": {"workload": WORKLOAD, "global_batch": world * PREFILL["B"] * PREFILL["H"],
                   "seq_len": PREFILL["N"], "parallelism": f"dp{world} (independent heads)",
                   "l2": "prefill: 256 MiB L2 flush between timed steps; decode: 3.19 GB fp32 "
                         "(1.66 GB mixed) state > L2",
                   "decode_steps": nsteps},
        "roofline": roof, "decode": decode, "prefill_dk32": prefill_dk32, "variants": variants,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    return line


# --------------------------------------------------------------- variants
def time_variants(sata, stream, dev, flush, pk, rank, steps=5, warmup=3):
    """Short measurements of the variants beyond the two benchmark workloads:
    P = 5 decode at d_K = 64 (its state is 212 MB per head) and two prefills
    on the CUDA-core path (many small fp32 heads; P = 5 bf16)."""
    import torch
    from sata_inputs import make_qkv

    def timed(fn, flush_l2):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(steps):
            if flush_l2:
                flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    out = {}
    # decode, P = 5, d_K = d_V = 64, B = 1, H = 2, state of a 64-token prefill
    B, H, N, d, P = 1, 2, 64, 64, 5
    m = basis_m(d, P)
    q, k, v = (t.to(dev) for t in make_qkv(B, H, N + 1, d, d, seed=20261210 + 1000 * rank,
                                            dtype="bf16"))
    st = torch.empty(B, H, m, d + 1, device=dev)
    sata.sata_prefill(q[:, :, :N].contiguous(), k[:, :, :N].contiguous(), v[:, :, :N].contiguous(),
                      torch.empty(B, H, N, d, device=dev), st, B, H, N, d, d, P, torch.bfloat16,
                      stream)
    qt, kt, vt = (x[:, :, N].contiguous() for x in (q, k, v))
    o = torch.empty(B, H, d, device=dev)
    ms = timed(lambda: sata.sata_decode_step(qt, kt, vt, st, o, B, H, d, d, P, torch.bfloat16,
                                             stream), False)
    nbytes = 2 * B * H * m * (d + 1) * 4
    out["decode_p5_dk64"] = {
        "workload": "decode B=1,H=2,dK=dV=64,P=5 fp32 state (814385 rows/head, 212 MB/head)",
        "ms_per_step": ms, "tokens_per_s": B / (ms / 1e3),
        "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "unit": "GB/s",
                     "peak": pk["hbm_gbs"], "frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                     "algorithmic_bytes_per_launch": nbytes}}
    del q, k, v, st
    # prefill on the CUDA-core path: many small fp32 heads, and P = 5 bf16
    for key, (B, H, N, d, P, dt, tdt) in {
            "prefill_f32_dk16_h64": (4, 64, 1024, 16, 4, "f32", torch.float32),
            "prefill_bf16_dk16_p5": (1, 8, 4096, 16, 5, "bf16", torch.bfloat16)}.items():
        m = basis_m(d, P)
        q, k, v = (t.to(dev) for t in make_qkv(B, H, N, d, d, seed=20261211 + 1000 * rank,
                                                dtype=dt))
        o = torch.empty(B, H, N, d, device=dev)
        st = torch.empty(B, H, m, d + 1, device=dev)
        ms = timed(lambda: sata.sata_prefill(q, k, v, o, st, B, H, N, d, d, P, tdt, stream), True)
        out[key] = {"workload": f"prefill B={B},H={H},N={N},dK=dV={d},P={P} {dt} (CUDA cores)",
                    "ms_per_step": ms, "tokens_per_s": B * N / (ms / 1e3),
                    "head_tokens_per_s": B * H * N / (ms / 1e3)}
        del q, k, v, o, st
    torch.cuda.synchronize()
    return out


# --------------------------------------------------------------- reference arm
def run_reference(args):
    per_step = []
    n = args.ref_tokens
    for i in range(args.warmup + args.steps):
        dt, tok = oracle_prefill_sample(n, seed=i)
        if i >= args.warmup:
            per_step.append((dt, tok))
    t = sum(d for d, _ in per_step)
    tok = sum(x for _, x in per_step)
    ddt, dtok = oracle_decode_sample(2)
    value = tok / t
    th = host_threads()
    sample = (f"each step: oracle.quadratic_form + oracle.final_state on the first {n} tokens "
              f"of 1 of 8 heads, fp64 numpy on the host cores, scaled to the workload by "
              f"(query, key) pairs and by tokens")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded i.i.d. N(0,1) q,k,v cast to bf16",
        "config": {"workload": WORKLOAD, "global_batch": PREFILL["B"] * PREFILL["H"],
                   "seq_len": PREFILL["N"], "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": th["cores"],
                         "numpy_threads": th["numpy_threads"], "kind": "oracle",
                         "sample": sample},
        "decode": {"value": dtok / ddt, "unit": "tokens/s",
                   "sample": "oracle.decode_step on 2 of 256 heads from a random state"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def profile_case(case: str):
    """Small cases for ncu captures: a few launches of one kernel on inputs
    larger than L2 but a few GB on the device at most."""
    import torch

    import linear_cost_attention_b200 as sata
    from sata_inputs import make_qkv

    torch.cuda.set_device(0)
    if case == "decode":
        B, H, N, d, P = 8, 8, 256, 64, 4          # state 797 MB (> L2)
        q, k, v = make_qkv(B, H, N, d, d, seed=3, dtype="bf16")
        _, state = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P)
        for t in range(5):
            qt, kt, vt = (x[:, :, t].contiguous().cuda() for x in (q, k, v))
            sata.decode_step(qt, kt, vt, state, P)
    elif case == "decode_mixed":
        B, H, N, d, P = 8, 8, 256, 64, 4          # mixed state 415 MB (> L2)
        q, k, v = make_qkv(B, H, N, d, d, seed=3, dtype="bf16")
        _, state = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P)
        lo, hi = sata.split_state(state, P)
        for t in range(5):
            qt, kt, vt = (x[:, :, t].contiguous().cuda() for x in (q, k, v))
            sata.decode_step_mixed(qt, kt, vt, lo, hi, P)
    elif case == "prefill":
        B, H, N, d, P = 1, 2, 8192, 64, 4         # one chunk-boundary snapshot per head
        q, k, v = make_qkv(B, H, N, d, d, seed=4, dtype="bf16")
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        for _ in range(3):
            sata.prefill(qd, kd, vd, P)
    elif case == "prefill_full":
        # the benchmark's prefill workload itself (about 0.4 GB on the device)
        w = PREFILL
        q, k, v = make_qkv(w["B"], w["H"], w["N"], w["dK"], w["dV"], seed=4, dtype="bf16")
        qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
        for _ in range(3):
            sata.prefill(qd, kd, vd, w["P"])
    else:
        raise SystemExit(f"unknown profile case {case}")
    torch.cuda.synchronize()
    assert sata.sata_get_error() == sata.SATA_OK


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--ref-tokens", type=int, default=1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["decode", "decode_mixed", "prefill", "prefill_full"],
                    default=None,
                    help="run a small case of one kernel for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    line = run_ours(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
