#!/usr/bin/env python
"""Benchmark of the CKDA recurrence library on one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: chunked-forward throughput (Mtok/s, tokens = B*T) on the 1.3B-layer-shaped workload
(B=2, T=2048, H=16, dk=dv=128, bf16, chunk 64, CKDA gate range).  One step = one
ckda_fwd_chunked call over that batch (q/k prologue, gate prep, intra-chunk factors, state pass
and output: the whole forward path).  Every rank runs its own replica on its own synthetic batch
(weak scaling, no collective on the data path); rank 0 prints one JSON line with the whole-job
throughput (all ranks' tokens / the slowest rank's device time).

The line also carries: the roofline of the one kernel a step launches (ckda_tc_fused, the whole
forward; against the measured HBM bandwidth), the same work timed as two kernels in sequence,
the decode step's HBM throughput on the batched-decode workload, the standalone q/k prologue's
HBM throughput (rotation then L2 norm at the layer shape), the backward's time at the layer
shape, the CKDA/KDA-range throughput ratio,
an end-to-end figure through the C ABI with host buffers, SM clocks sampled during the timed
region, and (rank 0, one GPU) the float64 CPU oracle's throughput on bounded samples of the
layer-shaped and long-context workloads, on all host cores and on one.

--impl reference times that float64 CPU oracle (the only reference implementation there is)
on the same workload, metric and unit.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CKDA chunked-fwd Mtok/s (H=16,d=128,bf16) + decode GB/s, % of roofline"
WORKLOAD = dict(name="layer_ckda_bf16", B=2, T=2048, H=16, dk=128, dv=128, chunk=64,
                kind="ckda", dtype="bf16")
# algorithmic bytes per head-token of the forward: q, k, v bf16 + alpha fp32 + beta fp32 + out bf16
FWD_BYTES_PER_HT = 3 * 256 + 512 + 4 + 256
INTRA_BYTES_PER_HT = 3 * 256 + 512 + 4          # what the chunk-factor kernel must read
STATE_BYTES_PER_HT = 256                        # what the state pass must write (plus states)
N_ROTATE = 4                                    # input sets cycled so no step finds its inputs in L2


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip decode / KDA-ratio / e2e / CPU-baseline legs")
    ap.add_argument("--profile-case", choices=["fwd", "decode", "prologue", "bwd", "seg", "simt"], default=None,
                    help="run only a few calls of one entry point (for ncu captures) and exit")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---- clocks ----------------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples with host timestamps.  Started well before the
    timed region (nvidia-smi takes a moment to produce its first line); window(t0, t1) keeps the
    samples taken while the timed region ran, widened to the nearest sample on each side when the
    region is shorter than the sampling interval."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.samples = []   # (host time, sm MHz, max MHz, reasons)
        self.raw = []

    def start(self, wait_first=5.0):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                   "-lms", "50"]
            if self.gpu_id:
                cmd.insert(1, f"--id={self.gpu_id}")
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t = time.time()
            while not self.samples and time.time() - t < wait_first and self.proc.poll() is None:
                time.sleep(0.02)
        except Exception as e:
            self.proc = None
            self.raw.append(repr(e))

    def _read(self):
        for line in self.proc.stdout:
            now = time.time()
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                self.raw.append(line.strip())
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                self.raw.append(line.strip())
                continue
            reasons = {n for n, val in zip(self.NAMES, f[5:9]) if val.lower() == "active"}
            self.samples.append((now, sm, mx, reasons))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def window(self, t0, t1):
        if not self.samples:
            return {"error": "no clock samples", "raw": self.raw[:3]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:   # region shorter than the interval: nearest sample on each side
            before = [s for s in self.samples if s[0] < t0][-1:]
            after = [s for s in self.samples if s[0] > t1][:1]
            inside = before + after
        sms = [s[1] for s in inside]
        reasons = set().union(*[s[3] for s in inside]) if inside else set()
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(s[2] for s in inside),
                "reasons": sorted(reasons), "samples": len(inside),
                "window_ms": round((t1 - t0) * 1e3, 2)}


# ---- helpers ---------------------------------------------------------------------------------

def event_time_ms(fn, steps, stream, queue_ahead_ms=0.0):
    """Device time of `steps` calls of fn, CUDA events recorded on the launching stream.  With
    queue_ahead_ms the stream first runs a GPU spin of that length, during which the host queues
    the calls: the events then time the device work back to back, without the host's per-call
    overhead (used where that overhead exceeds a call's device time)."""
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if queue_ahead_ms > 0:
        torch.cuda._sleep(int(queue_ahead_ms * 2.0e6))   # ~2 GHz: cycles per millisecond
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def kernel_source_hash(files=None):
    """Hash of the named sources under csrc/ (all of them when files is None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_82_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """DRAM bytes per launch for `kernel` from the committed ncu summary, if the sources the
    kernel is built from are unchanged since that capture (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    ent = d.get("kernels", {}).get(kernel)
    if ent is None or ent.get("source_hash") != kernel_source_hash(ent.get("sources")):
        return None
    return ent.get("dram_bytes_per_launch")


# ---- the reference arm: float64 CPU oracle ---------------------------------------------------

def cpu_oracle_leg(steps, warmup, budget_s=20.0, threads=None, heads=None, workload=None):
    """Time the float64 oracle on a bounded sample of a forward workload (the headline's by
    default).  The sample is the first `heads` (batch, head) pairs of the workload over its full
    sequence length, on `threads` host threads (default: every core, and as many heads);
    tokens/s is scaled to the workload's tokens (B*T tokens of H heads each)."""
    import numpy as np
    import oracle
    import synth
    w = workload or WORKLOAD
    cores = os.cpu_count() or 1
    threads = threads or cores
    heads = max(1, min(w["H"], heads or threads))
    d = synth.fwd_inputs(1, w["T"], heads, w["dk"], w["dv"], kind=w["kind"], dtype=w["dtype"],
                         h0_std=w.get("h0_std", 0.0), seed=4242)
    kw = dict(rope_theta=w.get("rope_theta", 0.0), nthreads=threads, want_state=True)
    run = lambda: oracle.fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["h0"], **kw)
    for _ in range(warmup):
        run()
    times = []
    t_start = time.perf_counter()
    for _ in range(steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > budget_s:
            break
    sec = statistics.median(times)
    head_tokens = w["T"] * heads
    mtok = head_tokens / w["H"] / sec / 1e6
    sample = (f"float64 oracle, {heads} head(s) of {w.get('name', 'the workload')}, T={w['T']}, "
              f"{threads} thread(s), {len(times)} timed run(s), median {sec * 1e3:.1f} ms")
    return mtok, threads, sample, len(times), sec


def reference_main(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    mtok, cores, sample, n, sec = cpu_oracle_leg(max(1, args.steps), max(0, min(args.warmup, 2)),
                                                 budget_s=120.0)
    w = WORKLOAD
    line = {"impl": "reference", "metric": METRIC, "value": round(mtok, 6), "unit": "Mtok/s",
            "n_gpus": args.gpus, "steps": n, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w['name']} (B={w['B']},T={w['T']},H={w['H']},"
                                   f"dk=dv={w['dk']},chunk={w['chunk']},{w['kind']} gates)",
                       "global_batch": w["B"], "seq_len": w["T"], "parallelism": "host threads"},
            "cpu_baseline": {"value": round(mtok, 6), "unit": "Mtok/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(mtok, 6), "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---- profiling cases (a few plain calls, no timing) ----------------------------------------------

def profile_case(case, calls, dev):
    """A few calls of one entry point on its benchmark workload, for ncu.  The first calls are
    the ones to capture (ncu -c); nothing is timed or printed."""
    import torch
    import gated_delta_rule_82_b200 as ck
    import synth
    calls = max(1, calls)
    if case == "fwd":
        w = WORKLOAD
        s = synth.torch_fwd_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], kind=w["kind"],
                                   seed=1, device=dev)
        ws = torch.empty(ck.workspace_bytes(w["B"], w["T"], w["H"], w["dk"], w["dv"]),
                         dtype=torch.uint8, device=dev)
        for _ in range(calls):
            ck.fwd_chunked(s["q"], s["k"], s["v"], s["alpha"], s["beta"], None, path="tc",
                           workspace=ws)
    elif case == "decode":
        wd = synth.WORKLOADS["decode_bf16"]
        d = synth.torch_decode_inputs(calls, wd["N"], wd["H"], 128, 128, seed=5, device=dev)
        state = 0.02 * torch.randn((wd["N"], wd["H"], 128, 128), device=dev)
        for i in range(calls):
            ck.decode_step(d["q"][i], d["k"][i], d["v"][i], d["alpha"][i], d["beta"][i], state)
    elif case == "bwd":
        w = WORKLOAD
        s = synth.torch_fwd_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], kind=w["kind"],
                                   h0_std=0.02, seed=1, device=dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(2)
        dout = torch.randn((w["B"], w["T"], w["H"], w["dv"]), generator=gen, device=dev).bfloat16()
        dhT = 0.02 * torch.randn((w["B"], w["H"], w["dk"], w["dv"]), generator=gen, device=dev)
        for _ in range(calls):
            ck.bwd_chunked(s["q"], s["k"], s["v"], s["alpha"], s["beta"], s["h0"], dout, dhT)
    elif case == "simt":
        w = WORKLOAD
        s = synth.torch_fwd_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], kind=w["kind"],
                                   h0_std=0.02, seed=1, device=dev)
        ws = torch.empty(ck.simt_workspace_bytes(w["B"], w["T"], w["H"], w["dk"], w["dv"]),
                         dtype=torch.uint8, device=dev)
        for _ in range(calls):
            ck.fwd_chunked(s["q"], s["k"], s["v"], s["alpha"], s["beta"], s["h0"], path="simt",
                           workspace=ws)
    elif case == "seg":
        wl = synth.WORKLOADS["long_rope_bf16"]
        s = synth.torch_fwd_inputs(1, wl["T"], 2, 128, 128, kind="ckda", dtype="bf16",
                                   h0_std=wl["h0_std"], seed=1, device=dev)
        for _ in range(calls):
            ck.fwd_segmented(s["q"], s["k"], s["v"], s["alpha"], s["beta"], s["h0"], segments=0,
                             rope_theta=wl["rope_theta"])
    else:
        w = WORKLOAD
        s = synth.torch_fwd_inputs(w["B"], w["T"], w["H"], w["dk"], w["dv"], seed=1, device=dev)
        for _ in range(calls):
            ck.qk_prologue(s["q"], s["k"], rope_theta=10000.0)
    torch.cuda.synchronize()
    return 0


# ---- rank plumbing (one process per GPU; also exercised by CPU tests with the gloo backend) ---

PG_TIMEOUT_S = 120


def init_ranks(world, backend="nccl", device=None, timeout_s=PG_TIMEOUT_S):
    """Join the process group of a world-size > 1 run (rendezvous from MASTER_ADDR/MASTER_PORT).
    A short timeout makes ranks that wait on a missing peer fail instead of hanging."""
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if device is not None else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def max_over_ranks(x, device, world):
    """The maximum of the scalar x over all ranks (one all_reduce(MAX)); x itself when world == 1."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_mtok_s(tokens_per_rank, world, ms_per_step_max):
    """Whole-job throughput: every rank processes its own batch of tokens_per_rank tokens per
    step; the job's step time is the slowest rank's."""
    return tokens_per_rank * world / (ms_per_step_max / 1e3) / 1e6


def input_seed(rank, i):
    """Seed of the i-th rotated input set on `rank`: disjoint synthetic batches per replica."""
    return 1000 * (rank + 1) + i


# ---- our arm -----------------------------------------------------------------------------------

def main():
    args = parse()
    if args.impl == "reference":
        return reference_main(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        init_ranks(world, "nccl", dev)

    from gated_delta_rule_82_b200 import build as ckbuild
    if rank == 0:
        ckbuild.build()
    if world > 1:
        dist.barrier()
    import gated_delta_rule_82_b200 as ck
    import synth

    if args.profile_case:
        return profile_case(args.profile_case, args.steps, dev)

    hbm_peak, tc_peak, peak_src = peaks()
    w = WORKLOAD
    B, T, H, dk, dv, C = w["B"], w["T"], w["H"], w["dk"], w["dv"], w["chunk"]
    stream = torch.cuda.current_stream(dev)

    # ---- inputs: N_ROTATE independent synthetic batches, resident in HBM --------------------
    sets = [synth.torch_fwd_inputs(B, T, H, dk, dv, kind=w["kind"], dtype=w["dtype"],
                                   seed=input_seed(rank, i), device=dev) for i in range(N_ROTATE)]
    out = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(ck.workspace_bytes(B, T, H, dk, dv, C, torch.bfloat16, "tc"),
                     dtype=torch.uint8, device=dev)

    def step(i, stages=0, inputs=None):
        s = (inputs or sets)[i % N_ROTATE]
        ck.fwd_chunked(s["q"], s["k"], s["v"], s["alpha"], s["beta"], None, chunk=C, path="tc",
                       out=out, hT=hT, workspace=ws, stages=stages)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()

    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id)
    sampler.start()
    for i in range(2):
        step(i)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_host0 = time.time()
    ms = event_time_ms(step, args.steps, stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    if world > 1:
        dist.barrier()
    time.sleep(0.12)
    clocks = sampler.window(t_host0, t_host1)
    ms_per_step = max_over_ranks(ms / args.steps, dev, world)
    value = weak_scaling_mtok_s(B * T, world, ms_per_step)

    # ---- roofline of the one kernel a step launches (ckda_tc_fused), from this rank's step time;
    # the step also clears the chunk-heads' ready flags (a 4-byte-per-chunk-head memset), which
    # this device time includes
    ht = B * T * H
    ms_local = ms / args.steps
    per_launch = ht * FWD_BYTES_PER_HT
    achieved = per_launch / (ms_local / 1e3) / 1e9
    path_gbs = ht * FWD_BYTES_PER_HT / (ms_per_step / 1e3) / 1e9
    roofline = {"kernel": "ckda_tc_fused", "bound": "hbm", "achieved": round(achieved, 1),
                "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                "traffic": ncu_traffic("ckda_tc_fused"), "algorithmic_bytes_per_launch": per_launch,
                "ms_per_launch": round(ms_local, 4), "peak_source": peak_src}
    # the same work as two kernels in sequence (the profiling split): the factor kernel alone,
    # then the state pass alone over the workspace it filled
    ms_intra = event_time_ms(lambda i: step(i, stages=1), args.steps, stream) / args.steps
    ms_state = event_time_ms(lambda i: step(i, stages=2), args.steps, stream) / args.steps
    intra_gbs = ht * INTRA_BYTES_PER_HT / (ms_intra / 1e3) / 1e9
    state_gbs = (ht * STATE_BYTES_PER_HT) / (ms_state / 1e3) / 1e9
    kernels = {"ckda_tc_fused": {"ms": round(ms_local, 4), "alg_GBps": round(achieved, 1)},
               "split": {"ckda_tc_intra": {"ms": round(ms_intra, 4), "alg_GBps": round(intra_gbs, 1)},
                         "ckda_tc_state": {"ms": round(ms_state, 4), "alg_GBps": round(state_gbs, 1)}}}
    path_roofline = {"bound": "hbm", "achieved": round(path_gbs, 1), "peak": hbm_peak,
                     "unit": "GB/s", "frac": round(path_gbs / hbm_peak, 4),
                     "roofline_mtok_s": round(hbm_peak * 1e9 / (H * FWD_BYTES_PER_HT) / 1e6, 1)}

    extras = {}
    if not args.no_extras:
        # ---- KDA gate range at the same shape: CKDA/KDA throughput ratio --------------------
        kda_sets = [synth.torch_fwd_inputs(B, T, H, dk, dv, kind="kda", dtype="bf16",
                                           seed=7000 + 10 * rank + i, device=dev)
                    for i in range(N_ROTATE)]
        for i in range(3):
            step(i, inputs=kda_sets)
        ms_kda = event_time_ms(lambda i: step(i, inputs=kda_sets), args.steps, stream) / args.steps
        extras["kda_range"] = {"mtok_s": round(B * T / (ms_kda / 1e3) / 1e6, 2),
                               "ckda_over_kda": round(ms_kda / (ms_per_step if world == 1 else ms / args.steps), 4)}
        del kda_sets

        # ---- gates given as logits (alpha = 2 sigma(a) - 1 from bf16 a, beta = 2 sigma(b)) ----
        gl_sets = [synth.torch_fwd_inputs(B, T, H, dk, dv, dtype="bf16", seed=8000 + 10 * rank + i,
                                          device=dev, gate_logits=True) for i in range(N_ROTATE)]

        def step_gl(i):
            s = gl_sets[i % N_ROTATE]
            ck.fwd_chunked(s["q"], s["k"], s["v"], s["alpha"], s["beta"], None, chunk=C, path="tc",
                           out=out, hT=hT, workspace=ws, gate_logits=True)
        for i in range(3):
            step_gl(i)
        ms_gl = event_time_ms(step_gl, args.steps, stream) / args.steps
        gl_bytes = FWD_BYTES_PER_HT - 256   # alpha as bf16 logits: 256 B instead of 512 per head-token
        extras["gate_logits"] = {
            "workload": f"{w['name']} with bf16 gate logits a and fp32 logits b",
            "mtok_s": round(B * T / (ms_gl / 1e3) / 1e6, 2), "ms_per_step": round(ms_gl, 4),
            "roofline_mtok_s": round(hbm_peak * 1e9 / (H * gl_bytes) / 1e6, 1),
            "path_hbm_frac": round(ht * gl_bytes / (ms_gl / 1e3) / 1e9 / hbm_peak, 4)}
        del gl_sets

        # ---- packed sequences of different lengths (cu_seqlens), the layer shape's tokens ----
        wp = synth.WORKLOADS["packed_bf16"]
        Tp, n_p = sum(wp["lens"]), len(wp["lens"])
        p_sets = [synth.torch_fwd_inputs(1, Tp, H, dk, dv, kind="ckda", dtype="bf16",
                                         seed=8500 + 10 * rank + i, device=dev)
                  for i in range(N_ROTATE)]
        cu_h = torch.tensor([sum(wp["lens"][:j]) for j in range(n_p + 1)], dtype=torch.int32)
        cu_d = cu_h.to(dev)
        out_p = torch.empty((1, Tp, H, dv), dtype=torch.bfloat16, device=dev)
        hT_p = torch.empty((n_p, H, dk, dv), dtype=torch.float32, device=dev)
        ws_p = torch.empty(ck.varlen_workspace_bytes(cu_h, H, dk, dv, C, torch.bfloat16),
                           dtype=torch.uint8, device=dev)

        def step_p(i):
            s = p_sets[i % N_ROTATE]
            ck.fwd_varlen(s["q"], s["k"], s["v"], s["alpha"], s["beta"], cu_d, None,
                          cu_seqlens_cpu=cu_h, chunk=C, path="tc", out=out_p, hT=hT_p,
                          workspace=ws_p)
        for i in range(3):
            step_p(i)
        ms_p_host = event_time_ms(step_p, args.steps, stream) / args.steps
        ms_p = event_time_ms(step_p, args.steps, stream,
                             queue_ahead_ms=max(20.0, 0.5 * args.steps)) / args.steps
        extras["varlen"] = {
            "workload": f"packed_bf16 ({n_p} sequences of {wp['lens']} tokens, H={H}, dk=dv=128)",
            "mtok_s": round(Tp / (ms_p / 1e3) / 1e6, 2), "ms_per_step": round(ms_p, 4),
            "ms_per_step_host_paced": round(ms_p_host, 4),
            "timing": "device time with the calls queued ahead of the timed region (the host's "
                      "per-call work for packed offsets is excluded; ms_per_step_host_paced "
                      "includes it)",
            "path_hbm_frac": round(Tp * H * FWD_BYTES_PER_HT / (ms_p / 1e3) / 1e9 / hbm_peak, 4)}
        del p_sets, ws_p

        # ---- long-context forward with RoPE and an initial state (one call per step) -------
        wl = synth.WORKLOADS["long_rope_bf16"]
        L = synth.torch_fwd_inputs(wl["B"], wl["T"], wl["H"], 128, 128, kind="ckda",
                                   dtype="bf16", h0_std=wl["h0_std"], seed=9000 + rank, device=dev)
        wsL = torch.empty(ck.workspace_bytes(wl["B"], wl["T"], wl["H"], 128, 128),
                          dtype=torch.uint8, device=dev)
        outL = torch.empty_like(L["v"])
        hL = torch.empty_like(L["h0"])
        fnL = lambda i: ck.fwd_chunked(L["q"], L["k"], L["v"], L["alpha"], L["beta"], L["h0"],
                                       rope_theta=wl["rope_theta"], path="tc", out=outL, hT=hL,
                                       workspace=wsL)
        for i in range(2):
            fnL(i)
        nL = max(3, args.steps // 10)
        ms_long = event_time_ms(fnL, nL, stream) / nL
        htL = wl["B"] * wl["T"] * wl["H"]
        extras["long_context"] = {
            "workload": "long_rope_bf16 (B=1,T=65536,H=16,dk=dv=128,RoPE 1e4 half-split,h0)",
            "ms": round(ms_long, 3), "mtok_s": round(wl["B"] * wl["T"] / (ms_long / 1e3) / 1e6, 2),
            "hbm_frac": round(htL * FWD_BYTES_PER_HT / (ms_long / 1e3) / 1e9 / hbm_peak, 4)}
        # the same workload with the segment-parallel state pass (8 segments, and the model's
        # count, which keeps the single fused launch here)
        wsS = torch.empty(ck.segmented_workspace_bytes(wl["B"], wl["T"], wl["H"], 128, 128, 8),
                          dtype=torch.uint8, device=dev)
        fnS = lambda i: ck.fwd_segmented(L["q"], L["k"], L["v"], L["alpha"], L["beta"], L["h0"],
                                         segments=8, rope_theta=wl["rope_theta"], out=outL,
                                         hT=hL, workspace=wsS)
        for i in range(2):
            fnS(i)
        ms_seg = event_time_ms(fnS, nL, stream) / nL
        extras["long_context"]["segments_8_ms"] = round(ms_seg, 3)
        extras["long_context"]["segments_auto"] = ck.segments_auto(wl["B"], wl["T"], wl["H"])
        del L, wsL, outL, hL, wsS

        # ---- one long sequence on two heads (a head-sharded layer's share of the long-context
        # workload): the single fused launch vs the segment-parallel state pass ----------------
        H2 = 2
        L2 = synth.torch_fwd_inputs(1, wl["T"], H2, 128, 128, kind="ckda", dtype="bf16",
                                    h0_std=wl["h0_std"], seed=9500 + rank, device=dev)
        P2 = ck.segments_auto(1, wl["T"], H2)
        ws2 = torch.empty(ck.segmented_workspace_bytes(1, wl["T"], H2, 128, 128, P2),
                          dtype=torch.uint8, device=dev)
        out2, h2 = torch.empty_like(L2["v"]), torch.empty_like(L2["h0"])
        fnF = lambda i: ck.fwd_chunked(L2["q"], L2["k"], L2["v"], L2["alpha"], L2["beta"],
                                       L2["h0"], rope_theta=wl["rope_theta"], path="tc",
                                       out=out2, hT=h2, workspace=ws2)
        fnG = lambda i: ck.fwd_segmented(L2["q"], L2["k"], L2["v"], L2["alpha"], L2["beta"],
                                         L2["h0"], segments=P2, rope_theta=wl["rope_theta"],
                                         out=out2, hT=h2, workspace=ws2)
        for i in range(2):
            fnF(i)
            fnG(i)
        ms_f2 = event_time_ms(fnF, nL, stream) / nL
        ms_g2 = event_time_ms(fnG, nL, stream) / nL
        ht2 = wl["T"] * H2
        extras["long_context_2_heads"] = {
            "workload": "B=1,T=65536,H=2,dk=dv=128,RoPE 1e4 half-split,h0",
            "fused_ms": round(ms_f2, 3), "segmented_ms": round(ms_g2, 3), "segments": P2,
            "segmented_mtok_s": round(wl["T"] / (ms_g2 / 1e3) / 1e6, 2),
            "segmented_hbm_frac": round(ht2 * FWD_BYTES_PER_HT / (ms_g2 / 1e3) / 1e9 / hbm_peak, 4)}
        del L2, ws2, out2, h2

        # ---- standalone q/k prologue: rotation (theta 1e4, half-split) then the L2 norm --------
        pq = [synth.torch_fwd_inputs(B, T, H, dk, dv, seed=6000 + 10 * rank + i, device=dev)
              for i in range(N_ROTATE)]
        pqo, pko = torch.empty_like(pq[0]["q"]), torch.empty_like(pq[0]["k"])
        fnP = lambda i: ck.qk_prologue(pq[i % N_ROTATE]["q"], pq[i % N_ROTATE]["k"],
                                       rope_theta=10000.0, q_out=pqo, k_out=pko)
        for i in range(3):
            fnP(i)
        # a call's device time (~10 us) is below the host's per-call work: queue the calls behind
        # a GPU spin so that the events time the device work back to back
        ms_pro = event_time_ms(fnP, args.steps, stream,
                               queue_ahead_ms=max(20.0, 0.5 * args.steps)) / args.steps
        pro_bytes = 4 * B * T * H * dk * 2          # q and k read, q and k written (bf16)
        pro_gbs = pro_bytes / (ms_pro / 1e3) / 1e9
        extras["prologue"] = {
            "workload": f"qk_prologue at the layer shape (B={B},T={T},H={H},dk={dk},bf16), "
                        "RoPE theta 1e4 half-split, then L2 norm",
            "us_per_call": round(ms_pro * 1e3, 2),
            "roofline": {"bound": "hbm", "achieved": round(pro_gbs, 1), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(pro_gbs / hbm_peak, 4),
                         "traffic": ncu_traffic("qk_prologue_kernel"),
                         "algorithmic_bytes_per_launch": pro_bytes}}
        del pq, pqo, pko

        # ---- backward at the layer shape: gradients of <dout, out> + <dhT, hT> ---------------
        bw = synth.torch_fwd_inputs(B, T, H, dk, dv, kind=w["kind"], dtype="bf16", h0_std=0.02,
                                    seed=6500 + rank, device=dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(6600 + rank)
        dout = torch.randn((B, T, H, dv), generator=gen, device=dev).to(torch.bfloat16)
        dhT = 0.02 * torch.randn((B, H, dk, dv), generator=gen, device=dev)
        wsb = torch.empty(ck.bwd_workspace_bytes(B, T, H, dk, dv), dtype=torch.uint8, device=dev)
        fnB = lambda i: ck.bwd_chunked(bw["q"], bw["k"], bw["v"], bw["alpha"], bw["beta"],
                                       bw["h0"], dout, dhT, workspace=wsb)
        for i in range(2):
            fnB(i)
        nB = max(3, args.steps // 10)
        ms_b = event_time_ms(fnB, nB, stream) / nB
        extras["backward"] = {
            "workload": f"{w['name']} (B={B},T={T},H={H},dk=dv={dk}) with h0, dout and dhT: dq, dk, "
                        "dv, dalpha, dbeta, dh0, fp32-grade (CUDA cores and split-tf32 warp tiles, "
                        "16-token chunks)",
            "ms": round(ms_b, 3), "mtok_s": round(B * T / (ms_b / 1e3) / 1e6, 3),
            "over_forward": round(ms_b / ms_local, 1)}
        # the same inputs through the CUDA-core forward (fp32-grade products; the path for
        # workloads whose state does not decay), in its record form
        wss = torch.empty(ck.simt_workspace_bytes(B, T, H, dk, dv), dtype=torch.uint8, device=dev)
        outS, hS = torch.empty_like(bw["v"]), torch.empty_like(bw["h0"])
        fnS = lambda i: ck.fwd_chunked(bw["q"], bw["k"], bw["v"], bw["alpha"], bw["beta"],
                                       bw["h0"], path="simt", out=outS, hT=hS, workspace=wss)
        for i in range(2):
            fnS(i)
        ms_s = event_time_ms(fnS, nB, stream) / nB
        extras["simt_forward"] = {
            "workload": f"{w['name']} (B={B},T={T},H={H},dk=dv={dk}) with h0, CUDA-core path, "
                        "record form (16-token chunks, split-tf32 warp tiles)",
            "ms": round(ms_s, 3), "mtok_s": round(B * T / (ms_s / 1e3) / 1e6, 2),
            "over_forward": round(ms_s / ms_local, 1)}
        del bw, dout, dhT, wsb, wss, outS, hS

        # ---- batched decode: 256 sequences x 32 heads, dk = dv = 128 ------------------------
        wd = synth.WORKLOADS["decode_bf16"]
        N, Hd, steps_d = wd["N"], wd["H"], args.decode_steps
        Din = synth.torch_decode_inputs(steps_d, N, Hd, 128, 128, kind="ckda", dtype="bf16",
                                        seed=5000 + rank, device=dev)
        state = 0.02 * torch.randn((N, Hd, 128, 128), device=dev)
        outd = torch.empty((N, Hd, 128), dtype=torch.bfloat16, device=dev)
        fnD = lambda i: ck.decode_step(Din["q"][i], Din["k"][i], Din["v"][i], Din["alpha"][i],
                                       Din["beta"][i], state, out=outd)
        for i in range(3):
            fnD(i)
        torch.cuda.synchronize()
        t_dec0 = time.time()
        ms_dec = event_time_ms(fnD, steps_d, stream) / steps_d
        t_dec1 = time.time()
        time.sleep(0.12)
        clocks_dec = sampler.window(t_dec0, t_dec1)
        bytes_step = N * Hd * (2 * 128 * 128 * 4 + 3 * 256 + 512 + 4 + 256)
        dec_gbs = bytes_step / (ms_dec / 1e3) / 1e9
        extras["decode"] = {
            "workload": f"decode_bf16 (N={N},H={Hd},dk=dv=128, {steps_d} sequential steps)",
            "us_per_step": round(ms_dec * 1e3, 2), "GBps": round(dec_gbs, 1),
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(dec_gbs / hbm_peak, 4),
                         "traffic": ncu_traffic("decode_kernel"),
                         "algorithmic_bytes_per_launch": bytes_step},
            "clocks": clocks_dec}
        del Din, state
    sampler.stop()

    # ---- end to end through the C ABI with host buffers --------------------------------------
    # Every step copies its inputs from pinned host memory and reads its output back.  The steps
    # are pipelined the way a serving loop would run them: two device input sets and two outputs,
    # the host->device copies on one stream, the forward on the launching stream and the
    # device->host copies on a third, ordered by events, so that step i's copies overlap the
    # neighbouring steps' work.  The clock starts before the first copy and stops after the last
    # output has reached host memory.
    e2e = None
    if not args.no_extras:
        keys = ("q", "k", "v", "alpha", "beta")
        host = [{k: sets[i][k].cpu().pin_memory() for k in keys} for i in range(2)]
        out_host = [torch.empty((B, T, H, dv), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        dev_in = [{k: torch.empty_like(sets[0][k]) for k in keys} for _ in range(2)]
        dev_out = [torch.empty_like(out) for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host[0].values())
        d2h = out_host[0].numel() * out_host[0].element_size()
        s_h2d = torch.cuda.Stream(device=dev)
        s_d2h = torch.cuda.Stream(device=dev)
        ev = {n: [torch.cuda.Event() for _ in range(2)]
              for n in ("ready", "in_free", "out_done", "out_read")}

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_event(ev["in_free"][b])      # the forward of step i-2 read set b
                for k in keys:
                    dev_in[b][k].copy_(host[b][k], non_blocking=True)
                ev["ready"][b].record(s_h2d)
            stream.wait_event(ev["ready"][b])
            stream.wait_event(ev["out_read"][b])        # output b of step i-2 is on the host
            ck.fwd_chunked(dev_in[b]["q"], dev_in[b]["k"], dev_in[b]["v"], dev_in[b]["alpha"],
                           dev_in[b]["beta"], None, chunk=C, path="tc", out=dev_out[b], hT=hT,
                           workspace=ws)
            ev["in_free"][b].record(stream)
            ev["out_done"][b].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev["out_done"][b])
                out_host[b].copy_(dev_out[b], non_blocking=True)
                ev["out_read"][b].record(s_d2h)

        def e2e_time(n):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            s_h2d.wait_event(e0)
            for i in range(n):
                e2e_step(i)
            for b in range(2):
                stream.wait_event(ev["out_read"][b])
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)

        e2e_time(3)
        n_e2e = max(6, args.steps // 5)
        ms_e2e = e2e_time(n_e2e) / n_e2e
        ms_e2e = max_over_ranks(ms_e2e, dev, world)
        e2e = {"value": round(weak_scaling_mtok_s(B * T, world, ms_e2e), 3), "unit": "Mtok/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(ms_e2e, 4),
               "pipelining": "two input and two output buffers; host->device copies, the forward "
                             "and device->host copies on three streams ordered by events"}
        del host, out_host, dev_in, dev_out

    # ---- CPU baseline: the float64 oracle on a bounded sample (rank 0, one GPU) --------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_extras:
        mtok, cores, sample, _, _ = cpu_oracle_leg(20, 1, budget_s=20.0)
        cpu = {"value": round(mtok, 6), "unit": "Mtok/s", "cores": cores, "kind": "oracle",
               "sample": sample}
        # the same sample on one host thread (one head), and the long-context workload (one
        # head per core, T = 65536, RoPE, h0) on every core
        m1, c1, s1, _, _ = cpu_oracle_leg(5, 0, budget_s=10.0, threads=1, heads=1)
        cpu["one_core"] = {"value": round(m1, 6), "unit": "Mtok/s", "cores": c1, "sample": s1}
        wl = dict(synth.WORKLOADS["long_rope_bf16"], name="long_rope_bf16")
        mL, cL, sL, _, _ = cpu_oracle_leg(1, 0, budget_s=1.0, workload=wl)
        cpu["long_context"] = {"value": round(mL, 6), "unit": "Mtok/s", "cores": cL,
                               "sample": sL}

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "Mtok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"{w['name']} (B={B},T={T},H={H},dk=dv={dk},chunk={C},"
                                   f"{w['kind']} gates, no RoPE, h0=0)",
                       "global_batch": B * world, "seq_len": T, "heads": H,
                       "parallelism": f"replicas x{world} (independent batches, no collective)",
                       "l2": f"{N_ROTATE} input sets rotated per step "
                             f"({N_ROTATE * 80} MB > 126 MB L2)"},
            "roofline": roofline, "path_roofline": path_roofline, "kernels": kernels,
            # one ckda_tc_fused launch per timed step (plus the flag reset, a driver memset)
            "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": args.steps,
            "clocks": clocks, **extras}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
