#!/usr/bin/env python3
"""Benchmark of the GDN-2 mixer hot path on B200.

One step = a training forward + backward over the batch (B=8, T=4096, H=16,
dk=dv=128, bf16 tokens, fp32 state, do ~ N(0,1), dS_T = 0) -- the 1.3B-layer
shape of the pages: gdn2_chunk_fwd_save (the forward that keeps its
chunk-boundary states) + gdn2_chunk_bwd_saved (the gate-aware backward using
them).  The plain forward (prefill, gdn2_chunk_fwd) and the decode step
(B=256, H=16, fp32 state of 268 MB updated in place) are timed in the same
run and reported under "prefill" and "decode", and the long-sequence forward
(B=1, H=16, T = 8192, 32768 and 131072) under "long".  Inputs are seeded
synthetic data of the pages' distributions (gated_delta_rule_gdn2_b200.inputs;
the long-sequence inputs are drawn on the GPU from the same distributions);
they are larger than L2 (about 1 GB per step), so no separate flush is needed.
After the K timed steps, "sustained" repeats the step for at least a second
with the clocks sampled throughout.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs its own batch (weak scaling, no collective on
the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import tempfile
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, T, H, D = 8, 4096, 16, 128  # B can be lowered with --batch for profiling captures
DEC_B, DEC_H = 256, 16
LONG_TS = (8192, 32768, 131072)  # the long-sequence forward legs (B1 H16)
SUSTAINED_S = 1.0  # seconds of back-to-back steps after the timed ones
WORKLOAD = "train fwd+bwd B8 T4096 H16 dk=dv=128 bf16 (prefill and decode B256 H16 alongside)"
METRIC = "GDN-2 chunk fwd+bwd tokens/s & TFLOP/s (H16 dk=dv=128); decode state GB/s"
# algorithmic work per (token, head), d = 128, C = 64: dense-counted products and bytes read + written once
FLOP_FWD = 6 * D * D + 10 * 64 * D          # 180,224
FLOP_BWD = 524288 - (4 * D * D + 8 * 64 * D)  # 393,216: backward without the state recompute
BYTES_FWD = 7 * D * 2                        # q,k,v,log_alpha,b,w in + o out, bf16
BYTES_BWD = 13 * D * 2                       # 6 inputs + dO in, 6 gradients out, bf16
# (the chunk-boundary states and per-chunk tiles the training forward keeps
# for the backward are intermediates: counted in the ncu traffic, not here)
STATE_BYTES = D * D * 4


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def run_config(world):
    """The workload as both arms report it."""
    return {"workload": WORKLOAD, "global_batch": B * world, "seq_len": T, "heads": H, "dk": D, "dv": D,
            "chunk": 64, "parallelism": "dp%d (independent batches)" % world,
            "l2": "inputs larger than L2 (about 1 GB per step)"}


def max_over_ranks(ms, world, device=None):
    """The slowest rank's time (every rank calls this at the same point; one
    rank returns its own).  The data path has no collective: this is the only
    exchange, on the host side of the timing."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = bus_id
        self.proc = None
        # the samples go to a file of their own (GDN2_CLOCKS_DIR, else the temp directory)
        self.path = os.path.join(os.environ.get("GDN2_CLOCKS_DIR", tempfile.gettempdir()),
                                 "gdn2_clocks_%d.csv" % os.getpid())

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "100"]
            if self.bus_id:
                cmd[1:1] = ["-i", self.bus_id]
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# roofline inputs


def kernel_traffic(name):
    """DRAM bytes per launch of `name` from the committed ncu summary, or None
    when the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(name)
    if not d:
        return None
    hs = hashlib.sha256()
    for f in d["sources"]:
        p = os.path.join(ROOT, f)
        if not os.path.exists(p):
            return None
        hs.update(open(p, "rb").read())
    return d["bytes_per_launch"] if hs.hexdigest()[:16] == d["source_sha"] else None


# ---------------------------------------------------------------------------


def make_device_inputs(torch, dev):
    from gated_delta_rule_gdn2_b200.inputs import WORKLOADS, make_workload
    w = WORKLOADS["train"]
    w = type(w)(**{**w.__dict__, "B": B})
    x = make_workload(w)
    bf = lambda a: torch.from_numpy(a).to(device=dev, dtype=torch.bfloat16)
    d = {n: bf(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "dO")}
    d["S0"] = torch.from_numpy(x["S0"]).to(dev)
    return x, d


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import gated_delta_rule_gdn2_b200 as g

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    x, d = make_device_inputs(torch, dev)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    grads = [torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev) for _ in range(6)]
    dS0 = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    nfw = g.gdn2_chunk_fwd_workspace(B, T, H, D, D, g.GDN2_BF16)
    nbw = g.gdn2_chunk_bwd_saved_workspace(B, T, H, D, D, g.GDN2_BF16)
    nst = g.gdn2_chunk_states_bytes(B, T, H, D, D, g.GDN2_BF16)
    wsf = torch.empty(max(nfw, 16), dtype=torch.uint8, device=dev)
    wsb = torch.empty(max(nbw, 16), dtype=torch.uint8, device=dev)
    states = torch.empty(nst, dtype=torch.uint8, device=dev)
    toks = [d[n] for n in ("q", "k", "v", "log_alpha", "b", "w")]

    def fwd():
        st = g.gdn2_chunk_fwd_save(*toks, d["S0"], o, ST, states, B, T, H, D, D, g.GDN2_BF16, wsf, nfw, sh)
        assert st == 0, st

    def bwd():
        st = g.gdn2_chunk_bwd_saved(*toks, d["S0"], d["dO"], None, states, *grads, dS0, B, T, H, D, D,
                                    g.GDN2_BF16, wsb, nbw, sh)
        assert st == 0, st

    def prefill():
        st = g.gdn2_chunk_fwd(*toks, d["S0"], o, ST, B, T, H, D, D, g.GDN2_BF16, wsf, nfw, sh)
        assert st == 0, st

    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    marks = [(ev(), ev(), ev()) for _ in range(args.steps)]
    bus = None
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        bus = u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    t_start, t_end = ev(), ev()
    with ClockSampler(None if bus is None else str(bus)) as clk:
        time.sleep(0.3)
        t_start.record(stream)
        for m in marks:
            m[0].record(stream)
            fwd()
            m[1].record(stream)
            bwd()
            m[2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        # ---- sustained: the same step back to back for at least SUSTAINED_S
        # seconds (the clocks are sampled across both regions)
        n_sus = 0
        s0, s1 = ev(), ev()
        s0.record(stream)
        t_wall = time.perf_counter()
        while time.perf_counter() - t_wall < SUSTAINED_S:
            for _ in range(50):
                fwd()
                bwd()
            n_sus += 50
            s1.record(stream)
            s1.synchronize()
        sus_ms = s0.elapsed_time(s1) / n_sus
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    assert g.gdn2_get_device_status() == 0
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = statistics.mean(m[0].elapsed_time(m[1]) for m in marks)
    bwd_ms = statistics.mean(m[1].elapsed_time(m[2]) for m in marks)
    total_ms = max_over_ranks(total_ms, world, dev)
    sus_ms = max_over_ranks(sus_ms, world, dev)
    ms_step = total_ms / args.steps

    # ---- prefill forward (gdn2_chunk_fwd, no states kept)
    for _ in range(3):
        prefill()
    torch.cuda.synchronize()
    p0, p1 = ev(), ev()
    p0.record(stream)
    for _ in range(args.steps):
        prefill()
    p1.record(stream)
    torch.cuda.synchronize()
    pre_ms = p0.elapsed_time(p1) / args.steps

    # ---- long-sequence forward (B1 H16: 16 sequences) at T = 8192, 32768, 131072;
    # inputs drawn on the device (the same distributions as the host recipe)
    from gated_delta_rule_gdn2_b200.inputs import WORKLOADS, make_inputs_device
    wl = WORKLOADS["long"]
    xl = make_inputs_device(1, max(LONG_TS), H, D, D, seed=wl.seed, device=dev, alpha_mu=wl.alpha_mu)
    long_legs = []
    for TL in LONG_TS:
        tl = [xl[n][:, :TL].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")]
        ol = torch.empty((1, TL, H, D), dtype=torch.bfloat16, device=dev)
        STl = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
        nlw = g.gdn2_chunk_fwd_workspace(1, TL, H, D, D, g.GDN2_BF16)
        wsl = torch.empty(max(nlw, 16), dtype=torch.uint8, device=dev)

        def long_fwd():
            st = g.gdn2_chunk_fwd(*tl, xl["S0"], ol, STl, 1, TL, H, D, D, g.GDN2_BF16, wsl, nlw, sh)
            assert st == 0, st

        for _ in range(3):
            long_fwd()
        torch.cuda.synchronize()
        reps = max(3, min(args.steps, int(2e6 // TL)))
        l0, l1 = ev(), ev()
        l0.record(stream)
        for _ in range(reps):
            long_fwd()
        l1.record(stream)
        torch.cuda.synchronize()
        ms = l0.elapsed_time(l1) / reps
        nbytes = TL * H * BYTES_FWD + 2 * H * STATE_BYTES
        long_legs.append({"T": TL, "ms": ms, "tokens_per_s": TL / (ms * 1e-3), "gbs": nbytes / (ms * 1e-3) / 1e9,
                          "reps": reps})
        del tl, ol, wsl
    del xl
    assert g.gdn2_get_device_status() == 0

    # ---- decode step, state of B256 H16 d128 resident and updated in place
    from gated_delta_rule_gdn2_b200.inputs import decode_initial_state, decode_step_inputs
    Sdec = torch.from_numpy(decode_initial_state(DEC_B, DEC_H, D, D, seed=1002)).to(dev)
    dec_inputs = []
    for s in range(4):
        xs = decode_step_inputs(DEC_B, DEC_H, D, D, seed=1002, step=s)
        dec_inputs.append([torch.from_numpy(xs[n]).to(device=dev, dtype=torch.bfloat16)
                           for n in ("q", "k", "v", "log_alpha", "b", "w")])
    odec = torch.empty((DEC_B, DEC_H, D), dtype=torch.bfloat16, device=dev)
    ndec = 1024  # one timed block of 1024 steps (four pre-staged token sets in turn)

    def dec(i):
        st = g.gdn2_decode_step(*dec_inputs[i % 4], Sdec, odec, DEC_B, DEC_H, D, D, g.GDN2_BF16, sh)
        assert st == 0, st

    for i in range(8):
        dec(i)
    torch.cuda.synchronize()
    d0, d1 = ev(), ev()
    d0.record(stream)
    for i in range(ndec):
        dec(i)
    d1.record(stream)
    torch.cuda.synchronize()
    dec_us = d0.elapsed_time(d1) * 1000.0 / ndec
    dec_bytes = DEC_B * DEC_H * (2 * STATE_BYTES + 8 * D * 2)

    # ---- end to end through the public API with pinned host buffers: every
    # step uploads its inputs, runs chunk_fwd(save_states=True) + chunk_bwd and
    # downloads every output; uploads and downloads run on their own streams
    # into preallocated pinned buffers, so step i + 1's upload overlaps step
    # i's compute and download (PCIe is full duplex)
    host = {n: torch.from_numpy(x[n]).to(torch.bfloat16).pin_memory() for n in
            ("q", "k", "v", "log_alpha", "b", "w", "dO")}
    host["S0"] = torch.from_numpy(x["S0"]).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    e2e_steps = max(2, min(args.steps, 8))
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    dev_in = [{n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in host.items()} for _ in range(2)]
    in_free = [ev(), ev()]
    for e in in_free:
        e.record(stream)
    outs_host = [None, None]
    keep = [None, None]

    def e2e_step(i):
        j = i % 2
        buf = dev_in[j]
        with torch.cuda.stream(up):
            up.wait_event(in_free[j])
            for n, t in host.items():
                buf[n].copy_(t, non_blocking=True)
            landed = ev()
            landed.record(up)
        stream.wait_event(landed)
        tk = [buf[n] for n in ("q", "k", "v", "log_alpha", "b", "w")]
        oo, SS, stt = g.chunk_fwd(*tk, S0=buf["S0"], save_states=True)
        gg = g.chunk_bwd(*tk, buf["S0"], buf["dO"], states=stt)
        res = [oo, SS] + [gg[n] for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")]
        in_free[j].record(stream)
        done = ev()
        done.record(stream)
        if outs_host[j] is None:
            outs_host[j] = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in res]
        with torch.cuda.stream(down):
            down.wait_event(done)
            for r, hb in zip(res, outs_host[j]):
                hb.copy_(r, non_blocking=True)
                r.record_stream(down)
        keep[j] = res
        return res

    res = e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    d2h = sum(r.numel() * r.element_size() for r in res)
    del res
    e0, e1 = ev(), ev()
    e0.record(stream)
    up.wait_event(e0)  # the first upload starts inside the timed region
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    hbm, tf_burst, tf_sus, src = peaks()
    tokens = B * T * world
    th = B * T * H
    # algorithmic bytes: token tensors in and out once, the fp32 S0 read and S_T
    # (or dS0) written once; the states kept between the passes are not counted
    fwd_gbs = (th * BYTES_FWD + 2 * B * H * STATE_BYTES) / (fwd_ms * 1e-3) / 1e9
    bwd_gbs = (th * BYTES_BWD + 2 * B * H * STATE_BYTES) / (bwd_ms * 1e-3) / 1e9
    pre_gbs = (th * BYTES_FWD + 2 * B * H * STATE_BYTES) / (pre_ms * 1e-3) / 1e9
    for leg in long_legs:
        leg["hbm_frac"] = leg["gbs"] / hbm
        leg["tflops"] = leg["T"] * H * FLOP_FWD / (leg["ms"] * 1e-3) / 1e12
        leg["tensor_frac_of_bf16"] = leg["tflops"] / tf_burst
    dom = "bwd" if bwd_ms >= fwd_ms else "fwd"
    kname = {"fwd": "chunk_fwd_tc_kernel (with state output)", "bwd": "chunk_bwd_tc_kernel"}[dom]
    achieved = bwd_gbs if dom == "bwd" else fwd_gbs
    traffic = kernel_traffic("chunk_fwd_tc_kernel" if dom == "fwd" else "chunk_bwd_tc_kernel")
    if traffic is not None:
        traffic = traffic * B / 8  # the committed figure is per launch at B = 8
    clocks = clk.summary()
    fwd_tf = th * FLOP_FWD / (fwd_ms * 1e-3) / 1e12
    bwd_tf = th * FLOP_BWD / (bwd_ms * 1e-3) / 1e12
    out = {
        "metric": METRIC,
        "value": tokens / (ms_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded normals of the pages' distributions; no dataset)",
        "config": run_config(world),
        "tflops": th * world * (FLOP_FWD + FLOP_BWD) / (ms_step * 1e-3) / 1e12,
        # every tensor fraction below is against the measured bf16 burst peak
        # (each leg is timed over well under a second); HBM fractions against
        # the measured copy bandwidth
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": tf_burst, "source": src},
        "breakdown": {
            "fwd_save_ms": fwd_ms, "bwd_saved_ms": bwd_ms,
            "fwd_tflops": fwd_tf, "fwd_tensor_frac": fwd_tf / tf_burst,
            "fwd_gbs": fwd_gbs, "fwd_hbm_frac": fwd_gbs / hbm,
            "bwd_tflops": bwd_tf, "bwd_tensor_frac": bwd_tf / tf_burst,
            "bwd_gbs": bwd_gbs, "bwd_hbm_frac": bwd_gbs / hbm,
        },
        "sustained": {"ms_per_step": sus_ms, "steps": n_sus, "seconds": sus_ms * n_sus / 1e3,
                      "tokens_per_s": tokens / (sus_ms * 1e-3)},
        "long": long_legs,
        "prefill": {"workload": "B8 T4096 H16 dk=dv=128 forward (gdn2_chunk_fwd)", "ms": pre_ms,
                    "tokens_per_s": B * T / (pre_ms * 1e-3), "tflops": th * FLOP_FWD / (pre_ms * 1e-3) / 1e12,
                    "gbs": pre_gbs, "hbm_frac": pre_gbs / hbm,
                    "tensor_frac_of_bf16": th * FLOP_FWD / (pre_ms * 1e-3) / 1e12 / tf_burst},
        "decode": {"workload": "B256 H16 dk=dv=128, fp32 state in place", "us_per_step": dec_us,
                   "tokens_per_s": DEC_B / (dec_us * 1e-6), "state_gbs": dec_bytes / (dec_us * 1e-6) / 1e9,
                   "hbm_frac": dec_bytes / (dec_us * 1e-6) / 1e9 / hbm, "peak_gbs": hbm},
        "roofline": {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic,
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs, copy)" % src,
                     "tensor_frac_of_bf16": (fwd_tf if dom == "fwd" else bwd_tf) / tf_burst},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * args.steps,  # chunk_fwd_tc_kernel (with states) + chunk_bwd_tc_kernel per step
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(x)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def cpu_baseline(x, target_s=12.0):
    """The fp64 oracle (as it stands) on the host cores: fwd + bwd of a sample
    of whole heads of the same workload, scaled to tokens/s of the batch."""
    import oracle
    cores = oracle.num_threads()
    heads = [(b, h) for b in range(B) for h in range(H)]
    n = min(len(heads), max(2, cores))
    sel = heads[:n]
    names = ("q", "k", "v", "log_alpha", "b", "w")
    xs = {m: np.stack([x[m][b, :, h] for b, h in sel])[:, :, None] for m in names + ("dO",)}
    S0 = np.stack([x["S0"][b, h] for b, h in sel])[:, None]
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.fwd(*[xs[m] for m in names], S0)
        oracle.bwd(*[xs[m] for m in names], S0, xs["dO"], None)
        reps += 1
        el = time.perf_counter() - t0
        if el > target_s or reps >= 100:
            break
    tok = reps * n * T / H  # head-tokens / H = tokens of the batch
    return {"value": tok / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d whole heads (T=%d) of the B%d H%d batch, fwd+bwd, %d rep(s), %.1f s" % (n, T, B, H, reps, el)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from gated_delta_rule_gdn2_b200.inputs import WORKLOADS, make_workload
    w = WORKLOADS["train"]
    x = make_workload(type(w)(**{**w.__dict__, "B": B}))
    vals = []
    cb = None
    per_step = max(1.0, min(5.0, 150.0 / max(1, args.steps)))
    for _ in range(args.steps):
        cb = cpu_baseline(x, target_s=per_step)
        vals.append(cb["value"])
    v = statistics.mean(vals)
    cb["value"] = v
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": B * T / v * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": run_config(world),
           "cpu_baseline": cb,
           "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=8,
                    help="batch of the fwd+bwd workload (8 = the benchmark; smaller only for ncu captures)")
    args = ap.parse_args()
    global B, WORKLOAD
    if args.batch != B:
        B = args.batch
        WORKLOAD = WORKLOAD.replace("B8 ", "B%d " % B)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
