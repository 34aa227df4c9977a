"""Benchmark of the gated delta rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one chunkwise forward (``gdn_chunk_fwd``) over the headline workload
(B=4, H=16, T=4096, Dk=Dv=128, chunk 64, bf16 q/k/v/o, float32 gates and state),
inputs resident in HBM.  The value is tokens/s over all ranks (weak scaling:
every rank runs its own copy of the workload, no collective on the data path).
The same run also times the recurrent decode step (batch 256, H 16, d 128,
float32 state in HBM updated in place) and reports its HBM bandwidth.

Rank 0 prints one JSON line.  ``--impl reference`` times the float64 CPU oracle
(the only other implementation of the rule) on a bounded sample of the same
workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_130_b200 import inputs as I  # noqa: E402

METRIC = "GDN chunk fwd tokens/s (bf16,H=16,d=128,T=4K); % TC peak; decode HBM GB/s"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def measured_traffic(path: str, w):
    """DRAM bytes of one call (both tcgen05-path kernels) from the committed ncu
    summary, or None if the call is not the captured workload or the kernel sources
    changed since the capture."""
    import hashlib
    f = os.path.join(ROOT, "profiles", "traffic_gdn_chunk_fwd_tc.txt")
    if path != "tcgen05" or not os.path.exists(f):
        return None
    value, ok = None, True
    for line in open(f):
        line = line.strip()
        if line.startswith("workload:"):
            name = line.split(":", 1)[1].strip()
            ok = ok and name in I.WORKLOADS and I.workload(name) == w
        elif line.startswith("dram_bytes_per_call:"):
            value = float(line.split(":", 1)[1])
        elif line.startswith("sha256 "):
            rel, digest = line[len("sha256 "):].split(":", 1)
            src = os.path.join(ROOT, rel.strip())
            if not os.path.exists(src) or \
                    hashlib.sha256(open(src, "rb").read()).hexdigest() != digest.strip():
                ok = False
    return value if ok else None


def chunk_flops(w) -> float:
    """Dense contraction FLOPs of the chunkwise algorithm, 2(3 C Dk + 2 C Dv + 3 Dk Dv)
    per token per head (the gated Gram matrix, the WY factors, the state update and
    the output)."""
    C = w.chunk
    return 2.0 * (3 * C * w.Dk + 2 * C * w.Dv + 3 * w.Dk * w.Dv) * w.B * w.T * w.H


def chunk_bytes(w, has_s0: bool) -> float:
    """Compulsory HBM bytes of one chunkwise forward: q, k, v read and o written
    once in the element type, both gates read once (float32), S0 read if given,
    S_T written (float32)."""
    esz = 2 if w.dtype == "bf16" else 4
    tok = w.B * w.T * w.H
    state = w.B * w.H * w.Dv * w.Dk * 4
    return tok * (esz * (2 * w.Dk + 2 * w.Dv) + 8) + state * (2 if has_s0 else 1)


def bwd_bytes(w, has_s0: bool) -> float:
    """Compulsory HBM bytes of one chunkwise backward: q, k, v and d_o read and dq,
    dk, dv written once in the element type, both gates read and both gate
    gradients written (float32); S0 (if given) and dS_T read, dS0 written."""
    esz = 2 if w.dtype == "bf16" else 4
    tok = w.B * w.T * w.H
    state = w.B * w.H * w.Dv * w.Dk * 4
    return tok * (esz * (4 * w.Dk + 3 * w.Dv) + 16) + state * (3 if has_s0 else 2)


def decode_bytes(w) -> float:
    """Compulsory HBM bytes of one decode step: the float32 state read and written,
    q, k, v read and o written in the element type, the two gates read."""
    esz = 2 if w.dtype == "bf16" else 4
    heads = w.B * w.H
    return heads * (8 * w.Dv * w.Dk + esz * (2 * w.Dk + 2 * w.Dv) + 8)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "reasons": reasons, "samples": len(rows)}


def _dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def _max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(ms_local: float, steps: int, tokens_per_rank: int, world: int, device):
    """Whole-job tokens/s and ms/step from this rank's device time: every rank
    processes its own batch, the job takes as long as the slowest rank."""
    ms_max = _max_over_ranks(ms_local, world, device)
    ms_step = ms_max / steps
    return world * tokens_per_rank / (ms_step * 1e-3), ms_step


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def time_loop(fn, steps, stream, world):
    """Device time of exactly `steps` calls, bracketed by barrier + synchronize."""
    _barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    return start.elapsed_time(end)  # ms


def cpu_baseline(w, inp, budget_s=15.0):
    """The float64 oracle on a bounded sample of whole heads, all host cores."""
    from oracle import oracle as O
    ncores = O.default_threads()
    one = I.sample_units(w, 1)
    t0 = time.perf_counter()
    O.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], units=one,
              nthreads=1)
    t_head = time.perf_counter() - t0
    n = max(1, min(w.B * w.H, int(budget_s / max(t_head, 1e-6))))
    units = I.sample_units(w, n)
    t0 = time.perf_counter()
    O.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], units=units,
              nthreads=ncores)
    wall = time.perf_counter() - t0
    tokens = len(units) * w.T / w.H  # token-heads processed, expressed in tokens
    return {"value": tokens / wall, "unit": UNIT, "cores": min(ncores, len(units)), "kind": "oracle",
            "sample": f"{len(units)} of {w.B * w.H} (b,h) heads, all {w.T} tokens each "
                      f"({wall:.2f} s wall); tokens/s = heads*T/H / wall"}


def run_reference(args):
    """--impl reference: the float64 oracle, timed on the host cores, rank 0 only."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as O
    w = I.workload(I.HEADLINE)
    inp = I.chunk_inputs(w)
    ncores = O.default_threads()
    # each step: the first n_tok tokens of a sample of heads, sized so that the
    # whole run takes about two minutes
    per_step = 120.0 / max(1, args.steps + args.warmup)
    units = I.sample_units(w, min(w.B * w.H, ncores))
    probe_tok = min(w.T, 256)
    sl = lambda x: x[:, :probe_tok].contiguous()
    t0 = time.perf_counter()
    O.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]), sl(inp["beta"]),
              None, units=units, nthreads=ncores)
    t_probe = max(time.perf_counter() - t0, 1e-6)
    n_tok = int(max(1, min(w.T, probe_tok * per_step / t_probe)))
    sl = lambda x: x[:, :n_tok].contiguous()
    args_ = [sl(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    for _ in range(args.warmup):
        O.forward(*args_, None, units=units, nthreads=ncores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.forward(*args_, None, units=units, nthreads=ncores)
    wall = time.perf_counter() - t0
    tokens = args.steps * len(units) * n_tok / w.H
    value = tokens / wall
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} T={w.T} Dk={w.Dk} Dv={w.Dv} "
                               f"chunk={w.chunk} {w.dtype}", "global_batch": w.B, "seq_len": w.T,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(ncores, len(units)),
                         "kind": "oracle",
                         "sample": f"per step: first {n_tok} tokens of {len(units)} of "
                                   f"{w.B * w.H} heads; tokens/s = heads*tokens/H / wall"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    world, rank, local = _dist_setup(args.gpus)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from gated_delta_rule_130_b200 import binding as G

    pk, pk_kind = peaks()
    w = parse_workload(args.workload) if args.chunk_only else I.workload(I.HEADLINE)
    inp_cpu = I.chunk_inputs(w, seed=w.seed + rank)
    inp = {n: (t.to(device) if t is not None else None) for n, t in inp_cpu.items()}
    path = G.chunk_fwd_path(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk, w.torch_dtype)
    # the parallel tile (UT) kernel and the sequential kernel; a split sequence adds
    # the map initialisation, the two first-pass walks and the scan
    variant = (G.chunk_fwd_variant(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk, w.torch_dtype)
               if path == "tcgen05" else None)
    launches_per_step = 6 if variant == "split" else 2
    o = torch.empty((w.B, w.T, w.H, w.Dv), dtype=w.torch_dtype, device=device)
    S_T = torch.empty((w.B, w.H, w.Dv, w.Dk), dtype=torch.float32, device=device)
    ws_bytes = G.chunk_fwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk, w.torch_dtype)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        G.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                    chunk=w.chunk, out=o, S_T=S_T, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    steps = args.steps
    if steps is None:  # about three seconds of timed work
        t_one = time_loop(step, 10, stream, 1) / 10
        steps = int(min(50000, max(100, 3000.0 / max(t_one, 1e-3))))
        steps = int(_max_over_ranks(steps, world, device))
    with ClockSampler(local) as clk:
        # the sampler polls every 100 ms: hold this load for about 1.5 s before
        # the timed region so that the clock record covers it even when the
        # timed region itself is only milliseconds long
        t_end = time.perf_counter() + 1.5
        while time.perf_counter() < t_end:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        ms = time_loop(step, steps, stream, world)
    clocks = clk.summary()
    clocks["window"] = "1.5 s of the same step back to back, then the timed region"
    tokens = w.B * w.T
    value, ms_step = weak_scaling_value(ms, steps, tokens, world, device)

    # roofline of the whole call (tcgen05 path: the parallel UT-transform kernel
    # and the sequential tensor-core kernel; SIMT path: its two CUDA-core kernels),
    # i.e. both launches together count against the algorithmic bytes and FLOPs
    F = chunk_flops(w)
    Bytes = chunk_bytes(w, inp["S0"] is not None)
    t_s = (ms / steps) * 1e-3
    gbs = Bytes / t_s / 1e9
    tflops = F / t_s / 1e12
    hbm_peak = pk["hbm_gbs"]
    tc_peak = pk["bf16_tflops"]
    roofline = {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": gbs / hbm_peak, "traffic": measured_traffic(path, w),
                "kernel": f"gdn_chunk_fwd ({path}, {launches_per_step} launches/step, timed together)",
                "algorithmic_bytes": Bytes, "peak_source": f"{pk_kind} hbm_gbs",
                "tc": {"achieved": tflops, "peak": tc_peak, "unit": "TFLOP/s",
                       "frac": tflops / tc_peak, "flops": F,
                       "peak_source": f"{pk_kind} bf16_tflops (burst)"}}

    decode, e2e = None, None
    if not args.chunk_only:  # (--chunk-only: the chunkwise step alone, for profiling)
        # decode step: batch 256, H 16, d 128, 1000 steps, state resident in HBM
        wd = I.workload("decode_b256")
        S = I.decode_state(wd, device=device)
        dec_in = [{n: t.to(device) for n, t in I.decode_step_inputs(wd, t).items()} for t in range(8)]
        od = torch.empty((wd.B, wd.H, wd.Dv), dtype=wd.torch_dtype, device=device)
        it = [0]

        def dstep():
            x = dec_in[it[0] % len(dec_in)]
            it[0] += 1
            G.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, out=od)

        for _ in range(20):
            dstep()
        dms = time_loop(dstep, wd.steps, stream, world)
        dms_max = _max_over_ranks(dms, world, device)
        d_us = 1e3 * dms / wd.steps
        d_gbs = decode_bytes(wd) / (d_us * 1e-6) / 1e9
        decode = {"workload": f"decode_b256: batch={wd.B} H={wd.H} Dk={wd.Dk} Dv={wd.Dv} bf16 "
                              f"q/k/v/o, f32 state in place, {wd.steps} steps",
                  "us_per_step": 1e3 * dms_max / wd.steps, "achieved": d_gbs, "unit": "GB/s",
                  "peak": hbm_peak, "frac": d_gbs / hbm_peak, "bytes_per_step": decode_bytes(wd),
                  "gpu_launches": wd.steps}

        # end to end through the public API with host buffers: every step copies its
        # inputs in from pinned host memory, makes the call and copies o and S_T back.
        # Consecutive steps are pipelined as a user would: uploads on one copy stream,
        # read-backs on another, the call on the launching stream, two buffer sets,
        # so one step's read-back overlaps the next step's upload (PCIe is duplex)
        host = {n: (t.pin_memory() if t is not None else None) for n, t in inp_cpu.items()}
        o_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        s_h = [torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory() for _ in range(2)]
        dev_in = [{n: (torch.empty_like(t, device=device) if t is not None else None)
                   for n, t in host.items()} for _ in range(2)]
        dev_o = [torch.empty_like(o) for _ in range(2)]
        dev_s = [torch.empty_like(S_T) for _ in range(2)]
        up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        uploaded, computed, read_back = ev(), ev(), ev()
        it = [0]

        def e2e_step():
            i, b = it[0], it[0] % 2
            it[0] += 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[b])        # step i - 2 has read these inputs
                for n, t in host.items():
                    if t is not None:
                        dev_in[b][n].copy_(t, non_blocking=True)
                uploaded[b].record(up)
            stream.wait_event(uploaded[b])
            if i >= 2:
                stream.wait_event(read_back[b])       # step i - 2's outputs are home
            d_ = dev_in[b]
            G.chunk_fwd(d_["q"], d_["k"], d_["v"], d_["log_alpha"], d_["beta"], d_["S0"],
                        chunk=w.chunk, out=dev_o[b], S_T=dev_s[b], workspace=ws)
            computed[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                o_h[b].copy_(dev_o[b], non_blocking=True)
                s_h[b].copy_(dev_s[b], non_blocking=True)
                read_back[b].record(down)

        def e2e_time(n):
            """Device time of n pipelined steps: from the first upload to the last read-back."""
            _barrier(world)
            torch.cuda.synchronize()
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(stream)
            up.wait_stream(stream)
            for _ in range(n):
                e2e_step()
            stream.wait_stream(up)
            stream.wait_stream(down)
            end.record(stream)
            torch.cuda.synchronize()
            _barrier(world)
            return start.elapsed_time(end)

        e2e_steps = max(6, min(steps, 30))
        e2e_time(3)
        ems = _max_over_ranks(e2e_time(e2e_steps), world, device)
        h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
        d2h = o_h[0].numel() * o_h[0].element_size() + s_h[0].numel() * s_h[0].element_size()
        e2e = {"value": world * tokens / (ems / e2e_steps * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "pipelining": "two buffer sets; uploads, calls and read-backs on three streams"}

    # the optional input prologue (q, k L2-normalised and gates given as logits),
    # fused into the kernels, against the plain call and against preparing the
    # inputs in a separate pass (torch device ops) before the plain call
    prologue = None
    if not args.chunk_only:
        raw = {n: (t.to(device) if t is not None else None)
               for n, t in I.raw_chunk_inputs(w, seed=w.seed + rank).items()}
        ws_p = torch.empty(max(G.chunk_fwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk,
                                                          w.torch_dtype, True, True), 1),
                           dtype=torch.uint8, device=device)

        def fused_step():
            G.chunk_fwd(raw["q"], raw["k"], raw["v"], raw["log_alpha"], raw["beta"], raw["S0"],
                        chunk=w.chunk, out=o, S_T=S_T, workspace=ws_p, l2norm_qk=True,
                        gate_logits=True)

        def unfused_step():
            F = torch.nn.functional
            qn = F.normalize(raw["q"].float(), dim=-1, eps=1e-6).to(w.torch_dtype)
            kn = F.normalize(raw["k"].float(), dim=-1, eps=1e-6).to(w.torch_dtype)
            la = -F.softplus(raw["log_alpha"])
            be = torch.sigmoid(raw["beta"])
            G.chunk_fwd(qn, kn, raw["v"], la, be, raw["S0"], chunk=w.chunk, out=o, S_T=S_T,
                        workspace=ws)

        n_p = max(20, min(steps, 400))
        for _ in range(3):
            fused_step()
            unfused_step()
        f_ms = _max_over_ranks(time_loop(fused_step, n_p, stream, world), world, device) / n_p
        u_ms = _max_over_ranks(time_loop(unfused_step, n_p, stream, world), world, device) / n_p
        prologue = {"what": "raw q, k and gate logits; normalisation and activations fused into "
                            "the kernels (l2norm_qk, gate_logits)",
                    "fused_ms_per_step": f_ms, "plain_ms_per_step": ms_step,
                    "unfused_prepass_ms_per_step": u_ms,
                    "fused_tokens_per_s": world * tokens / (f_ms * 1e-3), "steps": n_p}

    # packed variable-length batch of the same token count: 12 sequences of mixed
    # lengths (the serving form), one call over all of them
    varlen = None
    if not args.chunk_only:
        c = I.VARLEN_SERVING
        lengths = I.varlen_lengths(c["n"], c["total"], c["seed"])
        vin = I.varlen_inputs(lengths, c["H"], c["Dk"], c["Dv"], "bf16", seed=c["seed"] + rank,
                              device=device)
        cu = vin["cu_seqlens"]
        cu_d = torch.tensor(cu, dtype=torch.int32, device=device)
        vo = torch.empty((c["total"], c["H"], c["Dv"]), dtype=torch.bfloat16, device=device)
        vS = torch.empty((c["n"], c["H"], c["Dv"], c["Dk"]), dtype=torch.float32, device=device)
        vws = torch.empty(max(G.chunk_fwd_varlen_workspace_size(cu, c["H"], c["Dk"], c["Dv"]), 1),
                          dtype=torch.uint8, device=device)

        def varlen_step():
            G.chunk_fwd_varlen(vin["q"], vin["k"], vin["v"], vin["log_alpha"], vin["beta"], cu,
                               out=vo, S_T=vS, workspace=vws, cu_seqlens_device=cu_d)

        n_v = max(20, min(steps, 400))
        for _ in range(3):
            varlen_step()
        v_ms = _max_over_ranks(time_loop(varlen_step, n_v, stream, world), world, device) / n_v
        varlen = {"workload": f"{c['n']} packed sequences, {c['total']} tokens (lengths "
                              f"{min(lengths)}..{max(lengths)}), H={c['H']} Dk={c['Dk']} "
                              f"Dv={c['Dv']} bf16, S0=0",
                  "lengths": lengths, "ms_per_step": v_ms,
                  "tokens_per_s": world * c["total"] / (v_ms * 1e-3), "steps": n_v,
                  "path": "tcgen05" if G.chunk_fwd_path(1, max(lengths), c["H"], c["Dk"], c["Dv"])
                  == "tcgen05" else "simt"}

    # chunkwise backward of the headline call (given dL/do and dL/dS_T)
    backward = None
    if not args.chunk_only:
        gen = torch.Generator().manual_seed(w.seed + 99 + rank)
        bdo = torch.randn((w.B, w.T, w.H, w.Dv), generator=gen).to(w.torch_dtype).to(device)
        bdS = torch.randn((w.B, w.H, w.Dv, w.Dk), generator=gen).to(device)
        bws = torch.empty(max(G.chunk_bwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk,
                                                         w.torch_dtype), 1),
                          dtype=torch.uint8, device=device)

        def bwd_step():
            G.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                        bdo, bdS, chunk=w.chunk, workspace=bws)

        for _ in range(3):
            bwd_step()
        n_b = 20
        b_ms = _max_over_ranks(time_loop(bwd_step, n_b, stream, world), world, device) / n_b
        bb = bwd_bytes(w, inp["S0"] is not None)
        b_gbs = bb / (b_ms * 1e-3) / 1e9
        b_path = G.chunk_bwd_path(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk, w.torch_dtype)
        backward = {"workload": "headline_T4k backward: dq, dk, dv, dlog_alpha, dbeta, dS0 "
                                "from d_o and dS_T",
                    "path": b_path,
                    "kernels": BWD_KERNELS[b_path],
                    "ms_per_step": b_ms, "tokens_per_s": world * tokens / (b_ms * 1e-3),
                    "achieved": b_gbs, "unit": "GB/s", "peak": hbm_peak,
                    "frac": b_gbs / hbm_peak, "algorithmic_bytes": bb, "steps": n_b,
                    "gpu_launches": len(BWD_KERNELS[b_path]) * n_b}

    # channel-wise gates (decay per key channel, erase and write gates) on the
    # headline shape, and their decode step at batch 256
    channel_wise = None
    if not args.chunk_only:
        cin = I.cw_inputs(w, seed=w.seed + rank, device=device)
        cws = torch.empty(max(G.chunk_fwd_cw_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk,
                                                            w.torch_dtype), 1),
                          dtype=torch.uint8, device=device)

        def cw_step():
            G.chunk_fwd_cw(cin["q"], cin["k"], cin["v"], cin["log_alpha"], cin["b"], cin["w"],
                           cin["S0"], chunk=w.chunk, out=o, S_T=S_T, workspace=cws)

        for _ in range(3):
            cw_step()
        n_c = 10
        c_ms = _max_over_ranks(time_loop(cw_step, n_c, stream, world), world, device) / n_c
        esz = 2
        c_bytes = w.B * w.T * w.H * (esz * (2 * w.Dk + 2 * w.Dv) + 4 * (2 * w.Dk + w.Dv)) + \
            w.B * w.H * w.Dv * w.Dk * 4
        wd = I.workload("decode_b256")
        dcin = I.cw_inputs(I.workload("decode_b256", T=1, s0_law="normal002"), device=device)
        one = lambda x: x[:, 0].contiguous()
        xq, xk, xv, xl, xb, xw = (one(dcin[n]) for n in ("q", "k", "v", "log_alpha", "b", "w"))
        Sd = dcin["S0"].clone()
        od_cw = torch.empty((wd.B, wd.H, wd.Dv), dtype=wd.torch_dtype, device=device)

        def cw_dstep():
            G.decode_step_cw(xq, xk, xv, xl, xb, xw, Sd, out=od_cw)

        for _ in range(10):
            cw_dstep()
        n_d = 200
        cd_us = 1e3 * _max_over_ranks(time_loop(cw_dstep, n_d, stream, world), world,
                                      device) / n_d
        cd_bytes = wd.B * wd.H * (8 * wd.Dv * wd.Dk + esz * (2 * wd.Dk + 2 * wd.Dv) +
                                  4 * (2 * wd.Dk + wd.Dv))
        cw_path = G.chunk_fwd_cw_path(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk, w.torch_dtype)
        channel_wise = {
            "workload": "headline_T4k shape with a decay and an erase gate per key channel and "
                        "a write gate per value channel (float32 gates)",
            "path": ("tcgen05: per-chunk kernel (16-row blocks of the channel-wise decays, "
                     "mma.sync) + sequential tcgen05 kernel, 2 launches per call"
                     if cw_path == "tcgen05" else "CUDA cores, float32 arithmetic (2 launches)"),
            "ms_per_step": c_ms, "tokens_per_s": world * tokens / (c_ms * 1e-3),
            "achieved": c_bytes / (c_ms * 1e-3) / 1e9, "unit": "GB/s",
            "frac": c_bytes / (c_ms * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes": c_bytes,
            "steps": n_c,
            "decode": {"workload": "batch 256, H 16, d 128, bf16, state in place",
                       "us_per_step": cd_us, "achieved": cd_bytes / (cd_us * 1e-6) / 1e9,
                       "unit": "GB/s", "frac": cd_bytes / (cd_us * 1e-6) / 1e9 / hbm_peak,
                       "bytes_per_step": cd_bytes, "steps": n_d}}

    # the other chunkwise-forward shapes: d = 128 at T = 2K, one 32K-token sequence
    # (S0 != 0, strong decay) and the wide heads (Dk 256, Dv 512)
    configs = None
    if not args.chunk_only:
        configs = []
        for name, n_steps in (("bf16_T2k", 50), ("long_T32k", 20), ("wide_dk256_dv512", 20)):
            wc = I.workload(name)
            cin = I.chunk_inputs(wc, seed=wc.seed + rank, device=device)
            co = torch.empty((wc.B, wc.T, wc.H, wc.Dv), dtype=wc.torch_dtype, device=device)
            cS = torch.empty((wc.B, wc.H, wc.Dv, wc.Dk), dtype=torch.float32, device=device)
            cw_ = torch.empty(max(G.chunk_fwd_workspace_size(wc.B, wc.T, wc.H, wc.Dk, wc.Dv,
                                                             wc.chunk, wc.torch_dtype), 1),
                              dtype=torch.uint8, device=device)

            def cstep():
                G.chunk_fwd(cin["q"], cin["k"], cin["v"], cin["log_alpha"], cin["beta"],
                            cin["S0"], chunk=wc.chunk, out=co, S_T=cS, workspace=cw_)

            for _ in range(3):
                cstep()
            c_ms = _max_over_ranks(time_loop(cstep, n_steps, stream, world), world,
                                   device) / n_steps
            cb, cf = chunk_bytes(wc, cin["S0"] is not None), chunk_flops(wc)
            configs.append({
                "workload": f"{name}: B={wc.B} H={wc.H} T={wc.T} Dk={wc.Dk} Dv={wc.Dv} "
                            f"chunk={wc.chunk} bf16, gates {wc.gate_law}, S0 {wc.s0_law}",
                "path": G.chunk_fwd_path(wc.B, wc.T, wc.H, wc.Dk, wc.Dv, wc.chunk, wc.torch_dtype),
                "variant": G.chunk_fwd_variant(wc.B, wc.T, wc.H, wc.Dk, wc.Dv, wc.chunk,
                                               wc.torch_dtype),
                "ms_per_step": c_ms, "tokens_per_s": world * wc.B * wc.T / (c_ms * 1e-3),
                "hbm_frac": cb / (c_ms * 1e-3) / 1e9 / hbm_peak,
                "tc_frac": cf / (c_ms * 1e-3) / 1e12 / tc_peak, "tc_target": 0.5,
                "bound": "tensor" if cf / cb > tc_peak * 1e12 / (hbm_peak * 1e9) else "hbm",
                "steps": n_steps})
            del cin, co, cS, cw_

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.chunk_only:
        cpu = cpu_baseline(w, inp_cpu)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: B={w.B} H={w.H} T={w.T} Dk={w.Dk} Dv={w.Dv} "
                                   f"chunk={w.chunk} bf16 q/k/v/o, f32 gates and state, S0=0",
                       "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
                       "l2": "inputs larger than L2 (q,k,v,o = %.0f MB per rank)" %
                             (4 * o.numel() * o.element_size() / 1e6),
                       "path": path, "variant": variant},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": steps * launches_per_step, "clocks": clocks, "decode": decode,
            "prologue": prologue, "varlen": varlen, "backward": backward,
            "channel_wise": channel_wise, "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def parse_workload(spec: str):
    """'name' or 'name:B=2,T=1024' -- a workload of the table with its sizes overridden
    (for profiling a smaller case of the same kernel)."""
    name, _, rest = spec.partition(":")
    over = {}
    for item in filter(None, rest.split(",")):
        key, _, val = item.partition("=")
        over[key.strip()] = int(val)
    return I.workload(name, **over)


# the kernels one chunkwise backward launches, per path
BWD_KERNELS = {
    "tcgen05": ["gdn_utw_kernel (P, T'', W and T tiles)",
                "gdn_chunk_tcw_kernel (the chunk states, bf16)", "gdn_bwd_chain_kernel (dS', dS0)",
                "gdn_bwd_grads_kernel (dq, dk, dv, dlog_alpha, dbeta)"],
    "simt": ["chunk_prep (T, P, g)", "gdn_ut_kernel (the chunk states)",
             "gdn_chunk_tc_kernel (the chunk states)", "bwd_state", "bwd_grads"],
}


def run_bwd_only(args):
    """--bwd-only: the chunkwise backward alone on --workload (one GPU, for counter
    captures); prints one short JSON line."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from gated_delta_rule_130_b200 import binding as G
    w = parse_workload(args.workload)
    inp = {n: (t.to(device) if t is not None else None) for n, t in I.chunk_inputs(w).items()}
    gen = torch.Generator().manual_seed(w.seed + 99)
    bdo = torch.randn((w.B, w.T, w.H, w.Dv), generator=gen).to(w.torch_dtype).to(device)
    bdS = torch.randn((w.B, w.H, w.Dv, w.Dk), generator=gen).to(device)
    ws = torch.empty(max(G.chunk_bwd_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk,
                                                    w.torch_dtype), 1),
                     dtype=torch.uint8, device=device)

    def step():
        G.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                    bdo, bdS, chunk=w.chunk, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    steps = args.steps or 20
    ms = time_loop(step, steps, torch.cuda.current_stream(device), 1) / steps
    print(json.dumps({"leg": "backward", "workload": args.workload,
                      "path": G.chunk_bwd_path(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk, w.torch_dtype),
                      "ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3),
                      "steps": steps}), flush=True)


def run_cw_only(args):
    """--cw-only: the channel-wise-gate forward alone on --workload (one GPU, for
    counter captures); prints one short JSON line."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from gated_delta_rule_130_b200 import binding as G
    w = parse_workload(args.workload)
    cin = I.cw_inputs(w, device=device)
    o = torch.empty((w.B, w.T, w.H, w.Dv), dtype=w.torch_dtype, device=device)
    S = torch.empty((w.B, w.H, w.Dv, w.Dk), dtype=torch.float32, device=device)
    ws = torch.empty(max(G.chunk_fwd_cw_workspace_size(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk,
                                                       w.torch_dtype), 1),
                     dtype=torch.uint8, device=device)

    def step():
        G.chunk_fwd_cw(cin["q"], cin["k"], cin["v"], cin["log_alpha"], cin["b"], cin["w"],
                       cin["S0"], chunk=w.chunk, out=o, S_T=S, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    steps = args.steps or 20
    ms = time_loop(step, steps, torch.cuda.current_stream(device), 1) / steps
    print(json.dumps({"leg": "channel_wise", "workload": args.workload,
                      "path": G.chunk_fwd_cw_path(w.B, w.T, w.H, w.Dk, w.Dv, w.chunk,
                                                  w.torch_dtype),
                      "ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3),
                      "steps": steps}), flush=True)


def run_decode_only(args):
    """--decode-only: the decode step alone (batch 256, H 16, d 128, state in place),
    for counter captures of its kernel; prints one short JSON line."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from gated_delta_rule_130_b200 import binding as G
    pk, pk_kind = peaks()
    wd = I.workload("decode_b256")
    S = I.decode_state(wd, device=device)
    dec_in = [{n: t.to(device) for n, t in I.decode_step_inputs(wd, t).items()} for t in range(8)]
    od = torch.empty((wd.B, wd.H, wd.Dv), dtype=wd.torch_dtype, device=device)
    it = [0]

    def dstep():
        x = dec_in[it[0] % len(dec_in)]
        it[0] += 1
        G.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, out=od)

    for _ in range(max(args.warmup, 3)):
        dstep()
    steps = args.steps or 1000
    ms = time_loop(dstep, steps, torch.cuda.current_stream(device), 1)
    us = 1e3 * ms / steps
    gbs = decode_bytes(wd) / (us * 1e-6) / 1e9
    print(json.dumps({"leg": "decode", "us_per_step": us, "achieved": gbs, "unit": "GB/s",
                      "peak": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"],
                      "peak_source": f"{pk_kind} hbm_gbs", "bytes_per_step": decode_bytes(wd),
                      "steps": steps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--chunk-only", action="store_true",
                    help="time the chunkwise forward only (no decode, end-to-end or CPU legs)")
    ap.add_argument("--workload", default=I.HEADLINE,
                    help="with --chunk-only: the workload to time, 'name' or 'name:B=2,T=1024'")
    ap.add_argument("--decode-only", action="store_true",
                    help="time the decode step alone (one GPU, for counter captures)")
    ap.add_argument("--cw-only", action="store_true",
                    help="time the channel-wise-gate forward alone on --workload (one GPU)")
    ap.add_argument("--bwd-only", action="store_true",
                    help="time the chunkwise backward alone on --workload (one GPU)")
    args = ap.parse_args()
    if args.bwd_only:
        run_bwd_only(args)
    elif args.decode_only:
        run_decode_only(args)
    elif args.cw_only:
        run_cw_only(args)
    elif args.impl == "reference":
        if args.steps is None:
            args.steps = 10
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
