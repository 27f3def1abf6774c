"""Benchmark of the multi-scale retention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one chunkwise retention forward with the fused per-head
GroupNorm + swish gate over the RetNet-1.3B-shaped MSR workload (B=8, H=8,
L=4096, d_k=256, d_v=512, chunk 128, xPos rotation, bf16 in/out, fp32
accumulate): Q, K, V, G in, Y out, all resident in HBM.  Throughput is
tokens (B*L) per second over the whole job.  The same JSON line carries the
roofline of the dominant kernel, an end-to-end figure through host buffers,
the recurrent decode measurement (B=64, H=16, d_k=256, d_v=512, fp32 state,
256 steps in a CUDA graph after a chunkwise prefill of 8192 tokens), the
parallel form on the MSR workload, the CPU oracle baseline and the SM clocks
seen during the timed region.

With N > 1 (torchrun, one process per GPU) every rank runs its own copy of
the workload (independent sequences, no data exchange): weak scaling, value =
all ranks' tokens / max over ranks of the timed device time.

``--impl reference`` times the fp64 CPU oracle instead (the only other
implementation of the method here), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from retentive_network_scale_b200.synth import WORKLOADS, make_decode_inputs, make_inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (HGX HBM3e bandwidth; dense bf16), reported beside
# the measured denominators
SPEC_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
L2_BYTES = 126 * 2**20


# --------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(kernel_src, summary):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, scaled to the full workload; None unless the summary was taken
    on the current source of the kernel (its sha256 prefix matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "retentive_network_scale_b200", "csrc", kernel_src)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for line in open(path):
        if line.startswith("traffic_bytes_per_full_launch:"):
            # traffic_bytes_per_full_launch: <bytes> source_sha256: <16 hex>
            parts = line.split()
            if len(parts) >= 4 and parts[3] == digest:
                return float(parts[1])
    return None


def chunkwise_flops_per_token_head(C, dk, dv):
    """Algorithmic flops of the chunkwise form per token and head: causal
    pairs only inside a chunk ((C+1)/2 keys on average, 2 flops per
    multiply-add for q.k and for p.v) plus the carried-state read and the
    state update (2 dk dv each)."""
    return (C + 1) * (dk + dv) + 4 * dk * dv


def parallel_flops_per_token_head(L, dk, dv):
    return (L + 1) * (dk + dv)


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        self.lines, self.first = [], 0
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        if self.proc is not None:
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            # nvidia-smi's start-up (NVML) is over before the timed region
            # opens: wait for its first sample, then keep only later ones
            t0 = time.time()
            while not self.lines and self.proc.poll() is None and time.time() - t0 < 20:
                time.sleep(0.02)
            self.first = len(self.lines)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)
        taken = self.lines[self.first:] or self.lines
        self.out = "".join(taken)

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": seen, "samples": len(rows)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def whole_job_value(world, units_per_rank_step, ms_max):
    """Weak-scaling throughput: every rank processes the same number of
    units per step on its own shard, so the whole job does world * units in
    the slowest rank's step time (ms_max, the max over ranks)."""
    if world < 1 or ms_max <= 0:
        raise ValueError("need world >= 1 and a positive step time")
    return world * units_per_rank_step / (ms_max * 1e-3)


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- CPU oracle
def oracle_sample(w, max_seconds=20.0):
    """Time the fp64 oracle (recurrent form, then GroupNorm + gate) on whole
    (b, h) slices of the workload, adding slices until ~max_seconds of work.
    Returns (tokens/s equivalent, cores, description)."""
    from oracle import oracle as orc
    x = make_inputs(w, B=1)
    cores = os.cpu_count() or 1
    gam = orc.gammas(w.H)
    q, k, v = (x[n].double().numpy() for n in ("Q", "K", "V"))
    g = x["G"].double().numpy() if "G" in x else None
    slices, elapsed = 0, 0.0
    batch = min(w.H, cores)
    while elapsed < max_seconds / 2 and slices < w.B * w.H:
        hs = [(slices + i) % w.H for i in range(batch)]
        t0 = time.perf_counter()
        O, _ = orc.recurrent(q[:, hs], k[:, hs], v[:, hs], gam[hs], rotate=w.rotate,
                             theta_base=w.theta_base, nthreads=cores)
        if g is not None:
            gg = np.concatenate([g[:, :, h * w.d_v:(h + 1) * w.d_v] for h in hs], axis=-1)
            orc.gate_groupnorm(O, gg)
        elapsed += time.perf_counter() - t0
        slices += batch
    tokens = slices * w.L / w.H  # a token needs all H head slices
    desc = (f"{slices} (b,h) slices of L={w.L} (recurrent form"
            f"{' + GroupNorm/gate' if g is not None else ''}), fp64, {cores} threads")
    return tokens / elapsed, cores, desc, elapsed


def run_reference(args, world, rank):
    w = WORKLOADS["msr_1p3b"]
    if world > 1 and rank != 0:
        return
    values = []
    cores, desc = os.cpu_count(), ""
    for i in range(args.warmup + args.steps):
        v, cores, desc, _ = oracle_sample(w, max_seconds=max(2.0, 60.0 / (args.steps + args.warmup)))
        if i >= args.warmup:
            values.append(v)
    val = statistics.median(values)
    line = {"impl": "reference", "metric": "retention fwd tokens/s (RetNet-1.3B MSR chunkwise + GN/gate)",
            "value": val, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup,
            # each step is a bounded sample of the workload: the time a whole
            # step (B*L tokens) would take at the sampled rate
            "ms_per_step": w.B * w.L / val * 1e3, "ms_per_step_extrapolated": True,
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w):
    return {"workload": f"{w.name}: RetNet-1.3B-shaped MSR chunkwise forward + GroupNorm/swish gate, "
                        f"B={w.B} H={w.H} L={w.L} d_k={w.d_k} d_v={w.d_v} chunk={w.chunk}, "
                        f"xPos on, bf16 in/out",
            "global_batch": w.B, "seq_len": w.L, "heads": w.H, "d_k": w.d_k, "d_v": w.d_v,
            "chunk": w.chunk, "parallelism": "replicas",
            "l2": f"inputs ({w.B * w.H * w.L * (2 * w.d_k + 2 * w.d_v) * 2 / 1e6:.0f} MB) larger than L2; no flush"}


# ----------------------------------------------------------------- GPU timing
def time_launches(fn, n, stream):
    """Device time per call (ms) over n back-to-back calls, CUDA events on
    the launching stream."""
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(n):
        fn()
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / n


def bench_decode(R, pk, warm=2, reps=3, batch=None):
    w = WORKLOADS["decode"]
    if batch:
        w = dataclasses.replace(w, B=batch)
    x = make_inputs(w, device="cuda")
    steps = make_decode_inputs(w, device="cuda")
    g = R.msr_gammas(w.H)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    stream = torch.cuda.current_stream()
    prefill = lambda: R.ret_chunkwise(x["Q"], x["K"], x["V"], g, w.chunk, O=O, state_out=S,  # noqa: E731
                                      rotate=w.rotate)
    prefill()
    t_prefill = time_launches(prefill, 2, stream)
    del O, x
    o = torch.empty(w.decode_steps, w.B, w.H, w.d_v, device="cuda", dtype=torch.bfloat16)
    state = S.clone()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        # one eager pass first (lazy module loading), then capture
        for t in range(2):
            R.ret_recurrent_step(steps["q"][t], steps["k"][t], steps["v"][t], state, o[t], g,
                                 pos=w.L + t, rotate=w.rotate, stream=side)
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            for t in range(w.decode_steps):
                R.ret_recurrent_step(steps["q"][t], steps["k"][t], steps["v"][t], state, o[t], g,
                                     pos=w.L + t, rotate=w.rotate, stream=side)
    stream.wait_stream(side)
    for _ in range(warm):
        graph.replay()
    torch.cuda.synchronize()
    ms = time_launches(graph.replay, reps, stream) / w.decode_steps
    graph.reset()
    bytes_step = (2 * w.B * w.H * w.d_k * w.d_v * 4            # state read + write
                  + w.B * w.H * (2 * w.d_k + w.d_v) * 2       # q, k, v (bf16)
                  + w.B * w.H * w.d_v * 2)                    # o (bf16)
    gbs = bytes_step / (ms * 1e-3) / 1e9
    # several tokens per sequence and call (T = 8): one pass over the state
    T = 8
    calls = w.decode_steps // T
    group = lambda a, i: a[i * T:(i + 1) * T].permute(1, 2, 0, 3).contiguous()  # noqa: E731
    qs = [group(steps["q"], i) for i in range(calls)]
    ks = [group(steps["k"], i) for i in range(calls)]
    vs = [group(steps["v"], i) for i in range(calls)]
    del steps
    om = torch.empty(calls, w.B, w.H, T, w.d_v, device="cuda", dtype=torch.bfloat16)
    state_m = S.clone()
    graph_m = torch.cuda.CUDAGraph()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        R.ret_recurrent_step(qs[0], ks[0], vs[0], state_m, om[0], g, pos=w.L, rotate=w.rotate,
                             stream=side)
        side.synchronize()
        with torch.cuda.graph(graph_m, stream=side):
            for i in range(calls):
                R.ret_recurrent_step(qs[i], ks[i], vs[i], state_m, om[i], g, pos=w.L + i * T,
                                     rotate=w.rotate, stream=side)
    stream.wait_stream(side)
    for _ in range(warm):
        graph_m.replay()
    torch.cuda.synchronize()
    ms_m = time_launches(graph_m.replay, reps, stream) / calls
    graph_m.reset()
    bytes_call = (2 * w.B * w.H * w.d_k * w.d_v * 4
                  + T * w.B * w.H * (2 * w.d_k + w.d_v) * 2 + T * w.B * w.H * w.d_v * 2)
    gbs_m = bytes_call / (ms_m * 1e-3) / 1e9
    flop_prefill = w.B * w.H * w.L * chunkwise_flops_per_token_head(w.chunk, w.d_k, w.d_v)
    return {
        "workload": f"decode: B={w.B} H={w.H} d_k={w.d_k} d_v={w.d_v}, fp32 state, bf16 q/k/v/o, "
                    f"{w.decode_steps} steps in one CUDA graph after a {w.L}-token chunkwise prefill",
        "tokens_per_s": w.B / (ms * 1e-3), "ms_per_step": ms,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / pk["hbm_gbs"], "bytes_per_step": bytes_step,
                     "frac_of_spec": gbs / SPEC_PEAKS["hbm_gbs"]},
        "prefill": {"ms": t_prefill, "tokens_per_s": w.B * w.L / (t_prefill * 1e-3),
                    "tflops": flop_prefill / (t_prefill * 1e-3) / 1e12},
        "gpu_launches_per_step": 1,
        "multi_token": {
            "tokens_per_call": T, "ms_per_call": ms_m,
            "tokens_per_s": w.B * T / (ms_m * 1e-3),
            "workload": f"{T} tokens per sequence per call, {calls} calls in one CUDA graph",
            "roofline": {"bound": "hbm", "achieved": gbs_m, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs_m / pk["hbm_gbs"], "bytes_per_call": bytes_call}},
    }


def bench_parallel(R, w, d, pk, reps=3):
    g = R.msr_gammas(w.H)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    fn = lambda: R.ret_parallel(d["Q"], d["K"], d["V"], O, g, rotate=w.rotate)  # noqa: E731
    fn()
    ms = time_launches(fn, reps, torch.cuda.current_stream())
    fl = w.B * w.H * w.L * parallel_flops_per_token_head(w.L, w.d_k, w.d_v)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": f"parallel form on {w.name} (O bf16, no gate)", "ms": ms,
            "tokens_per_s": w.B * w.L / (ms * 1e-3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"]}}


def bench_backward(R, w, d, pk, reps=3):
    """Gradients of the retention output (dQ, dK, dV, fp32) on the workload,
    as the five tensor-core chunkwise products plus the copy passes."""
    g = R.msr_gammas(w.H)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed + 7)
    dO = torch.randn(w.B, w.H, w.L, w.d_v, device="cuda", generator=gen).bfloat16()
    dQ = torch.empty(w.B, w.H, w.L, w.d_k, device="cuda")
    dK = torch.empty_like(dQ)
    dV = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda")
    ws = torch.empty(R.lib_backward_workspace_size(w.B, w.H, w.L, w.d_k, w.d_v, g, w.chunk,
                                                   rotate=w.rotate),
                     dtype=torch.uint8, device="cuda")
    fn = lambda: R.ret_backward(d["Q"], d["K"], d["V"], dO, g, w.chunk, dQ=dQ, dK=dK, dV=dV,  # noqa: E731
                                rotate=w.rotate, workspace=ws)
    for _ in range(2):
        fn()
    ms = time_launches(fn, reps, torch.cuda.current_stream())
    C = w.chunk
    fl = lambda dqk, dval: (C + 1) * (dqk + dval) + 4 * dqk * dval  # noqa: E731
    per = 2 * fl(w.d_v, w.d_k) + fl(w.d_k, w.d_v)   # dQ^, dK^ (over d_v), dV
    flops = w.B * w.H * w.L * per
    tf = flops / (ms * 1e-3) / 1e12
    out = {"workload": f"retention backward (dQ, dK, dV fp32) on {w.name}", "ms": ms,
           "tokens_per_s": w.B * w.L / (ms * 1e-3),
           "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                        "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"], "flops": flops}}
    del dQ, dK, dV, ws
    out["gate_norm_backward"] = bench_gate_backward(R, w, d, pk, gen, reps=max(5, reps))
    return out


def bench_gate_norm(R, w, d, pk, reps=20):
    """The standalone GroupNorm + swish gate, Y from a bf16 O and G (the
    form used when the chunk loop writes O): one streaming kernel,
    HBM-bound.  Its inputs (0.54 GB) exceed L2."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed + 9)
    O = torch.randn(w.B, w.H, w.L, w.d_v, device="cuda", generator=gen).bfloat16()
    Y = torch.empty(w.B, w.L, w.H * w.d_v, device="cuda", dtype=torch.bfloat16)
    fn = lambda: R.ret_gate_norm(O, d["G"], Y, 1e-5)  # noqa: E731
    for _ in range(3):
        fn()
    ms = time_launches(fn, reps, torch.cuda.current_stream())
    nbytes = 3 * O.numel() * O.element_size()  # read O, G; write Y
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"GroupNorm + swish gate alone (bf16 O, G -> Y) on {w.name}", "ms": ms,
            "tokens_per_s": w.B * w.L / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "bytes": nbytes}}


def bench_gate_backward(R, w, d, pk, gen, reps=20):
    """dO and dG of the GroupNorm + swish gate given dY (bf16 O, G, dY, dO,
    dG): one streaming kernel, HBM-bound.  Its inputs (0.8 GB) exceed L2."""
    O = torch.randn(w.B, w.H, w.L, w.d_v, device="cuda", generator=gen).bfloat16()
    dY = torch.randn(w.B, w.L, w.H * w.d_v, device="cuda", generator=gen).bfloat16()
    dO = torch.empty_like(O)
    dG = torch.empty_like(dY)
    fn = lambda: R.ret_gate_norm_backward(O, d["G"], dY, dO, dG, 1e-5)  # noqa: E731
    for _ in range(3):
        fn()
    ms = time_launches(fn, reps, torch.cuda.current_stream())
    nbytes = 5 * O.numel() * O.element_size()  # read O, G, dY; write dO, dG
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"GroupNorm + swish gate backward (dO, dG bf16) on {w.name}", "ms": ms,
            "tokens_per_s": w.B * w.L / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "bytes": nbytes}}


def bench_seqshard(R, w, d, pk, reps=5, parts=8):
    """What splitting the sequence over ranks adds per rank: the state of
    a segment from zero (here the whole msr_1p3b sequence as one segment,
    the most a rank does) and the scan of `parts` gathered states.  The
    exchange itself needs several GPUs and is not timed here."""
    g = R.msr_gammas(w.H)
    U = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    ws = torch.empty(R.lib_segment_state_workspace_size(w.B, w.H, w.L, w.d_k, w.d_v, g, w.rotate),
                     dtype=torch.uint8, device="cuda")
    seg = lambda: R.ret_segment_state(d["K"], d["V"], g, U=U, rotate=w.rotate, workspace=ws)  # noqa: E731
    U_all = torch.randn(parts, w.B, w.H, w.d_k, w.d_v, device="cuda")
    Rout = torch.empty_like(U)
    lens = [w.L // parts] * parts
    scan = lambda: R.ret_state_scan(U_all, lens, parts, g, R=Rout)  # noqa: E731
    for _ in range(2):
        seg(); scan()
    stream = torch.cuda.current_stream()
    ms_seg = time_launches(seg, reps, stream)
    ms_scan = time_launches(scan, reps, stream)
    # K read and K~ written by the streaming pass, K~ and V read and U written by the GEMM
    rows = w.B * w.H * w.L
    seg_bytes = rows * w.d_k * 2 * 3 + rows * w.d_v * 2 + w.B * w.H * w.d_k * w.d_v * 4
    scan_bytes = (parts + 1) * w.B * w.H * w.d_k * w.d_v * 4
    return {"workload": f"segment state of {w.name} (B={w.B} H={w.H}, {w.L} rows) and the scan of "
                        f"{parts} gathered states",
            "segment_state_ms": ms_seg, "state_scan_ms": ms_scan,
            "roofline": {"bound": "hbm", "unit": "GB/s", "peak": pk["hbm_gbs"],
                         "segment_state": seg_bytes / (ms_seg * 1e-3) / 1e9,
                         "segment_state_frac": seg_bytes / (ms_seg * 1e-3) / 1e9 / pk["hbm_gbs"],
                         "state_scan": scan_bytes / (ms_scan * 1e-3) / 1e9,
                         "state_scan_frac": scan_bytes / (ms_scan * 1e-3) / 1e9 / pk["hbm_gbs"]}}


def bench_long_ctx(R, pk, reps=3, segments=8):
    """Long context (B=1 H=16 L=65536 d_k=128 d_v=256, chunk 256, xPos, O and
    the final state): the plain chunk loop (32 CTAs on 148 SMs) against the
    same sequences cut into `segments` segments that run at once."""
    w = WORKLOADS["long_ctx"]
    d = make_inputs(w, device="cuda")
    g = R.msr_gammas(w.H)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    ws_plain = torch.empty(R.ret_chunkwise_prep_size(w.B, w.H, w.L, w.d_k, w.d_v, R.RET_BF16,
                                                     R.RET_BF16, g, w.chunk, rotate=w.rotate),
                           dtype=torch.uint8, device="cuda")
    ws_seg = torch.empty(R.lib_segmented_workspace_size(w.B, w.H, w.L, w.d_k, w.d_v, g, w.chunk,
                                                        segments, w.rotate),
                         dtype=torch.uint8, device="cuda")
    plain = lambda: R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, O=O, state_out=S,  # noqa: E731
                                    rotate=w.rotate, workspace=ws_plain)
    seg = lambda: R.ret_chunkwise_segmented(d["Q"], d["K"], d["V"], g, w.chunk, segments, O=O,  # noqa: E731
                                            state_out=S, rotate=w.rotate, workspace=ws_seg)
    for _ in range(2):
        plain(); seg()
    stream = torch.cuda.current_stream()
    ms_plain = time_launches(plain, reps, stream)
    ms_seg = time_launches(seg, reps, stream)
    tokens = w.B * w.L
    # algorithmic bytes: Q, K, V read once, O written (bf16); algorithmic
    # flops of the chunkwise form at the workload's chunk
    alg_bytes = sum(t.numel() * t.element_size() for k, t in d.items() if k in ("Q", "K", "V")) + \
        O.numel() * O.element_size()
    flops = w.B * w.H * w.L * chunkwise_flops_per_token_head(w.chunk, w.d_k, w.d_v)
    gbs = alg_bytes / (ms_seg * 1e-3) / 1e9
    tf = flops / (ms_seg * 1e-3) / 1e12
    return {"workload": f"{w.name}: B={w.B} H={w.H} L={w.L} d_k={w.d_k} d_v={w.d_v} chunk={w.chunk}, "
                        f"O and the final state",
            "plain_ms": ms_plain, "segmented_ms": ms_seg, "segments": segments,
            "tokens_per_s_plain": tokens / (ms_plain * 1e-3),
            "tokens_per_s_segmented": tokens / (ms_seg * 1e-3),
            # the whole segmented call (key pass, segment states on the
            # tensor cores, scan, prep pass, chunk loop) against the
            # algorithmic work of the workload
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "bytes": alg_bytes,
                         "tensor": {"achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                    "frac": tf / pk["bf16_tflops"], "flops": flops}}}


def time_flushed(fn, n, stream, flush):
    """Median device time (ms) of n calls, each after writing a buffer larger
    than L2 (so no call finds its inputs in L2), CUDA events per call."""
    times = []
    for _ in range(n):
        flush.zero_()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        fn()
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e))
    return statistics.median(times)


def bench_msr_small(R, pk, reps=50):
    """The small MSR layer's retention (B=4 H=8 L=2048 d_k=d_v=64, chunk 64,
    no rotation, GroupNorm + swish gate, bf16): the chunkwise call for Y, and
    the parallel form for O.  Its inputs (42 MB) fit in L2, so L2 is flushed
    before every timed call."""
    w = WORKLOADS["msr_small"]
    d = make_inputs(w, device="cuda")
    g = R.msr_gammas(w.H)
    Y = torch.empty(w.B, w.L, w.H * w.d_v, device="cuda", dtype=torch.bfloat16)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    # the fast-path room: 32 heads of d_v 64 leave most SMs idle, so the call
    # cuts every sequence into segments that run at once
    ws = torch.empty(max(1, R.ret_chunkwise_fast_size(w.B, w.H, w.L, w.d_k, w.d_v, R.RET_BF16,
                                                      R.RET_BF16, g, w.chunk, rotate=w.rotate)),
                     dtype=torch.uint8, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    chunk = lambda: R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, G=d["G"], Y=Y,  # noqa: E731
                                    rotate=w.rotate, workspace=ws)
    par = lambda: R.ret_parallel(d["Q"], d["K"], d["V"], O, g, rotate=w.rotate)  # noqa: E731
    for _ in range(3):
        chunk(); par()
    stream = torch.cuda.current_stream()
    ms_c = time_flushed(chunk, reps, stream, flush)
    ms_p = time_flushed(par, reps, stream, flush)
    alg_bytes = sum(d[k].numel() * d[k].element_size() for k in ("Q", "K", "V", "G")) + \
        Y.numel() * Y.element_size()
    fl_c = w.B * w.H * w.L * chunkwise_flops_per_token_head(w.chunk, w.d_k, w.d_v)
    fl_p = w.B * w.H * w.L * parallel_flops_per_token_head(w.L, w.d_k, w.d_v)
    gbs = alg_bytes / (ms_c * 1e-3) / 1e9
    tf_p = fl_p / (ms_p * 1e-3) / 1e12
    return {"workload": f"{w.name}: B={w.B} H={w.H} L={w.L} d_k={w.d_k} d_v={w.d_v} chunk={w.chunk}, "
                        f"no rotation, Y = swish(G) GroupNorm(O), bf16; L2 flushed before each call; "
                        f"the chunkwise call in one launch, every 128-row block at once (fast-path "
                        f"workspace)",
            "chunkwise_ms": ms_c, "tokens_per_s": w.B * w.L / (ms_c * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "bytes": alg_bytes,
                         "tensor_frac": fl_c / (ms_c * 1e-3) / 1e12 / pk["bf16_tflops"]},
            "parallel": {"ms": ms_p, "tokens_per_s": w.B * w.L / (ms_p * 1e-3),
                         "roofline": {"bound": "tensor", "achieved": tf_p, "peak": pk["bf16_tflops"],
                                      "unit": "TFLOP/s", "frac": tf_p / pk["bf16_tflops"],
                                      "flops": fl_p}}}


def bench_layer(R, w, pk, reps=5):
    """The whole multi-scale retention layer on the RetNet-1.3B head shape:
    d_model = H*d_k, random bf16 weights (the shapes matter, not the values)."""
    dm = w.H * w.d_k
    n_proj = w.H * (2 * w.d_k + 2 * w.d_v)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed + 99)
    X = torch.randn(w.B, w.L, dm, device="cuda", generator=gen).bfloat16()
    W = (torch.randn(dm, n_proj, device="cuda", generator=gen) * dm ** -0.5).bfloat16()
    Wo = (torch.randn(w.H * w.d_v, dm, device="cuda", generator=gen) * (w.H * w.d_v) ** -0.5).bfloat16()
    out = torch.empty(w.B, w.L, dm, device="cuda", dtype=torch.bfloat16)
    g = R.msr_gammas(w.H)
    ws = torch.empty(R.lib_msr_layer_workspace_size(w.B, w.H, w.L, w.d_k, w.d_v, g, dm, w.chunk),
                     dtype=torch.uint8, device="cuda")
    fn = lambda: R.ret_msr_layer(X, W, Wo, g, w.chunk, w.d_k, w.d_v, out=out,  # noqa: E731
                                 rotate=w.rotate, workspace=ws)
    for _ in range(3):
        fn()
    ms = time_launches(fn, reps, torch.cuda.current_stream())
    rows = w.B * w.L
    flops = (2 * rows * dm * n_proj + 2 * rows * w.H * w.d_v * dm
             + w.B * w.H * w.L * chunkwise_flops_per_token_head(w.chunk, w.d_k, w.d_v))
    tf = flops / (ms * 1e-3) / 1e12
    # the two products alone, on the library's tensor-core GEMM (plain
    # epilogue)
    gemms = {}
    Xr = X.view(rows, dm)
    # random operands (an all-zero one draws less power and would run above
    # the power-capped peak)
    Yb = (torch.randn(rows, w.H * w.d_v, device="cuda", generator=gen) * 0.5).bfloat16()
    P = torch.empty(rows, n_proj, device="cuda", dtype=torch.bfloat16)
    for name, (a, b, c) in (("X W_qkvg", (Xr, W, P)), ("Y W_o", (Yb, Wo, out.view(rows, dm)))):
        g_fn = lambda a=a, b=b, c=c: R.ret_gemm_bf16(a, b, c)  # noqa: E731
        g_fn()
        g_ms = time_launches(g_fn, reps, torch.cuda.current_stream())
        g_fl = 2.0 * a.shape[0] * a.shape[1] * b.shape[1]
        g_tf = g_fl / (g_ms * 1e-3) / 1e12
        gemms[name] = {"shape": [a.shape[0], b.shape[1], a.shape[1]], "ms": g_ms, "achieved": g_tf,
                       "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": g_tf / pk["bf16_tflops"]}
    del P, Yb
    return {"workload": f"MSR layer: B={w.B} L={w.L} d_model={dm} H={w.H} d_k={w.d_k} d_v={w.d_v}, "
                        f"X W_qkvg (tensor-core GEMM, CTA pairs; the xPos turn and key weights in its "
                        f"epilogue) + fused chunkwise/GroupNorm/gate + Y W_o (the same GEMM)",
            "ms": ms, "tokens_per_s": rows / (ms * 1e-3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"], "flops": flops},
            "gemm": gemms}


def run_ours(args, world, rank, local):
    from retentive_network_scale_b200 import build as rbuild
    from retentive_network_scale_b200 import retention as R
    if rank == 0:
        rbuild.build()
    barrier(world)
    R.load_library()
    pk, pk_src = peaks()
    if args.only in ("decode", "parallel", "long_ctx", "msr_small", "backward", "layer",
                     "gate_norm"):
        if args.only == "decode":
            out = bench_decode(R, pk, warm=args.warmup, reps=max(1, args.steps), batch=args.decode_batch)
        elif args.only == "long_ctx":
            out = bench_long_ctx(R, pk)
        elif args.only == "msr_small":
            out = bench_msr_small(R, pk)
        else:
            w = WORKLOADS["msr_1p3b"]
            if args.batch:
                w = dataclasses.replace(w, B=args.batch)
            d = {k: v.cuda() for k, v in make_inputs(w).items()}
            if args.only == "backward":
                out = bench_backward(R, w, d, pk, reps=max(1, args.steps))
            elif args.only == "gate_norm":
                out = bench_gate_norm(R, w, d, pk, reps=max(1, args.steps))
            elif args.only == "layer":
                out = bench_layer(R, w, pk, reps=max(1, args.steps))
            else:
                out = bench_parallel(R, w, d, pk, reps=max(1, args.steps))
        if rank == 0:
            print(json.dumps({"only": args.only, **out}), flush=True)
        return
    w = WORKLOADS["msr_1p3b"]
    if args.batch:
        w = dataclasses.replace(w, B=args.batch)
    host = make_inputs(w, shard=rank)  # each replica its own sequences
    host = {k: v.pin_memory() for k, v in host.items()}
    d = {k: v.cuda(non_blocking=True) for k, v in host.items()}
    g = R.msr_gammas(w.H)
    Y = torch.empty(w.B, w.L, w.H * w.d_v, device="cuda", dtype=torch.bfloat16)
    stream = torch.cuda.current_stream()
    # workspace for the prepared Q^ / K~ (the call's streaming pass), once
    ws = torch.empty(R.ret_chunkwise_prep_size(w.B, w.H, w.L, w.d_k, w.d_v, R.RET_BF16, R.RET_BF16,
                                               g, w.chunk, rotate=w.rotate),
                     dtype=torch.uint8, device="cuda")

    def step():
        R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, G=d["G"], Y=Y, rotate=w.rotate,
                        workspace=ws)

    def prep_only():
        return R.ret_chunkwise_prepare(d["Q"], d["K"], g, w.chunk, ws, rotate=w.rotate)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n0 = R.ret_kernel_launches()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    launches = R.ret_kernel_launches() - n0
    # a bounded wait that ran out inside a kernel latches a status: such a
    # run measured nothing
    status = R.ret_last_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")
    ms_local = start.elapsed_time(end) / args.steps
    ms = max_over_ranks(ms_local, world)
    tokens_step = w.B * w.L
    value = whole_job_value(world, tokens_step, ms)

    # The step is the streaming pass that prepares Q^ / K~ and the chunk loop
    # (the dominant kernel); with the loop taking more than one wave of CTAs
    # the call cuts the batch into slices and the pass of the next slice runs
    # under the loop of the current one.  Each is timed alone here (same
    # stream, same buffers): the pass, then the loop over the whole batch in
    # one launch on the rows the pass prepared.
    for _ in range(2):
        qh, kt = prep_only()
    ms_prep = time_launches(prep_only, max(3, args.steps), stream)
    loop_only = lambda: R.ret_chunkwise_prepared(  # noqa: E731
        qh if w.rotate else d["Q"], kt, d["V"], g, w.chunk, G=d["G"], Y=Y, rotate=w.rotate)
    for _ in range(2):
        loop_only()
    ms_kernel = time_launches(loop_only, max(3, args.steps), stream)
    flops = w.B * w.H * w.L * chunkwise_flops_per_token_head(w.chunk, w.d_k, w.d_v)
    # algorithmic bytes of the chunk loop: Q^, K~ (same sizes as Q, K), V, G in; Y out
    bytes_alg = sum(t.numel() * t.element_size() for t in d.values()) + Y.numel() * Y.element_size()
    prep_bytes = 2 * ws.numel()  # Q, K read; Q^, K~ written
    tf = flops / (ms_kernel * 1e-3) / 1e12
    gbs = bytes_alg / (ms_kernel * 1e-3) / 1e9
    prep_gbs = prep_bytes / (ms_prep * 1e-3) / 1e9
    # flops / bytes = arithmetic intensity below the ridge (peak flops / peak
    # bandwidth): HBM is the roof that binds this kernel
    roofline = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"],
                "traffic": profiled_traffic("chunkwise_ws.cu", "chunkwise_ws_msr_1p3b.md"),
                "kernel": "chunkwise_ws_kernel<256, bf16, fused GroupNorm/gate>",
                "peak_source": f"{pk_src} (copy bandwidth)",
                "frac_of_spec": gbs / SPEC_PEAKS["hbm_gbs"], "spec_peak": SPEC_PEAKS["hbm_gbs"],
                "ms_per_launch": ms_kernel, "bytes_per_launch": bytes_alg,
                "flops_per_launch": flops,
                "intensity_flop_per_byte": flops / bytes_alg,
                "ridge_flop_per_byte": pk["bf16_tflops"] * 1e3 / pk["hbm_gbs"],
                "tensor": {"achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                           "frac": tf / pk["bf16_tflops"],
                           "peak_source": f"{pk_src} (bf16 burst)",
                           "frac_of_sustained": tf / pk["bf16_tflops_sustained"],
                           "frac_of_spec": tf / SPEC_PEAKS["bf16_tflops"],
                           "spec_peak": SPEC_PEAKS["bf16_tflops"]},
                "prep": {"kernel": "chunk_prep_kernel (rotate Q, rotate and decay-weight K)",
                         "ms_per_launch": ms_prep, "bytes_per_launch": prep_bytes,
                         "achieved": prep_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": prep_gbs / pk["hbm_gbs"]}}

    # end to end through the C ABI with host buffers: ret_chunkwise_host
    # copies each batch slice in, computes it and copies Y back, the three
    # overlapped across slices (page-locked host memory)
    Y_host = torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True)
    n_e2e = max(1, min(args.steps, 5))
    e2e_slices = w.B
    host_ws = torch.empty(R.ret_chunkwise_host_workspace_size(
        w.B, w.H, w.L, w.d_k, w.d_v, R.RET_BF16, R.RET_BF16, g, w.chunk, e2e_slices,
        want_O=False, want_Y=True, rotate=w.rotate), dtype=torch.uint8, device="cuda")

    def e2e_step():
        R.ret_chunkwise_host(host["Q"], host["K"], host["V"], g, w.chunk, G=host["G"], Y=Y_host,
                             rotate=w.rotate, slices=e2e_slices, workspace=host_ws)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    ms_e2e = max_over_ranks(time_launches(e2e_step, n_e2e, stream), world)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = Y.numel() * Y.element_size()

    extra = {}
    if not args.skip_extra:
        extra["parallel"] = bench_parallel(R, w, d, pk)
        extra["backward"] = bench_backward(R, w, d, pk)
        extra["gate_norm"] = bench_gate_norm(R, w, d, pk)
        extra["sequence_shard"] = bench_seqshard(R, w, d, pk)
        del d
        torch.cuda.empty_cache()
        extra["long_ctx"] = bench_long_ctx(R, pk)
        torch.cuda.empty_cache()
        extra["msr_small"] = bench_msr_small(R, pk)
        torch.cuda.empty_cache()
        extra["msr_layer"] = bench_layer(R, w, pk)
        torch.cuda.empty_cache()
        extra["decode"] = bench_decode(R, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        v, cores, desc, _ = oracle_sample(w, max_seconds=args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": "retention fwd tokens/s (RetNet-1.3B MSR chunkwise + GN/gate)",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w),
            "roofline": roofline,
            "e2e": {"value": whole_job_value(world, tokens_step, ms_e2e), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                    "call": f"ret_chunkwise_host (page-locked host buffers, {e2e_slices} batch slices pipelined)"},
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            **extra,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-extra", action="store_true", help="only the main step")
    ap.add_argument("--skip-cpu", action="store_true", help="no CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the MSR workload's batch (small cases for profiler captures)")
    ap.add_argument("--only", choices=["main", "parallel", "decode", "long_ctx", "msr_small",
                                       "backward", "layer", "gate_norm"],
                    default=None,
                    help="run one measurement alone (profiler captures)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="override the decode workload's batch (small cases for profiler captures)")
    args = ap.parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
