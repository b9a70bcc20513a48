#!/usr/bin/env python
"""Benchmark of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one gdr_chunk_fwd over the Gated DeltaNet workload (B=4, H=16,
T=4096, d_k=d_v=128, bf16, scalar decay, tied scalar beta, chunk 64): the
whole chunkwise path (load and log-decay scan, intra-chunk products, WY/UT
transform, inter-chunk state propagation, write-back). Inputs (274 MB) are
larger than the 126 MB L2, so no flush is needed between steps. The decode
step (256 x 32 heads, d = 128, 1000 sequential steps, fp32 state in HBM) is
measured in the same run and reported under "decode"; the KDA and Gated
DeltaNet-2 chunk workloads under "other_workloads".

With N > 1 (torchrun, one process per GPU) every rank runs its own copy of
the workload (heads are independent; no collective on the data path), the
timed region is bracketed by barriers and the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this project
has) on a bounded sample of the same workload on the host cores.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule fwd tokens/s and % roofline; decode state GB/s vs HBM peak"
# Algorithmic work per token-head (2 flops per multiply-add) of the chunkwise
# contractions at C = 64, d = 128 with general gates (tied scalar beta:
# workload_flops derives it from the head dims; 182,955 at d = 128).
FLOPS_PER_TOKEN_HEAD = {"general": 281259}
L2_BYTES = 126 * 2**20


# Sources of the kernel each workload runs; a recorded DRAM traffic figure is
# used only while these files are unchanged since the capture.
_CSRC = "gated_delta_rule_147_b200/csrc/"
KERNEL_SOURCES = {
    "general": (_CSRC + "chunk_sm100.cu", _CSRC + "chunk_common.cuh", _CSRC + "common.cuh"),
    "twopass": (_CSRC + "chunk_twopass_sm100.cu", _CSRC + "chunk_common.cuh", _CSRC + "common.cuh"),
    "twopass_general": (_CSRC + "chunk_twopass_general_sm100.cu", _CSRC + "chunk_common.cuh",
                        _CSRC + "common.cuh"),
    "erasefree": (_CSRC + "chunk_erasefree_sm100.cu", _CSRC + "chunk_common.cuh",
                  _CSRC + "common.cuh"),
    "twopass256": (_CSRC + "chunk_twopass256_sm100.cu", _CSRC + "chunk_common.cuh", _CSRC + "common.cuh"),
}


KERNEL_NAMES = {
    "general": "gdr::chunk::chunk_fwd_kernel / chunk_fwd_gdn_kernel (single pass)",
    "twopass": "gdr::twopass::prep_gdn_kernel + gdr::twopass::state_gdn_kernel (one call, two launches)",
    "erasefree": "gdr::erasefree::chunk_fwd_erasefree_kernel",
    "twopass_general": "gdr::twopass_g::prep_general_kernel + state_general_kernel (one call, two launches)",
    "twopass256": "gdr::twopass256::prep_gdn256_kernel + state_gdn256_kernel (one call, two launches)",
}
LAUNCHES_PER_CALL = {"general": 1, "twopass": 2, "erasefree": 1, "twopass_general": 2, "twopass256": 2}


def kernel_family(wl) -> str:
    if wl.b == "none":
        return "erasefree"
    gdn = wl.alpha == "scalar" and wl.b == "scalar" and wl.w == "tied"
    if wl.dtype == "bf16" and wl.dk == 256 and gdn and wl.dv % 64 == 0 and wl.dv <= 256 and wl.T > 0:
        return "twopass256"
    if wl.dtype == "bf16" and wl.dk == 128 and wl.dv in (64, 128) and wl.T > 0:
        if wl.alpha == "scalar" and wl.b == "scalar" and wl.w == "tied":
            return "twopass"
        return "twopass_general"
    return "general"


def kernel_source_hash(family: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[family]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
    the chunk kernel from the committed ncu summary, or None when the summary
    is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "chunk_fwd_traffic.json")
    try:
        d = json.load(open(path))
    except (OSError, ValueError):
        return None
    from gated_delta_rule_147_b200.inputs import WORKLOADS
    w = d.get("workloads", {}).get(workload)
    if w is None or w.get("source_sha256") != kernel_source_hash(kernel_family(WORKLOADS[workload])):
        return None
    return w.get("dram_bytes_per_launch")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def workload_bytes(wl):
    """Bytes that must cross HBM once: inputs read, o written, S0 read if
    given, S_T written."""
    el = 2 if wl.dtype == "bf16" else 4
    th = wl.B * wl.T * wl.H
    gate = lambda kind: 0 if kind in ("none", "tied") else (th if kind == "scalar" else th * wl.dk)
    n = wl.B * wl.T * wl.Hq * 2 * wl.dk + th * 2 * wl.dv + gate(wl.alpha) + gate(wl.b) + gate(wl.w)
    state = wl.B * wl.H * wl.dk * wl.dv * 4
    return n * el + state * (1 + int(wl.s0))


def workload_flops(wl):
    if wl.b == "none":
        # erase-free chunk form: (q.g) S, Bq V, the state increment and Bq itself
        C = 64
        per = 2 * (2 * wl.dk * wl.dv + C * wl.dv + C * wl.dk // 2)
        return per * wl.B * wl.T * wl.H
    if wl.w == "tied" and wl.b == "scalar":
        # per token-head: K K^T, Q K^T, -W (C d_k each), P, Aq U (C d_v each),
        # W S, Q S, the state step (d_k d_v each) and the solve (C^2 / 3)
        C = 64
        per = round(2 * (3 * wl.dk * wl.dv + C * (3 * wl.dk + 2 * wl.dv) + C * C / 3))
        return per * wl.B * wl.T * wl.H
    return FLOPS_PER_TOKEN_HEAD["general"] * wl.B * wl.T * wl.H


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
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
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


def dist_env():
    from gated_delta_rule_147_b200.dist_util import dist_env as env
    return env()


# ------------------------------------------------------------------ ours ---
def prepare_chunk(wl, dev):
    import torch
    from gated_delta_rule_147_b200.inputs import make_chunk_inputs
    inp = make_chunk_inputs(wl)
    d = {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in inp.items()}
    return inp, d


def alloc_workspace(d, wl):
    """The two-pass path's scratch (None when the gate form has no such path)."""
    import torch
    from gated_delta_rule_147_b200 import TIED, workspace_bytes
    w = TIED if wl.w == "tied" else d["w"]
    n = workspace_bytes(d["q"], d["v"], d["alpha"], d["b"], w)
    return torch.empty(n, dtype=torch.uint8, device=d["q"].device) if n else None


def chunk_call(d, wl, o, ST, stream, ws):
    from gated_delta_rule_147_b200 import TIED, chunk_fwd
    w = TIED if wl.w == "tied" else d["w"]
    chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], w, d["S0"], out=o, S_T=ST, stream=stream,
              workspace=ws)


def time_chunk(wl, dev, steps, warmup, barrier):
    """Device time per launch (CUDA events on the launching stream)."""
    import torch
    inp, d = prepare_chunk(wl, dev)
    o = torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=d["v"].dtype, device=dev)
    ST = torch.empty((wl.B, wl.H, wl.dk, wl.dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    ws = alloc_workspace(d, wl)
    for _ in range(warmup):
        chunk_call(d, wl, o, ST, stream, ws)
    torch.cuda.synchronize()
    barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        chunk_call(d, wl, o, ST, stream, ws)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total = ev[0].elapsed_time(ev[steps])
    barrier()
    return inp, d, total, per


def time_chunk_e2e(inp, wl, dev, steps, warmup):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory to the device and reads o back. Steps
    are pipelined as a caller streaming batches would run them: step i + 1's
    inputs cross PCIe (copy stream in) while step i computes and its o goes
    back (copy stream out, the other direction), with two device buffer sets.
    Device time from the first copy in to the last copy out."""
    import torch
    host = {k: (v.pin_memory() if hasattr(v, "pin_memory") else v) for k, v in inp.items()}
    tensors = [k for k, v in host.items() if hasattr(v, "pin_memory")]
    dbuf = [{k: (torch.empty_like(v, device=dev) if k in tensors else v) for k, v in host.items()}
            for _ in range(2)]
    o = [torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=host["v"].dtype, device=dev) for _ in range(2)]
    o_host = [torch.empty(o[0].shape, dtype=o[0].dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(host[k].numel() * host[k].element_size() for k in tensors)
    d2h = o[0].numel() * o[0].element_size()
    ws = alloc_workspace(dbuf[0], wl)
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(i):
        b = i & 1
        if used[b]:  # buffer set b: its inputs read by step i - 2's compute, its o read back
            s_in.wait_event(comp_done[b])
            s_comp.wait_event(out_done[b])
        with torch.cuda.stream(s_in):
            for k in tensors:
                dbuf[b][k].copy_(host[k], non_blocking=True)
        in_done[b].record(s_in)
        s_comp.wait_event(in_done[b])
        chunk_call(dbuf[b], wl, o[b], None, s_comp, ws)
        comp_done[b].record(s_comp)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            o_host[b].copy_(o[b], non_blocking=True)
        out_done[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        step(warmup + i)
    s_in.wait_event(out_done[(warmup + steps - 1) & 1])
    e1.record(s_in)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), h2d, d2h


# Tensor-core products of the Gated DeltaNet backward (d = 128, C = 64), per
# token-head, 2 flop per multiply-add:
# - the forward two-pass kernels, which checkpoint the state and U: the
#   forward's own count (182,955; workload_flops);
# - the chunkwise state-gradient pass: K K^T, Q K^T and X = (Diag(g_{n-1}/g)
#   T)^T K (C d_k each), Aq T (C^2) and the solve (C^2 / 3) in its first pass;
#   AqT^T dO (C d_v), X G, Q~^T dO and K^T Y' (d_k d_v each) in its state pass;
BWD_GRAD_FLOPS_PER_TOKEN_HEAD = round(2 * (3 * 64 * 128 + 64 * 64 + 64 * 128 + 3 * 128 * 128) + 2 * 64 * 64 / 3)
# - the chunk kernel, per (chunk, head): [dO;DR][S0|V|R]^T (128x256x128),
#   [Q;U]K^T (128x64x128), P[U;K], P^T[Q;E], [V';-R']G_e^T (128x128x128 each)
BWD_TC_FLOPS_PER_CHUNK = 2 * 128 * (256 * 128 + 64 * 128 + 3 * 128 * 128)


def time_backward(dev, steps, warmup, pk):
    """The backward pass (gdr_chunk_bwd) on the Gated DeltaNet workload: CUDA
    events per call (forward checkpoints, the chunkwise state-gradient pass and
    the chunk kernel, all on tensor cores)."""
    import torch
    from gated_delta_rule_147_b200 import TIED, chunk_bwd, gdr_chunk_bwd_workspace_size
    from gated_delta_rule_147_b200.inputs import WORKLOADS, make_cotangents
    wl = WORKLOADS["gdn"]
    _, d = prepare_chunk(wl, dev)
    cot = make_cotangents(wl)
    dO, dST = cot["dO"].to(dev), cot["dS_T"].to(dev)
    ws = torch.empty(gdr_chunk_bwd_workspace_size(wl.B, wl.T, wl.H, wl.dk, wl.dv), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def call():
        chunk_bwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], TIED, d["S0"], dO=dO, dS_T=dST,
                  workspace=ws, stream=stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        call()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.fmean(ev[i].elapsed_time(ev[i + 1]) for i in range(steps))
    th = wl.B * wl.T * wl.H
    state = wl.B * wl.H * wl.dk * wl.dv * 4
    # read q, k, v, dO (bf16), alpha, beta (bf16), dS_T; write dq, dk, dv (fp32), dalpha, dbeta, dS0
    bytes_ = th * (2 * (2 * wl.dk + 2 * wl.dv) + 2 * 2 + 4 * (2 * wl.dk + wl.dv) + 2 * 4) + 2 * state
    nch = wl.B * wl.H * ((wl.T + 63) // 64)
    tc_flops = BWD_TC_FLOPS_PER_CHUNK * nch
    flops = (workload_flops(wl) + BWD_GRAD_FLOPS_PER_TOKEN_HEAD * th) + tc_flops
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": f"Gated DeltaNet backward B={wl.B} H={wl.H} T={wl.T} d_k=d_v={wl.dk} bf16 "
                        f"inputs, fp32 gradients, dO and dS_T ~ N(0, 1)",
            "ms_per_call": ms, "tokens_per_s": wl.B * wl.T / (ms * 1e-3), "launches_per_call": 5,
            "kernel": "gdr::twopass::prep_gdn_kernel + state_gdn_kernel<1> (forward, checkpoints S and U) + "
                      "gdr::bwdgrad::prep_grad_kernel + state_grad_kernel (chunkwise state gradient) + "
                      "gdr::bwdtc::bwd_chunk_tc_kernel (chunk gradients)",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                         "note": "bf16 tensor-core products of all five launches over the whole call",
                         "algorithmic_flops": flops, "algorithmic_bytes": bytes_,
                         "hbm_frac": bytes_ / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "chunk_kernel_flops_per_call": tc_flops}


def time_decode(dev, nsteps, warmup):
    import torch
    from gated_delta_rule_147_b200 import decode_step
    from gated_delta_rule_147_b200.inputs import DECODE, make_decode_state, make_decode_steps
    dw = DECODE
    S = make_decode_state(dw).to(dev)
    steps = []
    for s0 in range(0, nsteps, 100):
        for st in make_decode_steps(dw, range(s0, min(s0 + 100, nsteps)), threads=os.cpu_count() or 8):
            steps.append({k: v.to(dev) for k, v in st.items()})
    o = torch.empty((dw.B, dw.H, dw.dv), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def run(i):
        d = steps[i % len(steps)]
        decode_step(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S, out=o, stream=stream)

    for i in range(warmup):
        run(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(nsteps):
        run(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / nsteps
    state = dw.B * dw.H * dw.dk * dw.dv * 4
    tok = dw.B * dw.H * (2 * dw.dk + dw.dv + 3 * dw.dk + dw.dv) * 2
    return {"workload": f"decode B={dw.B} H={dw.H} d_k=d_v={dw.dk} bf16 tokens, fp32 state, "
                        f"GDN-2 channel gates, {nsteps} sequential steps",
            "ms_per_step": ms, "launches": nsteps,
            "state_gbs": 2 * state / (ms * 1e-3) / 1e9,
            "total_gbs": (2 * state + tok) / (ms * 1e-3) / 1e9}


def cpu_baseline(wl, budget_s=15.0):
    """The oracle, untuned, on host cores over a bounded sample of heads (full
    sequence each); value in tokens/s of the same workload."""
    import oracle
    from gated_delta_rule_147_b200.inputs import make_chunk_inputs
    cores = len(os.sched_getaffinity(0))
    small = wl.with_(B=1, H=1, T=512)
    inp = make_chunk_inputs(small)
    t = time.perf_counter()
    oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"],
                      inp["gates"], nthreads=1)
    per_head_token = (time.perf_counter() - t) / small.T
    heads = max(1, min(wl.B * wl.H, int(budget_s * cores / (per_head_token * wl.T))))
    heads = max(cores, heads) if heads >= cores else heads
    sample = wl.with_(B=1, H=heads)
    inp = make_chunk_inputs(sample)
    t = time.perf_counter()
    oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"],
                      inp["gates"], nthreads=cores)
    dt = time.perf_counter() - t
    token_heads = heads * wl.T
    return {"value": token_heads / wl.H / dt, "unit": "tokens/s", "cores": min(cores, heads),
            "kind": "oracle",
            "sample": f"{heads} of {wl.B * wl.H} heads of the same workload, full T={wl.T}, "
                      f"fp64 token loop, {dt:.1f} s",
            # the same oracle on one thread (the calibration run): tokens/s of the workload per core
            "single_core": {"value": 1.0 / (per_head_token * wl.H), "unit": "tokens/s",
                            "sample": f"1 head, T={small.T}, 1 thread"}}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from gated_delta_rule_147_b200.inputs import WORKLOADS
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        barrier = lambda: dist.barrier(device_ids=[local])
    else:
        barrier = lambda: None
    from gated_delta_rule_147_b200.dist_util import max_over_ranks, shard_seed
    pk = peaks()
    wl = WORKLOADS["gdn"]
    # each rank processes its own shard of the global batch (disjoint sequences)
    wl_rank = wl.with_(seed=shard_seed(wl.seed, rank))
    with ClockSampler(local) as clk:
        inp, d, total_ms, per = time_chunk(wl_rank, dev, args.steps, args.warmup, barrier)
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms, device=dev)
    tokens = wl.B * wl.T
    value = ws * tokens * args.steps / (total_ms * 1e-3)
    bytes_ = workload_bytes(wl)
    flops = workload_flops(wl)
    avg_ms = statistics.fmean(per)
    t_hbm = bytes_ / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    achieved_gbs = bytes_ / (avg_ms * 1e-3) / 1e9
    result = None
    if rank == 0:
        e2e_ms, h2d, d2h = time_chunk_e2e(inp, wl, dev, max(3, args.steps // 2), args.warmup)
        e2e_steps = max(3, args.steps // 2)
        other = {}
        for name in ("kda", "gdn2", "gla", "gdn_gqa", "gdn256"):
            w2 = WORKLOADS[name]
            _, _, tot2, per2 = time_chunk(w2, dev, max(3, args.steps // 2), args.warmup, lambda: None)
            a2 = statistics.fmean(per2)
            b2, f2 = workload_bytes(w2), workload_flops(w2)
            rt = max(b2 / (pk["hbm_gbs"] * 1e9), f2 / (pk["bf16_tflops"] * 1e12))
            other[name] = {"workload": f"{name} B={w2.B} H={w2.H} (q/k heads {w2.Hq}) T={w2.T} d_k={w2.dk} d_v={w2.dv} bf16 alpha={w2.alpha} "
                                       f"b={w2.b} w={w2.w} S0={'random' if w2.s0 else 'zero'}",
                           "tokens_per_s": w2.B * w2.T / (a2 * 1e-3), "ms_per_launch": a2,
                           "hbm_gbs": b2 / (a2 * 1e-3) / 1e9, "roofline_frac": rt / (a2 * 1e-3),
                           "traffic": measured_traffic(name), "kernel": KERNEL_NAMES[kernel_family(w2)]}
            torch.cuda.empty_cache()
        bwd = time_backward(dev, max(3, args.steps // 2), args.warmup, pk)
        torch.cuda.empty_cache()
        dec = time_decode(dev, 1000, 10)
        dec["frac_of_hbm"] = dec["total_gbs"] / pk["hbm_gbs"]
        dec["peak_gbs"] = pk["hbm_gbs"]
        cpu = cpu_baseline(wl) if ws == 1 else None
        result = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"Gated DeltaNet chunk forward B={wl.B} H={wl.H} T={wl.T} "
                                   f"d_k=d_v={wl.dk} bf16, scalar alpha, tied scalar beta, chunk 64",
                       "global_batch": wl.B * ws, "seq_len": wl.T, "parallelism": f"replicas x{ws}",
                       "l2": f"inputs {bytes_ / 1e6:.0f} MB > 126 MB L2, no flush"},
            "roofline": {"bound": bound, "achieved": achieved_gbs if bound == "hbm" else flops / (avg_ms * 1e-3) / 1e12,
                         "peak": pk["hbm_gbs"] if bound == "hbm" else pk["bf16_tflops"],
                         "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                         "frac": (max(t_hbm, t_tc)) / (avg_ms * 1e-3), "traffic": measured_traffic("gdn"),
                         "kernel": KERNEL_NAMES[kernel_family(wl)],
                         "algorithmic_bytes": bytes_, "algorithmic_flops": flops,
                         "tensor_tflops": flops / (avg_ms * 1e-3) / 1e12,
                         "ms_per_launch": avg_ms, "peak_source": pk["source"]},
            "e2e": {"value": tokens * e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "pipelined": "step i + 1's inputs copied in while step i computes and its o is "
                                 "copied out (three streams, two device buffer sets)"},
            "gpu_launches": args.steps * LAUNCHES_PER_CALL[kernel_family(wl)],
            "clocks": clocks,
            "decode": dec,
            "backward": bwd,
            "other_workloads": other,
            "cpu_baseline": cpu,
        }
    if ws > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return result


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    from gated_delta_rule_147_b200.inputs import WORKLOADS, make_chunk_inputs
    wl = WORKLOADS["gdn"]
    cores = len(os.sched_getaffinity(0))
    heads = max(1, min(cores, wl.B * wl.H))
    sample = wl.with_(B=1, H=heads, T=1024)
    inp = make_chunk_inputs(sample)
    call = lambda: oracle.recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"],
                                     inp["S0"], inp["gates"], nthreads=cores)
    for _ in range(args.warmup):
        call()
    t = time.perf_counter()
    for _ in range(args.steps):
        call()
    dt = time.perf_counter() - t
    value = heads * sample.T * args.steps / wl.H / dt
    desc = (f"{heads} heads x T={sample.T} of the Gated DeltaNet workload per step, fp64 token "
            f"loop, OpenMP over heads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"Gated DeltaNet chunk forward B={wl.B} H={wl.H} T={wl.T} "
                                   f"d_k=d_v={wl.dk} bf16, scalar alpha, tied scalar beta, chunk 64",
                       "global_batch": wl.B, "seq_len": wl.T, "parallelism": "cpu"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    res = run_reference(args) if args.impl == "reference" else run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
