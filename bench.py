#!/usr/bin/env python
"""Benchmark of the context-parallel exact attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--pass fwd|bwd]
                    [--impl ours|reference]

One step = one pass of the hot path over one batch of synthetic input that is
already resident in HBM.  With no --workload the line is headed by the
packed-document ring forward: 131072 tokens of documents with lengths uniform
in [1024, 32768] (seed 4), 32 heads, dh 128, P = 8 virtual ranks in the
zigzag layout, bf16.  Its step is the zigzag reorder of Q, K, V, the ring-step
schedule, the block-attention launch over all live block pairs, the fp32 LSE
merge and the inverse reorder of O and LSE.  The same line carries, under one
clock record, a sub-object per other workload:

  ring_contig_32k    S=32768, P=4 contiguous causal (attention + merge)
  ring_zigzag_64k    S=65536, P=8 zigzag causal (+ zigzag reorders)
  ulysses_gqa_128k   S=131072, 32/8 heads, P=8 Ulysses (seq->head permutes,
                     per-group attention, head->seq permute)
  ring_striped_64k   S=65536, P=8 striped causal (+ striped reorders)
  usp_gqa_128k       S=131072, 32/4 heads, Ulysses over 4 x ring over 2
and the ring backward (dQ, dK, dV) of the 32K and packed-document workloads.

The metric is causal-effective TFLOP/s (4 * dh * hq per admitted (q, k) pair,
divided by the step time).  Each sub-object gives the attention kernel's own
TFLOP/s and fraction of the measured bf16 peak, and the merge, reorder and
permute kernels' GB/s and fraction of the measured HBM bandwidth, all timed
with CUDA events on the launching stream.

--gpus N > 1 launches N ranks (one process per GPU, torchrun) unless the
process already runs under torchrun; every rank times its own independent
problem (weak scaling: the virtual ranks of the path never exchange data) and
the time is the max over ranks.  With N > 1 the line also carries a `dist`
object: the ring (64K tokens, zigzag) and Ulysses (128K tokens, 32/8 heads)
run with the ranks on real GPUs, K/V rotating by NCCL send/recv and the
Ulysses all-to-alls over NCCL, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ring-attn fwd TFLOP/s & % BF16 tensor peak; a2a-permute GB/s % HBM"
METRIC_BWD = "ring-attn bwd TFLOP/s (causal-effective, 2.5x the forward's FLOP) & % BF16 tensor peak"

HEADLINE = "varlen_zigzag_128k"
SUITE = ["ring_contig_32k", "ring_zigzag_64k", "ulysses_gqa_128k", "ring_striped_64k", "usp_gqa_128k"]
BWD_SUITE = ["ring_contig_32k", "varlen_zigzag_128k"]

# DRAM traffic per launch of the block-attention kernel from an ncu capture,
# keyed by (hash of the kernel source it was taken on, workload): a kernel
# change makes the entry stale and the line reports null until the capture is
# repeated.  Filled from the profiles/ summaries.
ATTN_TRAFFIC = {
    # profiles/attn_fwd_kernel_dram_ring_workloads.md (one-pass DRAM read + write per launch), taken
    # on the source before the MMA descriptors were derived by offset: the current source reports
    # null until the capture is repeated on it.
    ("3f5eba916fea743e", "ring_contig_32k"): 2.1446e9,
    ("3f5eba916fea743e", "ring_zigzag_64k"): 9.7936e9,
    ("3f5eba916fea743e", "varlen_zigzag_128k"): 9.9624e9,
    ("3f5eba916fea743e", "ring_striped_64k"): 13.6513e9,
    ("3f5eba916fea743e", "ulysses_gqa_128k"): 6.7032e9,
}


def src_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def attn_src_hash():
    return src_hash(os.path.join(ROOT, "context_exact_attention_step_b200", "csrc", "attn_fwd.cu"))


# ----------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed
    regions run; start/stop may be called around several regions and the
    summary covers every sample taken."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.sm, self.mx, self.reasons = [], None, set()

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.proc = None
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    self.sm.append(float(parts[1]))
                    self.mx = float(parts[2])
                except ValueError:
                    continue
                for n, val in zip(self.NAMES, parts[5:9]):
                    if val.lower().startswith("active"):
                        self.reasons.add(n)
        os.unlink(self.path)

    def summary(self):
        if not self.sm:
            return None
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.mx, "reasons": sorted(self.reasons),
                "samples": len(self.sm)}


def dist_init(backend="nccl"):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch(n):
    """Runs this same command as n ranks under torchrun (one process per
    GPU) and returns its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.run(cmd).returncode


def ev():
    e = torch.cuda.Event(enable_timing=True)
    e.record()  # creates the CUDA handle
    return e


def tflops(flops, ms):
    return flops / (ms * 1e-3) / 1e12


def gbs(nbytes, ms):
    return nbytes / (ms * 1e-3) / 1e9


# ----------------------------------------------------------------- workloads
def make_workload(name, seq_len=None, pass_="fwd", host=False):
    """Inputs of a workload on the device and its step.  The step takes an
    optional list of four events recorded around the layout kernels that run
    outside the library's composite call (before: the forward reorder of Q,
    K, V; after: the inverse reorder of O and LSE)."""
    from context_exact_attention_step_b200 import api, synth
    cfg = dict(synth.CONFIGS[name])
    resized = bool(seq_len) and int(seq_len) != cfg["S"]
    if seq_len:
        cfg["S"] = int(seq_len)
    S, hq, hkv, dh, P = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"], cfg["P"]
    dtype = torch.float32 if cfg["dtype"] == "fp32" else torch.bfloat16
    q, k, v = synth.qkv(S, hq, hkv, dh, std=cfg["std"], dtype=dtype)
    cu = None
    if cfg.get("varlen"):
        cu = synth.cu_seqlens_from_lengths(synth.doc_lengths(S, cfg["doc_lo"], cfg["doc_hi"])).tolist()
    layout = cfg["layout"]
    dev = torch.device("cuda")
    w = dict(name=name, cfg=cfg, S=S, hq=hq, hkv=hkv, dh=dh, P=P, layout=layout, cu=cu, dtype=dtype, resized=resized)
    w["pairs"] = api.count_live_pairs(S, True, cu)
    w["flops"] = 4.0 * dh * hq * w["pairs"]
    if host:
        w["host"] = [t.pin_memory() for t in (q, k, v)]
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    del q, k, v
    w["in"] = (qd, kd, vd)
    o = torch.empty((S, hq, dh), device=dev, dtype=torch.float32)
    lse = torch.empty((hq, S), device=dev, dtype=torch.float32)
    w["out"] = (o, lse)
    w["reorder_bytes"] = 0
    mark = lambda marks, i: marks[i].record() if marks else None
    if layout == "ulysses":
        ws = torch.empty(api.ulysses_attn_workspace_size(S, hq, hkv, dh, P), device=dev, dtype=torch.uint8)

        def step(marks=None):
            api.ulysses_attn_fwd(qd, kd, vd, P, True, o=o, lse=lse, workspace=ws)
        # seq->head of Q, K, V (bf16) and head->seq of O (fp32): read + write once
        w["permute_bytes"] = 2 * (sum(t.numel() * t.element_size() for t in (qd, kd, vd)) + o.numel() * 4)
    elif layout == "usp":
        Pr, Pu, rl = cfg["Pr"], cfg["Pu"], cfg["ring_layout"]
        ws = torch.empty(api.usp_attn_workspace_size(S, hq, hkv, dh, Pr, Pu, rl, True), device=dev,
                         dtype=torch.uint8)
        qz, kz, vz = (torch.empty_like(t) for t in (qd, kd, vd))
        oz = torch.empty_like(o)
        lz = torch.empty_like(lse)
        reorder = api.zigzag_reorder if rl == "zigzag" else api.striped_reorder

        def step(marks=None):
            mark(marks, 0)
            reorder(qd, Pr, out=qz)
            reorder(kd, Pr, out=kz)
            reorder(vd, Pr, out=vz)
            mark(marks, 1)
            api.usp_attn_fwd(qz, kz, vz, Pr, Pu, rl, True, o=oz, lse=lz, workspace=ws)
            mark(marks, 2)
            reorder(oz, Pr, inverse=True, out=o)
            reorder(lz, Pr, inverse=True, seq_dim=1, out=lse)
            mark(marks, 3)
        w["reorder_bytes"] = 2 * sum(t.numel() * t.element_size() for t in (qd, kd, vd, o, lse))
    else:
        cu_dev = torch.tensor(cu, dtype=torch.int32, device=dev) if cu is not None else None
        w["cu_dev"] = cu_dev
        ws = torch.empty(max(256, api.ring_attn_workspace_size(S, hq, hkv, dh, P, layout, True, dtype, cu)),
                         device=dev, dtype=torch.uint8)
        if layout in ("zigzag", "striped"):
            qz, kz, vz = (torch.empty_like(t) for t in (qd, kd, vd))
            oz = torch.empty_like(o)
            lz = torch.empty_like(lse)
            reorder = api.zigzag_reorder if layout == "zigzag" else api.striped_reorder

            def step(marks=None):
                mark(marks, 0)
                reorder(qd, P, out=qz)
                reorder(kd, P, out=kz)
                reorder(vd, P, out=vz)
                mark(marks, 1)
                api.ring_attn_fwd(qz, kz, vz, P, layout, True, cu, cu_dev, o=oz, lse=lz, workspace=ws)
                mark(marks, 2)
                reorder(oz, P, inverse=True, out=o)
                reorder(lz, P, inverse=True, seq_dim=1, out=lse)
                mark(marks, 3)
            w["reorder_bytes"] = 2 * sum(t.numel() * t.element_size() for t in (qd, kd, vd, o, lse))
        else:
            def step(marks=None):
                api.ring_attn_fwd(qd, kd, vd, P, layout, True, cu, cu_dev, o=o, lse=lse, workspace=ws)
    w["fwd_ws"] = ws
    if pass_ == "bwd":
        make_bwd_step(w, api, synth, dev, ws, host)
    else:
        w["step"] = step
        w["ws_bytes"] = ws.numel()
    w["pass"] = pass_
    return w


def make_bwd_step(w, api, synth, dev, fwd_ws, host):
    """Backward step of a ring workload: cp_ring_attn_bwd on inputs already in
    the rank-major shard order, with O and LSE from one forward call made here
    (outside any timed region) and a seeded upstream gradient dO."""
    layout, P, cu = w["layout"], w["P"], w["cu"]
    if layout not in ("contiguous", "zigzag", "striped"):
        raise SystemExit(f"--pass bwd needs a ring workload, not {layout}")
    qd, kd, vd = w["in"]
    S, hq, hkv, dh = w["S"], w["hq"], w["hkv"], w["dh"]
    if w["dtype"] != torch.bfloat16:
        raise SystemExit("--pass bwd takes bf16 workloads")
    do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5).to(dev)
    if layout != "contiguous":
        reorder = api.zigzag_reorder if layout == "zigzag" else api.striped_reorder
        qd, kd, vd, do = (reorder(t, P) for t in (qd, kd, vd, do))
    cu_dev = w.get("cu_dev")
    o, lse = w["out"]
    api.ring_attn_fwd(qd, kd, vd, P, layout, True, cu, cu_dev, o=o, lse=lse, workspace=fwd_ws)
    dq = torch.empty((S, hq, dh), device=dev, dtype=torch.float32)
    dk = torch.empty((S, hkv, dh), device=dev, dtype=torch.float32)
    dv = torch.empty_like(dk)
    ws = torch.empty(api.ring_attn_bwd_workspace_size(S, hq, hkv, dh, P, layout, True, cu), device=dev,
                     dtype=torch.uint8)
    torch.cuda.synchronize()

    def step(marks=None):
        api.ring_attn_bwd(qd, kd, vd, o, lse, do, P, layout, True, cu, cu_dev, dq=dq, dk=dk, dv=dv, workspace=ws)

    w["step"] = step
    w["ws_bytes"] = ws.numel()
    if host:
        w["host"] = [t.cpu().pin_memory() for t in (qd, kd, vd, o, lse, do)]
    w["in"] = (qd, kd, vd, o, lse, do)
    w["out"] = (dq, dk, dv)
    w["fwd_flops"] = w["flops"]
    # five score-sized products (S, dP, dV, dK, dQ) against the forward's two
    w["flops"] = 2.5 * w["flops"]


def time_steps(w, steps, warmup, ws):
    """W untimed steps, then exactly K steps bracketed by a barrier and a
    synchronize on both sides.  Inside the timed region every step also
    records the library's phase events (attention begin / end, merge end; for
    the backward the dQ / dK-dV boundary) and the layout-kernel marks."""
    from context_exact_attention_step_b200 import api
    step = w["step"]
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    n_ev = 9
    evs = [[ev() for _ in range(n_ev)] for _ in range(steps)]
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    n0 = api.kernel_launch_count()
    t0.record()
    for i in range(steps):
        e = evs[i]
        e[0].record()
        api.set_profile_events(e[1], e[2], e[3])
        step(e[4:8])
        e[8].record()
    t1.record()
    api.set_profile_events(None, None, None)
    torch.cuda.synchronize()
    launches = api.kernel_launch_count() - n0
    barrier(ws)
    err = api.device_error()
    if err:
        raise RuntimeError(f"device error word {err:#x}: a kernel gave up waiting")
    has_marks = w["reorder_bytes"] > 0 and w.get("pass") != "bwd"
    r = {"ms": t0.elapsed_time(t1) / steps, "launches": launches}
    # per step: e0 start, e1 attention begin, e2 attention end, e3 merge end
    # (bwd: dQ end), e4..e7 reorder marks, e8 end
    r["attn"] = [e[1].elapsed_time(e[2]) for e in evs]
    if w.get("pass") == "bwd":
        r["dq"] = [e[1].elapsed_time(e[3]) for e in evs]
        r["dkdv"] = [e[3].elapsed_time(e[2]) for e in evs]
    elif w["layout"] == "ulysses":  # permutes: before and after the attention, inside the call
        r["permute"] = [e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[8]) for e in evs]
    else:
        r["merge"] = [e[2].elapsed_time(e[3]) for e in evs]
    if has_marks:
        r["reorder"] = [e[4].elapsed_time(e[5]) + e[6].elapsed_time(e[7]) for e in evs]
    return r


def merge_bytes(w):
    """Algorithmic bytes of the merge: every live partial (O fp32 + LSE) read
    once, the output O and LSE written once."""
    from context_exact_attention_step_b200 import api
    cfg = w["cfg"]
    if w["layout"] == "usp":  # Pu rings of Pr ranks over hq/Pu heads each
        sch = api.ring_schedule(w["S"], cfg["Pr"], cfg["ring_layout"], True, w["cu"])
    else:
        sch = api.ring_schedule(w["S"], w["P"], w["layout"], True, w["cu"])
    rows = int(sch["q_rows"].sum())
    per_row = w["hq"] * (w["dh"] + 1) * 4
    return rows * per_row + w["S"] * per_row


def summarize(w, r, pk, ws):
    """Per-workload figures: step, attention kernel, merge / reorder / permute
    kernels; times are means over the timed steps, max over ranks."""
    ms = max_over_ranks(r["ms"], ws)
    out = {"ms_per_step": ms, "tflops": tflops(w["flops"] * ws, ms), "flops_per_step": w["flops"],
           "admitted_pairs": w["pairs"]}
    am = max_over_ranks(statistics.mean(r["attn"]), ws)
    if w.get("pass") == "bwd":
        out["kernels"] = {"ms": am, "tflops": tflops(w["flops"], am), "frac": tflops(w["flops"], am) / pk["bf16"]}
        for name, gemms in (("dq", 3), ("dkdv", 4)):
            kms = max_over_ranks(statistics.mean(r[name]), ws)
            ex = gemms / 2.0 * w["fwd_flops"]  # tensor work the kernel executes (S, dP, dQ / S^T, dP^T, dV, dK)
            out[name] = {"ms": kms, "executed_tflops": tflops(ex, kms), "executed_frac": tflops(ex, kms) / pk["bf16"]}
        return out
    out["attn"] = {"ms": am, "tflops": tflops(w["flops"], am), "frac": tflops(w["flops"], am) / pk["bf16"],
                   "frac_of_sustained": tflops(w["flops"], am) / pk["bf16_sus"],
                   # the capture is of the full-size workload: none for a --seq-len override
                   "traffic": ATTN_TRAFFIC.get((attn_src_hash(), w["name"])) if not w.get("resized") else None}
    if "merge" in r:
        mb = merge_bytes(w)
        mm = max_over_ranks(statistics.mean(r["merge"]), ws)
        out["merge"] = {"ms": mm, "gbs": gbs(mb, mm), "frac_hbm": gbs(mb, mm) / pk["hbm_gbs"], "bytes": mb}
    if "reorder" in r:
        rm = max_over_ranks(statistics.mean(r["reorder"]), ws)
        rb = w["reorder_bytes"]
        out["reorder"] = {"ms": rm, "gbs": gbs(rb, rm), "frac_hbm": gbs(rb, rm) / pk["hbm_gbs"], "bytes": rb,
                          "what": f"{w['cfg'].get('ring_layout', w['layout'])} reorder of Q, K, V and inverse of O, LSE"}
    if "permute" in r:
        pm = max_over_ranks(statistics.mean(r["permute"]), ws)
        pb = w["permute_bytes"]
        out["permute"] = {"ms": pm, "gbs": gbs(pb, pm), "frac_hbm": gbs(pb, pm) / pk["hbm_gbs"], "bytes": pb,
                          "what": "seq->head of Q, K, V (bf16) + head->seq of O (fp32)"}
    return out


def time_e2e(w, steps):
    """Same step through the public API with host buffers: every step copies
    its pinned host inputs (Q, K, V; for the backward also O, LSE, dO) in and
    its outputs (O, LSE; for the backward dQ, dK, dV) out inside the timed
    region.  Steps are pipelined the way a serving loop runs them: the upload
    of step i+1 (H2D stream) and the download of step i-1 (D2H stream) overlap
    the computation of step i (compute stream), through two device staging
    slots; the device-to-device copies between a slot and the step's own
    tensors run on the compute stream and are timed too."""
    hosts_in = w["host"]
    devs_in = w["in"]
    devs_out = w["out"]
    hosts_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in devs_out] for _ in range(2)]
    stage_in = [[torch.empty_like(t) for t in devs_in] for _ in range(2)]
    stage_out = [[torch.empty_like(t) for t in devs_out] for _ in range(2)]
    s_h, s_c, s_d = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    plain = lambda: torch.cuda.Event()
    in_ready, in_free = [plain(), plain()], [plain(), plain()]
    out_ready, out_free = [plain(), plain()], [plain(), plain()]

    def one(i):
        slot = i % 2
        with torch.cuda.stream(s_h):
            s_h.wait_event(in_free[slot])
            for d, h in zip(stage_in[slot], hosts_in):
                d.copy_(h, non_blocking=True)
            in_ready[slot].record(s_h)
        with torch.cuda.stream(s_c):
            s_c.wait_event(in_ready[slot])
            for d, st in zip(devs_in, stage_in[slot]):
                d.copy_(st, non_blocking=True)
            in_free[slot].record(s_c)
            w["step"]()
            s_c.wait_event(out_free[slot])
            for st, d in zip(stage_out[slot], devs_out):
                st.copy_(d, non_blocking=True)
            out_ready[slot].record(s_c)
        with torch.cuda.stream(s_d):
            s_d.wait_event(out_ready[slot])
            for h, st in zip(hosts_out[slot], stage_out[slot]):
                h.copy_(st, non_blocking=True)
            out_free[slot].record(s_d)

    cur = torch.cuda.current_stream()
    for i in range(2):  # warm the pipeline
        one(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(cur)
    for s_ in (s_h, s_c, s_d):
        s_.wait_event(t0)
    for i in range(steps):
        one(i)
    for s_ in (s_h, s_c, s_d):
        cur.wait_stream(s_)
    t1.record(cur)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    h2d = sum(t.numel() * t.element_size() for t in hosts_in)
    d2h = sum(t.numel() * t.element_size() for t in hosts_out[0])
    return ms, h2d, d2h


# ----------------------------------------------------------------- multi-GPU ring, rank by rank
NVLINK_PEER_GBS = 770.0  # measured peer-copy bandwidth per direction on this hardware (B200, NVLink 5)


def time_per_rank(w, reps=5):
    """The kernel work of every rank of the multi-GPU ring (``distributed``),
    run rank after rank on this GPU through the same entry points: forward,
    the block pairs of the rank's live ring steps and its merge; backward, the
    prep and, per live step, the dK/dV and dQ block-pair kernels.  The
    exchanges cannot run on one GPU; their bytes per step and their time at
    the peer-copy bandwidth are reported beside the compute."""
    from context_exact_attention_step_b200 import api
    from context_exact_attention_step_b200 import distributed as D
    S, P, layout, cu = w["S"], w["P"], w["layout"], w["cu"]
    if layout not in ("contiguous", "zigzag", "striped"):
        raise SystemExit("--per-rank needs a ring workload")
    hq, hkv, dh = w["hq"], w["hkv"], w["dh"]
    n = S // P
    dev = torch.device("cuda")
    bwd = w.get("pass") == "bwd"
    cu_dev = torch.tensor(cu, dtype=torch.int32, device=dev) if cu is not None else None
    sch = api.ring_schedule(S, P, layout, True, cu)
    if bwd:
        qs, ks, vs, o, lse, dos = w["in"]
    else:
        qs, ks, vs = w["in"]
        if w["dtype"] != torch.bfloat16:
            raise SystemExit("--per-rank takes bf16 workloads")
        if layout != "contiguous":
            reorder = api.zigzag_reorder if layout == "zigzag" else api.striped_reorder
            qs, ks, vs = (reorder(t, P) for t in (qs, ks, vs))
    parts_o = [torch.empty((n, hq, dh), device=dev, dtype=torch.float32) for _ in range(P)]
    parts_l = [torch.empty((hq, n), device=dev, dtype=torch.float32) for _ in range(P)]
    o_r = torch.empty((n, hq, dh), device=dev, dtype=torch.float32)
    l_r = torch.empty((hq, n), device=dev, dtype=torch.float32)
    lg = torch.empty((hq, n), device=dev, dtype=torch.float32)
    dd = torch.empty_like(lg)
    dq = torch.empty((n, hq, dh), device=dev, dtype=torch.float32)
    dk = torch.empty((n, hkv, dh), device=dev, dtype=torch.float32)
    dv = torch.empty_like(dk)
    rows = lambda t, r: t[r * n:(r + 1) * n]
    lse_r = [lse[:, r * n:(r + 1) * n].contiguous() for r in range(P)] if bwd else None

    def rank_work(r):
        qc = D.query_chunks(S, P, layout, r)
        if bwd:
            api.attn_bwd_prep(rows(o, r), lse_r[r], rows(dos, r), lg=lg, dd=dd)
        used = 0
        for t in range(P):
            if not sch["launched"][r * P + t]:
                continue
            j = (r - t) % P
            kc = D.key_chunks(S, P, layout, r, j)
            if bwd:
                api.block_attn_bwd(rows(qs, r), rows(ks, j), rows(vs, j), rows(dos, r), lg, dd, qc, kc, True, cu_dev,
                                   dk=dk, dv=dv, parts=api.BWD_DKDV, accumulate=t > 0)
                api.block_attn_bwd(rows(qs, r), rows(ks, j), rows(vs, j), rows(dos, r), lg, dd, qc, kc, True, cu_dev,
                                   dq=dq, parts=api.BWD_DQ, accumulate=t > 0)
            else:
                api.block_attn_fwd(rows(qs, r), rows(ks, j), rows(vs, j), qc, kc, True, cu_dev,
                                   o=parts_o[used], lse=parts_l[used])
            used += 1
        if not bwd:
            api.lse_merge(parts_o[:used], parts_l[:used], o_out=o_r, lse_out=l_r)

    for r in range(P):  # warm-up
        rank_work(r)
    torch.cuda.synchronize()
    ms = []
    for r in range(P):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            rank_work(r)
        b.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b) / reps)
    if api.device_error():
        raise RuntimeError("device error word set during the per-rank runs")
    unit = (10.0 if bwd else 4.0) * dh * hq
    pairs = [int(sum(sch["live_pairs"][r * P + t] for t in range(P))) for r in range(P)]
    busiest = int(np.argmax(ms))
    kv_bytes = 2 * n * hkv * dh * 2
    grad_bytes = 2 * n * hkv * dh * 4 if bwd else 0
    live_steps = [int(sum(sch["launched"][r * P + t] for t in range(P))) for r in range(P)]
    return {
        "what": ("backward: prep, then per live ring step the dK/dV and dQ block-pair kernels" if bwd else
                 "forward: the block pairs of the rank's live ring steps, then its merge")
                + "; ranks run one after another on this GPU, exchanges not included",
        "ms": ms, "max_ms": max(ms), "live_steps": live_steps,
        "tflops_busiest_rank": unit * pairs[busiest] / (ms[busiest] * 1e-3) / 1e12,
        "tflops_P_gpus": w["flops"] / (max(ms) * 1e-3) / 1e12,
        "exchange_bytes_per_step": kv_bytes + grad_bytes,
        "exchange_ms_per_step_at_peer_bw": (kv_bytes + grad_bytes) / (NVLINK_PEER_GBS * 1e9) * 1e3,
        "compute_ms_per_live_step_busiest": ms[busiest] / max(1, live_steps[busiest]),
        "peer_bw_gbs": NVLINK_PEER_GBS,
    }


# ----------------------------------------------------------------- real multi-GPU legs
def time_dist(ws, rank, steps, warmup):
    """The ring and Ulysses with the ranks on real GPUs (``distributed``):
    every rank holds shard `rank` of the sequence; K/V rotate by NCCL
    send/recv into local buffers (ring) or move by NCCL all-to-all (Ulysses);
    no kernel reads another GPU's memory.  Time = max over ranks of the
    CUDA-event time of K calls."""
    from context_exact_attention_step_b200 import api, synth
    from context_exact_attention_step_b200 import distributed as D
    import torch.distributed as dist
    dev = torch.device("cuda")
    out = {}
    legs = [("ring_zigzag_64k", "ring"), ("ulysses_gqa_128k", "ulysses")]
    for name, kind in legs:
        cfg = synth.CONFIGS[name]
        S, hq, hkv, dh = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"]
        if kind == "ring" and S % (2 * ws):
            continue
        if kind == "ulysses" and hkv % ws:
            out[kind] = {"skipped": f"{ws} ranks do not divide the {hkv} KV heads"}
            continue
        q, k, v = (t.to(dev) for t in synth.qkv(S, hq, hkv, dh, std=cfg["std"], dtype=torch.bfloat16))
        n = S // ws
        if kind == "ring":
            q, k, v = (api.zigzag_reorder(t, ws) for t in (q, k, v))
        qs, ks, vs = (t[rank * n:(rank + 1) * n].contiguous() for t in (q, k, v))
        del q, k, v
        torch.cuda.empty_cache()
        if kind == "ring":
            call = lambda: D.ring_attn_fwd_dist(qs, ks, vs, "zigzag", True)
        else:
            call = lambda: D.ulysses_attn_fwd_dist(qs, ks, vs, True)
        for _ in range(warmup):
            call()
        torch.cuda.synchronize()
        barrier(ws)
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        for _ in range(steps):
            call()
        b.record()
        torch.cuda.synchronize()
        barrier(ws)
        ms = max_over_ranks(a.elapsed_time(b) / steps, ws)
        flops = 4.0 * dh * hq * S * (S + 1) / 2
        out[kind] = {"workload": name, "ranks": ws, "S": S, "ms_per_step": ms, "tflops": tflops(flops, ms),
                     "tflops_per_gpu": tflops(flops, ms) / ws,
                     "exchange": ("K/V of the shard to rank r+1 per ring step (NCCL send/recv, posted before the "
                                  "step's block attention)" if kind == "ring" else
                                  "all-to-all of Q, K, V to head blocks and of O, LSE back (NCCL)")}
        del qs, ks, vs
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------- CPU oracle
def oracle_sample_rate(w, target_s=12.0, max_rows=1024, seed=0, bwd=False):
    """Times the fp64 oracle on a bounded sample of the same workload: batches
    of 32 query rows (natural positions, seeded) against every key, all heads.
    Returns causal-effective TFLOP/s of the sample and what was sampled."""
    from oracle import ref
    from context_exact_attention_step_b200 import synth
    q, k, v = (t.to(torch.float64).numpy() for t in synth.qkv(w["S"], w["hq"], w["hkv"], w["dh"],
                                                                 std=w["cfg"]["std"], dtype=w["dtype"]))
    if w["dtype"] == torch.float32:  # the kernel consumes bf16-rounded values
        q, k, v = (torch.from_numpy(t).to(torch.bfloat16).double().numpy() for t in (q, k, v))
    if bwd:
        do = synth.normal((w["S"], w["hq"], w["dh"]), synth.SEED_DO, 0.5).double().numpy()
    rng = np.random.default_rng(seed)
    cu = w["cu"]
    t_total, flops, rows_done = 0.0, 0.0, 0
    while t_total < target_s and rows_done < max_rows:
        rows = np.sort(rng.integers(0, w["S"], 32))
        t0 = time.perf_counter()
        if bwd:  # the gradient work of these query rows (their dQ, their share of dK, dV)
            ref.attention_bwd(q[rows], k, v, do[rows], causal=True, cu_seqlens=cu, qpos=rows)
        else:
            ref.attention(q[rows], k, v, causal=True, cu_seqlens=cu, qpos=rows)
        t_total += time.perf_counter() - t0
        if cu is None:
            live = (rows + 1).sum()
        else:
            starts = np.asarray(cu)[np.searchsorted(cu, rows, side="right") - 1]
            live = (rows - starts + 1).sum()
        flops += (10.0 if bwd else 4.0) * w["dh"] * w["hq"] * float(live)
        rows_done += 32
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return dict(value=flops / t_total / 1e12, unit="TFLOP/s", cores=cores, kind="oracle",
                sample=f"{'gradient of ' if bwd else ''}{rows_done} query rows (seeded, uniform positions) x all "
                       f"{w['S']} keys x {w['hq']} heads, "
                       f"fp64 numpy, {t_total:.1f} s")


# ----------------------------------------------------------------- arms
def workload_identity(name, cfg, pairs, bwd):
    return {"workload": name, **{k_: cfg[k_] for k_ in ("S", "hq", "hkv", "dh", "P", "layout")},
            "causal": True, "input_dtype": cfg["dtype"], "admitted_pairs": pairs,
            "flops_per_step": (10.0 if bwd else 4.0) * cfg["dh"] * cfg["hq"] * pairs,
            **({k_: cfg[k_] for k_ in ("Pr", "Pu", "ring_layout")} if cfg["layout"] == "usp" else {}),
            **({"documents": "lengths uniform in [%d, %d], seed 4, last one truncated" % (cfg["doc_lo"], cfg["doc_hi"])}
               if cfg.get("varlen") else {})}


def run_reference(args, ws, rank):
    """Reference arm: the fp64 CPU oracle as it stands, on the same workload,
    metric and unit; every step is a bounded sample of 32 query rows."""
    if rank != 0:
        return
    from context_exact_attention_step_b200 import synth
    from oracle import ref
    name = args.workload or HEADLINE
    cfg = synth.CONFIGS[name]
    S, hq, hkv, dh = cfg["S"], cfg["hq"], cfg["hkv"], cfg["dh"]
    dtype = torch.float32 if cfg["dtype"] == "fp32" else torch.bfloat16
    q, k, v = (t.to(torch.bfloat16).double().numpy() for t in synth.qkv(S, hq, hkv, dh, std=cfg["std"], dtype=dtype))
    cu = None
    if cfg.get("varlen"):
        cu = synth.cu_seqlens_from_lengths(synth.doc_lengths(S, cfg["doc_lo"], cfg["doc_hi"])).tolist()
    rng = np.random.default_rng(1)
    rows_per_step = 32
    bwd = args.pass_ == "bwd"
    if bwd:
        do = synth.normal((S, hq, dh), synth.SEED_DO, 0.5).double().numpy()

    def step():
        rows = np.sort(rng.integers(0, S, rows_per_step))
        if bwd:  # the gradient work of these query rows (their dQ, their share of dK, dV)
            ref.attention_bwd(q[rows], k, v, do[rows], causal=True, cu_seqlens=cu, qpos=rows)
        else:
            ref.attention(q[rows], k, v, causal=True, cu_seqlens=cu, qpos=rows)
        if cu is None:
            return float((rows + 1).sum())
        starts = np.asarray(cu)[np.searchsorted(cu, rows, side="right") - 1]
        return float((rows - starts + 1).sum())

    # the workload's identity, as the GPU arm reports it (causal pairs in
    # closed form: S(S+1)/2, or the sum of L(L+1)/2 over the documents)
    lens = np.diff(np.asarray(cu, dtype=np.int64)) if cu is not None else np.array([S], dtype=np.int64)
    pairs = int((lens * (lens + 1) // 2).sum())
    ref_config = workload_identity(name, cfg, pairs, bwd)
    if bwd:
        ref_config["pass"] = "backward: the gradient of the sampled query rows"
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    live = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    val = (10.0 if bwd else 4.0) * dh * hq * live / dt / 1e12
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC_BWD if bwd else METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": ref_config,
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{'gradient of ' if bwd else ''}{rows_per_step} seeded query rows x all keys x "
                                   f"all heads per step"},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def free(w):
    for key in ("in", "out", "host", "fwd_ws", "step", "cu_dev"):
        w.pop(key, None)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run_ours(args, ws, rank, local):
    from context_exact_attention_step_b200 import build as _build
    _build.build()
    pk = peaks()
    bwd = args.pass_ == "bwd"
    name = args.workload or HEADLINE
    suite = args.workload is None and not args.no_suite and not bwd
    clocks = Clocks(local)

    w = make_workload(name, args.seq_len, args.pass_, host=True)
    clocks.start()
    r = time_steps(w, args.steps, args.warmup, ws)
    clocks.stop()
    head = summarize(w, r, pk, ws)
    e2e_ms, h2d, d2h = time_e2e(w, args.e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, ws)
    per_rank = time_per_rank(w) if args.per_rank else None
    ident = workload_identity(name, w["cfg"], w["pairs"], bwd)
    ident["S"] = w["S"]
    cpu = oracle_sample_rate(w, bwd=bwd) if (rank == 0 and ws == 1 and not args.no_cpu_baseline) else None
    head_flops = w["flops"]
    free(w)

    configs, bwd_configs = {}, {}
    if suite:
        for sname in SUITE:
            sw = make_workload(sname)
            clocks.start()
            sr = time_steps(sw, args.steps, args.warmup, ws)
            clocks.stop()
            configs[sname] = summarize(sw, sr, pk, ws)
            free(sw)
        for sname in BWD_SUITE:
            sw = make_workload(sname, pass_="bwd")
            clocks.start()
            sr = time_steps(sw, args.steps, args.warmup, ws)
            clocks.stop()
            bwd_configs[sname] = summarize(sw, sr, pk, ws)
            free(sw)
    dist_legs = time_dist(ws, rank, args.steps, args.warmup) if ws > 1 and not args.no_dist else None

    if bwd:
        kern = head["kernels"]
        roof = {"bound": "tensor", "kernel": "attn_bwd_dq_kernel + attn_bwd_dkdv_kernel", "achieved": kern["tflops"],
                "peak": pk["bf16"], "unit": "TFLOP/s", "frac": kern["frac"], "traffic": None,
                "peak_source": pk["source"] + " burst bf16", "ms": kern["ms"]}
    else:
        a = head["attn"]
        roof = {"bound": "tensor", "kernel": "attn_fwd_kernel", "achieved": a["tflops"], "peak": pk["bf16"],
                "unit": "TFLOP/s", "frac": a["frac"], "traffic": a["traffic"],
                "peak_source": pk["source"] + " burst bf16", "frac_of_sustained": a["frac_of_sustained"],
                "frac_of_nominal_2250": a["tflops"] / 2250.0, "attn_ms": a["ms"]}
    line = {
        "metric": METRIC_BWD if bwd else METRIC, "value": head["tflops"], "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**ident,
                   "l2": "inputs larger than L2 (%.0f MB read per step, no flush needed)" % (h2d / 1e6),
                   "per_gpu": "independent problem per GPU (the P virtual ranks of one problem share a GPU)",
                   **({"pass": "backward (prep + dQ kernel + dK/dV kernel), inputs in shard order"} if bwd else {})},
        "roofline": roof,
        "e2e": {"value": tflops(head_flops * ws, e2e_ms), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "H2D of step i+1 and D2H of step i-1 overlap step i (two staging slots)"},
        "gpu_launches": int(r["launches"]),
        "clocks": clocks.summary(),
    }
    for key in ("merge", "reorder", "permute", "dq", "dkdv"):
        if key in head:
            line[key] = head[key]
    if configs:
        line["configs"] = configs
        if "ulysses_gqa_128k" in configs:
            p = configs["ulysses_gqa_128k"]["permute"]
            line["a2a_permute"] = {**p, "workload": "ulysses_gqa_128k"}
    if bwd_configs:
        line["bwd"] = bwd_configs
    if dist_legs:
        line["dist"] = dist_legs
    if per_rank:
        line["per_rank"] = per_rank
    if cpu:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def check_launch(ws, rank):
    """--check-launch: the launcher and the rank bookkeeping without a GPU
    (gloo): every rank reports, rank 0 prints one line."""
    import torch.distributed as dist
    if ws > 1:
        t = torch.tensor([rank], dtype=torch.int64)
        got = [torch.zeros(1, dtype=torch.int64) for _ in range(ws)]
        dist.all_gather(got, t)
        ranks = [int(x.item()) for x in got]
        slowest = max_over_ranks(1.0 + rank, ws)
        barrier(ws)
    else:
        ranks, slowest = [0], 1.0
    if rank == 0:
        print(json.dumps({"n_gpus": ws, "ranks": ranks, "max_over_ranks": slowest}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--workload", default=None,
                    help=f"time only this workload (default: {HEADLINE} plus the per-config suite)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time the ring backward (dQ, dK, dV) of a ring workload instead of the forward")
    ap.add_argument("--no-suite", action="store_true", help="headline workload only")
    ap.add_argument("--no-dist", action="store_true", help="skip the multi-GPU ring / Ulysses legs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-rank", action="store_true",
                    help="also time each rank's kernel work of the multi-GPU ring (ring workloads)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's sequence length (smaller cases for profiler captures)")
    ap.add_argument("--check-launch", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks\n")
        sys.exit(2)
    if args.check_launch:
        ws, rank, _ = dist_init("gloo")
        try:
            check_launch(ws, rank)
        finally:
            if ws > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, world, int(os.environ.get("RANK", "0")))
        return
    ws, rank, local = dist_init()
    try:
        run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
