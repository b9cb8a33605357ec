#!/usr/bin/env python
"""Throughput of the Lighthouse Attention layer's hot path on B200.

One step = one pass of the whole hot path over one batch: pyramid + scores,
joint top-k and order, gather, causal attention, scatter-back (forward) and
scatter adjoint, attention backward (dK/dV and dQ), gather/pooling adjoint
(backward).  The workload is the pages' single-B200 shape: B=1, H=8, d=128,
N=524288, L=3, p=4, k=4096 (S=65536), bf16, seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  Under torchrun (N > 1) every rank runs its
own full workload (weak scaling, no collective on the data path); the
reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hierarchical_selection_attention_b200.inputs import WORKLOADS, make_dout, make_qkv  # noqa: E402

METRIC = "Lighthouse layer fwd & fwd+bwd tokens/s at N=512K on 1 B200; per-stage % roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = 3          # n512k_l3_p4_k4096
SELECT_NAMES = {0: "joint top-k", 1: "per-level quota", 2: "stratified"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=j["hbm_gbs"], tf_burst=j["bf16_tflops"],
                    tf_sust=j.get("bf16_tflops_sustained", j["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, tf_burst=1590.0, tf_sust=1400.0, src="fallback")


def sizes(w):
    B, N, H, d, L, p, k = (w[x] for x in ("B", "N", "H", "d", "L", "p", "k"))
    S = N // p ** (L - 1) + (L - 1) * p * k
    P = sum(N // p**l for l in range(L))
    R = P - N
    C = sum(N // p**l for l in range(L - 1))
    return B, N, H, d, L, p, k, S, P, R, C


def algorithmic(w):
    """Per-launch algorithmic bytes (HBM stages) and FLOPs (attention) of each
    stage: the bytes the method must move at least once, the FLOPs of the
    causal GEMMs over the S x S triangle (diagonal included)."""
    B, N, H, d, L, p, k, S, P, R, C = sizes(w)
    tok = B * N * H * d * 2          # one [B, N, H, d] bf16 tensor
    gat = B * H * S * d * 2          # one [B, H, S, d] bf16 tensor
    tri = B * H * d * S * (S + 1)    # one causal GEMM: sum over rows of 2 d (row + 1)
    return {
        "pyramid": ("hbm", 3 * tok + 3 * B * R * H * d * 2 + 2 * B * H * P * 4),
        "select": ("hbm", 2 * B * H * C * 4 + B * H * S * 4 + B * H * P * 4),
        "gather": ("hbm", 6 * gat + B * H * S * 4),
        "attn_fwd": ("tensor", 2 * tri),
        "scatter": ("hbm", gat + tok + B * H * P * 4),
        "scatter_bwd": ("hbm", tok + 2 * gat + B * H * S * 4),   # dO, og in; dog, D out
        "attn_bwd_dkdv": ("tensor", 4 * tri),
        "attn_bwd_dq": ("tensor", 1 * tri),    # dS K; S and dP are recomputed (2 more GEMMs)
        "gather_bwd": ("hbm", 3 * gat + 3 * tok + B * H * P * 4),
    }


def algorithmic_writes(w):
    """The part of each HBM stage's algorithmic bytes that is written."""
    B, N, H, d, L, p, k, S, P, R, C = sizes(w)
    tok = B * N * H * d * 2
    gat = B * H * S * d * 2
    return {
        "pyramid": 3 * B * R * H * d * 2 + 2 * B * H * P * 4,
        "select": B * H * S * 4 + B * H * P * 4,
        "gather": 3 * gat,
        "scatter": tok,
        "scatter_bwd": gat + B * H * S * 4,
        "gather_bwd": 3 * tok,
    }


def write_bandwidth(dev, nbytes=1 << 30):
    """Measured write-only bandwidth of this GPU (GB/s): a zero fill of
    `nbytes` (torch's fill kernel, CUDA events, best of 5).  HBM sustains far
    less writing alone than the read + write mix of a copy, so a stage that
    mostly writes is bounded by this figure, not by the copy peak."""
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    best = None
    for i in range(7):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        buf.zero_()
        b.record()
        torch.cuda.synchronize(dev)
        if i >= 2:
            t = a.elapsed_time(b)
            best = t if best is None else min(best, t)
    del buf
    return nbytes / (best / 1e3) / 1e9


EXECUTED_GEMMS = {"attn_fwd": 2, "attn_bwd_dkdv": 4, "attn_bwd_dq": 3}


class Clocks:
    """nvidia-smi sampling while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank time over all ranks (the slowest replica sets the
    job's time).  The reduction tensor lives where the process group's
    backend wants it: on the GPU for NCCL, on the CPU for gloo."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(ws: int, B: int, N: int, ms_step: float) -> float:
    """Whole-job throughput of ws independent replicas, each processing B x N
    tokens per step, with the step time taken as the max over ranks."""
    return ws * B * N / (ms_step / 1e3)


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------- our arm --

def bench_config(args, w, ws):
    """The workload description both arms print (the driver compares them)."""
    B, N, H, d, Lv, p, k, S, P, R, C = sizes(w)
    tok_gib = 3 * B * N * H * d * 2 / 2**30
    return {"workload": f"{w['name']}: B={B} N={N} H={H} d={d} L={Lv} p={p} k={k} S={S}",
            "step": "lh_forward + lh_backward stages (fwd+bwd)",
            "l2": f"inputs larger than L2 ({tok_gib:.2f} GiB of Q,K,V per step); no flush",
            "parallelism": (f"head split over {ws} ranks (one layer; no collective)"
                            if args.head_split and ws > 1 else
                            f"replicas x{ws} (independent layers, no collective)"),
            "selection": SELECT_NAMES[args.select_mode] +
            (f", {args.select_chunk} per chunk" if args.select_mode == 2 else "")}


def run_ours(args, w, ws, rank, local):
    from hierarchical_selection_attention_b200 import lighthouse as L

    B, N, H, d, Lv, p, k, S, P, R, C = sizes(w)
    dev = torch.device("cuda", local)
    qh, kh, vh = make_qkv(B, N, H, d, seed=args.workload)
    doh = make_dout(B, N, H, d, seed=args.workload)
    # head split: this rank runs the whole layer on its contiguous head range
    # of the one job-wide layer (the job's tokens are counted once)
    share, w_job = ws, w
    if args.head_split and ws > 1:
        from hierarchical_selection_attention_b200.heads import head_range
        h0, h1 = head_range(H, ws, rank)
        qh, kh, vh, doh = (x[:, :, h0:h1].contiguous() for x in (qh, kh, vh, doh))
        H, share = h1 - h0, 1
        w = dict(w, H=H)
    q, kk, v, dout = (t.to(dev) for t in (qh, kh, vh, doh))
    sel = dict(select_mode=args.select_mode, select_chunk=args.select_chunk)
    cfg = L.make_config(B, N, H, d, Lv, p, k, **sel)
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, device=dev, **sel)
    sv = layer.views()
    e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=dev)
    fws, _, _ = L.lh_workspace_bytes(cfg)
    ws_f = torch.empty(fws, dtype=torch.uint8, device=dev)
    q_lv, k_lv, v_lv = (e(max(B * R * H * d, 1)) for _ in range(3))
    qk, kq = e(B, H, P, dt=torch.float32), e(B, H, P, dt=torch.float32)
    o = torch.empty_like(q)
    dog, delta = e(B, H, S, d), e(B, H, S, dt=torch.float32)
    dqg, dkg, dvg = (e(B, H, S, d) for _ in range(3))
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    stages = [
        ("pyramid", lambda: L.lh_pyramid(cfg, q, kk, v, q_lv, k_lv, v_lv, qk, kq)),
        ("select", lambda: L.lh_score_topk(cfg, qk, kq, sv["sel_idx"], sv["slot_map"], ws_f)),
        ("gather", lambda: L.lh_gather(cfg, q, kk, v, q_lv, k_lv, v_lv, sv["sel_idx"], sv["qg"],
                                       sv["kg"], sv["vg"])),
        ("attn_fwd", lambda: L.lh_attn_fwd(cfg, sv["qg"], sv["kg"], sv["vg"], sv["og"], sv["lse"],
                                           og_lo=sv["og_lo"])),
        ("scatter", lambda: L.lh_scatter(cfg, sv["og"], sv["slot_map"], o)),
        ("scatter_bwd", lambda: L.lh_scatter_bwd(cfg, dout, sv["og"], sv["sel_idx"], dog, delta,
                                                 og_lo=sv["og_lo"])),
        ("attn_bwd_dkdv", lambda: L.lh_attn_bwd_dkdv(cfg, sv["qg"], sv["kg"], sv["vg"], dog,
                                                     sv["lse"], delta, dkg, dvg)),
        ("attn_bwd_dq", lambda: L.lh_attn_bwd_dq(cfg, sv["qg"], sv["kg"], sv["vg"], dog, sv["lse"],
                                                 delta, dqg)),
        ("gather_bwd", lambda: L.lh_gather_bwd(cfg, dqg, dkg, dvg, sv["slot_map"], dq, dk, dv)),
    ]
    n_fwd = 5
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        for i, (_, fn) in enumerate(stages):
            fn()
            if evs is not None:
                evs[i + 1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    L.check_device_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
           for _ in range(args.steps)]
    clk = Clocks(local)
    clk.start()
    barrier(ws)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(ws)
    clocks = clk.stop()
    L.check_device_status()
    total_ms = max_over_ranks(t0.elapsed_time(t1), ws)
    stage_ms = {name: statistics.mean(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(args.steps))
                for i, (name, _) in enumerate(stages)}
    fwd_ms = statistics.mean(evs[s][0].elapsed_time(evs[s][n_fwd]) for s in range(args.steps))
    fwd_ms = max_over_ranks(fwd_ms, ws)

    # ---- end to end through the public API with host buffers.  Every step
    # uploads its Q, K, V, dO from pinned host memory and downloads O, dQ,
    # dK, dV into pinned host memory; three streams (upload, compute,
    # download) and two sets of device buffers let step n+1's upload and step
    # n-1's download overlap step n's compute, as a training loop feeding the
    # layer from the host would.
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.pin_memory()
        hq, hk, hv, hdo = (pin(t) for t in (qh, kh, vh, doh))
        ho, hdq, hdk, hdv = (torch.empty_like(hq).pin_memory() for _ in range(4))
        ins = [(q, kk, v, dout), tuple(torch.empty_like(x) for x in (q, kk, v, dout))]
        outs = [(o, dq, dk, dv), tuple(torch.empty_like(x) for x in (o, dq, dk, dv))]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_ready, in_free = [ev(), ev()], [ev(), ev()]
        out_ready, out_free = [ev(), ev()], [ev(), ev()]
        for e in in_free + out_free:
            e.record(stream)

        def e2e_step(n):
            i = n & 1
            with torch.cuda.stream(up):
                up.wait_event(in_free[i])
                for dst, src in zip(ins[i], (hq, hk, hv, hdo)):
                    dst.copy_(src, non_blocking=True)
                in_ready[i].record(up)
            stream.wait_event(in_ready[i])
            stream.wait_event(out_free[i])
            xq, xk, xv, xdo = ins[i]
            yo, ydq, ydk, ydv = outs[i]
            layer.forward(xq, xk, xv, out=yo)
            layer.backward(xdo, grads=(ydq, ydk, ydv))
            in_free[i].record(stream)
            out_ready[i].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(out_ready[i])
                for dst, src in zip((ho, hdq, hdk, hdv), outs[i]):
                    dst.copy_(src, non_blocking=True)
                out_free[i].record(down)

        for n in range(max(1, min(args.warmup, 2))):
            e2e_step(n)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 10))
        barrier(ws)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(up)
        for n in range(n_e2e):
            e2e_step(n)
        b.record(down)
        torch.cuda.synchronize(dev)
        barrier(ws)
        L.check_device_status()
        e2e_ms = max_over_ranks(a.elapsed_time(b), ws) / n_e2e
        nbytes = B * N * H * d * 2
        e2e = {"value": share * B * N / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 4 * nbytes, "d2h_bytes_per_step": 4 * nbytes,
               "api": "LighthouseLayer.forward/backward (lh_forward + lh_backward), pinned host buffers; upload, compute and download on three streams, overlapped across steps"}

    # ---- roofline, per stage and for the dominant kernel
    pk = peaks()
    alg = algorithmic(w)
    wr = algorithmic_writes(w)
    wr_gbs = write_bandwidth(dev)
    per_stage = {}
    for name, ms in stage_ms.items():
        bound, amount = alg[name]
        if bound == "hbm":
            ach = amount / (ms / 1e3) / 1e9
            # the shortest time its bytes allow: all of them at the copy rate,
            # or its writes at the write-only rate, whichever is longer
            t_min = max(amount / pk["hbm"], wr[name] / wr_gbs) / 1e9 * 1e3
            per_stage[name] = {"ms": round(ms, 4), "bound": "hbm", "GB/s": round(ach, 1),
                               "frac": round(ach / pk["hbm"], 4), "algorithmic_bytes": amount,
                               "written_bytes": wr[name],
                               "frac_rw": round(t_min / ms, 4)}
        else:
            ach = amount / (ms / 1e3) / 1e12
            one_gemm = alg["attn_fwd"][1] / 2
            tc = EXECUTED_GEMMS[name] * one_gemm / (ms / 1e3) / 1e12
            per_stage[name] = {"ms": round(ms, 4), "bound": "tensor", "TFLOP/s": round(ach, 1),
                               "frac": round(ach / pk["tf_sust"], 4), "algorithmic_flops": amount,
                               "executed_TFLOP/s": round(tc, 1)}
    dom = max(stage_ms, key=stage_ms.get)
    bound, amount = alg[dom]
    if bound == "hbm":
        ach = amount / (stage_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": pk["hbm"],
                "unit": "GB/s", "frac": round(ach / pk["hbm"], 4), "traffic": None}
    else:
        ach = amount / (stage_ms[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 1), "peak": pk["tf_sust"],
                "unit": "TFLOP/s", "frac": round(ach / pk["tf_sust"], 4), "traffic": None}
    roof["peak_source"] = f"{pk['src']} (bf16 sustained for tensor, copy for HBM)"
    traffic = load_traffic(dom, w_job["name"])
    if traffic is not None:
        roof["traffic"] = traffic

    launches = args.steps * (L.lh_forward_launches(cfg) + L.lh_backward_launches(cfg))
    ms_step = total_ms / args.steps
    line = {
        "metric": METRIC, "value": job_tokens_per_s(share, B, N, ms_step), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong" if share == 1 and ws > 1 else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: N(0,1) x per-token lognormal(0,0.5), 64 heavy tokens x4)",
        "config": bench_config(args, w_job, ws),
        "heads_this_rank": H,
        "fwd_tokens_per_s": share * B * N / (fwd_ms / 1e3), "fwd_ms": fwd_ms,
        "stages": per_stage, "roofline": roof, "e2e": e2e, "gpu_launches": launches,
        "hbm_write_only_GB/s": round(wr_gbs, 1),
        "clocks": clocks,
    }
    return line


def load_traffic(kernel, workload):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary (profiles/traffic.json), if it was captured for this kernel on
    this workload (null otherwise: the bytes do not carry over)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    ent = json.load(open(p)).get(kernel)
    if ent is None or ent.get("workload_name") != workload:
        return None
    return ent.get("dram_bytes_per_launch")


# ----------------------------------------------------------- oracle timing --

def oracle_sample(w, rows_per_head: int, seed: int):
    """Time the CPU oracle on a bounded sample of the workload: one (b, h)
    head over all N tokens (scores, selection, order, pyramid, gather,
    scatter and both adjoints) plus the attention forward and backward of
    `rows_per_head` query rows spread evenly over S; the attention part is
    scaled by S / rows_per_head, and the head by H and B.  Returns
    (tokens/s, seconds measured, description)."""
    from oracle import lighthouse_oracle as lo

    B, N, H, d, Lv, p, k, S, P, R, C = sizes(w)
    q, kk, v = make_qkv(1, N, 1, d, seed=seed)
    dout = make_dout(1, N, 1, d, seed=seed)
    qh, kh, vh, doh = (x[0, :, 0, :].double().numpy() for x in (q, kk, v, dout))
    scale = 1.0 / math.sqrt(d)
    t0 = time.perf_counter()
    sel = lo.select_head(qh, kh, Lv, p, k)
    pyr = [lo.pyramid(x, Lv, p) for x in (qh, kh, vh)]
    qg, kg, vg = (lo.gather_rows(lv, sel["sel_idx"], N, Lv, p) for lv in pyr)
    dog = lo.scatter_bwd(doh, sel["sel_idx"], N, Lv, p)
    t_lin = time.perf_counter() - t0
    rows = np.linspace(0, S - 1, rows_per_head).astype(np.int64)
    t1 = time.perf_counter()
    og_rows, _ = lo.attention(qg, kg, vg, scale, rows=rows)
    dqg, dkg, dvg = lo.attention_bwd(qg, kg, vg, dog, scale, rows=rows)
    t_att = time.perf_counter() - t1
    t2 = time.perf_counter()
    og = np.zeros_like(qg)
    og[rows] = og_rows
    lo.scatter(og, sel["slot_map"], N, Lv, p)
    for g in (dqg, dkg, dvg):
        lo.pyramid_bwd(g, sel["slot_map"], N, Lv, p)
    t_lin += time.perf_counter() - t2
    head_s = t_lin + t_att * S / rows_per_head
    tok_s = B * N / (head_s * H * B)
    measured = time.perf_counter() - t0
    desc = (f"one (b,h) head of {w['name']}: all N={N} tokens through scores/top-k/order/pyramid/"
            f"gather/scatter/adjoints, attention fwd+bwd on {rows_per_head} of S={S} query rows "
            f"(scaled by S/{rows_per_head}), times B*H={B * H} heads; measured {measured:.1f} s")
    return tok_s, measured, desc


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def host_cores() -> dict:
    """Cores the oracle ran on: its matrix products use the BLAS threads; its
    element-wise passes, sorts and scans run on one thread."""
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:
        aff = os.cpu_count() or 1
    cpu = ""
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                cpu = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"blas_threads": blas_threads(), "affinity_cores": aff, "cpu_model": cpu}


def oracle_whole_head(wi: int = 1):
    """One (b, h) head of a workload through the whole oracle, forward and
    backward over every token and all S gathered rows, timed whole (no
    sampling, no extrapolation).  Returns (seconds, description)."""
    from oracle import lighthouse_oracle as lo
    w = WORKLOADS[wi]
    B, N, H, d, Lv, p, k, S, P, R, C = sizes(w)
    q, kk, v = make_qkv(1, N, 1, d, seed=wi)
    dout = make_dout(1, N, 1, d, seed=wi)
    qh, kh, vh, doh = (x[0, :, 0, :].double().numpy() for x in (q, kk, v, dout))
    t0 = time.perf_counter()
    st = lo.forward_head(qh, kh, vh, Lv, p, k, parity=True)
    lo.backward_head(st, doh)
    sec = time.perf_counter() - t0
    return sec, (f"one (b,h) head of {w['name']} (S={S}) forward+backward through the whole "
                 f"oracle, timed whole: {sec:.1f} s, i.e. {N / sec:.0f} head-tokens/s")


def run_reference(args, w):
    """The reference arm: the CPU oracle as it stands.  Each of the warm-up
    and timed steps is one bounded sample of the workload (oracle_sample);
    ms_per_step is the measured time of one such sample, and value the
    whole-workload throughput the sample's work fraction gives."""
    vals, secs = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        tok_s, sec, desc = oracle_sample(w, rows_per_head=args.oracle_rows, seed=args.workload)
        if i >= args.warmup:
            vals.append(tok_s)
            secs.append(sec)
    v = statistics.median(vals)
    cores = host_cores()
    return {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, same recipe)", "impl": "reference",
            "config": bench_config(args, w, 1),
            "arm": "CPU fp64 oracle (numpy) on the host cores; each step is one bounded sample "
                   "of the workload (cpu_baseline.sample); ms_per_step is the sample's measured "
                   "time, value the whole-workload tokens/s it extrapolates to",
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores["blas_threads"],
                             "kind": "oracle", "sample": desc, **cores},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_sweep(args):
    """Layer latency over sequence lengths (the paper's single-layer latency
    figure): B=1, H=8, d=128, L=3, p=4, k = N/128 (1:64 sparsity), N from 8K
    to 512K.  Forward and forward+backward through LighthouseLayer, CUDA
    events on the launch stream, 3 warm-up and 10 timed runs each (median).
    torch's causal scaled_dot_product_attention on the same Q, K, V is timed
    beside it as context only (fewer runs at the longest lengths)."""
    import torch.nn.functional as F
    from hierarchical_selection_attention_b200 import lighthouse as L
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    def med_ms(fn, reps, warm):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    for N in [8192 << i for i in range(7)]:
        B, H, d, Lv, p, k = 1, 8, 128, 3, 4, N // 128
        q, kk, v = (t.to(dev) for t in make_qkv(B, N, H, d, seed=0))
        dout = make_dout(B, N, H, d, seed=0).to(dev)
        layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, device=dev)
        o = torch.empty_like(q)
        grads = tuple(torch.empty_like(q) for _ in range(3))
        fwd = med_ms(lambda: layer.forward(q, kk, v, out=o), 10, 3)
        both = med_ms(lambda: (layer.forward(q, kk, v, out=o), layer.backward(dout, grads=grads)), 10, 3)
        L.check_device_status()
        line = {"N": N, "config": f"B=1 H=8 d=128 L=3 p=4 k={k} S={layer.S}",
                "lighthouse_fwd_ms": round(fwd, 3), "lighthouse_fwd_bwd_ms": round(both, 3),
                "lighthouse_fwd_tokens_per_s": B * N / (fwd / 1e3),
                "lighthouse_fwd_bwd_tokens_per_s": B * N / (both / 1e3)}
        if not args.no_sdpa:
            # context only: dense causal attention over all N tokens, [B, H, N, d] views
            try:
                qt, kt, vt = (x.permute(0, 2, 1, 3).detach().requires_grad_() for x in (q, kk, v))
                reps = 10 if N <= 65536 else 3
                dense_fwd = med_ms(lambda: F.scaled_dot_product_attention(qt, kt, vt, is_causal=True),
                                   reps, 2)

                def dense_step():
                    y = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
                    y.backward(dout.permute(0, 2, 1, 3))
                dense_both = med_ms(dense_step, reps, 2)
                line.update({"sdpa_causal_fwd_ms": round(dense_fwd, 3),
                             "sdpa_causal_fwd_bwd_ms": round(dense_both, 3),
                             "speedup_fwd": round(dense_fwd / fwd, 2),
                             "speedup_fwd_bwd": round(dense_both / both, 2)})
                del qt, kt, vt
            except RuntimeError as e:   # no dense kernel for this shape on this build
                line["sdpa_causal"] = f"unavailable: {str(e).splitlines()[0][:120]}"

        print(json.dumps(line), flush=True)
        del layer, q, kk, v, dout, o, grads
        torch.cuda.empty_cache()


def run_full_layer(args, w):
    """The layer with its projections (LighthouseProjectedLayer) on the bench
    workload, d_model = H d: forward + backward tokens/s, and the share of
    the step the Lighthouse layer itself takes.  Synthetic x, dy and weights
    (N(0,1) x 1/sqrt(d_model), bf16)."""
    from hierarchical_selection_attention_b200 import lighthouse as L
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    B, N, H, d, Lv, p, k = (w[x] for x in ("B", "N", "H", "d", "L", "p", "k"))
    Dm = H * d
    g = torch.Generator(device=dev).manual_seed(args.workload)
    x = torch.randn(B, N, Dm, generator=g, device=dev).to(torch.bfloat16)
    dy = torch.randn(B, N, Dm, generator=g, device=dev).to(torch.bfloat16)
    ws_ = [(torch.randn(*s_, generator=g, device=dev) / math.sqrt(Dm)).to(torch.bfloat16)
           for s_ in ((H * d, Dm),) * 3 + ((Dm, H * d),)]
    layer = L.LighthouseProjectedLayer(B, N, H, d, Dm, Lv, p, k, device=dev)
    y = torch.empty_like(x)
    grads = (torch.empty_like(x), *(torch.empty_like(ws_[0]) for _ in range(3)), torch.empty_like(ws_[3]))

    def step():
        layer.forward(x, *ws_, y=y)
        layer.backward(dy, grads=grads)

    def core_step():
        layer.core.forward(layer.q, layer.k, layer.v, out=layer.o)
        layer.core.backward(layer.do, grads=(layer.dq, layer.dk, layer.dv))

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / args.steps

    ms = timed(step)
    core_ms = timed(core_step)
    L.check_device_status()
    gemm_flop = 2 * B * N * Dm * H * d * (4 + 7)   # fwd: Q, K, V, y; bwd: dO, dW_o, dx (3), dW (3)
    gemm_ms = ms - core_ms
    return {"metric": "Lighthouse layer with projections, fwd+bwd tokens/s (1 B200)",
            "value": B * N / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
            "lighthouse_core_ms": core_ms, "projections_ms": gemm_ms,
            "projections_TFLOP/s": gemm_flop / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None,
            "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
            "config": {"workload": w["name"], "d_model": Dm}}


def run_ring(args, w):
    """The context-parallel layer with R shards on one GPU
    (ring.LighthouseRingLayer): shard-local stages (i)-(iii) and (iv), ring
    attention over the shards' gathered sub-sequences through the ring-step
    kernels.  One JSON line: forward and forward+backward tokens/s, and the
    ring attention's algorithmic TFLOP/s (R causal blocks of S rows and
    R (R - 1) / 2 full S x S blocks, fwd 2 GEMMs, bwd 5 algorithmic)."""
    from hierarchical_selection_attention_b200 import lighthouse as L, ring
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    B, N, H, d, Lv, p, k = (w[x] for x in ("B", "N", "H", "d", "L", "p", "k"))
    R = args.ring
    q, kk, v = (t.to(dev) for t in make_qkv(B, N, H, d, seed=args.workload))
    dout = make_dout(B, N, H, d, seed=args.workload).to(dev)
    layer = ring.LighthouseRingLayer(B, N, H, d, Lv, p, k, R, device=dev)
    o = torch.empty_like(q)
    grads = tuple(torch.empty_like(q) for _ in range(3))

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / args.steps

    fwd_ms = timed(lambda: layer.forward(q, kk, v, out=o))
    ms = timed(lambda: (layer.forward(q, kk, v, out=o), layer.backward(dout, grads=grads)))
    L.check_device_status()
    S = layer.S
    one = 2 * B * H * d                                  # FLOP per (row, key) per GEMM
    pairs = R * S * (S + 1) / 2 + R * (R - 1) / 2 * S * S
    return {"metric": f"context-parallel Lighthouse layer, {R} shards on 1 B200, fwd+bwd tokens/s",
            "value": B * N / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "fwd_ms": fwd_ms,
            "fwd_tokens_per_s": B * N / (fwd_ms / 1e3), "steps": args.steps, "warmup": args.warmup,
            "dtype": "bf16", "ring_attention_flop_fwd": 2 * one * pairs,
            "ring_attention_flop_bwd": 5 * one * pairs,
            "config": {"workload": w["name"], "shards": R, "shard_tokens": N // R,
                       "S_per_shard": S}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-rows", type=int, default=64,
                    help="query rows per head of the oracle's attention sample (both CPU legs)")
    ap.add_argument("--sweep", action="store_true",
                    help="latency over N = 8K..512K (one JSON line per N) instead of the bench line")
    ap.add_argument("--no-sdpa", action="store_true", help="--sweep without the dense SDPA context")
    ap.add_argument("--select-mode", type=int, default=0, choices=[0, 1, 2],
                    help="selection: 0 joint top-k (default), 1 per-level quota, 2 stratified")
    ap.add_argument("--select-chunk", type=int, default=0,
                    help="per-chunk quota m of the stratified selection")
    ap.add_argument("--head-split", action="store_true",
                    help="N > 1: split one layer's heads over the ranks (strong scaling) "
                         "instead of running N replicas (weak scaling)")
    ap.add_argument("--ring", type=int, default=0,
                    help="time the context-parallel layer with this many shards on one GPU")
    ap.add_argument("--full-layer", action="store_true",
                    help="time the layer with its Q/K/V/output projections (one JSON line)")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.sweep:
        run_sweep(args)
        return
    if args.full_layer:
        print(json.dumps(run_full_layer(args, w)), flush=True)
        return
    if args.ring:
        print(json.dumps(run_ring(args, w)), flush=True)
        return

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, w)), flush=True)
        return

    ws, rank, local = dist_init()
    if ws != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {ws} ranks were launched")
    try:
        line = run_ours(args, w, ws, rank, local)
        if rank == 0:
            if not args.no_cpu_baseline and ws == 1:
                samples = [oracle_sample(w, rows_per_head=args.oracle_rows, seed=args.workload)
                           for _ in range(3)]
                tok_s = statistics.median(x[0] for x in samples)
                desc = samples[0][2] + "; median of 3 such samples"
                cores = host_cores()
                line["cpu_baseline"] = {"value": tok_s, "unit": UNIT,
                                        "cores": cores["blas_threads"], "kind": "oracle",
                                        "sample": desc, **cores}
                sec, wdesc = oracle_whole_head(1)
                line["cpu_baseline"]["whole_head"] = {"seconds": sec, "workload": WORKLOADS[1]["name"],
                                                      "description": wdesc}
            print(json.dumps(line), flush=True)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
