#!/usr/bin/env python
"""Benchmark: chunk-WY forward throughput (Mtokens/s, % of HBM roofline) and decode GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one chunked forward pass over the whole workload: B=4, H=16, T=4096,
dk=dv=128, chunk 64, bf16 q/k/v, fp32 gates (seeded synthetic inputs, resident in
HBM).  The inputs (408 MB) are larger than the 126 MB L2, so no flush is needed
between steps.  Decode (256 sequences x 16 heads, fp32 state) is measured in the
same run and reported in the "decode" object, and the two other forward
workloads (B=16, H=12, T=4096 with slow decay and a random initial state; the
block-rotation variant at B=2, H=16, T=8192) each get an object of their own in
"workloads", timed the same way with their own roofline and clock record; the
backward pass (gradients of every input) on the headline workload is the "backward"
object.  Under
torchrun every rank runs its own independent batch (weak scaling, no data-path
collective); the time is the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated delta-rule fwd Mtokens/s and % roofline at H=16,dk=dv=128; decode GB/s"
WORKLOAD = "b4_h16_t4096_d128"
# every forward workload of the benchmark: the headline one, the 1.3B-layer training shape with
# slow decay and a random initial state, the block-rotation variant
FWD_WORKLOADS = ("b4_h16_t4096_d128", "b16_h12_t4096_d128_slow_s0", "b2_h16_t8192_d128_rot")
L2_BYTES = 126e6
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------- helpers ----

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws an independent batch (weak scaling)."""
    return base_seed + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "gdr_chunk_fwd_simt": ["simt_fwd.cuh", "common.cuh"],
    "gdr_chunk_fwd_tcgen05": ["tc_fwd.cuh", "tc_ptx.cuh", "common.cuh"],
    "gdr_chunk_fwd_tcgen05_split": ["tc_fwd.cuh", "tc_ptx.cuh", "common.cuh"],
    "gdr_chunk_fwd_tcgen05_waves": ["tc_fwd.cuh", "tc_ptx.cuh", "common.cuh"],
    "gdr_chunk_fwd_tcgen05_chains": ["split_fwd.cuh", "tc_ptx.cuh", "common.cuh"],
    "gdr_chunk_fwd_tcgen05_segments": ["split_fwd.cuh", "seg_combine.cuh", "tc_ptx.cuh", "common.cuh"],
    "gdr_decode_step": ["decode.cuh", "common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of one kernel's CUDA sources: a stored ncu traffic figure is only valid for it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "recurrent_state_memory_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        path = os.path.join(csrc, name)
        if os.path.exists(path):
            with open(path, "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        tab = json.load(f)
    ent = tab.get(f"{kernel}@{workload}")
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = open(os.devnull, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ our arm ----

def fwd_flops_per_token_head(dk, dv, C=64):
    """Algorithmic FLOPs per token and head, triangular products counted at half:
    6*dk*dv for the state products (Ktil S^T, Qtil S^T, E^T Kdec) and C*(3dk + 2dv)
    for the in-chunk products (A, Pm, Wk at half; U and Pm E at half)."""
    return 6 * dk * dv + C * (3 * dk + 2 * dv)


def workload_config(name, p):
    """The `config` object of the JSON line, identical in both arms for the same workload."""
    return {"workload": name, "B": p.B, "H": p.H, "T": p.T, "dk": p.dk, "dv": p.dv, "chunk": p.chunk,
            "inputs": "bf16 q/k/v, fp32 raw gate (-softplus fused) and beta" if p.dtype == "bf16" else
                      "fp32 q/k/v, gate and beta",
            "l2": f"inputs {p.nbytes_algorithmic / 1e6:.0f} MB vs L2 {L2_BYTES / 1e6:.0f} MB; no flush"}


def _to_torch(a):
    import torch
    if a is None:
        return None
    return torch.from_numpy(a.copy()).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)


def time_fwd(name, args, dev, stream, rank, ws, steps):
    """One forward workload: seeded inputs resident in HBM, W untimed warm-up launches, then
    `steps` launches timed with CUDA events on the launching stream (barrier + synchronize on
    both sides, max over ranks), with the SM clocks sampled meanwhile."""
    import torch
    import torch.distributed as dist
    from recurrent_state_memory_b200 import gdr
    from recurrent_state_memory_b200 import inputs as I

    cfg = dict(I.FWD_CONFIGS[name])
    cfg["seed"] = rank_seed(cfg["seed"], rank)
    p = I.make_fwd(name=name, **cfg)
    host = {k: _to_torch(getattr(p, k)) for k in ("q", "k", "v", "g", "beta", "theta", "S0")}
    dv_t = {k: (None if t is None else t.to(dev)) for k, t in host.items()}
    o = torch.empty((p.B, p.T, p.H, p.dv), dtype=dv_t["q"].dtype, device=dev)
    S_T = torch.empty((p.B, p.H, p.dv, p.dk), dtype=torch.float32, device=dev)
    desc = gdr.fwd_desc(p.B, p.H, p.T, p.dk, p.dv, dv_t["q"].dtype, o.dtype, p.gate_mode, p.rotation,
                        p.scale, args.algo)
    ws_bytes = gdr.workspace_bytes(desc)
    wsp = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None

    def step():
        gdr.chunk_fwd(dv_t["q"], dv_t["k"], dv_t["v"], dv_t["g"], dv_t["beta"], dv_t["theta"], dv_t["S0"],
                      gate_mode=p.gate_mode, scale=p.scale, algo=args.algo, o=o, S_T=S_T, stream=stream,
                      workspace=wsp)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t_all0, t_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        t_all0.record(stream)
        for i in range(steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    per_launch_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms_max = max_over_ranks(t_all0.elapsed_time(t_all1), dev)
    tokens = p.B * p.T
    tokens_all = sum_over_ranks(float(tokens * steps), dev)
    value = tokens_all / (total_ms_max * 1e-3) / 1e6

    peaks, peak_src = load_peaks()
    algo_bytes = p.nbytes_algorithmic
    avg_launch_s = statistics.mean(per_launch_ms) * 1e-3
    achieved_gbs = algo_bytes / avg_launch_s / 1e9
    resolved = gdr.resolved_algo(desc)
    kernel_name = "gdr_chunk_fwd_" + resolved
    roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
                "traffic": stored_traffic(kernel_name, name),
                "peak_source": f"{peak_src} HBM copy bandwidth",
                "algorithmic_bytes_per_launch": algo_bytes, "kernel": kernel_name}
    flops = fwd_flops_per_token_head(p.dk, p.dv) * tokens * p.H
    return {"p": p, "host": host, "dv_t": dv_t, "o": o, "S_T": S_T, "wsp": wsp, "desc": desc,
            "resolved": resolved, "kernel_name": kernel_name, "value": value, "total_ms_max": total_ms_max,
            "tokens": tokens, "peaks": peaks, "roofline": roofline, "tflops": flops / avg_launch_s / 1e12,
            "launches": gdr.kernel_launches(desc) * steps, "clocks": clk.summary(), "steps": steps}


def workload_summary(name, r):
    """The object a secondary forward workload gets in the JSON line."""
    return {"value": round(r["value"], 3), "unit": "Mtokens/s", "ms_per_step": round(r["total_ms_max"] / r["steps"], 4),
            "steps": r["steps"], "config": workload_config(name, r["p"]), "algo": r["resolved"],
            "tflops_algorithmic": round(r["tflops"], 2), "roofline": r["roofline"], "gpu_launches": r["launches"],
            "clocks": r["clocks"]}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from recurrent_state_memory_b200 import gdr
    from recurrent_state_memory_b200 import inputs as I

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    gdr.lib()
    stream = torch.cuda.current_stream(dev)
    main = time_fwd(args.workload, args, dev, stream, rank, ws, args.steps)
    p, host, dv_t, o, S_T, wsp = main["p"], main["host"], main["dv_t"], main["o"], main["S_T"], main["wsp"]
    cfg = dict(I.FWD_CONFIGS[args.workload])
    cfg["seed"] = rank_seed(cfg["seed"], rank)
    to = _to_torch
    value, total_ms_max, tokens = main["value"], main["total_ms_max"], main["tokens"]
    peaks, roofline, tflops = main["peaks"], main["roofline"], main["tflops"]
    resolved, kernel_name = main["resolved"], main["kernel_name"]
    algo_bytes = p.nbytes_algorithmic

    # ---- end to end through the public API with pinned host buffers ----
    e2e = None
    if not args.no_e2e:
        pinned = {k: (None if t is None else t.pin_memory()) for k, t in host.items()}
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        S_h = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
        d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()

        hdesc = gdr.fwd_desc(p.B, p.H, p.T, p.dk, p.dv, pinned["q"].dtype, o.dtype, p.gate_mode, p.theta is not None,
                             p.scale, args.algo)
        wsh = torch.empty(gdr.host_workspace_bytes(hdesc, S0=pinned.get("S0") is not None, S_T=True),
                          dtype=torch.uint8, device=dev)

        def e2e_step():
            # the public call on host tensors: gdr_chunk_fwd_host copies each batch slice in,
            # runs it and copies it out, overlapping neighbouring slices; returns when o and
            # S_T are in host memory
            gdr.chunk_fwd(pinned["q"], pinned["k"], pinned["v"], pinned["g"], pinned["beta"], pinned.get("theta"),
                          pinned.get("S0"), gate_mode=p.gate_mode, scale=p.scale, algo=args.algo, o=o_h, S_T=S_h,
                          stream=stream, workspace=wsh)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(2, min(args.steps, 5))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), dev)
        e_tok = sum_over_ranks(float(tokens * n_e2e), dev)
        e2e = {"value": round(e_tok / (e_ms * 1e-3) / 1e6, 3), "unit": "Mtokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n_e2e}

    # ---- separate erase / write strengths (CARVE): the same workload with a write strength w ----
    def time_variant(step, v_bytes):
        """Time one variant of the forward on the same workload (CUDA events, max over ranks)."""
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        n_v = max(3, min(args.steps, 10))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_v):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        v_ms = max_over_ranks(a.elapsed_time(b), dev)
        v_tok = sum_over_ranks(float(tokens * n_v), dev)
        v_gbs = v_bytes / (a.elapsed_time(b) / n_v * 1e-3) / 1e9
        return {"value": round(v_tok / (v_ms * 1e-3) / 1e6, 3), "unit": "Mtokens/s",
                "ms_per_step": round(v_ms / n_v, 4), "steps": n_v, "kernel": kernel_name,
                "roofline": {"bound": "hbm", "achieved": round(v_gbs, 1), "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": round(v_gbs / peaks["hbm_gbs"], 4),
                             "algorithmic_bytes_per_launch": int(v_bytes)}}

    def fwd_variant(**kw):
        return lambda: gdr.chunk_fwd(dv_t["q"], dv_t["k"], dv_t["v"], dv_t["g"], dv_t["beta"], dv_t["theta"],
                                     dv_t["S0"], gate_mode=p.gate_mode, scale=p.scale, algo=args.algo, o=o,
                                     S_T=S_T, stream=stream, workspace=wsp, **kw)

    untied = l2norm = cmean = None
    if not args.no_untied:
        # ---- separate erase / write strengths (CARVE): the same workload with a write strength w ----
        w_dev = torch.from_numpy(I.make_write_strength(rank_seed(cfg["seed"], rank) + 17, (p.B, p.T, p.H))).to(dev)
        untied = time_variant(fwd_variant(w=w_dev), algo_bytes + p.B * p.T * p.H * 4)     # plus w
        # ---- fused L2 normalisation of q and k: the same workload with the prologue on ----
        l2norm = time_variant(fwd_variant(qk_l2norm=True), algo_bytes)
        # ---- chunk means of o (the content signal of CARVE's content-aware erase) ----
        nc = (p.T + p.chunk - 1) // p.chunk
        m_dev = torch.empty((p.B, nc, p.H, p.dv), dtype=torch.float32, device=dev)
        cmean = time_variant(fwd_variant(chunk_mean=m_dev), algo_bytes + m_dev.numel() * 4)   # plus the means

    # ---- decode: 256 sequences x 16 heads, fp32 state, one launch per step ----
    decode = None
    if not args.no_decode:
        dc = dict(I.DECODE_CONFIG)
        pool = 8
        dcfg = I.make_decode(N=dc["N"], H=dc["H"], dk=dc["dk"], dv=dc["dv"], steps=pool,
                             dtype=dc["dtype"], seed=rank_seed(dc["seed"], rank), s_std=dc["s_std"])
        dd = {k: to(getattr(dcfg, k)).to(dev) for k in ("q", "k", "v", "g", "beta")}
        S = to(dcfg.S).to(dev)
        od = torch.empty((dc["N"], dc["H"], dc["dv"]), dtype=torch.bfloat16, device=dev)

        def dstep(i):
            j = i % pool
            gdr.decode_step(dd["q"][j], dd["k"][j], dd["v"][j], dd["g"][j], dd["beta"][j], S,
                            gate_mode=dcfg.gate_mode, o=od, stream=stream)

        for i in range(5):
            dstep(i)
        torch.cuda.synchronize()
        n_dec = args.decode_steps
        devs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_dec)]
        for i in range(n_dec):
            devs[i][0].record(stream)
            dstep(i)
            devs[i][1].record(stream)
        torch.cuda.synchronize()
        dms = sorted(x.elapsed_time(y) for x, y in devs)
        med_ms = max_over_ranks(dms[len(dms) // 2], dev)
        nh = dc["N"] * dc["H"]
        bytes_step = nh * (2 * dc["dv"] * dc["dk"] * 4 + 3 * dc["dk"] * 2 + dc["dk"] * 4 + 4 + dc["dv"] * 2)
        bytes_all = sum_over_ranks(float(bytes_step), dev)
        gbs = bytes_all / (med_ms * 1e-3) / 1e9
        decode = {"value": round(gbs, 1), "unit": "GB/s", "us_per_step_median": round(med_ms * 1e3, 2),
                  "bytes_per_step": int(bytes_step), "steps": n_dec, "N": dc["N"], "H": dc["H"],
                  "roofline": {"bound": "hbm", "achieved": round(bytes_step / (med_ms * 1e-3) / 1e9, 1),
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": round(bytes_step / (med_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                               "traffic": stored_traffic("gdr_decode_step", "decode_n256_h16_d128"),
                               "kernel": "gdr_decode_step"}}

    # ---- backward pass (gradients of every input) on the same workload ----
    bwd = None
    if not args.no_bwd and not p.rotation and p.dk == p.dv:
        dO_dev = torch.from_numpy(I.normal(rank_seed(cfg["seed"], rank) + 31, "dO", (p.B, p.T, p.H, p.dv))
                                  .astype(np.float32)).to(dev).to(o.dtype)
        dS_dev = torch.from_numpy(I.normal(rank_seed(cfg["seed"], rank) + 32, "dS_T", (p.B, p.H, p.dv, p.dk))
                                  .astype(np.float32)).to(dev)
        bdesc = gdr.fwd_desc(p.B, p.H, p.T, p.dk, p.dv, dv_t["q"].dtype, o.dtype, p.gate_mode, False, p.scale)
        bws = torch.empty(gdr.bwd_workspace_bytes(bdesc), dtype=torch.uint8, device=dev)

        def bstep():
            return gdr.chunk_bwd(dv_t["q"], dv_t["k"], dv_t["v"], dv_t["g"], dv_t["beta"], dv_t["S0"], dO_dev, dS_dev,
                                 gate_mode=p.gate_mode, scale=p.scale, workspace=bws, stream=stream)

        bstep()
        torch.cuda.synchronize()
        n_b = max(1, min(args.steps, 3))
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_b):
            bstep()
        b_.record(stream)
        torch.cuda.synchronize()
        b_ms = max_over_ranks(a.elapsed_time(b_) / n_b, dev)
        # bytes a backward must move: q, k, v, gates, beta and dO in; dq, dk, dv, dg (fp32), dbeta out
        esz = dv_t["q"].element_size()
        b_bytes = p.B * p.T * p.H * (3 * p.dk * esz + p.dk * 4 + 4 + p.dv * o.element_size() + 4 * p.dk * 4 + 4)
        b_gbs = b_bytes / (b_ms * 1e-3) / 1e9
        b_tok_all = sum_over_ranks(float(tokens), dev)
        bwd = {"value": round(b_tok_all / (b_ms * 1e-3) / 1e6, 3), "unit": "Mtokens/s", "ms_per_step": round(b_ms, 3),
               "steps": n_b, "kernel": "gdr_chunk_bwd",
               "scope": "value over all ranks (each the same workload, the slowest rank's time); roofline per GPU",
               "train_step_mtokens_s": round(b_tok_all / ((b_ms + total_ms_max / args.steps) * 1e-3) / 1e6, 3),
               "roofline": {"bound": "hbm", "achieved": round(b_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": round(b_gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes_per_launch": int(b_bytes)}}
        del bws

    # ---- Raven's routed slot memory (a second recurrence) at the headline shape ----
    raven = None
    if not args.no_raven:
        rcfg = dict(I.RAVEN_CONFIGS["raven_b4_h16_t4096_d128"])
        rcfg["seed"] = rank_seed(rcfg["seed"], rank)
        rp = I.make_raven(name="raven_b4_h16_t4096_d128", **rcfg)
        rt = {n: to(getattr(rp, n)).to(dev) for n in ("q", "k", "v", "z", "g")}
        rdesc = gdr.raven_desc(rp.B, rp.H, rp.T, rp.d, rp.K, scale=rp.scale)
        rws = torch.empty(max(16, gdr.raven_workspace_bytes(rdesc)), dtype=torch.uint8, device=dev)

        def rstep():
            return gdr.raven_fwd(rt["q"], rt["k"], rt["v"], rt["z"], rt["g"], topk=rp.K, scale=rp.scale,
                                 workspace=rws, stream=stream)

        for _ in range(max(3, args.warmup)):
            rstep()
        torch.cuda.synchronize()
        n_r = max(1, min(args.steps, 10))
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_r):
            rstep()
        b_.record(stream)
        torch.cuda.synchronize()
        r_ms = max_over_ranks(a.elapsed_time(b_) / n_r, dev)
        r_th = rp.B * rp.T * rp.H          # token-heads (the bytes); tokens are B*T, as in the headline
        # q, k, v bf16, 64 router logits fp32, the gate fp32 in; o bf16 out; the final states
        r_bytes = r_th * (3 * rp.d * 2 + 64 * 4 + 4 + rp.d * 2) + rp.B * rp.H * 2 * 64 * rp.d * 4
        r_gbs = r_bytes / (r_ms * 1e-3) / 1e9
        r_tok_all = sum_over_ranks(float(rp.B * rp.T), dev)
        raven = {"value": round(r_tok_all / (r_ms * 1e-3) / 1e6, 3), "unit": "Mtokens/s",
                 "us_per_step": round(r_ms * 1e3, 1),
                 "steps": n_r, "kernel": "gdr_raven_fwd", "workload": "raven_b4_h16_t4096_d128 (64 slots, top-8)",
                 "scope": "value over all ranks (each the same workload, the slowest rank's time); roofline per GPU",
                 "segments": gdr.raven_segments(rdesc), "launches_per_step": 3 if gdr.raven_segments(rdesc) > 1 else 2,
                 "roofline": {"bound": "hbm", "achieved": round(r_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": round(r_gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes_per_launch": int(r_bytes)}}
        del rt, rws
        torch.cuda.empty_cache()

    # ---- the other forward workloads, each timed the same way on its own inputs ----
    workloads = None
    if not args.no_workloads:
        workloads = {}
        for name in FWD_WORKLOADS:
            if name == args.workload:
                continue
            r = time_fwd(name, args, dev, stream, rank, ws, min(args.steps, 10))
            workloads[name] = workload_summary(name, r)
            del r
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        cpu = cpu_baseline(p, args.cpu_seconds)

    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "Mtokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if resolved.startswith("tcgen05") else "f32",
        "data": "synthetic (seeded SplitMix64; q,k L2-normalised, bf16)",
        "config": workload_config(args.workload, p),
        "algo": resolved, "per_rank_batch": p.B, "parallelism": f"replicas x{ws} (independent batches)",
        "tflops_algorithmic": round(tflops, 2),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": main["launches"],
        "decode": decode,
        "backward": bwd,
        "raven": raven,
        "untied": untied,
        "qk_l2norm": l2norm,
        "chunk_mean": cmean,
        "cpu_baseline": cpu,
        "clocks": main["clocks"],
        "workloads": workloads,
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(p, seconds: float):
    """The oracle, as it stands, on a bounded sample of whole heads of the workload.  Each group
    of heads is laid out for the oracle before its clock starts, so that only the oracle's own
    run is timed (as in the reference arm)."""
    import oracle
    heads_done, tokens, el = 0, 0, 0.0
    order = [(b, h) for b in range(p.B) for h in range(p.H)]
    batch = max(1, oracle.num_threads())
    i = 0
    while i < len(order) and el < seconds:
        grp = order[i:i + batch]
        sl = [p.head_slice(b, h) for (b, h) in grp]
        # the group as one oracle call, so that its OpenMP loop spreads over the cores
        cat = lambda key: None if getattr(sl[0], key) is None else np.concatenate([s.widened(key) for s in sl], axis=0)
        arrs = [cat(key) for key in ("q", "k", "v", "g", "beta", "theta", "S0")]
        t0 = time.perf_counter()
        oracle.gdr_fwd(*arrs, gate_mode=p.gate_mode, scale=p.scale)
        el += time.perf_counter() - t0
        heads_done += len(grp)
        tokens += len(grp) * p.T
        i += batch
    # per-head token throughput scaled to the workload's unit: tokens of B*T over all H heads
    value = (tokens / p.H) / el / 1e6
    return {"value": round(value, 6), "unit": "Mtokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{heads_done} whole heads (T={p.T}) of the workload, fp64 token recurrence, "
                      f"{el:.1f} s of oracle time; tokens counted as B*T over all H heads"}


# ------------------------------------------------------- reference arm ----

def run_reference(args):
    """The fp64 CPU oracle as the reference arm, on the host cores (rank 0 only)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from recurrent_state_memory_b200 import inputs as I
    p = I.make_config(args.workload)
    per_step = max(1, oracle.num_threads())
    sl = [p.head_slice(0, h % p.H) for h in range(per_step)]
    cat = lambda key: None if getattr(sl[0], key) is None else np.concatenate([s.widened(key) for s in sl], axis=0)
    arrs = {k: cat(k) for k in ("q", "k", "v", "g", "beta", "theta", "S0")}

    def step():
        oracle.gdr_fwd(arrs["q"], arrs["k"], arrs["v"], arrs["g"], arrs["beta"], arrs["theta"], arrs["S0"],
                       gate_mode=p.gate_mode, scale=p.scale)

    for _ in range(args.warmup):
        step()
    t0 = time.time()
    for _ in range(args.steps):
        step()
    el = time.time() - t0
    value = (per_step * p.T / p.H) * args.steps / el / 1e6
    sample = f"{per_step} whole heads (T={p.T}) per step; tokens counted as B*T over all H heads"
    line = {"metric": METRIC, "value": round(value, 6), "unit": "Mtokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SplitMix64)", "impl": "reference",
            "config": workload_config(args.workload, p),
            "cpu_baseline": {"value": round(value, 6), "unit": "Mtokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "Mtokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--algo", choices=["auto", "simt", "tcgen05", "tcgen05_split", "tcgen05_waves",
                                       "tcgen05_segments", "tcgen05_chains"], default="auto")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other forward workloads")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward pass")
    ap.add_argument("--no-raven", action="store_true", help="skip the Raven slot-memory forward")
    ap.add_argument("--no-untied", action="store_true", help="skip the separate-write-strength, "
                    "fused-L2-norm and chunk-mean measurements")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
