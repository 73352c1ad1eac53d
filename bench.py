"""Throughput of the spatial-spectral coupling (fwd + bwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload dense_60k|geo_60k|...] [--need-dv]

One step = the whole hot path over one synthetic shape pair resident in HBM:
the dense coupling forward (O, lse) and backward (dQ, dK) at n = 60,000,
d = 128, k = 196 (the headline), followed in the same line by the
Geo-FlashAttention step at the same size (patch scores + top-R selection,
forward, backward).  Throughput is effective TFLOP/s counted the
FlashAttention way (executed flops including the S recompute of the
backward): per (i, j) pair 2(d + k) forward and 2(2d + k) + 2d backward.

Under torchrun every rank runs its own shape pair (independent problems, weak
scaling, no collective on the data path); the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded row sample of the
same workload and extrapolates to the full size.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "coupling fwd+bwd ms & TFLOP/s at n=60k (dense, geo); % of bf16 tensor peak"


def pair_flops(d, k, need_dv):
    fwd = 2 * (d + k)
    bwd = 2 * (2 * d + k) + 2 * d + (2 * k if need_dv else 0)
    return fwd, bwd


# DRAM traffic of tc_bwd_dqk_kernel on the dense 60k workload, from one ncu
# capture of this bench's own launch at n = 60k (dram__bytes_read.sum +
# dram__bytes_write.sum, a 1-pass metric set).  It stands only while the
# kernel's source text is the one that was captured.
DQK_TRAFFIC = {"kernel_sha256_16": "d3a006df033c44d3", "n": 60000, "d": 128, "k": 196,
               "read_bytes": 179.66e6, "write_bytes": 70.50e6}


def dqk_kernel_hash():
    import hashlib
    path = os.path.join(ROOT, "spatial_spectral_attention_b200", "csrc", "coupling_tc.cu")
    try:
        s = open(path).read()
        i = s.index("template <int NCG, int QCH, int VF, int VR, bool kNoDK, bool kDqFlush>\n"
                    "__global__ void __launch_bounds__(128 * (2 + NCG), 1)\n    tc_bwd_dqk_kernel(")
        j = s.index("\n}\n", i) + 3
    except (OSError, ValueError):
        return None
    return hashlib.sha256(s[i:j].encode()).hexdigest()[:16]


def dqk_traffic(n, d, k):
    t = DQK_TRAFFIC
    if (n, d, k) != (t["n"], t["d"], t["k"]) or dqk_kernel_hash() != t["kernel_sha256_16"]:
        return None
    return t["read_bytes"] + t["write_bytes"]


DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16, nominal (no sparsity)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(tflops=j["bf16_tflops"], tflops_sustained=j["bf16_tflops_sustained"],
                    hbm=j["hbm_gbs"], source="measured")
    return dict(tflops=1590.0, tflops_sustained=1400.0, hbm=6650.0, source="fallback")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, polled through NVML every
    10 ms on a background thread (read-only queries)."""

    REASONS = {  # NVML clocks-event reason bits
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "sw_power_cap": 0x4,
    }

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.stop = threading.Event()
        self.window = (0.0, float("inf"))

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.nvml = None
        return self

    def _run(self):
        n = self.nvml
        while not self.stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                try:
                    r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = n.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), sm, r))
            except Exception:
                pass
            time.sleep(0.01)

    def mark(self, t0, t1):
        """Restrict the summary to samples taken between wall times t0 and t1."""
        self.window = (t0, t1)

    def __exit__(self, *a):
        self.stop.set()
        if self.nvml is not None:
            self.t.join(timeout=1)

    def summary(self):
        w0, w1 = self.window
        sel = [s for s in self.samples if w0 <= s[0] <= w1]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = sorted({nm for _, _, r in sel for nm, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": float(np.median([s[1] for s in sel])), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(sel)}


def dist_setup(ngpus):
    from spatial_spectral_attention_b200 import dist
    return dist.init("nccl")


def max_over_ranks(x, ws):
    from spatial_spectral_attention_b200 import dist
    return dist.max_over_ranks(x, ws, device="cuda")


def barrier(ws):
    from spatial_spectral_attention_b200 import dist
    dist.barrier(ws)


GEO_SWEEP_N = (20000, 40000, 60000, 100000, 160000)


def step_graph(step, torch, dev):
    """The launches of one step captured once into a CUDA graph (after the
    step has run eagerly, so every lazily made resource exists); a replay runs
    every launch of the step again on the same device-resident inputs."""
    gr = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(dev)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(gr, stream=cs):
        step()
    torch.cuda.synchronize()
    return gr


def timed_steps(run, flush, stream, torch, reps):
    """Mean ms of `reps` runs, each bracketed by CUDA events on `stream`, with
    L2 flushed (untimed) before each."""
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for e in evs:
        flush.zero_()
        e[0].record(stream)
        run()
        e[1].record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def run_geo_sweep(api, synth, torch, dev, need_dv, fpp, bpp):
    """Geo step (scores/top-R + fwd + bwd) against n with P = n/125 and R = 8:
    ms per step and peak device memory per size (160k is the warped,
    non-isometric pair).  Each size: patch tables once, 2 warm-up and 3 timed
    steps launched one by one, then 3 timed replays of the step as one CUDA
    graph; L2 flushed before each timed step."""
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    bf = lambda a: torch.tensor(a).to(torch.bfloat16).to(dev)
    out = []
    for n in GEO_SWEEP_N:
        gp = synth.make_workload("geo_160k_warped" if n == 160000 else "geo_60k", n=n)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev) - flush.numel()
        Q, K, V, dO = bf(gp.F_N), bf(gp.F_M), bf(gp.Phi_M), torch.tensor(gp.dO).to(dev)
        _, _, offN, memN = api.ssc_fps_patches(torch.tensor(gp.pts_N).to(dev), gp.P)
        _, _, offM, memM = api.ssc_fps_patches(torch.tensor(gp.pts_M).to(dev), gp.P)
        gws = torch.empty(api.lib().ssc_geo_coupling_workspace_size(n, n, gp.d, gp.k, gp.P, gp.P, gp.R, 0),
                          dtype=torch.uint8, device=dev)

        def step():
            topk = api.ssc_patch_scores_topk(Q, K, offN, memN, offM, memM, gp.R)
            O, lse = api.ssc_geo_coupling_fwd(Q, K, V, gp.scale, offN, memN, offM, memM, topk,
                                              workspace=gws)
            api.ssc_geo_coupling_bwd(Q, K, V, O, lse, dO, gp.scale, offN, memN, offM, memM, topk,
                                     need_dV=need_dv, workspace=gws, reuse_forward=True)

        for _ in range(2):
            step()
        eager_ms = timed_steps(step, flush, stream, torch, 3)
        peak = (torch.cuda.max_memory_allocated(dev) - flush.numel() - base) / 2**30
        gr = step_graph(step, torch, dev)
        ms = timed_steps(gr.replay, flush, stream, torch, 3)
        del gr
        U = float(np.mean(np.diff(offM.cpu().numpy()))) * gp.R
        out.append({"n": n, "P": gp.P, "ms_per_step": round(ms, 4),
                    "eager_ms_per_step": round(eager_ms, 4),
                    "tflops": round(float(n) * U * (fpp + bpp) / (ms * 1e-3) / 1e12, 2),
                    "peak_gib": round(peak, 3)})
        del Q, K, V, dO, offN, memN, offM, memM, gws
    return out


def run_fps_timing(api, synth, torch, dev, reps=5):
    """FPS + Voronoi + patch tables per shape on device-resident points, warmed:
    the FPS kernel's own launch time (CUDA events around each launch, on its
    stream) per call and per round, and the whole call.  60k (P 480) and the
    160k warped pair's target shape (P 1280)."""
    stream = torch.cuda.current_stream()
    out = []
    for name in ("geo_60k", "geo_160k_warped"):
        gp = synth.make_workload(name)
        pts = torch.tensor(gp.pts_N).to(dev)
        for _ in range(2):
            api.ssc_fps_patches(pts, gp.P)
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        api.ssc_profile_enable(True)
        for e in evs:
            e[0].record(stream)
            api.ssc_fps_patches(pts, gp.P)
            e[1].record(stream)
        api.ssc_profile_enable(False)
        torch.cuda.synchronize()
        kms, kn = api.ssc_profile_read(api.PROF_FPS)
        kms /= max(kn, 1)
        call_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
        out.append({"workload": name, "n": gp.n, "P": gp.P, "fps_kernel_ms": round(kms, 4),
                    "us_per_round": round(kms * 1e3 / gp.P, 3), "call_ms": round(call_ms, 4),
                    "calls": reps})
        del pts
    return out


def geo_tables_flops(offN, offM, topk, d, k, need_dv):
    """Support (algorithmic) and tile-padded (executed) (i, j) pair counts of one
    Geo step from the patch tables, and the flops per pair."""
    sN = np.diff(offN.cpu().numpy()).astype(np.float64)
    sM = np.diff(offM.cpu().numpy()).astype(np.float64)
    t = topk.cpu().numpy()
    U = sM[t].sum(axis=1)
    pairs = float((sN * U).sum())
    tilesN = np.ceil(sN / 128.0) * 128.0
    Upad = (np.ceil(sM / 128.0) * 128.0)[t].sum(axis=1)
    pairs_exec = float((tilesN * Upad).sum())
    fpp, bpp = pair_flops(d, k, need_dv)
    return pairs, pairs_exec, fpp, bpp


def _timed(torch, fn, flush, reps=5, warm=2):
    """Mean ms of fn() over reps calls, L2 flushed before each, CUDA events on
    the current stream."""
    stream = torch.cuda.current_stream()
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for e in evs:
        flush.zero_()
        e[0].record(stream)
        fn()
        e[1].record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def _relfro(a, b):
    return float((a.double() - b.double()).norm() / b.double().norm())


def run_extras(api, synth, torch, dev, pk):
    """The variants beside the headline step, each on its own resident inputs
    (L2 flushed before every timed call):
      linear   ELU linear-attention coupling fwd + bwd at 60k and 160k, kernel
               times and HBM throughput, and the accuracy gap to the exact
               dense coupling next to Geo's (relative Frobenius of O);
      deterministic  the run-to-run exact dense backward at 60k;
      e4m3     the dense forward with Q K^T on fp8 tensor cores at 60k;
      batched  8 pairs of 10k dense fwd + bwd and 8 pairs of 20k Geo in one call;
      mesh_fps geodesic FPS on the sphere meshes of the 60k and 160k shapes."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    bf = lambda a: torch.tensor(a).to(torch.bfloat16).to(dev)
    out = {}
    # ---- linear coupling and the accuracy gaps
    lin = []
    for name in ("geo_60k", "geo_160k_warped"):
        g = synth.make_workload(name)
        Q, K, V, dO = bf(g.F_N), bf(g.F_M), bf(g.Phi_M), torch.tensor(g.dO).to(dev)
        n, d, k = g.n, g.d, g.k
        ws = torch.empty(api.lib().ssc_linear_coupling_workspace_size(n, n, d, k), dtype=torch.uint8,
                         device=dev)
        res = {}
        fwd_ms = _timed(torch, lambda: api.ssc_linear_coupling_fwd(Q, K, V, workspace=ws), flush)
        O, den = api.ssc_linear_coupling_fwd(Q, K, V, workspace=ws)
        bwd_ms = _timed(torch, lambda: api.ssc_linear_coupling_bwd(Q, K, V, O, den, dO, workspace=ws),
                        flush)
        api.ssc_profile_enable(True)
        for _ in range(3):
            flush.zero_()
            o2, d2 = api.ssc_linear_coupling_fwd(Q, K, V, workspace=ws)
            api.ssc_linear_coupling_bwd(Q, K, V, o2, d2, dO, workspace=ws)
        api.ssc_profile_enable(False)
        torch.cuda.synchronize()
        red = api.ssc_profile_read(api.PROF_LIN_REDUCE)
        rows = api.ssc_profile_read(api.PROF_LIN_ROWS)
        kv = (k + 1 + 15) // 16 * 16
        # algorithmic bytes of one fwd + bwd: K,V read twice (both reductions
        # of K), Q read twice, Y written and read twice, O written, dO and O
        # read once, dQ and dK written
        step_bytes = (2.0 * n * (d + k) * 2 + 2.0 * n * d * 2 + 3.0 * n * kv * 2 + 4.0 * n * k
                      + 8.0 * n * k + 2 * 4.0 * n * d)
        # exact dense and Geo forwards on the same pair, for the accuracy gap
        Od, _ = api.ssc_dense_coupling_fwd(Q, K, V, g.scale)
        _, _, offN, memN = api.ssc_fps_patches(torch.tensor(g.pts_N).to(dev), g.P)
        _, _, offM, memM = api.ssc_fps_patches(torch.tensor(g.pts_M).to(dev), g.P)
        topk = api.ssc_patch_scores_topk(Q, K, offN, memN, offM, memM, g.R)
        Og, _ = api.ssc_geo_coupling_fwd(Q, K, V, g.scale, offN, memN, offM, memM, topk)
        torch.cuda.synchronize()
        res.update({"workload": name, "n": n, "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
                    "step_ms": round(fwd_ms + bwd_ms, 4),
                    "step_gbs": round(step_bytes / ((fwd_ms + bwd_ms) * 1e-3) / 1e9, 1),
                    "hbm_frac": round(step_bytes / ((fwd_ms + bwd_ms) * 1e-3) / 1e9 / pk["hbm"], 4),
                    "reduce_kernel_ms": round(red[0] / max(red[1], 1), 4),
                    "rows_kernel_ms": round(rows[0] / max(rows[1], 1), 4),
                    "O_relfro_vs_exact_dense": {"linear": round(_relfro(O, Od), 4),
                                                "geo": round(_relfro(Og, Od), 4)}})
        lin.append(res)
        del Q, K, V, dO, ws, O, den, Od, Og
    out["linear"] = {"sizes": lin, "note": "phi = elu + 1; step bytes = one pass over every "
                     "operand the two reductions and three row products read or write; the "
                     "accuracy gap is ||O - O_dense||_F / ||O_dense||_F on the same pair"}
    # ---- deterministic backward, e4m3 forward (60k dense)
    g = synth.make_workload("dense_60k")
    Q, K, V, dO = bf(g.F_N), bf(g.F_M), bf(g.Phi_M), torch.tensor(g.dO).to(dev)
    wsd = torch.empty(api.lib().ssc_dense_coupling_workspace_size(g.n, g.n, g.d, g.k, 0),
                      dtype=torch.uint8, device=dev)
    O, lse = api.ssc_dense_coupling_fwd(Q, K, V, g.scale, workspace=wsd)
    fpp, bpp = pair_flops(g.d, g.k, False)
    det = {}
    for dv in (False, True):
        ms = _timed(torch, lambda: api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, g.scale, need_dV=dv,
                                                              workspace=wsd, deterministic=True),
                    flush, reps=3)
        det["bwd_dV_ms" if dv else "bwd_ms"] = round(ms, 4)
    a = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, g.scale, workspace=wsd, deterministic=True)
    b = api.ssc_dense_coupling_bwd(Q, K, V, O, lse, dO, g.scale, workspace=wsd, deterministic=True)
    torch.cuda.synchronize()
    det["bit_identical_repeat"] = bool(all(torch.equal(x, y) for x, y in zip(a[:2], b[:2])))
    det["tflops_executed"] = round(float(g.n) * g.n * bpp / (det["bwd_ms"] * 1e-3) / 1e12, 2)
    det["note"] = ("dQ, key-stationary dK and (with dV) dV passes, no more CTAs than output tiles; "
                   "tflops on the default backward's executed-flop count")
    out["deterministic_backward"] = det
    ms8 = _timed(torch, lambda: api.ssc_dense_coupling_fwd_e4m3(Q, K, V, g.scale), flush, reps=3)
    O8, _ = api.ssc_dense_coupling_fwd_e4m3(Q, K, V, g.scale)
    torch.cuda.synchronize()
    out["e4m3_forward"] = {"fwd_ms": round(ms8, 4),
                           "tflops": round(float(g.n) * g.n * fpp / (ms8 * 1e-3) / 1e12, 2),
                           "O_relfro_vs_bf16_forward": round(_relfro(O8, O), 5),
                           "note": "single-CTA forward with S on kind::f8f6f4 (e4m3, per-tensor "
                                   "scales); P V bf16"}
    del Q, K, V, dO, wsd, O, lse, a, b, O8
    # ---- batches of pairs in one call
    B = 8
    g = synth.make_workload("dense_10k")
    Qb = torch.stack([bf(g.F_N)] * B)
    Kb = torch.stack([bf(g.F_M)] * B)
    Vb = torch.stack([bf(g.Phi_M)] * B)
    dOb = torch.stack([torch.tensor(g.dO).to(dev)] * B)
    ws = torch.empty(api.lib().ssc_dense_coupling_batched_workspace_size(B, g.n, g.n, g.d, g.k, 0),
                     dtype=torch.uint8, device=dev)

    def bstep():
        Ob, lb = api.ssc_dense_coupling_fwd_batched(Qb, Kb, Vb, g.scale, workspace=ws)
        api.ssc_dense_coupling_bwd_batched(Qb, Kb, Vb, Ob, lb, dOb, g.scale, workspace=ws)

    ms = _timed(torch, bstep, flush, reps=3)
    fpp, bpp = pair_flops(g.d, g.k, False)
    out["batched_dense"] = {"pairs": B, "n": g.n, "step_ms": round(ms, 4),
                            "tflops": round(B * float(g.n) * g.n * (fpp + bpp) / (ms * 1e-3) / 1e12, 2)}
    del Qb, Kb, Vb, dOb, ws
    # ---- geodesic FPS on meshes
    mesh = []
    for name in ("geo_60k", "geo_160k_warped"):
        g = synth.make_workload(name)
        off, adj, w = synth.sphere_mesh(g.pts_N)
        t = (torch.tensor(off).to(dev), torch.tensor(adj).to(dev), torch.tensor(w).to(dev))
        api.ssc_fps_patches_mesh(*t, g.P)
        torch.cuda.synchronize()
        api.ssc_profile_enable(True)
        for _ in range(2):
            api.ssc_fps_patches_mesh(*t, g.P)
        api.ssc_profile_enable(False)
        torch.cuda.synchronize()
        kms, cnt = api.ssc_profile_read(api.PROF_FPS)
        kms /= max(cnt, 1)
        mesh.append({"workload": name, "n": g.n, "edges": int(off[-1]) // 2, "P": g.P,
                     "fps_kernel_ms": round(kms, 3), "us_per_round": round(kms * 1e3 / g.P, 2)})
    out["mesh_fps"] = mesh
    return out


# ---------------------------------------------------------------- our arm
def run_ours(args, ws, rank, local):
    import torch
    from spatial_spectral_attention_b200 import api, synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pair = synth.make_workload(args.workload, n=args.n)
    gpair = synth.make_workload("geo_60k", n=args.n) if args.with_geo else None
    bf = lambda a: torch.tensor(a).to(torch.bfloat16)
    host = dict(Q=bf(pair.F_N).pin_memory(), K=bf(pair.F_M).pin_memory(),
                V=bf(pair.Phi_M).pin_memory(), dO=torch.tensor(pair.dO).pin_memory())
    Q, K, V, dO = (host[x].to(dev) for x in ("Q", "K", "V", "dO"))
    n, d, k = pair.n, pair.d, pair.k
    scale = pair.scale
    ws_bytes = api.lib().ssc_dense_coupling_workspace_size(n, n, d, k, 0)
    wsb = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()
    fpp, bpp = pair_flops(d, k, args.need_dv)
    flops_step = float(n) * n * (fpp + bpp)

    def dense_step(Qd, Kd, Vd, dOd, ev=None):
        if ev:
            ev[0].record(stream)
        O, lse = api.ssc_dense_coupling_fwd(Qd, Kd, Vd, scale, workspace=wsb)
        if ev:
            ev[1].record(stream)
        g = api.ssc_dense_coupling_bwd(Qd, Kd, Vd, O, lse, dOd, scale, need_dV=args.need_dv,
                                       workspace=wsb)
        if ev:
            ev[2].record(stream)
        return O, lse, g

    # geo inputs and tables (tables per shape, computed once: they depend on geometry only)
    geo = None
    if gpair is not None:
        gQ, gK, gV = bf(gpair.F_N).to(dev), bf(gpair.F_M).to(dev), bf(gpair.Phi_M).to(dev)
        gdO = torch.tensor(gpair.dO).to(dev)
        _, _, offN, memN = api.ssc_fps_patches(torch.tensor(gpair.pts_N).to(dev), gpair.P)
        _, _, offM, memM = api.ssc_fps_patches(torch.tensor(gpair.pts_M).to(dev), gpair.P)
        gws = torch.empty(api.lib().ssc_geo_coupling_workspace_size(
            gpair.n, gpair.n, gpair.d, gpair.k, gpair.P, gpair.P, gpair.R, 0),
            dtype=torch.uint8, device=dev)
        geo = dict(Q=gQ, K=gK, V=gV, dO=gdO, offN=offN, memN=memN, offM=offM, memM=memM, ws=gws)

    def geo_step():
        g = geo
        topk = api.ssc_patch_scores_topk(g["Q"], g["K"], g["offN"], g["memN"], g["offM"],
                                         g["memM"], gpair.R)
        O, lse = api.ssc_geo_coupling_fwd(g["Q"], g["K"], g["V"], gpair.scale, g["offN"],
                                          g["memN"], g["offM"], g["memM"], topk, workspace=g["ws"])
        api.ssc_geo_coupling_bwd(g["Q"], g["K"], g["V"], O, lse, g["dO"], gpair.scale, g["offN"],
                                 g["memN"], g["offM"], g["memM"], topk, need_dV=args.need_dv,
                                 workspace=g["ws"], reuse_forward=True)
        return topk

    # ---- the Geo step on its own, before any dense step (after the dense work
    # the clocks sit lower under the power cap for a while): K steps launched one
    # by one through the API and K replays of the same step captured as one
    # CUDA graph, alternating, L2 flushed before each; clocks sampled meanwhile
    geo_alone = None
    if geo:
        for _ in range(args.warmup):
            geo_step()
        gr = step_graph(geo_step, torch, dev)
        for _ in range(args.warmup):
            geo_step()
            gr.replay()
        torch.cuda.synchronize()
        reps = args.steps
        gclk = ClockSampler(local).__enter__()
        time.sleep(0.05)
        pairs_ev = []
        g0 = time.time()
        for _ in range(reps):
            for fn in (geo_step, gr.replay):
                e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                flush.zero_()
                e[0].record(stream)
                fn()
                e[1].record(stream)
                pairs_ev.append(e)
        torch.cuda.synchronize()
        g1 = time.time()
        gclk.mark(g0, g1)
        gclk.__exit__()
        tt = [a.elapsed_time(b) for a, b in pairs_ev]
        geo_alone = {"eager": max_over_ranks(float(np.mean(tt[0::2])), ws),
                     "graph": max_over_ranks(float(np.mean(tt[1::2])), ws),
                     "steps": reps, "clocks": gclk.summary()}
        del gr
        barrier(ws)

    clk = ClockSampler(local).__enter__()
    for _ in range(args.warmup):
        dense_step(Q, K, V, dO)
        if geo:
            geo_step()
    torch.cuda.synchronize()
    barrier(ws)

    # ---- timed region: device-resident inputs, L2 flushed between steps (untimed)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    launches0 = api.ssc_kernel_launches()
    torch.cuda.reset_peak_memory_stats(dev)
    mem0 = torch.cuda.memory_allocated(dev)
    torch.cuda.synchronize()
    w0 = time.time()
    # launch durations of the dense step's kernels (CUDA events the library
    # records on the launching stream; paused around the Geo step)
    api.ssc_profile_enable(True)
    for s in range(args.steps):
        flush.zero_()
        dense_step(Q, K, V, dO, evs[s])
        if geo:
            api.ssc_profile_enable(False)
            flush.zero_()
            gev[s][0].record(stream)
            geo_step()
            gev[s][1].record(stream)
            api.ssc_profile_enable(True, clear=False)
    api.ssc_profile_enable(False)
    torch.cuda.synchronize()
    w1 = time.time()
    kbwd_ms, kbwd_n = api.ssc_profile_read(api.PROF_BWD_DQK)
    kfwd_ms, kfwd_n = api.ssc_profile_read(api.PROF_DENSE_FWD)
    clk.mark(w0, w1)
    clk.__exit__()
    launches = api.ssc_kernel_launches() - launches0
    peak_gib = (torch.cuda.max_memory_allocated(dev) - mem0 + ws_bytes) / 2**30
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    step_ms = [a + b for a, b in zip(fwd_ms, bwd_ms)]
    dense_ms = max_over_ranks(float(np.mean(step_ms)), ws)
    geo_ms = max_over_ranks(float(np.mean([e[0].elapsed_time(e[1]) for e in gev])), ws) if geo else None
    barrier(ws)

    # ---- end to end through the public API with host buffers (pinned).  Every step
    # copies its inputs up and its results down inside the timed region; the copies
    # run on two copy streams and overlap the compute: a step's Q, K, V go up into
    # one of two device buffer sets while the previous step computes, its dO goes
    # up during its forward, O and lse come down during its backward and dQ, dK
    # after it.  The time runs from the first upload to the last download.
    out_host = dict(O=torch.empty((n, k), dtype=torch.float32).pin_memory(),
                    lse=torch.empty(n, dtype=torch.float32).pin_memory(),
                    dQ=torch.empty((n, d), dtype=torch.float32).pin_memory(),
                    dK=torch.empty((n, d), dtype=torch.float32).pin_memory())
    e2e_steps = max(3, min(args.steps, 8)) if args.e2e else 0
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nbuf = 2
    dev_in = [{x: torch.empty_like(host[x], device=dev) for x in host} for _ in range(nbuf)]
    ev = lambda: torch.cuda.Event(enable_timing=True)
    e0, e1 = ev(), ev()
    ev_qkv, ev_do = [ev() for _ in range(nbuf)], [ev() for _ in range(nbuf)]
    ev_done = [ev() for _ in range(nbuf)]
    parts = [[ev() for _ in range(3)] for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    barrier(ws)
    e0.record(up)
    for i in range(e2e_steps):
        bi = i % nbuf
        buf = dev_in[bi]
        with torch.cuda.stream(up):
            if i >= nbuf:
                up.wait_event(ev_done[bi])  # step i - 2 is done with these buffers
            for x in ("Q", "K", "V"):
                buf[x].copy_(host[x], non_blocking=True)
            ev_qkv[bi].record(up)
            buf["dO"].copy_(host["dO"], non_blocking=True)
            ev_do[bi].record(up)
        stream.wait_event(ev_qkv[bi])
        parts[i][0].record(stream)
        O, lse = api.ssc_dense_coupling_fwd(buf["Q"], buf["K"], buf["V"], scale, workspace=wsb)
        parts[i][1].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(parts[i][1])
            O.record_stream(down)
            lse.record_stream(down)
            out_host["O"].copy_(O, non_blocking=True)
            out_host["lse"].copy_(lse, non_blocking=True)
        stream.wait_event(ev_do[bi])
        dQ, dK, _ = api.ssc_dense_coupling_bwd(buf["Q"], buf["K"], buf["V"], O, lse, buf["dO"],
                                               scale, need_dV=args.need_dv, workspace=wsb)
        parts[i][2].record(stream)
        ev_done[bi].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(parts[i][2])
            dQ.record_stream(down)
            dK.record_stream(down)
            out_host["dQ"].copy_(dQ, non_blocking=True)
            out_host["dK"].copy_(dK, non_blocking=True)
    e1.record(down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / max(e2e_steps, 1), ws)
    e2e_compute = float(np.mean([p[0].elapsed_time(p[2]) for p in parts])) if parts else 0.0
    h2d = sum(host[x].numel() * host[x].element_size() for x in ("Q", "K", "V", "dO"))
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())

    # ---- the backward with dV as well (the dV pass after the dQ/dK kernel),
    # timed after the main region on the same resident inputs, L2 flushed
    with_dv = None
    if not args.need_dv:
        _, bpp_dv = pair_flops(d, k, True)
        O1, lse1 = api.ssc_dense_coupling_fwd(Q, K, V, scale, workspace=wsb)
        dv_steps = max(2, min(args.steps, 5))
        dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(dv_steps)]
        for s in range(dv_steps):
            flush.zero_()
            dev_ev[s][0].record(stream)
            api.ssc_dense_coupling_bwd(Q, K, V, O1, lse1, dO, scale, need_dV=True, workspace=wsb)
            dev_ev[s][1].record(stream)
        torch.cuda.synchronize()
        bwd_dv_ms = max_over_ranks(float(np.mean([e[0].elapsed_time(e[1]) for e in dev_ev])), ws)
        step_dv_ms = float(np.mean(fwd_ms)) + bwd_dv_ms
        with_dv = {"bwd_ms": round(bwd_dv_ms, 4), "step_ms": round(step_dv_ms, 4),
                   "tflops": round(float(n) * n * (fpp + bpp_dv) / (step_dv_ms * 1e-3) / 1e12, 2),
                   "bwd_tflops": round(float(n) * n * bpp_dv / (bwd_dv_ms * 1e-3) / 1e12, 2),
                   "flops_per_step": float(n) * n * (fpp + bpp_dv), "steps": dv_steps,
                   "note": "need_dV = 1: dQ/dK kernel + dV pass; step = forward (main region) "
                           "+ this backward"}
        barrier(ws)

    # ---- per-kernel launch times of the Geo step (library events on the
    # launching stream), L2 flushed before each step
    geo_kern = None
    if geo:
        gsteps = max(3, min(args.steps, 5))
        torch.cuda.synchronize()
        api.ssc_profile_enable(True)
        for _ in range(gsteps):
            flush.zero_()
            topk_last = geo_step()
        api.ssc_profile_enable(False)
        torch.cuda.synchronize()
        geo_kern = {nm: api.ssc_profile_read(kid) for nm, kid in (
            ("fwd", api.PROF_FWD), ("bwd_dqk", api.PROF_BWD_DQK), ("bwd_dv", api.PROF_BWD_DV),
            ("pool", api.PROF_POOL), ("scores", api.PROF_SCORES), ("topk", api.PROF_TOPK),
            ("gather", api.PROF_GATHER))}
        geo_kern = {nm: (ms / gsteps, n // gsteps) for nm, (ms, n) in geo_kern.items()}
        geo_kern["_topk"] = topk_last
    fps_timing = run_fps_timing(api, synth, torch, dev) if (geo and rank == 0) else None

    pk = peaks()
    tflops = ws * flops_step / (dense_ms * 1e-3) / 1e12
    # dominant kernel: the dQ/dK backward kernel (2/3 of the flops), its average
    # launch duration from the events around each launch; flops per launch =
    # executed flops per (i, j) pair x the n^2 pairs one launch processes
    bwd_flops = float(n) * n * bpp
    bwd_mean = float(np.mean(bwd_ms))
    kbwd_mean = kbwd_ms / max(kbwd_n, 1)
    achieved = bwd_flops / (kbwd_mean * 1e-3) / 1e12 if kbwd_n else 0.0
    achieved_model = float(n) * n * (2 * (2 * d + k) + (2 * k if args.need_dv else 0)) / (kbwd_mean * 1e-3) / 1e12 if kbwd_n else 0.0
    res = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dense_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded sphere workload: random-Fourier-feature descriptors, "
                "spherical-harmonic eigenbasis)",
        "config": {"workload": pair.name, "n": n, "d": d, "k": k, "need_dV": args.need_dv,
                   "flops_per_step": flops_step, "flop_convention":
                   "executed, fwd 2(d+k) + bwd 2(2d+k)+2d per (i,j) pair",
                   "l2": "flushed between timed steps (256 MiB write, untimed)",
                   "parallelism": f"replicas x{ws} (independent shape pairs)"},
        "dense": {"fwd_ms": round(float(np.mean(fwd_ms)), 4),
                  "bwd_ms": round(float(np.mean(bwd_ms)), 4),
                  "fwd_tflops": round(float(n) * n * fpp / (np.mean(fwd_ms) * 1e-3) / 1e12, 2),
                  "bwd_tflops": round(bwd_flops / (bwd_mean * 1e-3) / 1e12, 2),
                  "fwd_kernel_ms": round(kfwd_ms / max(kfwd_n, 1), 4),
                  "bwd_kernel_ms": round(kbwd_mean, 4),
                  "frac_of_peak": round(tflops / ws / pk["tflops"], 4),
                  "frac_of_datasheet_peak": round(tflops / ws / DATASHEET_BF16_TFLOPS, 4),
                  "peak_gib": round(peak_gib, 3),
                  "with_dV": with_dv},
        "roofline": {"bound": "tensor", "kernel": "tc_bwd_dqk_kernel (dense backward, dQ and dK)",
                     "achieved": round(achieved, 2), "peak": pk["tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / pk["tflops"], 4), "peak_source": pk["source"] +
                     " burst bf16 (MEASURED_PEAKS.json bf16_tflops)",
                     "frac_of_datasheet_peak": round(achieved / DATASHEET_BF16_TFLOPS, 4),
                     "frac_model_flops": round(achieved_model / pk["tflops"], 4),
                     "flops_per_launch": bwd_flops, "flop_convention": "executed (S recompute included)",
                     "achieved_model_flops": round(achieved_model, 2),
                     "launches_timed": kbwd_n, "traffic": dqk_traffic(n, d, k),
                     "traffic_unit": "bytes per launch (DRAM read + write, ncu)"},
        "e2e": ({"value": round(ws * flops_step / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                 "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d),
                 "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                 "compute_ms_per_step": round(e2e_compute, 4),
                 "overlap": "uploads and downloads on two copy streams overlap the compute; "
                            "two input buffer sets; time from the first upload to the last "
                            "download"} if e2e_steps > 0 else None),
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if args.extras and rank == 0:
        res["variants"] = run_extras(api, synth, torch, dev, pk)
    if args.geo_sweep and rank == 0:
        res["geo_sweep"] = {"note": "Geo step vs n, P = n/125, R = 8 (160k: warped pair); "
                                    "peak_gib = peak device memory of the size's inputs, "
                                    "tables, workspace and outputs",
                            "sizes": run_geo_sweep(api, synth, torch, dev, args.need_dv, fpp, bpp)}
    if geo:
        pairs, pairs_exec, gfpp, gbpp = geo_tables_flops(geo["offN"], geo["offM"],
                                                         geo_kern["_topk"], gpair.d, gpair.k,
                                                         args.need_dv)
        gflops = pairs * (gfpp + gbpp)
        gd, gk, gn = gpair.d, gpair.k, gpair.n
        kp = (gk + 15) // 16 * 16
        kp = kp + 16 if kp % 64 == 48 else kp

        def kern(nm, flops=None, nbytes=None, bound="tensor"):
            ms, cnt = geo_kern[nm]
            if cnt == 0:
                return None
            r = {"ms": round(ms, 4), "launches_per_step": cnt}
            if flops is not None:
                a = flops / (ms * 1e-3) / 1e12
                r.update({"bound": "tensor", "achieved": round(a, 2), "peak": pk["tflops"],
                          "unit": "TFLOP/s", "frac": round(a / pk["tflops"], 4),
                          "flops": flops})
            if nbytes is not None:
                g = nbytes / (ms * 1e-3) / 1e9
                r.update({"algorithmic_bytes": nbytes, "achieved_gbs": round(g, 1),
                          "hbm_frac": round(g / pk["hbm"], 4)})
                if flops is None:
                    r.update({"bound": bound, "peak": pk["hbm"], "unit": "GB/s"})
            return r

        geo_roof = {
            "fwd": kern("fwd", pairs * gfpp, 2.0 * gn * (gd + gd + kp) + 4.0 * gn * (gk + 1)),
            "bwd_dqk": kern("bwd_dqk", pairs * (gbpp - (2 * gk if args.need_dv else 0)),
                            2.0 * gn * (gd + gd + kp + kp) + 4.0 * gn * (2 * gd + 2)),
            "pool": kern("pool", None, 2.0 * (2.0 * gn * gd) + 2 * 4.0 * gn, "hbm"),
            "scores": kern("scores", None, 8.0 * gpair.P * gpair.P + 2 * 8.0 * gpair.P * gd, "hbm"),
            "topk": kern("topk", None, 8.0 * gpair.P * gpair.P, "hbm"),
            "gather": kern("gather", None, 2 * 2.0 * gn * (gd + gd + kp), "hbm"),
            "flop_convention": "support pairs sum_p |p| |U(p)| x per-pair flops (no tile padding)",
            "bytes_convention": "one read of each input row and one write of each output row "
                                "per launch (L2 re-reads not counted)",
            "peak_source": pk["source"] + " (MEASURED_PEAKS.json: bf16_tflops, hbm_gbs)",
        }
        geo_graph_ms = geo_alone["graph"]
        res["geo"] = {"workload": gpair.name, "ms_per_step": round(geo_graph_ms, 4),
                      "eager_ms_per_step": round(geo_alone["eager"], 4),
                      "eager_ms_per_step_beside_dense": round(geo_ms, 4),
                      "steps": geo_alone["steps"], "clocks": geo_alone["clocks"],
                      "tflops": round(gflops / (geo_graph_ms * 1e-3) / 1e12, 2),
                      "frac_of_peak": round(gflops / (geo_graph_ms * 1e-3) / 1e12 / pk["tflops"], 4),
                      "support_pairs": pairs, "tile_pairs": pairs_exec,
                      "tile_fill": round(pairs / pairs_exec, 4),
                      "support_per_row": round(pairs / gpair.n, 1),
                      "roofline": geo_roof,
                      "fps": fps_timing,
                      "note": "step = scores/top-R + fwd + bwd (the backward reuses the forward's "
                              "patch-major operands and schedule from the workspace); "
                              "ms_per_step: the step's launches replayed as one CUDA graph, "
                              "eager_ms_per_step: launched one by one through the API (the two "
                              "alternating, Geo steps only, before any dense step; clocks "
                              "sampled meanwhile); eager_ms_per_step_beside_dense: in the main "
                              "timed region, each after a dense step; FPS per shape, outside "
                              "the step, timed warm on resident points"}
    return res


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(pair, budget_s, need_dv):
    """Time the oracle's dense fwd+bwd on a row sample; extrapolate to all rows."""
    import oracle
    import torch
    bf = lambda a: torch.tensor(a).to(torch.bfloat16).double().numpy()
    Q, K, V = bf(pair.F_N), bf(pair.F_M), bf(pair.Phi_M)
    dO = bf(pair.dO)
    def run(r):
        t0 = time.perf_counter()
        oracle.dense_bwd(Q[:r], K, V, dO[:r], pair.scale)
        return time.perf_counter() - t0

    # grow the sample until a run takes an eighth of the budget, then one run
    # sized to fill the budget (about budget_s of host work in that last run)
    rows = 16
    dt = run(rows)
    while dt < budget_s / 8 and rows < pair.n:
        rows = min(pair.n, rows * 4)
        dt = run(rows)
    if rows < pair.n:
        rows = max(rows, min(pair.n, int(rows * budget_s / dt)))
        dt = run(rows)
    full_s = dt * pair.n / rows
    fpp, bpp = pair_flops(pair.d, pair.k, need_dv)
    tflops = float(pair.n) * pair.n * (fpp + bpp) / full_s / 1e12
    return tflops, full_s * 1e3, rows, dt


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, ws, rank):
    from spatial_spectral_attention_b200 import synth
    pair = synth.make_workload(args.workload, n=args.n)
    vals, times = [], []
    for s in range(args.warmup + args.steps):
        tf, ms, rows, dt = oracle_sample(pair, args.ref_budget, args.need_dv)
        if s >= args.warmup:
            vals.append(tf)
            times.append(ms)
    v = float(np.mean(vals))
    cores = cpu_cores()
    sample = f"{rows} of {pair.n} target rows per step (all {pair.n} source rows), extrapolated"
    return {
        "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(float(np.mean(times)), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": pair.name, "n": pair.n, "d": pair.d, "k": pair.k,
                   "need_dV": args.need_dv},
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dense_60k")
    ap.add_argument("--n", type=int, default=None, help="resize the workload (profiling runs)")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the linear, deterministic, e4m3, batched and mesh-FPS lines")
    ap.add_argument("--no-geo-sweep", dest="geo_sweep", action="store_false",
                    help="skip the Geo step sweep over n = 20k..160k")
    ap.add_argument("--need-dv", action="store_true")
    ap.add_argument("--no-geo", dest="with_geo", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--ref-budget", type=float, default=8.0, help="seconds of oracle time per step")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    ws, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, ws, rank)), flush=True)
        return
    res = run_ours(args, ws, rank, local)
    if rank == 0:
        if args.cpu_baseline:
            from spatial_spectral_attention_b200 import synth
            tf, ms, rows, dt = oracle_sample(synth.make_workload(args.workload, n=args.n), 12.0,
                                             args.need_dv)
            res["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": cpu_cores(),
                                   "kind": "oracle", "ms_full_step_est": round(ms, 1),
                                   "sample": f"{rows} of {res['config']['n']} target rows "
                                             f"({dt:.1f} s), extrapolated to all rows"}
        print(json.dumps(res), flush=True)
    from spatial_spectral_attention_b200 import dist
    dist.finalize(ws)


if __name__ == "__main__":
    main()
