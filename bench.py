#!/usr/bin/env python
"""Benchmark of the LoRAForge hot path on B200 (one JSON line on stdout, rank 0).

Headline workload (the "factor construction fleet"): 85 adapters of
Qwen2.5-7B-shaped LoRA modules (28 layers x q/k/v/o/gate/up/down = 196 modules
each, 16 660 modules), r = 64, fp32 factors with sigma_j ~ j^-1 * lognormal(0, 0.5),
compressed with LoRAForge-S at 1/12 of rank with floor 1.  One step = batched
TSQR + small SVD (lf_tsqr_batched) followed by allocation, fp64 boundary
refinement and export of the ragged fp32+bf16 pools (lf_truncate_export).
Metric: modules/s, plus the fraction of the HBM roofline.

Also reported in the same line:
* ``lora_path``: the rank-specialised side path y += s B'(A'x) on the decode
  workload (Llama-3-8B shapes, 32 layers x 7 projections, 256 tokens over 128
  adapters with Zipf(1) ids, ranks from the S allocation of synthetic spectra),
  with its padded-to-max and uncompressed rank-64 variants, and the prefill
  workload (Qwen2.5-7B layer, 32 requests x 512 tokens, k = 16 and uncompressed
  r = 64), in tokens/s;
* ``large_fleet``: 1024 Llama-3-8B-shaped adapters compressed in chunks of 64,
  then a mixed 4096-token batch through all 32 layers, ragged vs padded;
* ``library_qr_context``: torch.linalg.qr (cuSOLVER) on one adapter's modules
  next to this library's TSQR on the same bytes.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl loraforge|reference]
For N > 1 launch under torchrun; every rank compresses its own fleet (weak scaling).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

METRIC = "LoRA-path tokens/s and TSQR modules/s, each as % of B200 HBM roofline"
N_ADAPTERS = 85
POLICY = (1, 1, 12, 1)   # kind S, 1/12, floor 1
FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- clocks
def smi_device_id(dev_index: int) -> str:
    """nvidia-smi's --id for this process's CUDA device dev_index: its entry in
    CUDA_VISIBLE_DEVICES (an index or a UUID, both of which nvidia-smi takes) when that is
    set, else the index itself."""
    vis = [p.strip() for p in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if p.strip()]
    return vis[dev_index] if dev_index < len(vis) else str(dev_index)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region.

    The sampler is started, and its first sample awaited, on entry; the region is the
    body of the ``with`` block, and ``summary`` keeps only the samples taken inside it."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str, period_ms: int = 50, exe: str = "nvidia-smi"):
        self.gpu = gpu
        self.period_ms = period_ms
        self.exe = exe
        self.samples: list[tuple[float, str]] = []
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                [self.exe, f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            deadline = time.perf_counter() + 5.0
            while not self.samples and self.proc.poll() is None and time.perf_counter() < deadline:
                time.sleep(0.005)
        except OSError:
            self.proc = None
        self.t0 = time.perf_counter()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.perf_counter(), line.strip()))

    def __exit__(self, *a):
        self.t1 = time.perf_counter()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t1 = self.t1 if self.t1 is not None else float("inf")
        for t, ln in list(self.samples):
            if self.t0 is None or not (self.t0 <= t <= t1):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "period_ms": self.period_ms}


# ----------------------------------------------------------------- helpers
def algo_bytes_factor(mods, ranks_np):
    """Bytes the method must move for one step of the factor path.
    in: every B and A once (fp32); out: ragged fp32 + bf16 pools, R/sigma/U/V."""
    r = mods["r"].astype(np.int64); d_out = mods["d_out"].astype(np.int64); d_in = mods["d_in"].astype(np.int64)
    inp = int((4 * r * (d_out + d_in)).sum())
    k = ranks_np.astype(np.int64)
    out = int((6 * k * (d_out + d_in)).sum())
    rs = int(r.max()); n = len(r)
    small = n * (2 * 4 * rs * rs + 8 * rs + 2 * 8 * rs * rs)
    return inp, out, small


def timed(fn, steps, sync_all, stream):
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sync_all()
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    sync_all()
    return start.elapsed_time(end)



# ------------------------------------------------------------- roofline
# ALU peaks from unit counts x SM clock: fp32 SIMT 148 SMs x 128 lanes x 2 flop; fp64
# (mma.m8n8k4.f64 and DFMA share the rate) 148 SMs x 64 FMA/clk x 2 flop = 37.2 TF at 1965 MHz.
B200_SMS, FP32_LANES_PER_SM, FP64_FMA_PER_SM = 148, 128, 64


def alu_peak_tflops(sm_mhz):
    return B200_SMS * FP32_LANES_PER_SM * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


def fp64_peak_tflops(sm_mhz):
    return B200_SMS * FP64_FMA_PER_SM * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


def kernel_traffic(kernel, units):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json), scaled
    by the units one launch processes; None when the kernel's source changed since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["source_sha256"]:
        return None
    return int(rec["bytes_per_unit"] * units)


def dominant_roofline(dom, per_launch_ms, fr, hbm, peak_kind, sm_mhz):
    n = fr["n"]
    if dom == "tsqr_gram_leaf":
        # symmetric Gram X^T X of an m x r fp32 matrix in fp64: m r (r + 1) flop; both factors of every module
        flops = fr["gram_flops"]
        ach = flops / (per_launch_ms * 1e-3) / 1e12
        peak = fp64_peak_tflops(sm_mhz)
        gbs = fr["bytes_in"] / (per_launch_ms * 1e-3) / 1e9
        return {"kernel": dom, "bound": "alu", "achieved": round(ach, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": kernel_traffic(dom, n),
                "algo_flops": int(flops), "dtype": "f64",
                "peak_source": "derived: 148 SMs x 64 fp64 FMA/clk x 2 x SM clock",
                "hbm": {"achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                        "algo_bytes": int(fr["bytes_in"]), "peak_source": peak_kind}}
    if dom == "tsqr_householder":
        # Householder QR of an m x r matrix: 2 m r^2 - 2 r^3 / 3 flop; both factors of every module
        flops = fr["qr_flops"]
        ach = flops / (per_launch_ms * 1e-3) / 1e12
        peak = alu_peak_tflops(sm_mhz)
        gbs = fr["bytes_in"] / (per_launch_ms * 1e-3) / 1e9
        return {"kernel": dom, "bound": "alu", "achieved": round(ach, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": kernel_traffic(dom, n),
                "algo_flops": int(flops), "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x SM clock",
                "hbm": {"achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                        "algo_bytes": int(fr["bytes_in"]), "peak_source": peak_kind}}
    if dom == "tsqr_gram_i8":
        # every B and A^T row of the eligible matrices (all of this workload's) read once
        b = fr["bytes_in"]
        ach = b / (per_launch_ms * 1e-3) / 1e9
        return {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "traffic": kernel_traffic(dom, n), "algo_bytes": int(b),
                "peak_source": peak_kind}
    algo = {"export_stream": fr["bytes_in"] + fr["bytes_out"]}
    b = algo.get(dom)
    if b is None:
        return {"kernel": dom, "bound": "alu", "achieved": None, "peak": None, "unit": None, "frac": None,
                "traffic": None}
    ach = b / (per_launch_ms * 1e-3) / 1e9
    return {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(ach / hbm, 4), "traffic": kernel_traffic(dom, n), "algo_bytes": int(b),
            "peak_source": peak_kind}


# ------------------------------------------------------------ sharding
def shard_adapter_base(rank: int, n_adapters_per_rank: int) -> int:
    """Adapters are sharded across ranks with no exchange (the S budget is per adapter):
    rank r compresses adapters [r * n, (r + 1) * n) of the fleet."""
    return rank * n_adapters_per_rank


def max_over_ranks(x: float, pg, dev) -> float:
    """Max of a per-rank device time over all ranks (identity without a process group)."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, max_ms: float) -> float:
    """Units all ranks processed divided by the slowest rank's time (per second)."""
    return units_per_rank * world / (max_ms * 1e-3)


# ------------------------------------------------------------ factor path
def factor_bench(args, rank, world, dev, sync_all, stream, hbm, peak_kind):
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    n_ad = args.adapters
    lay = synth.fleet_layout(n_ad, synth.QWEN25_7B, r=64)
    mods = api.modules_from_layout(lay)
    B = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
    A = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
    synth.fill_fleet(lay, B, A, cfg_id=2, adapter_base=shard_adapter_base(rank, n_ad))
    pol = lf.lf_policy(*POLICY)
    F = api.alloc_factors(mods, dev)
    E = api.alloc_export(mods, pol, dev, bf16=True)
    ws_t = api.workspace(lf.lf_tsqr_workspace_size(mods), dev)
    ws_e = api.workspace(lf.lf_export_workspace_size(mods), dev)
    torch.cuda.synchronize()

    def step():
        api.tsqr(mods, B, A, out=F, ws=ws_t, stream=stream)
        api.truncate_export(mods, pol, B, A, F, out=E, ws=ws_e, stream=stream)

    for _ in range(args.warmup):
        step()
    assert lf.lf_get_device_status(stream) == 0
    lf.lf_profile_reset()
    lf.lf_profile_enable(True)
    launches0 = lf.lf_launch_count()
    with ClockSampler(smi_device_id(torch.cuda.current_device())) as clk:
        ms = timed(step, args.steps, sync_all, stream)
    launches = lf.lf_launch_count() - launches0
    lf.lf_profile_enable(False)
    phases = lf.lf_profile_read()
    st = lf.lf_get_device_status(stream)
    ranks = E.ranks.cpu().numpy()
    inp, out, small = algo_bytes_factor(mods, ranks)
    m_rows = (lay.d_out.astype(np.int64) + lay.d_in.astype(np.int64))
    rr = lay.r.astype(np.int64)
    qr_flops = float((2 * m_rows * rr * rr - 2 * (2 * rr ** 3) // 3).sum())
    gram_flops = float((m_rows * rr * (rr + 1)).sum())
    res = dict(ms=ms, launches=launches, phases=phases, clocks=clk.summary(), status=st, n=lay.n, qr_flops=qr_flops,
               gram_flops=gram_flops,
               bytes_in=inp, bytes_out=out, bytes_small=small, ranks_sum=int(ranks.sum()),
               params_frac=float((ranks.astype(np.int64) * (lay.d_in + lay.d_out)).sum() /
                                 (lay.r.astype(np.int64) * (lay.d_in + lay.d_out)).sum()))
    del B, A, F, E, ws_t, ws_e
    torch.cuda.empty_cache()
    return res


def factor_e2e(args, dev, stream, rank=0):
    """Same step through the C ABI with the inputs in pinned HOST memory: the H2D copy of
    B and A and the D2H copy of the rank table, offsets and bf16 pools are timed."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    n_ad = args.e2e_adapters
    lay = synth.fleet_layout(n_ad, synth.QWEN25_7B, r=64)
    mods = api.modules_from_layout(lay)
    Bh = torch.empty(lay.B_total, dtype=torch.float32, pin_memory=True)
    Ah = torch.empty(lay.A_total, dtype=torch.float32, pin_memory=True)
    Bd = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
    Ad = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
    synth.fill_fleet(lay, Bd, Ad, cfg_id=2, adapter_base=10_000 + shard_adapter_base(rank, n_ad))
    Bh.copy_(Bd); Ah.copy_(Ad)
    pol = lf.lf_policy(*POLICY)
    F = api.alloc_factors(mods, dev)
    E = api.alloc_export(mods, pol, dev, bf16=True)
    ws_t = api.workspace(lf.lf_tsqr_workspace_size(mods), dev)
    ws_e = api.workspace(lf.lf_export_workspace_size(mods), dev)
    # pinned host destinations, allocated once like the inputs: the rank table and offsets
    # come back first (they size the pools), then the used part of each bf16 pool
    ranks_h = torch.empty_like(E.ranks, device="cpu").pin_memory()
    offA_h = torch.empty_like(E.off_A, device="cpu").pin_memory()
    offB_h = torch.empty_like(E.off_Bt, device="cpu").pin_memory()
    A16_h = torch.empty_like(E.A_pool16, device="cpu").pin_memory()
    B16_h = torch.empty_like(E.Bt_pool16, device="cpu").pin_memory()
    outs_h = {}

    def step():
        with torch.cuda.stream(stream):
            Bd.copy_(Bh, non_blocking=True); Ad.copy_(Ah, non_blocking=True)
        api.tsqr(mods, Bd, Ad, out=F, ws=ws_t, stream=stream)
        api.truncate_export(mods, pol, Bd, Ad, F, out=E, ws=ws_e, stream=stream)
        with torch.cuda.stream(stream):
            ranks_h.copy_(E.ranks, non_blocking=True)
            offA_h.copy_(E.off_A, non_blocking=True); offB_h.copy_(E.off_Bt, non_blocking=True)
            stream.synchronize()
            na, nb = int(offA_h[-1]), int(offB_h[-1])
            A16_h[:na].copy_(E.A_pool16[:na], non_blocking=True); B16_h[:nb].copy_(E.Bt_pool16[:nb], non_blocking=True)
            stream.synchronize()
        outs_h["d2h"] = ranks_h.numel() * 4 + (offA_h.numel() + offB_h.numel()) * 8 + 2 * (na + nb)

    step()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    k = max(1, min(args.steps, 3))
    for _ in range(k):
        step()
    torch.cuda.synchronize()
    dt = (time.perf_counter() - t0) / k
    res = dict(value=lay.n / dt, h2d=int(4 * (lay.B_total + lay.A_total)), d2h=int(outs_h["d2h"]),
               adapters=n_ad, modules=lay.n)
    del Bh, Ah, Bd, Ad, F, E, ws_t, ws_e, ranks_h, offA_h, offB_h, A16_h, B16_h
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------- apply path
def apply_bytes(T, d_in, d_out, ranks_used):
    return 2 * T * d_in + 4 * T * d_out + 4 * T + sum(2 * k * (d_in + d_out) for k in ranks_used)


def _decode_e2e(args, calls, ids, ids_d, T, stream):
    """The decode step through the public call with host buffers: per step the token ids,
    every layer's inputs x and outputs y go up from pinned host memory, the 32
    lf_lora_shrink_expand_projections calls run, and every y comes back (y is updated in
    place, so it travels both ways).  Uploads, calls and read-backs run on three streams
    ordered by events layer by layer, so the two copy directions share the PCIe link at
    once: layer l's upload waits for the previous step's read-back of its buffers, its
    call for its upload, its read-back for its call.  Device-timed with events on the
    calling stream around all steps (it joins the read-back stream at the end).  One
    step with everything on the calling stream comes first; the overlapped steps must
    return the same bytes (``matches_serial``)."""
    import torch
    xs, ys = {}, {}
    for c in calls:
        for x, y, _ in c.items:
            xs.setdefault(x.data_ptr(), x)
            ys.setdefault(y.data_ptr(), y)
    xh = {k: v.cpu().pin_memory() for k, v in xs.items()}
    yh = {k: v.cpu().pin_memory() for k, v in ys.items()}
    yo = {k: torch.empty_like(v).pin_memory() for k, v in yh.items()}
    ids_h = torch.from_numpy(np.asarray(ids, np.int32)).pin_memory()
    xp = [sorted({x.data_ptr() for x, _, _ in c.items}) for c in calls]
    yp = [sorted({y.data_ptr() for _, y, _ in c.items}) for c in calls]

    def serial_step():
        with torch.cuda.stream(stream):
            ids_d.copy_(ids_h, non_blocking=True)
            for l, c in enumerate(calls):
                for p in xp[l]:
                    xs[p].copy_(xh[p], non_blocking=True)
                for p in yp[l]:
                    ys[p].copy_(yh[p], non_blocking=True)
                c(stream)
                for p in yp[l]:
                    yo[p].copy_(ys[p], non_blocking=True)

    serial_step()
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in yo.items()}

    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in calls]
    ev_call = [torch.cuda.Event() for _ in calls]
    ev_down = [torch.cuda.Event() for _ in calls]
    primed = [False]

    def step():
        with torch.cuda.stream(up):
            if primed[0]:
                up.wait_event(ev_call[-1])   # the previous step's calls have read ids
            ids_d.copy_(ids_h, non_blocking=True)
            for l in range(len(calls)):
                if primed[0]:
                    up.wait_event(ev_down[l])   # the previous step is done with x_l, y_l
                for p in xp[l]:
                    xs[p].copy_(xh[p], non_blocking=True)
                for p in yp[l]:
                    ys[p].copy_(yh[p], non_blocking=True)
                ev_up[l].record(up)
        for l, c in enumerate(calls):
            stream.wait_event(ev_up[l])
            c(stream)
            ev_call[l].record(stream)
        with torch.cuda.stream(down):
            for l in range(len(calls)):
                down.wait_event(ev_call[l])
                for p in yp[l]:
                    yo[p].copy_(ys[p], non_blocking=True)
                ev_down[l].record(down)
        primed[0] = True

    up.wait_stream(stream)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    reps = max(args.steps, 5)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    for _ in range(reps):
        step()
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    same = all(torch.equal(ref[k], yo[k]) for k in yo)
    h2d = ids_h.numel() * 4 + sum(v.numel() * 2 for v in xh.values()) + sum(v.numel() * 2 for v in yh.values())
    d2h = sum(v.numel() * 2 for v in yo.values())
    return {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "matches_serial": bool(same),
            "sample": "the whole decode step (32 layers) from pinned host memory, uploads, calls and "
                      "read-backs on three streams"}


def decode_bench(args, dev, stream, hbm, variant="ragged", fused=False, per_layer=True, e2e=False):
    """Config 3: Llama-3-8B shapes, 32 layers x 7 projections, T=256, 128 adapters.
    variant: "ragged" (retained ranks as allocated), "padded" (every adapter's factors
    of a projection zero-padded to the largest retained rank over the 128 resident
    adapters), "r64" (uncompressed rank-64 adapters).  per_layer: the 7 projections of
    a layer in one lf_lora_shrink_expand_projections call (32 calls per step); else
    fused: q/k/v and gate/up as one multi-slice call each (4 calls per layer), or one
    call per projection (7 per layer)."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.LLAMA3_8B
    n_ad, T = 128, 256
    per_layer = per_layer and not fused
    lay = synth.fleet_layout(n_ad, M, r=64)
    mods = api.modules_from_layout(lay)
    sig = synth.sigma_tables(n_ad, M, 64, cfg_id=3)
    ranks_all, _, _ = api.select_ranks(mods, lf.policy_S(1, 12, 1), torch.from_numpy(sig).to(dev))
    ranks_all = ranks_all.cpu().numpy().reshape(n_ad, 7, M.layers)
    ids = synth.zipf_ids(T, n_ad, 1.0, (3, 0))
    ids_d = torch.from_numpy(ids).to(dev)
    distinct = sorted(set(ids.tolist()))
    shapes = M.proj_shapes()
    calls = []
    total_bytes = 0
    for l in range(M.layers):
        x_h = synth.normal_bf16((T, M.hidden), (3, 1, l), device=dev)
        x_f = synth.normal_bf16((T, M.ffn), (3, 2, l), device=dev)
        groups = []
        for p, (_, d_out, d_in) in enumerate(shapes):
            rk_true = ranks_all[:, p, l].astype(np.int64)
            if variant == "ragged":
                rk = rk_true
            elif variant == "padded":
                rk = np.full(n_ad, int(rk_true.max()), dtype=np.int64)
            else:
                rk = np.full(n_ad, 64, dtype=np.int64)
            offA = np.concatenate([[0], np.cumsum(rk * d_in)]); offB = np.concatenate([[0], np.cumsum(rk * d_out)])
            Ap = synth.normal_bf16((int(offA[-1]),), (3, 3, l, p), std=d_in ** -0.5, device=dev)
            Bt = synth.normal_bf16((int(offB[-1]),), (3, 4, l, p), std=d_out ** -0.5, device=dev)
            if variant == "padded":   # rows past each adapter's retained rank are zero
                kmax = int(rk[0])
                pad = torch.from_numpy(np.arange(kmax)[None, :] >= rk_true[:, None]).to(dev)
                Ap.view(n_ad, kmax, d_in)[pad] = 0
                Bt.view(n_ad, kmax, d_out)[pad] = 0
            groups.append((d_in, d_out, rk, offA, offB, Ap, Bt))
            total_bytes += apply_bytes(T, d_in, d_out, [int(rk[a]) for a in distinct])
        lc, sets = _layer_calls(groups, lambda d: x_f if d == M.ffn else x_h, ids_d, n_ad, T, dev, (3, 5, l), fused,
                                per_layer=per_layer)
        calls += lc
        if fused:   # x is read once per call, not once per projection
            total_bytes -= sum(2 * T * groups[ps[0]][0] * (len(ps) - 1) for ps in sets)
    names = {"ragged": "S 1/12 floor 1 ranks (ragged)",
             "padded": "S 1/12 floor 1 ranks zero-padded to the per-projection max over resident adapters",
             "r64": "uncompressed rank-64 adapters"}
    how = ("; q/k/v and gate/up as one slice call each" if fused else
           ("; the 7 projections of a layer in one call" if per_layer else "; one call per projection"))
    out = _apply_run(args, calls, ids_d, n_ad, T, total_bytes, stream, hbm, dict(
        workload="decode: Llama-3-8B, 32 layers x 7 projections, 256 tokens, 128 adapters Zipf(1), "
                 + names[variant] + how,
        distinct_adapters=len(distinct), mean_rank=float(ranks_all.mean())))
    if e2e and per_layer:
        out["e2e"] = _decode_e2e(args, calls, ids, ids_d, T, stream)
    del calls
    torch.cuda.empty_cache()
    return out


def sandwich_bench(args, dev, stream, hbm, rank=16, diagonal=True):
    """Sigma-sandwich serving of jointly compressed adapters on the decode workload:
    Llama-3-8B shapes, 32 layers x 7 projections, 256 tokens over 128 adapters (Zipf(1));
    per projection a shared V^T (rank x d_in), U^T (rank x d_out) and a Sigma_a per adapter
    (diagonal or full rank x rank)."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.LLAMA3_8B
    n_ad, T = 128, 256
    ids = synth.zipf_ids(T, n_ad, 1.0, (3, 0))
    ids_d = torch.from_numpy(ids).to(dev)
    n_dist = len(set(ids.tolist()))
    calls, total_bytes = [], 0
    g = np.random.default_rng(6)
    for l in range(M.layers):
        x_h = synth.normal_bf16((T, M.hidden), (6, 1, l), device=dev)
        x_f = synth.normal_bf16((T, M.ffn), (6, 2, l), device=dev)
        for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
            Vt = synth.normal_bf16((rank, d_in), (6, 3, l, p), std=d_in ** -0.5, device=dev)
            Ut = synth.normal_bf16((rank, d_out), (6, 4, l, p), std=d_out ** -0.5, device=dev)
            shape = (n_ad, rank) if diagonal else (n_ad, rank, rank)
            sig = torch.from_numpy(g.standard_normal(shape).astype(np.float32)).to(dev)
            y = synth.normal_bf16((T, d_out), (6, 5, l, p), device=dev)
            x = x_f if d_in == M.ffn else x_h
            ws = api.workspace(lf.lf_apply_workspace_size(T, n_ad), dev)

            def run(st=None, x=x, y=y, Vt=Vt, Ut=Ut, sig=sig, ws=ws):
                lf.lf_lora_sigma_sandwich(x, y, ids_d, n_ad, Vt, Ut, sig, diagonal, 2.0, ws, stream=st)
            calls.append(run)
            total_bytes += 2 * T * d_in + 4 * T * d_out + 4 * T + 2 * rank * (d_in + d_out) \
                + 4 * n_dist * (rank if diagonal else rank * rank)
    out = _apply_run(args, calls, ids_d, n_ad, T, total_bytes, stream, hbm, dict(
        workload=f"Sigma-sandwich decode: Llama-3-8B, 32 layers x 7 projections, 256 tokens, 128 adapters "
                 f"Zipf(1), shared U, V of rank {rank}, {'diagonal' if diagonal else 'full'} Sigma per adapter"))
    del calls
    torch.cuda.empty_cache()
    return out


def prefill_bench(args, dev, stream, hbm, k, fused=False, route_once=True):
    """Config 4: Qwen2.5-7B layer, 7 projections, 32 requests x 512 tokens, request i -> adapter i.
    fused: q/k/v and gate/up as one multi-slice call each.  route_once: the batch is routed
    once per step (lf_route_tokens) and every projection call reuses the tables; otherwise
    every call routes the batch again."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.QWEN25_7B
    n_ad, T = 32, 32 * 512
    ids = np.repeat(np.arange(n_ad, dtype=np.int32), 512)
    ids_d = torch.from_numpy(ids).to(dev)
    x_h = synth.normal_bf16((T, M.hidden), (4, 1), device=dev)
    x_f = synth.normal_bf16((T, M.ffn), (4, 2), device=dev)
    groups, total_bytes = [], 0
    for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
        rk = np.full(n_ad, k, dtype=np.int64)
        offA = np.concatenate([[0], np.cumsum(rk * d_in)]); offB = np.concatenate([[0], np.cumsum(rk * d_out)])
        Ap = synth.normal_bf16((int(offA[-1]),), (4, 3, p, k), std=d_in ** -0.5, device=dev)
        Bt = synth.normal_bf16((int(offB[-1]),), (4, 4, p, k), std=d_out ** -0.5, device=dev)
        groups.append((d_in, d_out, rk, offA, offB, Ap, Bt))
        total_bytes += apply_bytes(T, d_in, d_out, [k] * n_ad)
    calls, sets = _layer_calls(groups, lambda d: x_f if d == M.ffn else x_h, ids_d, n_ad, T, dev, (4, 5), fused,
                               route_once)
    if fused:
        total_bytes -= sum(2 * T * groups[ps[0]][0] * (len(ps) - 1) for ps in sets)
    return _apply_run(args, calls, ids_d, n_ad, T, total_bytes, stream, hbm, dict(
        workload=f"prefill: Qwen2.5-7B layer x 7 projections, 32 requests x 512 tokens, k={k}"
                 + ("; q/k/v and gate/up as one slice call each" if fused else "")
                 + ("; routed once per step, projections reuse the tables" if route_once
                    else "; every call routes the batch")))


def _proj_call(x, y, ids_d, n_ad, rk, oa, ob, Ap, Bt, ws, scale=2.0):
    """One projection through lf_lora_shrink_expand."""
    from post_hoc_rank_b200 import loraforge as lf

    def run(st=None):
        lf.lf_lora_shrink_expand(x, y, ids_d, n_ad, rk, oa, ob, Ap, Bt, scale, ws, stream=st)
    return run


def _slices_call(x, y, ids_d, n_ad, slices, ws, scale=2.0):
    """Projections sharing x through one lf_lora_shrink_expand_slices call; slices:
    (d_out, y_offset, ranks, off_A, off_Bt, A_pool, Bt_pool, max_rank): device tensors and the
    largest rank of the slice."""
    from post_hoc_rank_b200 import loraforge as lf
    sl = [lf.make_slice(*t) for t in slices]

    def run(st=None, _keep=slices):
        lf.lf_lora_shrink_expand_slices(x, y, ids_d, n_ad, sl, scale, ws, stream=st)
    return run


def _routed_call(x, y, ids_d, n_ad, slices, ws, scale=2.0):
    """Projections through lf_lora_shrink_expand_slices_routed (tables already in ws)."""
    from post_hoc_rank_b200 import loraforge as lf
    sl = [lf.make_slice(*t) for t in slices]

    def run(st=None, _keep=slices):
        lf.lf_lora_shrink_expand_slices_routed(x, y, ids_d, n_ad, sl, scale, ws, stream=st)
    return run


def _projections_call(items, ids_d, n_ad, T, ws, scale=2.0):
    """Every projection of a layer through one lf_lora_shrink_expand_projections call;
    items: (x, y, (d_out, y_offset, ranks, off_A, off_Bt, A_pool, Bt_pool, max_rank)) device tensors
    and the largest rank of the projection."""
    from post_hoc_rank_b200 import loraforge as lf
    projs = [lf.make_projection(x, y, lf.make_slice(*t)) for x, y, t in items]

    def run(st=None, _keep=items):
        lf.lf_lora_shrink_expand_projections(T, ids_d, n_ad, projs, scale, ws, stream=st)
    run.items = items
    return run


def _layer_calls(groups, x_of, ids_d, n_ad, T, dev, key, fused, route_once=False, per_layer=False):
    """Calls of one layer.  groups: per projection (d_in, d_out, rk int64 array, offA,
    offB, Ap, Bt); fused: q/k/v and gate/up (projections reading the same x) go as
    one slice call each; route_once: one lf_route_tokens call, then routed projection
    calls on the same workspace; per_layer: all projections in one
    lf_lora_shrink_expand_projections call.  Returns (callables, the projection sets)."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf
    sets = [[0, 1, 2], [3], [4, 5], [6]] if fused else [[p] for p in range(len(groups))]
    if per_layer:
        items = []
        for p, (d_in, d_out, rk, offA, offB, Ap, Bt) in enumerate(groups):
            y = synth.normal_bf16((T, d_out), key + (p,), device=dev)
            items.append((x_of(d_in), y, (d_out, 0, torch.from_numpy(rk.astype(np.int32)).to(dev),
                                          torch.from_numpy(offA[:-1]).to(dev), torch.from_numpy(offB[:-1]).to(dev),
                                          Ap, Bt, int(rk.max()))))
        ws = api.workspace(lf.lf_apply_workspace_size(T, n_ad), dev)
        return [_projections_call(items, ids_d, n_ad, T, ws)], sets
    calls = []
    rws = None
    if route_once:
        rws = api.workspace(lf.lf_apply_slices_workspace_size(T, n_ad, max(len(ps) for ps in sets)), dev)

        def route(st=None):
            lf.lf_route_tokens(ids_d, n_ad, rws, stream=st)
        calls.append(route)
    for gi, ps in enumerate(sets):
        d_in = groups[ps[0]][0]
        x = x_of(d_in)
        widths = [groups[p][1] for p in ps]
        y = synth.normal_bf16((T, sum(widths)), key + (gi,), device=dev)
        tens = []
        y_off = 0
        for p in ps:
            _, d_out, rk, offA, offB, Ap, Bt = groups[p]
            tens.append((d_out, y_off, torch.from_numpy(rk.astype(np.int32)).to(dev),
                         torch.from_numpy(offA[:-1]).to(dev), torch.from_numpy(offB[:-1]).to(dev), Ap, Bt,
                         int(rk.max())))   # the caller's rank bound for the slice
            y_off += d_out
        if route_once:
            calls.append(_routed_call(x, y, ids_d, n_ad, tens, rws))
        elif len(ps) == 1:
            ws = api.workspace(lf.lf_apply_workspace_size(T, n_ad), dev)
            d_out, _, rk_d, oa_d, ob_d, Ap, Bt, _ = tens[0]
            calls.append(_proj_call(x, y, ids_d, n_ad, rk_d, oa_d, ob_d, Ap, Bt, ws))
        else:
            ws = api.workspace(lf.lf_apply_slices_workspace_size(T, n_ad, len(ps)), dev)
            calls.append(_slices_call(x, y, ids_d, n_ad, tens, ws))
    return calls, sets


def _apply_run(args, calls, ids_d, n_ad, T, total_bytes, stream, hbm, meta):
    import torch
    from post_hoc_rank_b200 import loraforge as lf

    def step(st=None):
        # st=None: torch's current stream (the capture stream inside torch.cuda.graph)
        for c in calls:
            c(st)

    for _ in range(max(args.warmup, 3)):
        step(stream)
    torch.cuda.synchronize()
    assert lf.lf_get_device_status(stream) == 0
    l0 = lf.lf_launch_count()
    step(stream)
    launches = lf.lf_launch_count() - l0
    # CUDA graph of one step (host launch cost out of the measurement)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=cap):
        step()
    torch.cuda.synchronize()
    reps = max(args.steps, 5) * 4
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    cs = torch.cuda.current_stream()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(cs)
    for _ in range(reps):
        g.replay()
    s1.record(cs)
    torch.cuda.synchronize()
    ms = s0.elapsed_time(s1) / reps
    # per-kernel device times (eager, profiled)
    lf.lf_profile_reset(); lf.lf_profile_enable(True)
    for _ in range(3):
        step(stream)
    lf.lf_profile_enable(False)
    ph = {k: v for k, v in lf.lf_profile_read().items() if v[1] > 0}
    gbs = total_bytes / (ms * 1e-3) / 1e9
    del g
    out = dict(meta)
    out.update(tokens_per_s=T / (ms * 1e-3), ms_per_step=ms, algo_bytes=int(total_bytes), achieved_gbs=gbs,
               hbm_frac=gbs / hbm, launches_per_step=launches,
               phases_ms={k: v[0] / 3 for k, v in ph.items()})
    return out


def large_fleet_bench(args, dev, stream, hbm):
    """Config 5: 1024 Llama-3-8B-shaped adapters (224 modules each, r = 64), compressed
    with LoRAForge-S 1/12 floor 1 in chunks of 64 adapters (each chunk generated in
    HBM, then one lf_tsqr_batched + lf_truncate_export, device-timed), then a mixed
    batch of 4096 tokens (64 prefill segments x 48 tokens + 1024 decode tokens, ids
    Zipf(1.2) over the 1024 adapters) through all 32 layers x 7 projections with the
    exported bf16 factors, ragged and padded to the per-projection max rank over the
    adapters the batch references."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.LLAMA3_8B
    n_total, chunk = args.large_adapters, 64
    nchunks = (n_total + chunk - 1) // chunk
    lay = synth.fleet_layout(chunk, M, r=64)
    mods = api.modules_from_layout(lay)
    B = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
    A = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
    pol = lf.lf_policy(*POLICY)
    F = api.alloc_factors(mods, dev)
    E = api.alloc_export(mods, pol, dev, bf16=True)
    ws_t = api.workspace(lf.lf_tsqr_workspace_size(mods), dev)
    ws_e = api.workspace(lf.lf_export_workspace_size(mods), dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    compress_ms, ranks_c, offA_c, offB_c, poolsA, poolsB = 0.0, [], [], [], [], []
    for c in range(nchunks):
        synth.fill_fleet(lay, B, A, cfg_id=5, adapter_base=c * chunk)
        torch.cuda.synchronize()
        e0.record(stream)
        api.tsqr(mods, B, A, out=F, ws=ws_t, stream=stream)
        api.truncate_export(mods, pol, B, A, F, out=E, ws=ws_e, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        compress_ms += e0.elapsed_time(e1)
        assert lf.lf_get_device_status(stream) == 0
        oa, ob = E.off_A.cpu().numpy(), E.off_Bt.cpu().numpy()
        ranks_c.append(E.ranks.cpu().numpy()); offA_c.append(oa); offB_c.append(ob)
        poolsA.append(E.A_pool16[:int(oa[-1])].clone()); poolsB.append(E.Bt_pool16[:int(ob[-1])].clone())
    n_mod = nchunks * lay.n
    del B, A, F, E, ws_t, ws_e
    torch.cuda.empty_cache()
    baseA = np.concatenate([[0], np.cumsum([p.numel() for p in poolsA])]).astype(np.int64)
    baseB = np.concatenate([[0], np.cumsum([p.numel() for p in poolsB])]).astype(np.int64)
    poolA = torch.cat(poolsA); poolB = torch.cat(poolsB)
    del poolsA, poolsB
    torch.cuda.empty_cache()
    # module index of (adapter, proj, layer) inside a chunk: (a_local * 7 + p) * layers + l
    a_all = np.arange(nchunks * chunk)
    cidx, aloc = a_all // chunk, a_all % chunk
    T = 4096
    seg_ids = synth.zipf_ids(64, n_total, 1.2, (5, 1))
    dec_ids = synth.zipf_ids(1024, n_total, 1.2, (5, 2))
    ids = np.concatenate([np.repeat(seg_ids, 48), dec_ids]).astype(np.int32)
    ids_d = torch.from_numpy(ids).to(dev)
    ref = np.unique(ids)
    shapes = M.proj_shapes()
    out = {"workload": f"large fleet: {n_total} adapters x Llama-3-8B (224 modules each, r=64), LoRAForge-S "
                       "1/12 floor 1, compressed in chunks of 64 adapters; then 4096 tokens (64 prefill segments "
                       "x 48 + 1024 decode tokens, Zipf(1.2) ids) through 32 layers x 7 projections, one call per layer",
           "modules": int(n_mod), "compress_ms": round(compress_ms, 2),
           "modules_per_s": round(n_mod / (compress_ms * 1e-3), 1), "distinct_adapters": int(len(ref))}
    ws = api.workspace(lf.lf_apply_workspace_size(T, n_total), dev)
    for variant in ("ragged", "padded"):
        calls, total_bytes = [], 0
        for l in range(M.layers):
            x_h = synth.normal_bf16((T, M.hidden), (5, 3, l), device=dev)
            x_f = synth.normal_bf16((T, M.ffn), (5, 4, l), device=dev)
            items = []   # the layer's 7 projections: one lf_lora_shrink_expand_projections call
            for p, (_, d_out, d_in) in enumerate(shapes):
                mi = (aloc * 7 + p) * M.layers + l
                rk = np.array([ranks_c[c][m] for c, m in zip(cidx, mi)], dtype=np.int64)
                oa = np.array([baseA[c] + offA_c[c][m] for c, m in zip(cidx, mi)], dtype=np.int64)
                ob = np.array([baseB[c] + offB_c[c][m] for c, m in zip(cidx, mi)], dtype=np.int64)
                y = synth.normal_bf16((T, d_out), (5, 5, l, p), device=dev)
                x = x_f if d_in == M.ffn else x_h
                if variant == "ragged":
                    k_used = rk[ref]
                    pa, pb, rk_d, oa_d, ob_d = poolA, poolB, rk, oa, ob
                else:
                    # padded pools for the referenced adapters: kmax rows each, rows past k zero
                    kmax = int(rk[ref].max())
                    jr = torch.arange(kmax, device=dev)
                    live = (jr[None, :] < torch.from_numpy(rk[ref]).to(dev)[:, None])
                    rows_a = torch.from_numpy(oa[ref]).to(dev)[:, None] + jr[None, :] * d_in
                    rows_b = torch.from_numpy(ob[ref]).to(dev)[:, None] + jr[None, :] * d_out
                    ia = (rows_a[:, :, None] + torch.arange(d_in, device=dev)[None, None, :]) * live[:, :, None]
                    ib = (rows_b[:, :, None] + torch.arange(d_out, device=dev)[None, None, :]) * live[:, :, None]
                    pa = (poolA[ia] * live[:, :, None]).reshape(-1).contiguous()
                    pb = (poolB[ib] * live[:, :, None]).reshape(-1).contiguous()
                    del ia, ib
                    rk_d = np.zeros(n_total, dtype=np.int64); rk_d[ref] = kmax
                    oa_d = np.zeros(n_total, dtype=np.int64); ob_d = np.zeros(n_total, dtype=np.int64)
                    oa_d[ref] = np.arange(len(ref)) * kmax * d_in; ob_d[ref] = np.arange(len(ref)) * kmax * d_out
                    k_used = np.full(len(ref), kmax)
                items.append((x, y, (d_out, 0, torch.from_numpy(rk_d.astype(np.int32)).to(dev),
                                     torch.from_numpy(oa_d).to(dev), torch.from_numpy(ob_d).to(dev), pa, pb,
                                     int(max(1, k_used.max())))))
                total_bytes += apply_bytes(T, d_in, d_out, [int(k) for k in k_used])
            calls.append(_projections_call(items, ids_d, n_total, T, ws))
        r = _apply_run(args, calls, ids_d, n_total, T, total_bytes, stream, hbm, {})
        out[variant] = {k: r[k] for k in ("tokens_per_s", "ms_per_step", "algo_bytes", "achieved_gbs", "hbm_frac",
                                          "launches_per_step", "phases_ms")}
        del calls
        torch.cuda.empty_cache()
    del poolA, poolB
    torch.cuda.empty_cache()
    return out


def jd_bench(dev, stream, hbm, sm_mhz, n_lora=64, r=16, rank=64, iters=10, with_cpu=True):
    """JD-Full eigenvalue iteration ("Compress then Serve", Appendix 8.2): n_lora
    Llama-3-8B-shaped LoRAs of rank r at each of one layer's 7 module positions (7 problems
    in one call), shared rank `rank`, `iters` steps, Sigma_i at the final bases."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.LLAMA3_8B
    lay = synth.fleet_layout(n_lora, M, r=r, n_layers=1)
    mods = api.modules_from_layout(lay)
    B = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
    A = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
    synth.fill_fleet(lay, B, A, cfg_id=7)
    positions = [[i for i in range(lay.n) if int(lay.proj[i]) == p] for p in range(7)]
    tabs = api.jd_tables(mods, positions, rank)
    U0 = torch.empty(tabs.U_total, dtype=torch.float32, device=dev)
    Vt0 = torch.empty(tabs.Vt_total, dtype=torch.float32, device=dev)
    for p, pr in enumerate(tabs.probs):
        d_out, d_in, uo, vo = int(pr["d_out"]), int(pr["d_in"]), int(pr["U_off"]), int(pr["Vt_off"])
        U0[uo:uo + d_out * rank] = synth.normal_f32((d_out * rank,), (7, 1, p), device=dev)
        Vt0[vo:vo + rank * d_in] = synth.normal_f32((rank * d_in,), (7, 2, p), device=dev)
    U, Vt = U0.clone(), Vt0.clone()
    sig = torch.empty(tabs.sigma_total, dtype=torch.float32, device=dev)
    ws = api.workspace(lf.lf_jd_workspace_size(mods, tabs.members, tabs.probs), dev)

    def solve():
        U.copy_(U0); Vt.copy_(Vt0)
        lf.lf_jd_full(mods, tabs.members, tabs.probs, B, A, None, iters, U, Vt, sig, ws, stream)

    for _ in range(2):
        solve()
    torch.cuda.synchronize()
    reps = 3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        solve()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    lf.lf_profile_reset(); lf.lf_profile_enable(True)
    l0 = lf.lf_launch_count()
    solve()
    launches = lf.lf_launch_count() - l0
    lf.lf_profile_enable(False)
    ph = lf.lf_profile_read()
    st = lf.lf_get_device_status(stream)
    # algorithmic work: each pass reads every factor once (fp32) and does 2 (d_out + d_in) r r~ flops per LoRA
    passes = 2 * iters + 1
    fac_bytes = 4 * int(((lay.d_out + lay.d_in).astype(np.int64) * lay.r).sum())
    pass_flops = 2.0 * float(((lay.d_out + lay.d_in).astype(np.int64) * lay.r).sum()) * rank
    state_bytes = 4 * int(((tabs.probs["d_out"] + tabs.probs["d_in"]).astype(np.int64)).sum()) * rank
    algo_bytes = passes * fac_bytes + (3 * passes + 6 * iters) * state_bytes
    algo_flops = passes * pass_flops
    dom = max(("jd_project", "jd_update"), key=lambda k: ph.get(k, (0.0, 1))[0])
    dom_ms, dom_n = ph[dom]
    dom_flops = (iters + 1 if dom == "jd_project" else iters) * pass_flops
    fp64 = fp64_peak_tflops(sm_mhz)
    ach = dom_flops / (dom_ms * 1e-3) / 1e12
    out = {
        "workload": f"JD-Full eigenvalue iteration: {n_lora} Llama-3-8B-shaped LoRAs (rank {r}) at each of the 7 "
                    f"module positions of one layer, shared rank {rank}, {iters} steps + Sigma",
        "ms_per_solve": round(ms, 3), "positions_per_s": round(7 / (ms * 1e-3), 2),
        "ms_per_step": round(ms / iters, 3),
        "algo_bytes": int(algo_bytes), "algo_gbs": round(algo_bytes / (ms * 1e-3) / 1e9, 1),
        "hbm_frac": round(algo_bytes / (ms * 1e-3) / 1e9 / hbm, 4),
        "algo_tflops": round(algo_flops / (ms * 1e-3) / 1e12, 2),
        "roofline": {"kernel": dom, "bound": "fp64_tensor", "achieved": round(ach, 2),
                     "peak": round(fp64, 1), "unit": "TFLOP/s", "frac": round(ach / fp64, 4),
                     "peak_source": "derived: 148 SMs x 64 fp64 FMA/clk x 2 x median SM clock"},
        "phases_ms": {k: round(v[0], 3) for k, v in ph.items()},
        "gpu_launches": int(launches), "device_status": st,
    }
    if with_cpu:
        out["cpu_baseline"] = cpu_jd_baseline(B, A, lay, tabs, U0, Vt0, rank, iters)
    del B, A, U, Vt, U0, Vt0, sig, ws
    torch.cuda.empty_cache()
    return out


def cpu_jd_baseline(B, A, lay, tabs, U0, Vt0, rank, iters):
    """The fp64 oracle's JD-Full on one module position of the same workload (q, 64 LoRAs),
    same start and step count; positions/s on the host cores."""
    import torch
    from oracle import jd as OJ
    pr = tabs.probs[0]
    m = tabs.members[int(pr["first"]):int(pr["first"]) + int(pr["count"])]
    Bh, Ah = B.cpu(), A.cpu()
    Bs = [Bh[int(lay.B_off[i]):int(lay.B_off[i]) + int(lay.d_out[i]) * int(lay.r[i])].double().numpy()
          .reshape(int(lay.d_out[i]), int(lay.r[i])) for i in m]
    As = [Ah[int(lay.A_off[i]):int(lay.A_off[i]) + int(lay.r[i]) * int(lay.d_in[i])].double().numpy()
          .reshape(int(lay.r[i]), int(lay.d_in[i])) for i in m]
    d_out, d_in = int(pr["d_out"]), int(pr["d_in"])
    Us = U0[:d_out * rank].cpu().double().numpy().reshape(d_out, rank)
    Vs = Vt0[:rank * d_in].cpu().double().numpy().reshape(rank, d_in).T
    t0 = time.perf_counter()
    OJ.jd_full(Bs, As, Us, Vs, iters)
    dt = time.perf_counter() - t0
    return {"kind": "oracle", "value": round(1.0 / dt, 4), "unit": "positions/s", "cores": torch.get_num_threads(),
            "sample": f"one position (q, 4096 x 4096) x {len(m)} LoRAs, {iters} steps + Sigma"}


def library_qr_context(dev, stream):
    """Matched library QR on the same modules: torch.linalg.qr (cuSOLVER geqrf, R only)
    on one Qwen2.5-7B-shaped adapter (196 modules, r = 64), B and A^T of each projection
    batched over the 28 layers, against this library's TSQR phases on the same bytes."""
    import torch
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.QWEN25_7B
    lay = synth.fleet_layout(1, M, r=64)
    mods = api.modules_from_layout(lay)
    B = torch.empty(lay.B_total, dtype=torch.float32, device=dev)
    A = torch.empty(lay.A_total, dtype=torch.float32, device=dev)
    synth.fill_fleet(lay, B, A, cfg_id=2, adapter_base=20_000)
    groups = []
    for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
        i0 = p * M.layers
        Bs = torch.stack([B[int(lay.B_off[i0 + l]):int(lay.B_off[i0 + l]) + d_out * 64].view(d_out, 64)
                          for l in range(M.layers)])
        As = torch.stack([A[int(lay.A_off[i0 + l]):int(lay.A_off[i0 + l]) + 64 * d_in].view(64, d_in)
                          for l in range(M.layers)]).transpose(1, 2)
        groups.append((Bs, As))

    def lib_step():
        for Bs, As in groups:
            torch.linalg.qr(Bs, mode="r"); torch.linalg.qr(As, mode="r")

    F = api.alloc_factors(mods, dev)
    ws = api.workspace(lf.lf_tsqr_workspace_size(mods), dev)
    for _ in range(2):
        lib_step(); api.tsqr(mods, B, A, out=F, ws=ws, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record(stream)
    for _ in range(reps):
        lib_step()
    e1.record(stream)
    torch.cuda.synchronize()
    lib_ms = e0.elapsed_time(e1) / reps
    lf.lf_profile_reset(); lf.lf_profile_enable(True)
    for _ in range(reps):
        api.tsqr(mods, B, A, out=F, ws=ws, stream=stream)
    lf.lf_profile_enable(False)
    ph = lf.lf_profile_read()
    # the R factors: integer leaf + root, and the fp64 leaf / Householder routes when they run
    qr_ms = sum(ph[k][0] for k in ("tsqr_gram_i8", "tsqr_gram_i8_root", "tsqr_gram_leaf", "tsqr_householder")
                if k in ph) / reps
    del B, A, F, ws, groups
    torch.cuda.empty_cache()
    return {"sample": "one Qwen2.5-7B-shaped adapter, 196 modules, B and A^T (R only)",
            "library": "torch.linalg.qr (cuSOLVER), per projection batched over 28 layers",
            "library_ms": round(lib_ms, 3), "tsqr_ms": round(qr_ms, 3),
            "library_modules_per_s": round(lay.n / (lib_ms * 1e-3), 1),
            "tsqr_modules_per_s": round(lay.n / (qr_ms * 1e-3), 1),
            "speedup_vs_library": round(lib_ms / qr_ms, 2)}


def cpu_apply_baseline():
    """The oracle's brute-force fp64 apply on the host: layer 0 of the decode workload
    (7 Llama-3-8B projections, 256 tokens, 128 adapters, S-policy ranks), scaled to the
    32-layer step."""
    import torch
    from oracle import apply as OP
    from post_hoc_rank_b200 import api, synth
    from post_hoc_rank_b200 import loraforge as lf

    M = synth.LLAMA3_8B
    n_ad, T = 128, 256
    sig = synth.sigma_tables(n_ad, M, 64, cfg_id=3)
    lay = synth.fleet_layout(n_ad, M, r=64)
    ranks = OA_spectral(sig, lay)
    ranks = ranks.reshape(n_ad, 7, M.layers)
    ids = synth.zipf_ids(T, n_ad, 1.0, (3, 0))
    t_total = 0.0
    for p, (_, d_out, d_in) in enumerate(M.proj_shapes()):
        rk = ranks[:, p, 0].astype(np.int64)
        offA = np.concatenate([[0], np.cumsum(rk * d_in)]); offB = np.concatenate([[0], np.cumsum(rk * d_out)])
        Ap = synth.normal_bf16((int(offA[-1]),), (3, 3, 0, p), std=d_in ** -0.5).float().numpy()
        Bt = synth.normal_bf16((int(offB[-1]),), (3, 4, 0, p), std=d_out ** -0.5).float().numpy()
        x = synth.normal_bf16((T, d_in), (3, 1, 0)).float().numpy()
        y = synth.normal_bf16((T, d_out), (3, 5, 0, p)).float().numpy()
        t0 = time.perf_counter()
        OP.lora_apply(x, y, ids, rk, offA[:-1], offB[:-1], Ap, Bt, 2.0)
        t_total += time.perf_counter() - t0
    step_s = t_total * M.layers
    return {"value": round(T / step_s, 1), "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": "layer 0 of the decode workload (7 projections, 256 tokens), fp64 brute force, "
                      "time x 32 layers"}


def OA_spectral(sig, lay):
    from oracle import allocate as OA
    ranks, _ = OA.spectral_ranks(sig, lay.r, lay.group, 1, 12, 1)
    return np.asarray(ranks)


# ----------------------------------------------------------- CPU baseline
def host_info():
    """The host the CPU baseline ran on: logical CPUs, the ones this process may use,
    the CPU model and whether SMT (more than one thread per core) is on."""
    info = {"os_cpu_count": os.cpu_count(), "usable_cpus": len(os.sched_getaffinity(0))}
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            k, _, v = line.partition(":")
            k, v = k.strip(), v.strip()
            if k == "Model name":
                info["model"] = v
            elif k == "Thread(s) per core":
                info["threads_per_core"] = int(v)
            elif k == "Socket(s)":
                info["sockets"] = int(v)
            elif k == "Core(s) per socket":
                info["cores_per_socket"] = int(v)
    except Exception:
        pass
    info["smt"] = info.get("threads_per_core", 1) > 1
    return info


# Worker side of the oracle's process pool (spawned processes, one BLAS thread each).
# A task names a module of the adapter held in a shared-memory block: its B (d_out x r)
# and A (r x d_in) element offsets.
_SHM = {}


def _pool_init():
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)


def _module_arrays(task):
    from multiprocessing import shared_memory
    name, nb, na, b0, a0, d_out, d_in, r = task[:8]
    if name not in _SHM:
        _SHM.clear()
        _SHM[name] = shared_memory.SharedMemory(name=name)
    buf = _SHM[name].buf
    Bf = np.frombuffer(buf, dtype=np.float32, count=nb)
    Af = np.frombuffer(buf, dtype=np.float32, count=na, offset=4 * nb)
    return Bf[b0:b0 + d_out * r].reshape(d_out, r), Af[a0:a0 + r * d_in].reshape(r, d_in)


def _cpu_spectrum(task):
    from oracle import factor as OF
    B, A = _module_arrays(task)
    return OF.spectrum_factor(B, A)[0]


def _cpu_export(task):
    from oracle import factor as OF
    B, A = _module_arrays(task)
    Bp, Ap = OF.export_factor(B, A, int(task[8]))
    return float(Bp[0, 0])


class OraclePool:
    """The fp64 oracle's fleet route (QR of B and A^T, SVD of R_B R_A^T per module; the
    LoRAForge-S allocation over the adapter; export per module) run by a pool of spawned
    worker processes with one BLAS thread each, on adapters of the same fleet recipe
    generated into shared memory."""

    def __init__(self, workers: int, model=None, n_layers=None):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        import torch
        from post_hoc_rank_b200 import synth
        self.model = model or synth.QWEN25_7B
        self.lay = synth.fleet_layout(1, self.model, r=64, n_layers=n_layers)
        nb, na = int(self.lay.B_total), int(self.lay.A_total)
        self.shm = shared_memory.SharedMemory(create=True, size=4 * (nb + na))
        arr = np.ndarray(nb + na, dtype=np.float32, buffer=self.shm.buf)
        self.Bh = torch.from_numpy(arr[:nb])
        self.Ah = torch.from_numpy(arr[nb:])
        self.nb, self.na = nb, na
        self.workers = workers
        self.pool = mp.get_context("spawn").Pool(workers, initializer=_pool_init)

    def tasks(self, idx):
        L = self.lay
        return [(self.shm.name, self.nb, self.na, int(L.B_off[i]), int(L.A_off[i]), int(L.d_out[i]),
                 int(L.d_in[i]), int(L.r[i])) for i in idx]

    def fill(self, adapter, cfg_id=2):
        from post_hoc_rank_b200 import synth
        synth.fill_fleet(self.lay, self.Bh, self.Ah, cfg_id=cfg_id, adapter_base=adapter)

    def run(self, idx=None):
        """Spectrum, S allocation over the modules idx (the whole adapter by default) and
        export; returns (modules, seconds)."""
        from oracle import allocate as OA
        L = self.lay
        idx = list(range(L.n)) if idx is None else list(idx)
        t = self.tasks(idx)
        t0 = time.perf_counter()
        sig = np.stack(self.pool.map(_cpu_spectrum, t, chunksize=1))
        ranks, _ = OA.spectral_ranks(sig, L.r[idx], np.zeros(len(idx), int), 1, 12, 1)
        self.pool.map(_cpu_export, [tt + (int(k),) for tt, k in zip(t, ranks)], chunksize=1)
        return len(idx), time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()
        del self.Bh, self.Ah
        self.shm.close()
        self.shm.unlink()


def cpu_definition_route(n_repeat=1):
    """The plain definition on the seven sample modules (layer 0 of adapter 0, one per
    projection): dense Delta W = B A and its SVD (numpy, the host's BLAS threads)."""
    import torch
    from post_hoc_rank_b200 import synth
    from oracle import factor as OF
    lay = synth.fleet_layout(1, synth.QWEN25_7B, r=64, n_layers=1)
    Bh = torch.empty(lay.B_total); Ah = torch.empty(lay.A_total)
    synth.fill_fleet(lay, Bh, Ah, cfg_id=2)
    mats = [tuple(t.numpy() for t in synth.module_view(lay, Bh, Ah, i)) for i in range(lay.n)]
    t0 = time.perf_counter()
    for _ in range(n_repeat):
        for Bm, Am in mats:
            OF.spectrum_dense(Bm, Am)
    dt = (time.perf_counter() - t0) / n_repeat
    return {"modules": lay.n, "seconds": round(dt, 2), "modules_per_s": round(lay.n / dt, 3),
            "sample": "layer 0 of adapter 0: q, k, v, o, gate, up, down (dense Delta W = B A, numpy SVD)"}


def cpu_baseline():
    """The oracle on the host cores: a process pool over all usable CPUs on one whole
    adapter (196 modules, the S budget's scope), one worker on a 14-module sample, and
    the dense definition route on the seven sample modules."""
    info = host_info()
    workers = max(1, info["usable_cpus"])
    P = OraclePool(workers)
    try:
        P.fill(0)
        P.run(range(min(P.lay.n, 2 * workers)))         # warm the workers (imports, first BLAS calls)
        n, dt = P.run()
    finally:
        P.close()
    P1 = OraclePool(1)
    try:
        P1.fill(0)
        sample = [p * 28 + l for p in range(7) for l in (0, 1)]
        P1.run(sample[:1])
        n1, dt1 = P1.run(sample)
    finally:
        P1.close()
    return {"value": round(n / dt, 2), "unit": "modules/s", "cores": workers, "kind": "oracle",
            "sample": f"one Qwen2.5-7B-shaped adapter of the same fleet recipe ({n} modules, r=64, S 1/12 over "
                      "the adapter): fp64 QR of B and A^T, SVD of R_B R_A^T, allocation, export; a spawned "
                      f"process pool of {workers} workers with one BLAS thread each",
            "one_core": {"value": round(n1 / dt1, 3), "unit": "modules/s",
                         "sample": "layers 0 and 1 of every projection (14 modules), one worker"},
            "definition_route": cpu_definition_route(),
            "host": info}


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="loraforge", choices=["loraforge", "reference"])
    ap.add_argument("--adapters", type=int, default=N_ADAPTERS)
    ap.add_argument("--e2e-adapters", type=int, default=8)
    ap.add_argument("--no-apply", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-large", action="store_true")
    ap.add_argument("--no-jd", action="store_true")
    ap.add_argument("--jd-only", action="store_true", help="run only the JD-Full workload and print its record")
    ap.add_argument("--large-adapters", type=int, default=1024)
    ap.add_argument("--lora-only", choices=["decode", "decode_per_projection", "prefill_k16", "prefill_r64",
                                            "large_fleet"],
                    help="run only this side-path workload and print its record")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, rank, world)
    if args.jd_only:
        import torch
        from post_hoc_rank_b200 import build as B
        B.build()
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        hbm, _ = peaks()
        print(json.dumps(jd_bench(dev, torch.cuda.current_stream(), hbm, None, with_cpu=not args.no_cpu)))
        return

    if args.lora_only:
        import torch
        from post_hoc_rank_b200 import build as B
        B.build()
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        hbm, _ = peaks()
        stream = torch.cuda.Stream()
        fn = {"decode": lambda: decode_bench(args, dev, stream, hbm),
              "decode_per_projection": lambda: decode_bench(args, dev, stream, hbm, per_layer=False),
              "prefill_k16": lambda: prefill_bench(args, dev, stream, hbm, 16),
              "prefill_r64": lambda: prefill_bench(args, dev, stream, hbm, 64),
              "large_fleet": lambda: large_fleet_bench(args, dev, stream, hbm)}[args.lora_only]
        print(json.dumps(fn()))
        return

    import torch
    from post_hoc_rank_b200 import build as B
    if rank == 0:
        B.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
        pg = dist
        dist.barrier()
        B.build()  # no-op once built by rank 0

    def sync_all():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
            torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    hbm, peak_kind = peaks()
    fr = factor_bench(args, rank, world, dev, sync_all, stream, hbm, peak_kind)
    ms = max_over_ranks(fr["ms"], pg, dev)
    value = whole_job_rate(fr["n"] * args.steps, world, ms)
    ms_step = ms / args.steps

    # dominant kernel roofline
    ph = fr["phases"]
    tot = {k: v[0] for k, v in ph.items()}
    dom = max(tot, key=tot.get)
    per_launch_ms = ph[dom][0] / max(ph[dom][1], 1)
    roof = dominant_roofline(dom, per_launch_ms, fr, hbm, peak_kind, fr["clocks"].get("sm_mhz"))
    step_bytes_2touch = 2 * fr["bytes_in"] + fr["bytes_out"] + fr["bytes_small"]
    step_gbs = step_bytes_2touch / (ms_step * 1e-3) / 1e9

    lora = None
    if not args.no_apply and rank == 0:   # per-GPU side-path figures: rank 0 only
        lora = {"decode": decode_bench(args, dev, stream, hbm, e2e=not args.no_e2e),
                "decode_padded_to_max": decode_bench(args, dev, stream, hbm, "padded"),
                "decode_uncompressed_r64": decode_bench(args, dev, stream, hbm, "r64"),
                "decode_fused_slices": decode_bench(args, dev, stream, hbm, fused=True),
                "decode_per_projection": decode_bench(args, dev, stream, hbm, per_layer=False),
                "decode_sigma_sandwich_r16_diag": sandwich_bench(args, dev, stream, hbm, 16, True),
                "decode_sigma_sandwich_r16_full": sandwich_bench(args, dev, stream, hbm, 16, False),
                "prefill_k16": prefill_bench(args, dev, stream, hbm, 16),
                "prefill_k16_route_per_call": prefill_bench(args, dev, stream, hbm, 16, route_once=False),
                "prefill_k16_fused_slices": prefill_bench(args, dev, stream, hbm, 16, fused=True),
                "prefill_r64": prefill_bench(args, dev, stream, hbm, 64)}
        if rank == 0 and not args.no_cpu:
            lora["decode"]["cpu_baseline"] = cpu_apply_baseline()
    large = None if (args.no_large or rank != 0) else large_fleet_bench(args, dev, stream, hbm)
    libqr = None if (args.no_apply or rank != 0) else library_qr_context(dev, stream)
    jd = None if (args.no_jd or rank != 0) else jd_bench(dev, stream, hbm, fr["clocks"].get("sm_mhz"),
                                                         with_cpu=not args.no_cpu)
    e2e = None
    if not args.no_e2e:
        e = factor_e2e(args, dev, stream, rank)
        if pg is not None:   # every rank compresses its own adapters: whole-job rate over the slowest rank
            e["value"] = whole_job_rate(e["modules"], world, max_over_ranks(1e3 * e["modules"] / e["value"], pg, dev))
        e2e = {"value": round(e["value"], 1), "unit": "modules/s", "h2d_bytes_per_step": e["h2d"],
               "d2h_bytes_per_step": e["d2h"],
               "sample": f"{e['adapters']} adapters ({e['modules']} modules) from pinned host memory"}
    if pg is not None:
        pg.barrier()
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    cpu = None if args.no_cpu else cpu_baseline()
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "modules/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": headline_config(args.adapters, world),
        "roofline": roof,
        "step_hbm": {"algo_bytes_2touch": int(step_bytes_2touch), "achieved_gbs": round(step_gbs, 1),
                     "frac": round(step_gbs / hbm, 4), "peak": hbm},
        "phases_ms_per_step": {k: round(v[0] / args.steps, 3) for k, v in ph.items()},
        "retained_params_frac": round(fr["params_frac"], 4),
        "gpu_launches": int(fr["launches"]),
        "clocks": fr["clocks"],
        "e2e": e2e,
        "lora_path": lora,
        "large_fleet": large,
        "library_qr_context": libqr,
        "jd_full": jd,
        "cpu_baseline": cpu,
        "device_status": fr["status"],
    }
    print(json.dumps(line))
    if pg is not None:
        pg.destroy_process_group()


def headline_config(n_adapters: int, world: int) -> dict:
    """The headline workload's config record (both arms print the same one)."""
    return {"workload": f"factor construction fleet: {n_adapters} adapters x Qwen2.5-7B (196 modules each, "
                        f"{196 * n_adapters} modules per GPU), r=64, LoRAForge-S 1/12 floor 1",
            "l2": "inputs (54.9 GB fp32 per GPU) larger than L2", "parallelism": f"dp{world} (adapters)"}


def reference_arm(args, rank, world):
    """The fp64 oracle, as it stands, on the host cores: each step is one whole adapter of
    the same fleet recipe (196 modules, the scope of the S budget), run by a process pool
    over all usable CPUs with one BLAS thread per worker."""
    if rank != 0:
        return
    info = host_info()
    workers = max(1, info["usable_cpus"])
    P = OraclePool(workers)
    steps = []
    try:
        for s in range(args.warmup + args.steps):
            P.fill(s)
            n, dt = P.run()
            if s >= args.warmup:
                steps.append((n, dt))
    finally:
        P.close()
    n = sum(a for a, _ in steps); t = sum(b for _, b in steps)
    v = n / t
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "modules/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t / len(steps), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": headline_config(args.adapters, 1),
            "cpu_baseline": {"kind": "oracle", "cores": workers, "value": round(v, 2), "unit": "modules/s",
                             "sample": "one whole adapter (196 modules, allocation over the adapter) per step; "
                                       f"spawned process pool of {workers} workers, one BLAS thread each",
                             "host": info},
            "e2e": {"value": round(v, 2), "unit": "modules/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
