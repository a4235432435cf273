"""Benchmark: LLA decode step on B200 -- latent-cache GB/s, token-loop reads/s, HBM roofline.

One step = one decode step of an Ouro-1.4B-shaped layer (T=4 loops, H=16 heads,
d=128, r_k=16 / r_v=32, rho = 21.3, B=64 sequences with context lengths uniform in
[2048, 4096]): the four loop queries of every sequence attend over the latent cache
(lla_decode_attn, absorbed form, all loops fused in one pass), then the finished
token's stacked K/V are encoded into the cache (lla_encode).  Inputs are resident
in HBM before timing; the latent cache (302 MB) is larger than L2 and the timed
loop also rotates over 3 independent cache replicas, so no step reads latents
another recent step left in L2.

Prints ONE JSON line on rank 0.  `python bench.py --gpus N --steps K --warmup W`;
N > 1 runs under torchrun as independent replicas (weak scaling, no collective on
the data path; the barrier and the max-over-ranks reduction are the only
communication).  `--impl reference` times the fp64 CPU oracle instead (the pages
ship no implementation to run); see `cpu_baseline`.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LLA decode latent-cache GB/s & token-loop reads/s (% of HBM roofline) at 1 B200"
WORKLOAD = "ouro1.4b-layer"
SPEC_HBM_GBS = 8000.0
L2_BYTES = 126 * 1000 * 1000
# committed ncu traffic summaries: profiles/<kernel>.<workload>.json, one per (decode kernel,
# workload) captured; the LLA-2D workloads run their own kernel
PROFILE_KERNEL = {"absorb": "decode_absorb_mma", "absorb2d": "decode_absorb_2d", "reconstruct": "decode_reconstruct",
                  "rope": "decode_reconstruct_rope"}
KERNEL_SOURCES = {
    "absorb": ("decode_mma.cu", "mma_common.cuh", "tmap.cuh", "decode_sched.cuh", "decode.cuh", "common.cuh"),
    "absorb2d": ("decode_mma2d.cu", "mma_common.cuh", "tmap.cuh", "decode_sched.cuh", "decode.cuh", "common.cuh"),
    "reconstruct": ("decode_recon_tc.cu", "tc_common.cuh", "mma_common.cuh", "tmap.cuh", "decode_sched.cuh",
                    "decode.cuh", "common.cuh"),
    "rope": ("decode_recon_tc.cu", "tc_common.cuh", "mma_common.cuh", "tmap.cuh", "decode_sched.cuh",
             "decode.cuh", "common.cuh"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--replicas", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--variant", default="absorb", choices=["absorb", "reconstruct"],
                    help="decode read form (the headline uses absorb)")
    ap.add_argument("--phase", default="step", choices=["step", "encode", "residual", "fit"],
                    help="step: decode step (headline); encode: prefill encode of one layer")
    ap.add_argument("--encode-seqs", type=int, default=0,
                    help="--phase encode: sequences of len_hi tokens to encode (default: B)")
    ap.add_argument("--rope", action="store_true",
                    help="faithful read: rotary embedding after reconstruction (reconstruct form, "
                         "query positions = context lengths, half-split pairs, base 10000)")
    ap.add_argument("--decoupled", type=int, default=0,
                    help="absorbed read with a decoupled rotary sub-key of this width (32 or 64) beside "
                         "each latent; queries placed after their contexts")
    ap.add_argument("--window", type=int, default=0,
                    help="hybrid form: W exact window rows per sequence (all in use) besides the "
                         "latents; 0 = latents only")
    ap.add_argument("--layers", type=int, default=0,
                    help="layers one decode step reads (0: every layer of the workload -- a whole-model "
                         "step; the rotary, decoupled and window forms read the first layer only)")
    ap.add_argument("--model-order", action="store_true",
                    help="one decode call per loop (Tq = 1, t = 0..T-1) instead of all loops fused")
    return ap.parse_args()


def rho_label(w) -> str:
    """Exact compression ratio of a workload as a reduced fraction: 2 T d / (r_k + r_v) per
    head per layer, with the H heads folded into one latent for LLA-2D."""
    num = 2 * w.T * w.d * (w.H if w.fold2d else 1)
    den = w.r_k + w.r_v
    g = math.gcd(num, den)
    num, den = num // g, den // g
    return str(num) if den == 1 else f"{num}/{den}"


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def kernel_source_hash(variant="absorb"):
    """Hash of the decode kernel's sources: a profile taken on other sources is stale."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[variant]:
        with open(os.path.join(ROOT, "decode_attention_12_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_path(variant, workload=WORKLOAD):
    return os.path.join(ROOT, "profiles", f"{PROFILE_KERNEL[variant]}.{workload}.json")


def profiled_traffic(units_per_launch, variant="absorb", workload=WORKLOAD):
    """DRAM bytes per launch from the committed ncu summary of this kernel on this workload,
    or None if stale (taken on other sources) or absent."""
    try:
        with open(profile_path(variant, workload)) as f:
            prof = json.load(f)
    except (OSError, ValueError):
        return None
    if prof.get("source_hash") != kernel_source_hash(variant) or prof.get("workload") != workload:
        return None
    per_unit = prof["dram_bytes_per_launch"] / prof["units_per_launch"]
    return per_unit * units_per_launch


def max_over_ranks(value: float, device) -> float:
    """Largest value over all ranks of the default process group (plain value at N = 1)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks: NVML samples during the timed region (read-only queries)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.005):
        self.samples, self.period, self.ok = [], period, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:  # a short timed region: take the samples nearest to it
            inside = sorted(self.samples, key=lambda s: abs(s[0] - 0.5 * (t0 + t1)))[:3]
        mhz = statistics.median(s[1] for s in inside)
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [n for n, b in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside)}


# ---------------------------------------------------------------------------
# the CPU oracle leg (cpu_baseline, and the --impl reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_rate(p, w, Tq, max_seconds, units_per_round=None):
    """Time the fp64 oracle on (b, h) units of the same step; returns (GB/s, info)."""
    import oracle
    import torch

    def f64(t):
        return t.detach().to(torch.float32).cpu().double().numpy()

    q = f64(p["q"])
    cK, cV = f64(p["k"][0]), f64(p["v"][0])
    WK, WV, mK, mV = (f64(p[n][0]) for n in ("W_up_k", "W_up_v", "mu_k", "mu_v"))
    if w.fold2d:  # one folded codec for all heads
        WK, WV, mK, mV = WK[0], WV[0], mK[0], mV[0]
    threads = os.cpu_count() or 1
    all_units = [(b, h) for b in range(w.B) for h in range(w.H)]
    if units_per_round is None:
        units_per_round = len(all_units)
    lens = p["lens"]
    bytes_done, t_spent, rounds, pos = 0, 0.0, 0, 0
    while t_spent < max_seconds or rounds == 0:
        units = [all_units[(pos + i) % len(all_units)] for i in range(units_per_round)]
        pos += units_per_round
        t0 = time.perf_counter()
        oracle.decode_layer("absorb", q, cK, cV, p["starts"], lens, WK, mK, WV, mV, 0, 1.0,
                            fold2d=w.fold2d, units=units, threads=threads)
        t_spent += time.perf_counter() - t0
        # latent bytes this share of the step covers (a folded latent serves all H heads)
        bytes_done += (sum(int(lens[b]) for b, _ in units) * (w.r_k + w.r_v) * w.elem_bytes
                       * w.heads_stored / w.H)
        rounds += 1
    info = {"cores": threads, "units": units_per_round, "rounds": rounds, "seconds": t_spent}
    return bytes_done / t_spent / 1e9, info


def run_reference(args, rank):
    """--impl reference: the oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import torch
    import lla_synth as S
    w = S.WORKLOADS[args.workload]
    p = S.decode_inputs(w, 0, "cpu")
    units = max(1, (w.B * w.H) // 16)          # each step: 1/16 of the layer's (b, h) units
    tot_units = w.B * w.H
    for _ in range(args.warmup):
        oracle_sample_rate(p, w, w.T, 0.0, units_per_round=units)
    t0 = time.perf_counter()
    rates = []
    for _ in range(args.steps):
        r, info = oracle_sample_rate(p, w, w.T, 0.0, units_per_round=units)
        rates.append(r)
    dt = time.perf_counter() - t0
    value = statistics.median(rates)
    S_tot = int(p["lens"].sum())
    step_bytes = S_tot * w.heads_stored * (w.r_k + w.r_v) * w.elem_bytes
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "d": w.d, "r_k": w.r_k, "r_v": w.r_v,
                   "B": w.B, "ctx_len": [w.len_lo, w.len_hi], "Tq": w.T,
                   "sample": f"{units} of {tot_units} (sequence, head) units per step"},
        "token_loop_reads_per_s": value * 1e9 / (step_bytes / (S_tot * w.T)),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": info["cores"], "kind": "oracle",
                         "sample": f"{units} (sequence, head) units x 4 loop queries per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# --phase encode: prefill encode of one layer (write path, tcgen05 for bf16)
# ---------------------------------------------------------------------------
def run_encode_phase(args, dev):
    import torch
    import decode_attention_12_b200 as lla
    import lla_synth as S

    w = S.WORKLOADS[args.workload]
    n_seq = args.encode_seqs or w.B
    n_tok = n_seq * w.len_hi
    # layers encoded per step (a prefill writes every layer's latents): one call covers them all
    nl = min(args.layers, w.L) if args.layers > 0 else w.L
    layers = list(range(nl))
    p = S.decode_inputs(w, layers, dev, lens=[1], Tq=1)
    dims = lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v, int(w.fold2d),
                         lla.F32 if w.dtype == "f32" else lla.BF16)
    bias_k = torch.zeros(w.L, w.heads_stored, w.r_k, device=dev)
    bias_v = torch.zeros(w.L, w.heads_stored, w.r_v, device=dev)
    codec = lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], bias_k=bias_k, bias_v=bias_v,
                           mu_k=p["mu_k"], mu_v=p["mu_v"])
    lla.codec_bias(dims, codec, bias_k, bias_v)
    ck = torch.empty(w.L, w.heads_stored, n_tok, w.r_k, dtype=w.torch_dtype, device=dev)
    cv = torch.empty(w.L, w.heads_stored, n_tok, w.r_v, dtype=w.torch_dtype, device=dev)
    cache = lla.make_cache(ck, cv, n_tok)
    xk = torch.empty(nl, n_tok, w.T, w.H, w.d, dtype=w.torch_dtype, device=dev)
    xv = torch.empty_like(xk)
    for l in layers:  # drawn layer by layer into place (no stacked copy)
        xk[l].copy_(S.draw_encode_tokens(w, l, "k", n_tok, dev))
        xv[l].copy_(S.draw_encode_tokens(w, l, "v", n_tok, dev))
    slot_idx = torch.arange(n_tok, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lla.encode(dims, 0, nl, xk, xv, n_tok, slot_idx, codec, cache, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index or 0).start()
    wall0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    sampler.stop()
    assert lla.status_fetch(None) == 0
    ms = e0.elapsed_time(e1) / args.steps
    e = w.elem_bytes
    bytes_moved = nl * (2 * n_tok * w.H * w.T * w.d * e + n_tok * w.heads_stored * (w.r_k + w.r_v) * e)
    flops = 2.0 * nl * n_tok * w.heads_stored * w.W * (w.r_k + w.r_v)
    peaks, kind = measured_peaks()
    gbs = bytes_moved / (ms * 1e-3) / 1e9
    tfl = flops / (ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "LLA prefill encode GB/s (K and V of every layer)", "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16 x bf16 -> f32" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "tokens": n_tok, "layers": nl, "H": w.H, "T": w.T, "d": w.d,
                   "r_k": w.r_k, "r_v": w.r_v, "rho": rho_label(w), "fold2d": w.fold2d},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": gbs / float(peaks["hbm_gbs"]), "peak_kind": kind},
        "tensor": {"achieved_tflops": tfl, "peak_tflops": float(peaks.get("bf16_tflops", 1590.0)),
                   "frac": tfl / float(peaks.get("bf16_tflops", 1590.0))},
        "clocks": sampler.summary(wall0, wall1),
    }), flush=True)


def run_residual_phase(args, dev):
    """Codec reconstruction residual of held-out tokens (one layer, K and V)."""
    import torch
    import decode_attention_12_b200 as lla
    import lla_synth as S

    w = S.WORKLOADS[args.workload]
    n_seq = args.encode_seqs or w.B
    n_tok = n_seq * w.len_hi
    layer = w.L - 1
    p = S.decode_inputs(w, layer, dev, lens=[1], Tq=1)
    dims = lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v, int(w.fold2d), lla.BF16)
    bias_k = torch.zeros(w.L, w.heads_stored, w.r_k, device=dev)
    bias_v = torch.zeros(w.L, w.heads_stored, w.r_v, device=dev)
    codec = lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], bias_k=bias_k, bias_v=bias_v,
                           W_up_k=p["W_up_k"], W_up_v=p["W_up_v"], mu_k=p["mu_k"], mu_v=p["mu_v"])
    lla.codec_bias(dims, codec, bias_k, bias_v)
    xk = S.draw_encode_tokens(w, layer, "k", n_tok, dev, seed_tag="held-out")
    xv = S.draw_encode_tokens(w, layer, "v", n_tok, dev, seed_tag="held-out")
    outs = [torch.empty(1, n_tok, w.heads_stored, device=dev) for _ in range(4)]
    stream = torch.cuda.current_stream(dev)

    def step():
        lla.codec_residual(dims, layer, 1, xk, xv, n_tok, codec, *outs, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index or 0).start()
    wall0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    e = w.elem_bytes
    # algorithmic bytes: each token's K and V stacks read once, 4 fp32 results written
    bytes_moved = 2 * n_tok * w.H * w.T * w.d * e + 4 * n_tok * w.heads_stored * 4
    # per (token, stored head, axis): 2 W r for c = x W_down and 2 r W for x_hat = c W_up
    flops = 4.0 * n_tok * w.heads_stored * w.W * (w.r_k + w.r_v)
    peaks, kind = measured_peaks()
    gbs = bytes_moved / (ms * 1e-3) / 1e9
    tfl = flops / (ms * 1e-3) / 1e12
    frac = (outs[0] / outs[1]).double()
    print(json.dumps({
        "metric": "LLA codec reconstruction residual GB/s (one layer, K and V)", "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16 x bf16 -> f32, 3xtf32", "data": "synthetic",
        "config": {"workload": w.name, "tokens": n_tok, "H": w.H, "T": w.T, "d": w.d, "r_k": w.r_k,
                   "r_v": w.r_v, "fold2d": w.fold2d},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": gbs / float(peaks["hbm_gbs"]), "peak_kind": kind},
        "tensor": {"achieved_tflops": tfl, "peak_tflops": float(peaks.get("bf16_tflops", 1590.0)),
                   "frac": tfl / float(peaks.get("bf16_tflops", 1590.0)),
                   "note": "algorithmic flop; the tf32 hi/lo rebuild issues 3 MMAs per product"},
        "residual_fraction_k": {"mean": float(frac.mean()), "max": float(frac.max())},
        "clocks": sampler.summary(wall0, wall1),
    }), flush=True)


def run_fit_phase(args, dev):
    """Codec fit (SVD initialisation) of every layer, head and axis from 256 calibration tokens."""
    import torch
    import decode_attention_12_b200 as lla
    import lla_synth as S

    w = S.WORKLOADS[args.workload]
    n = 256
    dims = lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v, int(w.fold2d), lla.BF16)
    Hs, Dp = w.heads_stored, w.d * (w.H if w.fold2d else 1)
    xs = {ax: torch.stack([S.draw_encode_tokens(w, l, ax, n, dev, seed_tag="calib") for l in range(w.L)])
          for ax in ("k", "v")}
    outs = {}
    for ax, r in (("k", w.r_k), ("v", w.r_v)):
        outs[f"W_down_{ax}"] = torch.empty(w.L, Hs, r, w.W, dtype=w.torch_dtype, device=dev)
        outs[f"W_up_{ax}"] = torch.empty(w.L, Hs, w.T, r, Dp, device=dev)
        outs[f"mu_{ax}"] = torch.empty(w.L, Hs, w.T, Dp, device=dev)
    codec = lla.make_codec(**outs)
    wsb = lla.codec_fit_workspace_bytes(dims, w.L, n)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lla.codec_fit(dims, 0, w.L, xs["k"], xs["v"], n, codec, ws, wsb, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ws[:8].zero_()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index or 0).start()
    wall0 = time.perf_counter()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    sampler.stop()
    head = ws[:8].view(torch.int32).cpu().tolist()
    assert head[0] == 0, "eigen-solver did not converge"
    sweeps_per_group = head[1] / (args.steps * 2 * w.L * Hs)
    ms = e0.elapsed_time(e1) / args.steps
    groups = 2 * w.L * Hs
    # algorithmic fp64 flop per group: Gram n^2 W and v_j = Y^T u_j (2 n W r) as FMAs (x2),
    # each Jacobi sweep (n - 1 rounds: 24 flop per 2x2 block of K, 6 per pair of U entries)
    r_avg = (w.r_k + w.r_v) / 2
    flop = groups * (2.0 * n * n * w.W + 2.0 * n * w.W * r_avg
                     + sweeps_per_group * (n - 1) * (24.0 * (n / 2) ** 2 + 6.0 * n * (n / 2)))
    # fp64 peak from unit counts and clocks: 148 SMs x 64 fp64 FMA lanes x 2 flop x 1.965 GHz
    fp64_peak = 148 * 64 * 2 * 1.965e9 / 1e12
    tfl = flop / (ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "LLA codec fit ms per model (SVD initialisation of K and V, every layer and head)",
        "value": ms, "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": False, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "layers": w.L, "heads_stored": Hs, "W": w.W, "r_k": w.r_k,
                   "r_v": w.r_v, "calibration_tokens": n, "groups": groups,
                   "jacobi_sweeps_per_group": sweeps_per_group},
        "roofline": {"bound": "alu", "achieved": tfl, "peak": fp64_peak, "unit": "TFLOP/s",
                     "frac": tfl / fp64_peak, "peak_kind": "fp64 units x clock (derived, not measured)"},
        "clocks": sampler.summary(wall0, wall1),
    }), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import decode_attention_12_b200 as lla
    import lla_synth as S

    if args.phase == "encode":
        run_encode_phase(args, dev)
        return
    if args.phase == "residual":
        run_residual_phase(args, dev)
        return
    if args.phase == "fit":
        run_fit_phase(args, dev)
        return
    w = S.WORKLOADS[args.workload]
    Tq = w.T
    # layers a step reads: a whole-model decode step walks every layer of the workload
    one_layer = bool(args.rope or args.decoupled or args.window)
    nl = 1 if one_layer else (min(args.layers, w.L) if args.layers > 0 else w.L)
    layers = list(range(nl))
    p = S.decode_inputs(w, layers, dev, gap=1)     # one free slot per sequence for the new token
    dims = lla.make_dims(w.T, w.L, w.H, w.d, w.r_k, w.r_v, int(w.fold2d),
                         lla.F32 if w.dtype == "f32" else lla.BF16)
    B, H = w.B, w.H
    lens = p["lens"]
    max_ctx = int(lens.max())
    S_tot = int(lens.sum())
    p["bias_k"] = torch.zeros(w.L, w.heads_stored, w.r_k, device=dev)
    p["bias_v"] = torch.zeros(w.L, w.heads_stored, w.r_v, device=dev)
    codec = lla.make_codec(W_down_k=p["W_down_k"], W_down_v=p["W_down_v"], bias_k=p["bias_k"],
                           bias_v=p["bias_v"], W_up_k=p["W_up_k"], W_up_v=p["W_up_v"],
                           mu_k=p["mu_k"], mu_v=p["mu_v"])
    lla.codec_bias(dims, codec, p["bias_k"], p["bias_v"])
    # independent cache replicas, rotated per step so that no step finds latents in L2: at
    # least enough that the replicas together span twice the 126 MB L2 (small planes, such
    # as the LLA-2D layer's 25 MB, need more than the default 3)
    plane_bytes = (p["k"][0].numel() + p["v"][0].numel()) * p["k"].element_size()  # one layer's latents
    step_plane_bytes = nl * plane_bytes                                           # what a step reads
    R = max(1, args.replicas, math.ceil(2 * L2_BYTES / max(step_plane_bytes, 1)) if args.replicas > 1 else 1)
    if nl > 1 and step_plane_bytes >= 2 * L2_BYTES:
        R = 1  # a whole-model step streams far more than L2 holds: no replica needed
    # (the extra replicas hold the layers a step reads)
    reps = [(p["k"], p["v"])] + [(p["k"][:nl].clone(), p["v"][:nl].clone()) for _ in range(R - 1)]
    caches = [lla.make_cache(k, v, p["slots"]) for k, v in reps]
    # hybrid form: every sequence holds a full window of W exact rows (steady state)
    Wn = max(0, args.window)
    windows = []
    if Wn:
        win = S.window_inputs(w, 0, B, Wn, dev, win_lens=np.full(B, Wn, dtype=np.int32))
        wreps = [(win["win_k"], win["win_v"])] + [(win["win_k"].clone(), win["win_v"].clone())
                                                  for _ in range(R - 1)]
        windows = [lla.make_window(k, v, win["win_len"], Wn, B) for k, v in wreps]
    # the finished tokens' stacked K/V of every layer the step reads: [layers][B][T][H][d]
    x_k = torch.stack([S.draw_encode_tokens(w, l, "k", B, dev, seed_tag="new") for l in layers])
    x_v = torch.stack([S.draw_encode_tokens(w, l, "v", B, dev, seed_tag="new") for l in layers])
    new_slot = (p["seq_start"] + p["ctx_lens"].to(torch.int64)).contiguous()
    if args.rope:
        args.variant = "reconstruct"
    variant = lla.RECONSTRUCT if args.variant == "reconstruct" else lla.ABSORB
    # faithful read: each sequence's query sits right after its context
    rope = lla.make_rope(p["ctx_lens"].clone(), 10000.0, lla.ROPE_HALF) if args.rope else None
    # decode calls of one step: all T loop queries fused (t0 = 0, Tq = T), or in model
    # order one call per loop (t0 = t, Tq = 1) with each loop's queries and outputs in
    # buffers of their own
    loop_calls = [(t, 1) for t in range(w.T)] if args.model_order else [(0, w.T)]
    calls = [(l, t0, n) for l in layers for t0, n in loop_calls]  # (layer, t0, Tq) per decode call
    # decoupled rotary sub-key planes (drawn unrotated: rotation does not change the timing)
    DRn = max(0, args.decoupled)
    if DRn:
        rope = lla.make_rope(p["ctx_lens"].clone(), 10000.0, lla.ROPE_HALF)
        kr0 = S.rope_subkeys(w, 0, p["slots"], DRn, dev).to(w.torch_dtype).unsqueeze(0)
        k_ropes = [kr0] + [kr0.clone() for _ in range(R - 1)]
        q_rope = S.rope_queries(w, B, w.T, DRn, dev)
        q_ropes = [q_rope[:, t0:t0 + n].contiguous() for _, t0, n in calls]
    Tq_call = calls[0][2]
    q_full = p["q"]
    # each layer's queries (the first layer's are the drawn inputs' own)
    q_layers = [q_full] + [S.draw_queries(B, w.T, H, w.d, S.seed_of(w.name, "q", l), dev, w.torch_dtype)
                           for l in layers[1:]]
    qs = [q_layers[l][:, t0:t0 + n].contiguous() for l, t0, n in calls]
    outs = [torch.empty(B, n, H, w.d, dtype=torch.float32, device=dev) for _, _, n in calls]
    lses = [torch.empty(B, n, H, dtype=torch.float32, device=dev) for _, _, n in calls]
    q, out, lse = q_full, outs[0], lses[0]
    if DRn:
        ws_bytes = lla.decode_decoupled_workspace_bytes(dims, B, Tq_call, max_ctx, DRn, args.num_splits)
    else:
        ws_fn = lla.decode_hybrid_workspace_bytes if Wn else lla.decode_workspace_bytes
        ws_bytes = ws_fn(dims, B, Tq_call, max_ctx, variant, args.num_splits)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    splits = lla.decode_num_splits(dims, B, Tq_call, max_ctx, variant, args.num_splits)

    def decode(i, q_in=None, out_buf=None, lse_buf=None):
        for c, (layer, t0, n) in enumerate(calls):
            if DRn:
                lla.decode_attn_decoupled(dims, layer, t0, n, (q_in or qs)[c], caches[i % R], p["seq_start"],
                                          p["ctx_lens"], B, max_ctx, codec, k_ropes[i % R],
                                          q_ropes[c], DRn,
                                          rope, 1.0, (out_buf or outs)[c], (lse_buf or lses)[c], ws, ws_bytes,
                                          num_splits=args.num_splits, stream=stream)
                continue
            if rope is not None:
                lla.decode_attn_rope(dims, layer, t0, n, (q_in or qs)[c], caches[i % R], p["seq_start"],
                                     p["ctx_lens"], B, max_ctx, codec, rope, 1.0, (out_buf or outs)[c],
                                     (lse_buf or lses)[c], ws, ws_bytes, num_splits=args.num_splits,
                                     stream=stream)
                continue
            if Wn:
                lla.decode_attn_hybrid(dims, layer, t0, n, (q_in or qs)[c], caches[i % R], p["seq_start"],
                                       p["ctx_lens"], B, max_ctx, codec, windows[i % R], 1.0,
                                       (out_buf or outs)[c], (lse_buf or lses)[c], ws, ws_bytes,
                                       variant=variant, num_splits=args.num_splits, stream=stream)
                continue
            lla.decode_attn(dims, layer, t0, n, (q_in or qs)[c], caches[i % R], p["seq_start"], p["ctx_lens"], B,
                            max_ctx, codec, 1.0, (out_buf or outs)[c], (lse_buf or lses)[c], ws, ws_bytes,
                            variant=variant, num_splits=args.num_splits, stream=stream)

    def encode(i, xk=x_k, xv=x_v, strm=None):
        lla.encode(dims, 0, nl, xk, xv, B, new_slot, codec, caches[i % R],
                   stream=strm if strm is not None else stream)

    # The encode of the finished tokens writes each sequence's next slot, which no decode
    # of the step reads: it runs on a side stream forked at the step's start and joined at
    # its end, so its CTAs can take the SM slots the decode grid frees.
    s_enc = torch.cuda.Stream(dev)

    def step(i, q_in=None, out_buf=None, lse_buf=None, xk=x_k, xv=x_v, ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record(stream)
        s_enc.wait_stream(stream)
        encode(i, xk=xk, xv=xv, strm=s_enc)
        decode(i, q_in=q_in, out_buf=out_buf, lse_buf=lse_buf)
        if ev_b is not None:
            ev_b.record(stream)
        stream.wait_stream(s_enc)

    # per decode call: prologue + decode + combine for each pass over the latents (32 loop
    # queries per pass, 16 with a rotary sub-key, 64 / H for LLA-2D), reconstruct: one decode
    # pass per 4 loop queries + combine; + the window pass; the encode of K and V is one launch
    if args.variant == "absorb":
        per_pass = 16 if DRn else (max(1, 64 // w.H) if w.fold2d else 32)
        per_call = 3 * -(-Tq_call // per_pass) + (1 if Wn else 0)
    else:
        per_call = -(-Tq_call // 4) + 1 + (1 if Wn else 0)
    launches_per_step = per_call * len(calls) + 1
    # ---- warm-up, then the device-timed region ------------------------------------------------
    sampler = ClockSampler(local).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    t_start.record(stream)
    for i in range(args.steps):
        step(i, ev_a=ev_a[i], ev_b=ev_b[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), dev)
    decode_ms = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    status = lla.status_fetch(ws)
    if status != 0:
        raise RuntimeError(f"device status {status}: {lla.status_string(status)}")

    # latents read per step: one pass over the layer's latents per decode call
    step_bytes = len(calls) * S_tot * w.heads_stored * (w.r_k + w.r_v) * w.elem_bytes
    # hybrid form: each loop query also reads its own loop's exact window keys and values once
    win_bytes = B * H * Tq * Wn * w.d * 2 * w.elem_bytes
    step_bytes += win_bytes
    # decoupled form: each call also reads every token's rotary sub-key once
    step_bytes += len(calls) * S_tot * w.heads_stored * DRn * w.elem_bytes
    ms_step = ms_total / args.steps
    value = world * step_bytes / (ms_step * 1e-3) / 1e9
    reads = world * S_tot * Tq * nl / (ms_step * 1e-3)  # (token, layer, loop) reads per second
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    mean_dec_ms = float(np.mean(decode_ms))
    achieved = step_bytes / (mean_dec_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": peak_kind,
                "traffic": profiled_traffic(S_tot * w.heads_stored,
                                            "absorb2d" if w.fold2d and args.variant == "absorb" else args.variant,
                                            w.name),
                "timed": "one lla_decode_attn call (q_tilde prologue + decode + combine "
                         "kernels), CUDA events per call on the launch stream",
                "algorithmic_bytes_per_launch": step_bytes}
    if args.variant == "reconstruct":
        # the reconstruct form rebuilds K_hat and V_hat on tensor cores: per (token, head,
        # loop) 2 d (r_k + r_v) flop for the rebuild and 4 d for the score and the P.V sum
        flop = nl * S_tot * w.heads_stored * Tq * (2 * w.d * (w.r_k + w.r_v) + 4 * w.d) * (w.H if w.fold2d else 1)
        tf_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1590.0)))
        tfl = flop / (mean_dec_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": tfl, "peak": tf_peak, "unit": "TFLOP/s",
                    "frac": tfl / tf_peak, "peak_kind": peak_kind + " (sustained bf16)",
                    "traffic": profiled_traffic(S_tot * w.heads_stored, "rope" if args.rope else args.variant, w.name),
                    "timed": "one decode call (one reconstruct pass per 4 loop queries + combine), "
                             "CUDA events per call on the launch stream",
                    "algorithmic_flop_per_step": flop, "hbm_gbs": achieved, "hbm_frac": achieved / peak}

    # ---- the dominant kernel alone: CUDA events around the latent-streaming grid ------------------
    # (lla_decode_attn_timed launches the call's grids in order, without programmatic overlap,
    # and records the events on the launch stream immediately around the decode grid)
    kern_ms = None
    if not (Wn or DRn or args.rope):
        n_k = min(args.steps, 200)
        kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
               for _ in range(n_k)]
        for step_ev in kev:  # create the events
            for e_a, e_b in step_ev:
                e_a.record(stream)
                e_b.record(stream)
        torch.cuda.synchronize()
        for i, step_ev in enumerate(kev):
            for c, (layer, t0, n) in enumerate(calls):
                lla.decode_attn_timed(dims, layer, t0, n, qs[c], caches[i % R], p["seq_start"], p["ctx_lens"], B,
                                      max_ctx, codec, 1.0, outs[c], lses[c], ws, ws_bytes, step_ev[c][0],
                                      step_ev[c][1], variant=variant, num_splits=args.num_splits, stream=stream)
            encode(i)
        torch.cuda.synchronize()
        # decode-grid time per step: the sum over the step's calls
        kern_ms = float(np.mean([sum(e_a.elapsed_time(e_b) for e_a, e_b in step_ev) for step_ev in kev]))
        call = {k: roofline[k] for k in ("achieved", "frac", "timed")}
        if roofline["bound"] == "tensor":
            roofline["achieved"] = roofline["algorithmic_flop_per_step"] / (kern_ms * 1e-3) / 1e12
        else:
            roofline["achieved"] = step_bytes / (kern_ms * 1e-3) / 1e9
        roofline["frac"] = roofline["achieved"] / roofline["peak"]
        roofline["timed"] = (f"the latent-streaming decode grid alone (mean of {n_k} steps): CUDA events "
                             "recorded around it on the launch stream by lla_decode_attn_timed, which "
                             "launches the call's grids in order without programmatic overlap")
        roofline["kernel_ms_per_step"] = kern_ms
        roofline["call"] = call  # the whole decode call (prologue + decode + combine), overlapped

    # ---- end to end through the public API with host buffers -------------------------------------
    # Every step copies its inputs (q and the new tokens' K/V) from pinned host memory and
    # reads its results (out, lse) back.  Two device slots let the copy engines move step
    # i+1's inputs and step i-1's results while step i computes (copy streams ordered by
    # events); the timed region runs from before the first input copy to after the last
    # result copy.
    # One packed buffer per direction and slot: the step's inputs (q of every call, the new
    # tokens' K and V) and its results (out and lse of every call) are views into them, so a
    # step issues one host-to-device and one device-to-host copy.
    def packed(tensors, device):
        sizes = [t.numel() * t.element_size() for t in tensors]
        offs = [0]
        for n in sizes:
            offs.append(offs[-1] + ((n + 255) // 256) * 256)
        buf = torch.empty(offs[-1], dtype=torch.uint8, device=device)
        if device == "cpu":
            buf = buf.pin_memory()
        views = [buf[o:o + n].view(t.dtype).view(t.shape) for t, o, n in zip(tensors, offs, sizes)]
        return buf, views

    in_h, in_views_h = packed(list(qs) + [x_k, x_v], "cpu")
    for v, t in zip(in_views_h, list(qs) + [x_k, x_v]):
        v.copy_(t)
    in_d, q_d, xk_d, xv_d = [], [], [], []
    for _ in range(2):
        buf, views = packed(list(qs) + [x_k, x_v], dev)
        in_d.append(buf)
        q_d.append(views[:len(qs)])
        xk_d.append(views[len(qs)])
        xv_d.append(views[len(qs) + 1])
    res_d, out_d, lse_d, res_h = [], [], [], []
    for _ in range(2):
        buf, views = packed(list(outs) + list(lses), dev)
        res_d.append(buf)
        out_d.append(views[:len(outs)])
        lse_d.append(views[len(outs):])
        res_h.append(torch.empty_like(buf, device="cpu").pin_memory())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(1, min(args.steps, 1000))

    def e2e_step(i):
        sl = i % 2
        if i >= 2:
            s_in.wait_event(comp_done[sl])      # step i-2 is done with this input slot
        with torch.cuda.stream(s_in):
            in_d[sl].copy_(in_h, non_blocking=True)
        in_ready[sl].record(s_in)
        stream.wait_event(in_ready[sl])
        if i >= 2:
            stream.wait_event(out_read[sl])    # step i-2's results have left this slot
        step(i, q_in=q_d[sl], out_buf=out_d[sl], lse_buf=lse_d[sl], xk=xk_d[sl], xv=xv_d[sl])
        comp_done[sl].record(stream)
        s_out.wait_event(comp_done[sl])
        with torch.cuda.stream(s_out):
            res_h[sl].copy_(res_d[sl], non_blocking=True)
        out_read[sl].record(s_out)

    for i in range(min(args.warmup, 10)):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    stream.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = world * step_bytes * e2e_steps / (e2e_ms * 1e-3) / 1e9
    h2d = in_h.numel()          # the packed buffers copied per step (256-byte aligned parts)
    d2h = res_h[0].numel()
    status = lla.status_fetch(ws)
    if status != 0:
        raise RuntimeError(f"device status after the end-to-end steps {status}: {lla.status_string(status)}")

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not Wn and not args.rope and not DRn:
        rate, info = oracle_sample_rate(p, w, Tq, args.cpu_seconds, units_per_round=max(1, B * H // 8))
        cpu = {"value": rate, "unit": "GB/s", "cores": info["cores"], "kind": "oracle",
               "sample": f"{info['rounds']} rounds of {info['units']} (sequence, head) units x "
                         f"{Tq} loop queries of this workload, {info['seconds']:.1f} s"}

    units_per_launch = S_tot * w.heads_stored
    clocks = sampler.summary(wall0, wall1)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "storage_dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name + (f"+window{Wn}" if Wn else "") + (f"+ropekey{DRn}" if DRn else ""),
                   "T": w.T, "L": w.L, "L_per_step": nl,
                   "H": H, "d": w.d, "window_rows": Wn, "window_bytes_per_step": win_bytes,
                   "r_k": w.r_k, "r_v": w.r_v, "rho": rho_label(w), "B": B,
                   "ctx_len": [w.len_lo, w.len_hi], "tokens": S_tot, "Tq": Tq_call, "decode_calls_per_step": len(calls),
                   "variant": args.variant + (" + rope" if args.rope else "")
                              + (f" + decoupled rotary sub-key {DRn}" if DRn else ""), "seg_max": splits,
                   "step": (f"{nl} layer(s) x "
                            + (f"{len(loop_calls)} x decode_attn(Tq = 1, one loop each, model order)"
                               if args.model_order else f"decode_attn(all {w.T} loop queries fused)")
                            + (f" with {Wn} exact window rows per sequence (decode_attn_hybrid)" if Wn else "")
                            + f" + encode(B new tokens, {nl} layer(s))"),
                   "l2": (f"{R} rotating cache replicas" if R > 1 else "no replicas (the step streams far more than L2)")
                         + f"; one layer's latents are {plane_bytes / 1e6:.0f} MB, a step reads {nl} layer(s) "
                         f"({R * step_plane_bytes / 1e6:.0f} MB of replicas together, L2 is 126 MB); "
                         f"{step_bytes / 1e6:.0f} MB read per step",
                   "parallelism": f"replicas x{world}"},
        "token_loop_reads_per_s": reads,
        "hbm_frac_of_8tbs_spec": value / world / SPEC_HBM_GBS,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "copies": "pinned host buffers; two device slots; per step one packed input copy "
                          "(q, new K/V) and one packed result copy (out, lse) on their own streams, "
                          "overlapping the neighbouring steps' kernels"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
