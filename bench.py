#!/usr/bin/env python3
"""Benchmark of the MATE block forward pass (MA + TE branches) through libmate.

One step = one full block forward (review pooling, fused in/qkv projection, bidirectional chunked
scan, TESA window attention, fused out projections and branch sum) on the 262,144-token latent grid
(T=256, H=W=32, d_model=1024, 16 Mamba heads x 64, d_state 128, chunk 256, 1024 review tokens, TESA
8 x 128 heads with 4x8x8 windows), bf16 storage with fp32 accumulation.  Steps cycle through layers
0..3, i.e. all four scan orders and both Swin shift phases.  Inputs (512 MiB) exceed the 126 MB L2.

Prints ONE JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle on a bounded sample of the
same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mate_inputs as mi  # noqa: E402

METRIC = "MATE-block tokens/s and ms/block at 1 B200; % of tensor-pipe/HBM roofline"
UNIT = "tokens/s"
WORKLOAD = "bf16_256x32x32"


def flops_per_block(cfg) -> dict:
    """Algorithmic FLOPs of one block (multiply-add = 2), per stage."""
    n, L = cfg.n * cfg.B, (cfg.n + cfg.R) * cfg.B
    nin = cfg.nh * cfg.P + 2 * cfg.N + cfg.nh
    return {
        "in_qkv_proj": 2.0 * n * cfg.d * (nin + 3 * cfg.th * cfg.tp) + 2.0 * cfg.R * cfg.B * cfg.d * nin,
        # chunked scan, both directions: states (2 per chunk-head), C.B^T per chunk, M.x and C.H^T per chunk-head
        "ssd": (L / cfg.Q) * (cfg.nh * (2 * 2 * cfg.Q * cfg.P * cfg.N) + 2 * cfg.Q * cfg.Q * cfg.N) +
               (n / cfg.Q) * cfg.nh * (2 * cfg.Q * cfg.Q * cfg.P + 2 * 2 * cfg.Q * cfg.N * cfg.P),
        "tesa": n * cfg.th * 2 * 2 * (cfg.wt * cfg.wh * cfg.ww) * cfg.tp,
        "out_proj": 2.0 * n * (cfg.nh * cfg.P + cfg.th * cfg.tp) * cfg.d,
    }


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    """{hbm, burst, sustained, source}: HBM GB/s and bf16 TFLOP/s (a burst of one GEMM timed alone, and a
    seconds-long loop under the power cap) from MEASURED_PEAKS.json, else the fallback figures."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm": p["hbm_gbs"], "burst": p["bf16_tflops"], "sustained": p["bf16_tflops_sustained"],
                "source": "measured"}
    except Exception:
        return {"hbm": 6650.0, "burst": 1590.0, "sustained": 1400.0, "source": "fallback"}


def tensor_peak(peaks, region_s, clocks):
    """The bf16 denominator for kernels timed in this run: the sustained figure only when the timed region
    is long enough for the power cap to pull the clock down (at least a second, median SM clock below its
    maximum); otherwise the burst figure."""
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    at_max = sm is not None and smax is not None and sm >= 0.97 * smax
    if region_s < 1.0 or at_max or sm is None:
        why = "timed region under 1 s" if region_s < 1.0 else ("median SM clock at its maximum" if at_max else
                                                               "no clock record")
        return peaks["burst"], f"{peaks['source']} bf16 burst ({why})"
    return peaks["sustained"], f"{peaks['source']} bf16 sustained (timed region {region_s:.1f} s, median SM " \
                               f"clock {sm:.0f} of {smax:.0f} MHz)"


# DRAM bytes per launch measured with ncu (dram__bytes_read.sum + dram__bytes_write.sum), scaled to the
# bench workload as the profile summary explains; valid only while the kernel source is the one captured.
MEASURED_TRAFFIC = {
    "in_projection": {"bytes": 2.675e9, "source": "linear_complexity_video_mate_b200/csrc/gemm_bf16.cuh",
                      "sha1": "8631257f47be87c82d568522e3bc0b600917d489",
                      "profile": "profiles/gemm_bf16_pair_in_projection_bf16_64x32x32.md",
                      "workload": "bf16_256x32x32"},
}


def measured_traffic(kernel, workload):
    """Per-launch DRAM bytes of `kernel` from the committed ncu capture, or None if there is none for
    this workload or the kernel source changed since it was taken."""
    import hashlib
    m = MEASURED_TRAFFIC.get(kernel)
    if m is None or m["workload"] != workload:
        return None
    try:
        with open(os.path.join(ROOT, m["source"]), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != m["sha1"]:
                return None
    except OSError:
        return None
    return m["bytes"]


def kernel_work(cfg, per_dir=False):
    """Algorithmic work per launch of each library kernel at this workload: {kernel: (flops or None, bytes)}.
    FLOPs count a multiply-add as 2 and only the products the method needs (each causal half once, the
    carried-state product C H^T once).  Bytes count each tensor once per kernel that must read or write it
    (inputs, outputs and the scan's stored intermediates: Gram matrix, chunk states, carried states, decay
    tables), nothing for re-reads."""
    es = 2 if cfg.dtype == "bf16" else 4
    B, n, R, d, nh, P, N, Q = cfg.B, cfg.n, cfg.R, cfg.d, cfg.nh, cfg.P, cfg.N, cfg.Q
    nin = nh * P + 2 * N + nh
    NI = nin + 3 * cfg.th * cfg.tp
    KO = nh * P + cfg.th * cfg.tp
    rows, rrows = B * n, B * R
    win = cfg.wt * cfg.wh * cfg.ww
    nVc, nRc = B * -(-n // Q), B * -(-R // Q)
    ldd = 2 * nh
    PN = P * N
    tbl = 2176 * 4 * 2        # decay tables per (video chunk, head): two 128-row tiles
    return {
        "in_projection": (2.0 * rows * d * NI, rows * d * es + rows * NI * es + rows * nh * 4 + NI * d * es),
        "in_projection_review": (2.0 * rrows * d * nin, rrows * d * es + rrows * nin * es + rrows * nh * 4),
        "out_projection": (2.0 * rows * KO * d, rows * KO * es + rows * d * es + d * KO * es),
        "tesa": (4.0 * rows * cfg.th * win * cfg.tp, rows * 3 * cfg.th * cfg.tp * es + rows * cfg.th * cfg.tp * es),
        "review_pool": (None, rows * d * es + rrows * d * es),
        "ssd_gram": (2.0 * nVc * Q * Q * N, rows * 2 * N * es + nVc * Q * Q * 2 + nVc * Q * 4),
        "ssd_state": (2.0 * (2 * nVc + (2 if per_dir else 1) * nRc) * nh * N * P * Q,
                      (rows + rrows) * (nh * P + N) * es + (rows + rrows) * ldd * 4 +
                      (2 * nVc + (2 if per_dir else 1) * nRc) * nh * PN * 4 + nVc * nh * tbl + nVc * Q * 4),
        "ssd_carry": (None, (2 * nVc + (2 if per_dir else 1) * nRc) * nh * PN * 4 + 2 * nVc * nh * 2 * PN * 2),
        "ssd_output": (nVc * nh * (2.0 * Q * Q * P + 2.0 * Q * N * 2 * P),
                       rows * (nh * P + N) * es + nVc * Q * Q * 2 + nVc * Q * 4 + 2 * nVc * nh * 2 * PN * 2 +
                       nVc * nh * tbl + rows * nh * P * es),
        "y_to_grid": (None, 2.0 * rows * nh * P * es),
        "conv_silu": (None, 2.0 * (rows + rrows) * (nh * P + 2 * N) * es),
        "gate_rmsnorm": (None, 3.0 * rows * nh * P * es),
        "pack_weights": (None, 2.0 * (NI * d + d * KO) * es),
        # the DiT block around the mixer
        "ln_modulate": (None, 2.0 * rows * d * es),
        "mlp_up": (2.0 * rows * d * 4 * d, rows * d * es + rows * 4 * d * es + 4 * d * d * es),
        "mlp_down": (2.0 * rows * 4 * d * d, rows * 4 * d * es + 2 * rows * d * es + 4 * d * d * es),
    }


def roofline_table(per, work, hbm_peak, tf_peak):
    """Per traced kernel: launches, ms per launch, and achieved TFLOP/s and GB/s against the peaks."""
    out = {}
    for k, (cnt, tot) in sorted(per.items(), key=lambda kv: -kv[1][1]):
        ms = tot / cnt
        row = {"launches": cnt, "ms_per_launch": ms}
        if k in work:
            fl, by = work[k]
            if fl is not None:
                row["tflops"] = fl / (ms * 1e-3) / 1e12
                row["tensor_frac"] = row["tflops"] / tf_peak
            row["algorithmic_bytes"] = by
            row["gbs"] = by / (ms * 1e-3) / 1e9
            row["hbm_frac"] = row["gbs"] / hbm_peak
        out[k] = row
    return out


def extras_weights(cfg, seed):
    """Random-init weights of the rest of a Mamba2 block: gate projection N(0, 1/d), convolution taps and
    bias U(-1/2, 1/2), norm weight 1 + N(0, 0.1^2)."""
    rng = np.random.default_rng(seed)
    nP, Cx = cfg.nh * cfg.P, cfg.nh * cfg.P + 2 * cfg.N
    return dict(W_z=(rng.standard_normal((nP, cfg.d)) / np.sqrt(cfg.d)).astype(np.float32),
                conv_w=rng.uniform(-0.5, 0.5, (Cx, 4)).astype(np.float32),
                conv_b=rng.uniform(-0.5, 0.5, Cx).astype(np.float32),
                norm_w=(1.0 + 0.1 * rng.standard_normal(nP)).astype(np.float32))


def time_block_variant(M, torch, cfg, wv, X, out, stream, steps):
    """ms per block of a MateBlock built from weights wv (3 warm-up forwards, `steps` timed ones cycling
    the layers) and per-kernel [launches, total ms] from the library trace."""
    blk = M.MateBlock(cfg, M.weights_to_device(wv, cfg))
    nl = 0
    for s in range(4):
        blk.forward(X, s, out)
        nl = max(nl, M.MateBlock.last_launch_count())
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    trace = M.KernelTrace(nl * steps + 16).start()
    e0.record(stream)
    for s in range(steps):
        blk.forward(X, s % 4, out)
    e1.record(stream)
    torch.cuda.synchronize()
    trace.stop()
    per = {}
    for name, kms in trace.read():
        a = per.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += kms
    del blk
    return e0.elapsed_time(e1) / steps, per


def measure_per_direction(M, torch, cfg, w, X, out, stream, base_ms, steps=20):
    """The block with separate backward-scan parameters (dt_bias_b, A_log_b, D_b), timed after the
    headline region: ms per block and the scan kernels' times."""
    rng = np.random.default_rng(4343)
    wp = dict(w)
    wp["dt_bias_b"] = (np.asarray(w["dt_bias"], np.float64) + rng.uniform(-1.0, 1.0, cfg.nh)).astype(np.float32)
    wp["A_log_b"] = rng.uniform(0.0, 1.0, cfg.nh).astype(np.float32)
    wp["D_b"] = rng.standard_normal(cfg.nh).astype(np.float32)
    ms, per = time_block_variant(M, torch, cfg, wp, X, out, stream, steps)
    res = {"ms_per_block": ms, "added_ms": ms - base_ms, "steps": steps}
    for k in ("in_projection", "ssd_state", "ssd_carry", "ssd_output"):
        if k in per:
            res[k + "_ms"] = per[k][1] / per[k][0]
    return res


def measure_extras(M, torch, cfg, w, X, out, stream, base_ms, hbm_peak, steps=20):
    """The block with the full Mamba2 core (convolution + SiLU, gate, gated RMSNorm), timed after the
    headline region: ms per block and the two added kernels against the HBM roofline (algorithmic bytes:
    the convolution reads and writes the x | B | C rows of the video and review rows, the gated norm reads
    y and z and writes y)."""
    we = dict(w)
    we.update(extras_weights(cfg, 4242))
    ms, per = time_block_variant(M, torch, cfg, we, X, out, stream, steps)
    es = 2 if cfg.dtype == "bf16" else 4
    nP, Cx = cfg.nh * cfg.P, cfg.nh * cfg.P + 2 * cfg.N
    nbytes = {"conv_silu": 2.0 * cfg.B * (cfg.n + cfg.R) * Cx * es, "gate_rmsnorm": 3.0 * cfg.B * cfg.n * nP * es}
    res = {"ms_per_block": ms, "added_ms": ms - base_ms, "steps": steps}
    for k, b in nbytes.items():
        if k in per:
            kms = per[k][1] / per[k][0]
            gbs = b / (kms * 1e-3) / 1e9
            res[k] = {"ms_per_launch": kms, "algorithmic_bytes": b, "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm_peak}
    return res


def timing_weights(cfg, seed):
    """Block weights with the workload's initialisation (linear weights N(0, 1/fan_in) rounded to bf16,
    A_log U[0, 1], D N(0, 1), dt_bias 0) from their own seeded stream, without drawing a latent grid."""
    rng = np.random.default_rng(seed)
    lin = lambda o, i: mi.round_to_bf16((rng.standard_normal((o, i)) / np.sqrt(i)).astype(np.float32))
    return dict(W_in=lin(cfg.d_in_proj, cfg.d), dt_bias=np.zeros(cfg.nh, np.float32),
                A_log=rng.uniform(0.0, 1.0, cfg.nh).astype(np.float32), D=rng.standard_normal(cfg.nh).astype(np.float32),
                W_out=lin(cfg.d, cfg.d_inner), W_qkv=lin(3 * cfg.d_attn, cfg.d), W_o=lin(cfg.d, cfg.d_attn))


def measure_scaling(M, torch, stream, headline, headline_name, headline_ms, steps=12):
    """ms per block of every bf16 workload (steps cycling the four layers; seeded Gaussian latents drawn on
    the device, weights from the workload's seeded generator), the headline workload's own number reused,
    and the per-token time of the three d = 1024 clips against the smallest one."""
    out = {}
    for name in ("bf16_16x32x32", "bf16_64x32x32", "bf16_256x32x32", "bf16_2x64x48x48_d2048"):
        cfg = mi.CONFIGS[name]
        if name == headline_name:
            ms = headline_ms
        else:
            blk = M.MateBlock(cfg, M.weights_to_device(timing_weights(cfg, cfg.seed), cfg))
            g = torch.Generator(device="cuda").manual_seed(cfg.seed)
            X = torch.randn((cfg.B, cfg.T, cfg.H, cfg.W, cfg.d), generator=g, device="cuda").to(torch.bfloat16)
            o = torch.empty_like(X)
            for s in range(4):
                blk.forward(X, s, o)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for s in range(steps):
                blk.forward(X, s % 4, o)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            del blk, X, o
        tokens = cfg.B * cfg.n
        out[name] = {"tokens": tokens, "ms_per_block": ms, "ns_per_token": ms * 1e6 / tokens}
    clips = ("bf16_16x32x32", "bf16_64x32x32", "bf16_256x32x32")   # the same block width, 16 to 256 frames
    base = out[clips[0]]["ns_per_token"]
    for name in clips[1:]:
        out[name]["per_token_vs_16x32x32"] = out[name]["ns_per_token"] / base
    # linear in the token count: ms = fixed + slope * tokens (least squares over the three clips); the fit's
    # largest relative residual says how far the measured times are from a straight line
    nt = np.array([out[k]["tokens"] for k in clips], np.float64)
    t = np.array([out[k]["ms_per_block"] for k in clips], np.float64)
    slope, fixed = np.polyfit(nt, t, 1)
    resid = float(np.max(np.abs(fixed + slope * nt - t) / t))
    out["affine_fit"] = {"fixed_ms": float(fixed), "ns_per_token": float(slope * 1e6), "max_rel_residual": resid}
    out["linear_within_15pct"] = resid <= 0.15
    return out


def dit_weights(cfg, dc, seed):
    """Seeded DiT-block weights and conditioning: W_ada N(0, 1/dc), W1 N(0, 1/d), W2 N(0, 1/(4 d)) rounded to
    bf16, biases N(0, 0.1^2), c N(0, 1)."""
    rng = np.random.default_rng(seed)
    d = cfg.d
    bf = lambda a: mi.round_to_bf16(a.astype(np.float32))
    dw = dict(W_ada=bf(rng.standard_normal((6 * d, dc)) / np.sqrt(dc)), b_ada=(0.1 * rng.standard_normal(6 * d)),
              W1=bf(rng.standard_normal((4 * d, d)) / np.sqrt(d)), b1=0.1 * rng.standard_normal(4 * d),
              W2=bf(rng.standard_normal((d, 4 * d)) / np.sqrt(4 * d)), b2=0.1 * rng.standard_normal(d))
    return dw, rng.standard_normal((cfg.B, dc)).astype(np.float32)


def measure_dit(M, torch, cfg, w, X, stream, hbm_peak, tf_peak, steps=12, dc=256):
    """The DiT block around the mixer (adaLN modulation, layer norms, the mixer behind a gated residual, the
    gated GELU MLP of width 4 d) at the headline workload, timed after the headline region: ms per block,
    algorithmic TFLOP/s and the per-kernel fractions.  Weights: W_ada N(0, 1/dc), W1 N(0, 1/d), W2
    N(0, 1/(4 d)), biases N(0, 0.1^2), c N(0, 1), seeded."""
    d = cfg.d
    dw, c = dit_weights(cfg, dc, 777)
    c = torch.as_tensor(c).cuda()
    blk = M.DitBlock(cfg, M.weights_to_device(w, cfg), M.dit_weights_to_device(dw, cfg), dc)
    out = torch.empty_like(X)
    nl = 0
    for s in range(4):
        blk.forward(X, c, s, out)
        nl = max(nl, M.MateBlock.last_launch_count())
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    trace = M.KernelTrace(nl * steps + 16).start()
    e0.record(stream)
    for s in range(steps):
        blk.forward(X, c, s % 4, out)
    e1.record(stream)
    torch.cuda.synchronize()
    trace.stop()
    per = {}
    for name, kms in trace.read():
        a = per.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += kms
    ms = e0.elapsed_time(e1) / steps
    rows = cfg.B * cfg.n
    flops = sum(flops_per_block(cfg).values()) + 16.0 * rows * d * d
    table = roofline_table(per, kernel_work(cfg), hbm_peak, tf_peak)
    del blk
    return {"ms_per_block": ms, "tokens_per_s": rows / (ms * 1e-3), "tflops": flops / (ms * 1e-3) / 1e12,
            "steps": steps, "conditioning_width": dc,
            "kernels": {k: table[k] for k in ("mlp_up", "mlp_down", "ln_modulate", "ada_modulation", "out_projection")
                        if k in table}}


def measure_permute(M, torch, cfg, X, stream, hbm_peak, steps=10):
    """The standalone Rotary Major Scan permute and unpermute (rms_permute / rms_unpermute, every order),
    timed after the headline region against the HBM roofline: each reads and writes the whole grid once."""
    Xp = torch.empty((cfg.B, cfg.n, cfg.d), dtype=X.dtype, device=X.device)
    Xb = torch.empty_like(X)
    for o in range(4):
        M.rms_permute(X, o, cfg, Xp)
        M.rms_unpermute(Xp, o, cfg, Xb)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(steps):
        M.rms_permute(X, s % 4, cfg, Xp)
        M.rms_unpermute(Xp, s % 4, cfg, Xb)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (2 * steps)
    nbytes = 2.0 * X.numel() * X.element_size()
    ok = bool(torch.equal(Xb, X))
    del Xp, Xb
    return {"ms_per_call": ms, "algorithmic_bytes": nbytes, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm_peak, "round_trip_exact": ok}


def measure_tesa_backward(M, torch, cfg, stream, tf_peak, steps=10):
    """TESA's backward pass (tesa_backward: dq | dk | dv from qkv, the forward output and its gradient) at
    the headline workload, timed after the headline region on seeded Gaussian qkv and output gradient;
    shifted and unshifted layers alternate.  Algorithmic work: five 256 x 256 x tp products per window and
    head (dV, dP, dS K, dS^T Q and the recomputed scores)."""
    g = torch.Generator(device="cuda").manual_seed(91)
    a = cfg.th * cfg.tp
    rows = cfg.B * cfg.n
    qkv = torch.randn((rows, 3 * a), generator=g, device="cuda").to(torch.bfloat16)
    dO = torch.randn((rows, a), generator=g, device="cuda").to(torch.bfloat16)
    O = M.tesa_forward(qkv, False, cfg)
    out = torch.empty_like(qkv)
    for s in range(2):
        M.tesa_backward(qkv, O, dO, s % 2 == 1, cfg, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(steps):
        M.tesa_backward(qkv, O, dO, s % 2 == 1, cfg, out)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    win = cfg.wt * cfg.wh * cfg.ww
    flops = 5 * 2.0 * rows * cfg.th * win * cfg.tp
    del qkv, dO, O, out
    return {"ms_per_call": ms, "algorithmic_tflops": flops / 1e12, "tflops": flops / (ms * 1e-3) / 1e12,
            "frac_of_bf16_peak": flops / (ms * 1e-3) / 1e12 / tf_peak, "steps": steps,
            "forward_tesa_ms": None}


def profile_run(M, torch, cfg, w, X, out):
    """Every kernel of the path a few times, untimed, for an ncu capture to select launches from: the
    block over the four layers, the block with the Mamba2 extras, the DiT block, and the standalone
    permute and unpermute."""
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    for s in range(4):
        blk.forward(X, s, out)
    del blk
    we = dict(w)
    we.update(extras_weights(cfg, 4242))
    blk = M.MateBlock(cfg, M.weights_to_device(we, cfg))
    for s in range(2):
        blk.forward(X, s, out)
    del blk
    dw, c = dit_weights(cfg, 256, 777)
    blk = M.DitBlock(cfg, M.weights_to_device(w, cfg), M.dit_weights_to_device(dw, cfg), 256)
    blk.forward(X, torch.as_tensor(c).cuda(), 1, out)
    del blk
    g = torch.Generator(device="cuda").manual_seed(91)
    a = cfg.th * cfg.tp
    qkv = torch.randn((cfg.B * cfg.n, 3 * a), generator=g, device="cuda").to(torch.bfloat16)
    dO = torch.randn((cfg.B * cfg.n, a), generator=g, device="cuda").to(torch.bfloat16)
    O = M.tesa_forward(qkv, True, cfg)
    M.tesa_backward(qkv, O, dO, True, cfg)
    del qkv, dO, O
    Xp = torch.empty((cfg.B, cfg.n, cfg.d), dtype=X.dtype, device=X.device)
    for o in range(2):
        M.rms_permute(X, o, cfg, Xp)
        M.rms_unpermute(Xp, o, cfg, out)
    torch.cuda.synchronize()
    print(json.dumps({"profile_run": cfg.name, "status": M.device_status()}), flush=True)


def oracle_sample_cfg(cfg, frames):
    """The workload restricted to its first `frames` frames, review tokens scaled in proportion."""
    import dataclasses
    R = max(16, cfg.R * frames // cfg.T // 16 * 16)
    return dataclasses.replace(cfg, T=frames, R=R, name=f"{cfg.name}[T={frames}]")


def run_oracle_sample(cfg, frames, steps, warmup):
    from oracle import mate_oracle as O
    scfg = oracle_sample_cfg(cfg, frames)
    w = mi.make_inputs(scfg)
    for s in range(warmup):
        O.mate_forward(w["X"], w, scfg, s % 4)
    t0 = time.perf_counter()
    for s in range(steps):
        O.mate_forward(w["X"], w, scfg, s % 4)
    dt = (time.perf_counter() - t0) / max(steps, 1)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    tokens = scfg.B * scfg.n
    return tokens / dt, dt, cores, scfg


# ------------------------------------------------------------------------------ multi-rank plumbing
# One process per GPU, each running its own block on its own seeded inputs (replicas: the block has no
# data-path collective); the job's time is the slowest rank's.

def replica_seed(cfg, rank: int) -> int:
    return cfg.seed + 1000 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of x over all ranks (x itself when world == 1)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job tokens/s: the tokens every rank processed in one step over the slowest rank's step time."""
    return tokens_per_rank * world / (ms * 1e-3)


def reference_arm(args, rank):
    if rank != 0:
        return 0
    cfg = mi.CONFIGS[args.config]
    value, dt, cores, scfg = run_oracle_sample(cfg, args.oracle_frames, args.steps, args.warmup)
    sample = (f"fp64 numpy oracle, {args.config} restricted to its first {scfg.T} frames "
              f"({scfg.B * scfg.n} tokens, R={scfg.R}), layers cycling 0..3")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.config, "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--oracle-frames", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the full-Mamba2-block side measurement")
    ap.add_argument("--no-scaling", action="store_true", help="skip the per-workload ms/block side measurement")
    ap.add_argument("--profile-run", action="store_true",
                    help="run every kernel of the path a few times without timing (for an ncu capture) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, rank)

    import torch
    import torch.distributed as dist
    from linear_complexity_video_mate_b200 import mate as M

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    cfg = mi.CONFIGS[args.config]
    w = mi.make_inputs(cfg, seed=replica_seed(cfg, rank))   # every rank runs its own block (weak scaling)
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    X = torch.as_tensor(w["X"]).to(device="cuda", dtype=torch.bfloat16)
    out = torch.empty_like(X)
    stream = torch.cuda.current_stream()
    if args.profile_run:
        profile_run(M, torch, cfg, w, X, out)
        return 0

    def barrier():
        if world > 1:
            dist.barrier()

    launches_per_step = 0
    for s in range(max(args.warmup, 4)):   # every layer at least once: the trace is sized by the largest
        blk.forward(X, s % 4, out)
        launches_per_step = max(launches_per_step, M.MateBlock.last_launch_count())
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    trace = M.KernelTrace(launches_per_step * args.steps + 16).start()   # events around every launch
    e0.record(stream)
    for s in range(args.steps):
        blk.forward(X, s % 4, out)
    e1.record(stream)
    torch.cuda.synchronize()
    trace.stop()
    barrier()
    clocks = sampler.stop()
    records = trace.read()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, "cuda")
    status = M.device_status()

    # per-kernel device times over the timed region; the roofline names the kernel with the largest total
    per = {}
    for name, kms in records:
        a = per.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += kms
    traced_ms = sum(a[1] for a in per.values())
    kernels = {k: {"launches": n, "ms_per_launch": t / n, "share": t / traced_ms}
               for k, (n, t) in sorted(per.items(), key=lambda kv: -kv[1][1])}
    work = kernel_work(cfg)
    peaks = measured_peaks()
    hbm_peak = peaks["hbm"]
    tf_peak, tf_src = tensor_peak(peaks, ms * args.steps * 1e-3, clocks)
    peak_src = tf_src
    table = roofline_table(per, work, hbm_peak, tf_peak)
    # the roofline names the kernel with the largest share of the traced time; a kernel with a FLOP model
    # is measured against the tensor pipe, the others against HBM
    dom = max((k for k in per if k in work), key=lambda k: per[k][1])
    dom_ms = per[dom][1] / per[dom][0]
    dflops, dbytes = work[dom]
    if dflops is not None:
        bound, runit, achieved, dpeak = "tensor", "TFLOP/s", dflops / (dom_ms * 1e-3) / 1e12, tf_peak
    else:
        bound, runit, achieved, dpeak = "hbm", "GB/s", dbytes / (dom_ms * 1e-3) / 1e9, hbm_peak
        peak_src = f"{peaks['source']} HBM copy bandwidth"

    # end to end through the host-buffer entry points: pinned host X in, pinned host Out back, every step;
    # the headline uses the pipelined calls (each call's input copy overlaps the previous call's output
    # copy), the one-call-at-a-time form is reported beside it
    xh = X.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()

    def e2e(pipelined):
        for s in range(3):
            blk.forward_host(xh, s, oh, pipelined=pipelined)
        M.MateBlock.flush_host()
        torch.cuda.synchronize()
        barrier()
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for s in range(args.e2e_steps):
            blk.forward_host(xh, s % 4, oh, pipelined=pipelined)
        M.MateBlock.flush_host()   # every step's output has reached the host before the end event
        h1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(h0.elapsed_time(h1) / args.e2e_steps, world, "cuda")
    e2e_ms = e2e(True)
    e2e_serial_ms = e2e(False)
    nbytes = X.numel() * X.element_size()

    # scan locality of the workload's grid (outside the timed region): mean sequence distance of
    # grid-adjacent tokens per index map, computed by the library's kernel
    locality = {}
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0.record(stream)
    for kind, name in enumerate(M.LOCALITY_MAPS):
        if kind == 5 and (cfg.H != cfg.W or cfg.H & (cfg.H - 1) or cfg.T % cfg.H):
            continue
        sm, npairs, mx = M.scan_locality(cfg.T, cfg.H, cfg.W, kind)
        locality[name] = {"mean": sm / npairs, "max": mx}
    l1.record(stream)
    torch.cuda.synchronize()
    locality["pairs"] = npairs
    locality["ms_all_maps"] = l0.elapsed_time(l1)

    # side measurements, outside the headline region: the block with the rest of the Mamba2 block, and with
    # separate backward-scan parameters; a failure is reported in the line instead of ending the run
    extras = per_direction = dit = permute = tesa_bwd = None
    try:
        permute = measure_permute(M, torch, cfg, X, stream, hbm_peak)
    except Exception as e:  # noqa: BLE001
        permute = {"error": f"{type(e).__name__}: {e}"}
    if not args.no_extras:
        try:
            tesa_bwd = measure_tesa_backward(M, torch, cfg, stream, tf_peak)
            if "tesa" in per:
                tesa_bwd["forward_tesa_ms"] = per["tesa"][1] / per["tesa"][0]
        except Exception as e:  # noqa: BLE001
            tesa_bwd = {"error": f"{type(e).__name__}: {e}"}
        try:
            dit = measure_dit(M, torch, cfg, w, X, stream, hbm_peak, tf_peak)
        except Exception as e:  # noqa: BLE001
            dit = {"error": f"{type(e).__name__}: {e}"}
        try:
            extras = measure_extras(M, torch, cfg, w, X, out, stream, ms, hbm_peak)
        except Exception as e:  # noqa: BLE001
            extras = {"error": f"{type(e).__name__}: {e}"}
        try:
            per_direction = measure_per_direction(M, torch, cfg, w, X, out, stream, ms)
        except Exception as e:  # noqa: BLE001
            per_direction = {"error": f"{type(e).__name__}: {e}"}

    # linear scaling in token count: ms per block of every workload in the same run (outside the headline
    # region), the 65,536-token clip over its four layers
    scaling = None
    if not args.no_scaling:
        try:
            scaling = measure_scaling(M, torch, stream, args.config, cfg.name, ms)
            torch.cuda.empty_cache()
        except Exception as e:  # noqa: BLE001
            scaling = {"error": f"{type(e).__name__}: {e}"}

    tokens_per_step = cfg.B * cfg.n
    value = job_value(tokens_per_step, world, ms)
    fl = flops_per_block(cfg)
    total_flops = sum(fl.values())
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian latents, random-init weights)",
        "config": {"workload": args.config, "B": cfg.B, "T": cfg.T, "H": cfg.H, "W": cfg.W, "d_model": cfg.d,
                   "tokens_per_block": tokens_per_step, "review_tokens": cfg.R, "layers": "cycling 0..3",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs (512 MiB) larger than L2"},
        "ms_per_block": ms,
        "block_tflops": total_flops / (ms * 1e-3) / 1e12,
        "block_frac_of_bf16_peak": total_flops / (ms * 1e-3) / 1e12 / tf_peak,
        "scaling_mode": "weak",
        "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": dpeak, "unit": runit,
                     "frac": achieved / dpeak, "traffic": measured_traffic(dom, args.config),
                     "traffic_unit": "bytes per launch", "peak_source": peak_src,
                     "algorithmic": dflops if dflops is not None else dbytes,
                     "kernel_ms": dom_ms, "launches_timed": per[dom][0],
                     "timing": "CUDA events around each launch inside the timed region (library trace)"},
        "kernels": kernels,
        "kernel_roofline": {"peaks": {"tensor_tflops": tf_peak, "hbm_gbs": hbm_peak, "tensor_source": tf_src},
                            "per_kernel": table},
        "scaling": scaling,
        "e2e": {"value": job_value(tokens_per_step, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": nbytes,
                "d2h_bytes_per_step": nbytes, "ms_per_step": e2e_ms, "api": "mate_forward_host_pipelined",
                "one_call_at_a_time_ms_per_step": e2e_serial_ms},
        "gpu_launches": len(records),
        "scan_locality": locality,
        "mamba_extras": extras,
        "per_direction_scan": per_direction,
        "dit_block": dit,
        "rms_permute": permute,
        "tesa_backward": tesa_bwd,
        "clocks": clocks,
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        value_c, dt_c, cores, scfg = run_oracle_sample(cfg, args.oracle_frames, 1, 0)
        line["cpu_baseline"] = {"value": value_c, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"fp64 oracle on {args.config} restricted to {scfg.T} frames "
                                          f"({scfg.n} tokens, R={scfg.R}), one block, layer 0"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
