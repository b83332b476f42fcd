"""KDA throughput on B200: tokens/s and fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is the production training pass of the recurrence: the chunked
prefill forward (which also stores the chunk states) and the chunked
backward that reuses them, on B=2, H=HV=96, T=4096, K=V=128, bf16 inputs,
fp32 state (all hot-path kernels except the decode step).  The prefill-only
workloads and the batched decode step are timed the same way and reported
under "paths".  A token is one (batch, time) position with all value heads.

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the per-GPU workload (independent batches, no data-path collective): weak
scaling; the timed region is bracketed by barriers and the slowest rank's
device time is reported.

``--impl reference`` times the float64 CPU oracle (the only reference this
method has) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from gated_delta_rule_66_b200.inputs import BY_NAME, make_erase_inputs, make_inputs, make_raw_inputs  # noqa: E402

HEADLINE = "fwdbwd"
PATHS = ("twin", "prefill_gqa", "fwdbwd", "decode", "prefill_prep", "decode_token", "erase")
# paths from the raw projections (fused preparation): workload they take their sizes from
PREP_PATHS = {"prefill_prep": "prefill_gqa", "decode_token": "decode"}
CONV_W = 4  # the host model's short-convolution width
METRIC = "KDA tokens/s at 1 B200 (prefill fwd, fwd+bwd, decode) + % of roofline"
L2_BYTES = 126 * 2 ** 20


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ---------------------------------------------------------------------------- algorithmic work

def esize(w):
    return 4 if w.dtype == "fp32" else 2


def algorithmic_bytes(w, kind):
    """Bytes a kernel must move at least once (inputs read, outputs written)."""
    B, T, H, HV, K, V, e = w.B, w.T, w.H, w.HV, w.K, w.V, esize(w)
    state = B * HV * K * V * 4
    if kind == "decode":
        return 2 * state + B * (2 * H * K * e + HV * V * e + HV * K * 4 + HV * 4 + HV * V * e)
    fwd_in = B * T * (2 * H * K * e + HV * V * e + HV * K * 4 + HV * 4)
    fwd_out = B * T * HV * V * e + state                      # o, S_T
    s0 = state if w.s0_std > 0 else 0
    if kind == "fwd":
        return fwd_in + fwd_out + s0
    # backward: reads the forward inputs and dO, writes dq, dk, dv, dg, dbeta, dS0
    bwd = fwd_in + s0 + B * T * HV * V * e + B * T * (2 * H * K * e + HV * V * e + HV * K * 4 + HV * 4) + state
    if kind == "bwd":
        return bwd
    return fwd_in + fwd_out + s0 + bwd


def prep_algorithmic_bytes(w, kind):
    """Bytes of the raw-projection paths: prefill_prep reads q, k, v, z, the
    output gate (input dtype) and the beta logits, writes o and S_T;
    decode_token also reads and writes the state and the convolution window
    (fp32) and reads the convolution weights."""
    B, T, H, HV, K, V, e = w.B, w.T, w.H, w.HV, w.K, w.V, esize(w)
    state = B * HV * K * V * 4
    per_tok = 2 * H * K * e + HV * V * e + HV * K * e + HV * V * e + HV * 4 + HV * V * e
    small = HV * 4 + HV * K * 4  # A_log, dt_bias
    if kind == "prefill_prep":
        return B * T * per_tok + state + small
    Cn = 2 * H * K + HV * V
    return B * per_tok + 2 * state + 2 * B * Cn * CONV_W * 4 + Cn * CONV_W * 4 + small


def chunk_flops_per_head_token(K, V, C):
    """Flops of the chunked form per (head, token): three K x V state
    contractions (residual, readout, carry), the two C x C x K interaction
    products, and the C x C x V solve and readout products (dense tiles)."""
    return 2 * (3 * K * V + 2 * C * K + 2 * C * V)


# The chunked backward's contractions per (head, token), as a multiple of the
# forward's: the state-gradient products, the recomputed residuals, the
# gradient products summed over the value columns and the interaction terms
# (dense tiles) come to about 2.5 times the forward's.
BWD_FLOPS_RATIO = 2.5
NOMINAL_HBM_GBS = 7700.0  # B200 HGX nominal HBM3e bandwidth, for context beside the measured copy peak


def tf32_peak_tflops(peaks):
    """Dense tf32 tensor peak: the measured dense bf16 peak times the nominal
    tf32 : bf16 ratio (1.1 : 2.25 PFLOP/s, i.e. one half)."""
    return peaks["bf16_tflops"] * 0.5


def two_rooflines(byts, flops, seconds, peaks):
    """Both fractions of a chunked call (HBM bytes and tf32 tensor flops) and
    the binding one (the bound whose ideal time is longer)."""
    hbm, tpk = peaks["hbm_gbs"], tf32_peak_tflops(peaks)
    gbs, tfs = byts / seconds / 1e9, flops / seconds / 1e12
    t_hbm, t_tc = byts / (hbm * 1e9), flops / (tpk * 1e12)
    hbm_part = {"achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm, "algorithmic_bytes": byts,
                "peak_source": f"{peaks['source']} copy bandwidth"}
    tc_part = {"achieved": tfs, "peak": tpk, "unit": "TFLOP/s", "frac": tfs / tpk, "algorithmic_flops": flops,
               "peak_source": f"{peaks['source']} dense bf16 x 1/2 (nominal tf32 : bf16 ratio)"}
    top = dict(tc_part, bound="tensor") if t_tc > t_hbm else dict(hbm_part, bound="hbm")
    top["hbm"], top["tensor"] = hbm_part, tc_part
    return top


# ---------------------------------------------------------------------------- GPU arm

class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _flush_l2(buf):
    buf.add_(1)


_HOST_INPUTS = {}  # workload name -> its host inputs, shared with the oracle sampler


def host_inputs(w):
    if w.name not in _HOST_INPUTS:
        _HOST_INPUTS[w.name] = make_inputs(w, with_do=(w.path == "fwdbwd"))
    return _HOST_INPUTS[w.name]


def gpu_prep_path(kda, name, steps, warmup, rank_barrier):
    """Times a raw-projection path: the prefill with the preparation and
    output gate fused (kda_fwd_prep, production prefill geometry) or the
    decode token (kda_decode_token: convolution step, preparation,
    recurrence, output gate; production decode geometry)."""
    w = BY_NAME[PREP_PATHS[name]].with_sizes(name=name, s0_std=0.0)  # (decode_token draws its own state)
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    if name == "prefill_prep":
        r = make_raw_inputs(w)
        d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in r.items()}
        ws = torch.empty(kda.prep_workspace_bytes(w.B, w.T, w.H, w.HV, w.K, w.V, w.torch_dtype), dtype=torch.uint8,
                         device=dev)

        def step():
            kda.fwd_prep(d["q"], d["k"], d["v"], d["z"], d["A_log"], d["dt_bias"], d["beta_logit"], scale=w.scale,
                         out_gate=d["og"], workspace=ws)
        tokens, launches = w.B * w.T, 4
        kernel = "kda_fwd_prep (kda_prep_gate_kernel + kda_fwd_intra_tc_kernel<1> + kda_fwd_state_tc_kernel<1> + kda_out_gate4_kernel, one call)"
        flush = None
    else:
        r = make_raw_inputs(w.with_sizes(T=1), conv_width=CONV_W)
        d = {n: (t[:, 0].contiguous().to(dev) if isinstance(t, torch.Tensor) and t.dim() >= 3 and n != "conv_state"
                 else (t.to(dev) if isinstance(t, torch.Tensor) else t)) for n, t in r.items()}
        S = torch.randn(w.B, w.HV, w.K, w.V, generator=torch.Generator().manual_seed(3)).mul_(0.02).to(dev)
        flush = None  # state and windows (1.8 GB) exceed L2

        def step():
            kda.decode_token(d["q"], d["k"], d["v"], d["conv_w"], d["conv_state"], d["z"], d["A_log"],
                             d["dt_bias"], d["beta_logit"], S, scale=w.scale, out_gate=d["og"])
        tokens, launches = w.B, 1
        kernel = "kda_decode_token_kernel"
    for _ in range(warmup):
        if flush is not None:
            _flush_l2(flush)
        step()
    torch.cuda.synchronize()
    rank_barrier()
    if flush is None:  # inputs larger than L2: the steps back to back
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / steps
    else:  # L2 flushed before every step, outside the timed span of the step
        spans = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e_s, e_e in spans:
            _flush_l2(flush)
            e_s.record(stream)
            step()
            e_e.record(stream)
        torch.cuda.synchronize()
        ms = sum(e_s.elapsed_time(e_e) for e_s, e_e in spans) / steps
    byts = prep_algorithmic_bytes(w, name)
    hbm = load_peaks()["hbm_gbs"]
    res = {"workload": name, "ms_per_step": ms, "tokens_per_step": tokens, "launches_per_step": launches,
           "l2": "inputs > L2", "calls": {"kernel_ms": ms}, "e2e_ms": None,
           "roofline": {"bound": "hbm", "kernel": kernel, "achieved": byts / (ms * 1e-3) / 1e9, "peak": hbm,
                        "unit": "GB/s", "frac": byts / (ms * 1e-3) / 1e9 / hbm, "algorithmic_bytes": byts}}
    return res, w


def gpu_erase_path(kda, steps, warmup, rank_barrier):
    """Times the asymmetric erase/write variant (kda_fwd_erase) on its
    workload: B=1, T=8192, 32 query heads over 8 state heads, K=64, V=128."""
    w = BY_NAME["erase"]
    d = {n: (None if t is None else t.cuda()) for n, t in make_erase_inputs(w).items()}
    stream = torch.cuda.current_stream()
    flush = None  # the inputs (151 MB) exceed L2

    def step():
        kda.fwd_erase(d["q"], d["k"], d["e"], d["z"], d["g"], scale=w.scale)
    for _ in range(warmup):
        if flush is not None:
            _flush_l2(flush)
        step()
    torch.cuda.synchronize()
    rank_barrier()
    if flush is None:  # inputs larger than L2: the steps back to back
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / steps
    else:  # L2 flushed before every step, outside the timed span of the step
        spans = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e_s, e_e in spans:
            _flush_l2(flush)
            e_s.record(stream)
            step()
            e_e.record(stream)
        torch.cuda.synchronize()
        ms = sum(e_s.elapsed_time(e_e) for e_s, e_e in spans) / steps
    e = esize(w)
    byts = (w.B * w.T * (w.H * w.K * e + 2 * w.HV * w.K * e + w.HV * w.V * e + w.HV * w.K * 4 + w.H * w.V * e)
            + w.B * w.HV * w.K * w.V * 4)
    hbm = load_peaks()["hbm_gbs"]
    res = {"workload": "erase", "ms_per_step": ms, "tokens_per_step": w.B * w.T, "launches_per_step": 1,
           "l2": "inputs > L2", "calls": {"kernel_ms": ms}, "e2e_ms": None,
           "roofline": {"bound": "hbm", "kernel": "kda_fwd_chunk_kernel<ERASE> (CUDA-core path)",
                        "achieved": byts / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                        "frac": byts / (ms * 1e-3) / 1e9 / hbm, "algorithmic_bytes": byts}}
    return res, w


def gpu_path(kda, name, steps, warmup, rank_barrier, shrink=None):
    """Times one workload on this rank's GPU.  Returns a result dict."""
    if name in PREP_PATHS:
        return gpu_prep_path(kda, name, steps, warmup, rank_barrier)
    if name == "erase":
        return gpu_erase_path(kda, steps, warmup, rank_barrier)
    w = BY_NAME[name]
    if shrink:  # a smaller batch and length of the same workload (profiler captures only)
        w = w.with_sizes(name=f"{name}_B{shrink[0]}_T{shrink[1]}", B=shrink[0], T=shrink[1])
    inp = host_inputs(w)
    dev = torch.device("cuda")
    d = {n: (None if t is None else t.to(dev)) for n, t in inp.items()}
    flush = None
    in_bytes = sum(t.numel() * t.element_size() for t in inp.values() if t is not None)
    if in_bytes < 2 * L2_BYTES:
        flush = torch.zeros(256 * 2 ** 20 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    launches_per_step = 0
    ws = None

    if w.path == "fwd":
        def step():
            kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"])
        # chunk-parallel kernel + state pass (tensor-core or CUDA-core path, with scratch)
        launches_per_step = 2
        tokens = w.B * w.T
    elif w.path == "fwdbwd":
        ws = torch.empty(kda.workspace_bytes("bwd", w.B, w.T, w.H, w.HV, w.K, w.V), dtype=torch.uint8,
                         device=dev)

        def step():
            kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"],
                    workspace=ws)
            kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], scale=w.scale,
                    initial_state=d["S0"], workspace=ws, states_from_fwd=True)
        # kda_fwd: chunk-parallel kernel + state pass; kda_bwd: state gradients,
        # gradient products, assembly (each launched twice when the heads leave
        # a partial last wave of SMs), +2 group sums when HV > H
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        heads = w.B * w.HV
        launches_per_step = 2 + (6 if heads > sms and heads % sms else 3) + (2 if w.HV > w.H else 0)
        tokens = w.B * w.T
    else:
        S = d["S"]

        def step():
            kda.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, scale=w.scale)
        launches_per_step = 1
        tokens = w.B

    for _ in range(warmup):
        if flush is not None:
            _flush_l2(flush)
        step()
    torch.cuda.synchronize()
    rank_barrier()
    if flush is None:  # inputs larger than L2: the steps back to back
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / steps
    else:  # L2 flushed before every step, outside the timed span of the step
        spans = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e_s, e_e in spans:
            _flush_l2(flush)
            e_s.record(stream)
            step()
            e_e.record(stream)
        torch.cuda.synchronize()
        ms = sum(e_s.elapsed_time(e_e) for e_s, e_e in spans) / steps
    res = {"workload": name, "ms_per_step": ms, "tokens_per_step": tokens,
           "launches_per_step": launches_per_step, "l2": "flushed" if flush is not None else "inputs > L2"}

    # per-call kernel timing (each C-ABI call below is the launch(es) named)
    calls = {}
    if w.path in ("fwd", "decode"):
        calls["kernel_ms"] = ms  # one kernel per step
    else:
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        t_f, t_b = 0.0, 0.0
        for _ in range(steps):
            e[0].record(stream)
            kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"],
                    workspace=ws)
            e[1].record(stream)
            kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], scale=w.scale,
                    initial_state=d["S0"], workspace=ws, states_from_fwd=True)
            e[2].record(stream)
            torch.cuda.synchronize()
            t_f += e[0].elapsed_time(e[1])
            t_b += e[1].elapsed_time(e[2])
        calls["fwd_ms"] = t_f / steps
        calls["bwd_ms"] = t_b / steps
    res["calls"] = calls

    # End to end through the public API with host buffers (pinned), copies
    # inside the timed region, pipelined the way a training or serving loop
    # would run it: step n's inputs go up on one copy stream while step n-1
    # computes and step n-2's results come down on another (two buffer sets).
    # The decode state stays resident in HBM between tokens (it is updated in
    # place there); a decode step moves the token's q, k, v, g, beta in and o out.
    resident = {"S"} if w.path == "decode" else set()
    pinned = {n: (None if t is None or n in resident else t.pin_memory()) for n, t in inp.items()}
    h2d = sum(t.numel() * t.element_size() for t in pinned.values() if t is not None)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    dev_in = [{n: (d[n] if n in resident else (None if t is None else torch.empty_like(d[n])))
               for n, t in pinned.items()} for _ in range(2)]
    host_out = [[], []]  # pinned result buffers per buffer set, allocated by the first (untimed) step
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_used = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_used:
        e.record(stream)

    def e2e_step(n):
        j = n % 2
        dd = dev_in[j]
        with torch.cuda.stream(up):
            up.wait_event(ev_used[j])  # the step that used this buffer set has finished computing
            for name, t in pinned.items():
                if t is not None and name not in resident:
                    dd[name].copy_(t, non_blocking=True)
            ev_in[j].record(up)
        stream.wait_event(ev_in[j])
        if flush is not None:  # as in the device-timed loop
            _flush_l2(flush)
        if w.path == "fwd":
            outs = kda.fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], scale=w.scale,
                           initial_state=dd["S0"])
        elif w.path == "fwdbwd":
            o, S_T = kda.fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], scale=w.scale,
                             initial_state=dd["S0"], workspace=ws)
            outs = (o, S_T) + kda.bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["dO"],
                                      scale=w.scale, initial_state=dd["S0"], workspace=ws,
                                      states_from_fwd=True)
        else:
            outs = (kda.decode_step(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S"],
                                    scale=w.scale),)
        outs = [t for t in outs if t is not None]
        ev_used[j].record(stream)
        if not host_out[j]:
            host_out[j].extend(torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs)
        with torch.cuda.stream(down):
            down.wait_event(ev_used[j])
            down.wait_event(ev_out[j])  # the previous read-back into these host buffers is done
            for hbuf, t in zip(host_out[j], outs):
                hbuf.copy_(t, non_blocking=True)
                t.record_stream(down)
            ev_out[j].record(down)
        return host_out[j]

    e2e_steps = max(4, min(steps, 10))
    for n in range(2):
        e2e_step(n)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    for n in range(e2e_steps):
        host = e2e_step(n)
    stream.wait_event(ev_out[0])
    stream.wait_event(ev_out[1])
    e1.record(stream)
    torch.cuda.synchronize()
    d2h = sum(t.numel() * t.element_size() for t in host)
    res["e2e_ms"] = e0.elapsed_time(e1) / e2e_steps
    res["h2d_bytes"] = h2d
    res["d2h_bytes"] = d2h
    del ws
    return res, w


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch of ``kernel`` on ``workload`` from the ncu capture
    recorded in profiles/dram_traffic.json, or None when there is none or the
    kernel's sources changed since (their sha256 is stored beside the figure)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    h = hashlib.sha256()
    for rel in rec["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    return rec["bytes_per_launch"].get(workload)


def roofline_for(res, w, peaks):
    hbm = peaks["hbm_gbs"]
    if w.path == "decode":
        byts = algorithmic_bytes(w, "decode")
        t = res["calls"]["kernel_ms"] * 1e-3
        return {"bound": "hbm", "kernel": "kda_decode_kernel", "achieved": byts / t / 1e9,
                "peak": hbm, "unit": "GB/s", "frac": byts / t / 1e9 / hbm, "algorithmic_bytes": byts,
                "frac_of_nominal": byts / t / 1e9 / NOMINAL_HBM_GBS, "nominal_peak": NOMINAL_HBM_GBS}
    C = 64 if w.K == 128 else 32
    head_tokens = w.B * w.T * w.HV
    fwd_flops = chunk_flops_per_head_token(w.K, w.V, C) * head_tokens
    if w.path == "fwd":
        r = two_rooflines(algorithmic_bytes(w, "fwd"), fwd_flops, res["calls"]["kernel_ms"] * 1e-3, peaks)
        r["kernel"] = ("kda_fwd (kda_fwd_intra_tc_kernel + kda_fwd_state_tc_kernel, one call)"
                       if w.K == 128 and w.dtype == "bf16" else "kda_fwd (CUDA-core chunk kernels)")
        return r
    # the step's dominant part is the backward call (state gradients, gradient
    # products, assembly); its algorithmic bytes are the backward's own I/O
    r = two_rooflines(algorithmic_bytes(w, "bwd"), BWD_FLOPS_RATIO * fwd_flops, res["calls"]["bwd_ms"] * 1e-3,
                      peaks)
    r["kernel"] = ("kda_bwd (kda_bwd_dstate_tc_kernel + kda_bwd_grads_tc_kernel + kda_bwd_assemble_kernel, "
                   "one call)")
    r["fwd"] = dict(two_rooflines(algorithmic_bytes(w, "fwd"), fwd_flops, res["calls"]["fwd_ms"] * 1e-3, peaks),
                    kernel="kda_fwd (kda_fwd_intra_tc_kernel + kda_fwd_state_tc_kernel, one call)")
    r["step"] = two_rooflines(algorithmic_bytes(w, "fwdbwd"), (1 + BWD_FLOPS_RATIO) * fwd_flops,
                              res["ms_per_step"] * 1e-3, peaks)
    return r


def job_throughput(ms_local, tokens_per_step, world, all_reduce_max):
    """Whole-job throughput of replicas: the slowest rank's step time (the
    all-reduce MAX of every rank's device time) and the tokens all ranks
    processed per step.  Returns (ms_per_step, tokens/s)."""
    ms = all_reduce_max(ms_local) if world > 1 else ms_local
    return ms, tokens_per_step * world / (ms * 1e-3)


def run_gpu(args):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    from gated_delta_rule_66_b200 import kda
    peaks = load_peaks()
    results = {}
    chosen = None if args.paths is None else set(args.paths.split(","))
    others = [p for p in PATHS if p != HEADLINE and args.all_paths and (chosen is None or p in chosen)]
    for name in [HEADLINE] + others:
        if name == HEADLINE:
            with Clocks(local) as clk:
                res, w = gpu_path(kda, name, args.steps, args.warmup, barrier, args.shrink)
            res["clocks"] = clk.summary()
        else:  # (--shrink B,T[,BD] reduces the decode batch to BD, else B, as well)
            small = (args.shrink[-1] if len(args.shrink) > 2 else args.shrink[0], 1) \
                if args.shrink and name == "decode" else None
            res, w = gpu_path(kda, name, args.steps, args.warmup, barrier, small)
        if "roofline" not in res:
            res["roofline"] = roofline_for(res, w, peaks)
        def reduce_max(x):
            t = torch.tensor([x], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())
        ms, res["tokens_per_s"] = job_throughput(res["ms_per_step"], res["tokens_per_step"], world, reduce_max)
        res["ms_per_step"] = ms
        res["e2e_tokens_per_s"] = (res["tokens_per_step"] * world / (res["e2e_ms"] * 1e-3)
                                   if res["e2e_ms"] else None)
        results[name] = (res, w)
        torch.cuda.empty_cache()

    head, w = results[HEADLINE]
    line = {
        "metric": METRIC,
        "value": head["tokens_per_s"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "tf32",  # arithmetic: tf32 tensor-core products, fp32 accumulation and CUDA-core steps
        "data": "synthetic (seeded; q,k L2-normalised, g = -5 sigmoid(N(0,1)), beta = sigmoid(N(0,1)))",
        "config": {"workload": f"fwdbwd: B={w.B} H=HV={w.HV} T={w.T} K=V={w.K}, bf16 q/k/v/dO, fp32 g/beta/state; "
                               "step = kda_fwd (stores chunk states and interaction records) + kda_bwd (reuses them)"
                               + ("" if not args.shrink else " [reduced for a profiler capture]"),
                   "arithmetic": "tf32 tensor-core products with fp32 accumulation, fp32 CUDA-core steps; "
                                 "bf16 q/k/v/o/dO storage",
                   "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"replicas x{world}",
                   "l2": head["l2"]},
        "roofline": dict({k: v for k, v in head["roofline"].items() if k != "fwd"},
                         traffic=recorded_traffic(head["roofline"]["kernel"].split()[0], HEADLINE)),
        "e2e": {"value": head["e2e_tokens_per_s"], "unit": "tokens/s",
                "h2d_bytes_per_step": head["h2d_bytes"], "d2h_bytes_per_step": head["d2h_bytes"]},
        "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": head.get("clocks"),
        "peaks": peaks,
        "paths": {n: {"tokens_per_s": r["tokens_per_s"], "ms_per_step": r["ms_per_step"],
                      "e2e_tokens_per_s": r["e2e_tokens_per_s"], "calls_ms": r["calls"],
                      "roofline": r["roofline"], "l2": r["l2"]} for n, (r, _) in results.items()},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- CPU oracle arm

def _oracle_head(job):
    """Runs the float64 oracle fwd (+bwd) on one (b, hv) head of a sample."""
    sys.path.insert(0, ROOT)
    import oracle
    path, arrays, scale = job
    q, k, v, g, beta, S0, dO = arrays
    t0 = time.perf_counter()
    oracle.kda_forward(q, k, v, g, beta, scale, S0)
    if path == "fwdbwd":
        oracle.kda_backward(q, k, v, g, beta, scale, S0, dO)
    return time.perf_counter() - t0


def _warm(_):
    sys.path.insert(0, ROOT)
    import oracle  # noqa: F401
    return 0


class OracleSampler:
    """The float64 oracle on the host's cores, on a bounded sample of a
    workload: whole (b, hv) heads at the workload's full length (a GQA head
    reads its own query/key head), one single-threaded worker process per
    core, as many heads as fit the time budget.  tokens/s = sampled head-tokens
    / HV / elapsed, i.e. scaled to all HV heads of a token."""

    def __init__(self, w, budget_s):
        for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ[var] = "1"   # one thread per worker: `cores` threads in total
        self.w = w
        self.cores = len(os.sched_getaffinity(0))
        inp = host_inputs(w)
        f64 = lambda t: None if t is None else t.to(torch.float64).numpy()
        G = w.HV // w.H
        if w.path == "decode":
            units = [(b, hv) for b in range(w.B) for hv in range(w.HV)]
            T = 1
            def arrays(b, hv):
                h = hv // G
                return (f64(inp["q"][b:b + 1, None, h:h + 1]), f64(inp["k"][b:b + 1, None, h:h + 1]),
                        f64(inp["v"][b:b + 1, None, hv:hv + 1]), f64(inp["g"][b:b + 1, None, hv:hv + 1]),
                        f64(inp["beta"][b:b + 1, None, hv:hv + 1]), f64(inp["S"][b:b + 1, hv:hv + 1]), None)
        else:
            units = [(b, hv) for b in range(w.B) for hv in range(w.HV)]
            T = w.T
            def arrays(b, hv):
                h = hv // G
                return (f64(inp["q"][b:b + 1, :, h:h + 1]), f64(inp["k"][b:b + 1, :, h:h + 1]),
                        f64(inp["v"][b:b + 1, :, hv:hv + 1]), f64(inp["g"][b:b + 1, :, hv:hv + 1]),
                        f64(inp["beta"][b:b + 1, :, hv:hv + 1]),
                        None if inp["S0"] is None else f64(inp["S0"][b:b + 1, hv:hv + 1]),
                        None if inp.get("dO") is None else f64(inp["dO"][b:b + 1, :, hv:hv + 1]))
        self.pool = mp.get_context("spawn").Pool(processes=self.cores)
        self.pool.map(_warm, range(self.cores))   # worker start-up stays outside the timing
        # calibrate on a short prefix of one head with every worker busy at once
        # (as in the timed run: shared cores and memory bandwidth), then size the sample
        cal = min(T, 64)
        q, k, v, g, beta, S0, dO = arrays(0, 0)
        cut = lambda x: None if x is None or w.path == "decode" else x[:, :cal]
        cal_job = (w.path, (cut(q), cut(k), cut(v), cut(g), cut(beta), S0, cut(dO)), w.scale)
        try:  # the first pass warms every worker's NumPy; the second is timed
            self.pool.map(_oracle_head, [cal_job] * self.cores, chunksize=1)
            t_cal = statistics.median(self.pool.map(_oracle_head, [cal_job] * self.cores, chunksize=1))
        except BaseException:
            self.pool.terminate()
            raise
        t_head = max(t_cal * T / cal, 1e-4)
        per_worker = max(1, int(budget_s / t_head))
        n = min(len(units), self.cores * per_worker)
        self.jobs = [(w.path, arrays(b, hv), w.scale) for (b, hv) in units[:n]]
        self.head_tokens = n * T
        self.desc = (f"{n} of {len(units)} (b, hv) heads, each the full {T} steps "
                     f"({'fwd+bwd' if w.path == 'fwdbwd' else w.path}), float64 NumPy, one single-threaded "
                     f"process per core; tokens/s = head-tokens / {w.HV} heads / elapsed")

    def run(self):
        t0 = time.perf_counter()
        self.pool.map(_oracle_head, self.jobs, chunksize=1)
        elapsed = time.perf_counter() - t0
        return {"value": self.head_tokens / self.w.HV / elapsed, "unit": "tokens/s", "cores": self.cores,
                "kind": "oracle", "sample": self.desc, "seconds": elapsed}

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(w, budget_s=20.0):
    smp = OracleSampler(w, budget_s)
    try:
        return smp.run()
    finally:
        smp.close()


def run_reference(args):
    """The reference arm: the float64 oracle on the host cores.  One step is
    one bounded sample of the headline workload (whole (b, hv) heads at the
    full length, as many as fit the step's time budget), so ms_per_step is the
    time the sample actually took and steps x ms_per_step is the time this
    run spent in timed steps.  The throughput scales the sample's head-tokens
    to all value heads of a token; the time a whole step (every head) would
    take at that rate is reported beside it, labelled as an extrapolation."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = BY_NAME[HEADLINE]
    # each step is one bounded sample; the whole run stays within a few minutes
    smp = OracleSampler(w, budget_s=max(2.0, 100.0 / (args.steps + args.warmup)))
    try:
        runs = [smp.run() for _ in range(args.warmup + args.steps)]
    finally:
        smp.close()
    timed = runs[args.warmup:]
    val = statistics.median(c["value"] for c in timed)
    sample_ms = statistics.median(c["seconds"] for c in timed) * 1e3
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": 1, "steps": len(timed),
            "warmup": len(runs) - len(timed), "ms_per_step": sample_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "fwdbwd: B=2 H=HV=96 T=4096 K=V=128 (float64 oracle); one step = one bounded "
                                   "sample of whole heads, tokens/s scaled to all value heads",
                       "global_batch": w.B, "seq_len": w.T, "parallelism": "none",
                       "step": timed[-1]["sample"],
                       "extrapolated_full_step_ms": w.B * w.T / val * 1e3},
            "cpu_baseline": {"kind": "oracle", "cores": timed[-1]["cores"], "sample": timed[-1]["sample"],
                             "value": val, "unit": "tokens/s"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", dest="all_paths", action="store_false")
    ap.add_argument("--shrink", type=lambda x: tuple(int(v) for v in x.split(",")), default=None,
                    metavar="B,T[,BD]", help="run the headline workload at batch B and length T and the decode "
                                             "path at batch BD (default B) (for ncu captures; the printed line "
                                             "is not a headline number)")
    ap.add_argument("--paths", default=None, metavar="NAME,...",
                    help="the other paths to run after the headline (default: all of them)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
