"""GPU parity of the preparation around the recurrence (through the C ABI)
against the float64 oracle: the prefill with the preparation fused into the
forward kernels (L2-normalised q/k, the decay gate from its pre-activation,
beta from its logit, the output gate), the short convolution, and the decode
token from raw projections; relative L2 bars 1e-5 (fp32) and 2e-3 (bf16).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_66_b200.inputs import BY_NAME, make_raw_inputs
from kda_testlib import f64, report, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from gated_delta_rule_66_b200 import kda as mod
    mod.device_status()
    yield mod
    assert mod.device_status() == 0, "a kernel gave up on a bounded wait"


def cuda(r):
    return {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in r.items()}


def oracle_prep(r, scale, gate=True):
    return oracle.kda_forward_prepared(f64(r["q"]), f64(r["k"]), f64(r["v"]), f64(r["z"]), f64(r["A_log"]),
                                       f64(r["dt_bias"]), r["lower_bound"], f64(r["beta_logit"]), scale,
                                       f64(r["S0"]), out_gate=f64(r["og"]) if gate else None)


def run_prep(kda, r, scale, gate=True, workspace=True):
    d = cuda(r)
    o, S = kda.fwd_prep(d["q"], d["k"], d["v"], d["z"], d["A_log"], d["dt_bias"], d["beta_logit"],
                        gate_lower_bound=r["lower_bound"], scale=scale, initial_state=d["S0"],
                        out_gate=d["og"] if gate else None, workspace=workspace)
    torch.cuda.synchronize()
    return o, S


PREP_CASES = [
    # name, workload, size overrides, gate lower bound, output gate, workspace
    ("tc_gqa_ragged", "prefill_gqa", dict(B=2, T=200, H=2, HV=4), -5.0, True, True),
    ("tc_single_kernel", "prefill_gqa", dict(B=1, T=130, H=1, HV=2), -5.0, True, None),
    ("tc_unbounded_no_gate", "fwdbwd", dict(B=1, T=257, H=2, HV=2, s0_std=0.02), 0.0, False, True),
    ("cuda_core_twin_fp32", "twin", dict(B=2, T=100), 0.0, True, None),
    ("cuda_core_bf16_k64", "prefill_gqa", dict(B=1, T=90, H=1, HV=3, K=64, V=32), -5.0, True, True),
    ("tiny_fp32", "tiny", {}, -5.0, True, None),
]


@pytest.mark.parametrize("name,wname,over,lb,gate,ws", PREP_CASES, ids=[c[0] for c in PREP_CASES])
def test_fwd_prep(kda, name, wname, over, lb, gate, ws):
    """Raw q, k (normalised in the kernel), z, beta logits and the output
    gate: tensor-core two-kernel and single-kernel paths, the CUDA-core path
    with the output-gate pass (in place for fp32, fp32 scratch for bf16)."""
    w = BY_NAME[wname].with_sizes(**over)
    r = make_raw_inputs(w, lower_bound=lb)
    o, S = run_prep(kda, r, w.scale, gate, ws)
    o_ref, S_ref = oracle_prep(r, w.scale, gate)
    tol = tol_for(w.torch_dtype)
    report(f"prep_{name} o", f64(o), o_ref, tol, w.torch_dtype)
    report(f"prep_{name} S_T", f64(S), S_ref, tol, torch.float32)


def test_fwd_prep_strong_unbounded_decay(kda):
    """Unbounded gate with a steep slope (A_log up to 1.5): in-chunk decays
    that leave the split-exponent range, on the tensor-core path."""
    w = BY_NAME["prefill_gqa"].with_sizes(B=1, T=192, H=1, HV=2)
    r = make_raw_inputs(w, lower_bound=0.0)
    r["A_log"] = r["A_log"] + 3.5
    o, S = run_prep(kda, r, w.scale)
    o_ref, S_ref = oracle_prep(r, w.scale)
    report("prep_strong o", f64(o), o_ref, tol_for(w.torch_dtype), w.torch_dtype)
    report("prep_strong S_T", f64(S), S_ref, tol_for(w.torch_dtype), torch.float32)


def test_fwd_prep_full_size(kda):
    """The production prefill geometry (B=1, H=16 -> HV=96, T=8192, K=V=128,
    bf16) from raw projections with the output gate, in full on the GPU; the
    oracle checks grouped-query block 3."""
    w = BY_NAME["prefill_gqa"]
    r = make_raw_inputs(w)
    o, S = run_prep(kda, r, w.scale)
    G = w.HV // w.H
    h, hv = 3, list(range(3 * G, 4 * G))
    sub = dict(r)
    for n in ("q", "k"):
        sub[n] = r[n][:, :, [h]]
    for n in ("v", "z", "og", "beta_logit"):
        sub[n] = r[n][:, :, hv]
    sub["A_log"], sub["dt_bias"] = r["A_log"][hv], r["dt_bias"][hv]
    o_ref, S_ref = oracle_prep(sub, w.scale)
    report("prep_full o[group 3]", f64(o[:, :, hv]), o_ref, tol_for(w.torch_dtype), w.torch_dtype)
    report("prep_full S_T[group 3]", f64(S[:, hv]), S_ref, tol_for(w.torch_dtype), torch.float32)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()


CONV_CASES = [
    # name, workload, size overrides, window, initial window
    ("bf16_gqa", "prefill_gqa", dict(B=2, T=77, H=1, HV=2, K=64, V=32), 4, True),
    ("fp32_shorter_than_window", "twin", dict(B=2, T=3), 4, True),
    ("bf16_w2_zero_window", "prefill_gqa", dict(B=1, T=40, H=2, HV=2, K=32, V=128), 2, False),
]


@pytest.mark.parametrize("name,wname,over,W,with_state", CONV_CASES, ids=[c[0] for c in CONV_CASES])
def test_short_conv(kda, name, wname, over, W, with_state):
    """The sequence form of the convolution; the final window is exact (it
    holds inputs), the activations within the dtype's bar."""
    w = BY_NAME[wname].with_sizes(**over)
    r = make_raw_inputs(w, conv_width=W)
    st0 = r["conv_state"] if with_state else None
    q, k, v, st = kda.short_conv(r["q"].cuda(), r["k"].cuda(), r["v"].cuda(), r["conv_w"].cuda(),
                                 None if st0 is None else st0.cuda())
    torch.cuda.synchronize()
    q_ref, k_ref, v_ref, st_ref = oracle.short_conv_qkv(f64(r["q"]), f64(r["k"]), f64(r["v"]), f64(r["conv_w"]),
                                                        None if st0 is None else f64(st0))
    tol = tol_for(w.torch_dtype)
    for n, x, ref in (("q", q, q_ref), ("k", k, k_ref), ("v", v, v_ref)):
        report(f"conv_{name} {n}", f64(x), ref, tol, w.torch_dtype)
    assert np.array_equal(f64(st), st_ref)


def _decode_inputs(w, W, steps, lb):
    return [make_raw_inputs(w.with_sizes(T=1), seed=900 + t, conv_width=W, lower_bound=lb) for t in range(steps)]


DECODE_CASES = [
    # name, workload, size overrides, window, lower bound, output gate
    ("bf16_gqa_gate", "decode", dict(B=3, H=2, HV=4), 4, -5.0, True),
    ("bf16_mha_in_place", "decode", dict(B=5, H=4, HV=4), 4, -5.0, True),
    ("fp32_twin_unbounded", "twin", dict(B=2, T=1), 4, 0.0, False),
]


@pytest.mark.parametrize("name,wname,over,W,lb,gate", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_token(kda, name, wname, over, W, lb, gate):
    """Three decode tokens from raw projections (window step, preparation,
    recurrence in place, output gate) against the oracle's decode token."""
    w = BY_NAME[wname].with_sizes(**over)
    steps = 3
    toks = _decode_inputs(w, W, steps, lb)
    first = toks[0]
    S = (torch.randn(w.B, w.HV, w.K, w.V, generator=torch.Generator().manual_seed(5)) * 0.02)
    S_gpu = S.cuda()
    win = first["conv_state"].cuda()
    in_place = w.H == w.HV
    S_ref, win_ref = f64(S), f64(first["conv_state"])
    tol = tol_for(w.torch_dtype)
    for t, r in enumerate(toks):
        d = {n: (x[:, 0].contiguous().cuda() if isinstance(x, torch.Tensor) and x.dim() >= 3 else x)
             for n, x in r.items() if n not in ("conv_w", "conv_state", "S0")}
        out = None if in_place else torch.empty_like(win)
        o = kda.decode_token(d["q"], d["k"], d["v"], first["conv_w"].cuda(), win, d["z"], r["A_log"].cuda(),
                             r["dt_bias"].cuda(), d["beta_logit"], S_gpu, gate_lower_bound=lb, scale=w.scale,
                             out_gate=d["og"] if gate else None, conv_out=out)
        if not in_place:
            win = out
        torch.cuda.synchronize()
        o_ref, S_ref, win_ref = oracle.kda_decode_token(
            f64(r["q"][:, 0]), f64(r["k"][:, 0]), f64(r["v"][:, 0]), f64(first["conv_w"]), win_ref,
            f64(r["z"][:, 0]), f64(r["A_log"]), f64(r["dt_bias"]), lb, f64(r["beta_logit"][:, 0]), S_ref, w.scale,
            out_gate=f64(r["og"][:, 0]) if gate else None)
        report(f"token_{name} step{t} o", f64(o), o_ref, tol, w.torch_dtype)
        assert np.array_equal(f64(win), win_ref)
    report(f"token_{name} S", f64(S_gpu), S_ref, tol, torch.float32)


def test_raw_prefill_then_decode(kda):
    """The host model's pipeline from raw projections: the convolution over
    the prompt, the prepared prefill, then decode tokens continuing from its
    final window and state.  The prompt's convolved activations are stored in
    the input dtype, so the oracle's prefill takes the same activations; the
    decode tokens run from the oracle's own state and window."""
    W, steps = 4, 3
    w = BY_NAME["prefill_gqa"].with_sizes(B=2, T=150, H=2, HV=4)
    r = make_raw_inputs(w, conv_width=W)
    d = cuda(r)
    q, k, v, win = kda.short_conv(d["q"], d["k"], d["v"], d["conv_w"], d["conv_state"])
    o, S = kda.fwd_prep(q, k, v, d["z"], d["A_log"], d["dt_bias"], d["beta_logit"], scale=w.scale,
                        out_gate=d["og"])
    toks = _decode_inputs(w.with_sizes(T=1), W, steps, -5.0)
    outs = []
    for t, tk in enumerate(toks):
        e = {n: tk[n][:, 0].contiguous().cuda() for n in ("q", "k", "v", "z", "beta_logit", "og")}
        win_next = torch.empty_like(win)
        outs.append(kda.decode_token(e["q"], e["k"], e["v"], d["conv_w"], win, e["z"], d["A_log"], d["dt_bias"],
                                     e["beta_logit"], S, scale=w.scale, out_gate=e["og"], conv_out=win_next))
        win = win_next
    torch.cuda.synchronize()
    conv_act = {"q": q.cpu(), "k": k.cpu(), "v": v.cpu()}
    o_ref, S_ref = oracle.kda_forward_prepared(
        f64(conv_act["q"]), f64(conv_act["k"]), f64(conv_act["v"]), f64(r["z"]), f64(r["A_log"]), f64(r["dt_bias"]),
        -5.0, f64(r["beta_logit"]), w.scale, None, out_gate=f64(r["og"]))
    tol = tol_for(w.torch_dtype)
    report("pipeline prefill o", f64(o), o_ref, tol, w.torch_dtype)
    _, _, _, win_ref = oracle.short_conv_qkv(f64(r["q"]), f64(r["k"]), f64(r["v"]), f64(r["conv_w"]),
                                             f64(r["conv_state"]))
    for t, tk in enumerate(toks):
        o_t, S_ref, win_ref = oracle.kda_decode_token(
            f64(tk["q"][:, 0]), f64(tk["k"][:, 0]), f64(tk["v"][:, 0]), f64(r["conv_w"]), win_ref, f64(tk["z"][:, 0]),
            f64(r["A_log"]), f64(r["dt_bias"]), -5.0, f64(tk["beta_logit"][:, 0]), S_ref, w.scale,
            out_gate=f64(tk["og"][:, 0]))
        report(f"pipeline decode step{t} o", f64(outs[t]), o_t, tol, w.torch_dtype)
    report("pipeline final S", f64(S), S_ref, tol, torch.float32)
    assert np.array_equal(f64(win), win_ref)


# ----------------------------------------------------------------------------- erase/write variant
from gated_delta_rule_66_b200.inputs import make_erase_inputs  # noqa: E402

ERASE_CASES = [
    # name, size overrides of the erase workload
    ("fp32_k32_ragged", dict(B=2, T=77, H=4, HV=2, K=32, V=32, dtype="fp32", s0_std=0.05)),
    ("bf16_k64_v128", dict(B=1, T=100, H=8, HV=2, K=64, V=128)),
    ("bf16_k128_mha", dict(B=2, T=65, H=2, HV=2, K=128, V=64, s0_std=0.05)),
]


def _erase_oracle(r, scale):
    return oracle.erase_forward(f64(r["q"]), f64(r["k"]), f64(r["e"]), f64(r["z"]), f64(r["g"]), scale,
                                f64(r["S0"]))


@pytest.mark.parametrize("scratch", [True, False], ids=["two_kernel", "single_kernel"])
@pytest.mark.parametrize("name,over", ERASE_CASES, ids=[c[0] for c in ERASE_CASES])
def test_fwd_erase(kda, name, over, scratch):
    """The asymmetric erase/write recurrence (separate erase and write
    vectors, query heads grouped over state heads) against the token loop, on
    the two-kernel path (chunk preparation, then one state pass per state
    head for all its query heads) and on the single-kernel path."""
    w = BY_NAME["erase"].with_sizes(**over)
    r = make_erase_inputs(w)
    d = {n: (None if t is None else t.cuda()) for n, t in r.items()}
    o, S = kda.fwd_erase(d["q"], d["k"], d["e"], d["z"], d["g"], scale=w.scale, initial_state=d["S0"],
                         scratch=scratch)
    torch.cuda.synchronize()
    o_ref, S_ref = _erase_oracle(r, w.scale)
    tol = tol_for(w.torch_dtype)
    tag = f"erase_{name}" + ("" if scratch else "_single")
    report(f"{tag} o", f64(o), o_ref, tol, w.torch_dtype)
    report(f"{tag} S_T", f64(S), S_ref, tol, torch.float32)


def test_fwd_erase_kda_special_case(kda):
    """e = beta k and z = beta v make the variant KDA: its output equals the
    KDA forward's on the same GPU (fp32, within the fp32 bar of each other)."""
    from gated_delta_rule_66_b200.inputs import make_inputs
    w = BY_NAME["twin"].with_sizes(B=1, T=96, H=2, HV=2)
    inp = make_inputs(w)
    d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    o_k, S_k = kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"])
    e = (d["beta"][..., None] * d["k"]).contiguous()
    z = (d["beta"][..., None] * d["v"]).contiguous()
    o_e, S_e = kda.fwd_erase(d["q"], d["k"], e, z, d["g"], scale=w.scale, initial_state=d["S0"])
    torch.cuda.synchronize()
    report("erase_as_kda o", f64(o_e), f64(o_k), 1e-5, torch.float32)
    report("erase_as_kda S_T", f64(S_e), f64(S_k), 1e-5, torch.float32)


def test_fwd_erase_full_size(kda):
    """The erase workload (B=1, T=8192, 32 query heads over 8 state heads,
    K=64, V=128, bf16) in full on the GPU; the oracle checks state head 3 and
    its four query heads."""
    w = BY_NAME["erase"]
    r = make_erase_inputs(w)
    d = {n: (None if t is None else t.cuda()) for n, t in r.items()}
    o, S = kda.fwd_erase(d["q"], d["k"], d["e"], d["z"], d["g"], scale=w.scale)
    torch.cuda.synchronize()
    QG = w.H // w.HV
    hq = list(range(3 * QG, 4 * QG))
    sub = {"q": r["q"][:, :, hq], "k": r["k"][:, :, [3]], "e": r["e"][:, :, [3]], "z": r["z"][:, :, [3]],
           "g": r["g"][:, :, [3]], "S0": None}
    o_ref, S_ref = _erase_oracle(sub, w.scale)
    report("erase_full o[state head 3]", f64(o[:, :, hq]), o_ref, tol_for(w.torch_dtype), w.torch_dtype)
    report("erase_full S_T[state head 3]", f64(S[:, [3]]), S_ref, tol_for(w.torch_dtype), torch.float32)
    assert torch.isfinite(o.float()).all()
