"""Pins for the oracle of the preparation steps around the recurrence (the
short convolution, L2 normalisation, the decay gate, the beta sigmoid and the
output gate): worked examples whose inputs the pages print (fixtures under
tests/golden), library routines for the special functions and the
convolution, closed forms and invariants.  The pins take the implementation
as an argument, and ``test_prep_pins_reject_planted_mistakes`` shows that a
plausible mistake in any step fails at least one of them.
"""
from __future__ import annotations

import json
import math
import os
import types

import numpy as np
import pytest
from scipy.special import expit

import oracle
from oracle import kda_decode_step, kda_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


ORACLE = types.SimpleNamespace(softplus=oracle.softplus, sigmoid=oracle.sigmoid, l2norm_rows=oracle.l2norm_rows,
                               kda_gate=oracle.kda_gate, conv_update=oracle.conv_update,
                               short_conv_silu=oracle.short_conv_silu, output_gate=oracle.output_gate)


# ---------------------------------------------------------------------------
# Pins (each takes an implementation namespace)
# ---------------------------------------------------------------------------

def pin_gate_worked_example(m):
    """"kimi_k3_host/kda.rs", test omitted_lower_bound_is_neg_exp_a_softplus."""
    fx = _fixture("gate_unbounded_softplus.json")
    z = np.array(fx["z"])[None]
    dt = np.array(fx["dt_bias"])[None]
    a_log = np.array(fx["A_log"])
    g = m.kda_gate(z, a_log, dt, 0.0)[0]
    sp = lambda x: max(x, 0.0) + math.log1p(math.exp(-abs(x)))
    ok = all(abs(g[c] - (-sp(fx["z"][c] + fx["dt_bias"][c]))) < fx["tolerance"] for c in range(2))
    g5 = m.kda_gate(z, a_log, dt, fx["bounded_lower_bound"])[0]
    return ok and abs(g5[0] - g[0]) > fx["bounded_min_difference_channel0"]


def pin_special_functions(m):
    """softplus against numpy's logaddexp(0, x), sigmoid against scipy's
    expit, over a range that reaches both overflow regions."""
    x = np.concatenate([np.linspace(-60, 60, 241), [-700.0, -30.5, 0.0, 30.5, 700.0]])
    return (np.abs(m.softplus(x) - np.logaddexp(0.0, x)).max() <= 1e-13 * np.maximum(1, np.abs(x)).max()
            and np.abs(m.sigmoid(x) - expit(x)).max() < 1e-15)


def pin_gate_closed_forms(m):
    """Bounded form lb sigmoid(e^A x): lb / 2 at x = 0, -> lb for large x,
    -> 0 for very negative x, and e^A scales x.  Unbounded form
    -e^A softplus(x): -e^A ln 2 at x = 0, ~ -e^A x for large x."""
    a_log = np.array([0.0, math.log(3.0)])
    dt = np.zeros((2, 3))
    zero = np.zeros((1, 2, 3))
    lb = -5.0
    g0 = m.kda_gate(zero, a_log, dt, lb)
    big = m.kda_gate(zero + 40.0, a_log, dt, lb)
    neg = m.kda_gate(zero - 40.0, a_log, dt, lb)
    z = np.array([[[0.3, -0.7, 1.1], [0.3, -0.7, 1.1]]])
    sl = m.kda_gate(z, a_log, dt, lb)
    slope = abs(sl[0, 1] - lb * expit(3.0 * z[0, 1])).max() < 1e-14
    u0 = m.kda_gate(zero, a_log, dt, 0.0)
    ubig = m.kda_gate(zero + 50.0, a_log, dt, 0.0)
    bias = m.kda_gate(zero, a_log, dt + 0.25, 0.0)
    return (np.allclose(g0, lb / 2, rtol=0, atol=1e-15) and np.allclose(big, lb, atol=1e-12)
            and np.abs(neg).max() < 1e-12 and slope
            and np.allclose(u0[0, 0], -math.log(2.0), atol=1e-15) and np.allclose(u0[0, 1], -3 * math.log(2.0), atol=1e-14)
            and np.allclose(ubig[0, 1], -3 * 50.0, rtol=1e-15, atol=1e-12)
            and np.allclose(bias[0, 0], -np.logaddexp(0.0, 0.25), atol=1e-15))


def pin_l2norm(m):
    """Row norms: |x_hat|^2 = s / (s + eps) with s the row's sum of squares;
    the direction is kept; a zero row stays zero; the eps default is the
    page's 1e-6."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 5, 16)) * np.array([1e-4, 1.0, 30.0, 1e-3, 2.0])[None, :, None]
    x[0, 0] = 0.0
    y = m.l2norm_rows(x)
    s = (x * x).sum(-1)
    ok = np.allclose((y * y).sum(-1), s / (s + 1e-6), rtol=1e-14, atol=0)
    nz = s > 0
    cos = (x * y).sum(-1)[nz] / np.sqrt(s[nz] * (y * y).sum(-1)[nz])
    return ok and np.allclose(cos, 1.0, atol=1e-14) and not np.any(y[0, 0])


def pin_conv_state_advances(m):
    """"kimi_k3_host/kda.rs", test conv_kernel_4_state_advances."""
    fx = _fixture("conv_state_advances.json")
    C, W = fx["channels"], fx["kernel"]
    st = np.zeros((C, W))
    w = np.ones((C, W))
    for t in range(fx["steps"]):
        x = np.full(C, t + 1.0)
        _, st = m.conv_update(st, x, w)
        if not np.array_equal(st[:, W - 1], x):
            return False
    return bool(np.all(st == np.array(fx["final_window"])[None]))


def pin_conv_library(m):
    """The sequence form against numpy's correlate on the padded sequence
    (window state first, oldest slot dropped) per channel, then SiLU with
    scipy's expit; the final window is the last W inputs; and the per-token
    update reproduces the sequence form step by step."""
    rng = np.random.default_rng(5)
    B, T, C, W = 2, 9, 5, 4
    x = rng.standard_normal((B, T, C))
    w = rng.standard_normal((C, W))
    st0 = rng.standard_normal((B, C, W))
    y, st = m.short_conv_silu(x, w, st0)
    ok = True
    for b in range(B):
        for c in range(C):
            u = np.concatenate([st0[b, c, 1:], x[b, :, c]])
            acc = np.correlate(u, w[c], mode="valid")
            ok &= np.abs(y[b, :, c] - acc * expit(acc)).max() < 1e-13
            ok &= np.array_equal(st[b, c], np.concatenate([st0[b, c], x[b, :, c]])[-W:])
    cur = st0
    for t in range(T):
        yt, cur = m.conv_update(cur, x[:, t], w)
        ok &= np.abs(yt - y[:, t]).max() < 1e-13
    yshort, stshort = m.short_conv_silu(x[:, :2], w, st0)  # fewer steps than the window
    ok &= np.array_equal(stshort, np.concatenate([st0, np.transpose(x[:, :2], (0, 2, 1))], axis=2)[:, :, -W:])
    return bool(ok)


def pin_output_gate(m):
    """With a zero gate (sigmoid 1/2) every row's RMS is
    sqrt(ms / (ms + eps)) / 2; with eps = 0 the output does not change when a
    row is scaled; with a saturated gate and eps = 0 every row has RMS 1."""
    rng = np.random.default_rng(9)
    o = rng.standard_normal((3, 4, 32)) * np.array([1e-3, 1.0, 10.0, 0.1])[None, :, None]
    ms = (o * o).mean(-1)
    half = m.output_gate(o, np.zeros_like(o), 1e-6)
    ok = np.allclose(np.sqrt((half * half).mean(-1)), 0.5 * np.sqrt(ms / (ms + 1e-6)), rtol=1e-13, atol=0)
    gate = rng.standard_normal(o.shape)
    ok &= np.allclose(m.output_gate(7.5 * o, gate, 0.0), m.output_gate(o, gate, 0.0), rtol=1e-13, atol=1e-15)
    sat = m.output_gate(o, np.full(o.shape, 40.0), 0.0)
    ok &= np.allclose(np.sqrt((sat * sat).mean(-1)), 1.0, atol=1e-14)
    ok &= np.array_equal(np.sign(m.output_gate(o, gate, 1e-6)), np.sign(o))
    return bool(ok)


PREP_PINS = [pin_gate_worked_example, pin_special_functions, pin_gate_closed_forms, pin_l2norm,
             pin_conv_state_advances, pin_conv_library, pin_output_gate]


@pytest.mark.parametrize("pin", PREP_PINS, ids=lambda p: p.__name__)
def test_prep_pins(pin):
    assert pin(ORACLE)


def _mistaken(which):
    m = types.SimpleNamespace(**vars(ORACLE))
    if which == "gate_no_exp":
        m.kda_gate = lambda z, A, dt, lb: (lb * expit(np.asarray(A)[:, None] * (z + dt)) if lb
                                           else -np.asarray(A)[:, None] * oracle.softplus(z + dt))
    elif which == "gate_bias_outside":
        m.kda_gate = lambda z, A, dt, lb: (lb * expit(np.exp(A)[:, None] * z + dt) if lb
                                           else -np.exp(A)[:, None] * oracle.softplus(z) + dt)
    elif which == "softplus_sign":
        m.softplus = lambda x: np.maximum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))
    elif which == "eps_outside_sqrt":
        m.l2norm_rows = lambda x, eps=1e-6: x / (np.sqrt((x * x).sum(-1, keepdims=True)) + eps)
    elif which == "conv_weights_reversed":
        def cu(state, x, w):
            new = np.concatenate([state[..., 1:], x[..., None]], axis=-1)
            acc = (new * w[:, ::-1]).sum(-1)
            return acc * expit(acc), new
        m.conv_update = cu
        m.short_conv_silu = lambda x, w, st=None: oracle.short_conv_silu(x, w[:, ::-1], st)
    elif which == "conv_no_silu":
        def cu(state, x, w):
            new = np.concatenate([state[..., 1:], x[..., None]], axis=-1)
            return (new * w).sum(-1), new
        m.conv_update = cu
    elif which == "rms_sum_not_mean":
        m.output_gate = lambda o, g, eps=1e-6: expit(g) * o / np.sqrt((o * o).sum(-1, keepdims=True) + eps)
    elif which == "gate_not_sigmoid":
        m.output_gate = lambda o, g, eps=1e-6: g * o / np.sqrt((o * o).mean(-1, keepdims=True) + eps)
    return m


@pytest.mark.parametrize("which", ["gate_no_exp", "gate_bias_outside", "softplus_sign", "eps_outside_sqrt",
                                   "conv_weights_reversed", "conv_no_silu", "rms_sum_not_mean",
                                   "gate_not_sigmoid"])
def test_prep_pins_reject_planted_mistakes(which):
    assert not all(p(_mistaken(which)) for p in PREP_PINS), f"no pin caught {which}"


# ---------------------------------------------------------------------------
# The compositions
# ---------------------------------------------------------------------------

def test_decode_token_prefix_snapshot_from_page():
    """"kimi_k3_host/kda.rs", test prefix_hit_wrong_slot_diverges, on the full
    decode token (window and recurrent state restored together)."""
    fx = _fixture("decode_prefix_snapshot.json")
    d, Wk = fx["head_dim"], fx["conv_kernel"]
    C = 3 * d
    conv_w = np.full((C, Wk), fx["conv_weight"])
    z = np.array(fx["z"])[None, None]
    dt = np.array(fx["dt_bias"])[None]
    a_log = np.array(fx["A_log"])
    bl = np.array(fx["beta_logit"])[None]
    scale = 1.0 / math.sqrt(d)

    def tok(val, st, S):
        x = np.full((1, 1, d), val)
        return oracle.kda_decode_token(x, x, x, conv_w, st, z, a_log, dt, fx["gate_lower_bound"], bl, S, scale)

    st, S = np.zeros((1, C, Wk)), np.zeros((1, 1, d, d))
    snaps = []
    for val in fx["prefix_inputs"]:
        _, S, st = tok(val, st, S)
        snaps.append((st.copy(), S.copy()))
    y_seq, _, st_seq = tok(fx["third_input"], st, S)
    y_hit, _, st_hit = tok(fx["third_input"], *snaps[1])
    y_wrong, _, _ = tok(fx["third_input"], *snaps[0])
    assert np.array_equal(y_hit, y_seq) and np.array_equal(st_hit, st_seq)
    assert np.abs(y_wrong - y_hit).max() > fx["min_divergence"]


def test_prepared_forward_worked_example_from_page():
    """The inputs of "kimi_k3_host/kda.rs" test beta_zero_is_sigmoid_half_not_zero
    through the prepared prefill (raw q, k normalised inside, beta logit 0):
    from a zero state the gate drops out and o = scale * (1/2) (q_hat . k_hat) v."""
    fx = _fixture("decode_beta_logit_zero.json")
    d, eps = fx["head_dim"], fx["l2_eps"]
    qkv = np.array(fx["qkv"])
    qr, kr, v = qkv[:d], qkv[d:2 * d], qkv[2 * d:]
    scale = 1.0 / math.sqrt(d)
    o, _ = oracle.kda_forward_prepared(qr[None, None, None], kr[None, None, None], v[None, None, None],
                                       np.zeros((1, 1, 1, d)), np.zeros(1), np.zeros((1, d)), -5.0,
                                       np.array(fx["beta_logit"])[None, None], scale)
    qh, kh = qr / math.sqrt((qr ** 2).sum() + eps), kr / math.sqrt((kr ** 2).sum() + eps)
    assert np.abs(o[0, 0, 0] - scale * 0.5 * float(qh @ kh) * v).max() < 1e-15


@pytest.mark.parametrize("lb", [-5.0, 0.0])
def test_decode_tokens_equal_prepared_prefill(lb):
    """T decode tokens from raw projections (window step per token) equal the
    sequence form of the convolution followed by the prepared prefill and the
    output gate; grouped heads (H = 1, HV = 2)."""
    rng = np.random.default_rng(17)
    B, T, H, HV, K, V, W = 2, 7, 1, 2, 3, 4, 4
    xq, xk = rng.standard_normal((B, T, H, K)), rng.standard_normal((B, T, H, K))
    xv = rng.standard_normal((B, T, HV, V))
    C = 2 * H * K + HV * V
    conv_w = rng.standard_normal((C, W)) * 0.5
    st0 = rng.standard_normal((B, C, W))
    z = rng.standard_normal((B, T, HV, K))
    a_log = rng.uniform(-2, 0, HV)
    dt = 0.1 * rng.standard_normal((HV, K))
    bl = rng.standard_normal((B, T, HV))
    og = rng.standard_normal((B, T, HV, V))
    S0 = 0.3 * rng.standard_normal((B, HV, K, V))
    q, k, v, st_end = oracle.short_conv_qkv(xq, xk, xv, conv_w, st0)
    o_ref, S_ref = oracle.kda_forward_prepared(q, k, v, z, a_log, dt, lb, bl, 0.5, S0, out_gate=og)
    st, S = st0, S0
    for t in range(T):
        o_t, S, st = oracle.kda_decode_token(xq[:, t], xk[:, t], xv[:, t], conv_w, st, z[:, t], a_log, dt, lb,
                                             bl[:, t], S, 0.5, out_gate=og[:, t])
        assert rel(o_t, o_ref[:, t]) < 1e-13
    assert rel(S, S_ref) < 1e-13 and rel(st, st_end) < 1e-15
