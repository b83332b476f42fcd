"""Pins for the float64 oracle: results fixed by the pages and by mathematics.

None of these re-types the oracle's loop.  Each checks the oracle against a
different statement of the same result: exact rational arithmetic of the
transition-matrix form, closed forms of special cases, invariants (the
delta-rule projection, linearity, state passing, grouped heads), an
independent chunked (triangular-solve) restatement, a worked example whose
inputs are printed on the pages, and central finite differences for every
gradient.  ``test_pins_reject_planted_mistakes`` shows that plausible
mistakes in the forward loop fail at least one pin.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import kda_backward, kda_decode_step, kda_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B, T, H, HV, K, V, beta_zero=False, gmin=-5.0):
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, HV, V))
    g = gmin / (1.0 + np.exp(-rng.standard_normal((B, T, HV, K))))
    beta = np.zeros((B, T, HV)) if beta_zero else 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, HV))))
    S0 = 0.3 * rng.standard_normal((B, HV, K, V))
    return q, k, v, g, beta, S0


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------------------
# Pin functions take a forward implementation so they can also be run on
# deliberately wrong variants (see test_pins_reject_planted_mistakes).
# ---------------------------------------------------------------------------

def _exact_transition_form(q, k, v, d, beta, S0, scale, G):
    """Exact rational evaluation of the recurrence as S_t = A_t S_{t-1} + B_t.

    From "K3/kda/ops/reference/recurrent.py" (module docstring formula):
    S_t = D_t S_{t-1} + beta_t k_t (v_t - k_t^T D_t S_{t-1})^T
        = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T (scale q_t), with D_t = diag(d_t), d = exp(g) given exactly.
    Computed with K x K transition matrices, not rank-1 updates.
    """
    B, T, H, K = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    HV, V = len(v[0][0]), len(v[0][0][0])
    o = [[[[None] * V for _ in range(HV)] for _ in range(T)] for _ in range(B)]
    S_out = []
    for b in range(B):
        S_heads = []
        for hv in range(HV):
            h = hv // G
            S = [[S0[b][hv][i][j] for j in range(V)] for i in range(K)]
            for t in range(T):
                kk, qq, vv = k[b][t][h], q[b][t][h], v[b][t][hv]
                bt = beta[b][t][hv]
                A = [[(1 if i == j else 0) * d[b][t][hv][j] - bt * kk[i] * kk[j] * d[b][t][hv][j]
                      for j in range(K)] for i in range(K)]
                S = [[sum(A[i][m] * S[m][j] for m in range(K)) + bt * kk[i] * vv[j]
                      for j in range(V)] for i in range(K)]
                for j in range(V):
                    o[b][t][hv][j] = scale * sum(qq[i] * S[i][j] for i in range(K))
            S_heads.append(S)
        S_out.append(S_heads)
    return o, S_out


def pin_exact_rational(fwd):
    """Tiny case in exact rational arithmetic (decays are powers of 1/2)."""
    rng = np.random.default_rng(7)
    B, T, H, HV, K, V = 1, 3, 1, 2, 2, 3
    G = HV // H
    fr = lambda x: Fraction(int(round(x * 8)), 8)
    q = [[[[fr(x) for x in rng.standard_normal(K)] for _ in range(H)] for _ in range(T)] for _ in range(B)]
    k = [[[[fr(x) for x in rng.standard_normal(K)] for _ in range(H)] for _ in range(T)] for _ in range(B)]
    v = [[[[fr(x) for x in rng.standard_normal(V)] for _ in range(HV)] for _ in range(T)] for _ in range(B)]
    pw = rng.integers(0, 3, size=(B, T, HV, K))
    d = [[[[Fraction(1, 2 ** int(pw[b, t, hv, i])) for i in range(K)] for hv in range(HV)]
          for t in range(T)] for b in range(B)]
    beta = [[[Fraction(int(rng.integers(1, 4)), 4) for _ in range(HV)] for _ in range(T)] for _ in range(B)]
    S0 = [[[[fr(x) for x in rng.standard_normal(V)] for _ in range(K)] for _ in range(HV)] for _ in range(B)]
    scale = Fraction(1, 2)
    o_ex, S_ex = _exact_transition_form(q, k, v, d, beta, S0, scale, G)
    f = lambda a: np.array(a, dtype=np.float64)
    g = np.log(f(d))
    o, S = fwd(f(q), f(k), f(v), g, f(beta), 0.5, f(S0))
    return max(rel(o, f(o_ex)), rel(S, f(S_ex))) < 1e-13


def pin_beta_zero(fwd):
    """beta = 0: no writes, S_t = diag(exp(sum_{s<=t} g_s)) S0 exactly."""
    rng = np.random.default_rng(11)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 9, 2, 4, 5, 3, beta_zero=True)
    scale = 0.37
    o, S = fwd(q, k, v, g, beta, scale, S0)
    c = np.cumsum(g, axis=1)                                   # [B,T,HV,K]
    S_t = np.exp(c)[..., None] * S0[:, None]                   # [B,T,HV,K,V]
    qe = np.repeat(q, 2, axis=2)
    o_ref = scale * np.einsum("bthk,bthkv->bthv", qe, S_t)
    return max(rel(o, o_ref), rel(S, S_t[:, -1])) < 1e-13


def pin_projection(fwd):
    """g = 0, beta = 1, |k| = 1: the write makes k_t^T S_t = v_t exactly
    ("K3/notes/sections/sec-01.tex", delta-rule intuition: the residual is
    the correction that makes the state's prediction along k_t equal v_t)."""
    rng = np.random.default_rng(13)
    B, T, H, HV, K, V = 1, 6, 1, 1, 4, 3
    q, k, v, g, beta, S0 = rand_inputs(rng, B, T, H, HV, K, V)
    g[:] = 0.0
    beta[:] = 1.0
    ok = True
    for t in range(1, T + 1):
        _, S = fwd(q[:, :t], k[:, :t], v[:, :t], g[:, :t], beta[:, :t], 1.0, S0)
        pred = np.einsum("bhk,bhkv->bhv", k[:, t - 1], S)
        ok &= rel(pred, v[:, t - 1]) < 1e-13
    return ok


def pin_gqa(fwd):
    """Value head hv reads query/key head hv // G ("recurrent.py",
    repeat_interleave along dim 2): each value head of a grouped run equals
    a single-head run on its own q/k head."""
    rng = np.random.default_rng(17)
    B, T, H, HV, K, V = 1, 7, 2, 6, 3, 2
    q, k, v, g, beta, S0 = rand_inputs(rng, B, T, H, HV, K, V)
    o, S = fwd(q, k, v, g, beta, 0.5, S0)
    worst = 0.0
    for hv in range(HV):
        h = hv // (HV // H)
        o1, S1 = fwd(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, hv:hv + 1], g[:, :, hv:hv + 1],
                     beta[:, :, hv:hv + 1], 0.5, S0[:, hv:hv + 1])
        worst = max(worst, rel(o[:, :, hv:hv + 1], o1), rel(S[:, hv:hv + 1], S1))
    return worst < 1e-14


PINS = [pin_exact_rational, pin_beta_zero, pin_projection, pin_gqa]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_forward_pins(pin):
    assert pin(kda_forward)


# ---------------------------------------------------------------------------
# Planted mistakes: each variant of the forward loop below is wrong in one
# plausible way; at least one pin must reject it.
# ---------------------------------------------------------------------------

def _variant(mistake):
    def fwd(q, k, v, g, beta, scale, S0=None):
        B, T, H, K = q.shape
        HV, V = v.shape[2], v.shape[3]
        G = HV // H
        idx = np.arange(HV) % H if mistake == "gqa_modulo" else np.arange(HV) // G
        qe = q[:, :, idx] * (1.0 if mistake == "no_scale" else scale)
        ke = k[:, :, idx]
        S = np.zeros((B, HV, K, V)) if S0 is None else S0.copy()
        o = np.empty((B, T, HV, V))
        for t in range(T):
            dec = np.exp(g[:, t])[..., None]
            S_dec = S if mistake == "decay_after_read" else S * dec
            p = np.einsum("bhk,bhkv->bhv", ke[:, t], S_dec)
            r = (p - v[:, t]) if mistake == "residual_sign" else (v[:, t] - p)
            a = ke[:, t] if mistake == "no_beta" else beta[:, t][..., None] * ke[:, t]
            S_new = S_dec + a[..., :, None] * r[..., None, :]
            if mistake == "decay_after_read":
                S_new = S_new * dec
            read = S if mistake == "read_before_write" else S_new
            if mistake == "read_before_write":
                read = S_dec
            o[:, t] = np.einsum("bhk,bhkv->bhv", qe[:, t], read)
            S = S_new
        return o, S
    return fwd


@pytest.mark.parametrize("mistake", ["gqa_modulo", "no_scale", "decay_after_read",
                                     "residual_sign", "no_beta", "read_before_write"])
def test_pins_reject_planted_mistakes(mistake):
    assert all(p(_variant("none")) for p in PINS), "the correct variant must pass every pin"
    assert not all(p(_variant(mistake)) for p in PINS), f"no pin caught {mistake}"


# ---------------------------------------------------------------------------
# Further forward invariants
# ---------------------------------------------------------------------------

def test_linear_in_v_and_S0():
    rng = np.random.default_rng(19)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 11, 1, 2, 4, 5)
    _, _, v2, _, _, S02 = rand_inputs(rng, 2, 11, 1, 2, 4, 5)
    o1, S1 = kda_forward(q, k, v, g, beta, 0.3, S0)
    o2, S2 = kda_forward(q, k, v2, g, beta, 0.3, S02)
    o3, S3 = kda_forward(q, k, 2.5 * v - v2, g, beta, 0.3, 2.5 * S0 - S02)
    assert rel(o3, 2.5 * o1 - o2) < 1e-12 and rel(S3, 2.5 * S1 - S2) < 1e-12


def test_split_time_state_passing():
    """fwd over [0,T) equals fwd over [0,T1) then [T1,T) with S_{T1} passed on
    (the initial/final state arguments of ``naive_kda_fwd``)."""
    rng = np.random.default_rng(23)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 20, 2, 4, 3, 3)
    o, S = kda_forward(q, k, v, g, beta, 0.5, S0)
    oa, Sa = kda_forward(q[:, :7], k[:, :7], v[:, :7], g[:, :7], beta[:, :7], 0.5, S0)
    ob, Sb = kda_forward(q[:, 7:], k[:, 7:], v[:, 7:], g[:, 7:], beta[:, 7:], 0.5, Sa)
    assert rel(np.concatenate([oa, ob], 1), o) < 1e-14 and rel(Sb, S) < 1e-14


def _chunked_forward(q, k, v, g, beta, scale, S0, C):
    """Independent chunked restatement (triangular solve inside each chunk).

    Algebra of ``delta_recurrence`` in "research_layers.py" with erase = write
    = k, z = v and the write strength beta folded into the residual: inside a
    chunk with cumulative decay c_i = sum_{s<=i} g_s and entering state M,
    u_i = beta_i r_i solves (I + A) U = diag(beta)(V - (K.e^c) M) with
    A_ij = beta_i sum_f k_if k_jf exp(c_if - c_jf) for j < i; then
    o_i = scale [(q_i.e^{c_i}) M + sum_{j<=i} (sum_f q_if k_jf e^{c_if-c_jf}) u_j]
    and M' = diag(e^{c_C}) M + (K.e^{c_C - c})^T U.  Exponents are formed as
    pairwise differences, never as exp(-c).
    """
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    G = HV // H
    qe, ke = np.repeat(q, G, 2) * scale, np.repeat(k, G, 2)
    o = np.empty((B, T, HV, V))
    M = S0.copy()
    for s in range(0, T, C):
        e = min(s + C, T)
        n = e - s
        c = np.cumsum(g[:, s:e], axis=1)                         # [B,n,HV,K]
        Kc, Qc, Vc, bc = ke[:, s:e], qe[:, s:e], v[:, s:e], beta[:, s:e]
        D = np.exp(c[:, :, None] - c[:, None, :])                 # [B,i,j,HV,K]
        A = np.einsum("bihk,bjhk,bijhk->bhij", Kc, Kc, D) * np.moveaxis(bc, 1, 2)[..., None]
        P = np.einsum("bihk,bjhk,bijhk->bhij", Qc, Kc, D)
        low = np.tril(np.ones((n, n)), -1)
        A, P = A * low, P * np.tril(np.ones((n, n)))
        E = np.exp(c)
        rhs = np.moveaxis(bc, 1, 2)[..., None] * (np.moveaxis(Vc, 1, 2)
                                                   - np.einsum("bihk,bhkv->bhiv", Kc * E, M))
        U = np.linalg.solve(np.eye(n) + A, rhs)
        o[:, s:e] = np.moveaxis(np.einsum("bihk,bhkv->bhiv", Qc * E, M) + P @ U, 2, 1)
        Ed = np.exp(c[:, -1:] - c)
        M = np.exp(c[:, -1])[..., None] * M + np.einsum("bihk,bhiv->bhkv", Kc * Ed, U)
    return o, M


@pytest.mark.parametrize("C", [1, 4, 16])
def test_chunked_restatement_matches_tokenwise(C):
    rng = np.random.default_rng(29)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 37, 2, 4, 6, 5)
    o, S = kda_forward(q, k, v, g, beta, 0.4, S0)
    oc, Sc = _chunked_forward(q, k, v, g, beta, 0.4, S0, C)
    assert rel(oc, o) < 1e-12 and rel(Sc, S) < 1e-12


def test_gate_bound_long_sequence_stays_finite():
    """At the production gate bound (-5 per step) the decay of a 64-step span
    reaches exp(-320); the oracle never forms exp(+|c|), so it stays finite."""
    rng = np.random.default_rng(31)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 300, 1, 1, 4, 4)
    g[:] = -5.0
    o, S = kda_forward(q, k, v, g, beta, 0.5, S0)
    assert np.isfinite(o).all() and np.isfinite(S).all()


# ---------------------------------------------------------------------------
# Decode step
# ---------------------------------------------------------------------------

def test_decode_step_equals_forward_and_sequence():
    rng = np.random.default_rng(37)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 5, 2, 4, 3, 4)
    o, S = kda_forward(q, k, v, g, beta, 0.6, S0)
    St = S0.copy()
    for t in range(5):
        ot, St_new = kda_decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], St, 0.6)
        assert rel(ot, o[:, t]) < 1e-14
        St = St_new
    assert rel(St, S) < 1e-14


def test_decode_prefix_snapshot_restore():
    """"kimi_k3_host/kda.rs", test prefix_hit_wrong_slot_diverges: decoding
    from the state saved after the prefix equals sequential decoding exactly;
    decoding from an earlier snapshot diverges."""
    rng = np.random.default_rng(41)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 3, 1, 1, 2, 2)
    S0[:] = 0.0
    snaps, S = [], S0
    for t in range(2):
        _, S = kda_decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, 0.7)
        snaps.append(S.copy())
    y_seq, _ = kda_decode_step(q[:, 2], k[:, 2], v[:, 2], g[:, 2], beta[:, 2], S, 0.7)
    y_hit, _ = kda_decode_step(q[:, 2], k[:, 2], v[:, 2], g[:, 2], beta[:, 2], snaps[1], 0.7)
    y_wrong, _ = kda_decode_step(q[:, 2], k[:, 2], v[:, 2], g[:, 2], beta[:, 2], snaps[0], 0.7)
    assert np.array_equal(y_hit, y_seq)
    assert np.abs(y_wrong - y_hit).max() > 1e-4


def test_decode_worked_example_from_page():
    """Inputs of "kimi_k3_host/kda.rs" test beta_zero_is_sigmoid_half_not_zero
    (fixture in tests/golden).  From a zero state one step gives
    o = scale * sigmoid(0) * (q_hat . k_hat) * v; the saturated logit differs."""
    with open(os.path.join(GOLDEN, "decode_beta_logit_zero.json")) as f:
        fx = json.load(f)
    d, eps = fx["head_dim"], fx["l2_eps"]
    qkv = np.array(fx["qkv"])
    qr, kr, v = qkv[:d], qkv[d:2 * d], qkv[2 * d:]
    qh, kh = qr / math.sqrt((qr ** 2).sum() + eps), kr / math.sqrt((kr ** 2).sum() + eps)
    scale = 1.0 / math.sqrt(d)
    g = np.array(fx["gate"])[None, None]
    S = np.zeros((1, 1, d, d))

    def step(logit):
        beta = np.array([[1.0 / (1.0 + math.exp(-logit))]])
        o, _ = kda_decode_step(qh[None, None], kh[None, None], v[None, None], g, beta, S, scale)
        return o[0, 0]

    o_half = step(fx["beta_logit"][0])
    expected = scale * 0.5 * float(qh @ kh) * v
    assert np.abs(o_half - expected).max() < 1e-15
    assert np.abs(o_half).max() > 1e-6
    assert not np.array_equal(o_half, step(fx["beta_logit_saturated"][0]))


# ---------------------------------------------------------------------------
# Backward
# ---------------------------------------------------------------------------

def _loss(inp, dO, dS_T, scale):
    o, S = kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], scale, inp["S0"])
    return float((o * dO).sum() + (S * dS_T).sum())


@pytest.mark.parametrize("shape", [(1, 5, 1, 2, 3, 2), (2, 4, 2, 2, 2, 3)])
def test_backward_matches_finite_differences(shape):
    """Every gradient, dS0 included, against central differences in float64
    ("recurrent.py" notes that the float64 path exists for gradient checks)."""
    B, T, H, HV, K, V = shape
    rng = np.random.default_rng(43)
    q, k, v, g, beta, S0 = rand_inputs(rng, B, T, H, HV, K, V)
    dO = rng.standard_normal((B, T, HV, V))
    dS_T = rng.standard_normal((B, HV, K, V))
    scale = 0.45
    grads = kda_backward(q, k, v, g, beta, scale, S0, dO, dS_T, segment=3)
    inp = dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0)
    h = 1e-6
    for name, grad in zip(["q", "k", "v", "g", "beta", "S0"], grads):
        fd = np.zeros_like(inp[name])
        for idx in np.ndindex(*inp[name].shape):
            x0 = inp[name][idx]
            inp[name][idx] = x0 + h
            lp = _loss(inp, dO, dS_T, scale)
            inp[name][idx] = x0 - h
            lm = _loss(inp, dO, dS_T, scale)
            inp[name][idx] = x0
            fd[idx] = (lp - lm) / (2 * h)
        assert rel(grad, fd) < 1e-7, name


def test_backward_beta_zero_closed_form():
    """beta = 0: S_t = D_t S0 with D_t = diag(exp(sum_{s<=t} g_s)), so
    dS0 = D_T dS_T + sum_t D_t (scale q_t) (x) dO_t, dq_t = scale (D_t S0) dO_t
    summed over the group, dv = dk = 0, and
    dg_s = sum_{t>=s} scale q_t (.) (D_t S0 dO_t) + rowsum(D_T S0 (.) dS_T)."""
    rng = np.random.default_rng(47)
    B, T, H, HV, K, V = 1, 6, 1, 2, 3, 4
    q, k, v, g, beta, S0 = rand_inputs(rng, B, T, H, HV, K, V, beta_zero=True)
    dO = rng.standard_normal((B, T, HV, V))
    dS_T = rng.standard_normal((B, HV, K, V))
    scale = 0.8
    dq, dk, dv, dg, dbeta, dS0 = kda_backward(q, k, v, g, beta, scale, S0, dO, dS_T)
    qe = np.repeat(q, HV // H, 2)
    D = np.exp(np.cumsum(g, 1))                                   # [B,T,HV,K]
    DS = D[..., None] * S0[:, None]                               # [B,T,HV,K,V]
    dS0_ref = D[:, -1][..., None] * dS_T + np.einsum("bthk,bthv->bhkv", D * qe * scale, dO)
    dq_ref = scale * np.einsum("bthkv,bthv->bthk", DS, dO).reshape(B, T, H, HV // H, K).sum(3)
    per_t = scale * qe * np.einsum("bthkv,bthv->bthk", DS, dO)    # d o / d c_t contributions
    dc = per_t.copy()
    dc[:, -1] += (DS[:, -1] * dS_T).sum(-1)
    dg_ref = np.flip(np.cumsum(np.flip(dc, 1), 1), 1)
    assert rel(dS0, dS0_ref) < 1e-13
    assert rel(dq, dq_ref) < 1e-13
    assert np.abs(dv).max() == 0.0 and np.abs(dk).max() == 0.0
    assert rel(dg, dg_ref) < 1e-13
    assert np.abs(dbeta).max() > 0.0   # beta still has a gradient at beta = 0


def test_backward_segment_length_does_not_matter():
    rng = np.random.default_rng(53)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 13, 1, 3, 4, 3)
    dO = rng.standard_normal((1, 13, 3, 3))
    a = kda_backward(q, k, v, g, beta, 0.5, S0, dO, None, segment=64)
    b = kda_backward(q, k, v, g, beta, 0.5, S0, dO, None, segment=4)
    for x, y in zip(a, b):
        assert rel(x, y) < 1e-13
