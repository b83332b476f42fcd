"""Pins for the oracle of the asymmetric erase/write delta recurrence
("research_layers.py", ``delta_token_reference`` / ``delta_recurrence``):
the page's chunk solve (an independent formulation the page states is
algebraically identical), the KDA special case (e = beta k, z = beta v)
against the pinned KDA oracle, exact rational arithmetic of the transition
form, the pure-write closed form (e = 0) and the query-head grouping.
Planted mistakes in the token loop fail at least one pin.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

from oracle import kda_forward
from oracle.kda_erase import erase_chunked, erase_forward


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


def rand(rng, B, T, HQ, HV, K, V, gscale=0.3):
    q = rng.standard_normal((B, T, HQ, K))
    k = rng.standard_normal((B, T, HV, K)) / np.sqrt(K)
    e = rng.standard_normal((B, T, HV, K)) / np.sqrt(K)
    z = rng.standard_normal((B, T, HV, V))
    g = -gscale / (1.0 + np.exp(-rng.standard_normal((B, T, HV, K))))
    S0 = 0.3 * rng.standard_normal((B, HV, K, V))
    return q, k, e, z, g, S0


def pin_chunk_solve(fwd):
    rng = np.random.default_rng(1)
    q, k, e, z, g, S0 = rand(rng, 2, 11, 4, 2, 3, 5)
    o, S = fwd(q, k, e, z, g, 0.7, S0)
    oc, Sc = erase_chunked(q, k, e, z, g, 0.7, S0, C=4)
    return rel(o, oc) < 1e-12 and rel(S, Sc) < 1e-12


def pin_kda_special_case(fwd):
    rng = np.random.default_rng(2)
    B, T, H, K, V = 2, 6, 2, 3, 4
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, V))
    g = -0.5 / (1.0 + np.exp(-rng.standard_normal((B, T, H, K))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.3 * rng.standard_normal((B, H, K, V))
    o_ref, S_ref = kda_forward(q, k, v, g, beta, 0.8, S0)
    o, S = fwd(q, k, beta[..., None] * k, beta[..., None] * v, g, 0.8, S0)
    return rel(o, o_ref) < 1e-13 and rel(S, S_ref) < 1e-13


def pin_exact_rational(fwd):
    """S_t = (I - k e^T) D S_{t-1} + k z^T, o_t = S_t^T q, in Fractions with
    decays given exactly (g = log of a rational)."""
    rng = np.random.default_rng(3)
    T, K, V = 3, 2, 2
    fr = lambda x: Fraction(int(round(x * 8)), 8)
    q = [[fr(x) for x in rng.standard_normal(K)] for _ in range(T)]
    k = [[fr(x) for x in rng.standard_normal(K)] for _ in range(T)]
    e = [[fr(x) for x in rng.standard_normal(K)] for _ in range(T)]
    z = [[fr(x) for x in rng.standard_normal(V)] for _ in range(T)]
    d = [[Fraction(rng.integers(1, 8), 8) for _ in range(K)] for _ in range(T)]
    S = [[Fraction(0)] * V for _ in range(K)]
    o_exact = []
    for t in range(T):
        Sd = [[d[t][f] * S[f][n] for n in range(V)] for f in range(K)]
        old = [sum(e[t][f] * Sd[f][n] for f in range(K)) for n in range(V)]
        S = [[Sd[f][n] + k[t][f] * (z[t][n] - old[n]) for n in range(V)] for f in range(K)]
        o_exact.append([sum(q[t][f] * S[f][n] for f in range(K)) for n in range(V)])
    arr = lambda x: np.array(x, dtype=np.float64)[None, :, None]
    g = np.log(np.array(d, dtype=np.float64))[None, :, None]
    o, S_T = fwd(arr(q), arr(k), arr(e), arr(z), g, 1.0, None)
    return (np.abs(o[0, :, 0] - np.array(o_exact, dtype=np.float64)).max() < 1e-14
            and np.abs(S_T[0, 0] - np.array(S, dtype=np.float64)).max() < 1e-14)


def pin_pure_write(fwd):
    """e = 0: nothing is erased, S_T = D_T..D_1 S0 + sum_t D_T..D_{t+1} k_t z_t^T."""
    rng = np.random.default_rng(4)
    q, k, e, z, g, S0 = rand(rng, 1, 5, 2, 2, 3, 2)
    e[:] = 0.0
    _, S = fwd(q, k, e, z, g, 1.0, S0)
    cum = np.cumsum(g[:, ::-1], axis=1)[:, ::-1]   # sum_{s>=t} g_s
    ref = np.exp(cum[:, 0])[..., None] * S0
    for t in range(5):
        after = np.exp(cum[:, t + 1]) if t + 1 < 5 else np.ones_like(cum[:, 0])
        ref = ref + after[..., None] * (k[:, t][..., :, None] * z[:, t][..., None, :])
    return rel(S, ref) < 1e-13


def pin_query_groups(fwd):
    """Query head hq reads state head hq // QG: each query head alone, with
    its own state head, gives the same output."""
    rng = np.random.default_rng(5)
    q, k, e, z, g, S0 = rand(rng, 1, 7, 6, 2, 3, 4)
    o, _ = fwd(q, k, e, z, g, 0.5, S0)
    worst = 0.0
    for hq in range(6):
        hv = hq // 3
        o1, _ = fwd(q[:, :, hq:hq + 1], k[:, :, hv:hv + 1], e[:, :, hv:hv + 1], z[:, :, hv:hv + 1],
                    g[:, :, hv:hv + 1], 0.5, S0[:, hv:hv + 1])
        worst = max(worst, rel(o[:, :, hq:hq + 1], o1))
    return worst < 1e-14


PINS = [pin_chunk_solve, pin_kda_special_case, pin_exact_rational, pin_pure_write, pin_query_groups]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_erase_pins(pin):
    assert pin(erase_forward)


def _variant(mistake):
    def fwd(q, k, e, z, g, scale=1.0, S0=None):
        B, T, HQ, K = q.shape
        HV, V = k.shape[2], z.shape[3]
        QG = HQ // HV
        S = np.zeros((B, HV, K, V)) if S0 is None else S0.copy()
        idx = np.arange(HQ) % HV if mistake == "groups_modulo" else np.arange(HQ) // QG
        o = np.empty((B, T, HQ, V))
        for t in range(T):
            rd, wr = (k[:, t], e[:, t]) if mistake == "erase_write_swapped" else (e[:, t], k[:, t])
            Sd = S if mistake == "decay_after_erase" else np.exp(g[:, t])[..., None] * S
            old = np.einsum("bhf,bhfv->bhv", rd, Sd)
            S_new = Sd + wr[..., :, None] * (z[:, t] - old)[..., None, :]
            if mistake == "decay_after_erase":
                S_new = np.exp(g[:, t])[..., None] * S_new
            read = Sd if mistake == "read_before_write" else S_new
            o[:, t] = np.einsum("bhf,bhfv->bhv", scale * q[:, t], read[:, idx])
            S = S_new
        return o, S
    return fwd


@pytest.mark.parametrize("mistake", ["erase_write_swapped", "groups_modulo", "decay_after_erase",
                                     "read_before_write"])
def test_erase_pins_reject_planted_mistakes(mistake):
    assert all(p(_variant("none")) for p in PINS), "the correct variant must pass every pin"
    assert not all(p(_variant(mistake)) for p in PINS), f"no pin caught {mistake}"
