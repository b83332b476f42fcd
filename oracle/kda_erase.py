"""Float64 CPU oracle of the asymmetric erase/write delta recurrence.

TEST INFRASTRUCTURE ONLY.  This module is imported by the test suite, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``; the
product path (the CUDA library and its Python binding) never imports, links or
executes it, and it imports nothing from the product package.

Source: "research_layers.py" -- ``delta_token_reference`` (the token loop)
and the docstring of ``delta_recurrence`` (the update it states and the chunk
solve that is algebraically identical to it).  Per state head the recurrence
keeps a K x V memory S and, for t = 0 .. T-1:

    S_bar = diag(exp(g_t)) S_{t-1}                    decay
    S_t   = S_bar + k_t (z_t - e_t^T S_bar)^T         erase along e_t, write along k_t
    o_t   = (scale q_t)^T S_t                         readout after the write

with a separate erase vector e (the page's ``erase``) and write vector k
(the page's ``k``).  KDA is the case e = beta k, z = beta v.

Heads follow the page's layer: the memory, k, e, z and g have HV state
("key/value") heads; q has HQ = HV * QG query heads, and query head hq reads
state head hq // QG (the memory is repeat-interleaved along the head axis).

Shapes (numpy float64, [batch, time, head, feature] like the rest of this
library; the page orders them [batch, head, time, feature]):

    q [B, T, HQ, K]   k, e, g [B, T, HV, K]   z [B, T, HV, V]   S0 [B, HV, K, V]

Readings: ``scale`` multiplies q (the page's loop has none: scale = 1
reproduces it); the page's chunk-size limit (<= 32) belongs to its bounded
decay factoring, not to the recurrence.
"""
from __future__ import annotations

import numpy as np

__all__ = ["erase_forward", "erase_chunked"]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _check(q, k, e, z, g):
    B, T, HQ, K = q.shape
    HV = k.shape[2]
    if k.shape != (B, T, HV, K) or e.shape != k.shape or g.shape != k.shape:
        raise ValueError("k, e and g must be [B,T,HV,K]")
    if z.ndim != 4 or z.shape[:3] != (B, T, HV):
        raise ValueError("z must be [B,T,HV,V]")
    if HQ % HV:
        raise ValueError("HQ must be a multiple of HV")
    return B, T, HQ, HV, K, z.shape[3]


def erase_forward(q, k, e, z, g, scale=1.0, S0=None):
    """Token loop of ``delta_token_reference``.  Returns (o [B,T,HQ,V], S_T [B,HV,K,V])."""
    q, k, e, z, g = map(_f64, (q, k, e, z, g))
    B, T, HQ, HV, K, V = _check(q, k, e, z, g)
    QG = HQ // HV
    S = np.zeros((B, HV, K, V)) if S0 is None else _f64(S0).copy()
    o = np.empty((B, T, HQ, V))
    for t in range(T):
        S = np.exp(g[:, t])[..., None] * S
        old = np.einsum("bhf,bhfv->bhv", e[:, t], S)
        S = S + k[:, t][..., :, None] * (z[:, t] - old)[..., None, :]
        o[:, t] = np.einsum("bhf,bhfv->bhv", scale * q[:, t], np.repeat(S, QG, axis=1))
    return o, S


def erase_chunked(q, k, e, z, g, scale=1.0, S0=None, C=16):
    """The chunk solve of ``delta_recurrence``, restated for checking the
    token loop (the page states the two are algebraically identical).  Per
    chunk, with the in-chunk cumulative decay d_i = exp(sum_{s<=i} g_s):
    write = k / d, read = e * d, U = (I + tril(read write^T, -1))^{-1}
    (z - read S), o = (q d) S + tril((q d) write^T) U, and the memory leaving
    the chunk is d_last * (S + write^T U).  (Without the page's bounded-decay
    safeguard: for the small decays of the checks only.)"""
    q, k, e, z, g = map(_f64, (q, k, e, z, g))
    B, T, HQ, HV, K, V = _check(q, k, e, z, g)
    QG = HQ // HV
    S = np.zeros((B, HV, K, V)) if S0 is None else _f64(S0).copy()
    o = np.empty((B, T, HQ, V))
    for t0 in range(0, T, C):
        t1 = min(t0 + C, T)
        n = t1 - t0
        d = np.exp(np.cumsum(g[:, t0:t1], axis=1))                 # [B, n, HV, K]
        write = k[:, t0:t1] / d
        read = e[:, t0:t1] * d
        inter = np.einsum("bihf,bjhf->bhij", read, write)
        system = np.tril(inter, -1) + np.eye(n)
        rhs = np.transpose(z[:, t0:t1], (0, 2, 1, 3)) - np.einsum("bihf,bhfv->bhiv", read, S)
        U = np.linalg.solve(system, rhs)                             # [B, HV, n, V]
        qd = scale * q[:, t0:t1] * np.repeat(d, QG, axis=2)
        wr = np.repeat(write, QG, axis=2)
        Ur = np.repeat(U, QG, axis=1)
        old = np.einsum("bihf,bhfv->bihv", qd, np.repeat(S, QG, axis=1))
        within = np.tril(np.einsum("bihf,bjhf->bhij", qd, wr))
        o[:, t0:t1] = old + np.transpose(np.einsum("bhij,bhjv->bhiv", within, Ur), (0, 2, 1, 3))
        S = np.transpose(d[:, -1], (0, 1, 2))[..., None] * (S + np.einsum("bjhf,bhjv->bhfv", write, U))
    return o, S
