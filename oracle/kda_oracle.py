"""Float64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.

TEST INFRASTRUCTURE ONLY.  This module is imported by the test suite, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``; the
product path (the CUDA library and its Python binding) never imports, links or
executes it, and it imports nothing from the product package.

It is deliberately the plainest possible restatement of the method: a
token-by-token loop over time, vectorised only over the independent
(batch, value-head) pairs, in float64, with no chunking, blocking or
re-association.  Every function names the passage it follows.

Sources (page title, then the section / function on it):

* "K3/kda/ops/reference/recurrent.py" -- module docstring (the per-step
  formula and the backward derivation notes), ``naive_kda_fwd`` (the forward
  loop), ``KDAFunction.backward`` (the BPTT loop, the grouped-head reduction
  and the scale on dq).
* "K3/notes/sections/sec-01.tex", section "KDA recurrence core", subsection
  of the step-by-step formulas (shape table and the four-step update:
  decay, residual, write, read) and the broadcast note on exp(g).
* "kimi_k3_host/kda.rs", ``kda_recurrent_step`` (single-token decode on a
  state updated in place, layout recurrent[h][k][v]).

Conventions (all arrays are numpy float64; the caller upcasts whatever bits
the GPU consumed, so both sides see identical inputs):

    q, k   [B, T, H,  K]    query / key, H query-key heads
    v      [B, T, HV, V]    value, HV value heads, HV % H == 0
    g      [B, T, HV, K]    log-space per-channel decay (any finite value)
    beta   [B, T, HV]       write strength, already in (0, 1)
    S0     [B, HV, K, V]    initial state (None means zeros)
    scale  float            multiplies q (default 1/sqrt(K) is the caller's)

Grouped heads: value head hv reads query/key head hv // G with G = HV // H
(a repeat-interleave along the head axis), and the backward sums the G copies.

Readings taken where the pages are silent or inconsistent:

* the readout uses the state *after* the rank-1 write (all three pages agree);
* beta is taken as given (post-sigmoid); L2 normalisation of q/k and the gate
  formula are input preparation, not part of the recurrence;
* the backward follows the code of ``KDAFunction.backward`` (dv = +dr), not
  the docstring's "dv = -dr" slip, and additionally returns dS0, the adjoint
  of the initial state left in the accumulator after the step at t = 0
  (the page computes it and then drops it); an optional upstream dS_T seeds
  that accumulator exactly as the page's ``dS`` argument does.
"""
from __future__ import annotations

import numpy as np

__all__ = ["kda_forward", "kda_backward", "kda_decode_step", "expand_heads"]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def expand_heads(x, hv):
    """Repeat-interleave the head axis (axis 2) from H to ``hv`` heads.

    "K3/kda/ops/reference/recurrent.py", ``naive_kda_fwd``: q and k are
    expanded with repeat_interleave(G, dim=2), so value head hv uses query/key
    head hv // G.
    """
    x = _f64(x)
    h = x.shape[2]
    if hv % h:
        raise ValueError(f"HV={hv} is not a multiple of H={h}")
    return np.repeat(x, hv // h, axis=2)


def _check(q, k, v, g, beta):
    B, T, H, K = q.shape
    if k.shape != q.shape:
        raise ValueError("q and k must have the same shape [B,T,H,K]")
    if v.ndim != 4 or v.shape[:2] != (B, T):
        raise ValueError("v must be [B,T,HV,V]")
    HV, V = v.shape[2], v.shape[3]
    if HV % H:
        raise ValueError("HV must be a multiple of H")
    if g.shape != (B, T, HV, K):
        raise ValueError("g must be [B,T,HV,K]")
    if beta.shape != (B, T, HV):
        raise ValueError("beta must be [B,T,HV]")
    return B, T, H, HV, K, V


def kda_forward(q, k, v, g, beta, scale, S0=None):
    """Token-by-token KDA forward.  Returns (o [B,T,HV,V], S_T [B,HV,K,V]).

    Follows ``naive_kda_fwd`` in "K3/kda/ops/reference/recurrent.py" and the
    four steps of "K3/notes/sections/sec-01.tex" ("KDA recurrence core"):

        S_dec = exp(g_t) (.) S_{t-1}          decay, exp(g_t) broadcast along V
        p_t   = k_t . S_dec                   read the old prediction
        r_t   = v_t - p_t                     delta-rule residual
        S_t   = S_dec + (beta_t k_t) (x) r_t  rank-1 write
        o_t   = (scale q_t) . S_t             readout after the write
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    B, T, H, HV, K, V = _check(q, k, v, g, beta)
    qe = expand_heads(q, HV) * scale
    ke = expand_heads(k, HV)
    S = np.zeros((B, HV, K, V)) if S0 is None else _f64(S0).copy()
    o = np.empty((B, T, HV, V))
    for t in range(T):
        q_t, k_t, v_t = qe[:, t], ke[:, t], v[:, t]
        S_dec = S * np.exp(g[:, t])[..., None]
        p_t = np.einsum("bhk,bhkv->bhv", k_t, S_dec)
        r_t = v_t - p_t
        a_t = beta[:, t][..., None] * k_t
        S = S_dec + a_t[..., :, None] * r_t[..., None, :]
        o[:, t] = np.einsum("bhk,bhkv->bhv", q_t, S)
    return o, S


def kda_decode_step(q, k, v, g, beta, S, scale):
    """One decode token on a state.  Returns (o [B,HV,V], S_new [B,HV,K,V]).

    "kimi_k3_host/kda.rs", ``kda_recurrent_step``: per head the state
    recurrent[h][kd][vd] is decayed row by row, the residual is formed from
    the column sums against k, the rank-1 update is added and the output is
    the q-weighted column sum times scale.  Here q, k are [B,H,K], v is
    [B,HV,V], g is [B,HV,K], beta is [B,HV] (already post-sigmoid; the Rust
    step applies the sigmoid and the q/k L2 normalisation itself, which this
    library leaves to input preparation).  The input S is not modified.
    """
    q, k, v, g, beta, S = map(_f64, (q, k, v, g, beta, S))
    HV = v.shape[1]
    qe = expand_heads(q[:, None], HV)[:, 0] * scale
    ke = expand_heads(k[:, None], HV)[:, 0]
    S_new = S * np.exp(g)[..., None]
    kv = np.einsum("bhk,bhkv->bhv", ke, S_new)
    delta = (v - kv) * beta[..., None]
    S_new = S_new + ke[..., :, None] * delta[..., None, :]
    o = np.einsum("bhk,bhkv->bhv", qe, S_new)
    return o, S_new


def kda_backward(q, k, v, g, beta, scale, S0, dO, dS_T=None, segment=64):
    """Back-propagation through time for ``kda_forward``.

    Returns (dq [B,T,H,K], dk [B,T,H,K], dv [B,T,HV,V], dg [B,T,HV,K],
    dbeta [B,T,HV], dS0 [B,HV,K,V]).

    Follows ``KDAFunction.backward`` in "K3/kda/ops/reference/recurrent.py",
    running t = T-1 ... 0 with an accumulator dS for the gradient reaching S_t:

        dS   += q~_t (x) do_t            (q~ = scale q, the expanded query)
        dq~_t = S_t do_t
        da_t  = dS r_t ;  dr_t = a_t^T dS
        dbeta_t = k_t . da_t
        dk_t  = beta_t da_t - S_dec,t dr_t
        dv_t  = dr_t
        dS_dec = dS - k_t (x) dr_t
        dg_t  = sum_v S_dec,t (.) dS_dec
        dS    = exp(g_t) (.) dS_dec

    then dq = scale * (sum of the G expanded copies of dq~) and dk likewise
    summed over its copies.  The page keeps every S_dec,t; to stay within host
    memory this restatement keeps the state every ``segment`` steps and
    recomputes the forward inside a segment before walking it backwards (the
    arithmetic of each step is unchanged).  dS_T (the upstream gradient of the
    final state) seeds dS; dS0 is dS after the step at t = 0.
    """
    q, k, v, g, beta, dO = map(_f64, (q, k, v, g, beta, dO))
    B, T, H, HV, K, V = _check(q, k, v, g, beta)
    G = HV // H
    qe = expand_heads(q, HV) * scale
    ke = expand_heads(k, HV)
    S = np.zeros((B, HV, K, V)) if S0 is None else _f64(S0).copy()

    checkpoints = {}
    for t in range(T):
        if t % segment == 0:
            checkpoints[t] = S.copy()
        S_dec = S * np.exp(g[:, t])[..., None]
        r_t = v[:, t] - np.einsum("bhk,bhkv->bhv", ke[:, t], S_dec)
        S = S_dec + (beta[:, t][..., None] * ke[:, t])[..., :, None] * r_t[..., None, :]

    dqe = np.zeros((B, T, HV, K))
    dke = np.zeros((B, T, HV, K))
    dv = np.zeros((B, T, HV, V))
    dg = np.zeros((B, T, HV, K))
    dbeta = np.zeros((B, T, HV))
    dS = np.zeros((B, HV, K, V)) if dS_T is None else _f64(dS_T).copy()

    for s0 in sorted(checkpoints, reverse=True):
        s1 = min(s0 + segment, T)
        S = checkpoints[s0].copy()
        S_decs, r_ts, S_ts = [], [], []
        for t in range(s0, s1):
            S_dec = S * np.exp(g[:, t])[..., None]
            r_t = v[:, t] - np.einsum("bhk,bhkv->bhv", ke[:, t], S_dec)
            S = S_dec + (beta[:, t][..., None] * ke[:, t])[..., :, None] * r_t[..., None, :]
            S_decs.append(S_dec)
            r_ts.append(r_t)
            S_ts.append(S)
        for i in range(s1 - s0 - 1, -1, -1):
            t = s0 + i
            S_dec, r_t, S_t = S_decs[i], r_ts[i], S_ts[i]
            q_t, k_t, do_t = qe[:, t], ke[:, t], dO[:, t]
            b_t = beta[:, t][..., None]
            a_t = b_t * k_t
            dS = dS + q_t[..., :, None] * do_t[..., None, :]
            dqe[:, t] = np.einsum("bhv,bhkv->bhk", do_t, S_t)
            da_t = np.einsum("bhv,bhkv->bhk", r_t, dS)
            dr_t = np.einsum("bhk,bhkv->bhv", a_t, dS)
            dbeta[:, t] = np.einsum("bhk,bhk->bh", k_t, da_t)
            dke[:, t] = b_t * da_t - np.einsum("bhv,bhkv->bhk", dr_t, S_dec)
            dv[:, t] = dr_t
            dS_dec = dS - k_t[..., :, None] * dr_t[..., None, :]
            dg[:, t] = np.einsum("bhkv,bhkv->bhk", S_dec, dS_dec)
            dS = np.exp(g[:, t])[..., None] * dS_dec

    dq = dqe.reshape(B, T, H, G, K).sum(axis=3) * scale
    dk = dke.reshape(B, T, H, G, K).sum(axis=3)
    return dq, dk, dv, dg, dbeta, dS
