"""Float64 CPU oracle of the preparation around the KDA recurrence: the short
causal convolution with SiLU, the per-row L2 normalisation of q and k, the
decay gate, the sigmoid on beta, and the full-rank output gate.

TEST INFRASTRUCTURE ONLY.  This module is imported by the test suite, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``; the
product path (the CUDA library and its Python binding) never imports, links or
executes it, and it imports nothing from the product package.

Sources (page title, then the function on it): "kimi_k3_host/kda.rs" --
``conv_update`` (one token of the depthwise causal convolution: shift the
per-channel window, append the new input, weighted sum, SiLU), ``softplus``,
``bounded_gate`` (the decay gate from its pre-activation), ``l2norm_rows``
with ``KDA_L2_EPS`` (eps added to the sum of squares inside the square root),
``kda_recurrent_step`` (L2-normalised q and k, sigmoid on the beta input,
then the recurrence step), ``full_rank_output_gate`` (RMS normalisation of
each head row times the sigmoid of the gate row) and ``kda_decode_token``
(convolution, then the recurrent step).

Conventions (numpy float64):

    q, k raw    [B, T, H,  K]    pre-normalisation query / key
    v           [B, T, HV, V]
    z           [B, T, HV, K]    gate pre-activation
    A_log       [HV]             per-head log decay rate
    dt_bias     [HV, K]          per-(head, channel) gate bias
    beta_logit  [B, T, HV]
    out_gate    [B, T, HV, V]    output-gate pre-activation
    conv weights [C, W], conv state [B, C, W]: channel c's window, oldest
    input first, newest in slot W - 1; channels in the order q | k | v
    (H*K query channels, H*K key channels, HV*V value channels).

Readings taken where the page is silent:

* the gate's lower bound 0 selects the unbounded form -exp(A_log) softplus(x)
  (the page turns a zero lower bound into "no bound" when it reads the model
  configuration);
* with grouped heads (HV > H) the convolution has separate channels for the
  H query/key heads and the HV value heads; the page has H = HV;
* the output gate's eps is a parameter on the page with no value given; the
  default here is the L2 eps, 1e-6;
* the prefill form of the convolution applies the per-token update to every
  step in order, starting from the given window (zeros when none).
"""
from __future__ import annotations

import numpy as np

from .kda_oracle import kda_decode_step, kda_forward

__all__ = ["L2_EPS", "sigmoid", "softplus", "l2norm_rows", "kda_gate", "conv_update", "short_conv_silu",
           "short_conv_qkv", "output_gate", "kda_forward_prepared", "kda_decode_token"]

L2_EPS = 1e-6  # "kimi_k3_host/kda.rs", KDA_L2_EPS


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    """Logistic function, evaluated without overflow for either sign."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def softplus(x):
    """"kimi_k3_host/kda.rs", ``softplus``: max(x, 0) + log1p(exp(-|x|))."""
    x = _f64(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def l2norm_rows(x, eps=L2_EPS):
    """"kimi_k3_host/kda.rs", ``l2norm_rows``: each row (last axis) times
    1 / sqrt(sum of squares + eps)."""
    x = _f64(x)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def kda_gate(z, A_log, dt_bias, lower_bound):
    """"kimi_k3_host/kda.rs", ``bounded_gate``: with decay = exp(A_log[h]) and
    x = z + dt_bias[h], the log-space decay is lower_bound * sigmoid(decay x)
    for a (negative) lower bound, else -decay * softplus(x).

    z is [..., HV, K], A_log [HV], dt_bias [HV, K].
    """
    z, A_log, dt_bias = _f64(z), _f64(A_log), _f64(dt_bias)
    decay = np.exp(A_log)[:, None]
    x = z + dt_bias
    if lower_bound:
        return float(lower_bound) * sigmoid(decay * x)
    return -decay * softplus(x)


def conv_update(state, x, w):
    """"kimi_k3_host/kda.rs", ``conv_update``: one token.  Every channel's
    window drops its oldest input and appends x; the output is the weighted
    sum of the window passed through SiLU (acc * sigmoid(acc)).

    state [..., C, W], x [..., C], w [C, W].  Returns (y [..., C], new state);
    the input state is not modified.
    """
    state, x, w = _f64(state), _f64(x), _f64(w)
    new = np.concatenate([state[..., 1:], x[..., None]], axis=-1)
    acc = (new * w).sum(axis=-1)
    return acc * sigmoid(acc), new


def short_conv_silu(x, w, state=None):
    """The convolution over a whole sequence: y_t = SiLU(sum_j w[c, j] u_{t-W+1+j})
    where u is the sequence preceded by the window's W - 1 newest inputs
    (the state's oldest slot drops out at the first step, as in
    ``conv_update``).  Returns (y [B, T, C], the window after the last step).

    Written as a sliding window over the padded sequence, not as repeated
    ``conv_update`` calls, so that the two forms check each other.
    """
    x, w = _f64(x), _f64(w)
    B, T, C = x.shape
    W = w.shape[1]
    st = np.zeros((B, C, W)) if state is None else _f64(state)
    full = np.concatenate([np.transpose(st, (0, 2, 1)), x], axis=1)  # [B, W + T, C], time order
    y = np.empty((B, T, C))
    for t in range(T):  # step t sees inputs t - W + 1 .. t, i.e. full[t + 1 .. t + W]
        acc = (full[:, t + 1:t + 1 + W, :] * w.T[None]).sum(axis=1)
        y[:, t] = acc * sigmoid(acc)
    return y, np.transpose(full[:, T:T + W, :], (0, 2, 1)).copy()


def _qkv_to_channels(q, k, v):
    B, T = q.shape[:2]
    return np.concatenate([q.reshape(B, T, -1), k.reshape(B, T, -1), v.reshape(B, T, -1)], axis=-1)


def short_conv_qkv(xq, xk, xv, w, state=None):
    """The convolution on the three projections laid side by side as the
    channels q | k | v; returns (q, k, v) in their own shapes and the window."""
    xq, xk, xv = _f64(xq), _f64(xk), _f64(xv)
    y, st = short_conv_silu(_qkv_to_channels(xq, xk, xv), w, state)
    nq, nk = xq[0, 0].size, xk[0, 0].size
    B, T = xq.shape[:2]
    return (y[..., :nq].reshape(xq.shape), y[..., nq:nq + nk].reshape(xk.shape),
            y[..., nq + nk:].reshape(xv.shape), st)


def output_gate(o, gate, eps=L2_EPS):
    """"kimi_k3_host/kda.rs", ``full_rank_output_gate``: each head row of o
    (last axis) divided by sqrt(mean of its squares + eps), times
    sigmoid(gate) element by element."""
    o, gate = _f64(o), _f64(gate)
    return sigmoid(gate) * o / np.sqrt((o * o).mean(axis=-1, keepdims=True) + eps)


def kda_forward_prepared(q, k, v, z, A_log, dt_bias, lower_bound, beta_logit, scale, S0=None,
                         out_gate=None, out_eps=L2_EPS):
    """Prefill from the raw projections: q, k L2-normalised per row, the gate
    from its pre-activation, beta = sigmoid(logit) ("kimi_k3_host/kda.rs",
    ``kda_recurrent_step`` and ``bounded_gate``), the recurrence, then the
    optional output gate (``full_rank_output_gate``).  Returns (o, S_T)."""
    o, S = kda_forward(l2norm_rows(q), l2norm_rows(k), v, kda_gate(z, A_log, dt_bias, lower_bound),
                       sigmoid(beta_logit), scale, S0)
    if out_gate is not None:
        o = output_gate(o, out_gate, out_eps)
    return o, S


def kda_decode_token(xq, xk, xv, conv_w, conv_state, z, A_log, dt_bias, lower_bound, beta_logit, S, scale,
                     out_gate=None, out_eps=L2_EPS):
    """"kimi_k3_host/kda.rs", ``kda_decode_token``: one token from the raw
    projections xq, xk [B, H, K], xv [B, HV, V]: the convolution step on the
    q | k | v channels, then (``kda_recurrent_step``) L2 normalisation of q
    and k, beta = sigmoid(logit), the gate from z [B, HV, K], the recurrence
    step on S, and the optional output gate.  Returns (o, S_new, conv_state_new);
    the inputs are not modified."""
    xq, xk, xv = _f64(xq), _f64(xk), _f64(xv)
    B = xq.shape[0]
    x = np.concatenate([xq.reshape(B, -1), xk.reshape(B, -1), xv.reshape(B, -1)], axis=-1)
    y, st = conv_update(conv_state, x, conv_w)
    nq, nk = xq[0].size, xk[0].size
    q = y[:, :nq].reshape(xq.shape)
    k = y[:, nq:nq + nk].reshape(xk.shape)
    v = y[:, nq + nk:].reshape(xv.shape)
    g = kda_gate(z, A_log, dt_bias, lower_bound)
    o, S_new = kda_decode_step(l2norm_rows(q), l2norm_rows(k), v, g, sigmoid(beta_logit), S, scale)
    if out_gate is not None:
        o = output_gate(o, out_gate, out_eps)
    return o, S_new, st
