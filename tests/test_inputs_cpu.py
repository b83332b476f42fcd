"""CPU checks of the seeded input recipe that both the CUDA path and the
oracle consume: the workload table (sizes, dtypes, gates), determinism of
the seeds, and the value ranges the recipe promises (unit-norm q/k rows,
gate ranges, beta in (0, 1), the state spreads)."""
from __future__ import annotations

import pytest
import torch

from gated_delta_rule_66_b200.inputs import BY_NAME, make_erase_inputs, make_inputs, make_raw_inputs


def test_workload_table():
    sizes = {n: (w.B, w.T, w.H, w.HV, w.K, w.V, w.dtype, w.path) for n, w in BY_NAME.items()}
    assert sizes["tiny"] == (1, 64, 2, 2, 32, 32, "fp32", "fwd")
    assert sizes["twin"] == (4, 1024, 8, 8, 32, 32, "fp32", "fwd")
    assert sizes["prefill_gqa"] == (1, 8192, 16, 96, 128, 128, "bf16", "fwd")
    assert sizes["fwdbwd"] == (2, 4096, 96, 96, 128, 128, "bf16", "fwdbwd")
    assert sizes["decode"] == (256, 1, 96, 96, 128, 128, "bf16", "decode")
    assert sizes["erase"] == (1, 8192, 32, 8, 64, 128, "bf16", "erase")
    assert BY_NAME["twin"].gate == "softplus" and BY_NAME["twin"].s0_std == 0.01
    assert BY_NAME["decode"].s0_std == 0.02
    assert all(BY_NAME[n].gate == "bounded" for n in ("tiny", "prefill_gqa", "fwdbwd", "decode"))


@pytest.mark.parametrize("name", ["tiny", "twin", "prefill_gqa", "fwdbwd"])
def test_seeded_and_deterministic(name):
    w = BY_NAME[name].with_sizes(B=1, T=40)
    a, b = make_inputs(w), make_inputs(w)
    for n in a:
        if a[n] is not None:
            assert torch.equal(a[n], b[n]), n
    c = make_inputs(w, seed=12345)
    assert not torch.equal(a["v"], c["v"])


def test_workloads_draw_different_numbers():
    a = make_inputs(BY_NAME["tiny"])
    b = make_inputs(BY_NAME["twin"].with_sizes(B=1, T=64, H=2, HV=2))
    assert not torch.equal(a["v"], b["v"])


@pytest.mark.parametrize("name, tol", [("tiny", 1e-5), ("fwdbwd", 1e-2)])
def test_query_key_rows_are_unit_norm(name, tol):
    w = BY_NAME[name].with_sizes(B=1, T=64, H=4, HV=4)
    x = make_inputs(w)
    for n in ("q", "k"):
        norms = x[n].double().norm(dim=-1)
        assert (norms - 1).abs().max() < tol, n


def test_value_ranges_and_outputs_by_path():
    fb = make_inputs(BY_NAME["fwdbwd"].with_sizes(B=1, T=128, H=4, HV=4))
    assert fb["q"].dtype == torch.bfloat16 and fb["g"].dtype == torch.float32
    assert (fb["g"] < 0).all() and (fb["g"] > -5).all()          # -5 sigmoid(z)
    assert (fb["beta"] > 0).all() and (fb["beta"] < 1).all()
    assert fb["S0"] is None and fb["dO"] is not None and fb["dO"].dtype == torch.bfloat16
    tw = make_inputs(BY_NAME["twin"].with_sizes(B=2, T=256))
    assert tw["q"].dtype == torch.float32 and tw["dO"] is None
    assert (tw["g"] < 0).all()                                    # -exp(A_log) softplus(.)
    assert 0.008 < float(tw["S0"].std()) < 0.012
    dec = make_inputs(BY_NAME["decode"].with_sizes(B=2))
    assert dec["q"].shape == (2, 96, 128) and dec["S"].shape == (2, 96, 128, 128)
    assert 0.018 < float(dec["S"].std()) < 0.022


def test_raw_and_erase_inputs_are_seeded():
    w = BY_NAME["prefill_gqa"].with_sizes(T=70, H=1, HV=2)
    a, b = make_raw_inputs(w), make_raw_inputs(w)
    for n, t in a.items():
        if isinstance(t, torch.Tensor):
            assert torch.equal(t, b[n]), n
    we = BY_NAME["erase"].with_sizes(T=50, H=4, HV=2)
    e1, e2 = make_erase_inputs(we), make_erase_inputs(we)
    for n, t in e1.items():
        if isinstance(t, torch.Tensor):
            assert torch.equal(t, e2[n]), n
    assert (e1["g"] < 0).all() and (e1["g"] > -0.25).all()       # -0.25 sigmoid(.)


def test_head_subset_keeps_whole_query_groups():
    """The full-size parity tests check a subset of query/key heads with all
    their value heads; on the oracle, the subset's results must equal the
    full problem's results at those heads (heads are independent, and dq/dk
    sum whole groups)."""
    import numpy as np

    import oracle
    from gated_delta_rule_66_b200.inputs import head_subset

    w = BY_NAME["prefill_gqa"].with_sizes(B=1, T=9, H=3, HV=6, K=32, V=32, dtype="fp32")
    full = make_inputs(w, with_do=True)
    sub, hv_idx = head_subset(full, w.H, w.HV, [2, 0])
    assert hv_idx == [4, 5, 0, 1]
    f64 = lambda d: [None if d[n] is None else d[n].double().numpy() for n in ("q", "k", "v", "g", "beta")]
    o_full, S_full = oracle.kda_forward(*f64(full), w.scale, None)
    o_sub, S_sub = oracle.kda_forward(*f64(sub), w.scale, None)
    assert np.allclose(o_sub, o_full[:, :, hv_idx], rtol=0, atol=1e-14)
    assert np.allclose(S_sub, S_full[:, hv_idx], rtol=0, atol=1e-14)
    g_full = oracle.kda_backward(*f64(full), w.scale, None, full["dO"].double().numpy())
    g_sub = oracle.kda_backward(*f64(sub), w.scale, None, sub["dO"].double().numpy())
    assert np.allclose(g_sub[0], g_full[0][:, :, [2, 0]], rtol=0, atol=1e-13)   # dq over whole groups
    assert np.allclose(g_sub[2], g_full[2][:, :, hv_idx], rtol=0, atol=1e-13)   # dv per value head
