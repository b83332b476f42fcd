"""kda_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a plugin whose host framework owns all device memory, a
running loop that forbids allocator calls) cannot hand kda_bwd a workspace;
kda_bwd_noalloc takes its scratch from a fixed device array inside the
library instead.  These tests call it through the C ABI twice in a row on each
problem (the second call reuses the array exactly as the first left it) and
check both results bit for bit against kda_bwd with a caller workspace (the
kernels are deterministic) and against the float64 oracle.  The file is named
so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import oracle
from gated_delta_rule_66_b200.inputs import BY_NAME, make_inputs
from kda_testlib import f64, rel_l2, tol_for

NOALLOC_BYTES = 64 * 1024 * 1024


def _lib():
    from gated_delta_rule_66_b200 import build as kbuild
    kbuild.build()
    from gated_delta_rule_66_b200 import kda
    lib = kda.library()
    vp, f, i = ctypes.c_void_p, ctypes.c_float, ctypes.c_int
    lib.kda_bwd_noalloc.restype = i
    lib.kda_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, f, i, i, i, i, i, i, i,
                                    vp, vp, vp, vp, vp, vp, vp]
    return kda, lib


def test_noalloc_rejects_problems_beyond_its_array():
    kda, lib = _lib()
    B, T, H, HV, K, V = 4, 4096, 8, 8, 128, 128
    assert kda.workspace_bytes("bwd", B, T, H, HV, K, V) > NOALLOC_BYTES
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the size check comes first
    rc = lib.kda_bwd_noalloc(*([fake] * 5), None, fake, None, 0.1, B, T, H, HV, K, V, 1,
                             *([fake] * 5), None, None)
    assert rc == 5
    assert "scratch" in lib.kda_last_error().decode()


def _noalloc_grads(kda, lib, d, w):
    dev = d["q"].device
    dq = torch.empty(w.B, w.T, w.H, w.K, dtype=d["q"].dtype, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty(w.B, w.T, w.HV, w.V, dtype=d["q"].dtype, device=dev)
    dg = torch.empty(w.B, w.T, w.HV, w.K, dtype=torch.float32, device=dev)
    dbeta = torch.empty(w.B, w.T, w.HV, dtype=torch.float32, device=dev)
    dS0 = torch.empty(w.B, w.HV, w.K, w.V, dtype=torch.float32, device=dev)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = lib.kda_bwd_noalloc(p(d["q"]), p(d["k"]), p(d["v"]), p(d["g"]), p(d["beta"]), p(d["S0"]),
                             p(d["dO"]), None, w.scale, w.B, w.T, w.H, w.HV, w.K, w.V,
                             0 if d["q"].dtype == torch.float32 else 1,
                             p(dq), p(dk), p(dv), p(dg), p(dbeta), p(dS0),
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.kda_last_error().decode()
    return dq, dk, dv, dg, dbeta, dS0


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    kda, lib = _lib()
    cases = [BY_NAME["prefill_gqa"].with_sizes(T=200, H=2, HV=4),          # bf16, grouped heads
             BY_NAME["twin"].with_sizes(B=2, T=150, H=2, HV=2, K=64, V=64)]  # fp32, S0 != 0
    names = ("dq", "dk", "dv", "dg", "dbeta", "dS0")
    for w in cases:
        assert kda.workspace_bytes("bwd", w.B, w.T, w.H, w.HV, w.K, w.V) <= NOALLOC_BYTES
        inp = make_inputs(w, with_do=True)
        d = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
        ref = kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], scale=w.scale,
                      initial_state=d["S0"])
        exact = oracle.kda_backward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                                    f64(inp["beta"]), w.scale, f64(inp["S0"]), f64(inp["dO"]))
        for call in range(2):  # the second call starts from what the first left in the array
            got = _noalloc_grads(kda, lib, d, w)
            torch.cuda.synchronize()
            for name, x, r, e in zip(names, got, ref, exact):
                assert torch.equal(x, r), (
                    f"{w.name} call {call} {name}: differs from kda_bwd "
                    f"(rel_l2 {rel_l2(f64(x), f64(r)):.3e})")
                err = rel_l2(f64(x), e)
                assert err <= tol_for(w.torch_dtype), f"{w.name} call {call} {name}: {err:.3e} vs oracle"
