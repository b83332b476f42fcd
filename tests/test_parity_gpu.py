"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Every case draws its inputs with the seeded generator, runs the library on
the GPU, upcasts the exact bits it consumed to float64, runs the oracle on
them, and compares whole tensors by relative L2 (1e-5 for fp32 inputs,
2e-3 for bf16 inputs).  Full-size workloads are checked on a seeded subset
of whole grouped-query blocks (or batch rows for decode).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_66_b200.inputs import BY_NAME, head_subset, make_inputs
from kda_testlib import f64, rel_l2, report, to_cuda, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from gated_delta_rule_66_b200 import kda as mod
    mod.device_status()
    yield mod
    assert mod.device_status() == 0, "a kernel gave up on a bounded wait"


def run_fwd(kda, inp, scale, scratch=True):
    d = to_cuda(inp)
    o, S = kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=scale, initial_state=d["S0"],
                   scratch=scratch)
    torch.cuda.synchronize()
    return o, S


def oracle_fwd(inp, scale):
    return oracle.kda_forward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                              f64(inp["beta"]), scale, f64(inp["S0"]))


def check_fwd(kda, inp, scale, dtype, label, scratch=True):
    o, S = run_fwd(kda, inp, scale, scratch)
    o_ref, S_ref = oracle_fwd(inp, scale)
    tol = tol_for(dtype)
    report(f"{label} o", f64(o), o_ref, tol, dtype)
    report(f"{label} S_T", f64(S), S_ref, tol, torch.float32)


# ----------------------------------------------------------------------------- forward

def test_fwd_tiny_workload(kda):
    w = BY_NAME["tiny"]
    check_fwd(kda, make_inputs(w), w.scale, w.torch_dtype, "tiny")


def test_fwd_twin_workload(kda):
    w = BY_NAME["twin"]
    check_fwd(kda, make_inputs(w), w.scale, w.torch_dtype, "twin")


FWD_CASES = [
    # name, base workload, overrides
    ("T1", "tiny", dict(T=1)),
    ("T31", "tiny", dict(T=31)),
    ("T33_s0", "twin", dict(B=1, T=33, H=2, HV=2)),
    ("K64V64_gqa_ragged", "twin", dict(B=2, T=77, H=2, HV=4, K=64, V=64)),
    ("K32V128", "twin", dict(B=1, T=70, H=1, HV=2, K=32, V=128)),
    ("K128V32_bf16", "prefill_gqa", dict(T=90, H=1, HV=3, K=128, V=32)),
    ("K128_bf16_gqa", "prefill_gqa", dict(T=200, H=2, HV=6)),
    ("K128_fp32", "prefill_gqa", dict(T=100, H=1, HV=2, dtype="fp32", s0_std=0.02)),
    ("K64V128_bf16", "fwdbwd", dict(B=1, T=65, H=2, HV=2, K=64, V=128, path="fwd")),
    # tensor-core prefill (K = V = 128, bf16): ragged tails, one step, S0, GQA
    ("tc_T1", "prefill_gqa", dict(T=1, H=1, HV=2)),
    ("tc_T63", "prefill_gqa", dict(T=63, H=1, HV=2)),
    ("tc_T64", "prefill_gqa", dict(T=64, H=1, HV=1)),
    ("tc_T129_s0", "prefill_gqa", dict(B=2, T=129, H=1, HV=2, s0_std=0.02)),
    ("tc_T300_gqa", "prefill_gqa", dict(B=1, T=300, H=2, HV=8)),
]


@pytest.mark.parametrize("name,base,over", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_fwd_shapes(kda, name, base, over):
    w = BY_NAME[base].with_sizes(**over)
    check_fwd(kda, make_inputs(w), w.scale, w.torch_dtype, name)


TC_CASES = [c for c in FWD_CASES if c[0].startswith("tc_")]
FMA_CASES = [c for c in FWD_CASES if not c[0].startswith("tc_")]


@pytest.mark.parametrize("name,base,over", FMA_CASES, ids=[c[0] for c in FMA_CASES])
def test_fwd_single_kernel(kda, name, base, over):
    """Without a workspace the CUDA-core shapes run one kernel per state slice
    (the default is the two-kernel path: chunk preparation, then the state
    pass); the same shapes against the oracle."""
    w = BY_NAME[base].with_sizes(**over)
    check_fwd(kda, make_inputs(w), w.scale, w.torch_dtype, name + "_single", scratch=False)


@pytest.mark.parametrize("name,base,over", TC_CASES, ids=[c[0] for c in TC_CASES])
def test_fwd_tc_single_kernel(kda, name, base, over):
    """The tensor-core forward without a workspace (one kernel carrying the
    whole chunk pipeline) on the same shapes as the two-kernel default."""
    w = BY_NAME[base].with_sizes(**over)
    check_fwd(kda, make_inputs(w), w.scale, w.torch_dtype, name + "_single", scratch=False)


def test_fwd_tc_training_workspace_same_output(kda):
    """With a training workspace (states and records stored) the two-kernel
    forward gives bitwise the o and S_T of the scratch-only run."""
    w = BY_NAME["prefill_gqa"].with_sizes(B=2, T=200, H=2, HV=4, s0_std=0.02)
    d = to_cuda(make_inputs(w))
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    o1, S1 = kda.fwd(*args, scale=w.scale, initial_state=d["S0"])
    ws = torch.empty(kda.workspace_bytes("fwd", w.B, w.T, w.H, w.HV, w.K, w.V), dtype=torch.uint8,
                     device="cuda")
    o2, S2 = kda.fwd(*args, scale=w.scale, initial_state=d["S0"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_bounded_wait_gives_up_then_recovers(kda):
    """The failure path of the bounded waits, without any fault: with one
    probe per wait the chunked forward's kernels give up at their first wait
    (the copy they just issued cannot have landed), drain the copies and
    products they issued, free their tensor memory and report bit 0; after
    the default is restored the same call on the same context matches the
    oracle."""
    w = BY_NAME["prefill_gqa"].with_sizes(T=130, H=1, HV=2)
    inp = make_inputs(w)
    d = to_cuda(inp)
    assert kda.device_status() == 0
    kda.set_wait_polls(1)
    try:
        kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"])
        torch.cuda.synchronize()
        flags = kda.device_status()
    finally:
        kda.set_wait_polls(0)
    assert flags & 1, f"no kernel reported giving up (flags {flags})"
    assert not flags & 2
    check_fwd(kda, inp, w.scale, w.torch_dtype, "after_give_up")
    assert kda.device_status() == 0


def test_bounded_wait_backward_gives_up_then_recovers(kda):
    """The same for the tensor-core backward's warp-specialised state-gradient
    pass: with one probe per wait its issuer gives up at its first wait (the
    builders cannot have formed the first operand yet), every role leaves,
    the issued copies drain and bit 0 is reported (the later kernels of the
    call run on undefined state gradients, which is no fault); with the
    default restored the backward matches the oracle."""
    w = BY_NAME["fwdbwd"].with_sizes(B=1, T=130, H=2, HV=2)
    inp = make_inputs(w, with_do=True)
    d = to_cuda(inp)
    B, T, H, K = d["q"].shape
    HV, V = d["v"].shape[2], d["v"].shape[3]
    ws = torch.empty(kda.workspace_bytes("bwd", B, T, H, HV, K, V), dtype=torch.uint8, device="cuda")
    kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"], workspace=ws)
    torch.cuda.synchronize()
    assert kda.device_status() == 0
    kda.set_wait_polls(1)
    try:
        kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], scale=w.scale, initial_state=d["S0"],
                workspace=ws, states_from_fwd=True)
        torch.cuda.synchronize()
        flags = kda.device_status()
    finally:
        kda.set_wait_polls(0)
    assert flags & 1, f"no kernel reported giving up (flags {flags})"
    check_bwd(kda, inp, w.scale, w.torch_dtype, "bwd_after_give_up", reuse=True)
    assert kda.device_status() == 0


def test_fwd_strong_unbounded_decay(kda):
    """Very strong decays (|g| up to 40 per step) take the pair-by-pair path
    for diagonal blocks; results stay finite and match."""
    w = BY_NAME["twin"].with_sizes(B=1, T=96, H=1, HV=2, K=32, V=32)
    inp = make_inputs(w)
    inp["g"] = inp["g"] * 20.0
    check_fwd(kda, inp, w.scale, w.torch_dtype, "strong_decay")


def test_fwd_tc_strong_unbounded_decay(kda):
    """bf16 K = V = 128 with decays far beyond the -5 bound: chunks whose
    in-half decay span is too wide for the split exponents form those
    entries pair by pair."""
    w = BY_NAME["prefill_gqa"].with_sizes(T=160, H=1, HV=2)
    inp = make_inputs(w)
    inp["g"] = inp["g"] * 8.0
    check_fwd(kda, inp, w.scale, w.torch_dtype, "tc_strong_decay")
    check_fwd(kda, inp, w.scale, w.torch_dtype, "tc_strong_decay_single", scratch=False)


def test_fwd_prefill_gqa_full_size(kda):
    """Production-head GQA prefill (B=1, H=16 -> HV=96, T=8192, K=V=128,
    bf16) on the GPU in full; the oracle checks grouped-query block 5."""
    w = BY_NAME["prefill_gqa"]
    inp = make_inputs(w)
    o, S = run_fwd(kda, inp, w.scale)
    sub, hv_idx = head_subset(inp, w.H, w.HV, [5])
    o_ref, S_ref = oracle_fwd(sub, w.scale)
    report("prefill_gqa o[group 5]", f64(o[:, :, hv_idx]), o_ref, tol_for(w.torch_dtype), w.torch_dtype)
    report("prefill_gqa S_T[group 5]", f64(S[:, hv_idx]), S_ref, tol_for(w.torch_dtype), torch.float32)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fwd_split_time_state_passing(kda, dtype):
    """A prefill split at T1 (S_T1 passed on as S0) matches the oracle's
    single pass over all T, as does the unsplit GPU run."""
    w = BY_NAME["prefill_gqa"].with_sizes(T=150, H=2, HV=4, dtype=dtype)
    cpu = make_inputs(w)
    inp = to_cuda(cpu)
    o, S = kda.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], scale=w.scale)
    T1 = 70
    sl = lambda x, a, b: x[:, a:b].contiguous()
    oa, Sa = kda.fwd(*(sl(inp[n], 0, T1) for n in ("q", "k", "v", "g", "beta")), scale=w.scale)
    ob, Sb = kda.fwd(*(sl(inp[n], T1, 150) for n in ("q", "k", "v", "g", "beta")), scale=w.scale,
                     initial_state=Sa)
    o_ref, S_ref = oracle_fwd(cpu, w.scale)
    tol = tol_for(w.torch_dtype)
    report(f"split_{dtype} o", f64(torch.cat([oa, ob], 1)), o_ref, tol, w.torch_dtype)
    report(f"split_{dtype} S_T", f64(Sb), S_ref, tol, torch.float32)
    report(f"unsplit_{dtype} S_T", f64(S), S_ref, tol, torch.float32)


def test_fwd_deterministic(kda):
    w = BY_NAME["prefill_gqa"].with_sizes(T=100, H=2, HV=4)
    inp = make_inputs(w)
    o1, S1 = run_fwd(kda, inp, w.scale)
    o2, S2 = run_fwd(kda, inp, w.scale)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


# ----------------------------------------------------------------------------- backward

def run_bwd(kda, inp, scale, dS_T=None, reuse=False):
    d = to_cuda(inp)
    ws = None
    if reuse:
        B, T, H, K = d["q"].shape
        HV, V = d["v"].shape[2], d["v"].shape[3]
        ws = torch.empty(kda.workspace_bytes("bwd", B, T, H, HV, K, V), dtype=torch.uint8, device="cuda")
        kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=scale, initial_state=d["S0"],
                workspace=ws)
    grads = kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], scale=scale,
                    initial_state=d["S0"], dS_T=None if dS_T is None else dS_T.cuda(),
                    workspace=ws, states_from_fwd=reuse)
    torch.cuda.synchronize()
    return grads


def oracle_bwd(inp, scale, dS_T=None):
    return oracle.kda_backward(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                               f64(inp["beta"]), scale, f64(inp["S0"]), f64(inp["dO"]),
                               None if dS_T is None else f64(dS_T))


GRAD_NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dS0")


def check_bwd(kda, inp, scale, dtype, label, dS_T=None, reuse=False):
    got = run_bwd(kda, inp, scale, dS_T, reuse)
    ref = oracle_bwd(inp, scale, dS_T)
    tol = tol_for(dtype)
    for n, x, r in zip(GRAD_NAMES, got, ref):
        out_dtype = dtype if n in ("dq", "dk", "dv") else torch.float32
        report(f"{label} {n}", f64(x), r, tol, out_dtype)


BWD_CASES = [
    ("fp32_K32_s0_dST", "twin", dict(B=1, T=70, H=1, HV=2)),
    ("fp32_K64_gqa", "twin", dict(B=2, T=64, H=1, HV=3, K=64, V=64)),
    ("bf16_K128_gqa_ragged", "prefill_gqa", dict(T=45, H=2, HV=4)),
    ("bf16_K128", "fwdbwd", dict(B=1, T=130, H=2, HV=2)),
    ("bf16_K128_T96_half_chunk", "fwdbwd", dict(B=1, T=96, H=1, HV=2, s0_std=0.02)),
    ("fp32_K128V32", "fwdbwd", dict(B=1, T=40, H=1, HV=1, V=32, dtype="fp32", s0_std=0.05)),
]


@pytest.mark.parametrize("name,base,over", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_bwd_shapes(kda, name, base, over):
    w = BY_NAME[base].with_sizes(**over)
    inp = make_inputs(w, with_do=True)
    dS_T = None
    if "dST" in name:
        dS_T = torch.randn(w.B, w.HV, w.K, w.V, generator=torch.Generator().manual_seed(5))
    check_bwd(kda, inp, w.scale, w.torch_dtype, name, dS_T)


def test_bwd_tc_strong_unbounded_decay(kda):
    """bf16 K = V = 128 with decays far beyond the -5 bound: chunks whose
    decay span rules out the split-exponent factors of the tensor-core
    assembly take the pair-by-pair route, the others the tensor cores."""
    w = BY_NAME["fwdbwd"].with_sizes(B=1, T=192, H=1, HV=2)
    inp = make_inputs(w, with_do=True)
    inp["g"] = inp["g"] * 8.0
    inp["g"][:, 64:128] = inp["g"][:, 64:128] / 8.0  # one chunk within range
    check_bwd(kda, inp, w.scale, w.torch_dtype, "tc_strong_decay")


@pytest.mark.parametrize("mag", [1e5, 1e-4], ids=["states_1e5", "states_1e-4"])
def test_bwd_tc_state_range(kda, mag):
    """The tensor-core path stores the chunk states and their gradients as
    fp16 with a power-of-two scale per value column and 32 key channels.
    v and S0 scaled by 1e5 put the states far past fp16's range (65504), and
    scaled by 1e-4 into its subnormals; with the scales both keep the bf16
    bar (the forward's states are reused by the backward, as in training)."""
    w = BY_NAME["fwdbwd"].with_sizes(B=1, T=130, H=2, HV=2, s0_std=0.5)
    inp = make_inputs(w, with_do=True)
    inp["v"] = (inp["v"].float() * mag).to(inp["v"].dtype)
    inp["S0"] = inp["S0"] * mag
    check_bwd(kda, inp, w.scale, w.torch_dtype, f"tc_state_range_{mag:g}", reuse=True)


def test_bwd_misaligned_dO_after_tensor_core_forward(kda):
    """A dO that is not 16-byte aligned keeps the backward off the tensor-core
    path; with states_from_fwd it must then not rely on the tensor-core
    forward's states (which keep only the chunk starts)."""
    w = BY_NAME["fwdbwd"].with_sizes(B=1, T=100, H=2, HV=2)
    inp = make_inputs(w, with_do=True)
    d = to_cuda(inp)
    buf = torch.empty(d["dO"].numel() + 1, dtype=d["dO"].dtype, device="cuda")
    dO = buf[1:].view(d["dO"].shape)
    dO.copy_(d["dO"])
    assert dO.data_ptr() % 16 != 0
    B, T, H, K = d["q"].shape
    HV, V = d["v"].shape[2], d["v"].shape[3]
    ws = torch.empty(kda.workspace_bytes("bwd", B, T, H, HV, K, V), dtype=torch.uint8, device="cuda")
    kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, workspace=ws)
    got = kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dO, scale=w.scale, workspace=ws,
                  states_from_fwd=True)
    torch.cuda.synchronize()
    ref = oracle_bwd(inp, w.scale)
    for n, x, r in zip(GRAD_NAMES, got, ref):
        out_dtype = w.torch_dtype if n in ("dq", "dk", "dv") else torch.float32
        report(f"misaligned_dO {n}", f64(x), r, tol_for(w.torch_dtype), out_dtype)


def test_bwd_reuses_forward_states(kda):
    w = BY_NAME["fwdbwd"].with_sizes(B=1, T=100, H=2, HV=2)
    inp = make_inputs(w, with_do=True)
    a = run_bwd(kda, inp, w.scale, reuse=False)
    b = run_bwd(kda, inp, w.scale, reuse=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("K,V", [(64, 32), (128, 128)], ids=["K64V32_split_readout", "K128V128_fp32"])
def test_bwd_reuses_two_kernel_cuda_core_states(kda, K, V):
    """CUDA-core shapes: the training forward runs as two (or three) kernels
    and stores every 32-step state; the backward that reuses them meets the
    fp32 bar (its own forward recomputation takes the single-kernel path)."""
    w = BY_NAME["twin"].with_sizes(B=1, T=100, H=2, HV=4, K=K, V=V)
    inp = make_inputs(w, with_do=True)
    grads = run_bwd(kda, inp, w.scale, reuse=True)
    for n, x, r in zip(GRAD_NAMES, grads, oracle_bwd(inp, w.scale)):
        report(f"fma_reuse_K{K}V{V} {n}", f64(x), r, tol_for(w.torch_dtype), torch.float32)


def test_fwdbwd_full_size(kda):
    """Production fwd+bwd (B=2, H=HV=96, T=4096, K=V=128, bf16) on the GPU in
    full, run exactly as the benchmark step runs it: the training forward
    stores its chunk states and records in the workspace and the backward
    reuses them (B * HV = 192 heads also exercise the backward's split of the
    partial last wave onto its side stream).  The oracle checks value heads 17
    and 60 of both batch rows."""
    w = BY_NAME["fwdbwd"]
    inp = make_inputs(w)
    d = to_cuda(inp)
    ws = torch.empty(kda.workspace_bytes("bwd", w.B, w.T, w.H, w.HV, w.K, w.V), dtype=torch.uint8,
                     device="cuda")
    o, S = kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"],
                   workspace=ws)
    grads = kda.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dO"], scale=w.scale,
                    initial_state=d["S0"], workspace=ws, states_from_fwd=True)
    # the same forward again gives the same bits (no data race in the pipelined kernels)
    o2, S2 = kda.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=w.scale, initial_state=d["S0"],
                     workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(S, S2), "two identical forwards differ"
    del o2, S2
    sub, hv_idx = head_subset(inp, w.H, w.HV, [17, 60])
    o_ref, S_ref = oracle_fwd(sub, w.scale)
    tol = tol_for(w.torch_dtype)
    report("fwdbwd o", f64(o[:, :, hv_idx]), o_ref, tol, w.torch_dtype)
    report("fwdbwd S_T", f64(S[:, hv_idx]), S_ref, tol, torch.float32)
    ref = oracle_bwd(sub, w.scale)
    sel = {"dq": lambda x: x[:, :, [17, 60]], "dk": lambda x: x[:, :, [17, 60]],
           "dv": lambda x: x[:, :, hv_idx], "dg": lambda x: x[:, :, hv_idx],
           "dbeta": lambda x: x[:, :, hv_idx], "dS0": lambda x: x[:, hv_idx]}
    for n, x, r in zip(GRAD_NAMES, grads, ref):
        out_dtype = w.torch_dtype if n in ("dq", "dk", "dv") else torch.float32
        report(f"fwdbwd {n}", f64(sel[n](x)), r, tol, out_dtype)
    for x in grads:
        assert torch.isfinite(x.float()).all()


# ----------------------------------------------------------------------------- decode

def check_decode(kda, inp, scale, dtype, label, rows=None):
    d = to_cuda(inp)
    S = d["S"].clone()
    o = kda.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, scale=scale)
    torch.cuda.synchronize()
    sel = slice(None) if rows is None else rows
    sub = {n: inp[n][sel] for n in ("q", "k", "v", "g", "beta", "S")}
    o_ref, S_ref = oracle.kda_decode_step(f64(sub["q"]), f64(sub["k"]), f64(sub["v"]), f64(sub["g"]),
                                          f64(sub["beta"]), f64(sub["S"]), scale)
    tol = tol_for(dtype)
    report(f"{label} o", f64(o[sel]), o_ref, tol, dtype)
    report(f"{label} S", f64(S[sel]), S_ref, tol, torch.float32)


def test_decode_full_size(kda):
    """Batched decode (B=256, HV=96, K=V=128, bf16 inputs, fp32 state, in
    place); the oracle checks batch rows 0, 131 and 255."""
    w = BY_NAME["decode"]
    check_decode(kda, make_inputs(w), w.scale, w.torch_dtype, "decode", rows=[0, 131, 255])


DEC_CASES = [
    ("K32V32_fp32", dict(B=3, H=2, HV=4, K=32, V=32, dtype="fp32")),
    ("K64V128_bf16", dict(B=2, H=1, HV=3, K=64, V=128)),
    ("K128V64_fp32_gqa", dict(B=2, H=2, HV=6, K=128, V=64, dtype="fp32")),
    ("K32V128_bf16", dict(B=5, H=4, HV=4, K=32, V=128)),
]


@pytest.mark.parametrize("name,over", DEC_CASES, ids=[c[0] for c in DEC_CASES])
def test_decode_shapes(kda, name, over):
    w = BY_NAME["decode"].with_sizes(**over)
    check_decode(kda, make_inputs(w), w.scale, w.torch_dtype, name)


def test_decode_sequence_equals_prefill(kda):
    """T decode steps from S0 equal one prefill over the same T tokens."""
    w = BY_NAME["prefill_gqa"].with_sizes(T=40, H=2, HV=4, dtype="fp32", s0_std=0.02)
    inp = to_cuda(make_inputs(w))
    o, S = kda.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], scale=w.scale,
                   initial_state=inp["S0"])
    St = inp["S0"].clone()
    outs = []
    for t in range(w.T):
        outs.append(kda.decode_step(*(inp[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")),
                                    St, scale=w.scale))
    torch.cuda.synchronize()
    assert rel_l2(f64(torch.stack(outs, 1)), f64(o)) < 1e-5
    assert rel_l2(f64(St), f64(S)) < 1e-5


# ----------------------------------------------------------------------------- packed sequences

VARLEN_CASES = [
    # name, sequence lengths, H, HV
    ("mixed", [5, 0, 195, 64, 1, 130], 2, 4),
    ("one_long", [300], 1, 2),
    ("all_short", [1, 2, 3, 63, 65], 1, 1),
]


def _varlen_inputs(lens, H, HV, seed=7):
    T = sum(lens)
    w = BY_NAME["prefill_gqa"].with_sizes(B=1, T=max(T, 1), H=H, HV=HV)
    inp = make_inputs(w, seed=seed)
    inp = {n: (t[0, :T] if t is not None and n != "S0" else t) for n, t in inp.items()}
    gen = torch.Generator().manual_seed(seed + 1)
    S0 = torch.randn(len(lens), HV, w.K, w.V, generator=gen) * 0.02
    return w, inp, S0


@pytest.mark.parametrize("scratch", [True, False], ids=["two_kernel", "single_kernel"])
@pytest.mark.parametrize("name,lens,H,HV", VARLEN_CASES, ids=[c[0] for c in VARLEN_CASES])
def test_fwd_varlen(kda, name, lens, H, HV, scratch):
    """N packed sequences (empty, one-step, exact-chunk and ragged lengths)
    against the oracle run on each sequence with its own initial state."""
    w, inp, S0 = _varlen_inputs(lens, H, HV)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    d = {n: t.cuda() for n, t in inp.items() if t is not None}
    ws = None
    if not scratch:  # the chunk table only: one kernel per (sequence, value head)
        nc = sum((n + 63) // 64 for n in lens)
        ws = torch.empty(((2 * nc + len(lens) + 1) * 4 + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
    o, S = kda.fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], cu, scale=w.scale,
                          initial_state=S0.cuda(), workspace=ws)
    torch.cuda.synchronize()
    o_ref = np.zeros((cu[-1], HV, w.V))
    S_ref = np.zeros((len(lens), HV, w.K, w.V))
    for s, (a0, a1) in enumerate(zip(cu[:-1], cu[1:])):
        if a1 == a0:
            S_ref[s] = f64(S0[s])
            continue
        sl = lambda t: f64(t[a0:a1].unsqueeze(0))
        os_, Ss = oracle.kda_forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]),
                                     w.scale, f64(S0[s:s + 1]))
        o_ref[a0:a1] = os_[0]
        S_ref[s] = Ss[0]
    tol = tol_for(w.torch_dtype)
    report(f"varlen_{name} o", f64(o), o_ref, tol, w.torch_dtype)
    report(f"varlen_{name} S_T", f64(S), S_ref, tol, torch.float32)


VARLEN_BWD_CASES = [
    ("mixed_gqa", [5, 0, 130, 64, 1], 1, 2),
    ("mha", [200, 70], 2, 2),
]


@pytest.mark.parametrize("name,lens,H,HV", VARLEN_BWD_CASES, ids=[c[0] for c in VARLEN_BWD_CASES])
def test_bwd_varlen(kda, name, lens, H, HV):
    """Backward of packed sequences against the oracle's backward run per
    sequence (its own S0, dO and dS_T); the result with the forward's stored
    states is bitwise the result of the backward's own forward pass."""
    w, inp, S0 = _varlen_inputs(lens, H, HV, seed=11)
    T = sum(lens)
    gen = torch.Generator().manual_seed(13)
    dO = torch.randn(T, HV, w.V, generator=gen).to(torch.bfloat16)
    dS_T = torch.randn(len(lens), HV, w.K, w.V, generator=gen)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    d = {n: t.cuda() for n, t in inp.items() if t is not None}
    args = (d["q"], d["k"], d["v"], d["g"], d["beta"])
    got = kda.bwd_varlen(*args, dO.cuda(), cu, scale=w.scale, initial_state=S0.cuda(), dS_T=dS_T.cuda())
    ws = torch.empty(kda.varlen_workspace_bytes("bwd", cu, H, HV, w.K, w.V), dtype=torch.uint8, device="cuda")
    kda.fwd_varlen(*args, cu, scale=w.scale, initial_state=S0.cuda(), workspace=ws)
    again = kda.bwd_varlen(*args, dO.cuda(), cu, scale=w.scale, initial_state=S0.cuda(), dS_T=dS_T.cuda(),
                           workspace=ws, states_from_fwd=True)
    torch.cuda.synchronize()
    for x, y in zip(got, again):
        assert torch.equal(x, y)
    ref = [np.zeros(tuple(t.shape)) for t in got]
    for s, (a0, a1) in enumerate(zip(cu[:-1], cu[1:])):
        if a1 == a0:
            ref[5][s] = f64(dS_T[s])
            continue
        sl = lambda t: f64(t[a0:a1].unsqueeze(0))
        r = oracle.kda_backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]), w.scale,
                                f64(S0[s:s + 1]), sl(dO), f64(dS_T[s:s + 1]))
        for n in range(5):
            ref[n][a0:a1] = r[n][0]
        ref[5][s] = r[5][0]
    tol = tol_for(w.torch_dtype)
    for n, x, r in zip(GRAD_NAMES, got, ref):
        out_dtype = w.torch_dtype if n in ("dq", "dk", "dv") else torch.float32
        report(f"varlen_{name} {n}", f64(x), r, tol, out_dtype)


def test_varlen_prefill_then_decode(kda):
    """Packed prefill hands each sequence's final state to batched decode: the
    decoded outputs equal the oracle run on each sequence's prompt followed by
    its decoded tokens."""
    lens, H, HV, steps = [70, 0, 1, 128, 33], 2, 4, 3
    N = len(lens)
    w, inp, S0 = _varlen_inputs(lens, H, HV, seed=21)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    d = {n: t.cuda() for n, t in inp.items() if t is not None}
    _, S = kda.fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], cu, scale=w.scale, initial_state=S0.cuda())
    dec_w = BY_NAME["decode"].with_sizes(B=N, H=H, HV=HV)
    dec = [make_inputs(dec_w, seed=40 + t) for t in range(steps)]
    outs = []
    for t in range(steps):
        outs.append(kda.decode_step(*(dec[t][n].cuda() for n in ("q", "k", "v", "g", "beta")), S, scale=w.scale))
    torch.cuda.synchronize()
    tol = tol_for(w.torch_dtype)
    for s, (a0, a1) in enumerate(zip(cu[:-1], cu[1:])):
        cat = {n: torch.cat([inp[n][a0:a1]] + [dec[t][n][s:s + 1] for t in range(steps)]).unsqueeze(0)
               for n in ("q", "k", "v", "g", "beta")}
        o_ref, S_ref = oracle.kda_forward(*(f64(cat[n]) for n in ("q", "k", "v", "g", "beta")), w.scale,
                                          f64(S0[s:s + 1]))
        got = torch.stack([outs[t][s] for t in range(steps)])
        report(f"prefill_then_decode seq{s} o", f64(got), o_ref[0, a1 - a0:], tol, w.torch_dtype)
        report(f"prefill_then_decode seq{s} S", f64(S[s]), S_ref[0], tol, torch.float32)
