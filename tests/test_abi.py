"""CPU checks of the C ABI: the library loads, exports every entry point that
include/kda.h declares, sizes its workspaces as documented, and rejects bad
arguments before it touches a GPU (no compute call is made here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from gated_delta_rule_66_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    from gated_delta_rule_66_b200 import kda
    return kda.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("kda_fwd", "kda_decode_step", "kda_bwd", "kda_fwd_workspace_bytes",
              "kda_bwd_workspace_bytes", "kda_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def fma_rec_bytes(K, QG=1, C=32):
    """One 32-step chunk record of the two-kernel CUDA-core forward: T diag(beta)
    and P (C x C per query head), the residual and carry operands and Q~ o e^c
    (C x K, the last per query head), e^{c_last} (K); fp32."""
    return 4 * (C * C + 2 * C * K + K + QG * (C * C + C * K))


def test_workspace_sizes(lib):
    """CUDA-core shapes: the training forward keeps the 32-step states and the
    scratch of the two-kernel forward (its chunk records); the backward
    overwrites the records with the state gradients (and dq/dk partials)."""
    B, T, H, HV, K, V = 2, 100, 2, 6, 64, 32
    NT = (T + 31) // 32
    states = B * HV * NT * K * V * 4
    prep = B * HV * NT * (fma_rec_bytes(K) + 4 * (K * V + 32 * V))  # records, then M and U per chunk
    assert lib.kda_fwd_scratch_bytes(B, T, HV, K, V) == prep
    assert lib.kda_fwd_workspace_bytes(B, T, HV, K, V) == states + prep
    assert lib.kda_bwd_workspace_bytes(B, T, H, HV, K, V) == states + max(states + 2 * B * T * HV * K * 4, prep)
    assert lib.kda_bwd_workspace_bytes(B, T, HV, HV, K, V) == states + max(states, prep)
    assert lib.kda_bwd_workspace_bytes(B, T, H, HV, K, V) >= lib.kda_fwd_workspace_bytes(B, T, HV, K, V)
    assert lib.kda_fwd_workspace_bytes(0, T, HV, K, V) == 0
    assert lib.kda_bwd_workspace_bytes(B, T, 4, HV, K, V) == 0   # HV % H != 0


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first


def fwd_call(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, S0=None, scale=0.5, B=1, T=8, H=1, HV=2,
             K=32, V=32, dtype=0, o=FAKE, S_T=None, ws=None, ws_bytes=0, stream=None)
    a.update(over)
    return lib.kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["scale"], a["B"],
                       a["T"], a["H"], a["HV"], a["K"], a["V"], a["dtype"], a["o"], a["S_T"],
                       a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over,code,needle", [
    (dict(T=0), 2, "sizes"),
    (dict(B=-1), 2, "sizes"),
    (dict(H=4, HV=6), 2, "multiple"),
    (dict(K=48), 4, "K=48"),
    (dict(V=256), 4, "V=256"),
    (dict(dtype=2), 3, "dtype"),
    (dict(scale=0.0), 7, "scale"),
    (dict(scale=float("nan")), 7, "scale"),
    (dict(q=None), 1, "non-NULL"),
    (dict(o=None), 1, "non-NULL"),
    (dict(ws=FAKE, ws_bytes=16), 5, "workspace"),
    (dict(ws=ctypes.c_void_p(0x1004), ws_bytes=1 << 30), 7, "aligned"),
    (dict(B=70000), 2, "65535"),
])
def test_fwd_rejects_bad_arguments(lib, over, code, needle):
    assert fwd_call(lib, **over) == code
    assert needle in lib.kda_last_error().decode()


def test_decode_rejects_bad_arguments(lib):
    rc = lib.kda_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0x1008), 0.5, 1, 1, 1,
                             32, 32, 0, FAKE, None)
    assert rc == 7 and "aligned" in lib.kda_last_error().decode()
    rc = lib.kda_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.5, 1, 1, 1, 32, 32, 0, FAKE, None)
    assert rc == 1
    rc = lib.kda_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, 1, 1, 1, 32, 96, 0, FAKE, None)
    assert rc == 4


def test_bwd_rejects_bad_arguments(lib):
    args = [FAKE] * 5 + [None, FAKE, None, 0.5, 1, 8, 1, 1, 32, 32, 0] + [FAKE] * 5 + [None]
    rc = lib.kda_bwd(*args, None, 0, 0, None)
    assert rc == 5 and "workspace" in lib.kda_last_error().decode()
    rc = lib.kda_bwd(*args, FAKE, 1 << 40, 2, None)
    assert rc == 7 and "flags" in lib.kda_last_error().decode()
    bad = list(args)
    bad[6] = None  # dO
    rc = lib.kda_bwd(*bad, FAKE, 1 << 40, 0, None)
    assert rc == 1


def test_last_error_clears_on_next_call(lib):
    fwd_call(lib, T=0)
    assert lib.kda_last_error().decode() != ""
    fwd_call(lib, K=48)
    assert "K=48" in lib.kda_last_error().decode()


def test_tensor_core_workspace_sizes(lib):
    """K = V = 128: the training forward keeps the 32-step states, a 64 KB
    interaction record and the scratch per 64-step chunk; the scratch holds the
    32 KB T and P images of the tensor-core path or the CUDA-core path's
    records (fp32 inputs), whichever is larger, since the dtype is not an
    argument; the backward overwrites it with its own buffers."""
    B, T, H, HV, K, V = 1, 130, 1, 2, 128, 128
    nt32, nt64 = (T + 31) // 32, (T + 63) // 64
    states = B * HV * nt32 * K * V * 4
    inter = B * HV * nt64 * 16384 * 4
    img = max(B * HV * nt64 * 32768, B * HV * nt32 * fma_rec_bytes(K))
    assert lib.kda_fwd_scratch_bytes(B, T, HV, K, V) == img
    assert lib.kda_fwd_workspace_bytes(B, T, HV, K, V) == states + inter + img
    tail = states + 2 * B * T * HV * K * 4 + B * HV * nt64 * 16592 * 4  # state grads, dq/dk partials, records
    assert lib.kda_bwd_workspace_bytes(B, T, H, HV, K, V) == states + inter + max(tail, img)
    assert lib.kda_bwd_workspace_bytes(B, T, H, HV, K, V) >= lib.kda_fwd_workspace_bytes(B, T, HV, K, V)
    assert lib.kda_fwd_scratch_bytes(B, T, HV, 64, 64) == B * HV * nt32 * (fma_rec_bytes(64) + 4 * (64 * 64 + 32 * 64))
    assert lib.kda_fwd_scratch_bytes(B, T, HV, 48, 64) == 0  # unsupported K


def _cu(vals):
    return (ctypes.c_int * len(vals))(*vals)


def test_varlen_workspace_and_validation(lib):
    HV = 3
    cu = _cu([0, 5, 5, 200])  # sequences of 5, 0 and 195 steps: 1 + 0 + 4 chunks
    table = ((2 * 5 + 4) * 4 + 255) // 256 * 256
    assert lib.kda_fwd_varlen_workspace_bytes(cu, 3, HV, 128, 128) == table + 5 * HV * 32768
    assert lib.kda_fwd_varlen_workspace_bytes(_cu([1, 5]), 1, HV, 128, 128) == 0      # must start at 0
    assert lib.kda_fwd_varlen_workspace_bytes(_cu([0, 9, 5]), 2, HV, 128, 128) == 0   # decreasing
    assert lib.kda_fwd_varlen_workspace_bytes(cu, 3, HV, 64, 64) == 0                 # tensor-core shapes only
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.5)
    rc = lib.kda_fwd_varlen(*args, _cu([0, 9, 5]), 2, 1, HV, 128, 128, 1, FAKE, None, FAKE, 1 << 40, None)
    assert rc == 7 and "cu_seqlens" in lib.kda_last_error().decode()
    rc = lib.kda_fwd_varlen(*args, cu, 3, 1, HV, 128, 128, 1, FAKE, None, None, 0, None)
    assert rc == 5 and "workspace" in lib.kda_last_error().decode()
    rc = lib.kda_fwd_varlen(*args, cu, 3, 1, HV, 128, 128, 0, FAKE, None, FAKE, 1 << 40, None)  # fp32
    assert rc == 7 and "tensor-core" in lib.kda_last_error().decode()


def test_prep_workspace_and_validation(lib):
    B, T, H, HV = 2, 100, 1, 2
    # tensor-core shape: see below; a CUDA-core bf16 shape: the fp32 output for the gate pass
    # (the T and P images, fp32 g and the fp32 rows of the output gate)
    assert lib.kda_fwd_prep_workspace_bytes(B, T, H, HV, 128, 128, 1) == (B * HV * 2 * 32768 + B * T * HV * 128 * 4
                                                                         + B * T * HV * 128 * 4)
    assert lib.kda_fwd_prep_workspace_bytes(B, T, H, HV, 64, 32, 1) == B * T * HV * 32 * 4
    assert lib.kda_fwd_prep_workspace_bytes(B, T, H, HV, 64, 32, 0) == 0
    assert lib.kda_fwd_prep_workspace_bytes(B, T, 2, 3, 64, 32, 0) == 0  # HV % H != 0

    def fwd_prep(**over):
        a = dict(q=FAKE, k=FAKE, v=FAKE, z=FAKE, A_log=FAKE, dt=FAKE, lb=-5.0, bl=FAKE, og=None, eps=1e-6,
                 S0=None, scale=0.5, B=1, T=8, H=1, HV=2, K=64, V=32, dtype=1, o=FAKE, S_T=None, ws=None,
                 ws_bytes=0)
        a.update(over)
        return lib.kda_fwd_prep(a["q"], a["k"], a["v"], a["z"], a["A_log"], a["dt"], a["lb"], a["bl"], a["og"],
                                a["eps"], a["S0"], a["scale"], a["B"], a["T"], a["H"], a["HV"], a["K"], a["V"],
                                a["dtype"], a["o"], a["S_T"], a["ws"], a["ws_bytes"], None)

    assert fwd_prep(z=None) == 1 and "z, A_log" in lib.kda_last_error().decode()
    assert fwd_prep(lb=0.5) == 7 and "gate_lower_bound" in lib.kda_last_error().decode()
    assert fwd_prep(lb=float("nan")) == 7
    assert fwd_prep(og=FAKE, eps=-1.0) == 7 and "out_eps" in lib.kda_last_error().decode()
    assert fwd_prep(og=FAKE) == 5 and "workspace" in lib.kda_last_error().decode()  # bf16 gate pass, no scratch
    assert fwd_prep(ws=ctypes.c_void_p(0x1004), ws_bytes=1 << 30) == 7
    assert fwd_prep(K=48) == 4

    def conv(**over):
        a = dict(xq=FAKE, xk=FAKE, xv=FAKE, w=FAKE, si=None, so=None, B=1, T=8, H=1, HV=2, K=32, V=32, W=4,
                 dtype=1, q=ctypes.c_void_p(0x100000), k=ctypes.c_void_p(0x200000), v=ctypes.c_void_p(0x300000))
        a.update(over)
        return lib.kda_short_conv(a["xq"], a["xk"], a["xv"], a["w"], a["si"], a["so"], a["B"], a["T"], a["H"],
                                  a["HV"], a["K"], a["V"], a["W"], a["dtype"], a["q"], a["k"], a["v"], None)

    assert conv(W=0) == 7 and conv(W=9) == 7
    assert conv(si=ctypes.c_void_p(0x400000), so=ctypes.c_void_p(0x400040)) == 7
    assert "overlap" in lib.kda_last_error().decode()
    assert conv(q=FAKE) == 7 and "alias" in lib.kda_last_error().decode()
    assert conv(w=None) == 1
    assert conv(T=65535 * 32 + 1) == 2 and "launch grid" in lib.kda_last_error().decode()

    def tok(**over):
        a = dict(xq=FAKE, xk=FAKE, xv=FAKE, cw=FAKE, ci=ctypes.c_void_p(0x400000), co=ctypes.c_void_p(0x400000),
                 W=4, z=FAKE, A_log=FAKE, dt=FAKE, lb=-5.0, bl=FAKE, og=None, eps=1e-6, S=FAKE, scale=0.5, B=1,
                 H=1, HV=2, K=32, V=32, dtype=1, o=FAKE)
        a.update(over)
        return lib.kda_decode_token(a["xq"], a["xk"], a["xv"], a["cw"], a["ci"], a["co"], a["W"], a["z"],
                                    a["A_log"], a["dt"], a["lb"], a["bl"], a["og"], a["eps"], a["S"], a["scale"],
                                    a["B"], a["H"], a["HV"], a["K"], a["V"], a["dtype"], a["o"], None)

    assert tok() == 7 and "H == HV" in lib.kda_last_error().decode()  # grouped heads share the q/k windows
    assert tok(S=ctypes.c_void_p(0x1008), H=2) == 7 and "aligned" in lib.kda_last_error().decode()
    assert tok(co=None) == 1
    assert tok(W=12, H=2) == 7


def test_erase_validation(lib):
    def call(**over):
        a = dict(q=FAKE, k=FAKE, e=FAKE, z=FAKE, g=FAKE, S0=None, scale=0.5, B=1, T=8, HQ=4, HV=2, K=64, V=128,
                 dtype=1, o=FAKE, S_T=None)
        a.update(over)
        return lib.kda_fwd_erase(a["q"], a["k"], a["e"], a["z"], a["g"], a["S0"], a["scale"], a["B"], a["T"],
                                 a["HQ"], a["HV"], a["K"], a["V"], a["dtype"], a["o"], a["S_T"],
                                 a.get("ws"), a.get("ws_bytes", 0), None)

    assert call(HQ=3) == 2 and "multiple of HV" in lib.kda_last_error().decode()
    assert call(e=None) == 1
    assert call(K=48) == 4
    assert call(scale=-1.0) == 7
    assert call(T=0) == 2
    # the two-kernel path's workspace: one record per 32-step chunk and state head
    # (then the state entering each chunk and its U, for the read-out kernel)
    assert lib.kda_fwd_erase_workspace_bytes(1, 8, 4, 2, 64, 128) == 1 * 2 * 1 * (fma_rec_bytes(64, QG=2) +
                                                                                 4 * (64 * 128 + 32 * 128))
    assert lib.kda_fwd_erase_workspace_bytes(1, 8, 3, 2, 64, 128) == 0  # HQ % HV != 0
    assert call(ws=FAKE, ws_bytes=16) == 5 and "workspace" in lib.kda_last_error().decode()


def test_training_forward_wants_aligned_o(lib):
    """bf16 K = V = 128 with aligned inputs and a training workspace: a
    misaligned o would send the forward down the CUDA-core path while a later
    tensor-core backward reads tensor-core records, so it is rejected before
    anything is enqueued."""
    B, T, H, HV, K, V = 1, 64, 1, 1, 128, 128
    ws_bytes = lib.kda_fwd_workspace_bytes(B, T, HV, K, V)
    rc = lib.kda_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.1, B, T, H, HV, K, V, 1, ctypes.c_void_p(0x1008), None,
                     FAKE, ws_bytes, None)
    assert rc == 7 and "aligned o" in lib.kda_last_error().decode()
