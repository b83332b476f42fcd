"""CPU checks of bench.py's bookkeeping: the algorithmic bytes behind the
roofline fractions and the recorded-traffic lookup (no GPU)."""
from __future__ import annotations

import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_decode_algorithmic_bytes():
    """The decode step reads and writes the fp32 state once (2 K V 4 bytes per
    (b, hv)) and moves the token's q, k, v, g, beta and o once."""
    b = _bench()
    w = b.BY_NAME["decode"]
    state = w.B * w.HV * w.K * w.V * 4
    io = w.B * (2 * w.H * w.K * 2 + w.HV * w.V * 2 + w.HV * w.K * 4 + w.HV * 4 + w.HV * w.V * 2)
    assert b.algorithmic_bytes(w, "decode") == 2 * state + io == 3259072512


def test_fwdbwd_algorithmic_bytes():
    """Forward: inputs once, o and S_T out.  Backward: the forward inputs and
    dO in, dq, dk, dv, dg, dbeta and dS0 out (S0 = 0 on this workload)."""
    b = _bench()
    w = b.BY_NAME["fwdbwd"]
    e = 2
    fwd_in = w.B * w.T * (2 * w.H * w.K * e + w.HV * w.V * e + w.HV * w.K * 4 + w.HV * 4)
    state = w.B * w.HV * w.K * w.V * 4
    assert b.algorithmic_bytes(w, "fwd") == fwd_in + w.B * w.T * w.HV * w.V * e + state
    bwd = b.algorithmic_bytes(w, "bwd")
    assert bwd == 2 * fwd_in + w.B * w.T * w.HV * w.V * e + state == 2233466880


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """The backward's DRAM traffic comes from profiles/dram_traffic.json only
    while the listed sources hash to the recorded value."""
    b = _bench()
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    got = b.recorded_traffic("kda_bwd", "fwdbwd")
    assert got in (None, rec["kda_bwd"]["bytes_per_launch"]["fwdbwd"])
    assert b.recorded_traffic("no_such_kernel", "fwdbwd") is None
    # a record whose hash does not match (a changed source) gives no figure
    bad = json.loads(json.dumps(rec))
    bad["kda_bwd"]["sources_sha256"] = "0" * 64
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(bad))
    for rel in rec["kda_bwd"]["sources"]:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(ROOT, rel), "rb").read())
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.recorded_traffic("kda_bwd", "fwdbwd") is None
