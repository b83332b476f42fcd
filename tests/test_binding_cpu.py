"""CPU checks of the Python binding's argument checks: every tensor must be a
contiguous CUDA tensor of the documented dtype and rank, on the calling
thread's current device (the one the library launches on).  No GPU call is
made: a stand-in object carries the attributes the checks read."""
from __future__ import annotations

import pytest
import torch

from gated_delta_rule_66_b200 import build as kbuild


@pytest.fixture(scope="module")
def kda():
    kbuild.build()
    from gated_delta_rule_66_b200 import kda as mod
    return mod


class FakeCudaTensor:
    """The attributes of a CUDA tensor that the binding's checks read."""

    is_cuda = True

    def __init__(self, index=0, dtype=torch.float32, shape=(1, 2, 3, 4), contiguous=True):
        self.index, self.dtype, self.shape, self.contiguous = index, dtype, shape, contiguous

    def get_device(self):
        return self.index

    def is_contiguous(self):
        return self.contiguous

    def dim(self):
        return len(self.shape)


@pytest.fixture
def on_device0(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)


def test_accepts_a_tensor_of_the_current_device(kda, on_device0):
    kda._req("g", FakeCudaTensor(0), torch.float32, 4)
    kda._req("workspace", None)


def test_rejects_a_tensor_of_another_device(kda, on_device0):
    with pytest.raises(ValueError, match=r"q is on cuda:1 but the current CUDA device is cuda:0"):
        kda._req("q", FakeCudaTensor(1), torch.float32, 4)


def test_rejects_host_tensors(kda, on_device0):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        kda._req("v", torch.zeros(1, 2, 3, 4), torch.float32, 4)


@pytest.mark.parametrize("bad, exc, needle", [
    (dict(contiguous=False), ValueError, "must be contiguous"),
    (dict(dtype=torch.bfloat16), TypeError, "must be torch.float32"),
    (dict(shape=(2, 3, 4)), ValueError, "must have 4 dims"),
])
def test_rejects_layout_dtype_and_rank(kda, on_device0, bad, exc, needle):
    with pytest.raises(exc, match=needle):
        kda._req("g", FakeCudaTensor(**bad), torch.float32, 4)
