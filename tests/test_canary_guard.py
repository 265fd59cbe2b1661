"""The canary guard of tests/test_gpu_canary.py catches writes just outside a
buffer (checked on CPU tensors, where planting the stray write is harmless)."""
import pytest
import torch

from tests.test_gpu_canary import Guarded


@pytest.mark.parametrize("where", ["before", "after", "none"])
def test_guard_detects_stray_writes(where):
    g = Guarded()
    v = g.view(torch.arange(37, dtype=torch.float32))           # 148 bytes: a ragged tail
    v += 1                                                      # writes inside are fine
    raw = g.blocks[0][0]
    if where == "before":
        raw[4096 // 4 - 1] = 0
    elif where == "after":
        raw[4096 // 4 + 40] = 0                                 # past the 16-byte-rounded end
    if where == "none":
        g.check()
    else:
        with pytest.raises(AssertionError):
            g.check()
