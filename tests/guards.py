"""Canary guard bands for GPU outputs: the output tensor is a view into a
larger buffer whose head and tail hold a known value, so any write outside
the tensor shows up as a changed canary."""
import numpy as np
import torch

CANARY = 12345.0
PAD = 4096


def guarded(shape, dtype=torch.bfloat16, fill=CANARY):
    """An output tensor inside a canary guard band: (band buffer, view)."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * PAD,), fill, dtype=dtype, device="cuda")
    return buf, buf[PAD:PAD + n].view(tuple(shape))


def check_guard(buf, fill=CANARY, what="out"):
    assert torch.all(buf[:PAD] == fill) and torch.all(buf[-PAD:] == fill), f"write outside {what}"
