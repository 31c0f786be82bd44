"""Guard bands for buffers handed to the library: a tensor placed inside a
larger allocation whose margins hold a fixed bit pattern, so that a write
outside the tensor shows up as a changed margin (a stand-in for a memory
checker, which is not available on the GPU pool)."""
import math

import torch

MARGIN_BYTES = 4096  # each side; keeps the tensor 4 KiB-aligned relative to the allocation
_PATTERN = {1: 0x5A, 2: 0x7FC1, 4: 0x7FC0DEAD}
_RAW = {1: torch.uint8, 2: torch.int16, 4: torch.int32}


def guarded(shape, dtype, device="cuda", fill=None):
    """(view, intact): `view` is a contiguous tensor of `shape` and `dtype`
    inside a larger buffer, `fill` (if given) copied into it; intact() is True
    while both margins still hold the pattern."""
    size = torch.empty((), dtype=dtype).element_size()
    margin = MARGIN_BYTES // size
    n = math.prod(shape)
    buf = torch.empty(n + 2 * margin, dtype=dtype, device=device)
    raw = buf.view(_RAW[size])
    raw.fill_(_PATTERN[size])
    view = buf[margin:margin + n].view(tuple(shape))
    if fill is not None:
        view.copy_(fill)

    def intact() -> bool:
        pat = _PATTERN[size]
        return bool((raw[:margin] == pat).all()) and bool((raw[margin + n:] == pat).all())

    return view, intact
