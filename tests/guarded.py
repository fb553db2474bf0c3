"""Output buffers with canary margins, for the GPU parity tests.

Every output a kernel writes (O, LSE, dQ, dK, dV, the workspace) is handed to
the library as a view into a larger device buffer whose margins before and
after the view are filled with a canary byte. After the call the margins must
be unchanged, so a store past the last row of a ragged tail, past the last
head or before the first element is caught even though the view itself has
exactly the size the call was given.
"""

from __future__ import annotations

import torch

CANARY = 0xA5
MARGIN = 4096  # bytes on each side; a multiple of 256 keeps every view aligned


class Guarded:
    """A tensor of ``shape``/``dtype`` inside a canary-filled device buffer."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        elem = torch.empty((), dtype=dtype).element_size()
        n = 1
        for s in shape:
            n *= int(s)
        self.nbytes = n * elem
        self.raw = torch.full((MARGIN + self.nbytes + MARGIN,), CANARY, dtype=torch.uint8, device=device)
        body = self.raw[MARGIN:MARGIN + self.nbytes]
        self.t = body.view(dtype).view(shape) if n else torch.empty(shape, dtype=dtype, device=device)
        if fill is not None and n:
            self.t.fill_(fill)

    def intact(self) -> bool:
        head = self.raw[:MARGIN]
        tail = self.raw[MARGIN + self.nbytes:]
        return bool(torch.all(head == CANARY)) and bool(torch.all(tail == CANARY))


def check_all(*guards):
    for name, g in guards:
        assert g.intact(), f"write outside {name}"
