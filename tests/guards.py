"""Guarded buffers for the library's outputs: every buffer is a view into a larger
byte buffer whose margins hold a fixed pattern, so that a write past either end of
the view shows up as a changed margin byte (a check of out-of-bounds writes that
needs no memory-checking tool)."""
import torch

MARGIN = 4096          # bytes on each side; keeps 256-byte alignment of the view
PATTERN = 0xA5


class Guarded:
    def __init__(self, shape, dtype, device, fill=None):
        self.shape, self.dtype = tuple(shape), dtype
        n = 1
        for d in self.shape:
            n *= d
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((self.nbytes + 2 * MARGIN,), PATTERN, dtype=torch.uint8,
                              device=device)
        self.t = self.raw[MARGIN:MARGIN + self.nbytes].view(dtype).view(self.shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self) -> bool:
        head = self.raw[:MARGIN]
        tail = self.raw[MARGIN + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())
