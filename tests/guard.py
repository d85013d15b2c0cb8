"""Guard bytes around GPU outputs: the tests' stand-in for an out-of-bounds
write checker.  Each output is a view, 256-byte aligned, inside a larger
allocation whose margins before and after hold a fixed byte pattern; after the
kernels ran, the margins must still hold it."""
import torch

MARGIN = 4096          # bytes on each side (a multiple of 256)
PATTERN = 0xA5


class Guarded:
    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype, device):
        n = 1
        for s in shape:
            n *= int(s)
        es = torch.empty((), dtype=dtype).element_size()
        nbytes = n * es
        body = (nbytes + 255) // 256 * 256
        raw = torch.full((MARGIN + body + MARGIN,), PATTERN, dtype=torch.uint8, device=device)
        view = raw[MARGIN:MARGIN + nbytes].view(dtype).view(tuple(shape))
        if raw.is_cuda:
            assert view.data_ptr() % 256 == 0
        self.bufs.append((raw, nbytes))
        return view

    def check(self):
        """Every margin byte still holds the pattern (and so does the padding
        between the end of an output and the next 256-byte boundary)."""
        for raw, nbytes in self.bufs:
            head = raw[:MARGIN]
            tail = raw[MARGIN + nbytes:]
            assert bool((head == PATTERN).all()), "write before the start of an output"
            assert bool((tail == PATTERN).all()), "write past the end of an output"
