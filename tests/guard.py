"""Guard zones around kernel outputs: the stand-in for a memory checker.

compute-sanitizer is closed on this machine, so the GPU tests place every output
buffer a kernel writes between two guard zones filled with a byte pattern,
and check after the call that the zones are untouched.  A kernel that writes
past the end (or before the start) of Y, Xq, beta, rowsum or the int32
accumulators of a ragged shape changes the pattern and fails the test.
"""
import numpy as np
import torch

PATTERN = 0xA5
GUARD_BYTES = 4096


class Guarded:
    """A device tensor of `shape` and `dtype` with GUARD_BYTES of pattern on
    each side (the tensor itself starts 16-byte aligned and is filled with
    the pattern too, so unwritten elements are visible)."""

    def __init__(self, shape, dtype, device="cuda:0"):
        self.shape = tuple(int(s) for s in shape)
        self.dtype = dtype
        n = int(np.prod(self.shape)) if self.shape else 1
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        pad = (-self.nbytes) % 16
        self.raw = torch.full((2 * GUARD_BYTES + self.nbytes + pad,), PATTERN,
                              dtype=torch.uint8, device=device)
        self.t = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(self.shape)

    def check(self, what="output"):
        """Assert both guard zones still hold the pattern."""
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[GUARD_BYTES + self.nbytes:]
        bad_h = int((head != PATTERN).sum().item())
        bad_t = int((tail != PATTERN).sum().item())
        assert bad_h == 0 and bad_t == 0, (
            "%s %s %s: %d bytes changed before it, %d after it"
            % (what, self.shape, self.dtype, bad_h, bad_t))


def check_all(*guarded):
    torch.cuda.synchronize()
    for i, g in enumerate(guarded):
        g.check("buffer %d" % i)
