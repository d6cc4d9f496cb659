"""L2 flush between timed launches.

The default flush writes a buffer larger than L2 (126 MB on B200), which evicts
every line a timed launch could reuse but leaves L2 full of the buffer's dirty
lines.  A bandwidth-bound launch then pays for their write-back to HBM: on the
paged decode that is about 14 us of a 199 us call, traffic of the flush and not
of the kernel.  `clean=True` reads a second buffer of the same size after the
write, so that L2 holds clean lines of no input (the state a profiler's cache
control leaves before it replays a kernel).  The compute-bound forward ran
fastest right after the plain write and 2-7 % slower after an extra (heavier,
widening) read or an idle gap, which points at the power and clock state rather
than at L2; so the timed regions use the plain write, and the decode is also
reported after the clean flush.
"""
import torch

FLUSH_BYTES = 256 << 20


class L2Flush:
    def __init__(self, device, nbytes: int = FLUSH_BYTES):
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.r = torch.zeros(nbytes // 4, dtype=torch.int32, device=device)
        self.sink = torch.empty((), dtype=torch.int32, device=device)

    def __call__(self, i: int, clean: bool = False) -> None:
        """Flush on the current stream: write the buffer, then (`clean`) read the other."""
        self.w.fill_(i & 0xff)
        if clean:   # a reduction in the buffer's own type: reads it, writes one word
            torch.amax(self.r, dim=0, out=self.sink)
