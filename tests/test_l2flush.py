"""The L2 flush used between timed launches writes its buffer and, when asked for
a clean L2, then reads the other one (here on the CPU, where only the operations
are checked)."""
import torch

from exact_tiled_attention_40_b200.l2flush import L2Flush


def test_clean_flush_writes_then_reads():
    f = L2Flush(torch.device("cpu"), nbytes=4096)
    f.r.fill_(3)
    f.r[17] = 9
    f(0x107, clean=True)
    assert f.w.numel() == 4096 and bool((f.w == 7).all())
    assert int(f.sink) == 9 and f.sink.dtype == f.r.dtype


def test_write_only_flush_leaves_the_read_buffer_alone():
    f = L2Flush(torch.device("cpu"), nbytes=4096)
    f.sink.fill_(-1)
    f(5)
    assert bool((f.w == 5).all()) and int(f.sink) == -1
