"""The L2 flush of bench.py reads its buffer (no writes left dirty in L2);
checked on CPU with a small buffer."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_flush_reads_and_leaves_buffer_untouched():
    f = bench.L2Flush.__new__(bench.L2Flush)
    f.torch = torch
    f.buf = torch.arange(1000, dtype=torch.int32)
    f.sink = torch.empty((), dtype=torch.int64)
    before = f.buf.clone()
    f()
    assert int(f.sink) == sum(range(1000))
    assert torch.equal(f.buf, before)
