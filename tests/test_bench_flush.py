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
    f.buf = torch.arange(1000, dtype=torch.float32)
    f.sink = torch.empty((), dtype=torch.float32)
    before = f.buf.clone()
    f()
    assert float(f.sink) == float(sum(range(1000)))
    assert torch.equal(f.buf, before)


def test_flush_reduction_needs_no_conversion_copy():
    """The flush must only read: a float32 sum into a float32 scalar runs one
    reduction (an int32 buffer summed with dtype=int64 would be converted --
    written -- first).  On CPU, check that no temporary as large as the
    buffer is created by watching the profiler's allocations."""
    from torch.profiler import ProfilerActivity, profile
    f = bench.L2Flush.__new__(bench.L2Flush)
    f.torch = torch
    f.buf = torch.zeros(1 << 22, dtype=torch.float32)
    f.sink = torch.empty((), dtype=torch.float32)
    with profile(activities=[ProfilerActivity.CPU], profile_memory=True) as prof:
        f()
    big = [e for e in prof.events() if e.cpu_memory_usage >= f.buf.numel() * 4]
    assert not big
