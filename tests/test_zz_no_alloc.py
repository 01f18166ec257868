"""The host round trip that allocates nothing (ep_roundtrip_host_noalloc).

Who needs it: callers that cannot allocate device memory when they need a
dispatch/combine pass -- code running while another component owns the
device allocator (a caching allocator or a memory pool fixed at start-up),
plugins loaded into a host that forbids allocation after initialisation,
latency paths that cannot take the implicit synchronisation of an
allocation.  Instead of caller-provided device scratch, this entry point
uses a fixed array inside the library.

These checks call it through the C ABI and compare its output with
ep_roundtrip_host, which runs the same pass in device memory the caller
allocated, on two calls in a row with different batches.  The file runs
last so that a run stopping at its first failure has run everything else.
"""
import numpy as np
import pytest
import torch

from combine_ep_layout_07_b200 import epx
from combine_ep_layout_07_b200 import workloads as wlmod

from gpu_helpers import assert_combine_close, torch_to_bits

pytestmark = pytest.mark.gpu


def _host(wl):
    x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    idx = torch.from_numpy(wl["topk_idx"]).pin_memory()
    w = torch.from_numpy(wl["topk_weights"]).pin_memory()
    out = torch.empty((wl["T"], wl["H"]), dtype=torch.bfloat16).pin_memory()
    return x, idx, w, out


def _with_caller_memory(wl):
    x, idx, w, out = _host(wl)
    nbytes = epx.roundtrip_device_bytes(wl["T"], wl["H"], wl["k"], wl["E"], wl["R"])
    dev = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    epx.roundtrip_host(x, idx, w, wl["E"], wl["R"], dev, out)
    torch.cuda.synchronize()
    return torch_to_bits(out)


def _without_allocation(wl):
    x, idx, w, out = _host(wl)
    epx.roundtrip_host_noalloc(x, idx, w, wl["E"], wl["R"], out)
    torch.cuda.synchronize()
    return torch_to_bits(out)


def test_noalloc_matches_caller_memory_path_on_two_calls():
    first = wlmod.make("decode", seed=5)
    second = wlmod.make("lowbatch8")        # different shapes, routing and values
    got = [_without_allocation(first), _without_allocation(second)]
    want = [_with_caller_memory(first), _with_caller_memory(second)]
    for g, w in zip(got, want):
        assert_combine_close(g, w)
    # the second batch's output does not depend on what the first left behind
    assert np.all(wlmod.bf16_bits_to_f32(got[1])[0] == 1.234375)
    assert np.all(got[1][1:] == 0)


def test_noalloc_rejects_batches_beyond_its_scratch():
    wl = wlmod.make("tiny", seed=0)
    T, H, k, E, R = 4096, 7168, 8, 256, 16
    assert epx.roundtrip_device_bytes(T, H, k, E, R) > epx.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    idx = torch.zeros((T, k), dtype=torch.int64)
    w = torch.zeros((T, k), dtype=torch.float32)
    out = torch.empty((T, H), dtype=torch.bfloat16)
    with pytest.raises(epx.EpxError) as ei:
        epx.roundtrip_host_noalloc(x, idx, w, E, R, out)
    assert ei.value.status == 6          # EP_ERR_UNSUPPORTED
    # a batch that fits still works after the rejection
    assert_combine_close(_without_allocation(wl), _with_caller_memory(wl))
