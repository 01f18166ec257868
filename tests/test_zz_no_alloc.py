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
allocated, bit for bit, on two calls in a row with different batches, and
with the CPU oracle within the combine tolerance; they also check that a
call changes no allocation and that dropped routes reach the caller through
the error word.  The file runs
last so that a run stopping at its first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle

from combine_ep_layout_07_b200 import epx
from combine_ep_layout_07_b200 import workloads as wlmod

from gpu_helpers import assert_combine_close, torch_to_bits

pytestmark = pytest.mark.gpu


def _host(wl, idx_dtype=torch.int64):
    x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    idx = torch.from_numpy(wl["topk_idx"]).to(idx_dtype).pin_memory()
    w = torch.from_numpy(wl["topk_weights"]).pin_memory()
    out = torch.empty((wl["T"], wl["H"]), dtype=torch.bfloat16).pin_memory()
    return x, idx, w, out


def _with_caller_memory(wl, idx_dtype=torch.int64):
    x, idx, w, out = _host(wl, idx_dtype)
    bits = 64 if idx_dtype == torch.int64 else 32
    nbytes = epx.roundtrip_device_bytes(wl["T"], wl["H"], wl["k"], wl["E"], wl["R"], bits)
    dev = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    err = ctypes.c_int32(-1)
    epx.roundtrip_host(x, idx, w, wl["E"], wl["R"], dev, out, dev_err=err)
    torch.cuda.synchronize()
    return torch_to_bits(out), err.value


def _without_allocation(wl, idx_dtype=torch.int64):
    x, idx, w, out = _host(wl, idx_dtype)
    err = ctypes.c_int32(-1)
    epx.roundtrip_host_noalloc(x, idx, w, wl["E"], wl["R"], out, dev_err=err)
    torch.cuda.synchronize()
    return torch_to_bits(out), err.value


def test_noalloc_matches_caller_memory_path_on_two_calls():
    first = wlmod.make("decode", seed=5)
    second = wlmod.make("lowbatch8")        # different shapes, routing and values
    got = [_without_allocation(first), _without_allocation(second)]
    want = [_with_caller_memory(first), _with_caller_memory(second)]
    for (g, ge), (w, we) in zip(got, want):
        # the same kernels on the same inputs: identical bits, clean error word
        np.testing.assert_array_equal(g, w)
        assert ge == 0 and we == 0
    # and the result is the oracle's, within the combine tolerance
    assert_combine_close(got[0][0], oracle.run_all(first)["out"])
    # the second batch's output does not depend on what the first left behind
    assert np.all(wlmod.bf16_bits_to_f32(got[1][0])[0] == 1.234375)
    assert np.all(got[1][0][1:] == 0)


def test_noalloc_int32_indices():
    wl = wlmod.make("tiny", seed=3)
    g, ge = _without_allocation(wl, torch.int32)
    w, we = _with_caller_memory(wl, torch.int32)
    np.testing.assert_array_equal(g, w)
    assert ge == 0 and we == 0
    assert_combine_close(g, oracle.run_all(wl)["out"])


def test_noalloc_allocates_no_device_memory():
    wl = wlmod.make("decode", seed=2)
    _without_allocation(wl)              # warm-up: first-call set-up, lazy module load
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    reserved0 = torch.cuda.memory_reserved()
    for _ in range(3):
        _without_allocation(wl)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0


def test_noalloc_reports_dropped_routes():
    """An index >= E is dropped and flagged in the device error word, which
    the call hands back to the host (its status only covers host checks)."""
    wl = wlmod.make("tiny", seed=1)
    wl = dict(wl)
    idx = wl["topk_idx"].copy()
    idx[5, 1] = wl["E"] + 3
    wl["topk_idx"] = idx
    g, ge = _without_allocation(wl)
    w, we = _with_caller_memory(wl)
    assert ge & 0x1 and we & 0x1          # EP_DEVERR_BAD_INDEX
    np.testing.assert_array_equal(g, w)
    assert_combine_close(g, oracle.run_all(wl)["out"])


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
    np.testing.assert_array_equal(_without_allocation(wl)[0], _with_caller_memory(wl)[0])
