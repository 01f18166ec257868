"""Failure paths on the GPU, made without a GPU fault: the bulk copy engine's
bounded wait is made to give up (a test setting of its first poll limit), and
the host sees the error word, while the context stays usable and the next
normal call is exact.  Also the latency-floor helper's chain of launches."""
import numpy as np
import pytest
import torch

from combine_ep_layout_07_b200 import epx

from gpu_helpers import assert_all_equal, gpu_inputs, oracle_run, run_gpu, torch_to_bits

pytestmark = pytest.mark.gpu


def test_bulk_dispatch_wait_gives_up_then_recovers():
    wl, o = oracle_run("decode", 0)
    x, idx, _ = gpu_inputs(wl)
    lay = epx.layout(idx, wl["E"], wl["R"])
    recv = torch.zeros((lay.recv_cap, wl["H"]), dtype=torch.bfloat16, device="cuda")
    ex = torch.zeros((lay.exp_cap, wl["H"]), dtype=torch.bfloat16, device="cuda")
    epx.debug_dispatch_first_wait_limit(0)
    try:
        epx.dispatch_expand(x, lay, recv=recv, expanded=ex, variant=2)
        t = epx.read_totals(lay, raise_on_error=False)
    finally:
        epx.debug_dispatch_first_wait_limit(-1)
    assert t["dev_err"] & 0x10              # EP_DEVERR_TIMEOUT
    assert t["status"] == 5                 # EP_ERR_CUDA
    # every CTA gave up on its first (only) token: no row was written
    assert torch.count_nonzero(recv.view(torch.int16)) == 0
    assert torch.count_nonzero(ex.view(torch.int16)) == 0
    # the context is fine and the next normal pass is exact
    g = run_gpu(wl, dispatch_variant=2)
    assert g["totals"]["status"] == 0
    assert_all_equal(g, o)


def test_latency_floor_chain_runs_in_order():
    n = 3
    buf = torch.arange(64 * (2 * n + 2), dtype=torch.int32, device="cuda")
    epx.latency_floor(buf, n)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    for i in range(n):
        assert b[64 * (n + 1 + i)] == 64 * i + 1
    with pytest.raises(epx.EpxError):
        epx.latency_floor(buf[:64], n)      # buffer too small
