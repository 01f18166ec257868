"""GPU parity of the two-stage combine (local reduce per (token, rank), then
the epilogue with an optional residual add) against the CPU oracle.

Tolerances: fp32 partials |gpu - oracle| <= 2^-18 |oracle| (an fp32 FMA chain
of at most 32 same-sign terms against one rounding of the double sum); bf16
partials within one bf16 step, 2^-7 |oracle|.  Epilogue outputs: the combine
tolerance 2^-7 |oracle| + 1e-3 with fp32 partials; with bf16 partials each
summand may sit one bf16 step apart, so 2^-6 |oracle| + 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import epx
from combine_ep_layout_07_b200 import workloads as wlmod

from gpu_helpers import (assert_combine_close, bits_to_torch, gpu_inputs, oracle_run, run_gpu,
                         torch_to_bits)

pytestmark = pytest.mark.gpu

NAMES = ["tiny", "decode", "prefill", "lowbatch1", "lowbatch8", "dp_padded", "dp_compact"]


def _f(bits):
    return wlmod.bf16_bits_to_f32(bits).astype(np.float64)


def _close(got, want, rtol, atol=0.0):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    bad = np.abs(got - want) > rtol * np.abs(want) + atol
    assert not bad.any(), (f"{bad.sum()} of {bad.size} out of tolerance; first "
                           f"{np.argwhere(bad)[0]}: {got[bad][0]} vs {want[bad][0]}")


@pytest.mark.parametrize("bits", [32, 16])
@pytest.mark.parametrize("name", NAMES)
def test_local_reduce_and_epilogue(name, bits):
    wl, o = oracle_run(name, 0)
    lay_o = o["layout"]
    g = run_gpu(wl)
    lay = g["layout"]
    w = torch.from_numpy(wl["topk_weights"]).cuda()
    dt = torch.float32 if bits == 32 else torch.bfloat16
    part = epx.combine_local_reduce(g["y"], w, lay, partial_dtype=dt)
    want_part = oracle.combine_local(o["y"], wl["topk_weights"], lay_o, part_bits=bits)
    n = lay_o["N_recv"]
    if bits == 32:
        _close(part[:n].cpu().numpy(), want_part, 2.0 ** -18)
    else:
        _close(_f(torch_to_bits(part[:n])), _f(want_part), 2.0 ** -7)
    out = epx.combine_epilogue(part, lay)
    want_out = oracle.combine_epilogue(want_part, lay_o)
    _close(_f(torch_to_bits(out)), _f(want_out), 2.0 ** -7 if bits == 32 else 2.0 ** -6, 1e-3)
    # and against the single-stage oracle result
    _close(_f(torch_to_bits(out)), _f(o["out"]), 2.0 ** -7 if bits == 32 else 2.0 ** -6, 1e-3)
    assert epx.read_totals(lay)["status"] == 0


@pytest.mark.parametrize("bits", [32, 16])
@pytest.mark.parametrize("name", ["decode", "lowbatch4"])
def test_epilogue_on_oracle_partials_with_residual(name, bits):
    wl, o = oracle_run(name, 0)
    lay_o = o["layout"]
    g = run_gpu(wl)
    part_o = oracle.combine_local(o["y"], wl["topk_weights"], lay_o, part_bits=bits)
    n, H = lay_o["N_recv"], wl["H"]
    cap = g["layout"].recv_cap
    if bits == 32:
        part = torch.zeros((cap, H), dtype=torch.float32, device="cuda")
        part[:n] = torch.from_numpy(part_o).cuda()
    else:
        part = torch.zeros((cap, H), dtype=torch.bfloat16, device="cuda")
        part[:n] = bits_to_torch(part_o)
    x, _, _ = gpu_inputs(wl)
    out = epx.combine_epilogue(part, g["layout"], residual=x)
    want = oracle.combine_epilogue(part_o, lay_o, residual=wl["x"])
    _close(_f(torch_to_bits(out)), _f(want), 2.0 ** -7, 1e-3)


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_two_stage_worked_example_issue760_exact(T):
    """Unit expert outputs: every partial is 1/16, the real row is exactly 1,
    padding rows are +0 (DeepEP issue #760, Reproduction)."""
    wl = wlmod.make_lowbatch(T)
    g = run_gpu(wl)
    lay = g["layout"]
    ones = torch.ones_like(g["y"])
    w = torch.from_numpy(wl["topk_weights"]).cuda()
    for dt in (torch.float32, torch.bfloat16):
        part = epx.combine_local_reduce(ones, w, lay, partial_dtype=dt)
        assert torch.all(part[:16].float() == 0.0625)
        out = torch_to_bits(epx.combine_epilogue(part, lay))
        assert np.all(out[0] == 0x3F80) and np.all(out[1:] == 0)


def test_partial_guard_bands_and_capacity():
    wl, o = oracle_run("tiny", 1)
    g = run_gpu(wl)
    lay = g["layout"]
    w = torch.from_numpy(wl["topk_weights"]).cuda()
    n, H = o["layout"]["N_recv"], wl["H"]
    big = torch.full((lay.recv_cap + 6, H), -7.0, dtype=torch.float32, device="cuda")
    part = big[3:-3]
    epx.combine_local_reduce(g["y"], w, lay, partial=part)
    assert torch.all(big[:3] == -7.0) and torch.all(big[3 + n:] == -7.0)
    assert epx.read_totals(lay)["status"] == 0
    small = torch.zeros((10, H), dtype=torch.float32, device="cuda")
    epx.combine_local_reduce(g["y"], w, lay, partial=small)
    t = epx.read_totals(lay, raise_on_error=False)
    assert t["status"] == 3 and (t["dev_err"] & 2)
