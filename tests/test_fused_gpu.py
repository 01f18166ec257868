"""GPU parity of ep_layout_dispatch_expand -- the one-launch kernel (variant
1), the layout kernel followed by a dispatch that reads x before its wait
(variant 2) and the automatic choice between them (0): every array of the
layout, the received and the expanded rows bit-exact against the CPU oracle,
the combine on top of it within tolerance, on the seeded workloads and on
edge shapes (padding rows, bad indices, duplicates)."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import epx

from gpu_helpers import (assert_all_equal, assert_layout_equal, gpu_inputs, oracle_run,
                         torch_to_bits)
from test_edge_gpu import _random_wl

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "decode", "lowbatch1", "lowbatch2", "lowbatch4", "lowbatch8", "dp_compact",
         "dp_padded"]


def _arrays(lay):
    """Every array of a layout (the block's padding between them is never written)."""
    return [lay.cnt_e, lay.off_e, lay.cnt_r, lay.off_r, lay.pos, lay.recv_pos, lay.totals]


def run_fused(wl, variant=0, idx_dtype=torch.int64, caps=None):
    x, idx, w = gpu_inputs(wl, idx_dtype)
    E, R = wl["E"], wl["R"]
    lay, recv, ex = epx.layout_dispatch_expand(idx, x, E, R, variant=variant)
    y = epx.standin_expert(ex, lay)
    out = epx.combine_reduce(y, w, lay)
    tot = epx.read_totals(lay, raise_on_error=False)
    return dict(layout=lay, recv=recv, expanded=ex, y=y, out=out, totals=tot)


@pytest.mark.parametrize("name", SMALL)
@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("variant", [0, 1, 2])
@pytest.mark.parametrize("idx_dtype", [torch.int64, torch.int32], ids=["i64", "i32"])
def test_fused_matches_oracle(name, seed, variant, idx_dtype):
    wl, o = oracle_run(name, seed)
    if variant == 1 and wl["T"] * wl["k"] > epx.FUSED_MAX_ROUTES:
        x, idx, _ = gpu_inputs(wl, idx_dtype)
        with pytest.raises(epx.EpxError) as ei:   # beyond the one-launch limit
            epx.layout_dispatch_expand(idx, x, wl["E"], wl["R"], variant=1)
        assert ei.value.status == 6
        return
    g = run_fused(wl, variant, idx_dtype)
    assert_all_equal(g, o)


def test_auto_on_large_batch_runs_two_kernels_and_matches():
    wl, o = oracle_run("prefill", 0)
    assert_all_equal(run_fused(wl, 0), o)
    assert_all_equal(run_fused(wl, 2), o)


def test_one_launch_refuses_beyond_its_limit():
    wl, _ = oracle_run("prefill", 0)
    x, idx, _ = gpu_inputs(wl)
    with pytest.raises(epx.EpxError) as ei:
        epx.layout_dispatch_expand(idx, x, wl["E"], wl["R"], variant=1)
    assert ei.value.status == 6


FUSED_CASES = [
    dict(T=1, H=8, E=1, R=1, k=1),
    dict(T=2, H=8, E=2, R=2, k=2),
    dict(T=33, H=296, E=12, R=3, k=6),          # k does not divide 32; ragged H
    dict(T=77, H=64, E=64, R=4, k=32),          # k = 32
    dict(T=5, H=8, E=8, R=8, k=1),
    dict(T=3, H=14336, E=16, R=4, k=4),         # wide rows: four vectors per thread
    dict(T=512, H=64, E=256, R=16, k=8),        # at the one-launch limit (4096 routes)
    dict(T=128, H=136, E=4096, R=64, k=32),     # E, R and k at their maxima
    dict(T=4096, H=8, E=8, R=2, k=1),           # one route per token, many tokens
    dict(T=200, H=128, E=96, R=48, k=12),       # R > 32: 64-bit rank sets
]


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "T{T}k{k}E{E}R{R}H{H}".format(**c))
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_fused_edge_shapes(case, variant):
    wl = _random_wl(seed=case["T"] * 7 + case["k"], p_pad=0.2, distinct=False, **case)
    idx = wl["topk_idx"]
    if case["T"] > 3:
        idx[2, 0] = case["E"] + 5      # bad index: dropped and flagged
        idx[3, :] = -1                 # all-padding row
    if case["T"] > 1 and case["k"] > 1:
        idx[1, 1] = idx[1, 0]          # same expert twice in one token
    o = oracle.run_all(wl)
    g = run_fused(wl, variant)
    assert_all_equal(g, o)


def test_fused_layout_equals_layout_kernel_on_every_array():
    wl, _ = oracle_run("decode", 1)
    x, idx, _ = gpu_inputs(wl)
    lay_f, _, _ = epx.layout_dispatch_expand(idx, x, wl["E"], wl["R"], variant=1)
    lay_k = epx.layout(idx, wl["E"], wl["R"])
    torch.cuda.synchronize()
    for a, b in zip(_arrays(lay_f), _arrays(lay_k)):
        assert torch.equal(a, b)


def test_fused_empty_batch():
    idx = torch.zeros((0, 8), dtype=torch.int64, device="cuda")
    x = torch.zeros((0, 7168), dtype=torch.bfloat16, device="cuda")
    lay, recv, ex = epx.layout_dispatch_expand(idx, x, 256, 16, variant=1)
    t = epx.read_totals(lay)
    assert (t["N_route"], t["N_recv"], t["T_real"], t["dev_err"]) == (0, 0, 0, 0)
    assert lay.off_e.cpu().sum().item() == 0 and lay.cnt_r.cpu().sum().item() == 0


@pytest.mark.parametrize("T,variant,H", [(64, 1, 64), (64, 1, 4096), (64, 2, 64), (1536, 2, 64)],
                         ids=["one_launch", "one_launch_bulk", "paired_vec", "paired_bulk"])
@pytest.mark.parametrize("which", ["recv", "expanded", "both"])
def test_fused_capacity_overflow_flagged_not_written(T, variant, H, which):
    # "both": tokens whose every row lies beyond the capacities have their
    # chunk of x loaded before the dispatch's wait (paired path) and nothing
    # to write
    wl = _random_wl(T=T, H=H, E=16, R=4, k=4, seed=10)
    o = oracle.run_all(wl)
    x, idx, _ = gpu_inputs(wl)
    cap = 10
    canary = {n: torch.full((cap + 4, H), 7, dtype=torch.int16, device="cuda")
              for n in ("recv", "expanded")}
    bufs = {n: (canary[n][:cap].view(torch.bfloat16) if which in (n, "both") else
                torch.empty((T * 4, H), dtype=torch.bfloat16, device="cuda"))
            for n in ("recv", "expanded")}
    lay, _, _ = epx.layout_dispatch_expand(idx, x, 16, 4, recv=bufs["recv"],
                                           expanded=bufs["expanded"], variant=variant)
    t = epx.read_totals(lay, raise_on_error=False)
    want_err = {"recv": 2, "expanded": 4, "both": 6}[which]
    assert t["status"] == 3 and (t["dev_err"] & want_err) == want_err
    for n in ("recv", "expanded"):
        if which in (n, "both"):
            np.testing.assert_array_equal(torch_to_bits(bufs[n]), o[n][:cap])
            assert torch.all(canary[n][cap:] == 7)
        else:
            rows = o["layout"]["N_recv" if n == "recv" else "N_route"]
            np.testing.assert_array_equal(torch_to_bits(bufs[n][:rows]), o[n])
    assert_layout_equal(lay, o["layout"])


@pytest.mark.parametrize("H", [136, 4096], ids=["spread_stores", "bulk_stores"])
def test_fused_guard_bands_untouched(H):
    wl = _random_wl(T=200, H=H, E=32, R=8, k=6, seed=11, p_pad=0.3)
    o = oracle.run_all(wl)
    T, k, R = 200, 6, 8
    x, idx, _ = gpu_inputs(wl)
    G = 3
    big_r = torch.full((T * min(k, R) + 2 * G, H), -3, dtype=torch.int16, device="cuda")
    big_e = torch.full((T * k + 2 * G, H), -5, dtype=torch.int16, device="cuda")
    recv = big_r[G:-G].view(torch.bfloat16)
    ex = big_e[G:-G].view(torch.bfloat16)
    epx.layout_dispatch_expand(idx, x, 32, 8, recv=recv, expanded=ex, variant=1)
    torch.cuda.synchronize()
    nr, ne = o["layout"]["N_recv"], o["layout"]["N_route"]
    assert torch.all(big_r[:G] == -3) and torch.all(big_r[G + nr:] == -3)
    assert torch.all(big_e[:G] == -5) and torch.all(big_e[G + ne:] == -5)
    np.testing.assert_array_equal(torch_to_bits(recv[:nr]), o["recv"])
    np.testing.assert_array_equal(torch_to_bits(ex[:ne]), o["expanded"])


def test_fused_deterministic_across_runs():
    wl, _ = oracle_run("dp_compact", 0)
    x, idx, _ = gpu_inputs(wl)
    ref = None
    for _ in range(10):
        lay, recv, ex = epx.layout_dispatch_expand(idx, x, wl["E"], wl["R"], variant=1)
        t = epx.read_totals(lay)
        cur = [a.clone() for a in _arrays(lay)] + [recv[:t["N_recv"]].clone(),
                                                   ex[:t["N_route"]].clone()]
        if ref is None:
            ref = cur
        else:
            assert all(torch.equal(a, b) for a, b in zip(ref, cur))
