"""GPU checks of the multi-GPU expert-parallel pieces on one GPU: the routing
that travels with every sent row (ep_route_meta) against its definition, the
expand-only dispatch, and the whole ep_dist path in its one-rank case
against the CPU oracle and the single-GPU path."""
import numpy as np
import pytest
import torch

from combine_ep_layout_07_b200 import ep_dist, epx

from gpu_helpers import (assert_combine_close, gpu_inputs, oracle_run, run_gpu,
                         torch_to_bits)

pytestmark = pytest.mark.gpu


def _expected_meta(wl, lay_o):
    E, R, k = wl["E"], wl["R"], wl["k"]
    epr = E // R
    idx, w = wl["topk_idx"].astype(np.int64), wl["topk_weights"]
    n = lay_o["N_recv"]
    mi = np.full((n, k), -1, np.int32)
    mw = np.zeros((n, k), np.float32)
    for r in range(R):
        rows = lay_o["recv_pos"][:, r]
        sel = rows >= 0
        e = idx[sel]
        keep = (e >= 0) & (e < E) & (e // epr == r)
        mi[rows[sel]] = np.where(keep, e, -1)
        mw[rows[sel]] = np.where(keep, w[sel], 0.0)
    return mi, mw


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "lowbatch8", "dp_padded"])
@pytest.mark.parametrize("idx_dtype", [torch.int64, torch.int32], ids=["i64", "i32"])
def test_route_meta_matches_definition(name, idx_dtype):
    wl, o = oracle_run(name, 0)
    x, idx, w = gpu_inputs(wl, idx_dtype)
    lay = epx.layout(idx, wl["E"], wl["R"])
    mi, mw = epx.route_meta(idx, w, lay)
    n = o["layout"]["N_recv"]
    emi, emw = _expected_meta(wl, o["layout"])
    np.testing.assert_array_equal(mi[:n].cpu().numpy(), emi)
    np.testing.assert_array_equal(mw[:n].cpu().numpy(), emw)
    assert epx.read_totals(lay)["status"] == 0


def test_route_meta_capacity_flagged():
    wl, o = oracle_run("tiny", 0)
    x, idx, w = gpu_inputs(wl)
    lay = epx.layout(idx, wl["E"], wl["R"])
    cap = 7
    mi = torch.full((cap + 2, wl["k"]), 99, dtype=torch.int32, device="cuda")
    mw = torch.zeros((cap + 2, wl["k"]), dtype=torch.float32, device="cuda")
    epx.route_meta(idx, w, lay, meta_idx=mi[:cap], meta_w=mw[:cap])
    t = epx.read_totals(lay, raise_on_error=False)
    assert t["status"] == 3 and (t["dev_err"] & 2)
    emi, _ = _expected_meta(wl, o["layout"])
    np.testing.assert_array_equal(mi[:cap].cpu().numpy(), emi[:cap])
    assert torch.all(mi[cap:] == 99)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_expand_only_dispatch(name):
    wl, o = oracle_run(name, 0)
    x, idx, _ = gpu_inputs(wl)
    lay = epx.layout(idx, wl["E"], wl["R"])
    for v in (1, 2):
        recv, ex = epx.dispatch_expand(x, lay, expand_only=True, variant=v)
        assert recv is None
        ne = o["layout"]["N_route"]
        np.testing.assert_array_equal(torch_to_bits(ex[:ne]), o["expanded"])
        assert epx.read_totals(lay)["status"] == 0


@pytest.mark.parametrize("name", ["tiny", "decode", "lowbatch8", "dp_padded"])
def test_one_rank_expert_parallel_path(name):
    """ep_dist with no process group: every expert on this GPU, the
    exchanges the identity.  The expanded rows must be the oracle's bit for
    bit and the output the single-GPU combine's."""
    wl, o = oracle_run(name, 0)
    x, idx, w = gpu_inputs(wl)
    h = ep_dist.dispatch(x, idx, w, wl["E"])
    ne = o["layout"]["N_route"]
    np.testing.assert_array_equal(torch_to_bits(h.expanded[:ne]), o["expanded"])
    y = epx.standin_expert(h.expanded, h.layout_in)
    out = ep_dist.combine(h, y)
    assert_combine_close(torch_to_bits(out), o["out"])
    np.testing.assert_array_equal(torch_to_bits(out), torch_to_bits(run_gpu(wl)["out"]))
