"""GPU edge cases: empty and ragged inputs, limits, duplicates, bad indices,
capacities, misalignment, guard bands around outputs."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import epx
from combine_ep_layout_07_b200 import workloads as wlmod

from gpu_helpers import (assert_all_equal, assert_combine_close, assert_layout_equal, run_gpu,
                         torch_to_bits)

pytestmark = pytest.mark.gpu


def _random_wl(T, H, E, R, k, seed, p_pad=0.0, dup=False, distinct=True):
    rng = np.random.default_rng(seed)
    x = wlmod.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    if distinct and k <= E:
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    else:
        idx = rng.integers(0, E, size=(T, k))
    if dup and T:
        idx[:, -1] = idx[:, 0]
    if p_pad:
        idx = np.where(rng.random((T, k)) < p_pad, -1, idx)
    w = rng.random((T, k), dtype=np.float32)
    w = np.where(idx >= 0, w, 0).astype(np.float32)
    return dict(x=x, topk_idx=idx.astype(np.int64), topk_weights=w, T=T, H=H, E=E, R=R, k=k)


def _check(wl, **kw):
    o = oracle.run_all(wl)
    g = run_gpu(wl, **kw)
    assert_all_equal(g, o)
    return g, o


@pytest.mark.parametrize("case", [
    dict(T=1, H=8, E=1, R=1, k=1),
    dict(T=3, H=8, E=4, R=4, k=4),
    dict(T=33, H=296, E=12, R=3, k=6),           # k does not divide 32; ragged H
    dict(T=257, H=1000, E=20, R=5, k=12),
    dict(T=5000, H=64, E=96, R=8, k=6),         # multi-CTA cluster, ragged split
    dict(T=8192, H=64, E=256, R=16, k=8),       # 8-CTA cluster
    dict(T=700, H=128, E=4096, R=64, k=32),     # every limit at its maximum
    dict(T=64, H=7168, E=64, R=64, k=32),       # k = R = 64 ranks... k=32 routes
    dict(T=40, H=14336, E=256, R=16, k=8),      # wide rows
])
@pytest.mark.parametrize("dv", [1, 2])
def test_random_shapes(case, dv):
    wl = _random_wl(seed=case["T"] + case["E"], p_pad=0.2, **case)
    for cv in (1, 2):
        _check(wl, dispatch_variant=dv, combine_variant=cv)


# shapes for both layout schedules: k not dividing 32 (idle lanes), k = 32,
# R not a multiple of 4 (scalar -1 fill), several passes of the warps, a
# cluster with a ragged last CTA, duplicates and bad indices in one batch
LAYOUT_CASES = [
    dict(T=1, H=8, E=1, R=1, k=1),
    dict(T=33, H=8, E=12, R=3, k=3),
    dict(T=300, H=8, E=60, R=6, k=6),
    dict(T=77, H=8, E=64, R=4, k=32),
    dict(T=3000, H=8, E=70, R=7, k=7),
    dict(T=5, H=8, E=8, R=8, k=1),
    dict(T=960, H=8, E=256, R=16, k=8),
    dict(T=8192, H=8, E=256, R=16, k=8),
]


@pytest.mark.parametrize("case", LAYOUT_CASES, ids=lambda c: "T{T}k{k}E{E}R{R}".format(**c))
@pytest.mark.parametrize("lv", [1, 2])
def test_layout_schedules_shapes(case, lv):
    wl = _random_wl(seed=case["T"] * 3 + case["k"], p_pad=0.2, distinct=False, **case)
    idx = wl["topk_idx"]
    if case["T"] > 3:
        idx[2, 0] = case["E"] + 5      # bad index: dropped and flagged
        idx[3, :] = -1                 # all-padding row
    if case["T"] > 1 and case["k"] > 1:
        idx[1, 1] = idx[1, 0]          # same expert twice in one token
    lay_o = oracle.layout(idx, case["E"], case["R"])
    lay = epx.layout(torch.from_numpy(idx).cuda(), case["E"], case["R"], variant=lv)
    torch.cuda.synchronize()
    assert_layout_equal(lay, lay_o)


GRID_CASES = [c for c in LAYOUT_CASES if c["T"] * c["k"] > 256] + [
    dict(T=4096, H=8, E=256, R=16, k=8),       # the prefill shape: 128 CTAs
    dict(T=16384, H=8, E=256, R=16, k=8),      # one CTA per SM, several passes
    dict(T=2000, H=8, E=1024, R=64, k=5),      # wide tables, k not dividing 32
]


@pytest.mark.parametrize("case", GRID_CASES, ids=lambda c: "T{T}k{k}E{E}R{R}".format(**c))
def test_layout_grid_schedule_shapes(case):
    """The grid schedule (variant 3): bit-exact, twice in a row on the same
    block (its barrier words are left zero by every call)."""
    wl = _random_wl(seed=case["T"] * 5 + case["k"], p_pad=0.2, distinct=False, **case)
    idx = wl["topk_idx"]
    idx[2, 0] = case["E"] + 5
    idx[3, :] = -1
    idx[1, 1] = idx[1, 0]
    lay_o = oracle.layout(idx, case["E"], case["R"])
    it = torch.from_numpy(idx).cuda()
    lay = epx.Layout(case["T"], case["k"], case["E"], case["R"], 64)
    for _ in range(2):
        epx.layout(it, case["E"], case["R"], out=lay, variant=3)
        torch.cuda.synchronize()
        assert_layout_equal(lay, lay_o)
        off = lay.c.work - lay.mem.data_ptr()
        assert torch.count_nonzero(lay.mem[off:off + 64]) == 0   # header back to zero


def test_layout_grid_schedule_refuses_single_cta():
    idx = torch.zeros((16, 8), dtype=torch.int64, device="cuda")
    with pytest.raises(epx.EpxError) as ei:
        epx.layout(idx, 16, 4, variant=3)
    assert ei.value.status == 6


def test_layout_grid_schedule_deterministic_and_interleaved():
    wl = _random_wl(T=4096, H=8, E=256, R=16, k=8, seed=21)
    it = torch.from_numpy(wl["topk_idx"]).cuda()
    lay_o = oracle.layout(wl["topk_idx"], 256, 16)
    lay = epx.Layout(4096, 8, 256, 16, 64)
    ref = None
    for i in range(20):
        epx.layout(it, 256, 16, out=lay, variant=(3, 1, 2, 0)[i % 4])
        snap = [a.clone() for a in (lay.cnt_e, lay.off_e, lay.cnt_r, lay.off_r, lay.pos,
                                    lay.recv_pos, lay.totals)]
        if ref is None:
            ref = snap
        assert all(torch.equal(a, b) for a, b in zip(snap, ref))
    assert_layout_equal(lay, lay_o)


def test_layout_warp_schedule_unsupported_shape():
    # the per-warp count table of E = 4096, R = 64 for 129 tokens of top-5
    # does not fit in shared memory: variant 1 refuses, auto and 2 agree
    wl = _random_wl(T=129, H=8, E=4096, R=64, k=5, seed=9)
    idx = torch.from_numpy(wl["topk_idx"]).cuda()
    with pytest.raises(RuntimeError, match="UNSUPPORTED|unsupported"):
        epx.layout(idx, 4096, 64, variant=1)
    lay_o = oracle.layout(wl["topk_idx"], 4096, 64)
    for lv in (0, 2):
        lay = epx.layout(idx, 4096, 64, variant=lv)
        torch.cuda.synchronize()
        assert_layout_equal(lay, lay_o)


def test_duplicates_within_row():
    wl = _random_wl(T=100, H=64, E=16, R=4, k=4, seed=3, dup=True)
    g, o = _check(wl)
    assert o["layout"]["N_route"] == 400


def test_non_distinct_random_routes():
    wl = _random_wl(T=300, H=64, E=8, R=2, k=8, seed=4, distinct=False)
    _check(wl)


def test_all_padding_rows():
    T, H, E, R, k = 64, 256, 16, 4, 4
    wl = dict(x=np.full((T, H), 0x3F80, np.uint16), topk_idx=-np.ones((T, k), np.int64),
              topk_weights=np.zeros((T, k), np.float32), T=T, H=H, E=E, R=R, k=k)
    g, o = _check(wl)
    assert g["totals"]["N_route"] == 0 and g["totals"]["N_recv"] == 0
    assert np.all(torch_to_bits(g["out"]) == 0)


def test_empty_batch():
    idx = torch.zeros((0, 8), dtype=torch.int64, device="cuda")
    lay = epx.layout(idx, 256, 16)
    x = torch.zeros((0, 7168), dtype=torch.bfloat16, device="cuda")
    recv, ex = epx.dispatch_expand(x, lay)
    y = epx.standin_expert(ex, lay)
    out = epx.combine_reduce(y, torch.zeros((0, 8), device="cuda"), lay)
    t = epx.read_totals(lay)
    assert (t["N_route"], t["N_recv"], t["T_real"], t["dev_err"]) == (0, 0, 0, 0)
    assert out.shape == (0, 7168)
    assert lay.off_e.cpu().sum().item() == 0 and lay.off_r.cpu().sum().item() == 0


def test_bad_indices_flagged_and_dropped():
    wl = _random_wl(T=50, H=64, E=16, R=4, k=4, seed=8)
    wl["topk_idx"][3, 1] = 16
    wl["topk_idx"][7, 0] = -2
    wl["topk_idx"][49, 3] = 1 << 40
    o = oracle.run_all(wl)
    assert o["layout"]["n_bad"] == 3
    x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).cuda()
    idx = torch.from_numpy(wl["topk_idx"]).cuda()
    lay = epx.layout(idx, 16, 4)
    with pytest.raises(epx.EpxError) as ei:
        epx.read_totals(lay)
    assert ei.value.status == 4
    recv, ex = epx.dispatch_expand(x, lay)
    y = epx.standin_expert(ex, lay)
    out = epx.combine_reduce(y, torch.from_numpy(wl["topk_weights"]).cuda(), lay)
    np.testing.assert_array_equal(lay.pos.cpu().numpy(), o["layout"]["pos"])
    np.testing.assert_array_equal(torch_to_bits(ex[:o["layout"]["N_route"]]), o["expanded"])
    assert_combine_close(torch_to_bits(out), o["out"])
    # int32 width: the 2^40 index cannot be represented; drop that case
    wl["topk_idx"][49, 3] = 99
    lay32 = epx.layout(torch.from_numpy(wl["topk_idx"]).to(torch.int32).cuda(), 16, 4)
    assert epx.read_totals(lay32, raise_on_error=False)["status"] == 4


def test_error_word_reset_by_next_layout():
    wl = _random_wl(T=8, H=64, E=16, R=4, k=4, seed=9)
    idx = torch.from_numpy(wl["topk_idx"]).cuda()
    bad = idx.clone()
    bad[0, 0] = 77
    lay = epx.layout(bad, 16, 4)
    assert epx.read_totals(lay, raise_on_error=False)["status"] == 4
    epx.layout(idx, 16, 4, out=lay)
    assert epx.read_totals(lay)["status"] == 0


def test_capacity_overflow_is_flagged_not_written():
    wl = _random_wl(T=64, H=64, E=16, R=4, k=4, seed=10)
    o = oracle.run_all(wl)
    x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).cuda()
    lay = epx.layout(torch.from_numpy(wl["topk_idx"]).cuda(), 16, 4)
    cap = 10
    canary = torch.full((cap + 4, 64), 7, dtype=torch.int16, device="cuda")
    recv = canary[:cap].view(torch.bfloat16)
    ex = torch.empty((64 * 4, 64), dtype=torch.bfloat16, device="cuda")
    for v in (1, 2):
        epx.dispatch_expand(x, lay, recv=recv, expanded=ex, variant=v)
        t = epx.read_totals(lay, raise_on_error=False)
        assert t["status"] == 3 and (t["dev_err"] & 2)
        np.testing.assert_array_equal(torch_to_bits(recv), o["recv"][:cap])
        assert torch.all(canary[cap:] == 7)


def test_guard_bands_untouched():
    wl = _random_wl(T=200, H=136, E=32, R=8, k=6, seed=11, p_pad=0.3)
    o = oracle.run_all(wl)
    T, H, k, R = 200, 136, 6, 8
    x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).cuda()
    w = torch.from_numpy(wl["topk_weights"]).cuda()
    lay = epx.layout(torch.from_numpy(wl["topk_idx"]).cuda(), 32, 8)
    G = 3
    for dv in (1, 2):
        for cv in (1, 2):
            big_r = torch.full((T * min(k, R) + 2 * G, H), -3, dtype=torch.int16, device="cuda")
            big_e = torch.full((T * k + 2 * G, H), -5, dtype=torch.int16, device="cuda")
            big_o = torch.full((T + 2 * G, H), -9, dtype=torch.int16, device="cuda")
            recv = big_r[G:-G].view(torch.bfloat16)
            ex = big_e[G:-G].view(torch.bfloat16)
            out = big_o[G:-G].view(torch.bfloat16)
            epx.dispatch_expand(x, lay, recv=recv, expanded=ex, variant=dv)
            y = epx.standin_expert(ex, lay)
            epx.combine_reduce(y, w, lay, out=out, variant=cv)
            nr, ne = o["layout"]["N_recv"], o["layout"]["N_route"]
            assert torch.all(big_r[:G] == -3) and torch.all(big_r[G + nr:] == -3)
            assert torch.all(big_e[:G] == -5) and torch.all(big_e[G + ne:] == -5)
            assert torch.all(big_o[:G] == -9) and torch.all(big_o[-G:] == -9)
            np.testing.assert_array_equal(torch_to_bits(recv[:nr]), o["recv"])
            assert_combine_close(torch_to_bits(out), o["out"])


def test_invalid_arguments_rejected():
    with pytest.raises(epx.EpxError) as ei:
        epx.Layout(16, 4, 10, 4)              # E % R != 0
    assert ei.value.status == 1
    with pytest.raises(epx.EpxError) as ei:
        epx.Layout(16, 33, 64, 4)             # k > 32
    assert ei.value.status == 6
    lay = epx.layout(torch.zeros((4, 2), dtype=torch.int64, device="cuda"), 4, 2)
    xb = torch.zeros(4 * 16 + 1, dtype=torch.bfloat16, device="cuda")
    x = xb[1:].view(4, 16)                    # 2-byte offset: misaligned rows
    with pytest.raises(epx.EpxError) as ei:
        epx.dispatch_expand(x, lay)
    assert ei.value.status == 2
    with pytest.raises(epx.EpxError) as ei:
        epx.dispatch_expand(torch.zeros((4, 12), dtype=torch.bfloat16, device="cuda"), lay)
    assert ei.value.status == 1               # H % 8 != 0


def test_roundtrip_host_matches_device_path():
    wl, _ = wl_o = (wlmod.make("decode", seed=0), None)
    o = oracle.run_all(wl)
    T, H, k, E, R = wl["T"], wl["H"], wl["k"], wl["E"], wl["R"]
    x_h = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    i_h = torch.from_numpy(wl["topk_idx"]).pin_memory()
    w_h = torch.from_numpy(wl["topk_weights"]).pin_memory()
    out_h = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    dev = torch.empty(epx.roundtrip_device_bytes(T, H, k, E, R), dtype=torch.uint8, device="cuda")
    epx.roundtrip_host(x_h, i_h, w_h, E, R, dev, out_h)
    torch.cuda.synchronize()
    assert_combine_close(torch_to_bits(out_h), o["out"])
