"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Layout, recv, expanded and the stand-in expert output are compared bit for
bit; the combine output elementwise within |gpu - oracle| <= 2^-7 |oracle| + 1e-3.
All five workloads (the low-batch one at T = 1, 2, 4, 8; the DP batch compact
and padded) at their full sizes, seeds 0-2, both index widths, both layout
schedules, both copy engines and both combine schedules.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import epx
from combine_ep_layout_07_b200 import workloads as wlmod

from gpu_helpers import (assert_all_equal, assert_combine_close, assert_layout_equal,
                         bits_to_torch, oracle_run, run_gpu, torch_to_bits)

pytestmark = pytest.mark.gpu

ALL = ["tiny", "decode", "prefill", "lowbatch1", "lowbatch2", "lowbatch4", "lowbatch8",
       "dp_compact", "dp_padded"]
SEEDED = ["tiny", "decode", "prefill", "dp_compact", "dp_padded"]


@pytest.mark.parametrize("name", ALL)
def test_default_path_matches_oracle(name):
    wl, o = oracle_run(name, 0)
    g = run_gpu(wl)
    assert g["totals"]["status"] == 0
    assert_all_equal(g, o)


@pytest.mark.parametrize("seed", [1, 2])
@pytest.mark.parametrize("name", SEEDED)
def test_other_seeds(name, seed):
    wl, o = oracle_run(name, seed)
    assert_all_equal(run_gpu(wl), o)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "lowbatch8", "dp_padded"])
def test_int32_indices(name):
    wl, o = oracle_run(name, 0)
    assert_all_equal(run_gpu(wl, idx_dtype=torch.int32), o)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("name", ALL)
def test_layout_schedules(name, variant):
    wl, o = oracle_run(name, 0)
    assert_all_equal(run_gpu(wl, layout_variant=variant), o)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("name", ["decode", "prefill", "lowbatch8"])
def test_layout_schedules_int32(name, variant):
    wl, o = oracle_run(name, 1)
    assert_all_equal(run_gpu(wl, idx_dtype=torch.int32, layout_variant=variant), o)


@pytest.mark.parametrize("idx_dtype", [torch.int64, torch.int32], ids=["i64", "i32"])
@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "dp_compact", "dp_padded"])
def test_layout_grid_schedule(name, idx_dtype):
    wl, o = oracle_run(name, 0)
    assert_all_equal(run_gpu(wl, idx_dtype=idx_dtype, layout_variant=3), o)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "lowbatch1", "dp_padded"])
def test_dispatch_engines(name, variant):
    wl, o = oracle_run(name, 0)
    assert_all_equal(run_gpu(wl, dispatch_variant=variant), o)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "lowbatch1", "lowbatch8",
                                  "dp_compact"])
def test_combine_schedules(name, variant):
    wl, o = oracle_run(name, 0)
    assert_all_equal(run_gpu(wl, combine_variant=variant), o)


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_combine_on_oracle_expert_output(name):
    """Combine alone, fed the oracle's expert output rows."""
    wl, o = oracle_run(name, 0)
    y = torch.zeros((wl["T"] * wl["k"], wl["H"]), dtype=torch.bfloat16, device="cuda")
    y[:o["layout"]["N_route"]] = bits_to_torch(o["y"])
    g = run_gpu(wl, y_override=y)
    assert_combine_close(torch_to_bits(g["out"]), o["out"])


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_lowbatch_worked_example_exact(T):
    """DeepEP issue #760 reproduction shape: row 0 is 79/64 exactly with the
    stand-in experts and x = 1, padding rows are +0."""
    wl = wlmod.make_lowbatch(T)
    g = run_gpu(wl)
    out = torch_to_bits(g["out"])
    assert np.all(out[0] == 0x3F9E)          # 1.234375 = 79/64
    assert np.all(out[1:] == 0)
    for v in (1, 2):
        g2 = run_gpu(wl, combine_variant=v)
        np.testing.assert_array_equal(torch_to_bits(g2["out"]), out)


def test_identity_experts_round_trip_x():
    wl, o = oracle_run("decode", 0)
    g = run_gpu(wl, y_override=None)
    out = epx.combine_reduce(g["expanded"], torch.from_numpy(wl["topk_weights"]).cuda(),
                             g["layout"])
    np.testing.assert_array_equal(torch_to_bits(out), wl["x"])


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_deterministic_across_runs(name):
    wl, o = oracle_run(name, 0)
    rows = {"recv": o["layout"]["N_recv"], "expanded": o["layout"]["N_route"],
            "out": wl["T"]}    # rows past N_recv / N_route are never written
    g0 = run_gpu(wl)
    ref = {k: torch_to_bits(g0[k][:n]) for k, n in rows.items()}
    pos0 = g0["layout"].pos.cpu().numpy()
    rp0 = g0["layout"].recv_pos.cpu().numpy()
    for _ in range(20):
        g = run_gpu(wl)
        np.testing.assert_array_equal(g["layout"].pos.cpu().numpy(), pos0)
        np.testing.assert_array_equal(g["layout"].recv_pos.cpu().numpy(), rp0)
        for k, n in rows.items():
            np.testing.assert_array_equal(torch_to_bits(g[k][:n]), ref[k])


@pytest.mark.parametrize("layout_variant", [0, 2])
def test_dp_compact_and_padded_agree_on_gpu(layout_variant):
    # the same 127 real tokens laid out compact (127 rows) and padded (960
    # rows, group g at rows 120g...): identical totals and copies, identical
    # real output rows, +0.0 padding rows
    c = run_gpu(wlmod.make("dp_compact", seed=0), layout_variant=layout_variant)
    p = run_gpu(wlmod.make("dp_padded", seed=0), layout_variant=layout_variant)
    for key in ("N_route", "N_recv", "T_real"):
        assert c["totals"][key] == p["totals"][key]
    np.testing.assert_array_equal(c["layout"].cnt_e.cpu().numpy(), p["layout"].cnt_e.cpu().numpy())
    n_route, n_recv = c["totals"]["N_route"], c["totals"]["N_recv"]
    np.testing.assert_array_equal(torch_to_bits(c["expanded"][:n_route]),
                                  torch_to_bits(p["expanded"][:n_route]))
    np.testing.assert_array_equal(torch_to_bits(c["recv"][:n_recv]),
                                  torch_to_bits(p["recv"][:n_recv]))
    rows = np.concatenate([np.arange(120), 120 * np.arange(1, 8)])
    out_c, out_p = torch_to_bits(c["out"]), torch_to_bits(p["out"])
    np.testing.assert_array_equal(out_p[rows], out_c)
    mask = np.ones(960, bool)
    mask[rows] = False
    assert np.all(out_p[mask] == 0)
