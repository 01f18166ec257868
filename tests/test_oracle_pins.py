"""Pins for the CPU oracle, checked against things other than itself.

* bf16 rounding: brute-force nearest search over the whole bf16 grid (exact
  rationals), and torch's CPU float->bf16 cast.
* layout: a sort-based brute force on tiny random cases (a different algorithm
  from the oracle's count / scan / cursor walk), invariants on every workload,
  and the low-batch closed form printed in DeepEP issue #760, Reproduction.
* dispatch / expand: the defining byte equalities.
* stand-in expert: torch fp32 arithmetic and torch's bf16 cast.
* combine: the closed form out[t] = sum_j w[t,j] (1 + e[t,j]/E) x[t] within the
  bf16 error bound, bit-exact round trip of x through identity experts with
  normalised weights, weights used without renormalisation, zero rows for
  padding tokens, and the worked example of issue #760 (golden fixture).
* two-stage combine (local reduce, then epilogue): with unit expert outputs
  every partial is the token's local gate-weight sum (the issue #760 fake
  expert output); the issue #760 worked example through both stages; the
  partials of all ranks add up to the single-stage sum; the residual-add
  epilogue returns the residual for zero partials.
"""
import bisect
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import workloads as wlmod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- bf16 pins

def _all_finite_nonneg_bf16():
    vals = []
    for b in range(0x0000, 0x7F80):
        u = np.array([b << 16], dtype=np.uint32).view(np.float32)[0]
        vals.append((Fraction(float(u)), b))
    vals.sort()
    return vals


_BF16_GRID = None


def _brute_bf16(v: float) -> int:
    """Nearest bf16 to v by search over every finite bf16 value, ties to the
    even bit pattern; beyond max-finite + half ulp -> inf."""
    global _BF16_GRID
    if _BF16_GRID is None:
        _BF16_GRID = _all_finite_nonneg_bf16()
    sign = 0x8000 if np.signbit(v) else 0
    a = Fraction(abs(v))
    keys = [g[0] for g in _BF16_GRID]
    i = bisect.bisect_left(keys, a)
    cands = []
    for j in (i - 1, i):
        if 0 <= j < len(_BF16_GRID):
            cands.append(_BF16_GRID[j])
    top_val, top_bits = _BF16_GRID[-1]
    half_ulp = (Fraction(2) ** 127 * 2 - top_val) / 2   # (2^128 - max)/2
    if a >= top_val + half_ulp:
        return sign | 0x7F80
    best = min(cands, key=lambda c: (abs(c[0] - a), c[1] & 1))
    return sign | best[1]


def test_bf16_rounding_matches_bruteforce_on_edge_values():
    rng = np.random.default_rng(5)
    vals = [0.0, 1.0, -1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,   # exact ties
            1.0 + 2.0 ** -8 + 2.0 ** -40,                          # just above a tie
            1.0 + 2.0 ** -8 - 2.0 ** -40,
            1.0 + 2.0 ** -8 + 2.0 ** -30,                          # double-rounding trap
            2.0 ** -126, 2.0 ** -133, 3 * 2.0 ** -134, 2.0 ** -135, 2.0 ** -134,
            2.0 ** -130 * 1.5, 3.3895313892515355e38, 3.4e38, 3.39e38, -3.5e38,
            65504.0, 1e-40, -7.25e-39]
    vals += list(rng.standard_normal(300))
    vals += list(rng.standard_normal(100) * 1e-39)
    vals += list((rng.standard_normal(100) * 2.0 ** rng.integers(-60, 60, 100)))
    for v in vals:
        assert oracle.bf16_from_double(v) == _brute_bf16(float(v)), v


def test_bf16_rounding_matches_torch_cast_of_floats():
    rng = np.random.default_rng(6)
    f = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e-38).astype(np.float32),
        # exact ties: a bf16 value plus half its ulp, in float32
        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        (np.arange(0x3F80, 0x4100, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
    ])
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_double(float(v)) for v in f], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)


def test_bf16_to_double_exact():
    for b in (0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x4049):
        want = float(np.array([b << 16], np.uint32).view(np.float32)[0])
        assert oracle.bf16_to_double(b) == want


# --------------------------------------------------------------- layout pins

def _brute_layout(idx, E, R):
    """Sort-based definition: a route's row is its rank among all valid routes
    ordered by (expert, token, slot); a (token, rank) pair's row is its rank
    among all pairs ordered by (rank, token)."""
    T, k = idx.shape
    epr = E // R
    routes = [(int(idx[t, j]), t, j) for t in range(T) for j in range(k)
              if 0 <= idx[t, j] < E]
    routes.sort()
    pos = -np.ones((T, k), np.int64)
    for n, (_, t, j) in enumerate(routes):
        pos[t, j] = n
    pairs = sorted({(int(idx[t, j]) // epr, t) for t in range(T) for j in range(k)
                    if 0 <= idx[t, j] < E})
    recv_pos = -np.ones((T, R), np.int64)
    for n, (r, t) in enumerate(pairs):
        recv_pos[t, r] = n
    cnt_e = np.zeros(E, np.int64)
    for e, _, _ in routes:
        cnt_e[e] += 1
    cnt_r = np.zeros(R, np.int64)
    for r, _ in pairs:
        cnt_r[r] += 1
    n_bad = int(((idx < -1) | (idx >= E)).sum())
    t_real = len({t for _, t, _ in routes})
    return dict(pos=pos, recv_pos=recv_pos, cnt_e=cnt_e, cnt_r=cnt_r,
                N_route=len(routes), N_recv=len(pairs), n_bad=n_bad, T_real=t_real)


def _check_against_brute(idx, E, R):
    b = _brute_layout(idx, E, R)
    for dt in (np.int64, np.int32):
        o = oracle.layout(idx.astype(dt), E, R)
        np.testing.assert_array_equal(o["pos"], b["pos"])
        np.testing.assert_array_equal(o["recv_pos"], b["recv_pos"])
        np.testing.assert_array_equal(o["cnt_e"], b["cnt_e"])
        np.testing.assert_array_equal(o["cnt_r"], b["cnt_r"])
        np.testing.assert_array_equal(o["off_e"], np.concatenate([[0], np.cumsum(b["cnt_e"])]))
        np.testing.assert_array_equal(o["off_r"], np.concatenate([[0], np.cumsum(b["cnt_r"])]))
        assert (o["N_route"], o["N_recv"], o["n_bad"], o["T_real"]) == (
            b["N_route"], b["N_recv"], b["n_bad"], b["T_real"])


@pytest.mark.parametrize("seed", range(60))
def test_layout_matches_bruteforce_on_micro_cases(seed):
    rng = np.random.default_rng(1000 + seed)
    T = int(rng.integers(0, 9))
    E = int(rng.choice([1, 2, 4, 6, 8]))
    R = int(rng.choice([r for r in (1, 2, 4) if E % r == 0]))
    k = int(rng.integers(1, 5))
    # -1 padding, duplicates, and a few bad indices
    idx = rng.integers(-1, E, size=(T, k))
    if T and rng.random() < 0.3:
        idx[rng.integers(0, T), rng.integers(0, k)] = rng.choice([E, E + 3, -2, -7])
    _check_against_brute(idx, E, R)


def test_layout_matches_bruteforce_on_tiny_workload():
    wl = wlmod.make("tiny", seed=0)
    _check_against_brute(wl["topk_idx"], wl["E"], wl["R"])


def test_layout_rejects_uneven_expert_split():
    with pytest.raises(ValueError):
        oracle.layout(np.zeros((2, 2), np.int64), 6, 4)


def _check_invariants(idx, E, R, o):
    T, k = idx.shape
    valid = (idx >= 0) & (idx < E)
    assert o["cnt_e"].sum() == o["N_route"] == valid.sum()
    ranks = [set((idx[t][valid[t]] // (E // R)).tolist()) for t in range(T)]
    assert o["cnt_r"].sum() == o["N_recv"] == sum(len(s) for s in ranks)
    assert o["T_real"] == sum(1 for s in ranks if s)
    assert np.all(np.diff(o["off_e"]) >= 0) and o["off_e"][-1] == o["N_route"]
    assert np.all(np.diff(o["off_r"]) >= 0) and o["off_r"][-1] == o["N_recv"]
    p = o["pos"][valid]
    assert np.array_equal(np.sort(p), np.arange(o["N_route"]))     # bijection
    assert np.all(o["pos"][~valid] == -1)
    # each route lands in its expert's segment, in (token, slot) order
    e = idx[valid]
    assert np.all((p >= o["off_e"][e]) & (p < o["off_e"][e + 1]))
    order = np.lexsort((np.nonzero(valid)[1], np.nonzero(valid)[0], e))
    assert np.all(np.diff(p[order]) == 1)
    rp = o["recv_pos"]
    hit = rp >= 0
    assert hit.sum() == o["N_recv"]
    assert np.array_equal(np.sort(rp[hit]), np.arange(o["N_recv"]))
    for r in range(R):
        col = rp[:, r][hit[:, r]]
        assert np.all(np.diff(col) == 1)
        if col.size:
            assert col[0] == o["off_r"][r] and col[-1] == o["off_r"][r + 1] - 1


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "lowbatch1", "lowbatch8",
                                  "dp_compact", "dp_padded"])
def test_layout_invariants_on_workloads(name):
    wl = wlmod.make(name, seed=0)
    o = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    _check_invariants(wl["topk_idx"], wl["E"], wl["R"], o)
    o32 = oracle.layout(wl["topk_idx"].astype(np.int32), wl["E"], wl["R"])
    for key in ("pos", "recv_pos", "cnt_e", "cnt_r", "off_e", "off_r", "totals"):
        np.testing.assert_array_equal(o[key], o32[key])


def _golden():
    with open(os.path.join(GOLDEN, "lowbatch_combine_issue760.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_layout_lowbatch_closed_form(T):
    g = _golden()
    wl = wlmod.make_lowbatch(T)
    o = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    want_e = np.zeros(wl["E"], np.int32)
    want_e[np.arange(16) * 28] = 1
    np.testing.assert_array_equal(o["cnt_e"], want_e)
    np.testing.assert_array_equal(o["cnt_r"], g["layout"]["cnt_r"])
    assert o["N_route"] == g["layout"]["N_route"]
    assert o["N_recv"] == g["layout"]["N_recv"]
    assert o["T_real"] == g["layout"]["T_real"]
    np.testing.assert_array_equal(o["pos"][0], np.arange(16))
    np.testing.assert_array_equal(o["recv_pos"][0, :16], np.arange(16))
    assert np.all(o["recv_pos"][0, 16:] == -1)
    assert np.all(o["pos"][1:] == -1) and np.all(o["recv_pos"][1:] == -1)


# ---------------------------------------------------- dispatch / expand pins

@pytest.mark.parametrize("name", ["tiny", "decode", "dp_padded", "lowbatch4"])
def test_dispatch_expand_definition(name):
    wl = wlmod.make(name, seed=1)
    lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    recv, expanded = oracle.dispatch_expand(wl["x"], lay)
    x = wl["x"]
    T, R = lay["T"], lay["R"]
    for t in range(T):
        for r in range(R):
            d = lay["recv_pos"][t, r]
            if d >= 0:
                assert np.array_equal(recv[d], x[t])
        for j in range(lay["k"]):
            p = lay["pos"][t, j]
            if p >= 0:
                assert np.array_equal(expanded[p], x[t])
    assert recv.shape[0] == lay["N_recv"] and expanded.shape[0] == lay["N_route"]


# ------------------------------------------------------------ stand-in pins

def _torch_standin(expanded_bits, expert_of_row, E):
    xf = torch.from_numpy(expanded_bits.view(np.int16)).view(torch.bfloat16).float()
    e = torch.from_numpy(expert_of_row.astype(np.float32))
    scale = 1.0 + e / float(E)                      # fp32 tensor ops (IEEE)
    return (xf * scale[:, None]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name", ["tiny", "decode", "lowbatch1"])
def test_standin_matches_torch(name):
    wl = wlmod.make(name, seed=2)
    lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    _, expanded = oracle.dispatch_expand(wl["x"], lay)
    y = oracle.standin(expanded, lay)
    expert_of_row = np.repeat(np.arange(wl["E"]), lay["cnt_e"])
    np.testing.assert_array_equal(y, _torch_standin(expanded, expert_of_row, wl["E"]))


# ------------------------------------------------------------- combine pins

def _closed_form(wl):
    x = wlmod.bf16_bits_to_f32(wl["x"]).astype(np.float64)
    idx = wl["topk_idx"]
    w = wl["topk_weights"].astype(np.float64)
    valid = idx >= 0
    scale = np.where(valid, 1.0 + idx.astype(np.float64) / wl["E"], 0.0)
    coef = (w * scale * valid).sum(axis=1)
    return coef[:, None] * x


@pytest.mark.parametrize("name", ["tiny", "decode", "dp_padded", "lowbatch2"])
def test_combine_closed_form(name):
    wl = wlmod.make(name, seed=0)
    res = oracle.run_all(wl)
    cf = _closed_form(wl)
    got = wlmod.bf16_bits_to_f32(res["out"]).astype(np.float64)
    # y rounding (2^-8 relative) + final rounding (2^-8 relative); every term
    # of a row has the sign of x (w >= 0, scale > 0) so nothing cancels
    assert np.all(np.abs(got - cf) <= 2.0 ** -7 * np.abs(cf) + 1e-300)


@pytest.mark.parametrize("name", ["tiny", "decode", "dp_compact"])
def test_combine_identity_experts_round_trip_x(name):
    wl = wlmod.make(name, seed=3)
    lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    _, expanded = oracle.dispatch_expand(wl["x"], lay)
    out = oracle.combine(expanded, wl["topk_weights"], lay)   # identity experts
    real = lay["pos"].max(axis=1) >= 0
    np.testing.assert_array_equal(out[real], wl["x"][real])
    assert np.all(out[~real] == 0)


def test_combine_uses_weights_as_given():
    T, H, E, R = 3, 16, 4, 2
    rng = np.random.default_rng(9)
    x = wlmod.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    idx = np.array([[0, 3], [1, -1], [-1, -1]])
    w = np.array([[0.25, 0.25], [0.5, 7.0], [3.0, 3.0]], np.float32)
    lay = oracle.layout(idx, E, R)
    _, expanded = oracle.dispatch_expand(x, lay)
    out = oracle.combine(expanded, w, lay)
    xf = wlmod.bf16_bits_to_f32(x)
    # 0.5 x and 0.5 x: power-of-two scaling is exact; -1 routes ignore weight
    np.testing.assert_array_equal(wlmod.bf16_bits_to_f32(out[0]), 0.5 * xf[0])
    np.testing.assert_array_equal(wlmod.bf16_bits_to_f32(out[1]), 0.5 * xf[1])
    assert np.all(out[2] == 0)


def test_combine_duplicate_expert_counts_twice():
    T, H, E, R = 1, 8, 4, 2
    x = wlmod.to_bf16_bits(np.full((T, H), 1.5, np.float32))
    idx = np.array([[2, 2]])
    w = np.array([[0.25, 0.5]], np.float32)
    lay = oracle.layout(idx, E, R)
    assert lay["N_route"] == 2 and lay["N_recv"] == 1
    res = oracle.run_all(dict(x=x, topk_idx=idx, topk_weights=w, E=E, R=R))
    # expert 2 of 4 scales by 1.5: 0.75 * (1.5 * 1.5) = 1.6875 (exact in bf16)
    np.testing.assert_array_equal(wlmod.bf16_bits_to_f32(res["out"]), np.full((1, H), 1.6875))


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_combine_worked_example_issue760(T):
    g = _golden()
    for case in g["cases"]:
        val = case.get("x_value", 1.0)
        wl = wlmod.make_lowbatch(T, value=val)
        lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
        _, expanded = oracle.dispatch_expand(wl["x"], lay)
        if case["expert_output"] == "ones":
            y = np.full_like(expanded, 0x3F80)
        elif case["expert_output"] == "identity":
            y = expanded
        else:
            y = oracle.standin(expanded, lay)
        out = wlmod.bf16_bits_to_f32(oracle.combine(y, wl["topk_weights"], lay))
        assert np.all(out[0] == case["expected_real_row"]), case["what"]
        assert np.all(out[1:] == case["expected_padding_rows"])
        assert not np.any(np.signbit(out[1:]))


def test_dp_compact_and_padded_agree():
    c = oracle.run_all(wlmod.make("dp_compact", seed=0))
    p = oracle.run_all(wlmod.make("dp_padded", seed=0))
    for key in ("N_route", "N_recv", "T_real"):
        assert c["layout"][key] == p["layout"][key]
    np.testing.assert_array_equal(c["layout"]["cnt_e"], p["layout"]["cnt_e"])
    np.testing.assert_array_equal(c["expanded"], p["expanded"])
    np.testing.assert_array_equal(c["recv"], p["recv"])
    rows = np.concatenate([np.arange(120), 120 * np.arange(1, 8)])
    np.testing.assert_array_equal(p["out"][rows], c["out"])
    mask = np.ones(960, bool)
    mask[rows] = False
    assert np.all(p["out"][mask] == 0)


def test_empty_batch():
    idx = np.zeros((0, 4), np.int64)
    lay = oracle.layout(idx, 16, 4)
    assert lay["N_route"] == lay["N_recv"] == lay["T_real"] == 0
    assert np.all(lay["off_e"] == 0) and np.all(lay["off_r"] == 0)


def test_bad_indices_are_counted_and_dropped():
    idx = np.array([[0, 16, -1, -5], [3, 3, 99, 15]])
    lay = oracle.layout(idx, 16, 4)
    assert lay["n_bad"] == 3
    assert lay["N_route"] == 4
    assert list(lay["pos"][0]) == [0, -1, -1, -1]


# ------------------------------------------------ two-stage combine pins

def _rank_of(idx, E, R):
    return np.where(idx >= 0, idx // (E // R), -1)


@pytest.mark.parametrize("name", ["tiny", "decode", "dp_padded"])
def test_local_partials_of_unit_expert_output_are_local_weight_sums(name):
    """DeepEP issue #760, Reproduction: the fake expert output makes each
    received row the sum of its valid local gate weights (top-k weights
    masked to the rank's own experts).  With every expert output = 1 that is
    exactly what the local reduce must produce, per (token, rank)."""
    wl = wlmod.make(name, seed=4)
    lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    ones = np.full((lay["N_route"], wl["H"]), 0x3F80, np.uint16)
    part = oracle.combine_local(ones, wl["topk_weights"], lay, part_bits=32)
    rk = _rank_of(wl["topk_idx"], wl["E"], wl["R"])
    w = wl["topk_weights"].astype(np.float64)
    for t in range(lay["T"]):
        for r in range(lay["R"]):
            d = lay["recv_pos"][t, r]
            if d < 0:
                assert not np.any(rk[t] == r)
                continue
            masked = np.where(rk[t] == r, w[t], 0.0).sum()   # masked_fill(idx<0, 0).sum
            assert np.all(part[d] == np.float32(masked))


def test_two_stage_worked_example_issue760():
    """Sixteen ranks each hold one route of weight 1/16: every partial row is
    1/16 and the epilogue gives exactly 1 for the real row, 0 for padding
    rows (the value the page checks with an all-reduced max error)."""
    for T in (1, 2, 4, 8):
        wl = wlmod.make_lowbatch(T)
        lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
        ones = np.full((lay["N_route"], wl["H"]), 0x3F80, np.uint16)
        for bits in (32, 16):
            part = oracle.combine_local(ones, wl["topk_weights"], lay, part_bits=bits)
            pf = part if bits == 32 else wlmod.bf16_bits_to_f32(part)
            assert part.shape[0] == 16 and np.all(pf == 0.0625)
            out = wlmod.bf16_bits_to_f32(oracle.combine_epilogue(part, lay))
            assert np.all(out[0] == 1.0) and np.all(out[1:] == 0)


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill"])
def test_two_stage_sums_to_single_stage(name):
    """The partials of all ranks add up to the whole weighted sum: summed in
    double they match the single-stage sum up to fp32 rounding of each
    partial, and the epilogue output matches the closed form."""
    wl = wlmod.make(name, seed=0)
    res = oracle.run_all(wl)
    lay = res["layout"]
    _, exact = oracle.combine(res["y"], wl["topk_weights"], lay, exact=True)
    part = oracle.combine_local(res["y"], wl["topk_weights"], lay, part_bits=32)
    acc = np.zeros_like(exact)
    for t in range(lay["T"]):
        rows = lay["recv_pos"][t][lay["recv_pos"][t] >= 0]
        if rows.size:
            acc[t] = part[rows].astype(np.float64).sum(axis=0)
    scale = np.abs(part).astype(np.float64).max() if part.size else 0.0
    assert np.all(np.abs(acc - exact) <= lay["R"] * 2.0 ** -23 * scale + 1e-30)
    out = wlmod.bf16_bits_to_f32(oracle.combine_epilogue(part, lay)).astype(np.float64)
    cf = _closed_form(wl)
    assert np.all(np.abs(out - cf) <= 2.0 ** -7 * np.abs(cf) + 1e-30)


def test_epilogue_residual_add():
    wl = wlmod.make("tiny", seed=6)
    res = oracle.run_all(wl)
    lay = res["layout"]
    part = oracle.combine_local(res["y"], wl["topk_weights"], lay, part_bits=32)
    # zero partials: the output is the residual row, bit for bit
    out0 = oracle.combine_epilogue(np.zeros_like(part), lay, residual=wl["x"])
    np.testing.assert_array_equal(out0, wl["x"])
    # residual = x: out = x + sum  (every term has the sign of x: no cancellation)
    out = wlmod.bf16_bits_to_f32(oracle.combine_epilogue(part, lay, residual=wl["x"]))
    want = wlmod.bf16_bits_to_f32(wl["x"]).astype(np.float64) + _closed_form(wl)
    assert np.all(np.abs(out - want) <= 2.0 ** -7 * np.abs(want) + 1e-30)


# ------------------------------------------- dispatch without expand pins

@pytest.mark.parametrize("name", ["tiny", "decode", "dp_padded", "lowbatch2"])
def test_expand_index_serves_every_expanded_row(name):
    """Reading recv through the gather index gives exactly the expanded rows
    (the copy a do_expand=False consumer avoids), and every index stays in the
    owning rank's receive segment."""
    wl = wlmod.make(name, seed=2)
    lay = oracle.layout(wl["topk_idx"], wl["E"], wl["R"])
    recv, expanded = oracle.dispatch_expand(wl["x"], lay)
    src = oracle.expand_index(lay)
    assert src.shape == (lay["N_route"],) and np.all(src >= 0)
    np.testing.assert_array_equal(recv[src], expanded)
    epr = wl["E"] // wl["R"]
    expert_of_row = np.repeat(np.arange(wl["E"]), lay["cnt_e"])
    rank_of_row = expert_of_row // epr
    assert np.all(src >= lay["off_r"][rank_of_row]) and np.all(src < lay["off_r"][rank_of_row + 1])
