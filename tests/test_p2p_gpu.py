"""GPU parity of the peer-memory transport (ep_dispatch_p2p,
ep_combine_local_reduce_p2p), with the ranks emulated on one GPU: every
logical rank's buffers are separate allocations of this GPU, the kernels of
one rank run one after another (none waits on another), and the pointers the
kernels get are the same kind a real run gets from CUDA IPC.

What the pages' setting fixes (DeepEP issue #48: a token goes once to every
rank that owns one of its experts, with its routing; the partials reduced
per rank go back): rank r's buffer must hold, from row 0, the rows every
source sends it -- source by source, each in its own send order -- which
are bit for bit the rows ep_dispatch + ep_route_meta put in the source's
send block for r; and the partials stored back must be bit for bit what
ep_combine_local_reduce computes on the receiving rank, at the source's
receive-layout rows, so the source's epilogue gives the single-GPU result."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import ep_dist, epx
from combine_ep_layout_07_b200 import workloads as wlmod

from gpu_helpers import assert_combine_close, torch_to_bits

pytestmark = pytest.mark.gpu


def _sources(R, E, k, H, T_of, seed, p_pad=0.15, idx_dtype=torch.int64):
    out = []
    for g, T in enumerate(T_of):
        rng = np.random.default_rng(seed * 100 + g)
        x = wlmod.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int64)
        idx[rng.random((T, k)) < p_pad] = -1
        if T > 3:
            idx[3, :] = -1                    # a token that goes nowhere
        w = rng.random((T, k), dtype=np.float32)
        out.append(dict(
            T=T, x_bits=x, idx=idx, w=w,
            x=torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda(),
            idx_t=torch.from_numpy(idx).to(idx_dtype).cuda(),
            w_t=torch.from_numpy(w).cuda()))
    return out


def _emulate(R, E, k, H, T_of, seed, partial_dtype=torch.float32, idx_dtype=torch.int64):
    src = _sources(R, E, k, H, T_of, seed, idx_dtype=idx_dtype)
    lays = [epx.layout(s["idx_t"], E, R) for s in src]
    counts = torch.stack([l.cnt_r.cpu() for l in lays])
    cap = sum(T_of)
    bufs = [dict(rows=torch.full((cap, H), -7, dtype=torch.int16, device="cuda"),
                 meta_idx=torch.full((cap, k), 99, dtype=torch.int32, device="cuda"),
                 meta_w=torch.full((cap, k), 9.0, dtype=torch.float32, device="cuda"))
            for _ in range(R)]
    for g, s in enumerate(src):
        plan = ep_dist.p2p_plan(counts, g)
        peers = [epx.PeerRows(bufs[r]["rows"].view(torch.bfloat16), cap,
                              row0=plan["dispatch_row0"][r], meta_idx=bufs[r]["meta_idx"],
                              meta_w=bufs[r]["meta_w"]) for r in range(R)]
        epx.dispatch_p2p(s["x"], s["idx_t"], s["w_t"], lays[g], peers)
    torch.cuda.synchronize()
    return src, lays, counts, cap, bufs


CASES = [
    dict(R=2, E=16, k=4, H=64, T_of=[37, 50]),
    dict(R=4, E=32, k=6, H=136, T_of=[1, 0, 64, 9]),     # a rank with no tokens, k not 2^n
    dict(R=8, E=256, k=8, H=7168, T_of=[16] * 8),        # the decode shape, 16 tokens per rank
    dict(R=64, E=128, k=32, H=8, T_of=[3] * 63 + [0]),   # R and k at their maxima
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R{R}E{E}k{k}H{H}".format(**c))
@pytest.mark.parametrize("idx_dtype", [torch.int64, torch.int32], ids=["i64", "i32"])
def test_p2p_dispatch_places_rows_and_routing(case, idx_dtype):
    R, E, k, H = case["R"], case["E"], case["k"], case["H"]
    src, lays, counts, cap, bufs = _emulate(R, E, k, H, case["T_of"], seed=1, idx_dtype=idx_dtype)
    # the source-side reference: send blocks of ep_dispatch + ep_route_meta
    sends = []
    for s, lay in zip(src, lays):
        send = epx.dispatch(s["x"], lay)
        mi, mw = epx.route_meta(s["idx_t"], s["w_t"], lay)
        sends.append((torch_to_bits(send), mi.cpu().numpy(), mw.cpu().numpy(),
                      lay.off_r.cpu().numpy()))
    for r in range(R):
        want_rows, want_mi, want_mw = [], [], []
        for g in range(R):
            rows, mi, mw, off = sends[g]
            a, b = off[r], off[r + 1]
            want_rows.append(rows[a:b])
            want_mi.append(mi[a:b])
            want_mw.append(mw[a:b])
        n = int(counts[:, r].sum())
        np.testing.assert_array_equal(bufs[r]["rows"][:n].cpu().numpy().view(np.uint16),
                                      np.concatenate(want_rows))
        np.testing.assert_array_equal(bufs[r]["meta_idx"][:n].cpu().numpy(), np.concatenate(want_mi))
        np.testing.assert_array_equal(bufs[r]["meta_w"][:n].cpu().numpy(), np.concatenate(want_mw))
        assert torch.all(bufs[r]["rows"][n:] == -7) and torch.all(bufs[r]["meta_idx"][n:] == 99)
    for lay in lays:
        assert epx.read_totals(lay)["status"] == 0


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R{R}E{E}k{k}H{H}".format(**c))
@pytest.mark.parametrize("partial_dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
def test_p2p_combine_returns_partials_to_sources(case, partial_dtype):
    R, E, k, H = case["R"], case["E"], case["k"], case["H"]
    src, lays, counts, cap, bufs = _emulate(R, E, k, H, case["T_of"], seed=2)
    back_cap = max(max(case["T_of"]) * min(k, R), 1)
    backs = [torch.full((back_cap, H), -5, dtype=torch.int16 if partial_dtype == torch.bfloat16
                        else torch.int32, device="cuda").view(partial_dtype) for _ in range(R)]
    local = []
    for r in range(R):
        plan = ep_dist.p2p_plan(counts, r)
        n = plan["n_recv"]
        rows = bufs[r]["rows"][:n].view(torch.bfloat16)
        mi, mw = bufs[r]["meta_idx"][:n], bufs[r]["meta_w"][:n]
        lay_in = epx.layout(mi, E, R)
        _, expanded = epx.dispatch_expand(rows, lay_in, expand_only=True)
        y = epx.standin_expert(expanded, lay_in)
        part = epx.combine_local_reduce(y, mw, lay_in, partial_dtype=partial_dtype)
        peers = [epx.PeerRows(backs[s], back_cap, row0=plan["back_row0"][s],
                              first=plan["back_first"][s], count=plan["back_count"][s])
                 for s in range(R)]
        epx.combine_local_reduce_p2p(y, mw, lay_in, peers, partial_dtype=partial_dtype)
        assert epx.read_totals(lay_in)["status"] == 0
        local.append((plan, part))
    torch.cuda.synchronize()
    raw = lambda t: t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu().numpy()  # noqa: E731
    for s in range(R):
        n_send = int(counts[s].sum())
        for r in range(R):
            plan, part = local[r]
            f, c, r0 = plan["back_first"][s], plan["back_count"][s], plan["back_row0"][s]
            np.testing.assert_array_equal(raw(backs[s][r0:r0 + c]), raw(part[f:f + c]))
        assert np.all(raw(backs[s][n_send:]) == -5)        # rows past the sent ones untouched
        # the source's epilogue: the single-GPU result of its batch
        out = epx.combine_epilogue(backs[s], lays[s])
        wl = dict(name="p2p", T=src[s]["T"], H=H, E=E, R=R, k=k, x=src[s]["x_bits"],
                  topk_idx=src[s]["idx"], topk_weights=src[s]["w"])
        o = oracle.run_all(wl)
        assert_combine_close(torch_to_bits(out), o["out"])


def test_p2p_capacity_overflow_flagged_not_written():
    R, E, k, H = 2, 16, 4, 64
    src = _sources(R, E, k, H, [40, 40], seed=3)
    lays = [epx.layout(s["idx_t"], E, R) for s in src]
    counts = torch.stack([l.cnt_r.cpu() for l in lays])
    cap = 10
    canary = [torch.full((cap + 4, H), -7, dtype=torch.int16, device="cuda") for _ in range(R)]
    plan = ep_dist.p2p_plan(counts, 1)
    peers = [epx.PeerRows(canary[r][:cap].view(torch.bfloat16), cap, row0=plan["dispatch_row0"][r])
             for r in range(R)]
    epx.dispatch_p2p(src[1]["x"], src[1]["idx_t"], src[1]["w_t"], lays[1], peers)
    t = epx.read_totals(lays[1], raise_on_error=False)
    assert t["status"] == 3 and (t["dev_err"] & 2)
    for r in range(R):
        assert torch.all(canary[r][cap:] == -7)


def test_one_rank_p2p_transport_matches_nccl_transport():
    """ep_dist with transport 'p2p' and one rank (PeerBuffers are local
    allocations) gives bit for bit the 'nccl' transport's rows and output."""
    wl = wlmod.make("decode", seed=0)
    x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).cuda()
    idx = torch.from_numpy(wl["topk_idx"]).cuda()
    w = torch.from_numpy(wl["topk_weights"]).cuda()
    bufs = ep_dist.PeerBuffers(t_max=wl["T"], H=wl["H"], k=wl["k"])
    for _ in range(2):                       # the buffers are reused across steps
        hp = ep_dist.dispatch(x, idx, w, wl["E"], transport="p2p", buffers=bufs)
        hn = ep_dist.dispatch(x, idx, w, wl["E"], transport="nccl")
        n = epx.read_totals(hp.layout_in)["N_route"]
        assert n == epx.read_totals(hn.layout_in)["N_route"]
        assert torch.equal(hp.expanded[:n], hn.expanded[:n])
        yp = epx.standin_expert(hp.expanded, hp.layout_in)
        yn = epx.standin_expert(hn.expanded, hn.layout_in)
        op = ep_dist.combine(hp, yp)
        on = ep_dist.combine(hn, yn)
        assert torch.equal(op, on)
    bufs.close()
