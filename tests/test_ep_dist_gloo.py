"""Host logic of the multi-GPU expert-parallel path (ep_dist), on CPU with
world-size-2 gloo groups.  The kernels' part of each step is played by the
CPU oracle; what is under test is the plan and the exchanges: the counts
all-gather, the all-to-all send plan, the order of received rows and the
return trip of the partials.

The check is the one the pages' setting fixes: with the ranks' batches
concatenated in rank order, rank r must receive exactly the rows a single
GPU puts in rank r's block of `recv` (DeepEP issue #48: a token goes once to
every rank that owns one of its experts), with routing restricted to rank
r's experts, and the combine that comes back must equal the single-GPU
two-stage combine of the same tokens."""
import os
import socket
import sys
import traceback

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, K, H = 16, 4, 64
T_OF = [37, 50]          # ranks hold different batch sizes


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _batch(g):
    """Rank g's tokens (the same on every process): x bf16 bits, idx, w."""
    from combine_ep_layout_07_b200 import workloads as wlmod
    rng = np.random.default_rng(100 + g)
    T = T_OF[g]
    x = wlmod.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :K].astype(np.int64)
    idx[rng.random((T, K)) < 0.15] = -1
    if T > 3:
        idx[3, :] = -1          # a token that goes nowhere
    w = rng.random((T, K), dtype=np.float32)
    return x, idx, w


def _meta(idx, w, lay, R):
    """Expected routing of every sent row (recv_pos order): the token's
    routes on the destination rank, -1 / 0 elsewhere."""
    epr = E // R
    n = lay["N_recv"]
    mi = np.full((n, K), -1, np.int32)
    mw = np.zeros((n, K), np.float32)
    for t in range(lay["T"]):
        for r in range(R):
            row = lay["recv_pos"][t, r]
            if row < 0:
                continue
            for j in range(K):
                e = idx[t, j]
                if e >= 0 and e // epr == r:
                    mi[row, j] = e
                    mw[row, j] = w[t, j]
    return mi, mw


def _worker(rank, world, port, out_q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        import oracle
        from combine_ep_layout_07_b200 import ep_dist
        dist.init_process_group("gloo", rank=rank, world_size=world)
        pg = dist.group.WORLD
        R = world
        x, idx, w = _batch(rank)
        # ---- source side (oracle standing in for the kernels)
        lay = oracle.layout(idx, E, R)
        send, _ = oracle.dispatch_expand(x, lay)
        mi, mw = _meta(idx, w, lay, R)
        counts = ep_dist.exchange_counts(torch.from_numpy(lay["cnt_r"]), pg)
        plan = ep_dist.send_plan(counts, rank)
        assert plan["n_send"] == lay["N_recv"]
        recv_x = ep_dist.exchange_rows(torch.from_numpy(send.view(np.int16)), plan, pg)
        recv_i = ep_dist.exchange_rows(torch.from_numpy(mi), plan, pg)
        recv_w = ep_dist.exchange_rows(torch.from_numpy(mw), plan, pg)

        # ---- the single-GPU view of all ranks' tokens
        parts = [_batch(g) for g in range(world)]
        gx = np.concatenate([p[0] for p in parts])
        gidx = np.concatenate([p[1] for p in parts])
        gw = np.concatenate([p[2] for p in parts])
        glay = oracle.layout(gidx, E, R)
        grecv, _ = oracle.dispatch_expand(gx, glay)
        gmi, gmw = _meta(gidx, gw, glay, R)
        lo, hi = glay["off_r"][rank], glay["off_r"][rank + 1]
        assert list(counts[:, rank]) == [int(v) for v in plan["recv_splits"]]
        assert plan["n_recv"] == hi - lo
        np.testing.assert_array_equal(recv_x.numpy().view(np.uint16), grecv[lo:hi])
        np.testing.assert_array_equal(recv_i.numpy(), gmi[lo:hi])
        np.testing.assert_array_equal(recv_w.numpy(), gmw[lo:hi])

        # ---- receiving side: every received route is on this rank
        lay_in = oracle.layout(recv_i.numpy(), E, R)
        assert lay_in["cnt_r"][rank] == plan["n_recv"] and lay_in["N_recv"] == plan["n_recv"]
        np.testing.assert_array_equal(lay_in["recv_pos"][:, rank], np.arange(plan["n_recv"]))
        _, ex_in = oracle.dispatch_expand(recv_x.numpy().view(np.uint16), lay_in)
        y_in = oracle.standin(ex_in, lay_in)
        part = oracle.combine_local(y_in, recv_w.numpy(), lay_in, 32)
        back = ep_dist.exchange_rows(torch.from_numpy(np.ascontiguousarray(part)), plan, pg,
                                     reverse=True).numpy()
        out = oracle.combine_epilogue(back, lay)

        # ---- against the single-GPU two-stage combine of all tokens
        _, gex = oracle.dispatch_expand(gx, glay)
        gy = oracle.standin(gex, glay)
        gpart = oracle.combine_local(gy, gw, glay, 32)
        gout = oracle.combine_epilogue(gpart, glay)
        t0 = sum(T_OF[:rank])
        for t in range(lay["T"]):
            for r in range(R):
                row = lay["recv_pos"][t, r]
                if row >= 0:
                    np.testing.assert_array_equal(back[row],
                                                  gpart[glay["recv_pos"][t0 + t, r]])
        np.testing.assert_array_equal(out, gout[t0:t0 + lay["T"]])
        out_q.put((rank, "ok"))
    except Exception:
        out_q.put((rank, traceback.format_exc()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_send_plan_is_the_counts_matrix():
    from combine_ep_layout_07_b200 import ep_dist
    c = torch.tensor([[3, 0, 2], [1, 4, 0], [0, 5, 6]])
    p = ep_dist.send_plan(c, 1)
    assert p["send_splits"] == [1, 4, 0] and p["recv_splits"] == [0, 4, 5]
    assert p["recv_offsets"] == [0, 0, 4] and p["n_send"] == 5 and p["n_recv"] == 9
    with pytest.raises(ValueError):
        ep_dist.send_plan(torch.tensor([[1, -1], [0, 0]]), 0)
    with pytest.raises(ValueError):
        ep_dist.send_plan(c, 3)


def test_exchange_on_one_rank_is_the_identity():
    from combine_ep_layout_07_b200 import ep_dist
    plan = ep_dist.send_plan(torch.tensor([[5]]), 0)
    rows = torch.arange(20, dtype=torch.int32).view(5, 4)
    assert torch.equal(ep_dist.exchange_rows(rows, plan), rows)
    assert torch.equal(ep_dist.exchange_rows(rows, plan, reverse=True), rows)
    assert ep_dist.exchange_counts(torch.tensor([5])).tolist() == [[5]]


def test_two_ranks_match_the_single_gpu_layout_split_by_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    for r in range(world):
        assert res[r] == "ok", res[r]


def test_p2p_plan_places_rows_where_the_all_to_all_does():
    """The peer-memory transport's placements (ep_dist.p2p_plan) against
    the all-to-all plan (send_plan): source s's rows for rank r start, in
    r's buffer, where the all-to-all puts them (recv_offsets of r, entry s),
    and r's partials for s go back to the start of s's send block for r."""
    from combine_ep_layout_07_b200 import ep_dist
    rng = np.random.default_rng(7)
    for world in (1, 2, 3, 5):
        counts = torch.from_numpy(rng.integers(0, 9, size=(world, world)))
        counts[0, world - 1] = 0                     # an empty block
        plans = [ep_dist.p2p_plan(counts, g) for g in range(world)]
        sends = [ep_dist.send_plan(counts, g) for g in range(world)]
        for s in range(world):
            for r in range(world):
                assert plans[s]["dispatch_row0"][r] == sends[r]["recv_offsets"][s]
                assert plans[r]["back_first"][s] == sends[r]["recv_offsets"][s]
                assert plans[r]["back_count"][s] == int(counts[s, r])
                assert plans[r]["back_row0"][s] == sum(sends[s]["send_splits"][:r])
            assert plans[s]["n_recv"] == sends[s]["n_recv"]
            assert plans[s]["n_send"] == sends[s]["n_send"]
    with pytest.raises(ValueError):
        ep_dist.p2p_plan(torch.zeros(2, 3), 0)
    with pytest.raises(ValueError):
        ep_dist.p2p_plan(-torch.ones(2, 2), 0)


def _peer_buffers_worker(rank, world, port, out_q, H_of):
    """PeerBuffers' exchange on a gloo group, with the CUDA IPC calls of the
    binding replaced by fakes that record what they were given: every rank
    must map every other rank's handle, learn every rank's capacities, and
    refuse a group whose ranks disagree on the row width."""
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        from combine_ep_layout_07_b200 import ep_dist, epx
        calls = dict(malloc=[], open=[], close=[], free=[])

        def fake_malloc(nbytes):
            ptr = 0x1000 * (rank + 1) + len(calls["malloc"])
            calls["malloc"].append((nbytes, ptr))
            return ptr, bytes([rank, len(calls["malloc"]) - 1]) + bytes(62)

        epx.ipc_malloc = fake_malloc
        epx.ipc_open = lambda h: calls["open"].append(h) or 0x900000 + h[0] * 16 + h[1]
        epx.ipc_close = lambda p: calls["close"].append(p)
        epx.ipc_free = lambda p: calls["free"].append(p)
        epx.tensor_at = lambda ptr, shape, dtype, device: torch.zeros(shape, dtype=dtype)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        pg = dist.group.WORLD
        t_max = [5, 7][rank]
        H = H_of[rank]
        if len(set(H_of)) > 1:
            try:
                ep_dist.PeerBuffers(t_max, H, 4, pg, device=torch.device("cpu"))
                raise AssertionError("mismatched H accepted")
            except ValueError:
                pass
            assert len(calls["free"]) == 4 and not calls["open"]   # own buffers freed, none mapped
            out_q.put((rank, "ok"))
            return
        b = ep_dist.PeerBuffers(t_max, H, 4, pg, device=torch.device("cpu"))
        assert b.peer_recv_cap == [2 * 5, 2 * 7] and b.peer_back_cap == [5 * 2, 7 * 2]
        assert b.recv_cap == 2 * t_max and b.local["rows"].shape == (2 * t_max, H)
        other = 1 - rank
        for i, name in enumerate(("rows", "meta_idx", "meta_w", "back")):
            assert b.peer[name][rank] == calls["malloc"][i][1]             # own allocation
            assert b.peer[name][other] == 0x900000 + other * 16 + i        # the other's, mapped
        assert calls["malloc"][0][0] == 2 * t_max * H * 2                  # bf16 rows
        assert calls["malloc"][3][0] == t_max * 2 * H * 4                  # fp32 partials
        b.close()
        assert sorted(calls["close"]) == sorted(0x900000 + other * 16 + i for i in range(4))
        assert sorted(calls["free"]) == sorted(p for _, p in calls["malloc"])
        out_q.put((rank, "ok"))
    except Exception:
        out_q.put((rank, traceback.format_exc()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.parametrize("H_of", [(64, 64), (64, 128)], ids=["agree", "mismatch"])
def test_peer_buffers_exchange_on_two_ranks(H_of):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_buffers_worker, args=(r, world, port, q, H_of))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    for r in range(world):
        assert res[r] == "ok", res[r]


def test_p2p_placement_is_the_single_gpu_layout_split_by_rank():
    """The peer-memory dispatch's placement rule -- source s writes its row
    for (t, r) at p2p_plan(counts, s).dispatch_row0[r] + (recv_pos_s[t, r] -
    off_r_s[r]) of rank r's buffer, with the routing kept on r -- computed
    here with the oracle's layouts of each source's batch, must fill rank
    r's buffer exactly as the single-GPU layout of all batches concatenated
    in rank order fills rank r's block of recv (rows and routing), with no
    row written twice or left empty; and the partials' return rule must put
    every partial back at the source's own recv_pos row."""
    sys.path.insert(0, ROOT)
    import oracle
    from combine_ep_layout_07_b200 import ep_dist
    for world in (2, 4):                 # E = 16 experts split evenly
        parts = [_batch(g % 2) for g in range(world)]
        lays = [oracle.layout(p[1], E, world) for p in parts]
        counts = torch.tensor(np.stack([l["cnt_r"] for l in lays]))
        gidx = np.concatenate([p[1] for p in parts])
        gw = np.concatenate([p[2] for p in parts])
        gx = np.concatenate([p[0] for p in parts])
        glay = oracle.layout(gidx, E, world)
        grecv, _ = oracle.dispatch_expand(gx, glay)
        gmi, gmw = _meta(gidx, gw, glay, world)
        for r in range(world):
            n = int(counts[:, r].sum())
            rows = np.full((n, H), 0xFFFF, np.uint16)
            mi = np.full((n, K), -7, np.int32)
            mw = np.full((n, K), -7.0, np.float32)
            written = np.zeros(n, np.int64)
            for s, (x, idx, w) in enumerate(parts):
                plan = ep_dist.p2p_plan(counts, s)
                lay = lays[s]
                smi, smw = _meta(idx, w, lay, world)
                for t in range(lay["T"]):
                    q = lay["recv_pos"][t, r]
                    if q < 0:
                        continue
                    row = plan["dispatch_row0"][r] + (q - lay["off_r"][r])
                    rows[row], mi[row], mw[row] = x[t], smi[q], smw[q]
                    written[row] += 1
            assert np.all(written == 1)
            lo, hi = glay["off_r"][r], glay["off_r"][r + 1]
            np.testing.assert_array_equal(rows, grecv[lo:hi])
            np.testing.assert_array_equal(mi, gmi[lo:hi])
            np.testing.assert_array_equal(mw, gmw[lo:hi])
            # the return trip: received row d from source s goes to the
            # source's row back_row0[s] + (d - back_first[s]), which must be
            # that source's own recv_pos row for (t, r)
            plan_r = ep_dist.p2p_plan(counts, r)
            for s in range(world):
                lay = lays[s]
                mine = [t for t in range(lay["T"]) if lay["recv_pos"][t, r] >= 0]
                for i, t in enumerate(mine):
                    d = plan_r["back_first"][s] + i
                    assert plan_r["back_row0"][s] + (d - plan_r["back_first"][s]) == \
                        lay["recv_pos"][t, r]


def test_dispatch_arguments_are_checked_before_any_device_work():
    """Bad transport arguments fail on the host, before a layout is launched
    (the inputs here are CPU tensors a kernel could not take)."""
    from combine_ep_layout_07_b200 import ep_dist
    x = torch.zeros((4, 8), dtype=torch.bfloat16)
    idx = torch.zeros((4, 2), dtype=torch.int64)
    w = torch.zeros((4, 2), dtype=torch.float32)
    with pytest.raises(ValueError, match="unknown transport"):
        ep_dist.dispatch(x, idx, w, 4, transport="rdma")
    with pytest.raises(ValueError, match="needs PeerBuffers"):
        ep_dist.dispatch(x, idx, w, 4, transport="p2p")

    class Fake:
        world, rank, recv_cap, H = 2, 0, 8, 8
    with pytest.raises(ValueError, match="another process group"):
        ep_dist.dispatch(x, idx, w, 4, transport="p2p", buffers=Fake())
    Fake.world, Fake.recv_cap = 1, 2
    with pytest.raises(ValueError, match="larger than"):
        ep_dist.dispatch(x, idx, w, 4, transport="p2p", buffers=Fake())
