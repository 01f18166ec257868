"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the CPU oracle on the same seeded inputs."""
import functools

import numpy as np
import torch

import oracle
from combine_ep_layout_07_b200 import epx
from combine_ep_layout_07_b200 import workloads as wlmod

# combine tolerance: |gpu - oracle| <= 2^-7 |oracle| + 1e-3, elementwise
RTOL = 2.0 ** -7
ATOL = 1e-3


def bits_to_torch(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def torch_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@functools.lru_cache(maxsize=32)
def oracle_run(name: str, seed: int):
    wl = wlmod.make(name, seed=seed)
    return wl, oracle.run_all(wl)


def gpu_inputs(wl, idx_dtype=torch.int64):
    x = bits_to_torch(wl["x"])
    idx = torch.from_numpy(wl["topk_idx"]).to(idx_dtype).cuda()
    w = torch.from_numpy(wl["topk_weights"]).cuda()
    return x, idx, w


def run_gpu(wl, idx_dtype=torch.int64, dispatch_variant=0, combine_variant=0, y_override=None,
            layout_variant=0):
    x, idx, w = gpu_inputs(wl, idx_dtype)
    lay = epx.layout(idx, wl["E"], wl["R"], variant=layout_variant)
    recv, expanded = epx.dispatch_expand(x, lay, variant=dispatch_variant)
    y = epx.standin_expert(expanded, lay)
    y_in = y if y_override is None else y_override
    out = epx.combine_reduce(y_in, w, lay, variant=combine_variant)
    tot = epx.read_totals(lay)
    return dict(layout=lay, recv=recv, expanded=expanded, y=y, out=out, totals=tot)


def assert_layout_equal(g, o):
    lay = g["layout"] if isinstance(g, dict) else g
    np.testing.assert_array_equal(lay.cnt_e.cpu().numpy(), o["cnt_e"])
    np.testing.assert_array_equal(lay.off_e.cpu().numpy(), o["off_e"])
    np.testing.assert_array_equal(lay.cnt_r.cpu().numpy(), o["cnt_r"])
    np.testing.assert_array_equal(lay.off_r.cpu().numpy(), o["off_r"])
    np.testing.assert_array_equal(lay.pos.cpu().numpy(), o["pos"])
    np.testing.assert_array_equal(lay.recv_pos.cpu().numpy(), o["recv_pos"])
    t = lay.totals.cpu().numpy()
    assert (t[0], t[1], t[2]) == (o["N_route"], o["N_recv"], o["T_real"])
    assert (t[3] & 1) == (1 if o["n_bad"] else 0)


def assert_combine_close(out_gpu_bits: np.ndarray, out_oracle_bits: np.ndarray):
    g = wlmod.bf16_bits_to_f32(out_gpu_bits).astype(np.float64)
    o = wlmod.bf16_bits_to_f32(out_oracle_bits).astype(np.float64)
    err = np.abs(g - o)
    bound = RTOL * np.abs(o) + ATOL
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} elements out of tolerance; first at {tuple(i)}: "
                             f"gpu={g[tuple(i)]} oracle={o[tuple(i)]}")


def assert_all_equal(g, o):
    assert_layout_equal(g, o["layout"])
    nr, ne = o["layout"]["N_recv"], o["layout"]["N_route"]
    np.testing.assert_array_equal(torch_to_bits(g["recv"][:nr]), o["recv"])
    np.testing.assert_array_equal(torch_to_bits(g["expanded"][:ne]), o["expanded"])
    np.testing.assert_array_equal(torch_to_bits(g["y"][:ne]), o["y"])
    assert_combine_close(torch_to_bits(g["out"]), o["out"])
