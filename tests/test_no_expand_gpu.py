"""GPU parity of dispatch without expand: ep_dispatch (recv rows only), the
gather index ep_expand_index, and the stand-in expert reading recv through it
(ep_standin_expert_gather), against the CPU oracle.  Everything here is
bit-exact except the final combine (usual tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from combine_ep_layout_07_b200 import epx

from gpu_helpers import assert_combine_close, gpu_inputs, oracle_run, torch_to_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "decode", "prefill", "lowbatch1", "lowbatch8",
                                  "dp_padded", "dp_compact"])
def test_dispatch_without_expand(name):
    wl, o = oracle_run(name, 0)
    lay_o = o["layout"]
    x, idx, w = gpu_inputs(wl)
    lay = epx.layout(idx, wl["E"], wl["R"])
    recv = epx.dispatch(x, lay)
    nr, ne = lay_o["N_recv"], lay_o["N_route"]
    np.testing.assert_array_equal(torch_to_bits(recv[:nr]), o["recv"])
    src = epx.expand_index(lay)
    np.testing.assert_array_equal(src[:ne].cpu().numpy(), oracle.expand_index(lay_o))
    y = epx.standin_expert_gather(recv, lay, src)
    np.testing.assert_array_equal(torch_to_bits(y[:ne]), o["y"])
    out = epx.combine_reduce(y, w, lay)
    assert_combine_close(torch_to_bits(out), o["out"])
    assert epx.read_totals(lay)["status"] == 0


def test_gather_index_guards():
    wl, o = oracle_run("tiny", 2)
    x, idx, w = gpu_inputs(wl)
    lay = epx.layout(idx, wl["E"], wl["R"])
    ne = o["layout"]["N_route"]
    big = torch.full((lay.exp_cap + 8,), -9, dtype=torch.int32, device="cuda")
    epx.expand_index(lay, src=big[4:-4])
    assert torch.all(big[:4] == -9) and torch.all(big[4 + ne:] == -9)
    small = torch.zeros((5,), dtype=torch.int32, device="cuda")
    epx.expand_index(lay, src=small)
    t = epx.read_totals(lay, raise_on_error=False)
    assert t["status"] == 3 and (t["dev_err"] & 4)
