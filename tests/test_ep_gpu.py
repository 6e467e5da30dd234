"""Expert-parallel split on one GPU: the ranks' partial layers (each with its
own slot table, the other ranks' experts marked absent; the shared expert and
the residual on rank 0) run one after the other through moe_layer_forward,
and their rank-order sum equals the unsplit call within fp32 rounding and the
oracle within the usual bound. Decode (fused kernel) and prefill (grouped
GEMM path) both."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_router_b200 import ep as EP
from bit_expert_ffn_router_b200 import moe as M

from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,bits", [(4, 2), (40, 2), (300, 3)])
@pytest.mark.parametrize("world", [2, 3])
def test_partials_sum_to_the_unsplit_layer(T, bits, world):
    cfg = M.FULL.replace(bits=bits, residual=1, out_fp32=1)
    L = H.Layer(cfg, T, seed=800 + T + world, zipf=True)
    full, _ = L.forward()
    dv = L.device()
    ctx = H.ctx()
    parts = []
    for r in range(world):
        rc = EP.rank_cfg(cfg, r)
        table = EP.rank_slot_table(dv["slot_of"], r, world)
        ws = M.workspace(rc, T)
        part = torch.empty(T, cfg.d, dtype=torch.float32, device="cuda")
        ctx.layer_forward(rc, dv["x"], T, dv["wr"], dv["bias"], table, L.n_slots, dv["pool"], dv["stride"],
                          dv["shared"] if r == 0 else None, ws, part)
        torch.cuda.synchronize()
        # the routing views leave out exactly the pairs of experts this rank does not hold
        rt = ctx.layer_routing(rc, T, ws)
        idx = rt["idx"].cpu().numpy()
        pos = rt["pair_pos"].cpu().numpy().reshape(T, cfg.k)
        assert np.array_equal(pos < 0, ~EP.held(cfg.E, r, world)[idx])
        parts.append(part)
    assert ctx.check_device_status() == M.OK
    y = EP.combine_partials(parts)
    assert torch.allclose(y, full, rtol=2e-5, atol=1e-6 * float(full.abs().max()))
    H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"])
