"""moe_layer_forward_static (scratch in a static device array, no workspace
argument) against moe_layer_forward on the same inputs, two calls in a row.

The file name sorts last so that the static scratch is also exercised after
every other test has used the library."""
from __future__ import annotations

import pytest
import torch

import harness as H
from bit_expert_ffn_router_b200 import moe as M

pytestmark = pytest.mark.gpu


def _static(L, cfg, y):
    dv = L.device()
    return H.ctx().layer_forward_static_status(cfg, dv["x"], L.T, dv["wr"], dv["bias"], dv["slot_of"], L.n_slots,
                                               dv["pool"], dv["stride"], dv["shared"], y)


@pytest.mark.parametrize("cfg,T,zipf", [(M.TINY, 4, False), (M.FULL, 1, True), (M.FULL, 4, True),
                                        (M.FULL.replace(bits=3), 8, True), (M.TINY, 40, False)])
def test_static_scratch_matches_workspace_path(cfg, T, zipf):
    L = H.Layer(cfg, T, seed=31, zipf=zipf)
    y_ref, _ = L.forward()
    outs = []
    for _ in range(2):  # two calls in a row reuse the same scratch
        y = L.out_tensor()
        assert _static(L, cfg, y) == M.OK
        outs.append(y)
    torch.cuda.synchronize()
    assert H.ctx().check_device_status() == M.OK
    for y in outs:  # the same kernels on the same inputs: the same bits
        assert torch.equal(y, y_ref)


def test_static_scratch_rejects_workspaces_beyond_its_size():
    T = 64  # the full-size layer needs ~11 MB of scratch here
    assert M.workspace_bytes(M.FULL, T) > 4 << 20
    L = H.Layer(M.FULL, T, seed=32)
    y = L.out_tensor()
    assert _static(L, M.FULL, y) == M.ENOSPACE
