"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
exports every function include/moe.h declares, and its host-only calls
(record layout, workspace size, argument checks, status strings) behave."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_expert_ffn_router_b200 import build as B
from bit_expert_ffn_router_b200 import moe as M
from oracle import moe_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "moe.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", txt)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 13
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(M._SIGS), "binding and header disagree"


def test_status_strings():
    for s in range(7):
        assert M.status_string(s)
    assert M.status_string(99) == "unknown status"


@pytest.mark.parametrize("d,f,bits", [(2048, 768, 2), (2048, 768, 3), (256, 128, 2), (256, 128, 3), (4096, 1536, 3)])
def test_layout_matches_oracle(d, f, bits):
    lib = M.expert_layout(M.LayerCfg(d=d, f=f, E=16, k=2, bits=bits))
    ora = O.expert_layout(d, f, bits)
    for name in ("gu_codes", "dn_codes", "gu_scales", "dn_scales"):
        assert lib[name] == ora[name][0]
    assert lib["bytes"] == ora["bytes"]


def test_workspace_and_argument_checks():
    assert M.workspace_bytes(M.FULL, 1) > 0
    assert M.workspace_bytes(M.FULL, 8192) > M.workspace_bytes(M.FULL, 4)
    assert M.workspace_bytes(M.FULL, 0) > 0
    bad = [M.FULL.replace(bits=4), M.FULL.replace(block=16), M.FULL.replace(k=33), M.TINY.replace(k=17),
           M.FULL.replace(E=2048), M.FULL.replace(d=2000), M.FULL.replace(f=100), M.FULL.replace(n_shared=2),
           M.FULL.replace(k=0)]
    for cfg in bad:
        assert M.workspace_bytes(cfg, 4) == 0, cfg
    with pytest.raises(M.MoeError) as e:
        M.expert_layout(M.FULL.replace(bits=4))
    assert e.value.status == M.EUNSUPPORTED
    with pytest.raises(M.MoeError) as e:
        M.expert_layout(M.FULL.replace(k=600))
    assert e.value.status == M.EINVAL


def test_null_context_rejected_without_gpu():
    lib = M.load_library()
    cfg = M.TINY.c()
    assert lib.moe_router_topk(None, ctypes.byref(cfg), None, None, None, 1, None, None, None, None) == M.EINVAL
    assert lib.moe_check_device_status(None, None) == M.EINVAL
    assert lib.moe_ctx_create(0, None) == M.EINVAL


def test_prepared_layer_forward_passes_the_same_arguments():
    """PreparedLayer marshals each argument once; its calls must hand the C entry
    point exactly what Context.layer_forward_status hands it."""
    import torch

    calls = []

    class FakeLib:
        def moe_layer_forward(self, *args):
            calls.append(args)
            return 0

    class FakeCtx:
        lib = FakeLib()
        h = ctypes.c_void_p(1234)

    class FakeStream:
        cuda_stream = 4321

    def norm(a):
        if isinstance(a, ctypes.c_void_p):
            return ("p", a.value)
        if type(a).__name__ == "CArgObject":  # ctypes.byref(struct)
            return ("ref", bytes(a._obj))
        return ("v", a)

    cfg = M.FULL.replace(bits=3, out_fp32=0, residual=1)
    t = lambda n: torch.zeros(n, dtype=torch.uint8)  # noqa: E731  (CPU tensors: only data_ptr is read)
    w, bias, slots, pool, shared, ws = t(64), t(16), t(32), t(256), t(128), t(4096)
    x, y = t(8), t(8)
    args = (cfg, 3, w, bias, slots, 40, pool, 1536, shared, ws)
    prep = M.PreparedLayer(FakeCtx(), *args, stream=FakeStream())
    assert prep.status(x, y) == 0
    M.Context.layer_forward_status(FakeCtx(), cfg, x, 3, w, bias, slots, 40, pool, 1536, shared, ws, y,
                                   stream=FakeStream())
    assert len(calls) == 2
    a, b = [tuple(norm(v) for v in c) for c in calls]
    assert a == b
    # the pointers are the tensors' own addresses, the sizes the workspace's bytes
    assert ("p", x.data_ptr()) in a and ("p", y.data_ptr()) in a and ("v", 4096) in a
