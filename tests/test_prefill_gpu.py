"""GPU parity of the prefill path (T > 8): x gather, the tcgen05 grouped GEMMs
(gate/up + SwiGLU, down + gate) and the combine, against the fp64 oracle.

Sizes span several token tiles (128 pairs) and weight tiles (128 rows) with
ragged tails; the full layer at T = 8,192 (the prefill chunk of the pages) is
checked on sampled tokens.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import harness as H
from bit_expert_ffn_router_b200 import moe as M
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def forced_bias(T: int, E: int, sets) -> np.ndarray:
    """Logit bias that makes token t pick the experts in sets[t] (router still runs)."""
    b = np.zeros((T, E), dtype=np.float32)
    for t, s in enumerate(sets):
        b[t, list(s)] = 20.0
    return b


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [9, 37, 300])
def test_layer_prefill_tiny(bits, T):
    L = H.Layer(M.TINY.replace(bits=bits), T, seed=11 + T)
    y, _ = L.forward()
    ref = L.oracle()
    H.assert_close_rows(H.y_as_f64(y), ref["y"])


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("count", [127, 128, 129, 255, 256, 257])
def test_prefill_tile_boundaries(bits, count):
    # every token picks experts {3, 5}: two experts with `count` pairs each,
    # the shared expert with `count` rows, all other experts empty
    T = count
    cfg = M.TINY.replace(bits=bits)
    L = H.Layer(cfg, T, seed=3, bias=forced_bias(T, cfg.E, [(3, 5)] * T))
    y, _ = L.forward()
    H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"])


def test_prefill_one_expert_takes_everything_but_one():
    # one hot expert with 2T-1 pairs is impossible at k=2 (distinct experts);
    # instead expert 0 is in every token's set and the partner varies
    T, cfg = 400, M.TINY
    sets = [(0, 1 + (t % 15)) for t in range(T)]
    L = H.Layer(cfg, T, seed=4, bias=forced_bias(T, cfg.E, sets))
    y, _ = L.forward()
    H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"])


@pytest.mark.parametrize("bits", [2, 3])
def test_layer_prefill_full_zipf(bits):
    L = H.Layer(M.FULL.replace(bits=bits), 300, seed=6, zipf=True)
    y, _ = L.forward()
    toks = list(range(0, 300, 10))
    ref = L.oracle(tokens=toks)
    H.assert_close_rows(H.y_as_f64(y)[toks], ref["y"])


def test_layer_prefill_256_experts():
    # the pages' pruned variant: 256 experts per layer (news.blueqat.app/post/3262,
    # section 量子化の種類とサイズ), top-10 + shared
    L = H.Layer(M.FULL.replace(E=256), 300, seed=61, zipf=True)
    y, _ = L.forward()
    toks = list(range(3, 300, 13))
    ref = L.oracle(tokens=toks)
    H.assert_close_rows(H.y_as_f64(y)[toks], ref["y"])


@pytest.mark.parametrize("bits", [2, 3])
def test_layer_prefill_chunk_8192_sampled(bits):
    # the pages' prefill chunk: 8,192 tokens x top-10 of 512 + shared expert
    T = 8192
    L = H.Layer(M.FULL.replace(bits=bits), T, seed=5, zipf=True)
    y, _ = L.forward()
    toks = sorted(np.random.default_rng(bits).choice(T, 12, replace=False).tolist())
    ref = L.oracle(tokens=toks)
    H.assert_close_rows(H.y_as_f64(y)[toks], ref["y"])
    assert H.ctx().check_device_status() == M.OK


def test_prefill_bf16_residual_no_shared_renorm0():
    for cfg in (M.TINY.replace(out_fp32=0, residual=1), M.TINY.replace(n_shared=0, renorm=0)):
        L = H.Layer(cfg, 77, seed=8)
        y, _ = L.forward()
        H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"], bf16=not cfg.out_fp32)


def test_prefill_deterministic_and_token_permutation():
    T, cfg = 200, M.TINY
    L = H.Layer(cfg, T, seed=9)
    y1, ws = L.forward()
    y2, _ = L.forward(ws=ws)
    assert torch.equal(y1, y2), "prefill is not run-to-run deterministic"
    perm = np.random.default_rng(1).permutation(T)
    Lp = H.Layer(cfg, T, seed=9)
    Lp.x = L.x[perm].copy()
    yp, _ = Lp.forward()
    # the same token lands in another column of the same expert's tile
    H.assert_close_rows(H.y_as_f64(yp), H.y_as_f64(y1)[perm], tol=1e-5)


@pytest.mark.parametrize("bits", [2, 3])
def test_expert_ffn_z_rows_and_combine(bits):
    """The unfused entry points: grouping -> moe_expert_ffn_q{bits} (z_rows, gated,
    pair order) -> moe_combine, each output compared with the oracle."""
    T, cfg = 45, M.TINY.replace(bits=bits)
    L = H.Layer(cfg, T, seed=12)
    dv = L.device()
    ref = L.oracle()
    ctx = H.ctx()
    ws = M.workspace(cfg, T)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    gate = torch.from_numpy(ref["gate"].astype(np.float32)).cuda()
    g = ctx.group_tokens(cfg, idx, gate, T, dv["slot_of"], L.n_slots, ws)
    n_rows = g.n_rows
    z = torch.full((n_rows, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    ctx.expert_ffn(cfg, dv["x"], g, dv["pool"], dv["stride"], dv["shared"], ws, z_rows=z)
    y = torch.empty(T, cfg.d, dtype=torch.float32, device="cuda")
    ctx.combine(cfg, g, z, dv["x"], T, y)
    torch.cuda.synchronize()
    assert ctx.check_device_status() == M.OK

    grp = O.group(ref["idx"], ref["gate"].astype(np.float32).astype(np.float64), cfg.E)
    xd = O.bf16_to_f64(L.x)
    zg = z.cpu().numpy().astype(np.float64)
    for p in range(T * cfg.k):
        t, e = int(grp["pair_token"][p]), int(ref["idx"][grp["pair_token"][p], grp["pair_j"][p]])
        wg, wu, wd = O.expert_weights(L.sections[e], cfg.d, cfg.f, bits)
        zr = float(np.float32(ref["gate"][t, grp["pair_j"][p]])) * O.expert_forward(xd[t], wg, wu, wd)
        H.assert_close_rows(zg[p:p + 1], zr[None])
    sh = O.expert_weights(L.shared, cfg.d, cfg.f, bits)
    for t in range(T):
        H.assert_close_rows(zg[T * cfg.k + t:T * cfg.k + t + 1], O.expert_forward(xd[t], *sh)[None])
    H.assert_close_rows(H.y_as_f64(y), ref["y"])


def test_prefill_unsupported_geometry_is_refused():
    # f = 192 is a valid decode shape but not a multiple of the 128-code chunk
    cfg = M.LayerCfg(d=256, f=192, E=16, k=2)
    L = H.Layer(cfg, 20, seed=1)
    dv = L.device()
    ws = M.workspace(cfg, 20)
    y = L.out_tensor()
    st = H.ctx().layer_forward_status(cfg, dv["x"], 20, dv["wr"], None, dv["slot_of"], L.n_slots, dv["pool"],
                                      dv["stride"], dv["shared"], ws, y)
    assert st == M.EUNSUPPORTED
