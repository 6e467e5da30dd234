"""GPU parity of the routing and grouping that the whole-step call computes
itself, read back through moe_layer_routing, against the fp64 oracle.

On the decode path the fused decode kernel runs its own router, top-k and
grouping (separate code from moe_router_topk / moe_group_tokens), so these
tests compare what that kernel published: logits within 1e-5 of the fp64
oracle; the selected experts bit-exactly equal to the oracle's selection on
the kernel's own fp32 logits, and equal to the fp64 selection except at fp64
near-ties; the gates; and every grouping array bit-exactly. Tie cases set
W_r = 0 so that the logits are exactly the given bias rows: heavy ties, +-0,
+-inf and NaN, and rows where 32 or 33 values tie at the top. Inputs scaled
by 2^40 and 2^90 make the CTAs' partial logits large enough to use the upper
parts of the kernel's fixed-point accumulators."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_router_b200 import moe as M
from bit_expert_ffn_router_b200 import synth
from oracle import moe_oracle as O

from tests import harness as H

pytestmark = pytest.mark.gpu

_LAYERS = {}


def _layer(cfg, seed):
    key = (cfg, seed)
    if key not in _LAYERS:
        _LAYERS.clear()  # one full-size pool on the device at a time
        _LAYERS[key] = H.Layer(cfg, 8, seed=seed)
    return _LAYERS[key]


def _np(t):
    return t.cpu().numpy()


def check_published_routing(L, ws=None, check_fp64=True, ws_routing=None):
    """Compares the routing published in ws (or the routing views given as
    numpy arrays) with the oracle; returns the routing dict."""
    cfg, T = L.cfg, L.T
    r = ws_routing if ws_routing is not None else {k: _np(v) for k, v in H.ctx().layer_routing(cfg, T, ws).items()}
    logits = r["logits"].astype(np.float64)
    # the selection is exact on the kernel's own fp32 logits
    want = O.topk(logits, cfg.k)
    assert np.array_equal(r["idx"], want)
    fin = np.all(np.isfinite(np.take_along_axis(logits, want.astype(np.int64), 1)), axis=1)
    g_own = O.gates(logits, want, renorm=bool(cfg.renorm))
    assert np.allclose(r["gate"][fin], g_own[fin], rtol=1e-5, atol=1e-7)
    if check_fp64:
        l_ref, idx_ref, g_ref = O.route(L.x, L.wr, cfg.k, L.bias, renorm=bool(cfg.renorm))
        scale = np.abs(l_ref).max(axis=1, keepdims=True)
        assert np.all(np.abs(logits - l_ref) <= 1e-5 * scale)
        H.assert_routing_matches(r["idx"], idx_ref, l_ref)
    # grouping of the published selection, every array (of the kept pairs,
    # when low-ranked non-resident ones are left out)
    keep = O.kept_pairs(r["idx"].astype(np.int64), L.slot_of, cfg.skip_from, cfg.hot_slots)
    ref = O.group(r["idx"], r["gate"], cfg.E, L.slot_of, keep=keep)
    n = int(keep.sum())
    nu = int(r["n_uniq"][0])
    assert nu == ref["n_uniq"]
    assert np.array_equal(r["expert_count"], ref["expert_count"])
    assert np.array_equal(r["expert_offset"], ref["expert_offset"])
    assert np.array_equal(r["pair_token"][:n], ref["pair_token"])
    assert np.array_equal(r["pair_j"][:n], ref["pair_j"])
    assert np.array_equal(r["pair_gate"][:n], ref["pair_gate"].astype(np.float32), equal_nan=True)
    assert np.array_equal(r["pair_pos"], ref["pair_pos"].reshape(-1))
    flat = r["idx"].reshape(-1)
    kept_idx = np.nonzero(keep.reshape(-1))[0]
    order = kept_idx[np.argsort(flat[kept_idx], kind="stable")]
    assert np.array_equal(r["pair_slot"][:n], L.slot_of[flat[order]])
    assert np.array_equal(r["uniq_expert"][:nu], ref["uniq_expert"])
    assert np.array_equal(r["uniq_slot"][:nu], ref["uniq_slot"])
    assert np.array_equal(r["uniq_offset"][:nu + 1], np.append(ref["expert_offset"][ref["uniq_expert"]], n))
    return r


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("zipf", [True, False])
def test_fused_decode_routing_full_size(bits, zipf):
    """Full-size layer (512 experts, top-10 + shared), T = 1..8 on one pool:
    the published routing and grouping, and y against the oracle at every T."""
    base = _layer(M.FULL.replace(bits=bits), 80 + bits)
    for T in (1, 2, 3, 4, 5, 8):
        x = synth.activations(T, base.cfg.d, 1000 + T)
        bias = synth.bias_from_sets(synth.zipf_sets(T, base.cfg.E, base.cfg.k, 2000 + T), base.cfg.E) if zipf else None
        L = base.with_inputs(x, bias)
        y, ws = L.forward()
        torch.cuda.synchronize()
        assert H.ctx().check_device_status() == M.OK
        check_published_routing(L, ws)
        H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"])


def _tie_rows(E, seed):
    g = np.random.default_rng(seed)
    rows = np.zeros((8, E), dtype=np.float32)                      # 0: all equal
    rows[1] = g.integers(-2, 3, size=E)                            # 1: heavy ties, > 32 at the threshold
    rows[2] = g.standard_normal(E)                                 # 2: distinct, a few exact ties and +inf
    rows[2, 7] = rows[2, 300 % E] = rows[2, 11] = np.float32(9.0)
    rows[2, 5] = np.inf
    rows[3] = np.nan                                               # 3: six numbers among NaN
    rows[3, g.choice(E, 6, replace=False)] = g.standard_normal(6)
    rows[4] = -np.inf                                              # 4: three numbers among -inf
    rows[4, g.choice(E, 3, replace=False)] = [1.0, -1.0, 0.5]
    rows[5] = np.where(np.arange(E) % 2 == 0, 0.0, -0.0)           # 5: +0 / -0 ties under five positives
    rows[5, g.choice(E, 5, replace=False)] = [3.0, 1.0, 2.0, 2.0, 1.0]
    rows[6] = -1.0                                                 # 6: exactly 32 values at the top
    rows[6, g.choice(E, min(32, E), replace=False)] = 4.0
    rows[7] = -1.0                                                 # 7: 33 values at the top
    rows[7, g.choice(E, min(33, E), replace=False)] = 4.0
    return rows


@pytest.mark.parametrize("cfg", [M.FULL, M.FULL.replace(bits=3), M.TINY], ids=["full-q2", "full-q3", "tiny"])
def test_fused_decode_selection_on_ties_nan_and_zeros(cfg):
    """W_r = 0 makes the logits exactly the bias rows, so the fused selection is
    checked bit for bit on crafted rows, including its more-than-32-candidates
    branch."""
    base = _layer(cfg, 90)
    rows = _tie_rows(cfg.E, 91)
    x = synth.activations(8, cfg.d, 92)
    L = base.with_inputs(x, rows, wr=np.zeros((cfg.E, cfg.d), dtype=np.float32))
    y, ws = L.forward()
    torch.cuda.synchronize()
    assert H.ctx().check_device_status() == M.OK
    r = check_published_routing(L, ws, check_fp64=False)
    # the logits are the bias itself (x * 0 sums to +0; -0 + 0 = +0 compares equal)
    lg = r["logits"]
    assert np.array_equal(np.isnan(lg), np.isnan(rows))
    num = ~np.isnan(rows)
    assert np.array_equal(lg[num], rows[num])
    assert np.array_equal(r["idx"], O.topk(rows.astype(np.float64), cfg.k))


@pytest.mark.parametrize("shift", [40, 90])
def test_fused_decode_logits_of_large_inputs(shift):
    """x ~ N(0, 2^(2 shift)): each CTA's partial logits are ~2^(shift-4), above
    2^22 (shift 40) and above 2^76 (shift 90), so they are carried by the
    accumulators in units of 2^22 and 2^76. The logits stay within 1e-5 of the
    fp64 oracle's and the selection is exact."""
    base = _layer(M.FULL, 82)
    x = synth.activations(2, base.cfg.d, 1700 + shift, scale=2.0 ** shift)
    L = base.with_inputs(x, None)
    y, ws = L.forward()
    torch.cuda.synchronize()
    assert H.ctx().check_device_status() == M.OK
    r = check_published_routing(L, ws)
    assert np.abs(r["logits"]).max() > 2.0 ** (shift - 10)


def test_fused_decode_routing_256_experts_and_renorm0():
    cfg = M.FULL.replace(E=256, renorm=0)
    base = _layer(cfg, 95)
    x = synth.activations(3, cfg.d, 96)
    L = base.with_inputs(x, synth.bias_from_sets(synth.zipf_sets(3, cfg.E, cfg.k, 97), cfg.E))
    _, ws = L.forward()
    torch.cuda.synchronize()
    check_published_routing(L, ws)


@pytest.mark.parametrize("cfg,T", [(M.LayerCfg(d=256, f=128, E=600, k=4), 2), (M.TINY, 40), (M.FULL, 300)],
                         ids=["decode-E600", "prefill-tiny", "prefill-full"])
def test_routing_views_on_the_other_paths(cfg, T):
    """The separate router / top-k / grouping kernels (E > 512 decode, prefill)
    leave the same views in the workspace."""
    L = H.Layer(cfg, T, seed=98 + T, zipf=True)
    _, ws = L.forward()
    torch.cuda.synchronize()
    check_published_routing(L, ws)
