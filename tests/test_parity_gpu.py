"""GPU parity: libmoe (through the C ABI) against the fp64 oracle on the same
seeded inputs. Routing and grouping are compared element by element and must
match bit for bit; FFN outputs must be within 2e-3 (per-token max-norm
relative error) of the fp64 oracle."""
import copy

import numpy as np
import pytest
import torch

from bit_expert_ffn_router_b200 import moe as M
from bit_expert_ffn_router_b200 import synth
from oracle import moe_oracle as O

from tests import harness as H

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ router + top-k

@pytest.mark.parametrize("cfg,T,zipf", [(M.TINY, 4, False), (M.TINY, 1, False), (M.FULL, 1, True),
                                        (M.FULL, 4, True), (M.FULL, 8, False), (M.FULL, 37, True),
                                        (M.FULL, 1000, False), (M.TINY, 300, False),
                                        (M.FULL.replace(E=1024, k=32), 200, False)])
def test_router_topk_matches_oracle(cfg, T, zipf):
    L = H.Layer(cfg.replace(n_shared=0), T, seed=T, zipf=zipf)
    dv = L.device()
    logits = torch.empty(T, cfg.E, device="cuda")
    idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, cfg.k, device="cuda")
    H.ctx().router_topk(cfg, dv["x"], dv["wr"], dv["bias"], T, logits, idx, gate)
    l_ref, idx_ref, g_ref = O.route(L.x, L.wr, cfg.k, L.bias)
    lg = logits.cpu().numpy().astype(np.float64)
    assert np.allclose(lg, l_ref, rtol=1e-5, atol=1e-5 * np.abs(l_ref).max())
    idx_g = idx.cpu().numpy()
    ties = H.assert_routing_matches(idx_g, idx_ref, l_ref)
    if zipf:
        assert ties == 0
    same = np.all(idx_g == idx_ref, axis=1)
    assert np.allclose(gate.cpu().numpy()[same], g_ref[same], rtol=1e-5, atol=1e-6)


def _fp32_logit_cases():
    g = np.random.default_rng(7)
    small = g.integers(-2, 3, size=(64, 16)).astype(np.float32)  # heavy ties
    small[0] = np.nan
    small[1, :4] = [np.nan, -0.0, 0.0, -np.inf]
    small[2] = -0.0
    big = g.integers(-4, 5, size=(300, 512)).astype(np.float32)
    big[:50] = g.standard_normal((50, 512)).astype(np.float32)
    return [(M.TINY, small), (M.FULL, big), (M.FULL.replace(E=1024, k=32), g.standard_normal((33, 1024)).astype(np.float32)),
            (M.FULL.replace(E=40, k=32), g.integers(0, 3, size=(9, 40)).astype(np.float32))]


@pytest.mark.parametrize("case", range(4))
def test_topk_bit_exact_on_given_fp32_logits(case):
    """Selection from the same fp32 logits is exact, ties and NaN included."""
    cfg, l = _fp32_logit_cases()[case]
    T = l.shape[0]
    idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, cfg.k, device="cuda")
    H.ctx().topk(cfg, torch.from_numpy(l).cuda(), T, idx, gate)
    want = O.topk(l.astype(np.float64), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), want)
    finite = np.all(np.isfinite(np.take_along_axis(l, want.astype(np.int64), 1)), axis=1)
    g_ref = O.gates(l.astype(np.float64), want)
    assert np.allclose(gate.cpu().numpy()[finite], g_ref[finite], rtol=1e-5, atol=1e-7)


def test_topk_full_softmax_gates():
    cfg = M.FULL.replace(renorm=0)
    l = np.random.default_rng(3).standard_normal((20, 512)).astype(np.float32) * 4
    idx = torch.empty(20, cfg.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(20, cfg.k, device="cuda")
    H.ctx().topk(cfg, torch.from_numpy(l).cuda(), 20, idx, gate)
    want = O.topk(l.astype(np.float64), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), want)
    assert np.allclose(gate.cpu().numpy(), O.gates(l.astype(np.float64), want, renorm=False), rtol=1e-5, atol=1e-8)


# ------------------------------------------------------------------ grouping

@pytest.mark.parametrize("T,E,k", [(1, 512, 10), (4, 512, 10), (4, 16, 2), (51, 512, 10), (52, 512, 10),
                                   (1000, 64, 7), (8192, 512, 10), (333, 1024, 32)])
def test_grouping_bit_exact(T, E, k):
    cfg = M.FULL.replace(E=E, k=k)
    g = np.random.default_rng(T * 31 + E)
    if T == 8192:
        idx = synth.zipf_sets(T, E, k, seed=0)  # Zipf-skewed load, as in the prefill chunk
    else:
        idx = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    gate = g.random((T, k)).astype(np.float32)
    n_slots = E + 5
    slot_of = g.permutation(n_slots)[:E].astype(np.int32)
    ws = M.workspace(cfg, T)
    grp = H.ctx().group_tokens(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(gate).cuda(), T,
                               torch.from_numpy(slot_of).cuda(), n_slots, ws)
    torch.cuda.synchronize()
    ref = O.group(idx, gate, E, slot_of)

    def dev(ptr, n, dtype=torch.int32):
        return ws.view(torch.uint8)[ptr - ws.data_ptr():][: n * 4].view(dtype).cpu().numpy()

    n_pairs = T * k
    assert grp.n_pairs == n_pairs
    assert np.array_equal(dev(grp.expert_count, E), ref["expert_count"])
    assert np.array_equal(dev(grp.expert_offset, E + 1), ref["expert_offset"])
    assert np.array_equal(dev(grp.pair_token, n_pairs), ref["pair_token"])
    assert np.array_equal(dev(grp.pair_j, n_pairs), ref["pair_j"])
    assert np.array_equal(dev(grp.pair_gate, n_pairs, torch.float32), ref["pair_gate"].astype(np.float32))
    assert np.array_equal(dev(grp.pair_pos, n_pairs), ref["pair_pos"].reshape(-1))
    assert np.array_equal(dev(grp.pair_slot, n_pairs), slot_of[idx.reshape(-1)][np.argsort(idx.reshape(-1), kind="stable")])
    nu = int(dev(grp.n_uniq, 1)[0])
    assert nu == ref["n_uniq"]
    assert np.array_equal(dev(grp.uniq_expert, nu), ref["uniq_expert"])
    assert np.array_equal(dev(grp.uniq_slot, nu), ref["uniq_slot"])
    assert np.array_equal(dev(grp.uniq_offset, nu + 1),
                          np.append(ref["expert_offset"][ref["uniq_expert"]], n_pairs))
    assert H.ctx().check_device_status() == M.OK


def test_grouping_reports_bad_indices():
    cfg = M.TINY
    T = 3
    idx = np.array([[0, 1], [2, 99], [3, 4]], dtype=np.int32)
    gate = np.ones((T, 2), dtype=np.float32)
    ws = M.workspace(cfg, T)
    H.ctx().group_tokens(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(gate).cuda(), T,
                         torch.arange(16, dtype=torch.int32, device="cuda"), 16, ws)
    assert H.ctx().check_device_status() == M.EDEVICE
    assert H.ctx().check_device_status() == M.OK  # cleared
    idx[1, 1] = 5
    slot_of = torch.arange(16, dtype=torch.int32, device="cuda")
    slot_of[5] = 16  # out of the pool
    H.ctx().group_tokens(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(gate).cuda(), T, slot_of, 16, ws)
    assert H.ctx().check_device_status() == M.EDEVICE


def test_multi_cta_grouping_reports_bad_index_and_keeps_a_permutation():
    """T*k > 512 takes the multi-CTA grouping; an expert index = E is reported
    as MOE_EDEVICE, filed under expert 0 by both of its passes, and the sorted
    positions still form a permutation of [0, T*k)."""
    cfg = M.FULL
    T = 60
    g = np.random.default_rng(17)
    idx = np.stack([g.choice(cfg.E, size=cfg.k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[7, 3] = cfg.E
    idx[40, 0] = -1
    gate = g.random((T, cfg.k)).astype(np.float32)
    ws = M.workspace(cfg, T)
    ws.fill_(0xAB)  # stale contents must not survive anywhere in the result
    grp = H.ctx().group_tokens(cfg, torch.from_numpy(idx).cuda(), torch.from_numpy(gate).cuda(), T,
                               torch.arange(cfg.E, dtype=torch.int32, device="cuda"), cfg.E, ws)
    assert H.ctx().check_device_status() == M.EDEVICE
    n = T * cfg.k
    raw = ws.view(torch.uint8)

    def dev(ptr, count):
        return raw[ptr - ws.data_ptr():][: count * 4].view(torch.int32).cpu().numpy()

    pos = dev(grp.pair_pos, n)
    assert np.array_equal(np.sort(pos), np.arange(n))
    mapped = np.where((idx < 0) | (idx >= cfg.E), 0, idx)
    ref = O.group(mapped, gate, cfg.E)
    assert np.array_equal(pos, ref["pair_pos"].reshape(-1))
    assert np.array_equal(dev(grp.pair_token, n), ref["pair_token"])
    assert np.array_equal(dev(grp.expert_count, cfg.E), ref["expert_count"])
    assert H.ctx().check_device_status() == M.OK


# ------------------------------------------------------------------ whole layer, decode path

@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_layer_decode_tiny(bits, T):
    L = H.Layer(M.TINY.replace(bits=bits), T, seed=10 + T)
    y, _ = L.forward()
    ref = L.oracle()
    worst = H.assert_close_rows(H.y_as_f64(y), ref["y"])
    assert worst < 1e-4, worst  # fp32 arithmetic on exact weights: far inside the bar


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 4])
def test_layer_decode_full(bits, T):
    L = H.Layer(M.FULL.replace(bits=bits), T, seed=20 + T, zipf=True)
    y, _ = L.forward()
    ref = L.oracle()
    H.assert_close_rows(H.y_as_f64(y), ref["y"])


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 4])
def test_layer_decode_256_experts(bits, T):
    # the pages' pruned variant keeps 256 of each layer's 512 experts
    # (news.blueqat.app/post/3262, section 量子化の種類とサイズ); top-10 of
    # 256 + shared
    L = H.Layer(M.FULL.replace(bits=bits, E=256), T, seed=60 + T, zipf=True)
    y, _ = L.forward()
    ref = L.oracle()
    H.assert_close_rows(H.y_as_f64(y), ref["y"])


@pytest.mark.parametrize("bits", [2, 3])
def test_decode_expert_ffn_on_given_grouping(bits):
    """The unfused decode entry points: moe_group_tokens on the oracle's routing,
    then moe_expert_ffn_q{bits} with no pair buffer (the fused down + combine
    writes y), against the oracle's layer output."""
    T, cfg = 3, M.FULL.replace(bits=bits)
    L = H.Layer(cfg, T, seed=71, zipf=True)
    dv = L.device()
    ref = L.oracle()
    ctx = H.ctx()
    ws = M.workspace(cfg, T)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    gate = torch.from_numpy(ref["gate"].astype(np.float32)).cuda()
    g = ctx.group_tokens(cfg, idx, gate, T, dv["slot_of"], L.n_slots, ws)
    y = L.out_tensor()
    ctx.expert_ffn(cfg, dv["x"], g, dv["pool"], dv["stride"], dv["shared"], ws, z_rows=None, y=y)
    torch.cuda.synchronize()
    assert ctx.check_device_status() == M.OK
    H.assert_close_rows(H.y_as_f64(y), ref["y"])


def test_layer_decode_more_than_512_experts():
    # E > 512 routes with the separate router / top-k / grouping kernels and
    # runs the decode expert kernel on the published grouping
    cfg = M.LayerCfg(d=256, f=128, E=600, k=4)
    L = H.Layer(cfg, 2, seed=72, zipf=True)
    y, _ = L.forward()
    H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"])


def test_layer_decode_full_unbiased_router_T8():
    L = H.Layer(M.FULL, 8, seed=5)
    y, ws = L.forward()
    ref = L.oracle()
    H.assert_close_rows(H.y_as_f64(y), ref["y"])


def test_layer_bf16_output_and_residual():
    cfg = M.FULL.replace(out_fp32=0, residual=1)
    L = H.Layer(cfg, 2, seed=41, zipf=True)
    y, _ = L.forward()
    ref = L.oracle()
    H.assert_close_rows(H.y_as_f64(y), ref["y"], bf16=True)


def test_layer_no_shared_and_renorm0():
    cfg = M.TINY.replace(n_shared=0, renorm=0)
    L = H.Layer(cfg, 3, seed=42)
    y, _ = L.forward()
    H.assert_close_rows(H.y_as_f64(y), L.oracle()["y"])


def test_decode_batch_invariance_and_determinism():
    """A T=4 verify batch gives each token the bits it gets alone (speculation is lossless)."""
    L4 = H.Layer(M.FULL, 4, seed=50, zipf=True)
    y4, ws = L4.forward()
    y4b, _ = L4.forward(ws=ws)
    assert torch.equal(y4, y4b)  # same call twice: same bits
    for t in range(4):
        L1 = copy.copy(L4)
        L1.T, L1.x, L1.bias = 1, L4.x[t:t + 1], L4.bias[t:t + 1]
        L1._dev = None
        y1, _ = L1.forward()
        assert torch.equal(y1[0], y4[t]), t


def test_decode_token_and_slot_permutation_invariance():
    L = H.Layer(M.FULL, 4, seed=60, zipf=True)
    y, _ = L.forward()
    perm = np.array([2, 0, 3, 1])
    P = copy.copy(L)
    P.x, P.bias = L.x[perm], L.bias[perm]
    P.slot_of = synth.rng(61).permutation(P.n_slots)[:P.cfg.E].astype(np.int32)
    P._dev = None
    yp, _ = P.forward()
    assert torch.equal(yp, y[torch.from_numpy(perm).cuda()])


def test_empty_batch_is_a_noop():
    L = H.Layer(M.TINY, 1, seed=1)
    dv = L.device()
    ws = M.workspace(M.TINY, 0)
    y = torch.full((1, 256), 7.0, device="cuda")
    st = H.ctx().layer_forward_status(M.TINY, dv["x"], 0, dv["wr"], None, dv["slot_of"], L.n_slots, dv["pool"],
                                      dv["stride"], dv["shared"], ws, y)
    assert st == M.OK
    assert torch.all(y == 7.0)


def test_host_argument_errors():
    L = H.Layer(M.TINY, 2, seed=2)
    dv = L.device()
    ws = M.workspace(M.TINY, 2)
    y = L.out_tensor()
    c = H.ctx()
    args = dict(cfg=M.TINY, x=dv["x"], T=2, w_router=dv["wr"], bias=None, slot_of=dv["slot_of"], n_slots=L.n_slots,
                pool=dv["pool"], stride=dv["stride"], shared=dv["shared"], ws=ws, y=y)
    assert c.layer_forward_status(**args) == M.OK
    assert c.layer_forward_status(**{**args, "cfg": M.TINY.replace(bits=5)}) == M.EUNSUPPORTED
    assert c.layer_forward_status(**{**args, "x": None}) == M.EINVAL
    assert c.layer_forward_status(**{**args, "stride": dv["stride"] - 256}) == M.EINVAL
    assert c.layer_forward_status(**{**args, "ws": ws[: ws.numel() // 2]}) == M.ENOSPACE
    assert c.layer_forward_status(**{**args, "x": dv["x"].view(torch.uint8)[2:]}) == M.EINVAL  # misaligned
    assert c.layer_forward_status(**{**args, "shared": None}) == M.EINVAL
    assert c.check_device_status() == M.OK


def test_device_wait_timeout_is_reported_and_context_recovers(monkeypatch):
    """A 1 us wait limit makes the decode kernel's waits run out: the call
    reports MOE_ETIMEOUT through the status word, and the context (after
    moe_check_device_status clears it) computes correct results again."""
    L = H.Layer(M.FULL, 1, seed=70, zipf=True)
    dv = L.device()
    monkeypatch.setenv("MOE_TIMEOUT_US", "1")
    short = M.Context(torch.cuda.current_device())
    monkeypatch.delenv("MOE_TIMEOUT_US")
    ws = M.workspace(M.FULL, 1)
    y = L.out_tensor()
    st = short.layer_forward_status(M.FULL, dv["x"], 1, dv["wr"], dv["bias"], dv["slot_of"], L.n_slots, dv["pool"],
                                    dv["stride"], dv["shared"], ws, y)
    assert st == M.OK  # the launch itself is fine
    assert short.check_device_status() == M.ETIMEOUT
    assert short.check_device_status() == M.OK
    short.close()
    y2, _ = L.forward()
    H.assert_close_rows(H.y_as_f64(y2), L.oracle()["y"])
