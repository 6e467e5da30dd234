"""Pins of the fp64 oracle to facts fixed outside itself.

Each test checks the oracle against something it does not compute with:
hand-worked format examples, the size figures the pages print, library
routines in special cases (scipy's expit/softmax, torch's silu/linear),
closed forms built from permutation matrices, brute-force enumeration on tiny
inputs, and invariants. A plausible slip in the oracle (a swapped bit plane,
gate/up rows swapped, a transposed matrix, a missing shared expert, a wrong
tie-break, an unstable grouping) fails at least one of them.
"""
import itertools
import os

import numpy as np
import pytest
import scipy.special

from oracle import moe_oracle as O
from bit_expert_ffn_router_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1) if ":" in line else line.split(None, 1)
            out[key.strip()] = val.split()
    return out


# ------------------------------------------------------------------ format

def test_golden_q2_bytes_and_weights():
    g = _golden("format_q2.txt")
    codes = np.array([int(c) for c in g["codes"]])[None, :]
    want = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)[None, :]
    assert np.array_equal(O.pack_codes(codes, 2), want)
    assert np.array_equal(O.unpack_codes(want, 32, 2), codes)
    scales = np.array([[float(g["scale"][0])]], dtype=np.float16)
    w = O.dequant(want, scales, 32, 2)
    assert np.array_equal(w[0], np.array([float(v) for v in g["weights"]]))


def test_golden_q3_bytes_and_weights():
    g = _golden("format_q3.txt")
    codes = np.array([int(c) for c in g["codes"]])[None, :]
    want = np.array([int(b, 16) for b in g["bytes"]], dtype=np.uint8)[None, :]
    assert np.array_equal(O.pack_codes(codes, 3), want)
    assert np.array_equal(O.unpack_codes(want, 64, 3), codes)
    scales = np.array([[float(s) for s in g["scale"]]], dtype=np.float16)
    w = O.dequant(want, scales, 64, 3)
    assert np.array_equal(w[0, :32], np.array([float(v) for v in g["weights_block0"]]))
    assert np.all(w[0, 32:] == float(g["weights_block1"][0]))


@pytest.mark.parametrize("bits", [2, 3])
def test_dequant_value_set_and_round_trip(bits):
    g = np.random.default_rng(1)
    K = 128
    packed = g.integers(0, 256, size=(5, O.row_bytes(K, bits)), dtype=np.uint8)
    scales = synth.random_scales((5, K // 32), g)
    w = O.dequant(packed, scales, K, bits)
    s = np.repeat(scales.astype(np.float64), 32, axis=1)
    ratio = w / s
    allowed = np.arange(-(1 << (bits - 1)), 1 << (bits - 1))
    assert np.all(np.isin(ratio, allowed))
    # every code value appears (uniform random bytes hit all of them)
    assert set(np.unique(ratio).astype(int)) == set(allowed)
    # quantise(dequant(codes)) gives the codes back, bit for bit
    assert np.array_equal(O.quantize(w, scales, bits), packed)


@pytest.mark.parametrize("bits", [2, 3])
def test_quantize_clamps_and_rounds_half_even(bits):
    off = 1 << (bits - 1)
    scales = np.full((1, 1), 1.0, dtype=np.float16)
    w = np.zeros((1, 32))
    w[0, :6] = [100.0, -100.0, 0.5, 1.5, -0.5, -1.5]
    q = O.unpack_codes(O.quantize(w, scales, bits), 32, bits)[0]
    assert q[0] == (1 << bits) - 1 and q[1] == 0
    # ties go to the even integer: 0.5 -> 0, -0.5 -> 0, -1.5 -> -2, 1.5 -> 2 (clamped to 1 at 2 bits)
    assert q[2] == off and q[4] == off and q[5] == off - 2
    assert q[3] == min(off + 2, (1 << bits) - 1)


def test_record_layout_closed_form_sizes():
    # three 768x2048 matrices at 2 bits + one fp16 scale per 32 weights = 2.5 bits per weight
    lay2 = O.expert_layout(2048, 768, 2)
    lay3 = O.expert_layout(2048, 768, 3)
    n = 3 * 768 * 2048
    assert lay2["bytes"] == n * 2.5 / 8 == 1_474_560
    assert lay3["bytes"] == n * 3.5 / 8 == 2_064_384
    for lay in (lay2, lay3):
        offs = [lay[k][0] for k in ("gu_codes", "dn_codes", "gu_scales", "dn_scales")]
        assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    # tiny layer: d=256, f=128
    assert O.expert_layout(256, 128, 2)["bytes"] == 3 * 256 * 128 * 2.5 / 8


def test_record_round_trip():
    sec = synth.expert_sections(256, 128, 3, seed=5)
    rec = O.record_from_sections(sec, 256, 128, 3)
    back = O.sections_from_record(rec, 256, 128, 3)
    for k in sec:
        assert np.array_equal(np.asarray(sec[k]).view(np.uint8), np.asarray(back[k]).view(np.uint8))


def test_expert_shape_against_page_sizes():
    """d=2048, f=768 reproduce the pages' size figures within a few percent."""
    p = {k: float(v[0]) for k, v in _golden("page_sizes.txt").items()}
    n = 3 * 768 * 2048  # weights per expert
    assert p["layers"] * p["experts_per_layer"] == p["total_experts"]
    per_expert_q2_0 = n * p["q2_0_bpw"] / 8  # bytes
    assert abs(per_expert_q2_0 * p["total_experts"] / 1e9 - p["q2_0_expert_gb"]) / p["q2_0_expert_gb"] < 0.03
    assert abs(per_expert_q2_0 * p["experts_per_layer"] / 1e9 - p["layer_expert_gb"]) / p["layer_expert_gb"] < 0.05
    assert abs(1e9 / per_expert_q2_0 - p["experts_per_gb"]) / p["experts_per_gb"] < 0.02
    per_token = p["layers"] * p["topk"] * per_expert_q2_0 / 1e9
    assert abs(per_token - (p["read_per_token_gb"] - p["shared_part_gb"])) < 0.05
    # this project's two formats land on the 2.50 and 3.50 bpw rows of the table
    ours2 = O.expert_layout(2048, 768, 2)["bytes"] * p["total_experts"] / 1e9
    ours3 = O.expert_layout(2048, 768, 3)["bytes"] * p["total_experts"] / 1e9
    assert abs(ours2 - p["iq2_xs_expert_gb"]) / p["iq2_xs_expert_gb"] < 0.03
    assert abs(ours3 - p["iq3_s_expert_gb"]) / p["iq3_s_expert_gb"] < 0.03


# ------------------------------------------------------------------ top-k and gates

def _brute_topk(row, k):
    # Python's sorted is stable; NaN is pushed below every number by the key
    key = lambda e: (0 if np.isnan(row[e]) else 1, -0.0 if np.isnan(row[e]) else row[e])
    return sorted(range(len(row)), key=lambda e: (-key(e)[0], -key(e)[1], e))[:k]


def test_topk_exhaustive_ties_E16_k2():
    rows = np.array(list(itertools.product([0.0, 1.0], repeat=16)))
    idx = O.topk(rows, 2)
    for r, got in zip(rows, idx):
        assert list(got) == _brute_topk(list(r), 2)


@pytest.mark.parametrize("E,k", [(16, 2), (64, 10), (512, 10)])
def test_topk_random_with_ties(E, k):
    g = np.random.default_rng(E)
    rows = g.integers(-3, 4, size=(50, E)).astype(np.float64)  # many ties
    rows[:10] = g.standard_normal((10, E))
    idx = O.topk(rows, k)
    for r, got in zip(rows, idx):
        assert list(got) == _brute_topk(list(r), k)
        assert len(set(got)) == k and got.min() >= 0 and got.max() < E


def test_topk_nan_signed_zero_and_inf():
    row = np.array([np.nan, -0.0, 0.0, -np.inf, np.nan, 0.0])
    assert list(O.topk(row[None], 6)[0]) == [1, 2, 5, 3, 0, 4]


def test_gates_closed_forms():
    g = np.random.default_rng(3)
    l = g.standard_normal((20, 16)) * 3
    idx = O.topk(l, 2)
    gt = O.gates(l, idx)
    l0 = np.take_along_axis(l, idx.astype(np.int64), 1)
    # two experts: g0 = sigmoid(l0 - l1)
    assert np.allclose(gt[:, 0], scipy.special.expit(l0[:, 0] - l0[:, 1]), rtol=0, atol=1e-15)
    assert np.allclose(gt.sum(1), 1.0, atol=1e-15)
    # k=1 gives gate 1
    assert np.all(O.gates(l, O.topk(l, 1)) == 1.0)
    # renorm=0 is the full softmax read at the chosen experts
    idx10 = O.topk(l, 10)
    full = scipy.special.softmax(l, axis=1)
    assert np.allclose(O.gates(l, idx10, renorm=False), np.take_along_axis(full, idx10.astype(np.int64), 1),
                       rtol=1e-13, atol=0)
    # renorm=1 is a softmax over the chosen logits
    assert np.allclose(O.gates(l, idx10), scipy.special.softmax(np.take_along_axis(l, idx10.astype(np.int64), 1), axis=1),
                       rtol=1e-13, atol=0)
    # gates are in descending order, like the logits
    assert np.all(np.diff(O.gates(l, idx10), axis=1) <= 0)


def test_ten_of_512_per_token():
    """10 distinct experts of 512 per token, as the pages state."""
    x = synth.activations(8, 2048, seed=0)
    wr = synth.router_weights(512, 2048, seed=1)
    _, idx, _ = O.route(x, wr, 10)
    assert idx.shape == (8, 10)
    for row in idx:
        assert len(set(row.tolist())) == 10 and row.min() >= 0 and row.max() < 512


def test_router_logits_against_bruteforce_sum():
    x = synth.activations(2, 64, seed=4)
    wr = synth.router_weights(5, 64, seed=5)
    l = O.router_logits(x, wr)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(2):
        for e in range(5):
            s = 0.0
            for i in range(64):
                s += float(xf[t, i]) * float(wr[e, i])
            assert abs(l[t, e] - s) < 1e-12


# ------------------------------------------------------------------ grouping

def _brute_group(idx, E):
    T, k = idx.shape
    pairs = []
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    pairs.append((e, t, j))
    return pairs


@pytest.mark.parametrize("T,E,k", [(4, 16, 2), (1, 512, 10), (4, 512, 10), (300, 64, 10)])
def test_grouping_matches_enumeration_and_invariants(T, E, k):
    g = np.random.default_rng(T + E)
    idx = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    gate = g.random((T, k))
    slot_of = g.permutation(E).astype(np.int32)
    gr = O.group(idx, gate, E, slot_of)
    pairs = _brute_group(idx, E)
    assert list(zip(gr["pair_token"], gr["pair_j"])) == [(t, j) for _, t, j in pairs]
    cnt, off = gr["expert_count"], gr["expert_offset"]
    assert cnt.sum() == T * k and off[0] == 0 and off[-1] == T * k
    assert np.array_equal(np.diff(off), cnt)
    for e in range(E):
        seg = slice(off[e], off[e + 1])
        assert np.all(idx[gr["pair_token"][seg], gr["pair_j"][seg]] == e)
        assert np.all(np.diff(gr["pair_token"][seg]) > 0)  # stable: tokens ascending
    # pair_pos is the inverse permutation
    for t in range(T):
        for j in range(k):
            p = gr["pair_pos"][t, j]
            assert gr["pair_token"][p] == t and gr["pair_j"][p] == j and gr["pair_gate"][p] == gate[t, j]
    assert np.array_equal(gr["uniq_expert"], np.unique(idx))
    assert np.array_equal(gr["uniq_slot"], slot_of[np.unique(idx)])


# ------------------------------------------------------------------ expert FFN

def test_silu_against_library_and_identities():
    import torch
    z = np.linspace(-30, 30, 601)
    s = O.silu(z)
    assert np.allclose(s, z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)
    assert np.allclose(s, torch.nn.functional.silu(torch.from_numpy(z)).numpy(), rtol=1e-14, atol=1e-300)
    assert O.silu(0.0) == 0.0
    assert np.allclose(O.silu(-z), O.silu(z) - z, atol=1e-12)
    assert O.silu(-1000.0) == 0.0 and O.silu(1000.0) == 1000.0


def _perm_expert(d, f, bits, seed):
    """An expert whose dequantised matrices are signed permutation-like matrices.

    W_g[c, p1[c]] = +1, W_u[c, p2[c]] = -2, W_d[i, p3[i]] = +1, zeros elsewhere,
    built through the quantiser with all scales 1.0.
    """
    g = np.random.default_rng(seed)
    p1 = g.permutation(d)[:f]
    p2 = g.permutation(d)[:f]
    p3 = g.integers(0, f, size=d)
    wg = np.zeros((f, d)); wg[np.arange(f), p1] = 1.0
    wu = np.zeros((f, d)); wu[np.arange(f), p2] = -2.0
    wd = np.zeros((d, f)); wd[np.arange(d), p3] = 1.0
    wgu = np.empty((2 * f, d)); wgu[0::2] = wg; wgu[1::2] = wu
    ones_gu = np.ones((2 * f, d // 32), dtype=np.float16)
    ones_dn = np.ones((d, f // 32), dtype=np.float16)
    sec = {"gu_codes": O.quantize(wgu, ones_gu, bits), "gu_scales": ones_gu,
           "dn_codes": O.quantize(wd, ones_dn, bits), "dn_scales": ones_dn}
    return sec, p1, p2, p3


@pytest.mark.parametrize("bits", [2, 3])
def test_expert_closed_form_permutations(bits):
    d, f = 64, 32
    sec, p1, p2, p3 = _perm_expert(d, f, bits, seed=bits)
    wg, wu, wd = O.expert_weights(sec, d, f, bits)
    x = synth.activations(3, d, seed=9)
    xd = O.bf16_to_f64(x)
    z = O.expert_forward(xd, wg, wu, wd)
    for t in range(3):
        xt = xd[t]
        for i in range(d):
            c = p3[i]
            a = xt[p1[c]]
            want = (a / (1.0 + np.exp(-a))) * (-2.0 * xt[p2[c]])
            assert z[t, i] == pytest.approx(want, rel=1e-14, abs=1e-300)


def _tiny_layer(d, f, E, bits, seed):
    secs = [synth.expert_sections(d, f, bits, seed + 10 + e) for e in range(E)]
    shared = synth.expert_sections(d, f, bits, seed + 5)
    return secs, shared


def test_one_hot_gate_reduces_to_dense_ffn_torch():
    """One expert at gate 1 (its logit +1e4): y = FFN_e(x) + FFN_shared(x), checked with torch fp64."""
    import torch
    F = torch.nn.functional
    d, f, E, k, bits = 256, 128, 16, 2, 2
    secs, shared = _tiny_layer(d, f, E, bits, seed=0)
    x = synth.activations(4, d, seed=1)
    wr = synth.router_weights(E, d, seed=2)
    bias = np.zeros((4, E), dtype=np.float64)
    hot = [3, 7, 11, 3]
    for t, e in enumerate(hot):
        bias[t, e] = 1e4
    cache = O.ExpertCache(lambda e: secs[e], d, f, bits)
    sh = O.expert_weights(shared, d, f, bits)
    out = O.layer_forward(x, wr, k, cache, sh, bias=bias)
    assert np.all(out["gate"][:, 0] == 1.0) and np.all(out["gate"][:, 1] == 0.0)

    def torch_ffn(sec, xt):
        wgu = torch.from_numpy(O.dequant(sec["gu_codes"], sec["gu_scales"], d, bits))
        wd = torch.from_numpy(O.dequant(sec["dn_codes"], sec["dn_scales"], f, bits))
        wg, wu = wgu[0::2], wgu[1::2]  # gate rows are the even rows, up rows the odd rows
        return F.linear(F.silu(F.linear(xt, wg)) * F.linear(xt, wu), wd)

    xt = torch.from_numpy(O.bf16_to_f64(x))
    for t, e in enumerate(hot):
        want = torch_ffn(secs[e], xt[t]) + torch_ffn(shared, xt[t])
        assert np.allclose(out["y"][t], want.numpy(), rtol=1e-12, atol=1e-14)


def test_gate_split_between_identical_experts_is_linear():
    d, f, E, k, bits = 256, 128, 16, 2, 3
    secs, shared = _tiny_layer(d, f, E, bits, seed=4)
    secs[5] = secs[9]  # two experts with the same weights
    x = synth.activations(2, d, seed=6)
    wr = synth.router_weights(E, d, seed=7)
    bias = np.zeros((2, E)); bias[:, 5] = 50.0; bias[:, 9] = 50.0 + np.array([0.3, -1.2])
    cache = O.ExpertCache(lambda e: secs[e], d, f, bits)
    out = O.layer_forward(x, wr, k, cache, None, bias=bias)
    wg, wu, wd = cache(5)
    want = O.expert_forward(O.bf16_to_f64(x), wg, wu, wd)
    assert np.allclose(out["y"], want, rtol=1e-12, atol=1e-13)


def test_token_permutation_invariance_and_residual():
    d, f, E, k, bits = 256, 128, 16, 2, 2
    secs, shared = _tiny_layer(d, f, E, bits, seed=8)
    x = synth.activations(6, d, seed=9)
    wr = synth.router_weights(E, d, seed=10)
    cache = O.ExpertCache(lambda e: secs[e], d, f, bits)
    sh = O.expert_weights(shared, d, f, bits)
    a = O.layer_forward(x, wr, k, cache, sh)
    perm = np.array([4, 0, 5, 2, 1, 3])
    b = O.layer_forward(x[perm], wr, k, cache, sh)
    assert np.array_equal(b["idx"], a["idx"][perm])
    assert np.allclose(b["y"], a["y"][perm], rtol=1e-13, atol=1e-15)
    r = O.layer_forward(x, wr, k, cache, sh, residual=True)
    assert np.allclose(r["y"], a["y"] + O.bf16_to_f64(x), rtol=1e-13, atol=1e-15)
    # dropping the shared expert changes the output by exactly the shared FFN
    c = O.layer_forward(x, wr, k, cache, None)
    assert np.allclose(a["y"] - c["y"], O.expert_forward(O.bf16_to_f64(x), *sh), rtol=1e-10, atol=1e-13)


def _bit(byte_val, bit):
    return (byte_val >> bit) & 1


def _brute_weight(sec_codes, sec_scales, r, c, K, bits):
    """One dequantised weight read straight off the bit-level definition."""
    row = sec_codes[r]
    low = (int(row[c // 4]) >> (2 * (c % 4))) & 3
    q = low
    if bits == 3:
        q += 4 * _bit(int(row[K // 4 + c // 8]), c % 8)
    return float(sec_scales[r, c // 32]) * (q - (1 << (bits - 1)))


@pytest.mark.parametrize("bits", [2, 3])
def test_brute_force_tiny_layer(bits):
    """Scalar loops over a tiny layer (d=32, f=32, E=4, k=2, T=2) from the bit-level definition."""
    import math
    d, f, E, k, T = 32, 32, 4, 2, 2
    secs, shared = _tiny_layer(d, f, E, bits, seed=20 + bits)
    x = synth.activations(T, d, seed=30)
    wr = synth.router_weights(E, d, seed=31) * 20
    cache = O.ExpertCache(lambda e: secs[e], d, f, bits)
    out = O.layer_forward(x, wr, k, cache, O.expert_weights(shared, d, f, bits))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)

    def ffn(sec, xt):
        h = []
        for c in range(f):
            gsum = sum(_brute_weight(sec["gu_codes"], sec["gu_scales"], 2 * c, i, d, bits) * xt[i] for i in range(d))
            usum = sum(_brute_weight(sec["gu_codes"], sec["gu_scales"], 2 * c + 1, i, d, bits) * xt[i] for i in range(d))
            h.append(gsum / (1 + math.exp(-gsum)) * usum)
        return [sum(_brute_weight(sec["dn_codes"], sec["dn_scales"], r, c, f, bits) * h[c] for c in range(f))
                for r in range(d)]

    for t in range(T):
        logits = [sum(xf[t, i] * float(wr[e, i]) for i in range(d)) for e in range(E)]
        order = sorted(range(E), key=lambda e: (-logits[e], e))[:k]
        ex = [math.exp(logits[e] - logits[order[0]]) for e in order]
        gts = [v / sum(ex) for v in ex]
        y = ffn(shared, xf[t])
        acc = [0.0] * d
        for j, e in enumerate(order):
            z = ffn(secs[e], xf[t])
            acc = [a + gts[j] * zz for a, zz in zip(acc, z)]
        y = [a + b for a, b in zip(acc, y)]
        assert list(out["idx"][t]) == order
        assert np.allclose(out["y"][t], y, rtol=1e-11, atol=1e-13)


def test_skipping_low_ranked_non_resident_pairs():
    """Leaving out pairs of rank >= skip_from on non-resident slots: the cases
    that reduce to no skipping (every slot resident; skip_from = k), the case
    that keeps only the top expert (skip_from = 1, nothing resident), and the
    general case against the full layer minus the dropped pairs' terms."""
    d, f, E, k, bits = 256, 128, 16, 4, 2
    secs, shared = _tiny_layer(d, f, E, bits, seed=40)
    x = synth.activations(5, d, seed=41)
    wr = synth.router_weights(E, d, seed=42)
    cache = O.ExpertCache(lambda e: secs[e], d, f, bits)
    sh = O.expert_weights(shared, d, f, bits)
    slot_of = synth.rng(43).permutation(E)
    full = O.layer_forward(x, wr, k, cache, sh)
    same = O.layer_forward(x, wr, k, cache, sh, skip_from=1, hot_slots=E, slot_of=slot_of)
    assert np.array_equal(same["y"], full["y"]) and same["keep"].all()
    same = O.layer_forward(x, wr, k, cache, sh, skip_from=k, hot_slots=0, slot_of=slot_of)
    assert np.array_equal(same["y"], full["y"])
    top = O.layer_forward(x, wr, k, cache, sh, skip_from=1, hot_slots=0, slot_of=slot_of)
    xd = O.bf16_to_f64(x)
    for t in range(5):
        e0 = int(full["idx"][t, 0])
        want = full["gate"][t, 0] * O.expert_forward(xd[t], *cache(e0)) + O.expert_forward(xd[t], *sh)
        assert np.allclose(top["y"][t], want, rtol=1e-12, atol=1e-14)
    part = O.layer_forward(x, wr, k, cache, sh, skip_from=2, hot_slots=E // 2, slot_of=slot_of)
    keep = part["keep"]
    assert keep[:, :2].all()
    assert np.array_equal(keep[:, 2:], slot_of[full["idx"][:, 2:]] < E // 2)
    for t in range(5):
        drop = sum(full["gate"][t, j] * O.expert_forward(xd[t], *cache(int(full["idx"][t, j])))
                   for j in range(k) if not keep[t, j])
        assert np.allclose(part["y"][t], full["y"][t] - drop, rtol=1e-10, atol=1e-12)
    g = O.group(full["idx"], full["gate"], E, slot_of, keep=keep)
    assert g["expert_count"].sum() == keep.sum()
    assert np.all(g["pair_pos"][~keep] == -1)
    kept_pos = np.sort(g["pair_pos"][keep])
    assert np.array_equal(kept_pos, np.arange(keep.sum()))
