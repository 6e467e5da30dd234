"""Plant plausible mistakes in the oracle (on the CPU) and check that its pins catch each one.

Every mutation below replaces one oracle function with a wrong variant; at
least one pin from test_oracle_pins must then fail. This guards the pins
themselves: a pin set that passes a broken oracle pins nothing.
"""
import numpy as np
import pytest

import tests.test_oracle_pins as P
from oracle import moe_oracle as O

PINS = [
    lambda: P.test_golden_q2_bytes_and_weights(),
    lambda: P.test_golden_q3_bytes_and_weights(),
    lambda: P.test_dequant_value_set_and_round_trip(2),
    lambda: P.test_dequant_value_set_and_round_trip(3),
    lambda: P.test_topk_exhaustive_ties_E16_k2(),
    lambda: P.test_topk_random_with_ties(64, 10),
    lambda: P.test_topk_nan_signed_zero_and_inf(),
    lambda: P.test_gates_closed_forms(),
    lambda: P.test_grouping_matches_enumeration_and_invariants(4, 16, 2),
    lambda: P.test_silu_against_library_and_identities(),
    lambda: P.test_expert_closed_form_permutations(2),
    lambda: P.test_expert_closed_form_permutations(3),
    lambda: P.test_one_hot_gate_reduces_to_dense_ffn_torch(),
    lambda: P.test_token_permutation_invariance_and_residual(),
    lambda: P.test_brute_force_tiny_layer(2),
    lambda: P.test_brute_force_tiny_layer(3),
]

_orig = {name: getattr(O, name) for name in
         ("expert_weights", "topk", "gates", "group", "silu", "unpack_codes", "dequant", "layer_forward",
          "expert_forward", "router_logits")}


def _swap_gate_up(sec, d, f, bits):
    wg, wu, wd = _orig["expert_weights"](sec, d, f, bits)
    return wu, wg, wd


def _ties_to_upper(logits, k):
    l = np.asarray(logits, dtype=np.float64)
    E = l.shape[1]
    return np.stack([np.lexsort((-np.arange(E), -row))[:k] for row in l]).astype(np.int32)


def _gates_no_renorm(logits, idx, renorm=True):
    return _orig["gates"](logits, idx, False)


def _group_unstable(idx, gate, E, slot_of=None):
    g = _orig["group"](idx, gate, E, slot_of)
    # reverse the tokens inside every expert's segment
    off = g["expert_offset"]
    for key in ("pair_token", "pair_j", "pair_gate"):
        a = g[key].copy()
        for e in range(E):
            a[off[e]:off[e + 1]] = a[off[e]:off[e + 1]][::-1]
        g[key] = a
    return g


def _silu_wrong(z):
    return np.asarray(z, dtype=np.float64) / (1.0 + np.exp(np.asarray(z, dtype=np.float64)))


def _unpack_planes_swapped(packed, K, bits):
    q = _orig["unpack_codes"](packed, K, bits)
    if bits == 3:
        return (q >> 2) + 2 * (q & 3) % 8
    return q


def _unpack_bits_reversed(packed, K, bits):
    q = _orig["unpack_codes"](packed, K, bits)
    out = q.copy()
    for s in range(4):
        out[:, s::4] = q[:, (3 - s)::4]
    return out


def _dequant_wrong_offset(packed, scales, K, bits):
    w = _orig["dequant"](packed, scales, K, bits)
    s = np.repeat(np.asarray(scales, dtype=np.float64), 32, axis=1)
    return w + s


def _expert_transposed_down(xd, wg, wu, wd):
    x2 = np.atleast_2d(xd)
    h = O.silu(x2 @ wg.T) * (x2 @ wu.T)
    wdt = wd.reshape(wd.shape[1], wd.shape[0]) if wd.shape[0] != wd.shape[1] else wd.T
    z = h @ wdt if wd.shape[0] != wd.shape[1] else h @ wdt.T
    return z if np.ndim(xd) == 2 else z[0]


def _layer_drop_shared(x_bits, w_router, k, experts, shared=None, **kw):
    return _orig["layer_forward"](x_bits, w_router, k, experts, None, **kw)


def _layer_ungated(x_bits, w_router, k, experts, shared=None, bias=None, renorm=True, residual=False, tokens=None):
    out = _orig["layer_forward"](x_bits, w_router, k, experts, shared, bias=bias, renorm=renorm,
                                 residual=residual, tokens=tokens)
    xd = O.bf16_to_f64(x_bits)
    ys = []
    for t in range(xd.shape[0]):
        y = sum(O.expert_forward(xd[t], *experts(int(e))) for e in out["idx"][t])
        if shared is not None:
            y = y + O.expert_forward(xd[t], *shared)
        ys.append(xd[t] + y if residual else y)
    out["y"] = np.array(ys)
    return out


def _router_transposed_bias(x_bits, w_router, bias=None):
    return _orig["router_logits"](x_bits, w_router, None if bias is None else -np.asarray(bias))


MUTATIONS = {
    "gate_up_swapped": ("expert_weights", _swap_gate_up),
    "ties_to_upper_index": ("topk", _ties_to_upper),
    "gates_not_renormalised": ("gates", _gates_no_renorm),
    "grouping_unstable": ("group", _group_unstable),
    "silu_wrong_sign": ("silu", _silu_wrong),
    "bit_planes_swapped": ("unpack_codes", _unpack_planes_swapped),
    "code_order_in_byte_reversed": ("unpack_codes", _unpack_bits_reversed),
    "dequant_offset_off_by_one": ("dequant", _dequant_wrong_offset),
    "down_projection_transposed": ("expert_forward", _expert_transposed_down),
    "shared_expert_dropped": ("layer_forward", _layer_drop_shared),
    "gates_ignored_in_combine": ("layer_forward", _layer_ungated),
    "bias_sign_flipped": ("router_logits", _router_transposed_bias),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except Exception:  # an assertion or a shape error both count as caught
            caught += 1
    assert caught >= 1, f"no pin caught mutation {name}"
