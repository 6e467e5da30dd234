"""Seeded synthetic inputs for the sparse-MoE FFN step.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no routing, no dequantisation, no matrix products).
Both the fp64 CPU oracle (through the tests) and the CUDA path (through the
tests and the benchmark) take their inputs from here, so that the two sides
see the same bytes.

Recipe (every draw uses NumPy's PCG64 unless stated):

* activations x: N(0, 1) rounded to bf16 (round to nearest even), seed as given;
* router weights W_r: N(0, 0.02) as fp32;
* expert codes: uniform random bytes, which makes every 2-bit or 3-bit code
  uniform over its range whatever its position in the packed row;
* expert scales: U(0.005, 0.02) rounded to fp16;
* Zipf routing: each layer draws a permutation that gives every expert a
  popularity rank r in 1..E; a token's expert set is a Gumbel-top-k sample of
  p_e ~ r_e^-s (Plackett-Luce sampling without replacement, s = 1.1), turned
  into a logit bias of +20 on the chosen experts;
* layer l of a stack uses seed + 1000*l.

Large pools (tens of GB) are filled on the device with torch's seeded
generator instead of NumPy, so that no host round trip is needed; the
scale sections are written where the caller says they are.
"""
from __future__ import annotations

import numpy as np

ZIPF_S = 1.1
BIAS = 20.0


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns raw uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(a)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def activations(T: int, d: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """x [T, d] as raw bf16 bits, N(0, scale^2) (a power-of-two scale only
    moves the exponent of the N(0,1) draw)."""
    return f32_to_bf16_bits(rng(seed).standard_normal((T, d), dtype=np.float32) * np.float32(scale))


def router_weights(E: int, d: int, seed: int, std: float = 0.02) -> np.ndarray:
    """W_r [E, d] fp32, N(0, std)."""
    return (rng(seed).standard_normal((E, d), dtype=np.float32) * np.float32(std)).astype(np.float32)


def random_scales(shape, g: np.random.Generator) -> np.ndarray:
    return g.uniform(0.005, 0.02, size=shape).astype(np.float16)


def expert_sections(d: int, f: int, bits: int, seed: int) -> dict:
    """One expert's packed weights as four separate arrays.

    gu_codes [2f, d*bits/8] uint8, dn_codes [d, f*bits/8] uint8,
    gu_scales [2f, d/32] fp16, dn_scales [d, f/32] fp16.
    """
    g = rng(seed)
    return {
        "gu_codes": g.integers(0, 256, size=(2 * f, d * bits // 8), dtype=np.uint8),
        "dn_codes": g.integers(0, 256, size=(d, f * bits // 8), dtype=np.uint8),
        "gu_scales": random_scales((2 * f, d // 32), g),
        "dn_scales": random_scales((d, f // 32), g),
    }


def zipf_ranks(E: int, seed: int) -> np.ndarray:
    """ranks[e] in 1..E: a seeded permutation (rank 1 = most popular)."""
    return rng(seed).permutation(E) + 1


def zipf_logp(ranks: np.ndarray, s: float = ZIPF_S) -> np.ndarray:
    return -s * np.log(ranks.astype(np.float64))


def gumbel_topk_sets(T: int, k: int, logp: np.ndarray, g: np.random.Generator,
                     exclude=None) -> np.ndarray:
    """T unordered k-subsets drawn without replacement with P(e) ~ exp(logp[e])."""
    E = logp.shape[0]
    keys = logp[None, :] + g.gumbel(size=(T, E))
    if exclude is not None:
        keys = np.where(exclude, -np.inf, keys)
    return np.argpartition(-keys, k - 1, axis=1)[:, :k].astype(np.int32)


def zipf_sets(T: int, E: int, k: int, seed: int, s: float = ZIPF_S) -> np.ndarray:
    """Expert sets [T, k] for one layer; the layer's popularity permutation comes from `seed`."""
    ranks = zipf_ranks(E, seed)
    return gumbel_topk_sets(T, k, zipf_logp(ranks, s), rng(seed + 1))


def bias_from_sets(sets: np.ndarray, E: int, big: float = BIAS) -> np.ndarray:
    T = sets.shape[0]
    b = np.zeros((T, E), dtype=np.float32)
    np.put_along_axis(b, sets.astype(np.int64), np.float32(big), axis=1)
    return b


def correlated_sets(steps: int, T: int, E: int, k: int, keep: int, seed: int,
                    s: float = ZIPF_S) -> np.ndarray:
    """Expert sets [steps, T, k] for one layer with temporal reuse.

    Step 0 is a fresh Zipf draw. At step i, each token position keeps `keep`
    experts of its step i-1 set (uniform choice) and draws k-keep new ones by
    Zipf among the experts it did not keep.
    """
    ranks = zipf_ranks(E, seed)
    logp = zipf_logp(ranks, s)
    g = rng(seed + 1)
    out = np.empty((steps, T, k), dtype=np.int32)
    out[0] = gumbel_topk_sets(T, k, logp, g)
    for i in range(1, steps):
        for t in range(T):
            kept = g.choice(out[i - 1, t], size=keep, replace=False)
            excl = np.zeros((1, E), dtype=bool)
            excl[0, kept] = True
            new = gumbel_topk_sets(1, k - keep, logp, g, exclude=excl)[0]
            out[i, t, :keep] = kept
            out[i, t, keep:] = new
    return out


def hot_slot_table(L: int, E: int, n_hot: int, seed: int, s: float = ZIPF_S) -> np.ndarray:
    """slot_of [L*E] int32: the n_hot most popular (layer, expert) pairs get slots 0..n_hot-1.

    Popularity is the per-layer Zipf rank drawn with seed + 1000*l (the same
    permutation `zipf_sets` uses); equal ranks across layers are ordered by
    layer. The remaining experts follow in (layer, expert) order.
    """
    rank = np.stack([zipf_ranks(E, seed + 1000 * l) for l in range(L)])  # [L, E]
    flat_rank = rank.reshape(-1)
    layer = np.repeat(np.arange(L), E)
    expert = np.tile(np.arange(E), L)
    order = np.lexsort((expert, layer, flat_rank))  # by rank, then layer, then expert
    hot = order[:n_hot]
    cold = np.setdiff1d(np.arange(L * E), hot)  # ascending (layer, expert)
    slot_of = np.empty(L * E, dtype=np.int32)
    slot_of[hot] = np.arange(n_hot, dtype=np.int32)
    slot_of[cold] = np.arange(n_hot, L * E, dtype=np.int32)
    return slot_of


# ---------------------------------------------------------------- torch (device) fills

def fill_random_bytes_(t, seed: int, chunk_bytes: int = 1 << 30) -> None:
    """Fill a uint8 torch tensor (any device) with seeded uniform random bytes."""
    import torch
    flat = t.view(-1)
    g = torch.Generator(device=t.device)
    g.manual_seed(seed)
    for s in range(0, flat.numel(), chunk_bytes):
        flat[s:s + chunk_bytes].random_(0, 256, generator=g)


def fill_scales_(t_u8, seed: int) -> None:
    """Overwrite a uint8 torch view (an even number of bytes per row) with fp16 U(0.005, 0.02)."""
    import torch
    g = torch.Generator(device=t_u8.device)
    g.manual_seed(seed)
    v = torch.empty(t_u8.shape[:-1] + (t_u8.shape[-1] // 2,), dtype=torch.float16, device=t_u8.device)
    v.uniform_(0.005, 0.02, generator=g)
    t_u8.copy_(v.view(torch.uint8))
