"""fp64 CPU oracle of the per-layer sparse-MoE FFN step.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline may import or run this module. It shares no code with the CUDA path
and imports nothing from it.

What it follows. The pages describe Qwen3.8-Flash-Next as 48 layers of 512
experts, of which each token uses 10 plus one always-on shared expert
(Strataとは, news.blueqat.app/post/3262, first section; geekoyaji.com
"freetoken-vs-strata-moe-offload", section 共通の仕組み), with expert weights
stored at 2 to 3 bits (geekoyaji.com comparison table; news.blueqat.app
section 量子化の種類とサイズ). They give no formula for any step, so every
function below is the plain definition of a top-k MoE layer with SwiGLU
experts on block-quantised weights, in fp64:

  1. logits   l[t,e] = sum_i x[t,i] W_r[e,i]  (+ an optional bias)
  2. top-k    the k largest logits, ties to the lower expert index
  3. gates    softmax over the k chosen logits (renorm=1) or the full
              softmax restricted to them (renorm=0)
  4. grouping stable sort of the (token, j) pairs by expert
  5. expert   h = silu(W_g x) * (W_u x),  z = W_d h, with W = s*(q - 2^(b-1))
  6. combine  y[t] = sum_j gate[t,j] z_(t,j)  (j ascending)  +  z_shared[t]

The block format (32 weights along the reduction axis per fp16 scale, codes
packed little-end first, 3-bit rows split into a 2-bit plane and a 1-bit
plane) is this project's own definition: the pages name Q2_0 and the IQ
formats but do not describe their bits.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
SECTION_ALIGN = 256


# ------------------------------------------------------------------ scalar types

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 raw bits -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def fp16_to_f64(h) -> np.ndarray:
    return np.asarray(h, dtype=np.float16).astype(np.float64)


# ------------------------------------------------------------------ block format

def row_bytes(K: int, bits: int) -> int:
    """Packed code bytes of one row of K weights."""
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    if bits == 2:
        return K // 4
    if bits == 3:
        return K // 4 + K // 8
    raise ValueError("bits must be 2 or 3")


def _align(n: int, a: int = SECTION_ALIGN) -> int:
    return (n + a - 1) // a * a


def expert_layout(d: int, f: int, bits: int) -> dict:
    """Byte offsets of one expert record: gate/up codes, down codes, gate/up scales, down scales.

    Gate/up is [2f, d] with gate row c at 2c and up row c at 2c+1; down is [d, f].
    Each section starts on a 256-byte boundary; the record size is rounded up to 256.
    """
    sizes = {
        "gu_codes": 2 * f * row_bytes(d, bits),
        "dn_codes": d * row_bytes(f, bits),
        "gu_scales": 2 * f * (d // BLOCK) * 2,
        "dn_scales": d * (f // BLOCK) * 2,
    }
    off = 0
    lay = {}
    for name in ("gu_codes", "dn_codes", "gu_scales", "dn_scales"):
        lay[name] = (off, sizes[name])
        off = _align(off + sizes[name])
    lay["bytes"] = off
    return lay


def sections_from_record(record: np.ndarray, d: int, f: int, bits: int) -> dict:
    lay = expert_layout(d, f, bits)
    r = np.asarray(record, dtype=np.uint8).reshape(-1)

    def sec(name, rows, cols, dtype):
        o, n = lay[name]
        return r[o:o + n].view(dtype).reshape(rows, cols)

    return {
        "gu_codes": sec("gu_codes", 2 * f, row_bytes(d, bits), np.uint8),
        "dn_codes": sec("dn_codes", d, row_bytes(f, bits), np.uint8),
        "gu_scales": sec("gu_scales", 2 * f, d // BLOCK, np.float16),
        "dn_scales": sec("dn_scales", d, f // BLOCK, np.float16),
    }


def record_from_sections(sec: dict, d: int, f: int, bits: int) -> np.ndarray:
    lay = expert_layout(d, f, bits)
    r = np.zeros(lay["bytes"], dtype=np.uint8)
    for name in ("gu_codes", "dn_codes", "gu_scales", "dn_scales"):
        o, n = lay[name]
        r[o:o + n] = np.ascontiguousarray(sec[name]).view(np.uint8).reshape(-1)
    return r


def unpack_codes(packed: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Packed rows [R, row_bytes] -> integer codes [R, K].

    2-bit: code c of a row sits in byte c//4 at bits 2*(c%4).
    3-bit: the row holds that same 2-bit plane (K/4 bytes) for the low bits,
    then a 1-bit plane (K/8 bytes) with the high bit of code c at bit c%8 of
    byte c//8; q = low + 4*high.
    """
    p = np.asarray(packed, dtype=np.uint8)
    R = p.shape[0]
    low = np.empty((R, K), dtype=np.int64)
    lowp = p[:, :K // 4].astype(np.int64)
    for s in range(4):
        low[:, s::4] = (lowp >> (2 * s)) & 3
    if bits == 2:
        return low
    highp = p[:, K // 4:K // 4 + K // 8].astype(np.int64)
    high = np.empty((R, K), dtype=np.int64)
    for s in range(8):
        high[:, s::8] = (highp >> s) & 1
    return low + 4 * high


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """Integer codes [R, K] -> packed rows (inverse of unpack_codes)."""
    q = np.asarray(q, dtype=np.int64)
    R, K = q.shape
    if q.min() < 0 or q.max() >= (1 << bits):
        raise ValueError("code out of range")
    low = q & 3
    lowp = np.zeros((R, K // 4), dtype=np.int64)
    for s in range(4):
        lowp |= low[:, s::4] << (2 * s)
    if bits == 2:
        return lowp.astype(np.uint8)
    high = q >> 2
    highp = np.zeros((R, K // 8), dtype=np.int64)
    for s in range(8):
        highp |= high[:, s::8] << s
    return np.concatenate([lowp, highp], axis=1).astype(np.uint8)


def dequant(packed: np.ndarray, scales: np.ndarray, K: int, bits: int) -> np.ndarray:
    """w[r, c] = s[r, c//32] * (q[r, c] - 2^(bits-1)) in fp64."""
    q = unpack_codes(packed, K, bits)
    s = np.repeat(fp16_to_f64(scales), BLOCK, axis=1)
    return s * (q - (1 << (bits - 1))).astype(np.float64)


def quantize(w: np.ndarray, scales: np.ndarray, bits: int) -> np.ndarray:
    """q = clamp(round_half_even(w / s) + 2^(bits-1), 0, 2^bits - 1), packed."""
    w = np.asarray(w, dtype=np.float64)
    s = np.repeat(fp16_to_f64(scales), BLOCK, axis=1)
    off = 1 << (bits - 1)
    q = np.clip(np.rint(w / s) + off, 0, (1 << bits) - 1).astype(np.int64)
    return pack_codes(q, bits)


def expert_weights(sec: dict, d: int, f: int, bits: int):
    """Dequantised (W_g [f,d], W_u [f,d], W_d [d,f]) of one expert."""
    wgu = dequant(sec["gu_codes"], sec["gu_scales"], d, bits)
    wd = dequant(sec["dn_codes"], sec["dn_scales"], f, bits)
    return wgu[0::2], wgu[1::2], wd


# ------------------------------------------------------------------ router

def router_logits(x_bits: np.ndarray, w_router: np.ndarray, bias=None) -> np.ndarray:
    """l[t, e] = sum_i x[t,i] W_r[e,i] in fp64, plus bias[t, e] if given.

    The router runs on the GPU for every token (news.blueqat.app/post/3262,
    section GPU・CPU・RAM・SSDの分担, placement table).
    """
    xd = bf16_to_f64(x_bits)
    wr = np.asarray(w_router, dtype=np.float64)
    l = xd @ wr.T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)
    return l


def topk(logits: np.ndarray, k: int) -> np.ndarray:
    """idx[t, 0..k): experts ordered by descending logit, ties to the lower index.

    NaN ranks below every number (it is never chosen while k numbers exist);
    -0.0 and +0.0 are equal. Each token uses 10 of its layer's 512 experts
    (Strataとは, news.blueqat.app/post/3262, first section).
    """
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    out = np.empty((T, k), dtype=np.int32)
    e = np.arange(E)
    for t in range(T):
        order = np.lexsort((e, -l[t]))  # primary: -l ascending (NaN last); secondary: e
        out[t] = order[:k]
    return out


def gates(logits: np.ndarray, idx: np.ndarray, renorm: bool = True) -> np.ndarray:
    """Gate weights [T, k] in fp64.

    renorm=1: g_j = exp(l_j - l_0) / sum_{j'<k} exp(l_j' - l_0), a softmax over
    the k chosen logits. renorm=0: the full softmax over all E logits, read at
    the chosen experts. The pages do not say which; renormalising is the
    default reading.
    """
    l = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(l, idx.astype(np.int64), axis=1)
    top = sel[:, :1]
    ex = np.exp(sel - top)
    if renorm:
        return ex / ex.sum(axis=1, keepdims=True)
    full = np.exp(l - top).sum(axis=1, keepdims=True)
    return ex / full


def route(x_bits, w_router, k, bias=None, renorm=True):
    l = router_logits(x_bits, w_router, bias)
    idx = topk(l, k)
    return l, idx, gates(l, idx, renorm)


# ------------------------------------------------------------------ grouping

def group(idx: np.ndarray, gate: np.ndarray, E: int, slot_of=None, keep=None) -> dict:
    """Token -> expert grouping: a stable sort of the pairs p = t*k + j by expert.

    The result is in (expert, token, j) order. slot_of maps an expert to its
    slot in the expert pool, the indirection that stands for the pages' hot
    expert cache (vramglass.com, section その1：よく使うエキスパートを選んでGPUに置く).
    keep (from kept_pairs) restricts the sort to the kept pairs; a pair left
    out has pair_pos -1.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    cand = np.arange(flat.size) if keep is None else np.nonzero(np.asarray(keep).reshape(-1))[0]
    order = cand[np.argsort(flat[cand], kind="stable")]
    count = np.bincount(flat[cand], minlength=E)
    offset = np.concatenate([[0], np.cumsum(count)])
    pos = np.full(flat.size, -1, dtype=np.int64)
    pos[order] = np.arange(order.size)
    uniq = np.nonzero(count)[0]
    g = {
        "expert_count": count.astype(np.int32),
        "expert_offset": offset.astype(np.int32),
        "pair_token": (order // k).astype(np.int32),
        "pair_j": (order % k).astype(np.int32),
        "pair_gate": np.asarray(gate, dtype=np.float64).reshape(-1)[order],
        "pair_pos": pos.astype(np.int32).reshape(T, k),
        "uniq_expert": uniq.astype(np.int32),
        "n_uniq": int(uniq.size),
    }
    if slot_of is not None:
        g["uniq_slot"] = np.asarray(slot_of, dtype=np.int32)[uniq]
    return g


# ------------------------------------------------------------------ expert FFN

def silu(z):
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_forward(xd: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray) -> np.ndarray:
    """SwiGLU expert: z = W_d (silu(W_g x) * (W_u x)); xd may be [d] or [n, d]."""
    x2 = np.atleast_2d(xd)
    h = silu(x2 @ wg.T) * (x2 @ wu.T)
    z = h @ wd.T
    return z if np.ndim(xd) == 2 else z[0]


class ExpertCache:
    """Dequantised expert weights, keyed by an id, built on first use."""

    def __init__(self, load, d, f, bits):
        self.load, self.d, self.f, self.bits = load, d, f, bits
        self.cache = {}

    def __call__(self, key):
        if key not in self.cache:
            self.cache[key] = expert_weights(self.load(key), self.d, self.f, self.bits)
        return self.cache[key]


def kept_pairs(idx: np.ndarray, slot_of, skip_from: int, hot_slots: int) -> np.ndarray:
    """Which (token, j) pairs a step that skips low-ranked non-resident
    experts keeps: all when skip_from == 0; else pair (t, j) is left out when
    j >= skip_from and its expert's slot is >= hot_slots. The pages' engine
    leaves out low-ranked experts that are not in GPU memory (news.blueqat.app
    /post/3262, section どう見るか); "low-ranked" is read as rank >= skip_from
    of the token's k, "not in GPU memory" as a slot outside the hot set, and
    the remaining gates keep their values. Independently of skipping, a pair
    whose expert has slot -1 (not held by this device, the expert-parallel
    split) is left out."""
    keep = np.ones(idx.shape, dtype=bool)
    if slot_of is not None:
        slots = np.asarray(slot_of)[idx]
        keep &= slots != -1
        if skip_from:
            keep[:, skip_from:] &= slots[:, skip_from:] < hot_slots
    return keep


def layer_forward(x_bits, w_router, k, experts, shared=None, bias=None, renorm=True,
                  residual=False, tokens=None, skip_from=0, hot_slots=0, slot_of=None):
    """One MoE layer in fp64.

    experts(e) -> (W_g, W_u, W_d) of routed expert e; shared -> the shared
    expert's triple or None. Each token's 10 routed experts plus the shared one
    are summed as y = sum_j g_j z_j + z_shared (the pages split exactly these
    experts of each layer between GPU and CPU and wait for both before the next
    layer: vramglass.com, section その2：GPUとCPUで同時に計算する).
    residual=True returns x + y. `tokens` restricts the FFN to a subset of the
    tokens (routing is still computed for all). skip_from > 0 leaves out the
    pairs kept_pairs() drops (slot_of: the layer's slot table).
    Returns dict(logits, idx, gate, y, keep) with y fp64 [len(tokens), d].
    """
    l, idx, g = route(x_bits, w_router, k, bias, renorm)
    keep = kept_pairs(idx, slot_of, skip_from, hot_slots)
    xd = bf16_to_f64(x_bits)
    toks = range(xd.shape[0]) if tokens is None else tokens
    ys = []
    for t in toks:
        y = np.zeros(xd.shape[1])
        for j in range(k):
            if not keep[t, j]:
                continue
            wg, wu, wd = experts(int(idx[t, j]))
            y = y + g[t, j] * expert_forward(xd[t], wg, wu, wd)
        if shared is not None:
            y = y + expert_forward(xd[t], *shared)
        if residual:
            y = xd[t] + y
        ys.append(y)
    return {"logits": l, "idx": idx, "gate": g, "keep": keep, "y": np.array(ys).reshape(len(ys), xd.shape[1])}
