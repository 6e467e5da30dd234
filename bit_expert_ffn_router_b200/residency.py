"""Hot-set policy over a slot table.

The pages' engine keeps the experts it uses most in GPU memory, chosen from
usage statistics and swapped as a conversation goes on (vramglass.com,
section その1：よく使うエキスパートを選んでGPUに置く; news.blueqat.app/post/3262,
section GPU・CPU・RAM・SSDの分担). Here the hot set is the pool's first n_hot
slots: plan_swaps picks which slot-table entries trade slots so that the
n_hot most used experts sit there, and Context.slot_swap carries the trades
out on the device (moe_slot_swap). Host logic only."""
from __future__ import annotations

import numpy as np


def hot_order(counts) -> np.ndarray:
    """Entries by descending count, ties to the lower entry index."""
    counts = np.asarray(counts, dtype=np.int64).ravel()
    return np.lexsort((np.arange(counts.size), -counts))


def plan_swaps(counts, slot_of, n_hot: int, max_swaps: int | None = None):
    """Exchanges that bring the n_hot most used entries into slots [0, n_hot).

    counts, slot_of: host integer arrays over the same flat entries (layer * E
    + expert). Returns (a, b) int32: entry a[i], wanted but outside the hot
    slots, trades slots with entry b[i], the least used occupant of a hot slot
    that is not wanted, and only while the newcomer's count is the larger one
    (so the set the table starts from, e.g. one seeded from popularity, stays
    until observed usage beats it). The most used newcomers go first; at most
    max_swaps pairs. All 2n entries are distinct."""
    counts = np.asarray(counts, dtype=np.int64).ravel()
    slot_of = np.asarray(slot_of).ravel()
    if counts.shape != slot_of.shape:
        raise ValueError("counts and slot_of must cover the same entries")
    want = hot_order(counts)[:n_hot]
    hot = slot_of < n_hot
    incoming = want[~hot[want]]
    wanted = np.zeros(counts.size, dtype=bool)
    wanted[want] = True
    leaving = np.nonzero(hot & ~wanted)[0]
    leaving = leaving[np.lexsort((leaving, counts[leaving]))]  # least used first, then lower index
    n = min(incoming.size, leaving.size)
    beats = counts[incoming[:n]] > counts[leaving[:n]]
    n = int(np.argmin(beats)) if not beats.all() else n  # the prefix where the newcomer is used more
    if max_swaps is not None:
        n = min(n, max_swaps)
    return incoming[:n].astype(np.int32), leaving[:n].astype(np.int32)


def apply_swaps(slot_of, a, b) -> np.ndarray:
    """The slot table after the exchanges (what moe_slot_swap does to it)."""
    out = np.array(slot_of, copy=True).ravel()
    a = np.asarray(a, dtype=np.int64)
    b = np.asarray(b, dtype=np.int64)
    out[a], out[b] = out[b], out[a].copy()
    return out


def hot_hit_rate(experts_by_layer, slot_of, E: int, n_hot: int) -> float:
    """Share of routed (token, j) pairs whose expert sits in a hot slot.
    experts_by_layer: list of int arrays (the routed experts of layer l)."""
    slot_of = np.asarray(slot_of).ravel()
    hits = total = 0
    for l, ex in enumerate(experts_by_layer):
        ex = np.asarray(ex, dtype=np.int64).ravel()
        hits += int((slot_of[l * E + ex] < n_hot).sum())
        total += ex.size
    return hits / max(total, 1)
