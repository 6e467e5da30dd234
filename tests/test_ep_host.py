"""Expert-parallel split, host side, on CPU: two gloo ranks each compute
their partial of a layer with the oracle (only their experts: slot -1 marks
the others; the shared expert and the residual on rank 0), all-gather the
partials and sum them in rank order; the sum equals the unsplit layer, and
every rank gets the same bits. Plus the partition itself."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_expert_ffn_router_b200 import ep as EP
from bit_expert_ffn_router_b200 import moe as M
from bit_expert_ffn_router_b200 import synth
from oracle import moe_oracle as O


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed=50):
    cfg = M.TINY.replace(k=3, residual=1)
    d, f, E = cfg.d, cfg.f, cfg.E
    secs = [synth.expert_sections(d, f, cfg.bits, seed + e) for e in range(E)]
    shared = synth.expert_sections(d, f, cfg.bits, seed + 99)
    x = synth.activations(7, d, seed + 1)
    wr = synth.router_weights(E, d, seed + 2)
    slot_of = synth.rng(seed + 3).permutation(E).astype(np.int32)
    return cfg, secs, shared, x, wr, slot_of


def _partial(cfg, secs, shared, x, wr, slot_of, rank, world):
    rc = EP.rank_cfg(cfg, rank)
    cache = O.ExpertCache(lambda e: secs[e], cfg.d, cfg.f, cfg.bits)
    sh = O.expert_weights(shared, cfg.d, cfg.f, cfg.bits) if rc.n_shared else None
    table = EP.rank_slot_table(slot_of, rank, world)
    return O.layer_forward(x, wr, cfg.k, cache, sh, residual=bool(rc.residual), slot_of=table)["y"]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, secs, shared, x, wr, slot_of = _layer()
        part = torch.from_numpy(_partial(cfg, secs, shared, x, wr, slot_of, rank, world))
        parts = [torch.empty_like(part) for _ in range(world)]
        dist.all_gather(parts, part)
        q.put((rank, EP.combine_partials(parts).numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_to_the_unsplit_layer():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    assert np.array_equal(got[0], got[1])  # the same bits on every rank
    cfg, secs, shared, x, wr, slot_of = _layer()
    cache = O.ExpertCache(lambda e: secs[e], cfg.d, cfg.f, cfg.bits)
    full = O.layer_forward(x, wr, cfg.k, cache, O.expert_weights(shared, cfg.d, cfg.f, cfg.bits), residual=True)
    assert np.allclose(got[0], full["y"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_partition_covers_every_expert_once(world):
    E = 512
    masks = np.stack([EP.held(E, r, world) for r in range(world)])
    assert np.array_equal(masks.sum(axis=0), np.ones(E))
    # interleaved: a Zipf-shaped load (rank of popularity = expert index) spreads within one expert per rank
    counts = masks.sum(axis=1)
    assert counts.max() - counts.min() <= 1
    slot_of = np.arange(E, dtype=np.int32)[::-1].copy()
    for r in range(world):
        t = EP.rank_slot_table(slot_of, r, world)
        assert np.array_equal(t[masks[r]], slot_of[masks[r]]) and np.all(t[~masks[r]] == EP.SLOT_ABSENT)
    assert EP.rank_cfg(M.FULL.replace(residual=1, out_fp32=0), 1).n_shared == 0


def test_oracle_leaves_out_absent_experts():
    cfg, secs, shared, x, wr, slot_of = _layer(seed=60)
    table = slot_of.copy()
    table[::2] = -1
    cache = O.ExpertCache(lambda e: secs[e], cfg.d, cfg.f, cfg.bits)
    part = O.layer_forward(x, wr, cfg.k, cache, None, slot_of=table)
    full = O.layer_forward(x, wr, cfg.k, cache, None)
    xd = O.bf16_to_f64(x)
    for t in range(x.shape[0]):
        want = sum(full["gate"][t, j] * O.expert_forward(xd[t], *cache(int(e)))
                   for j, e in enumerate(full["idx"][t]) if e % 2 == 1)
        assert np.allclose(part["y"][t], want, rtol=1e-12, atol=1e-13)
