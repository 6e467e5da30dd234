"""GPU checks of the residency calls: moe_usage_count tallies exactly the
pairs the routing record holds, per layer and accumulated; moe_slot_swap
exchanges exactly the named records and table entries, leaves every later
result bit-for-bit unchanged, and rejects or reports bad input."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_router_b200 import moe as M
from bit_expert_ffn_router_b200 import residency as R

from tests import harness as H
from tests.test_stack_gpu import Stack

pytestmark = pytest.mark.gpu


def _routed_counts(ctx, cfg, st, ws):
    out = np.zeros(st.L * cfg.E, dtype=np.int64)
    for l in range(st.L):
        idx = ctx.layer_routing(cfg, st.T, ws, stack_layers=st.L, layer=l)["idx"].cpu().numpy()
        np.add.at(out, l * cfg.E + idx.reshape(-1), 1)
    return out


@pytest.mark.parametrize("T", [1, 4])
def test_usage_count_matches_the_routing_and_accumulates(T):
    cfg = M.FULL.replace(bits=2, out_fp32=0, residual=1)
    st = Stack(cfg, 3, T, seed=700 + T)
    y, ws = st.forward()
    torch.cuda.synchronize()
    ctx = H.ctx()
    counts = torch.zeros(st.L * cfg.E, dtype=torch.int32, device="cuda")
    ctx.usage_count(cfg, st.L, T, ws, counts)
    ctx.usage_count(cfg, st.L, T, ws, counts)
    torch.cuda.synchronize()
    want = _routed_counts(ctx, cfg, st, ws)
    assert np.array_equal(counts.cpu().numpy(), 2 * want)
    assert int(want.sum()) == st.L * T * cfg.k
    assert ctx.check_device_status() == M.OK


def test_usage_count_on_a_single_layer_workspace():
    L = H.Layer(M.FULL, 40, seed=710, zipf=True)  # prefill path
    y, ws = L.forward()
    torch.cuda.synchronize()
    ctx = H.ctx()
    counts = torch.zeros(M.FULL.E, dtype=torch.int32, device="cuda")
    ctx.usage_count(M.FULL, 1, 40, ws, counts)
    idx = ctx.layer_routing(M.FULL, 40, ws)["idx"].cpu().numpy()
    assert np.array_equal(counts.cpu().numpy(), np.bincount(idx.reshape(-1), minlength=M.FULL.E))


def _one_record_per_entry(st, seed):
    """Re-homes a Stack on a pool with one record per (layer, expert) entry
    behind a random permutation table (as the bench's pool), so that distinct
    entries always name distinct slots."""
    dv = st.dev
    old = dv["slot_of"].cpu().numpy().reshape(-1)
    n = old.size
    perm = np.random.default_rng(seed).permutation(n)
    pool = torch.empty(n, st.stride, dtype=torch.uint8, device="cuda")
    pool[torch.from_numpy(perm).cuda()] = dv["pool"][torch.from_numpy(old.astype(np.int64)).cuda()]
    dv["pool"] = pool
    dv["slot_of"] = torch.from_numpy(perm.astype(np.int32).reshape(st.L, -1)).cuda()
    st.n_slots = n


@pytest.mark.parametrize("cfg", [M.TINY.replace(out_fp32=0), M.FULL.replace(bits=3, out_fp32=0, residual=1)],
                         ids=["tiny", "full-q3"])
def test_slot_swap_moves_records_and_entries_and_keeps_results_bitwise(cfg):
    st = Stack(cfg, 3, 4, seed=720)
    ref0, _ = st.forward()
    _one_record_per_entry(st, 5)
    ref, _ = st.forward()
    torch.cuda.synchronize()
    assert torch.equal(ref, ref0)  # the slot assignment does not enter the results
    ctx = H.ctx()
    dv = st.dev
    table = dv["slot_of"].view(-1)
    pool_before = dv["pool"].clone()
    table_before = table.cpu().numpy().copy()
    rng = np.random.default_rng(3)
    m = min(150, table.numel() // 2)
    ent = rng.permutation(table.numel())[:2 * m].astype(np.int32)
    a, b = ent[:m], ent[m:]
    ctx.slot_swap(cfg, dv["pool"], st.stride, table, st.n_slots, a, b)
    torch.cuda.synchronize()
    assert ctx.check_device_status() == M.OK
    after = table.cpu().numpy()
    assert np.array_equal(after, R.apply_swaps(table_before, a, b))
    # every entry reaches its own record; slots no pair names are untouched
    for i in range(table.numel()):
        assert torch.equal(dv["pool"][after[i]], pool_before[table_before[i]])
    y2, _ = st.forward()
    torch.cuda.synchronize()
    assert torch.equal(y2, ref)


def test_slot_swap_argument_checks_and_device_bad_slot():
    cfg = M.TINY.replace(out_fp32=0)
    st = Stack(cfg, 2, 2, seed=730)
    ctx = H.ctx()
    dv = st.dev
    table = dv["slot_of"].view(-1)
    n = table.numel()
    ok = ctx.slot_swap_status(cfg, dv["pool"], st.stride, table, st.n_slots, [0], [1])
    assert ok == M.OK
    assert ctx.slot_swap_status(cfg, dv["pool"], st.stride, table, st.n_slots, [0, 2], [1, 0]) == M.EINVAL
    assert ctx.slot_swap_status(cfg, dv["pool"], st.stride, table, st.n_slots, [n], [0]) == M.EINVAL
    assert ctx.slot_swap_status(cfg, dv["pool"], st.stride, table, st.n_slots, [], []) == M.OK
    assert ctx.slot_swap_status(cfg, dv["pool"], st.stride + 16, table, st.n_slots, [0], [1]) == M.EINVAL
    torch.cuda.synchronize()
    assert ctx.check_device_status() == M.OK
    # a table entry outside the pool: the kernel reports it and leaves the pair alone
    saved = table[3].item()
    table[3] = st.n_slots
    before = dv["pool"].clone()
    assert ctx.slot_swap_status(cfg, dv["pool"], st.stride, table, st.n_slots, [3], [4]) == M.OK
    assert ctx.check_device_status() == M.EDEVICE
    assert torch.equal(dv["pool"], before)
    assert table[3].item() == st.n_slots
    table[3] = saved
    torch.cuda.synchronize()
    assert ctx.check_device_status() == M.OK
