"""GPU parity of moe_stack_forward: L chained decode layers in one launch.

Each layer has its own router, Zipf bias, shared expert and slot-table row
over one pool of expert records. The oracle runs layer by layer on the
GPU's own bf16 input of that layer (x for layer 0, y[l-1] after), so every
layer is compared with its plain definition: routing bit-exactly (except at
fp64 near-ties), output within 2e-3 per token plus one bf16 ulp. The stack
must also give the same bits as L single-layer calls chained by hand."""
import numpy as np
import pytest
import torch

from bit_expert_ffn_router_b200 import moe as M
from bit_expert_ffn_router_b200 import synth
from oracle import moe_oracle as O

from tests import harness as H
from tests.test_routing_gpu import check_published_routing

pytestmark = pytest.mark.gpu


class Stack:
    def __init__(self, cfg, L, T, seed, zipf=True):
        self.cfg, self.L, self.T, self.seed = cfg, L, T, seed
        d, f, E, k, bits = cfg.d, cfg.f, cfg.E, cfg.k, cfg.bits
        self.n_slots = E + 3
        self.sections = [synth.expert_sections(d, f, bits, seed + 100 + s) for s in range(self.n_slots)]
        self.shared = [synth.expert_sections(d, f, bits, seed + 50 + l) for l in range(L)] if cfg.n_shared else None
        self.wr = np.stack([synth.router_weights(E, d, seed + 1000 * l + 1) for l in range(L)])
        self.bias = (np.stack([synth.bias_from_sets(synth.zipf_sets(T, E, k, seed + 1000 * l + 2), E)
                               for l in range(L)]) if zipf else None)
        self.slot_of = np.stack([synth.rng(seed + 1000 * l + 3).permutation(self.n_slots)[:E]
                                 for l in range(L)]).astype(np.int32)
        self.x = synth.activations(T, d, seed + 7)
        pool, self.stride = M.place_records(cfg, self.sections)
        shared = M.place_records(cfg, self.shared, stride=self.stride)[0] if self.shared else None
        self.dev = {
            "x": torch.from_numpy(self.x.view(np.int16)).cuda(),
            "wr": torch.from_numpy(self.wr).cuda(),
            "bias": None if self.bias is None else torch.from_numpy(self.bias).cuda(),
            "slot_of": torch.from_numpy(self.slot_of).cuda(),
            "pool": pool, "shared": shared,
        }

    def out(self, L=None):
        dt = torch.float32 if self.cfg.out_fp32 else torch.bfloat16
        return torch.empty(L or self.L, self.T, self.cfg.d, dtype=dt, device="cuda")

    def forward(self):
        dv = self.dev
        ws = M.stack_workspace(self.cfg, self.L, self.T)
        y = self.out()
        H.ctx().stack_forward(self.cfg, self.L, dv["x"], self.T, dv["wr"], dv["bias"], dv["slot_of"], self.n_slots,
                              dv["pool"], self.stride, dv["shared"], ws, y)
        return y, ws

    def layer_view(self, l, x_bits):
        """Layer l as a harness Layer (for the oracle and the routing checks) on input x_bits."""
        L = H.Layer.__new__(H.Layer)
        L.cfg, L.T, L.seed = self.cfg, self.T, self.seed
        L.x = x_bits
        L.wr = self.wr[l]
        L.bias = None if self.bias is None else self.bias[l]
        L.sections = [self.sections[s] for s in self.slot_of[l]]
        L.shared = self.shared[l] if self.shared else None
        L.n_slots = self.n_slots
        L.slot_of = self.slot_of[l]
        L._dev = None
        return L


def _bits(y_l):
    return y_l.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 4])
def test_stack_matches_oracle_layer_by_layer(bits, T):
    cfg = M.FULL.replace(bits=bits, out_fp32=0, residual=1)
    st = Stack(cfg, 3, T, seed=300 + 10 * bits + T)
    y, ws = st.forward()
    torch.cuda.synchronize()
    assert H.ctx().check_device_status() == M.OK
    x = st.x
    for l in range(st.L):
        Lv = st.layer_view(l, x)
        r = {k: v.cpu().numpy() for k, v in H.ctx().layer_routing(cfg, T, ws, stack_layers=st.L, layer=l).items()}
        check_published_routing(Lv, ws_routing=r)
        H.assert_close_rows(H.y_as_f64(y[l]), Lv.oracle()["y"], bf16=True)
        x = _bits(y[l])


@pytest.mark.parametrize("bits", [2, 3])
def test_stack_equals_chained_single_layer_calls(bits):
    """One launch of L layers gives the bits of L moe_layer_forward calls."""
    cfg = M.FULL.replace(bits=bits, out_fp32=0, residual=1)
    st = Stack(cfg, 4, 2, seed=400 + bits)
    y, _ = st.forward()
    dv = st.dev
    x = dv["x"]
    ws1 = M.workspace(cfg, st.T)
    for l in range(st.L):
        y1 = torch.empty(st.T, cfg.d, dtype=torch.bfloat16, device="cuda")
        H.ctx().layer_forward(cfg, x, st.T, dv["wr"][l], None if dv["bias"] is None else dv["bias"][l],
                              dv["slot_of"][l], st.n_slots, dv["pool"], st.stride, dv["shared"][l], ws1, y1)
        assert torch.equal(y1, y[l]), l
        x = y1.view(torch.int16)
    y2, _ = st.forward()  # and the same launch again: the same bits
    assert torch.equal(y, y2)
    assert H.ctx().check_device_status() == M.OK


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_stack_tiny_many_layers(bits, T):
    cfg = M.TINY.replace(bits=bits, out_fp32=0, residual=1)
    st = Stack(cfg, 8, T, seed=500 + T, zipf=False)
    y, ws = st.forward()
    torch.cuda.synchronize()
    assert H.ctx().check_device_status() == M.OK
    x = st.x
    for l in range(st.L):
        Lv = st.layer_view(l, x)
        r = {k: v.cpu().numpy() for k, v in H.ctx().layer_routing(cfg, T, ws, stack_layers=st.L, layer=l).items()}
        check_published_routing(Lv, ws_routing=r)
        H.assert_close_rows(H.y_as_f64(y[l]), Lv.oracle()["y"], bf16=True)
        x = _bits(y[l])


def test_stack_without_residual_or_shared():
    cfg = M.TINY.replace(out_fp32=0, n_shared=0)
    st = Stack(cfg, 3, 2, seed=600)
    y, _ = st.forward()
    torch.cuda.synchronize()
    x = st.x
    for l in range(st.L):
        H.assert_close_rows(H.y_as_f64(y[l]), st.layer_view(l, x).oracle()["y"], bf16=True)
        x = _bits(y[l])


def test_stack_argument_errors():
    cfg = M.TINY.replace(out_fp32=0)
    st = Stack(cfg, 2, 2, seed=601)
    dv = st.dev
    ws = M.stack_workspace(cfg, 2, 2)
    c = H.ctx()
    args = dict(cfg=cfg, L=2, x=dv["x"], T=2, w_router=dv["wr"], bias=dv["bias"], slot_of=dv["slot_of"],
                n_slots=st.n_slots, pool=dv["pool"], stride=st.stride, shared=dv["shared"], ws=ws, y=st.out())
    assert c.stack_forward_status(**args) == M.OK
    assert c.stack_forward_status(**{**args, "cfg": cfg.replace(out_fp32=1), "y": st.out().float()}) == M.EINVAL
    assert c.stack_forward_status(**{**args, "T": 9}) == M.EINVAL
    assert c.stack_forward_status(**{**args, "ws": ws[:ws.numel() // 2]}) == M.ENOSPACE
    assert c.stack_forward_status(**{**args, "L": 0}) == M.EINVAL
    assert c.check_device_status() == M.OK


@pytest.mark.parametrize("limit_us", [1, 5, 20])
def test_stack_wait_limits_report_timeout_and_recover(monkeypatch, limit_us):
    """Short wait limits make the stack kernel give up at different points
    (an exchange, a weight stage, the routing of a later layer): every launch
    ends, reports MOE_ETIMEOUT (or finishes), and the same context then gives
    the exact results of an unlimited one."""
    cfg = M.FULL.replace(bits=2, out_fp32=0, residual=1)
    st = Stack(cfg, 3, 4, seed=610)
    ref, _ = st.forward()
    torch.cuda.synchronize()
    dv = st.dev
    monkeypatch.setenv("MOE_TIMEOUT_US", str(limit_us))
    short = M.Context(torch.cuda.current_device())
    monkeypatch.delenv("MOE_TIMEOUT_US")
    ws = M.stack_workspace(cfg, st.L, st.T)
    seen = set()
    for _ in range(4):
        y = st.out()
        assert short.stack_forward_status(cfg, st.L, dv["x"], st.T, dv["wr"], dv["bias"], dv["slot_of"], st.n_slots,
                                          dv["pool"], st.stride, dv["shared"], ws, y) == M.OK
        s = short.check_device_status()
        assert s in (M.OK, M.ETIMEOUT)
        seen.add(s)
        assert short.check_device_status() == M.OK
        if s == M.OK:
            assert torch.equal(y, ref)
    if limit_us == 1:
        assert M.ETIMEOUT in seen
    short.close()
    y2, _ = st.forward()
    torch.cuda.synchronize()
    assert torch.equal(y2, ref)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 4])
def test_stack_leaves_out_low_ranked_non_resident_pairs(bits, T):
    """skip_from / hot_slots: every layer against the oracle that leaves the
    same pairs out (routing views of the kept pairs, outputs within the usual
    bound); with every slot resident the bits equal the plain stack's."""
    base = M.FULL.replace(bits=bits, out_fp32=0, residual=1)
    st = Stack(base, 3, T, seed=740 + 10 * bits + T)
    plain, _ = st.forward()
    st.cfg = base.replace(skip_from=4, hot_slots=st.n_slots)
    same, _ = st.forward()
    torch.cuda.synchronize()
    assert torch.equal(same, plain)
    cfg = base.replace(skip_from=4, hot_slots=st.n_slots // 2)
    st.cfg = cfg
    y, ws = st.forward()
    torch.cuda.synchronize()
    assert H.ctx().check_device_status() == M.OK
    x = st.x
    dropped = 0
    for l in range(st.L):
        Lv = st.layer_view(l, x)
        r = {k: v.cpu().numpy() for k, v in H.ctx().layer_routing(cfg, T, ws, stack_layers=st.L, layer=l).items()}
        check_published_routing(Lv, ws_routing=r)
        ref = Lv.oracle()
        dropped += int((~ref["keep"]).sum())
        H.assert_close_rows(H.y_as_f64(y[l]), ref["y"], bf16=True)
        x = _bits(y[l])
    assert dropped > 0
    assert not torch.equal(y, plain)
