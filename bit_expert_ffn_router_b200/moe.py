"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every step of the MoE FFN runs inside libmoe's CUDA kernels; this module turns
torch tensors into device pointers and the current torch stream into a
cudaStream_t. If libmoe.so is missing, loading fails with an error: there is
no fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libmoe.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT, EDEVICE, ENOSPACE = range(7)
DECODE_MAX_T = 8


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_string(status)} ({status})"
        if status == ECUDA:
            msg += f" [{load_library().moe_last_cuda_error().decode()}]"
        super().__init__(msg)


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("d", "f", "E", "k", "n_shared", "bits", "block", "renorm", "out_fp32", "residual",
                 "skip_from", "hot_slots")]


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("gu_codes", "dn_codes", "gu_scales", "dn_scales", "bytes")]


class Grouping(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("k", ctypes.c_int), ("E", ctypes.c_int),
                ("n_pairs", ctypes.c_int), ("n_rows", ctypes.c_int)] + [
        (n, ctypes.c_void_p) for n in
        ("expert_count", "expert_offset", "pair_token", "pair_j", "pair_gate", "pair_slot", "pair_pos",
         "uniq_expert", "uniq_slot", "uniq_offset", "n_uniq", "internal")]


class Routing(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("k", ctypes.c_int), ("E", ctypes.c_int),
                ("logits", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("gate", ctypes.c_void_p),
                ("grouping", Grouping)]


@dataclasses.dataclass(frozen=True)
class LayerCfg:
    d: int
    f: int
    E: int
    k: int
    n_shared: int = 1
    bits: int = 2
    block: int = 32
    renorm: int = 1
    out_fp32: int = 1
    residual: int = 0
    skip_from: int = 0  # 0: off; else pairs of rank >= skip_from on a slot >= hot_slots are left out (decode)
    hot_slots: int = 0

    def c(self) -> _Cfg:
        return _Cfg(*(getattr(self, f.name) for f in dataclasses.fields(self)))

    def replace(self, **kw) -> "LayerCfg":
        return dataclasses.replace(self, **kw)


# Named shapes: the tiny parity layer and the full Qwen3.8-Flash-Next-shaped layer.
TINY = LayerCfg(d=256, f=128, E=16, k=2)
FULL = LayerCfg(d=2048, f=768, E=512, k=10)

_P, _I, _Z, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
_SIGS = {
    "moe_ctx_create": (_I, [_I, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_ctx_destroy": (None, [_P]),
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_check_device_status": (_I, [_P, _S]),
    "moe_last_device_error_detail": (_I, [_P]),
    "moe_trace_fetch": (_I, [_P, ctypes.c_void_p, _I, _S]),
    "moe_expert_layout_get": (_I, [ctypes.POINTER(_Cfg), ctypes.POINTER(_Layout)]),
    "moe_workspace_bytes": (_Z, [ctypes.POINTER(_Cfg), _I]),
    "moe_router_topk": (_I, [_P, ctypes.POINTER(_Cfg), _P, _P, _P, _I, _P, _P, _P, _S]),
    "moe_topk": (_I, [_P, ctypes.POINTER(_Cfg), _P, _I, _P, _P, _S]),
    "moe_group_tokens": (_I, [_P, ctypes.POINTER(_Cfg), _P, _P, _I, _P, _I, _P, _Z,
                              ctypes.POINTER(Grouping), _S]),
    "moe_expert_ffn_q2": (_I, [_P, ctypes.POINTER(_Cfg), _P, ctypes.POINTER(Grouping), _P, _Z, _P, _P, _Z,
                               _P, _P, _S]),
    "moe_expert_ffn_q3": (_I, [_P, ctypes.POINTER(_Cfg), _P, ctypes.POINTER(Grouping), _P, _Z, _P, _P, _Z,
                               _P, _P, _S]),
    "moe_combine": (_I, [_P, ctypes.POINTER(_Cfg), ctypes.POINTER(Grouping), _P, _P, _I, _P, _S]),
    "moe_layer_forward": (_I, [_P, ctypes.POINTER(_Cfg), _P, _I, _P, _P, _P, _I, _P, _Z, _P, _P, _Z, _P,
                               _S]),
    "moe_layer_routing": (_I, [ctypes.POINTER(_Cfg), _I, _P, _Z, ctypes.POINTER(Routing)]),
    "moe_stack_workspace_bytes": (_Z, [ctypes.POINTER(_Cfg), _I, _I]),
    "moe_stack_forward": (_I, [_P, ctypes.POINTER(_Cfg), _I, _P, _I, _P, _P, _P, _I, _P, _Z, _P, _P, _Z, _P, _S]),
    "moe_stack_routing": (_I, [ctypes.POINTER(_Cfg), _I, _I, _P, _Z, _I, ctypes.POINTER(Routing)]),
    "moe_layer_forward_static": (_I, [_P, ctypes.POINTER(_Cfg), _P, _I, _P, _P, _P, _I, _P, _Z, _P, _P, _S]),
    "moe_usage_count": (_I, [_P, ctypes.POINTER(_Cfg), _I, _I, _P, _Z, _P, _S]),
    "moe_slot_swap": (_I, [_P, ctypes.POINTER(_Cfg), _P, _Z, _P, _I, _I, _P, _P, _I, _S]),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Opens libmoe.so (built in-tree by bit_expert_ffn_router_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: build it with `python -m bit_expert_ffn_router_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load_library().moe_status_string(s).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise MoeError(status, what)


def expert_layout(cfg: LayerCfg) -> dict:
    lay = _Layout()
    _check(load_library().moe_expert_layout_get(ctypes.byref(cfg.c()), ctypes.byref(lay)), "moe_expert_layout_get")
    return {n: getattr(lay, n) for n, _ in _Layout._fields_}


def workspace_bytes(cfg: LayerCfg, T: int) -> int:
    return int(load_library().moe_workspace_bytes(ctypes.byref(cfg.c()), T))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Context:
    """One libmoe context (device status word + SM count) on a CUDA device."""

    def __init__(self, device: int = 0):
        self.lib = load_library()
        h = ctypes.c_void_p()
        _check(self.lib.moe_ctx_create(device, ctypes.byref(h)), "moe_ctx_create")
        self.h = h
        self.device = device

    def close(self):
        if self.h:
            self.lib.moe_ctx_destroy(self.h)
            self.h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- raw entry points (status codes returned, not raised) --------------------
    def router_topk_status(self, cfg, x, w_router, bias, T, logits, idx, gate, stream=None):
        return self.lib.moe_router_topk(self.h, ctypes.byref(cfg.c()), _ptr(x), _ptr(w_router), _ptr(bias), T,
                                        _ptr(logits), _ptr(idx), _ptr(gate), _stream(stream))

    def layer_forward_status(self, cfg, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, y,
                             stream=None):
        return self.lib.moe_layer_forward(self.h, ctypes.byref(cfg.c()), _ptr(x), T, _ptr(w_router), _ptr(bias),
                                          _ptr(slot_of), n_slots, _ptr(pool), stride, _ptr(shared), _ptr(ws),
                                          0 if ws is None else ws.numel() * ws.element_size(), _ptr(y),
                                          _stream(stream))

    def stack_forward_status(self, cfg, L, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, y,
                             stream=None):
        return self.lib.moe_stack_forward(self.h, ctypes.byref(cfg.c()), L, _ptr(x), T, _ptr(w_router), _ptr(bias),
                                          _ptr(slot_of), n_slots, _ptr(pool), stride, _ptr(shared), _ptr(ws),
                                          0 if ws is None else ws.numel() * ws.element_size(), _ptr(y),
                                          _stream(stream))

    def stack_forward(self, cfg, L, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, y,
                      stream=None):
        """moe_stack_forward: L chained decode layers in one launch (layer l + 1 reads y[l])."""
        _check(self.stack_forward_status(cfg, L, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws,
                                         y, stream), "moe_stack_forward")

    def layer_forward_static_status(self, cfg, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, y,
                                    stream=None):
        """moe_layer_forward with the library's static scratch (no workspace argument)."""
        return self.lib.moe_layer_forward_static(self.h, ctypes.byref(cfg.c()), _ptr(x), T, _ptr(w_router),
                                                 _ptr(bias), _ptr(slot_of), n_slots, _ptr(pool), stride,
                                                 _ptr(shared), _ptr(y), _stream(stream))

    # -- checked wrappers ---------------------------------------------------------
    def router_topk(self, cfg, x, w_router, bias, T, logits, idx, gate, stream=None):
        _check(self.router_topk_status(cfg, x, w_router, bias, T, logits, idx, gate, stream), "moe_router_topk")

    def topk(self, cfg, logits, T, idx, gate, stream=None):
        _check(self.lib.moe_topk(self.h, ctypes.byref(cfg.c()), _ptr(logits), T, _ptr(idx), _ptr(gate),
                                 _stream(stream)), "moe_topk")

    def group_tokens(self, cfg, idx, gate, T, slot_of, n_slots, ws, stream=None) -> Grouping:
        g = Grouping()
        _check(self.lib.moe_group_tokens(self.h, ctypes.byref(cfg.c()), _ptr(idx), _ptr(gate), T, _ptr(slot_of),
                                         n_slots, _ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(g),
                                         _stream(stream)), "moe_group_tokens")
        return g

    def expert_ffn(self, cfg, x, grouping, pool, stride, shared, ws, z_rows=None, y=None, stream=None):
        fn = self.lib.moe_expert_ffn_q2 if cfg.bits == 2 else self.lib.moe_expert_ffn_q3
        _check(fn(self.h, ctypes.byref(cfg.c()), _ptr(x), ctypes.byref(grouping), _ptr(pool), stride, _ptr(shared),
                  _ptr(ws), ws.numel() * ws.element_size(), _ptr(z_rows), _ptr(y), _stream(stream)),
               f"moe_expert_ffn_q{cfg.bits}")

    def combine(self, cfg, grouping, z_rows, x, T, y, stream=None):
        _check(self.lib.moe_combine(self.h, ctypes.byref(cfg.c()), ctypes.byref(grouping), _ptr(z_rows), _ptr(x),
                                    T, _ptr(y), _stream(stream)), "moe_combine")

    def layer_forward(self, cfg, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, y,
                      stream=None):
        _check(self.layer_forward_status(cfg, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, y,
                                         stream), "moe_layer_forward")

    def prepare_layer_forward(self, cfg, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws,
                              stream=None) -> "PreparedLayer":
        """moe_layer_forward with every argument but x and y marshalled once (for launch loops)."""
        return PreparedLayer(self, cfg, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, stream)

    def usage_count_status(self, cfg, L, T, ws, counts, stream=None) -> int:
        return self.lib.moe_usage_count(self.h, ctypes.byref(cfg.c()), L, T, _ptr(ws),
                                        ws.numel() * ws.element_size(), _ptr(counts), _stream(stream))

    def usage_count(self, cfg, L, T, ws, counts, stream=None) -> None:
        """moe_usage_count: counts [L*E] int32 (device) += pairs routed to each expert by the call that
        used ws (L = 1 for a single-layer workspace)."""
        _check(self.usage_count_status(cfg, L, T, ws, counts, stream), "moe_usage_count")

    def slot_swap_status(self, cfg, pool, stride, slot_of, n_slots, a, b, stream=None) -> int:
        import numpy as np
        a = np.ascontiguousarray(a, dtype=np.int32)
        b = np.ascontiguousarray(b, dtype=np.int32)
        if a.shape != b.shape or a.ndim != 1:
            return EINVAL
        return self.lib.moe_slot_swap(self.h, ctypes.byref(cfg.c()), _ptr(pool), stride, _ptr(slot_of),
                                      slot_of.numel(), n_slots, a.ctypes.data, b.ctypes.data, a.size,
                                      _stream(stream))

    def slot_swap(self, cfg, pool, stride, slot_of, n_slots, a, b, stream=None) -> None:
        """moe_slot_swap: the records at slots slot_of[a[i]] and slot_of[b[i]] trade places, and so
        do the two table entries (a, b: host index arrays into the flat device table slot_of)."""
        _check(self.slot_swap_status(cfg, pool, stride, slot_of, n_slots, a, b, stream), "moe_slot_swap")

    def layer_routing(self, cfg, T, ws, stack_layers=None, layer=0) -> dict:
        """The routing a whole-step call with workspace `ws` computed (moe_layer_routing; with
        stack_layers=L, layer `layer` of a moe_stack_forward workspace), as torch views into ws:
        logits [T,E], idx [T,k], gate [T,k] and the grouping arrays. Read them after the call has
        completed on its stream."""
        import torch
        r = Routing()
        nbytes = ws.numel() * ws.element_size()
        if stack_layers is None:
            _check(self.lib.moe_layer_routing(ctypes.byref(cfg.c()), T, _ptr(ws), nbytes, ctypes.byref(r)),
                   "moe_layer_routing")
        else:
            _check(self.lib.moe_stack_routing(ctypes.byref(cfg.c()), stack_layers, T, _ptr(ws), nbytes, layer,
                                              ctypes.byref(r)), "moe_stack_routing")
        raw = ws.view(torch.uint8).view(-1)
        base = ws.data_ptr()

        def view(ptr, n, dtype):
            off = ptr - base
            return raw[off:off + 4 * n].view(dtype)

        g = r.grouping
        n_pairs, nu_max = T * cfg.k, min(T * cfg.k, cfg.E)
        return {
            "logits": view(r.logits, T * cfg.E, torch.float32).view(T, cfg.E),
            "idx": view(r.idx, T * cfg.k, torch.int32).view(T, cfg.k),
            "gate": view(r.gate, T * cfg.k, torch.float32).view(T, cfg.k),
            "expert_count": view(g.expert_count, cfg.E, torch.int32),
            "expert_offset": view(g.expert_offset, cfg.E + 1, torch.int32),
            "pair_token": view(g.pair_token, n_pairs, torch.int32),
            "pair_j": view(g.pair_j, n_pairs, torch.int32),
            "pair_gate": view(g.pair_gate, n_pairs, torch.float32),
            "pair_slot": view(g.pair_slot, n_pairs, torch.int32),
            "pair_pos": view(g.pair_pos, n_pairs, torch.int32),
            "uniq_expert": view(g.uniq_expert, nu_max, torch.int32),
            "uniq_slot": view(g.uniq_slot, nu_max, torch.int32),
            "uniq_offset": view(g.uniq_offset, nu_max + 1, torch.int32),
            "n_uniq": view(g.n_uniq, 1, torch.int32),
        }

    def prepare_stack_forward(self, cfg, L, T, w_router, slot_of, n_slots, pool, stride, shared, ws,
                              stream=None) -> "PreparedStack":
        """moe_stack_forward with every argument but x, the bias and y marshalled once (for launch loops)."""
        return PreparedStack(self, cfg, L, T, w_router, slot_of, n_slots, pool, stride, shared, ws, stream)

    def check_device_status(self, stream=None) -> int:
        return self.lib.moe_check_device_status(self.h, _stream(stream))

    def last_device_error_detail(self) -> int:
        return self.lib.moe_last_device_error_detail(self.h)

    def trace_fetch(self, n_ctas: int, stream=None):
        """Phase timestamps of the last decode-layer launches (MOE_TRACE set at creation)."""
        import numpy as np
        buf = np.zeros((n_ctas, 64), dtype=np.uint64)
        _check(self.lib.moe_trace_fetch(self.h, buf.ctypes.data, buf.size, _stream(stream)), "moe_trace_fetch")
        return buf


class PreparedLayer:
    """A moe_layer_forward call whose layer arguments (configuration, weights,
    slot table, pool, workspace, stream) are converted to ctypes values once;
    each call marshals only x and y. It passes exactly the arguments
    Context.layer_forward_status would, and keeps the tensors it points into
    alive."""

    def __init__(self, ctx, cfg, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, stream=None):
        self._fn = ctx.lib.moe_layer_forward
        self._cfg = cfg.c()
        self._keep = (ctx, w_router, bias, slot_of, pool, shared, ws)
        self._head = (ctx.h, ctypes.byref(self._cfg))
        self._mid = (T, _ptr(w_router), _ptr(bias), _ptr(slot_of), n_slots, _ptr(pool), stride, _ptr(shared),
                     _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size())
        self._stream = _stream(stream)

    def status(self, x, y) -> int:
        return self._fn(*self._head, _ptr(x), *self._mid, _ptr(y), self._stream)

    def __call__(self, x, y) -> None:
        _check(self.status(x, y), "moe_layer_forward")


class PreparedStack:
    """A moe_stack_forward call whose fixed arguments (configuration, routers,
    slot table, pool, shared experts, workspace, stream) are converted to
    ctypes values once; each call marshals only x, the bias and y."""

    def __init__(self, ctx, cfg, L, T, w_router, slot_of, n_slots, pool, stride, shared, ws, stream=None):
        self._fn = ctx.lib.moe_stack_forward
        self._cfg = cfg.c()
        self._keep = (ctx, w_router, slot_of, pool, shared, ws)
        self._head = (ctx.h, ctypes.byref(self._cfg), L)
        self._T = T
        self._mid = (_ptr(w_router),)
        self._tail = (_ptr(slot_of), n_slots, _ptr(pool), stride, _ptr(shared), _ptr(ws),
                      ws.numel() * ws.element_size())
        self._stream = _stream(stream)

    def status(self, x, bias, y) -> int:
        return self._fn(*self._head, _ptr(x), self._T, *self._mid, _ptr(bias), *self._tail, _ptr(y), self._stream)

    def __call__(self, x, bias, y) -> None:
        _check(self.status(x, bias, y), "moe_stack_forward")


# ------------------------------------------------------------------ buffers

def workspace(cfg: LayerCfg, T: int, device="cuda"):
    import torch
    n = workspace_bytes(cfg, T)
    if n == 0:
        raise MoeError(EINVAL, "moe_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def stack_workspace(cfg: LayerCfg, L: int, T: int, device="cuda"):
    import torch
    n = int(load_library().moe_stack_workspace_bytes(ctypes.byref(cfg.c()), L, T))
    if n == 0:
        raise MoeError(EINVAL, "moe_stack_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def place_records(cfg: LayerCfg, sections: list, device="cuda", stride: int | None = None):
    """Packs per-expert section arrays (gu_codes, dn_codes, gu_scales, dn_scales)
    into one uint8 pool tensor [n, stride] at libmoe's record offsets."""
    import numpy as np
    import torch
    lay = expert_layout(cfg)
    stride = stride or lay["bytes"]
    host = np.zeros((len(sections), stride), dtype=np.uint8)
    for i, sec in enumerate(sections):
        for name in ("gu_codes", "dn_codes", "gu_scales", "dn_scales"):
            raw = np.ascontiguousarray(sec[name]).view(np.uint8).reshape(-1)
            host[i, lay[name]:lay[name] + raw.size] = raw
    return torch.from_numpy(host).to(device), stride
