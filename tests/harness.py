"""Shared set-up for the GPU parity tests: one synthetic layer whose inputs
both sides read (the oracle as numpy arrays, libmoe as device buffers), and
comparison helpers with the tolerances the tests use.

Tolerances:
* routing indices and grouping: bit-exact, except that an index may differ
  where the oracle's fp64 logits of the two experts involved are within
  TIE_TOL * max|l| of each other (the GPU selects on fp32 logits);
* FFN output: per token, max|y - y*| <= 2e-3 * max|y*| against the fp64
  oracle (fp32 output); bf16 output may add one bf16 ulp of y*.
"""
from __future__ import annotations

import copy

import numpy as np
import torch

from bit_expert_ffn_router_b200 import moe as M
from bit_expert_ffn_router_b200 import synth
from oracle import moe_oracle as O

REL_TOL = 2e-3
TIE_TOL = 1e-5

_ctx = None


def ctx() -> M.Context:
    global _ctx
    if _ctx is None:
        M.load_library()
        _ctx = M.Context(torch.cuda.current_device())
    return _ctx


class Layer:
    """A seeded layer: x [T,d] bf16, W_r, optional Zipf bias, E routed experts
    behind a shuffled slot table, one shared expert."""

    def __init__(self, cfg: M.LayerCfg, T: int, seed: int = 0, zipf: bool = False, extra_slots: int = 3,
                 bias=None):
        self.cfg, self.T, self.seed = cfg, T, seed
        d, f, E, k, bits = cfg.d, cfg.f, cfg.E, cfg.k, cfg.bits
        self.x = synth.activations(T, d, seed)
        self.wr = synth.router_weights(E, d, seed + 1)
        if bias is not None:
            self.bias = np.asarray(bias, dtype=np.float32)
        elif zipf:
            self.bias = synth.bias_from_sets(synth.zipf_sets(T, E, k, seed + 2), E)
        else:
            self.bias = None
        self.sections = [synth.expert_sections(d, f, bits, seed + 100 + e) for e in range(E)]
        self.shared = synth.expert_sections(d, f, bits, seed + 99) if cfg.n_shared else None
        self.n_slots = E + extra_slots
        self.slot_of = synth.rng(seed + 3).permutation(self.n_slots)[:E].astype(np.int32)
        self._dev = None

    # ---- oracle side
    def oracle(self, tokens=None):
        cache = O.ExpertCache(lambda e: self.sections[e], self.cfg.d, self.cfg.f, self.cfg.bits)
        sh = O.expert_weights(self.shared, self.cfg.d, self.cfg.f, self.cfg.bits) if self.shared else None
        return O.layer_forward(self.x, self.wr, self.cfg.k, cache, sh, bias=self.bias, renorm=bool(self.cfg.renorm),
                               residual=bool(self.cfg.residual), tokens=tokens, skip_from=self.cfg.skip_from,
                               hot_slots=self.cfg.hot_slots, slot_of=self.slot_of)

    # ---- device side
    def device(self):
        if self._dev is None:
            cfg = self.cfg
            filler = synth.expert_sections(cfg.d, cfg.f, cfg.bits, self.seed + 98)
            by_slot = [filler] * self.n_slots
            for e in range(cfg.E):
                by_slot[self.slot_of[e]] = self.sections[e]
            pool, stride = M.place_records(cfg, by_slot)
            shared = M.place_records(cfg, [self.shared])[0] if self.shared else None
            self._dev = {
                "x": torch.from_numpy(self.x.view(np.int16)).cuda(),
                "wr": torch.from_numpy(self.wr).cuda(),
                "bias": None if self.bias is None else torch.from_numpy(self.bias).cuda(),
                "slot_of": torch.from_numpy(self.slot_of).cuda(),
                "pool": pool, "stride": stride, "shared": shared,
            }
        return self._dev

    def with_inputs(self, x, bias, wr=None):
        """The same experts, pool and slot table with other tokens (x [T,d] bf16 bits, bias [T,E] or
        None) and optionally another router matrix; the device pool is shared, not rebuilt."""
        L = copy.copy(self)
        L.T = x.shape[0]
        L.x = x
        L.bias = None if bias is None else np.asarray(bias, dtype=np.float32)
        if wr is not None:
            L.wr = np.asarray(wr, dtype=np.float32)
        dv = dict(self.device())
        dv["x"] = torch.from_numpy(np.ascontiguousarray(L.x).view(np.int16)).cuda()
        dv["bias"] = None if L.bias is None else torch.from_numpy(L.bias).cuda()
        dv["wr"] = torch.from_numpy(L.wr).cuda()
        L._dev = dv
        return L

    def out_tensor(self):
        dt = torch.float32 if self.cfg.out_fp32 else torch.bfloat16
        return torch.empty(self.T, self.cfg.d, dtype=dt, device="cuda")

    def forward(self, cfg=None, y=None, ws=None):
        cfg = cfg or self.cfg
        dv = self.device()
        ws = ws if ws is not None else M.workspace(cfg, self.T)
        y = y if y is not None else self.out_tensor()
        ctx().layer_forward(cfg, dv["x"], self.T, dv["wr"], dv["bias"], dv["slot_of"], self.n_slots, dv["pool"],
                            dv["stride"], dv["shared"], ws, y)
        return y, ws


def y_as_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


def assert_close_rows(y_gpu: np.ndarray, y_ref: np.ndarray, bf16: bool = False, tol: float = REL_TOL) -> float:
    """Per-row max-norm relative error; returns the worst one."""
    worst = 0.0
    for t in range(y_ref.shape[0]):
        scale = np.max(np.abs(y_ref[t]))
        err = np.abs(y_gpu[t] - y_ref[t])
        if bf16:
            ulp = np.ldexp(1.0, np.frexp(np.abs(y_ref[t]))[1] - 8)
            err = np.maximum(err - ulp, 0.0)
        rel = float(err.max() / scale) if scale > 0 else float(err.max())
        worst = max(worst, rel)
        assert rel <= tol, f"token {t}: relative error {rel:.3e} > {tol}"
    return worst


def assert_routing_matches(idx_gpu: np.ndarray, idx_ref: np.ndarray, logits_ref: np.ndarray) -> int:
    """Indices must agree, except at fp64 near-ties; returns the number of tie-explained differences."""
    ties = 0
    for t in range(idx_ref.shape[0]):
        if np.array_equal(idx_gpu[t], idx_ref[t]):
            continue
        scale = np.max(np.abs(logits_ref[t]))
        for a, b in zip(idx_gpu[t], idx_ref[t]):
            if a != b:
                gap = abs(logits_ref[t, a] - logits_ref[t, b])
                assert gap <= TIE_TOL * scale, f"token {t}: expert {a} vs {b}, fp64 gap {gap:.3e}"
                ties += 1
    return ties
