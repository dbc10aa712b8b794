"""Test infrastructure: one MoE layer built from the seeded inputs on both sides.

The CUDA path receives the f32 weights and quantises them with its own kernel;
the oracle quantises its own copy of the same f32 weights (experts on demand).
Only tests, the smoke check and the benchmark's CPU-baseline leg use this.
"""
from __future__ import annotations

import numpy as np

import oracle
from quantized_routed_expert_tc_b200.layer import expert_f32, router_weights


class OracleLayer:
    """Oracle-side experts, quantised on demand and cached per (format, expert)."""

    def __init__(self, wl):
        self.wl = wl
        self.Wr, self.bias = router_weights(wl)
        self._cache = {}

    def expert(self, e: int, bits: int | None = None) -> oracle.Expert:
        bits = self.wl.wbits if bits is None else bits
        key = (bits, e)
        if key not in self._cache:
            self._cache[key] = oracle.quantize_expert(*expert_f32(self.wl, e), bits)
        return self._cache[key]

    def experts(self, ids, bits=None) -> dict:
        return {int(e): self.expert(int(e), bits) for e in np.unique(np.asarray(ids))}

    def shared(self, bits=None) -> oracle.Expert:
        return self.expert(self.wl.n_experts, bits)

    def forward_tokens(self, wl, x: np.ndarray, tokens, bias=None, topp: float = 0.0):
        """Oracle layer output rows for the listed tokens of batch x (routing uses the
        tokens' own rows; every token is independent).  topp in (0, 1): adaptive
        expert top-p on the router's output (r then holds the pruned idx, w)."""
        bias = self.bias if bias is None else bias
        r = oracle.router(wl, x, self.Wr, bias)
        if 0.0 < topp < 1.0:
            r["idx"], r["w"], _ = oracle.topp_prune(r["idx"], r["w"], topp, wl.rsf)
        outs = []
        for t in tokens:
            w1 = wl.with_(T=1)
            xt = x[t:t + 1]
            idx = r["idx"][t:t + 1]
            p = oracle.permute(idx, wl.n_experts)
            ex = self.experts(idx.ravel()[idx.ravel() >= 0], wl.wbits)
            _, ys = oracle.expert_ffn(w1, ex, p, xt)
            _, ysh = oracle.shared_ffn(w1, self.shared(wl.wbits), xt)
            outs.append(oracle.combine(w1, ys, ysh, r["w"][t:t + 1], p["inv"])[0])
        return r, np.stack(outs)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max|got - ref| / max|ref| (the parity measure on f32 outputs)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    m = np.abs(ref).max()
    d = np.abs(got - ref).max()
    return float(d / m) if m > 0 else float(d)


TOL = 1e-3   # max|gpu - oracle| <= 1e-3 * max|oracle| on f32 outputs
