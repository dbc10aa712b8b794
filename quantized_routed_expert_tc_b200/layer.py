"""A routed-MoE layer resident on the GPU, built from the seeded synthetic inputs.

Weights are drawn as f32 on the host (``synth``), copied to the device and
packed there by the library's own quantiser (qrx_quantize_weights), one expert
at a time, into the layout of include/qrx.h.  All formats requested are packed
from the same f32 draw, so a format sweep compares like with like.
"""
from __future__ import annotations

import numpy as np
import torch

from . import qrx, synth, workloads as W


def expert_f32(wl, e: int):
    """f32 gate [I,H], up [I,H], down [H,I] of expert e (e == E: the shared expert)."""
    H, I, s = wl.hidden, wl.inter, wl.layer_seed
    g = synth.normal_f32(s, W.stream(W.K_GATE, e), I * H, 0.0, W.W_STD).reshape(I, H)
    u = synth.normal_f32(s, W.stream(W.K_UP, e), I * H, 0.0, W.W_STD).reshape(I, H)
    d = synth.normal_f32(s, W.stream(W.K_DOWN, e), H * I, 0.0, W.W_STD).reshape(H, I)
    return g, u, d


def router_weights(wl):
    """Router weight Wr [E,H] (layer seed) and score-correction bias [E] (workload seed)."""
    E, H = wl.n_experts, wl.hidden
    Wr = synth.normal_f32(wl.layer_seed, W.stream(W.K_WR), E * H, 0.0, W.W_STD).reshape(E, H)
    bias = synth.normal_f32(wl.seed, W.stream(W.K_BIAS), E, 0.0, wl.bias_std)
    return Wr, bias


def activations(wl, T: int | None = None, batch: int = 0) -> np.ndarray:
    """x [T,H] of batch `batch`: f32, or uint16 bf16 bit patterns for bf16 workloads."""
    T = wl.T if T is None else T
    n = T * wl.hidden
    if wl.afmt == W.A_BF16:
        return synth.normal_bf16(wl.seed, W.stream(W.K_X, batch), n).reshape(T, wl.hidden)
    return synth.normal_f32(wl.seed, W.stream(W.K_X, batch), n).reshape(T, wl.hidden)


def activations_correlated(wl, T: int, rho: float, batch: int = 0) -> np.ndarray:
    """A verify batch whose T tokens share router input structure: token i is
    sqrt(rho) * z + sqrt(1 - rho) * z_i with z common to the batch and z_i its own
    (all N(0,1) draws; pairwise correlation rho per coordinate), formed in double
    and rounded to f32 (bf16 workloads: then to bf16, nearest-even).  rho = 0 gives
    independent tokens, rho = 1 identical ones."""
    n = wl.hidden
    z = synth.normal_f32(wl.seed, W.stream(W.K_XC, batch), n).astype(np.float64)
    zi = synth.normal_f32(wl.seed, W.stream(W.K_X, batch), T * n).reshape(T, n).astype(np.float64)
    x = (np.sqrt(rho) * z[None, :] + np.sqrt(1.0 - rho) * zi).astype(np.float32)
    if wl.afmt == W.A_BF16:
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return x


def to_device_act(wl, x: np.ndarray, device="cuda") -> torch.Tensor:
    """Activation array -> device tensor of the workload's dtype (f32 or bf16)."""
    if wl.afmt == W.A_BF16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(x).to(device)


class GpuLayer:
    """Packed routed experts, shared expert, router weight and bias on one device."""

    def __init__(self, wl, formats=None, device="cuda"):
        self.wl = wl
        self.device = device
        formats = tuple(formats or (wl.wbits,))
        E, H, I = wl.n_experts, wl.hidden, wl.inter
        self.routed = {b: qrx.Experts.empty(E, H, I, b, device) for b in formats}
        self.shared = {b: qrx.Experts.empty(1, H, I, b, device) for b in formats}
        Wr, bias = router_weights(wl)
        self.Wr = torch.from_numpy(Wr).to(device)
        self.bias = torch.from_numpy(bias).to(device)
        stream = torch.cuda.current_stream(device)
        for e in range(E + 1):
            g, u, d = (torch.from_numpy(a).to(device) for a in expert_f32(wl, e))
            for b in formats:
                dst, slot = (self.routed[b], e) if e < E else (self.shared[b], 0)
                qrx.quantize_expert_into(dst, slot, g, u, d, b, stream)
        torch.cuda.synchronize(device)

    def set_bias(self, wl) -> None:
        """Use the bias of another workload on the same layer."""
        _, bias = router_weights(wl)
        self.bias = torch.from_numpy(bias).to(self.device)
