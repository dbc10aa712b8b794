"""Thin Python binding of libqrx (include/qrx.h): argument marshalling only.

Every function named ``qrx_*`` here calls the C entry point of the same name
with the tensors' device pointers and the current torch CUDA stream.  Every
step of the layer runs in the library's CUDA kernels; there is no Python or
CPU fallback: if libqrx.so is missing or a call fails, a QrxError is raised.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

from . import build as _build

QRX_OK, QRX_EINVAL, QRX_EUNSUPPORTED, QRX_ECUDA, QRX_ETIMEOUT, QRX_EDEVICE, QRX_ENOSPACE = \
    0, -1, -2, -3, -4, -5, -6
QRX_ENGINE_GEMV, QRX_ENGINE_TC = 0, 1
W_INT8, W_INT4, W_INT2 = 8, 4, 2
A_F32, A_Q8_0, A_BF16 = 0, 1, 2

HEADER = os.path.join(os.path.dirname(_build.HERE), "include", "qrx.h")


class QrxError(RuntimeError):
    def __init__(self, name: str, code: int, detail: str | None = None):
        self.code = code
        super().__init__(f"{name}: {detail or qrx_strerror(code)} ({code})")


class Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("wfmt", ctypes.c_int32),
                ("afmt", ctypes.c_int32)]


class CMat(ctypes.Structure):
    """qrx_mat: one packed matrix of every expert."""
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("expert_stride_q", ctypes.c_int64), ("expert_stride_s", ctypes.c_int64)]


class CExperts(ctypes.Structure):
    """qrx_experts: the gate, up and down matrices of an expert set."""
    _fields_ = [("gate", CMat), ("up", CMat), ("down", CMat)]


class COpts(ctypes.Structure):
    """qrx_moe_opts."""
    _fields_ = [("expert_top_p", ctypes.c_float), ("usage", ctypes.c_void_p)]


class CPerm(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("counts", "offsets", "sorted", "inv", "union_ids", "n_union")]


class CAct(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("xq", ctypes.c_void_p), ("xd", ctypes.c_void_p)]


_lib = None
vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
P = ctypes.POINTER

_SIGS = {
    "qrx_validate": ([P(Cfg)], ctypes.c_int),
    "qrx_workspace_bytes": ([P(Cfg), i32], sz),
    "qrx_ffn_engine": ([P(Cfg), i32], ctypes.c_int),
    "qrx_last_error": ([], ctypes.c_int),
    "qrx_strerror": ([ctypes.c_int], ctypes.c_char_p),
    "qrx_quantize_weights": ([vp, i64, i64, i32, vp, i64, vp, i64, vp], ctypes.c_int),
    "qrx_quantize_act_q8": ([vp, i64, i64, vp, vp, vp], ctypes.c_int),
    "qrx_requant_fp8": ([vp, i64, i64, i64, vp, i32, vp, i64, vp, i64, vp], ctypes.c_int),
    "qrx_block_dots_q8": ([i32, vp, i64, i64, vp, vp, vp], ctypes.c_int),
    "qrx_route": ([P(Cfg), vp, i32, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
    "qrx_permute": ([P(Cfg), vp, i32, P(CPerm), vp], ctypes.c_int),
    "qrx_topp_prune": ([P(Cfg), vp, vp, i32, ctypes.c_float, vp], ctypes.c_int),
    "qrx_usage_accumulate": ([P(Cfg), P(CPerm), vp, vp], ctypes.c_int),
    "qrx_expert_ffn": ([P(Cfg), P(CExperts), P(CPerm), P(CAct), i32, vp, vp, vp, sz, vp],
                       ctypes.c_int),
    "qrx_expert_ffn_noalloc": ([P(Cfg), P(CExperts), P(CPerm), P(CAct), i32, vp, vp],
                               ctypes.c_int),
    "qrx_expert_down": ([P(Cfg), P(CExperts), P(CPerm), vp, i32, vp, vp, sz, vp], ctypes.c_int),
    "qrx_expert_gateup_q8_sums": ([P(Cfg), P(CExperts), P(CPerm), P(CAct), i32, vp, vp, vp, sz, vp],
                                  ctypes.c_int),
    "qrx_expert_down_q8_sums": ([P(Cfg), P(CExperts), P(CPerm), vp, i32, vp, vp, vp, sz, vp],
                                ctypes.c_int),
    "qrx_shared_ffn": ([P(Cfg), P(CExperts), P(CAct), i32, vp, vp, vp, sz, vp], ctypes.c_int),
    "qrx_combine": ([P(Cfg), vp, vp, vp, vp, i32, vp, vp], ctypes.c_int),
    "qrx_moe_forward": ([P(Cfg), vp, i32, vp, vp, P(CExperts), P(CExperts), vp, vp, vp, vp, sz,
                         vp], ctypes.c_int),
    "qrx_moe_forward_opts": ([P(Cfg), vp, i32, vp, vp, P(CExperts), P(CExperts), vp, vp, vp, vp,
                              sz, P(COpts), vp], ctypes.c_int),
    "qrx_moe_forward_hostio": ([P(Cfg), vp, i32, vp, vp, P(CExperts), P(CExperts), vp, vp, sz,
                                vp], ctypes.c_int),
    "qrx_moe_forward_profiled": ([P(Cfg), vp, i32, vp, vp, P(CExperts), P(CExperts), vp, vp, vp,
                                  vp, sz, ctypes.POINTER(vp), i32, P(COpts), vp], ctypes.c_int),
}


def lib_path() -> str:
    """libqrx.so, or with QRX_CHECK=1 in the environment the bounds-checked
    libqrx_check.so (same entry points and results; misses are reported by
    qrx_last_error)."""
    return _build.CHECK_LIB if os.environ.get("QRX_CHECK") == "1" else _build.LIB


def lib():
    """Load libqrx.so (built in-tree by build()).  Raises if it is missing."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise QrxError("load", QRX_ECUDA,
                           f"{path} is missing: build it with "
                           "quantized_routed_expert_tc_b200.build.build()")
        L = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions include/qrx.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(qrx_\w+)\s*\(", txt, re.M)))


# ------------------------------------------------------------------ marshalling helpers
def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _st(stream):
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream
    return torch.cuda.current_stream().cuda_stream


def _check(name: str, rc: int):
    if rc != QRX_OK:
        raise QrxError(name, rc)


def cfg_of(w) -> Cfg:
    """qrx_cfg from a workload-like object (hidden, n_experts, ..., wbits, afmt)."""
    return Cfg(w.hidden, w.n_experts, w.inter, w.n_group, w.topk_group, w.top_k, w.rsf,
               w.wbits, w.afmt)


@dataclass
class Experts:
    """Packed experts on the device (layout of include/qrx.h): three matrices,
    each [n][rows][K*b/8] uint8 with row scales [n][rows] f32."""
    gate: torch.Tensor     # [n, I, H*b/8] uint8
    gate_s: torch.Tensor   # [n, I] f32
    up: torch.Tensor       # [n, I, H*b/8] uint8
    up_s: torch.Tensor     # [n, I] f32
    down: torch.Tensor     # [n, H, I*b/8] uint8
    down_s: torch.Tensor   # [n, H] f32

    @staticmethod
    def _cmat(q, s) -> CMat:
        if q.dim() != 3 or s.dim() != 2 or q.stride(2) != 1 or q.stride(1) != q.shape[2] or s.stride(1) != 1:
            raise ValueError("expert matrices must have contiguous rows and scales")
        return CMat(q.data_ptr(), s.data_ptr(), q.stride(0) * q.element_size(), s.stride(0))

    def c(self) -> CExperts:
        """The qrx_experts struct of these tensors, built once: a call passes it
        without rebuilding it, and assigning any of the six tensors drops it."""
        cs = self.__dict__.get("_cstruct")
        if cs is None:
            cs = CExperts(self._cmat(self.gate, self.gate_s), self._cmat(self.up, self.up_s),
                          self._cmat(self.down, self.down_s))
            self.__dict__["_cstruct"] = cs
        return cs

    def __setattr__(self, name, value):
        self.__dict__.pop("_cstruct", None)
        super().__setattr__(name, value)

    @staticmethod
    def empty(n: int, H: int, I: int, wbits: int, device="cuda") -> "Experts":
        u8, f32 = torch.uint8, torch.float32
        return Experts(torch.empty((n, I, H * wbits // 8), dtype=u8, device=device),
                       torch.empty((n, I), dtype=f32, device=device),
                       torch.empty((n, I, H * wbits // 8), dtype=u8, device=device),
                       torch.empty((n, I), dtype=f32, device=device),
                       torch.empty((n, H, I * wbits // 8), dtype=u8, device=device),
                       torch.empty((n, H), dtype=f32, device=device))

    def tensors(self):
        return (self.gate, self.gate_s, self.up, self.up_s, self.down, self.down_s)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.tensors())


@dataclass
class Perm:
    counts: torch.Tensor
    offsets: torch.Tensor
    sorted: torch.Tensor
    inv: torch.Tensor
    union_ids: torch.Tensor
    n_union: torch.Tensor

    def c(self) -> CPerm:
        return CPerm(*(_p(t) for t in (self.counts, self.offsets, self.sorted, self.inv,
                                        self.union_ids, self.n_union)))

    @staticmethod
    def empty(T: int, k: int, E: int, device="cuda") -> "Perm":
        z = lambda n: torch.empty(n, dtype=torch.int32, device=device)
        return Perm(z(E), z(E + 1), z(T * k), z(T * k), z(E), z(1))


def workspace(cfg: Cfg, T: int, device="cuda") -> torch.Tensor:
    n = qrx_workspace_bytes(cfg, T)
    if n == 0:
        raise QrxError("qrx_workspace_bytes", QRX_EINVAL)
    return torch.empty(n, dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ C entry points
def qrx_validate(cfg: Cfg) -> int:
    return lib().qrx_validate(ctypes.byref(cfg))


def qrx_workspace_bytes(cfg: Cfg, T: int) -> int:
    return lib().qrx_workspace_bytes(ctypes.byref(cfg), T)


def qrx_ffn_engine(cfg: Cfg, T: int) -> int:
    """QRX_ENGINE_TC or QRX_ENGINE_GEMV: the expert-FFN engine for this cfg and T."""
    v = lib().qrx_ffn_engine(ctypes.byref(cfg), T)
    if v < 0:
        raise QrxError("qrx_ffn_engine", v)
    return v


def qrx_last_error() -> int:
    return lib().qrx_last_error()


def qrx_strerror(code: int) -> str:
    if _lib is None and not os.path.exists(lib_path()):
        return f"error {code}"
    return lib().qrx_strerror(code).decode()


def qrx_quantize_weights(w, wbits, q, ldq, scale, lds, stream=None):
    rows, K = w.shape
    _check("qrx_quantize_weights", lib().qrx_quantize_weights(
        _p(w), rows, K, wbits, _p(q), ldq, _p(scale), lds, _st(stream)))


def qrx_quantize_act_q8(x, xq, xd, stream=None):
    T, H = x.shape
    _check("qrx_quantize_act_q8", lib().qrx_quantize_act_q8(_p(x), T, H, _p(xq), _p(xd),
                                                            _st(stream)))


def qrx_block_dots_q8(wbits, q, K, xq, acc, stream=None):
    _check("qrx_block_dots_q8", lib().qrx_block_dots_q8(wbits, _p(q), q.shape[0], K, _p(xq),
                                                        _p(acc), _st(stream)))


def qrx_route(cfg, x, Wr, bias, topk_idx, topk_w, ws, stream=None):
    _check("qrx_route", lib().qrx_route(ctypes.byref(cfg), _p(x), x.shape[0], _p(Wr), _p(bias),
                                        _p(topk_idx), _p(topk_w), _p(ws), ws.numel(), _st(stream)))


def qrx_permute(cfg, topk_idx, perm: Perm, stream=None):
    _check("qrx_permute", lib().qrx_permute(ctypes.byref(cfg), _p(topk_idx), topk_idx.shape[0],
                                            ctypes.byref(perm.c()), _st(stream)))


def _act(cfg, x=None, xq=None, xd=None) -> CAct:
    return CAct(_p(x), _p(xq), _p(xd))


def qrx_expert_ffn(cfg, routed: Experts, perm: Perm, T, y_sorted, ws, x=None, xq=None, xd=None,
                   h_sorted=None, stream=None):
    _check("qrx_expert_ffn", lib().qrx_expert_ffn(
        ctypes.byref(cfg), ctypes.byref(routed.c()), ctypes.byref(perm.c()),
        ctypes.byref(_act(cfg, x, xq, xd)), T, _p(h_sorted), _p(y_sorted), _p(ws), ws.numel(),
        _st(stream)))


def qrx_expert_ffn_noalloc(cfg, routed: Experts, perm: Perm, T, y_sorted, x=None, xq=None,
                           xd=None, stream=None):
    """qrx_expert_ffn with no caller workspace (the library's fixed 8 MiB array)."""
    _check("qrx_expert_ffn_noalloc", lib().qrx_expert_ffn_noalloc(
        ctypes.byref(cfg), ctypes.byref(routed.c()), ctypes.byref(perm.c()),
        ctypes.byref(_act(cfg, x, xq, xd)), T, _p(y_sorted), _st(stream)))


def qrx_expert_down(cfg, routed: Experts, perm: Perm, h_sorted, T, y_sorted, ws, stream=None):
    _check("qrx_expert_down", lib().qrx_expert_down(
        ctypes.byref(cfg), ctypes.byref(routed.c()), ctypes.byref(perm.c()), _p(h_sorted), T,
        _p(y_sorted), _p(ws), ws.numel(), _st(stream)))


def qrx_expert_gateup_q8_sums(cfg, routed: Experts, perm: Perm, T, h_sorted, acc, ws, xq, xd,
                              stream=None):
    """Gate/up of the routed FFN (Q8_0, T <= 4) with its int32 block accumulators
    acc [T*k, 2, I, H/32]."""
    _check("qrx_expert_gateup_q8_sums", lib().qrx_expert_gateup_q8_sums(
        ctypes.byref(cfg), ctypes.byref(routed.c()), ctypes.byref(perm.c()),
        ctypes.byref(_act(cfg, None, xq, xd)), T, _p(h_sorted), _p(acc), _p(ws), ws.numel(),
        _st(stream)))


def qrx_expert_down_q8_sums(cfg, routed: Experts, perm: Perm, h_sorted, T, y_sorted, acc, ws,
                            stream=None):
    """Down of the routed FFN from a given h (Q8_0, T <= 4) with its int32 block
    accumulators acc [T*k, H, I/32]."""
    _check("qrx_expert_down_q8_sums", lib().qrx_expert_down_q8_sums(
        ctypes.byref(cfg), ctypes.byref(routed.c()), ctypes.byref(perm.c()), _p(h_sorted), T,
        _p(y_sorted), _p(acc), _p(ws), ws.numel(), _st(stream)))


def qrx_shared_ffn(cfg, shared: Experts, T, y_sh, ws, x=None, xq=None, xd=None, h_sh=None,
                   stream=None):
    _check("qrx_shared_ffn", lib().qrx_shared_ffn(
        ctypes.byref(cfg), ctypes.byref(shared.c()), ctypes.byref(_act(cfg, x, xq, xd)), T,
        _p(h_sh), _p(y_sh), _p(ws), ws.numel(), _st(stream)))


def qrx_combine(cfg, y_sorted, y_sh, topk_w, inv, out, stream=None):
    _check("qrx_combine", lib().qrx_combine(ctypes.byref(cfg), _p(y_sorted), _p(y_sh),
                                            _p(topk_w), _p(inv), topk_w.shape[0], _p(out),
                                            _st(stream)))


def qrx_moe_forward(cfg, x, Wr, bias, routed: Experts, shared: Experts | None, topk_idx, topk_w,
                    out, ws, stream=None, topp: float = 0.0, usage=None):
    """The whole layer.  topp > 0 or a usage tensor (uint64/int64 [E] on the
    device) go through qrx_moe_forward_opts."""
    sh = ctypes.byref(shared.c()) if shared is not None else None
    if topp or usage is not None:
        opts = COpts(float(topp), _p(usage))
        _check("qrx_moe_forward_opts", lib().qrx_moe_forward_opts(
            ctypes.byref(cfg), _p(x), x.shape[0], _p(Wr), _p(bias), ctypes.byref(routed.c()), sh,
            _p(topk_idx), _p(topk_w), _p(out), _p(ws), ws.numel(), ctypes.byref(opts), _st(stream)))
        return
    _check("qrx_moe_forward", lib().qrx_moe_forward(
        ctypes.byref(cfg), _p(x), x.shape[0], _p(Wr), _p(bias), ctypes.byref(routed.c()), sh,
        _p(topk_idx), _p(topk_w), _p(out), _p(ws), ws.numel(), _st(stream)))


def qrx_requant_fp8(w8, bscale, wbits: int, q, scale, stream=None):
    """FP8 e4m3 rows (uint8 [rows][K]) with 128x128 block scales -> packed codes q
    [rows][K*wbits/8] and row scales [rows]."""
    rows, K = w8.shape
    if w8.stride(1) != 1 or not w8.is_cuda:
        raise ValueError("w8 rows must be contiguous device memory (a row stride is allowed)")
    _check("qrx_requant_fp8", lib().qrx_requant_fp8(w8.data_ptr(), rows, K, w8.stride(0), _p(bscale), wbits,
                                                    _p(q), q.stride(0), _p(scale), 1, _st(stream)))


def qrx_topp_prune(cfg, topk_idx, topk_w, p: float, stream=None):
    """Adaptive expert top-p in place on a router output [T][k]."""
    _check("qrx_topp_prune", lib().qrx_topp_prune(ctypes.byref(cfg), _p(topk_idx), _p(topk_w),
                                                  topk_idx.shape[0], float(p), _st(stream)))


def qrx_usage_accumulate(cfg, perm, usage, stream=None):
    """usage[e] += perm.counts[e] (usage: uint64/int64 [E] device tensor)."""
    _check("qrx_usage_accumulate", lib().qrx_usage_accumulate(ctypes.byref(cfg), ctypes.byref(perm.c()),
                                                              _p(usage), _st(stream)))


def qrx_moe_forward_profiled(cfg, x, Wr, bias, routed: Experts, shared: Experts | None,
                             topk_idx, topk_w, out, ws, events, stream=None, topp: float = 0.0,
                             usage=None):
    """qrx_moe_forward recording 7 torch.cuda.Event objects between its stages."""
    sh = ctypes.byref(shared.c()) if shared is not None else None
    for ev in events:                     # torch creates the CUDA event on first record
        if not ev.cuda_event:
            ev.record(stream)
    arr = (vp * 7)(*[ev.cuda_event for ev in events])
    _check("qrx_moe_forward_profiled", lib().qrx_moe_forward_profiled(
        ctypes.byref(cfg), _p(x), x.shape[0], _p(Wr), _p(bias), ctypes.byref(routed.c()), sh,
        _p(topk_idx), _p(topk_w), _p(out), _p(ws), ws.numel(), arr, len(events),
        ctypes.byref(COpts(float(topp), _p(usage))), _st(stream)))


def qrx_moe_forward_hostio(cfg, x_host, Wr, bias, routed: Experts, shared: Experts | None,
                           out_host, ws, stream=None):
    sh = ctypes.byref(shared.c()) if shared is not None else None
    _check("qrx_moe_forward_hostio", lib().qrx_moe_forward_hostio(
        ctypes.byref(cfg), _p(x_host), x_host.shape[0], _p(Wr), _p(bias),
        ctypes.byref(routed.c()), sh, _p(out_host), _p(ws), ws.numel(), _st(stream)))


# ------------------------------------------------------------------ weight packing
def quantize_expert_into(ex: Experts, e: int, gate: torch.Tensor, up: torch.Tensor,
                         down: torch.Tensor, wbits: int, stream=None) -> None:
    """Quantise one expert's f32 gate [I,H], up [I,H], down [H,I] (device tensors)
    into slot e of `ex` with the library's per-row quantiser."""
    for w, q, sc in ((gate, ex.gate, ex.gate_s), (up, ex.up, ex.up_s), (down, ex.down, ex.down_s)):
        qrx_quantize_weights(w, wbits, q[e].data_ptr(), q.shape[2], sc[e].data_ptr(), 1, stream)
