"""ctypes wrapper of the CPU oracle (``qrx_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The oracle is the plain, slow reference that the
CUDA path is checked against.  Only ``tests/``, the smoke check and the
benchmark's CPU-baseline leg may import this package; the product path never
does.  It shares no code with the CUDA library.

Parity status: every function below is pinned by tests/test_oracle_pins.py to
something other than itself (hand-worked fixtures in tests/golden, brute force,
closed forms, numpy/f64 recomputation).  The colibri pages print no example of
a whole layer; the layer composition is pinned by a closed form (structured
tokens, router and expert rows under which every stage is a scalar expression).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qrx_oracle.c")
_LIB = os.path.join(_HERE, "libqrx_oracle.so")
_lock = threading.Lock()
_lib = None

vp = ctypes.c_void_p
i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float


def build(force: bool = False) -> str:
    """Compile the oracle: gcc -O2 -fopenmp -ffp-contract=off (no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int), ("inter", ctypes.c_int),
                ("n_group", ctypes.c_int), ("topk_group", ctypes.c_int), ("top_k", ctypes.c_int),
                ("routed_scaling_factor", ctypes.c_float), ("wbits", ctypes.c_int),
                ("afmt", ctypes.c_int)]


class CExpert(ctypes.Structure):
    _fields_ = [("gate_q", vp), ("gate_s", vp), ("up_q", vp), ("up_s", vp),
                ("down_q", vp), ("down_s", vp)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER
            sig = {
                "qo_max_threads": ([], ctypes.c_int),
                "qo_set_threads": ([ctypes.c_int], None),
                "qo_quantize_rows": ([vp, i64, i64, ctypes.c_int, vp, vp], None),
                "qo_unpack_rows": ([vp, i64, i64, ctypes.c_int, vp], None),
                "qo_quantize_q8": ([vp, i64, vp, vp], None),
                "qo_block_dots_q8": ([vp, i64, i64, ctypes.c_int, vp, vp], None),
                "qo_f32_to_bf16": ([f32], ctypes.c_uint16),
                "qo_bf16_to_f32": ([ctypes.c_uint16], f32),
                "qo_router": ([P(Cfg), vp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp], None),
                "qo_permute": ([vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp,
                                vp], None),
                "qo_ffn_token": ([P(Cfg), P(CExpert), vp, i64, vp, vp], None),
                "qo_expert_ffn": ([P(Cfg), vp, vp, vp, vp, ctypes.c_int, vp, vp, vp], None),
                "qo_expert_ffn_per_token": ([P(Cfg), vp, vp, vp, ctypes.c_int, vp, vp], None),
                "qo_expert_down": ([P(Cfg), vp, vp, vp, ctypes.c_int, vp, vp], None),
                "qo_shared_ffn": ([P(Cfg), P(CExpert), vp, ctypes.c_int, vp, vp], None),
                "qo_combine": ([P(Cfg), ctypes.c_int, vp, vp, vp, vp, vp], None),
                "qo_moe_forward": ([P(Cfg), vp, ctypes.c_int, vp, vp, vp, P(CExpert), vp, vp, vp],
                                   None),
                "qo_moe_forward_opts": ([P(Cfg), vp, ctypes.c_int, vp, vp, vp, P(CExpert),
                                         ctypes.c_double, vp, vp, vp], None),
                "qo_topp_prune": ([ctypes.c_int, ctypes.c_int, ctypes.c_double, f32, vp, vp],
                                  i64),
                "qo_fp8_e4m3_to_f32": ([ctypes.c_uint8], f32),
                "qo_requant_fp8": ([vp, i64, i64, i64, vp, ctypes.c_int, vp, vp], None),
            }
            for name, (args, res) in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def max_threads() -> int:
    return _load().qo_max_threads()


def set_threads(n: int) -> None:
    _load().qo_set_threads(n)


def cfg_struct(w) -> Cfg:
    """Oracle configuration from a Workload-like object."""
    return Cfg(w.hidden, w.n_experts, w.inter, w.n_group, w.topk_group, w.top_k,
               w.rsf, w.wbits, w.afmt)


# --------------------------------------------------------------------------- codes
def row_bytes(bits: int, K: int) -> int:
    return K * bits // 8


def quantize_rows(w: np.ndarray, bits: int):
    w = _c(w, np.float32)
    rows, K = w.shape
    q = np.zeros((rows, row_bytes(bits, K)), dtype=np.uint8)
    s = np.zeros(rows, dtype=np.float32)
    _load().qo_quantize_rows(_p(w), rows, K, bits, _p(q), _p(s))
    return q, s


def unpack_rows(q: np.ndarray, K: int, bits: int) -> np.ndarray:
    q = _c(q, np.uint8)
    rows = q.shape[0]
    codes = np.zeros((rows, K), dtype=np.int8)
    _load().qo_unpack_rows(_p(q), rows, K, bits, _p(codes))
    return codes


def quantize_q8(x: np.ndarray):
    x = _c(x, np.float32)
    n = x.size
    q = np.zeros(x.shape, dtype=np.int8)
    d = np.zeros(x.shape[:-1] + (x.shape[-1] // 32,), dtype=np.float32)
    _load().qo_quantize_q8(_p(x), n, _p(q), _p(d))
    return q, d


def block_dots_q8(q: np.ndarray, K: int, bits: int, xq: np.ndarray) -> np.ndarray:
    q = _c(q, np.uint8)
    xq = _c(xq, np.int8)
    rows = q.shape[0]
    acc = np.zeros((rows, K // 32), dtype=np.int32)
    _load().qo_block_dots_q8(_p(q), rows, K, bits, _p(xq), _p(acc))
    return acc


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    lib = _load()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib.qo_f32_to_bf16(float(v)) for v in x], dtype=np.uint16)


# --------------------------------------------------------------------------- experts
@dataclass
class Expert:
    """One expert's packed weights (oracle-side arrays)."""
    gate_q: np.ndarray
    gate_s: np.ndarray
    up_q: np.ndarray
    up_s: np.ndarray
    down_q: np.ndarray
    down_s: np.ndarray

    def cstruct(self) -> CExpert:
        return CExpert(_p(self.gate_q), _p(self.gate_s), _p(self.up_q), _p(self.up_s),
                       _p(self.down_q), _p(self.down_s))


def quantize_expert(gate: np.ndarray, up: np.ndarray, down: np.ndarray, bits: int) -> Expert:
    gq, gs = quantize_rows(gate, bits)
    uq, us = quantize_rows(up, bits)
    dq, ds = quantize_rows(down, bits)
    return Expert(gq, gs, uq, us, dq, ds)


def _expert_table(experts: dict, E: int):
    arr = (CExpert * E)()
    for e, ex in experts.items():
        arr[e] = ex.cstruct()
    return arr


def _act(w, act):
    if w.afmt == 2:
        assert act.dtype == np.uint16
        return _c(act, np.uint16)
    return _c(act, np.float32)


# --------------------------------------------------------------------------- layer steps
def router(w, act: np.ndarray, Wr: np.ndarray, bias: np.ndarray):
    act = _act(w, act)
    T = act.shape[0]
    Wr, bias = _c(Wr, np.float32), _c(bias, np.float32)
    idx = np.zeros((T, w.top_k), dtype=np.int32)
    wt = np.zeros((T, w.top_k), dtype=np.float32)
    logits = np.zeros((T, w.n_experts), dtype=np.float32)
    scores = np.zeros((T, w.n_experts), dtype=np.float32)
    ties = np.zeros(T, dtype=np.int32)
    c = cfg_struct(w)
    _load().qo_router(ctypes.byref(c), _p(act), T, _p(Wr), _p(bias), _p(idx), _p(wt),
                      _p(logits), _p(scores), _p(ties))
    return dict(idx=idx, w=wt, logits=logits, scores=scores, ties=ties)


def permute(idx: np.ndarray, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    A = T * k
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    sorted_ = np.zeros(A, np.int32)
    inv = np.zeros(A, np.int32)
    uid = np.zeros(E, np.int32)
    nu = np.zeros(1, np.int32)
    _load().qo_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(sorted_), _p(inv),
                       _p(uid), _p(nu))
    n = int(nu[0])
    return dict(counts=counts, offsets=offsets, sorted=sorted_, inv=inv, union_ids=uid[:n].copy(),
                n_union=n)


def ffn_token(w, ex: Expert, act: np.ndarray, t: int):
    act = _act(w, act)
    h = np.zeros(w.inter, np.float32)
    y = np.zeros(w.hidden, np.float32)
    c, ce = cfg_struct(w), ex.cstruct()
    _load().qo_ffn_token(ctypes.byref(c), ctypes.byref(ce), _p(act), t, _p(h), _p(y))
    return h, y


def expert_ffn(w, experts: dict, perm: dict, act: np.ndarray):
    """Batch-union routed FFN -> (h_sorted [A, I], y_sorted [A, H])."""
    act = _act(w, act)
    A = perm["sorted"].size
    h = np.zeros((A, w.inter), np.float32)
    y = np.zeros((A, w.hidden), np.float32)
    uid = _c(perm["union_ids"], np.int32)
    tab = _expert_table(experts, w.n_experts)
    c = cfg_struct(w)
    _load().qo_expert_ffn(ctypes.byref(c), tab, _p(perm["offsets"]), _p(perm["sorted"]),
                          _p(uid), perm["n_union"], _p(act), _p(h), _p(y))
    return h, y


def expert_ffn_per_token(w, experts: dict, idx: np.ndarray, perm: dict, act: np.ndarray):
    act = _act(w, act)
    T = act.shape[0]
    y = np.zeros((T * w.top_k, w.hidden), np.float32)
    tab = _expert_table(experts, w.n_experts)
    c = cfg_struct(w)
    idx = _c(idx, np.int32)
    _load().qo_expert_ffn_per_token(ctypes.byref(c), tab, _p(idx), _p(perm["inv"]), T,
                                    _p(act), _p(y))
    return y


def expert_down(w, experts: dict, perm: dict, h_sorted: np.ndarray):
    h_sorted = _c(h_sorted, np.float32)
    A = perm["sorted"].size
    y = np.zeros((A, w.hidden), np.float32)
    uid = _c(perm["union_ids"], np.int32)
    tab = _expert_table(experts, w.n_experts)
    c = cfg_struct(w)
    _load().qo_expert_down(ctypes.byref(c), tab, _p(perm["offsets"]), _p(uid), perm["n_union"],
                           _p(h_sorted), _p(y))
    return y


def shared_ffn(w, shared: Expert, act: np.ndarray):
    act = _act(w, act)
    T = act.shape[0]
    h = np.zeros((T, w.inter), np.float32)
    y = np.zeros((T, w.hidden), np.float32)
    c, ce = cfg_struct(w), shared.cstruct()
    _load().qo_shared_ffn(ctypes.byref(c), ctypes.byref(ce), _p(act), T, _p(h), _p(y))
    return h, y


def combine(w, y_sorted: np.ndarray, y_sh, wt: np.ndarray, inv: np.ndarray):
    y_sorted = _c(y_sorted, np.float32)
    wt = _c(wt, np.float32)
    T = wt.shape[0]
    ysh = None if y_sh is None else _c(y_sh, np.float32)
    out = np.zeros((T, w.hidden), np.float32)
    c = cfg_struct(w)
    _load().qo_combine(ctypes.byref(c), T, _p(y_sorted), _p(ysh), _p(wt), _p(_c(inv, np.int32)),
                       _p(out))
    return out


def topp_prune(idx: np.ndarray, wt: np.ndarray, p: float, rsf: float):
    """Adaptive expert top-p on the router's output (copies): (idx, w, kept)."""
    idx = _c(idx, np.int32).copy()
    wt = _c(wt, np.float32).copy()
    T, k = idx.shape
    # p and rsf are f32 values at the library's boundary: the threshold is
    # (double)p * (double)rsf of those
    kept = _load().qo_topp_prune(T, k, float(np.float32(p)), float(np.float32(rsf)), _p(idx), _p(wt))
    return idx, wt, int(kept)


def fp8_e4m3_to_f32(codes) -> np.ndarray:
    """FP8 e4m3 byte codes -> f32 (NaN for S.1111.111)."""
    codes = np.asarray(codes, np.uint8).ravel()
    f = _load().qo_fp8_e4m3_to_f32
    return np.array([f(int(b)) for b in codes], np.float32)


def requant_fp8(w8: np.ndarray, bscale: np.ndarray, bits: int):
    """FP8 [rows][K] with 128x128 block scales -> packed per-row codes and scales."""
    w8 = _c(w8, np.uint8)
    rows, K = w8.shape
    bscale = _c(bscale, np.float32)
    assert bscale.shape == ((rows + 127) // 128, (K + 127) // 128)
    q = np.zeros((rows, K * bits // 8), np.uint8)
    s = np.zeros(rows, np.float32)
    _load().qo_requant_fp8(_p(w8), rows, K, K, _p(bscale), bits, _p(q), _p(s))
    return q, s


def usage(idx: np.ndarray, E: int) -> np.ndarray:
    """Expert-usage histogram of one layer call: assignments per expert (dropped
    slots, idx = -1, not counted)."""
    idx = np.asarray(idx).ravel()
    return np.bincount(idx[idx >= 0], minlength=E).astype(np.uint64)


def moe_forward(w, act: np.ndarray, Wr: np.ndarray, bias: np.ndarray, experts: dict,
                shared: Expert | None, topp: float = 0.0):
    act = _act(w, act)
    T = act.shape[0]
    idx = np.zeros((T, w.top_k), np.int32)
    wt = np.zeros((T, w.top_k), np.float32)
    out = np.zeros((T, w.hidden), np.float32)
    tab = _expert_table(experts, w.n_experts)
    c = cfg_struct(w)
    sh = None if shared is None else ctypes.byref(shared.cstruct())
    _load().qo_moe_forward_opts(ctypes.byref(c), _p(act), T, _p(_c(Wr, np.float32)),
                                _p(_c(bias, np.float32)), tab, sh, float(np.float32(topp)), _p(idx), _p(wt),
                                _p(out))
    return idx, wt, out
