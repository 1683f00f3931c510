"""CPU oracle for the routed-MoE FFN (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package; the product library never does. The arithmetic lives
in moe_oracle.cpp (plain loops, double accumulation); this module marshals
numpy arrays into it and strings the per-token steps together in the order
the layer runs them:
  1. router logits over all experts (plus an optional per-expert bias),
  2. softmax over all experts, the k largest, renormalised over the k,
  3. per selected expert gate/up (one packed matrix), SwiGLU, down,
  4. sigmoid-gated shared expert, weighted combine, fp32 then bf16.
Routing fan-out: Swiftlet article (xix.ai), paragraph 4; Runnel README,
"Target". Low-bit groups: Swiftlet article, paragraph 8. Packed gate/up:
Runnel README, introduction and "Streaming CLI".
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.cpp into oracle/_build/liboracle.so with g++."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-pthread", _SRC, "-o", _LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class QMat(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("K", ctypes.c_int64)]


def lib():
    global _lib
    if _lib is None:
        # MOE_ORACLE_LIB points the tests' mutation check at a deliberately
        # broken build of this file; normally the library is built here.
        _lib = ctypes.CDLL(os.environ.get("MOE_ORACLE_LIB") or build())
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        _lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.orc_bf16_to_f32.restype = ctypes.c_float
        _lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        _lib.orc_dequant.argtypes = [ctypes.POINTER(QMat), I32, I32, P]
        _lib.orc_router_logits.argtypes = [P, I64, I64, P, I64, P, P]
        _lib.orc_softmax_topk.argtypes = [P, I64, I64, I32, P, P]
        _lib.orc_shared_gate.argtypes = [P, P, I64]
        _lib.orc_shared_gate.restype = D
        _lib.orc_expert_ffn.argtypes = [P, P, I64, I64, P, P, P]
        _lib.orc_moe_token.argtypes = [I64, I64, I64, I32, I32, P, I64, ctypes.POINTER(QMat),
                                       ctypes.POINTER(QMat), P, ctypes.POINTER(QMat),
                                       ctypes.POINTER(QMat), D, P, P, P, I32]
        _lib.orc_sort_by_expert.argtypes = [P, I64, I64, I64, I32, P, P]
        _lib.orc_residual_rmsnorm.argtypes = [P, P, I64, I64, D, P, P]
        for f in ("orc_dequant", "orc_router_logits", "orc_softmax_topk", "orc_expert_ffn",
                  "orc_moe_token", "orc_sort_by_expert", "orc_residual_rmsnorm"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def bf16_to_f32(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (via the C routine)."""
    a = np.asarray(x, dtype=np.float32)
    f = lib().orc_f32_to_bf16
    return np.array([f(float(v)) for v in a.ravel()], dtype=np.uint16).reshape(a.shape)


class QMatrix:
    """Host view of one quantised matrix [rows][K]: codes, bf16 scales and biases."""

    def __init__(self, q, scales, biases, rows: int, K: int):
        self.q = _c(q, np.uint8)
        self.scales = _c(scales, np.uint16)
        self.biases = _c(biases, np.uint16)
        self.rows, self.K = int(rows), int(K)

    def c(self) -> QMat:
        return QMat(self.q.ctypes.data, self.scales.ctypes.data, self.biases.ctypes.data,
                    self.rows, self.K)


def dequant(m: QMatrix, bits: int, group: int) -> np.ndarray:
    out = np.empty((m.rows, m.K), dtype=np.float32)
    cm = m.c()
    _check(lib().orc_dequant(ctypes.byref(cm), bits, group, out.ctypes.data), "dequant")
    return out


def router_logits(x_bits, wr_bits, rbias=None) -> np.ndarray:
    x = _c(np.atleast_2d(x_bits), np.uint16)
    wr = _c(wr_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    assert wr.shape[1] == H
    rb = None if rbias is None else _c(rbias, np.float32)
    out = np.empty((T, E), dtype=np.float64)
    _check(lib().orc_router_logits(x.ctypes.data, T, H, wr.ctypes.data, E, _ptr(rb), out.ctypes.data),
           "router_logits")
    return out


def softmax_topk(logits, k: int, renorm: bool = True):
    lg = _c(logits, np.float64)
    idx = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float64)
    _check(lib().orc_softmax_topk(lg.ctypes.data, lg.shape[0], k, int(renorm), idx.ctypes.data,
                                  w.ctypes.data), "softmax_topk")
    return idx, w


def topk_gap(logits, k: int) -> float:
    """Gap between the k-th and (k+1)-th largest logit (inf when k == E)."""
    s = np.sort(np.asarray(logits, dtype=np.float64))[::-1]
    return float("inf") if k >= s.shape[0] else float(s[k - 1] - s[k])


def shared_gate(x_bits, wsg_bits) -> float:
    x = _c(x_bits, np.uint16)
    w = _c(wsg_bits, np.uint16)
    return float(lib().orc_shared_gate(x.ctypes.data, w.ctypes.data, x.shape[0]))


def expert_ffn(wgu: np.ndarray, wd: np.ndarray, x: np.ndarray):
    """o = Wd (silu(Wg x) * (Wu x)) on dequantised fp32 matrices; returns (o f64, h f32)."""
    wgu = _c(wgu, np.float32)
    wd = _c(wd, np.float32)
    xd = _c(x, np.float64)
    H = xd.shape[0]
    I = wgu.shape[0] // 2
    o = np.empty(H, dtype=np.float64)
    h = np.empty(I, dtype=np.float32)
    _check(lib().orc_expert_ffn(wgu.ctypes.data, wd.ctypes.data, H, I, xd.ctypes.data, o.ctypes.data,
                                h.ctypes.data), "expert_ffn")
    return o, h


def moe_token(H: int, I: int, Is: int, bits: int, group: int, x_bits, gate_up: Sequence[QMatrix],
              down: Sequence[QMatrix], w, shared_gate_up: Optional[QMatrix] = None,
              shared_down: Optional[QMatrix] = None, gate: float = 0.0, threads: int = 1):
    """Routed experts + shared expert for one token; returns (y f64, y f32, y bf16 bits)."""
    x = _c(x_bits, np.uint16)
    n = len(gate_up)
    GU = (QMat * max(n, 1))(*[m.c() for m in gate_up])
    DN = (QMat * max(n, 1))(*[m.c() for m in down])
    wv = _c(w, np.float64)
    sgu = ctypes.byref(shared_gate_up.c()) if shared_gate_up is not None else None
    sdn = ctypes.byref(shared_down.c()) if shared_down is not None else None
    y64 = np.empty(H, dtype=np.float64)
    y32 = np.empty(H, dtype=np.float32)
    y16 = np.empty(H, dtype=np.uint16)
    _check(lib().orc_moe_token(H, I, Is if shared_gate_up is not None else 0, bits, group, x.ctypes.data,
                               n, GU, DN, wv.ctypes.data, sgu, sdn, float(gate), y64.ctypes.data,
                               y32.ctypes.data, y16.ctypes.data, int(threads)), "moe_token")
    return y64, y32, y16


def sort_by_expert(idx, E: int, with_shared: bool = True):
    ix = _c(np.atleast_2d(idx), np.int32)
    T, k = ix.shape
    n = T * k + (T if with_shared else 0)
    perm = np.empty(n, dtype=np.int32)
    offsets = np.empty(E + (2 if with_shared else 1), dtype=np.int32)
    _check(lib().orc_sort_by_expert(ix.ctypes.data, T, k, E, int(with_shared), perm.ctypes.data,
                                    offsets.ctypes.data), "sort_by_expert")
    return perm, offsets


def residual_rmsnorm(r, y_bits, eps: float = 1e-6):
    rr = _c(np.atleast_2d(r), np.float64)
    yy = _c(np.atleast_2d(y_bits), np.uint16)
    T, H = rr.shape
    r_out = np.empty_like(rr)
    x_out = np.empty((T, H), dtype=np.uint16)
    _check(lib().orc_residual_rmsnorm(rr.ctypes.data, yy.ctypes.data, T, H, float(eps), r_out.ctypes.data,
                                      x_out.ctypes.data), "residual_rmsnorm")
    return r_out, x_out


class HostLayer:
    """A layer's weights as host numpy arrays (bf16 as uint16 bit patterns).

    gate_up / down / shared_* are (q, scales, biases) with a leading expert
    axis; `expert(e)` returns the QMatrix pair of expert e. Subclasses may
    fetch experts lazily (e.g. from device memory) by overriding `expert`.
    """

    def __init__(self, H, E, k, I, Is, bits, group, router_w, router_bias, gate_up, down,
                 shared_gate_up=None, shared_down=None, shared_gate_w=None):
        self.H, self.E, self.k, self.I, self.Is = H, E, k, I, Is
        self.bits, self.group = bits, group
        self.router_w = _c(router_w, np.uint16)
        self.router_bias = None if router_bias is None else _c(router_bias, np.float32)
        self.gate_up, self.down = gate_up, down
        self.shared_gate_up, self.shared_down = shared_gate_up, shared_down
        self.shared_gate_w = None if shared_gate_w is None else _c(shared_gate_w, np.uint16)

    def expert(self, e: int):
        gq, gs, gb = self.gate_up
        dq, ds, db = self.down
        return (QMatrix(gq[e], gs[e], gb[e], 2 * self.I, self.H),
                QMatrix(dq[e], ds[e], db[e], self.H, self.I))

    def shared(self):
        if self.shared_gate_up is None or self.Is == 0:
            return None, None
        gq, gs, gb = self.shared_gate_up
        dq, ds, db = self.shared_down
        return (QMatrix(gq[0], gs[0], gb[0], 2 * self.Is, self.H),
                QMatrix(dq[0], ds[0], db[0], self.H, self.Is))


def layer_forward(layer: HostLayer, x_bits, force_idx=None, threads: int = 1):
    """Whole layer for T tokens x_bits [T][H] (bf16 bits).

    force_idx [T][k] (optional) replaces the oracle's own selection for the
    expert part (the weights are then the renormalised softmax of the forced
    experts), which lets a caller evaluate the output under another selection.
    Returns dict with logits f64 [T][E], idx [T][k], w f64 [T][k],
    gap [T], gate [T], y64 [T][H], y32 [T][H], y16 [T][H].
    """
    x = _c(np.atleast_2d(x_bits), np.uint16)
    T, H = x.shape
    k = layer.k
    logits = router_logits(x, layer.router_w, layer.router_bias)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    gap = np.empty(T, dtype=np.float64)
    gate = np.zeros(T, dtype=np.float64)
    y64 = np.empty((T, H), dtype=np.float64)
    y32 = np.empty((T, H), dtype=np.float32)
    y16 = np.empty((T, H), dtype=np.uint16)
    sgu, sdn = layer.shared()
    for t in range(T):
        i_t, w_t = softmax_topk(logits[t], k)
        gap[t] = topk_gap(logits[t], k)
        if force_idx is not None:
            fi = np.asarray(force_idx[t], dtype=np.int64)
            sel = logits[t][fi]
            p = np.exp(sel - logits[t].max())
            i_t, w_t = fi.astype(np.int32), p / p.sum()
        idx[t], w[t] = i_t, w_t
        mats = [layer.expert(int(e)) for e in i_t]
        if sgu is not None:
            gate[t] = shared_gate(x[t], layer.shared_gate_w)
        y64[t], y32[t], y16[t] = moe_token(H, layer.I, layer.Is, layer.bits, layer.group, x[t],
                                           [m[0] for m in mats], [m[1] for m in mats], w_t,
                                           sgu, sdn, gate[t], threads)
    return dict(logits=logits, idx=idx, w=w, gap=gap, gate=gate, y64=y64, y32=y32, y16=y16)
