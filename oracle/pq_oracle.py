"""Python access to the CPU oracle of the weight fake-quantizer.

TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's CPU
baseline leg call this module; the product path never imports it. The oracle
itself is the plain C file next to this one (``pq_oracle.c``); this module
compiles it with gcc on first use (no FMA contraction, no fast-math) and wraps
its functions for numpy arrays.

Quantizer arithmetic lives only in the C file; this wrapper marshals arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "pq_oracle.c")
_LIB = os.path.join(_HERE, "libpq_oracle.so")
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
          "-shared", "-fPIC", "-Wall", "-Wextra"]

# Quantizer identifiers (same numbering as the library's C ABI).
BINARY, TERNARY, SEQ2, SEQ2_B, LSQ2, LSQ3, LSQ4 = 1, 2, 3, 4, 5, 6, 7
ALL_QUANTIZERS = (BINARY, TERNARY, SEQ2, SEQ2_B, LSQ2, LSQ3, LSQ4)

_lock = threading.Lock()
_default = None


def compile_source(src: str, out: str) -> str:
    """Compile an oracle C source into a shared library at ``out``."""
    tmp = out + f".{os.getpid()}.tmp"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle into ``libpq_oracle.so`` (if missing or stale)."""
    stale = (not os.path.exists(_LIB)
             or os.path.getmtime(_LIB) < os.path.getmtime(SRC))
    if force or stale:
        compile_source(SRC, _LIB)
    return _LIB


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class AdamW(ctypes.Structure):
    """Hyperparameters of one AdamW step (t >= 1 is the step count)."""
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("weight_decay", ctypes.c_double), ("step", ctypes.c_int64)]

    @classmethod
    def at_step(cls, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
        return cls(lr, beta1, beta2, eps, weight_decay, t)


class Oracle:
    """One loaded copy of the oracle library."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        L.pqo_fwd.argtypes = [ctypes.c_int, i64, i64, p, p, p, p, p]
        L.pqo_fwd.restype = ctypes.c_int
        L.pqo_bwd.argtypes = [ctypes.c_int, i64, i64, p, p, p, p, p,
                              ctypes.c_float, p]
        L.pqo_bwd.restype = ctypes.c_int
        L.pqo_pack.argtypes = [ctypes.c_int, i64, i64, p, p, p]
        L.pqo_pack.restype = ctypes.c_int
        L.pqo_dequant.argtypes = [ctypes.c_int, i64, i64, p, p, p]
        L.pqo_dequant.restype = ctypes.c_int
        L.pqo_bwd_adamw.argtypes = [ctypes.c_int, i64, i64, p, p, p, p, p, p, p,
                                    ctypes.c_float, ctypes.POINTER(AdamW),
                                    ctypes.POINTER(AdamW), p]
        L.pqo_bwd_adamw.restype = ctypes.c_int
        L.pqo_reduce_bwd_adamw.argtypes = [ctypes.c_int, i64, i64, p, p, ctypes.c_int, p,
                                           ctypes.c_float, p, p, p, p, ctypes.c_float,
                                           ctypes.POINTER(AdamW), ctypes.POINTER(AdamW), p, p]
        L.pqo_reduce_bwd_adamw.restype = ctypes.c_int
        L.pqo_wq_matmul.argtypes = [ctypes.c_int, i64, i64, i64, p, p, p, p]
        L.pqo_wq_matmul.restype = ctypes.c_int
        L.pqo_adamw_step.argtypes = [i64, p, p, p, p, ctypes.POINTER(AdamW)]
        L.pqo_adamw_step.restype = ctypes.c_int
        L.pqo_default_grad_scale.argtypes = [ctypes.c_int, i64]
        L.pqo_default_grad_scale.restype = ctypes.c_float
        L.pqo_code_bits.argtypes = [ctypes.c_int]
        L.pqo_code_bits.restype = ctypes.c_int
        L.pqo_bf16_rne.argtypes = [ctypes.c_float]
        L.pqo_bf16_rne.restype = ctypes.c_uint16
        L.pqo_quantize_scalar.argtypes = [
            ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_float,
            ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float),
            ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int),
            ctypes.POINTER(ctypes.c_float)]
        L.pqo_quantize_scalar.restype = ctypes.c_int
        self.lib = L
        self.path = path

    def code_bits(self, q: int) -> int:
        return int(self.lib.pqo_code_bits(q))

    def fwd(self, q: int, w, alpha, pack: bool = False):
        """Returns (wq_bf16 bits uint16 [R,C], codes int8 [R,C], packed uint8
        [R, C*bits/8] or None)."""
        w = np.ascontiguousarray(w, np.float32)
        rows, cols = w.shape
        alpha = np.ascontiguousarray(alpha, np.float32).reshape(rows)
        wq = np.empty((rows, cols), np.uint16)
        codes = np.empty((rows, cols), np.int8)
        packed = (np.empty((rows, cols * self.code_bits(q) // 8), np.uint8)
                  if pack else None)
        rc = self.lib.pqo_fwd(q, rows, cols, _ptr(w), _ptr(alpha), _ptr(wq),
                              _ptr(codes), _ptr(packed))
        if rc != 0:
            raise ValueError(f"oracle fwd rejected q={q} shape={w.shape} "
                             f"pack={pack}")
        return wq, codes, packed

    def bwd(self, q: int, w, alpha, g_bf16, grad_scale: float):
        """Returns (dw fp32 [R,C], dalpha fp32 [R], row_abs fp64 [R]) where
        row_abs is the per-row sum of |term| before grad_scale."""
        w = np.ascontiguousarray(w, np.float32)
        rows, cols = w.shape
        alpha = np.ascontiguousarray(alpha, np.float32).reshape(rows)
        g = np.ascontiguousarray(g_bf16).view(np.uint16)
        assert g.shape == w.shape
        dw = np.empty((rows, cols), np.float32)
        da = np.empty(rows, np.float32)
        row_abs = np.empty(rows, np.float64)
        rc = self.lib.pqo_bwd(q, rows, cols, _ptr(w), _ptr(alpha), _ptr(g),
                              _ptr(dw), _ptr(da), ctypes.c_float(grad_scale),
                              _ptr(row_abs))
        if rc != 0:
            raise ValueError(f"oracle bwd rejected q={q}")
        return dw, da, row_abs

    def pack(self, q: int, w, alpha):
        w = np.ascontiguousarray(w, np.float32)
        rows, cols = w.shape
        alpha = np.ascontiguousarray(alpha, np.float32).reshape(rows)
        out = np.empty((rows, cols * self.code_bits(q) // 8), np.uint8)
        rc = self.lib.pqo_pack(q, rows, cols, _ptr(w), _ptr(alpha), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle pack rejected q={q} shape={w.shape}")
        return out

    def dequant(self, q: int, packed, alpha, cols: int):
        """bf16 bits [R, cols] from packed codes [R, cols*bits/8]."""
        packed = np.ascontiguousarray(packed, np.uint8)
        rows = packed.shape[0]
        alpha = np.ascontiguousarray(alpha, np.float32).reshape(rows)
        out = np.empty((rows, cols), np.uint16)
        rc = self.lib.pqo_dequant(q, rows, cols, _ptr(packed), _ptr(alpha), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle dequant rejected q={q} cols={cols}")
        return out

    def bwd_adamw(self, q, w, alpha, g_bf16, m_w, v_w, m_a, v_a, grad_scale,
                  hw, ha):
        """Fused backward + AdamW on copies; returns (w, alpha, m_w, v_w, m_a,
        v_a, dalpha), all fp32."""
        w = np.array(w, np.float32, order="C", copy=True)
        rows, cols = w.shape
        alpha = np.array(alpha, np.float32, copy=True).reshape(rows)
        g = np.ascontiguousarray(g_bf16).view(np.uint16)
        m_w = np.array(m_w, np.float32, order="C", copy=True)
        v_w = np.array(v_w, np.float32, order="C", copy=True)
        m_a = np.array(m_a, np.float32, copy=True).reshape(rows)
        v_a = np.array(v_a, np.float32, copy=True).reshape(rows)
        da = np.empty(rows, np.float32)
        rc = self.lib.pqo_bwd_adamw(q, rows, cols, _ptr(w), _ptr(alpha), _ptr(g),
                                    _ptr(m_w), _ptr(v_w), _ptr(m_a), _ptr(v_a),
                                    ctypes.c_float(grad_scale), ctypes.byref(hw),
                                    ctypes.byref(ha), _ptr(da))
        if rc != 0:
            raise ValueError("oracle bwd_adamw rejected its arguments")
        return w, alpha, m_w, v_w, m_a, v_a, da

    def reduce_bwd_adamw(self, q, w, alpha, g_list, grad_mult, m_w, v_w, m_a, v_a,
                         grad_scale, hw, ha):
        """Backward + AdamW with the upstream gradient summed over the bf16
        arrays of g_list; returns (w, alpha, m_w, v_w, m_a, v_a, dalpha,
        row_abs), row_abs the per-row sum of |term| before grad_scale."""
        w = np.array(w, np.float32, order="C", copy=True)
        rows, cols = w.shape
        alpha = np.array(alpha, np.float32, copy=True).reshape(rows)
        gs = [np.ascontiguousarray(g).view(np.uint16) for g in g_list]
        ptrs = (ctypes.c_void_p * len(gs))(*[g.ctypes.data for g in gs])
        m_w = np.array(m_w, np.float32, order="C", copy=True)
        v_w = np.array(v_w, np.float32, order="C", copy=True)
        m_a = np.array(m_a, np.float32, copy=True).reshape(rows)
        v_a = np.array(v_a, np.float32, copy=True).reshape(rows)
        da = np.empty(rows, np.float32)
        row_abs = np.empty(rows, np.float64)
        rc = self.lib.pqo_reduce_bwd_adamw(q, rows, cols, _ptr(w), _ptr(alpha), len(gs),
                                           ctypes.cast(ptrs, ctypes.c_void_p),
                                           ctypes.c_float(grad_mult), _ptr(m_w), _ptr(v_w),
                                           _ptr(m_a), _ptr(v_a), ctypes.c_float(grad_scale),
                                           ctypes.byref(hw), ctypes.byref(ha), _ptr(da),
                                           _ptr(row_abs))
        if rc != 0:
            raise ValueError("oracle reduce_bwd_adamw rejected its arguments")
        return w, alpha, m_w, v_w, m_a, v_a, da, row_abs

    def wq_matmul(self, q, x_bf16, packed, alpha, k):
        """Y = X * (alpha * levels(codes))^T in fp64; x_bf16 [M, K] bits,
        packed [N, K*bits/8]."""
        x = np.ascontiguousarray(x_bf16).view(np.uint16)
        packed = np.ascontiguousarray(packed, np.uint8)
        m, n = x.shape[0], packed.shape[0]
        alpha = np.ascontiguousarray(alpha, np.float32).reshape(n)
        y = np.empty((m, n), np.float64)
        rc = self.lib.pqo_wq_matmul(q, m, n, k, _ptr(x), _ptr(packed), _ptr(alpha), _ptr(y))
        if rc != 0:
            raise ValueError("oracle wq_matmul rejected its arguments")
        return y

    def adamw_step(self, p, g, m, v, h):
        """One AdamW step on copies of fp32 arrays; returns (p, m, v)."""
        p = np.array(p, np.float32, copy=True).ravel()
        g = np.ascontiguousarray(g, np.float32).ravel()
        m = np.array(m, np.float32, copy=True).ravel()
        v = np.array(v, np.float32, copy=True).ravel()
        rc = self.lib.pqo_adamw_step(len(p), _ptr(p), _ptr(g), _ptr(m), _ptr(v),
                                     ctypes.byref(h))
        if rc != 0:
            raise ValueError("oracle adamw rejected its arguments")
        return p, m, v

    def quantize_scalar(self, q: int, w: float, alpha: float,
                        clip_hi: float = 0.0):
        """One element: dict(code, level, wq32, inside, x). ``clip_hi`` > 0
        replaces the symmetric SEQ/ternary clip value."""
        c, lev, wq = ctypes.c_int(), ctypes.c_float(), ctypes.c_float()
        ins, x = ctypes.c_int(), ctypes.c_float()
        rc = self.lib.pqo_quantize_scalar(q, w, alpha, clip_hi,
                                          ctypes.byref(c), ctypes.byref(lev),
                                          ctypes.byref(wq), ctypes.byref(ins),
                                          ctypes.byref(x))
        if rc != 0:
            raise ValueError(f"unknown quantizer {q}")
        return dict(code=c.value, level=lev.value, wq32=wq.value,
                    inside=bool(ins.value), x=x.value)

    def bf16_rne(self, f) -> np.ndarray:
        """Elementwise fp32 -> bf16 bits via the oracle's own conversion."""
        f = np.asarray(f, np.float32).ravel()
        return np.array([self.lib.pqo_bf16_rne(float(v)) for v in f],
                        np.uint16)

    def default_grad_scale(self, q: int, cols: int) -> float:
        return float(self.lib.pqo_default_grad_scale(q, cols))


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def fwd(q, w, alpha, pack=False):
    return default().fwd(q, w, alpha, pack)


def bwd(q, w, alpha, g_bf16, grad_scale):
    return default().bwd(q, w, alpha, g_bf16, grad_scale)


def pack(q, w, alpha):
    return default().pack(q, w, alpha)


def quantize_scalar(q, w, alpha, clip_hi=0.0):
    return default().quantize_scalar(q, w, alpha, clip_hi)


def dequant(q, packed, alpha, cols):
    return default().dequant(q, packed, alpha, cols)


def bf16_rne(f):
    return default().bf16_rne(f)


def default_grad_scale(q, cols):
    return default().default_grad_scale(q, cols)


def code_bits(q):
    return default().code_bits(q)


def bf16_bits_to_float(h) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact widening)."""
    return (np.asarray(h).view(np.uint16).astype(np.uint32) << 16).view(np.float32)
