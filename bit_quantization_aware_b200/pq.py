"""Thin ctypes binding over the C ABI in ``include/pq.h`` (``lib/libpq.so``).

Argument marshalling only: every step of the quantizer runs in the CUDA
kernels of the library. Tensors are passed as device pointers; torch is used
for device memory and streams. There is no CPU fallback: loading fails
loudly when the library is missing.

Function names match the C entry points. Each takes torch tensors (CUDA,
contiguous) and an optional stream (torch.cuda.Stream or a raw cudaStream_t
int; default: torch's current stream), and raises ``PQError`` on a non-OK
status.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libpq.so")

PQ_BINARY, PQ_TERNARY, PQ_SEQ2, PQ_SEQ2_B, PQ_LSQ2, PQ_LSQ3, PQ_LSQ4 = range(1, 8)
QUANTIZERS = {"binary": PQ_BINARY, "ternary": PQ_TERNARY, "seq2": PQ_SEQ2,
              "seq2_b": PQ_SEQ2_B, "lsq2": PQ_LSQ2, "lsq3": PQ_LSQ3,
              "lsq4": PQ_LSQ4}
PQ_OK, PQ_ERR_INVALID_ARG, PQ_ERR_UNSUPPORTED, PQ_ERR_MISALIGNED, \
    PQ_ERR_CUDA, PQ_ERR_TIMEOUT = range(6)

_lock = threading.Lock()
_lib = None


class PQError(RuntimeError):
    def __init__(self, fn, status, cuda_err=0):
        msg = f"{fn}: status {status} ({status_string(status)})"
        if status == PQ_ERR_CUDA:
            msg += f", cudaError {cuda_err}"
        super().__init__(msg)
        self.status = status


class PQMatrix(ctypes.Structure):
    """``pq_matrix_t``: one weight matrix of a batched call (device pointers)."""
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("w", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("wq_bf16_out", ctypes.c_void_p), ("packed_out", ctypes.c_void_p),
                ("g_bf16", ctypes.c_void_p), ("dw_out", ctypes.c_void_p),
                ("dalpha_out", ctypes.c_void_p), ("grad_scale", ctypes.c_float)]


class PQAdamW(ctypes.Structure):
    """``pq_adamw_t``: hyperparameters of one AdamW step (step >= 1)."""
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("weight_decay", ctypes.c_double), ("step", ctypes.c_int64)]


class PQAdamWMatrix(ctypes.Structure):
    """``pq_adamw_matrix_t``: one matrix of the fused backward + AdamW."""
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("w", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("g_bf16", ctypes.c_void_p), ("m_w", ctypes.c_void_p),
                ("v_w", ctypes.c_void_p), ("m_alpha", ctypes.c_void_p),
                ("v_alpha", ctypes.c_void_p), ("dalpha_out", ctypes.c_void_p),
                ("grad_scale", ctypes.c_float)]


class PQShard(ctypes.Structure):
    """``pq_shard_t``: one row shard of a matrix owned by this GPU."""
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("w", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("m_w", ctypes.c_void_p), ("v_w", ctypes.c_void_p),
                ("m_alpha", ctypes.c_void_p), ("v_alpha", ctypes.c_void_p),
                ("dalpha_out", ctypes.c_void_p), ("g_offset", ctypes.c_int64),
                ("grad_scale", ctypes.c_float)]


class PQGemmProblem(ctypes.Structure):
    """``pq_gemm_problem_t``: one matrix of a grouped weight-only matmul."""
    _fields_ = [("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("x_bf16", ctypes.c_void_p), ("packed", ctypes.c_void_p),
                ("alpha", ctypes.c_void_p), ("y_bf16", ctypes.c_void_p)]


class PQIpcHandle(ctypes.Structure):
    """``pq_ipc_handle_t``: a CUDA IPC handle of one device allocation."""
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


def _declare(L):
    i64, p, i32, f32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.pq_fakequant_fwd_batch.argtypes = [i32, i32, ctypes.POINTER(PQMatrix), p]
    L.pq_fakequant_fwd_batch.restype = i32
    L.pq_fakequant_bwd_batch.argtypes = [i32, i32, ctypes.POINTER(PQMatrix), p]
    L.pq_fakequant_bwd_batch.restype = i32
    L.pq_fakequant_bwd_adamw.argtypes = [i32, i32, ctypes.POINTER(PQAdamWMatrix),
                                         ctypes.POINTER(PQAdamW), ctypes.POINTER(PQAdamW), p]
    L.pq_fakequant_bwd_adamw.restype = i32
    L.pq_reduce_bwd_adamw.argtypes = [i32, i32, ctypes.POINTER(ctypes.c_void_p), f32, i32,
                                      ctypes.POINTER(PQShard), ctypes.POINTER(PQAdamW),
                                      ctypes.POINTER(PQAdamW), p]
    L.pq_reduce_bwd_adamw.restype = i32
    L.pq_wq_gemm.argtypes = [i32, i64, i64, i64, p, p, p, p, p, i64, p]
    L.pq_wq_gemm.restype = i32
    L.pq_wq_gemm_batch.argtypes = [i32, i64, i32, ctypes.POINTER(PQGemmProblem), p, i64, p]
    L.pq_wq_gemm_batch.restype = i32
    L.pq_wq_gemm_batch_workspace_bytes.argtypes = [i32, i64, i32, ctypes.POINTER(PQGemmProblem)]
    L.pq_wq_gemm_batch_workspace_bytes.restype = i64
    L.pq_wq_gemm_noalloc.argtypes = [i32, i64, i64, i64, p, p, p, p, p]
    L.pq_wq_gemm_noalloc.restype = i32
    L.pq_wq_gemm_workspace_bytes.argtypes = [i32, i64, i64, i64]
    L.pq_wq_gemm_workspace_bytes.restype = i64
    L.pq_device_status.argtypes = []
    L.pq_device_status.restype = i32
    L.pq_launch_count.argtypes = []
    L.pq_launch_count.restype = i64
    L.pq_ipc_export.argtypes = [p, ctypes.POINTER(PQIpcHandle), ctypes.POINTER(ctypes.c_int64)]
    L.pq_ipc_export.restype = i32
    L.pq_ipc_open.argtypes = [ctypes.POINTER(PQIpcHandle), ctypes.POINTER(ctypes.c_void_p)]
    L.pq_ipc_open.restype = i32
    L.pq_ipc_close.argtypes = [p]
    L.pq_ipc_close.restype = i32
    L.pq_debug_abort_waits.argtypes = [i32]
    L.pq_debug_abort_waits.restype = i32
    L.pq_dequant_codes_batch.argtypes = [i32, i32, ctypes.POINTER(PQMatrix), p]
    L.pq_dequant_codes_batch.restype = i32
    L.pq_dequant_codes.argtypes = [i32, i64, i64, p, p, p, p]
    L.pq_dequant_codes.restype = i32
    L.pq_scaled_weights.argtypes = [i64, i64, p, p, p, p]
    L.pq_scaled_weights.restype = i32
    L.pq_fakequant_fwd.argtypes = [i32, i64, i64, p, p, p, p, p]
    L.pq_fakequant_fwd.restype = i32
    L.pq_fakequant_bwd.argtypes = [i32, i64, i64, p, p, p, p, p, f32, p]
    L.pq_fakequant_bwd.restype = i32
    L.pq_pack_codes.argtypes = [i32, i64, i64, p, p, p, p]
    L.pq_pack_codes.restype = i32
    L.pq_code_bits.argtypes = [i32]
    L.pq_code_bits.restype = i32
    L.pq_default_grad_scale.argtypes = [i32, i64]
    L.pq_default_grad_scale.restype = f32
    L.pq_status_string.argtypes = [i32]
    L.pq_status_string.restype = ctypes.c_char_p
    L.pq_last_cuda_error.argtypes = []
    L.pq_last_cuda_error.restype = i32
    return L


def lib(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise ImportError(
                    f"CUDA library {path} is missing; build it with "
                    "`python -m bit_quantization_aware_b200.build` (there is no "
                    "CPU fallback)")
            _lib = _declare(ctypes.CDLL(path))
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, status):
    if status != PQ_OK:
        raise PQError(fn, status, lib().pq_last_cuda_error())


def _shape(w, rows, cols):
    if rows is None or cols is None:
        rows, cols = w.shape
    return int(rows), int(cols)


def pq_fakequant_fwd(q, w, alpha, wq_out, packed_out=None, stream=None,
                     rows=None, cols=None):
    """Forward: ``wq_out`` (bf16 [rows, cols]) and optional ``packed_out``
    (uint8 [rows, cols*bits/8])."""
    rows, cols = _shape(w, rows, cols)
    _check("pq_fakequant_fwd", lib().pq_fakequant_fwd(
        q, rows, cols, _ptr(w), _ptr(alpha), _ptr(wq_out), _ptr(packed_out),
        _stream(stream)))


def pq_fakequant_bwd(q, w, alpha, g, dw_out, dalpha_out, grad_scale,
                     stream=None, rows=None, cols=None):
    """Backward: ``dw_out`` (fp32 [rows, cols]) and ``dalpha_out`` (fp32
    [rows]) from the bf16 upstream gradient ``g``."""
    rows, cols = _shape(w, rows, cols)
    _check("pq_fakequant_bwd", lib().pq_fakequant_bwd(
        q, rows, cols, _ptr(w), _ptr(alpha), _ptr(g), _ptr(dw_out),
        _ptr(dalpha_out), ctypes.c_float(grad_scale), _stream(stream)))


def pq_pack_codes(q, w, alpha, packed_out, stream=None, rows=None, cols=None):
    """Packed code export only."""
    rows, cols = _shape(w, rows, cols)
    _check("pq_pack_codes", lib().pq_pack_codes(
        q, rows, cols, _ptr(w), _ptr(alpha), _ptr(packed_out),
        _stream(stream)))


def pq_dequant_codes(q, packed, alpha, wq_out, stream=None, rows=None, cols=None):
    """bf16 weights [rows, cols] from packed codes [rows, cols*bits/8]."""
    if rows is None or cols is None:
        rows, cols = wq_out.shape
    _check("pq_dequant_codes", lib().pq_dequant_codes(
        q, int(rows), int(cols), _ptr(packed), _ptr(alpha), _ptr(wq_out),
        _stream(stream)))


def pq_dequant_codes_batch(q, mats, stream=None):
    """Dequantization over a ``pq_matrix_t[]`` (packed read, wq written)."""
    _check("pq_dequant_codes_batch", lib().pq_dequant_codes_batch(
        q, len(mats), mats, _stream(stream)))


def pq_scaled_weights(w, alpha, x_out, stream=None, rows=None, cols=None):
    """x = fl(w / alpha_row) (fp32 [rows, cols])."""
    rows, cols = _shape(w, rows, cols)
    _check("pq_scaled_weights", lib().pq_scaled_weights(
        rows, cols, _ptr(w), _ptr(alpha), _ptr(x_out), _stream(stream)))


def matrix_array(descs):
    """Build a ``pq_matrix_t[]`` from dicts with keys rows, cols, w, alpha,
    wq, packed, g, dw, dalpha, grad_scale (tensors or raw pointers; missing
    keys are NULL / 0)."""
    arr = (PQMatrix * len(descs))()
    for i, d in enumerate(descs):
        m = arr[i]
        m.rows, m.cols = int(d["rows"]), int(d["cols"])
        m.w, m.alpha = _ptr(d.get("w")), _ptr(d.get("alpha"))
        m.wq_bf16_out, m.packed_out = _ptr(d.get("wq")), _ptr(d.get("packed"))
        m.g_bf16, m.dw_out = _ptr(d.get("g")), _ptr(d.get("dw"))
        m.dalpha_out = _ptr(d.get("dalpha"))
        m.grad_scale = float(d.get("grad_scale", 0.0))
    return arr


def pq_fakequant_fwd_batch(q, mats, stream=None):
    """Forward over a ``pq_matrix_t[]`` (see ``matrix_array``)."""
    _check("pq_fakequant_fwd_batch", lib().pq_fakequant_fwd_batch(
        q, len(mats), mats, _stream(stream)))


def pq_fakequant_bwd_batch(q, mats, stream=None):
    """Backward over a ``pq_matrix_t[]`` (see ``matrix_array``)."""
    _check("pq_fakequant_bwd_batch", lib().pq_fakequant_bwd_batch(
        q, len(mats), mats, _stream(stream)))


def adamw_matrix_array(descs):
    """Build a ``pq_adamw_matrix_t[]`` from dicts with keys rows, cols, w,
    alpha, g, m_w, v_w, m_alpha, v_alpha, dalpha (optional), grad_scale."""
    arr = (PQAdamWMatrix * len(descs))()
    for i, d in enumerate(descs):
        m = arr[i]
        m.rows, m.cols = int(d["rows"]), int(d["cols"])
        m.w, m.alpha, m.g_bf16 = _ptr(d.get("w")), _ptr(d.get("alpha")), _ptr(d.get("g"))
        m.m_w, m.v_w = _ptr(d.get("m_w")), _ptr(d.get("v_w"))
        m.m_alpha, m.v_alpha = _ptr(d.get("m_alpha")), _ptr(d.get("v_alpha"))
        m.dalpha_out = _ptr(d.get("dalpha"))
        m.grad_scale = float(d.get("grad_scale", 0.0))
    return arr


def adamw(step, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
    return PQAdamW(lr, beta1, beta2, eps, weight_decay, step)


def pq_fakequant_bwd_adamw(q, mats, hp_w, hp_alpha, stream=None):
    """Backward fused with one AdamW step over a ``pq_adamw_matrix_t[]``."""
    _check("pq_fakequant_bwd_adamw", lib().pq_fakequant_bwd_adamw(
        q, len(mats), mats, ctypes.byref(hp_w), ctypes.byref(hp_alpha),
        _stream(stream)))


def shard_array(descs):
    """Build a ``pq_shard_t[]`` from dicts with keys rows, cols, w, alpha,
    m_w, v_w, m_alpha, v_alpha, dalpha (optional), g_offset, grad_scale."""
    arr = (PQShard * len(descs))()
    for i, d in enumerate(descs):
        m = arr[i]
        m.rows, m.cols = int(d["rows"]), int(d["cols"])
        m.w, m.alpha = _ptr(d.get("w")), _ptr(d.get("alpha"))
        m.m_w, m.v_w = _ptr(d.get("m_w")), _ptr(d.get("v_w"))
        m.m_alpha, m.v_alpha = _ptr(d.get("m_alpha")), _ptr(d.get("v_alpha"))
        m.dalpha_out = _ptr(d.get("dalpha"))
        m.g_offset = int(d.get("g_offset", 0))
        m.grad_scale = float(d.get("grad_scale", 0.0))
    return arr


def pq_reduce_bwd_adamw(q, g_sources, grad_mult, shards, hp_w, hp_alpha, stream=None):
    """Reduce over replicas' bf16 gradients fused with backward + AdamW.
    ``g_sources``: device pointers (ints) or CUDA tensors, one per replica."""
    srcs = (ctypes.c_void_p * len(g_sources))(*[_ptr(g) for g in g_sources])
    _check("pq_reduce_bwd_adamw", lib().pq_reduce_bwd_adamw(
        q, len(g_sources), srcs, ctypes.c_float(grad_mult), len(shards), shards,
        ctypes.byref(hp_w), ctypes.byref(hp_alpha), _stream(stream)))


def pq_wq_gemm_workspace_bytes(q, m, n, k) -> int:
    return int(lib().pq_wq_gemm_workspace_bytes(q, m, n, k))


def pq_wq_gemm(q, x, packed, alpha, y_out, workspace=None, stream=None):
    """Y = X (alpha * levels(codes))^T; x bf16 [m, k], packed uint8 [n, k/4],
    alpha fp32 [n], y_out bf16 [m, n]. Tensor cores (integer mode for
    m <= 16, bf16 beyond), one row times this one matrix on the CUDA cores;
    include/pq.h states each mode's arithmetic and error bound."""
    m, k = x.shape
    n = packed.shape[0]
    if (packed.dim() != 2 or packed.shape[1] * 8 != k * pq_code_bits(q)
            or alpha.numel() != n or tuple(y_out.shape) != (m, n)
            or not (x.is_contiguous() and packed.is_contiguous() and y_out.is_contiguous())):
        raise ValueError("pq_wq_gemm: shapes must be x [m, k], packed [n, k*bits/8], "
                         "alpha [n], y_out [m, n], all contiguous")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pq_wq_gemm", lib().pq_wq_gemm(
        q, m, n, k, _ptr(x), _ptr(packed), _ptr(alpha), _ptr(y_out), _ptr(workspace),
        ws_bytes, _stream(stream)))


def gemm_problem_array(descs):
    """Build a ``pq_gemm_problem_t[]`` from dicts with keys x (bf16 [m, k]),
    packed (uint8 [n, k/4]), alpha (fp32 [n]) and y (bf16 [m, n])."""
    arr = (PQGemmProblem * len(descs))()
    for i, d in enumerate(descs):
        pr = arr[i]
        pr.n, pr.k = int(d["packed"].shape[0]), int(d["x"].shape[1])
        pr.x_bf16, pr.packed = _ptr(d["x"]), _ptr(d["packed"])
        pr.alpha, pr.y_bf16 = _ptr(d["alpha"]), _ptr(d["y"])
    return arr


def pq_wq_gemm_batch_workspace_bytes(q, m, problems) -> int:
    return int(lib().pq_wq_gemm_batch_workspace_bytes(q, m, len(problems), problems))


def pq_wq_gemm_batch(q, m, problems, workspace=None, stream=None):
    """Grouped weight-only matmul over a ``pq_gemm_problem_t[]`` (see
    ``gemm_problem_array``); all matrices share q and the activation rows m."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("pq_wq_gemm_batch", lib().pq_wq_gemm_batch(
        q, m, len(problems), problems, _ptr(workspace), ws_bytes, _stream(stream)))


def wq_gemm_batch(q, xs, packeds, alphas, stream=None):
    """Allocate outputs and workspace and run pq_wq_gemm_batch; returns the
    list of Y (bf16 [m, n])."""
    m = xs[0].shape[0]
    ys = [torch.empty((m, pk.shape[0]), dtype=torch.bfloat16, device=pk.device) for pk in packeds]
    arr = gemm_problem_array([dict(x=x, packed=pk, alpha=a, y=y)
                              for x, pk, a, y in zip(xs, packeds, alphas, ys)])
    need = pq_wq_gemm_batch_workspace_bytes(q, m, arr)
    if need < 0:
        raise PQError("pq_wq_gemm_batch_workspace_bytes", PQ_ERR_INVALID_ARG)
    ws = torch.empty(need, dtype=torch.uint8, device=xs[0].device) if need > 0 else None
    pq_wq_gemm_batch(q, m, arr, ws, stream)
    return ys


WQ_GEMM_NOALLOC_SCRATCH_BYTES = 8 << 20  # PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES


def pq_wq_gemm_noalloc(q, x, packed, alpha, y_out, stream=None):
    """pq_wq_gemm with the library's fixed split-K scratch: allocates nothing,
    on the device or through torch. Problems needing more than
    WQ_GEMM_NOALLOC_SCRATCH_BYTES of scratch are rejected; calls that may
    overlap on the GPU race on the shared scratch."""
    m, k = x.shape
    n = packed.shape[0]
    if (packed.dim() != 2 or packed.shape[1] * 8 != k * pq_code_bits(q)
            or alpha.numel() != n or tuple(y_out.shape) != (m, n)
            or not (x.is_contiguous() and packed.is_contiguous() and y_out.is_contiguous())):
        raise ValueError("pq_wq_gemm_noalloc: shapes must be x [m, k], packed [n, k*bits/8], "
                         "alpha [n], y_out [m, n], all contiguous")
    status = lib().pq_wq_gemm_noalloc(q, m, n, k, _ptr(x), _ptr(packed), _ptr(alpha),
                                      _ptr(y_out), _stream(stream))
    if status == PQ_ERR_UNSUPPORTED:
        need = pq_wq_gemm_workspace_bytes(q, m, n, k)
        if need > WQ_GEMM_NOALLOC_SCRATCH_BYTES:
            raise PQError(f"pq_wq_gemm_noalloc (needs {need} B of split-K scratch, over the "
                          f"fixed {WQ_GEMM_NOALLOC_SCRATCH_BYTES} B; use pq_wq_gemm)", status)
    _check("pq_wq_gemm_noalloc", status)


def pq_device_status() -> int:
    """PQ_OK, or PQ_ERR_TIMEOUT once after a bounded device wait gave up."""
    return int(lib().pq_device_status())


def ipc_export(t):
    """(handle bytes, byte offset) of the device allocation holding the
    contiguous CUDA tensor ``t`` (pq_ipc_export)."""
    h = PQIpcHandle()
    off = ctypes.c_int64()
    _check("pq_ipc_export", lib().pq_ipc_export(_ptr(t), ctypes.byref(h), ctypes.byref(off)))
    return bytes(h.bytes), int(off.value)


def ipc_open(handle: bytes) -> int:
    """Maps another process's exported allocation; returns its base address
    in this process (pq_ipc_open)."""
    h = PQIpcHandle()
    ctypes.memmove(h.bytes, handle, 64)
    base = ctypes.c_void_p()
    _check("pq_ipc_open", lib().pq_ipc_open(ctypes.byref(h), ctypes.byref(base)))
    return int(base.value)


def ipc_close(base: int) -> None:
    """Unmaps a base returned by ``ipc_open`` (pq_ipc_close)."""
    _check("pq_ipc_close", lib().pq_ipc_close(base))


def pq_launch_count() -> int:
    """Kernel launches the library has enqueued since it was loaded (the
    launches of a call are the difference of two readings)."""
    return int(lib().pq_launch_count())


def pq_debug_abort_waits(on: bool) -> None:
    """Test switch: later matmul launches give up their waits at once."""
    _check("pq_debug_abort_waits", lib().pq_debug_abort_waits(1 if on else 0))


def wq_gemm(q, x, packed, alpha, stream=None):
    """Allocate the output and workspace and run pq_wq_gemm."""
    m, k = x.shape
    n = packed.shape[0]
    y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    need = pq_wq_gemm_workspace_bytes(q, m, n, k)
    if need < 0:
        raise PQError("pq_wq_gemm_workspace_bytes", PQ_ERR_UNSUPPORTED)
    ws = torch.empty(need, dtype=torch.uint8, device=x.device) if need > 0 else None
    pq_wq_gemm(q, x, packed, alpha, y, ws, stream)
    return y


def pq_code_bits(q) -> int:
    return int(lib().pq_code_bits(q))


def pq_default_grad_scale(q, cols) -> float:
    return float(lib().pq_default_grad_scale(q, cols))


def status_string(status) -> str:
    return lib().pq_status_string(status).decode()


# --------------------------------------------------------------- conveniences
def fakequant_fwd(q, w, alpha, pack=False, stream=None):
    """Allocate outputs and run the forward; returns (wq bf16, packed|None)."""
    rows, cols = w.shape
    wq = torch.empty((rows, cols), dtype=torch.bfloat16, device=w.device)
    packed = (torch.empty((rows, cols * pq_code_bits(q) // 8), dtype=torch.uint8,
                          device=w.device) if pack else None)
    pq_fakequant_fwd(q, w, alpha, wq, packed, stream)
    return wq, packed


def fakequant_bwd(q, w, alpha, g, grad_scale=None, stream=None):
    """Allocate outputs and run the backward; returns (dw fp32, dalpha fp32)."""
    rows, cols = w.shape
    if grad_scale is None:
        grad_scale = pq_default_grad_scale(q, cols)
    dw = torch.empty((rows, cols), dtype=torch.float32, device=w.device)
    da = torch.empty((rows,), dtype=torch.float32, device=w.device)
    pq_fakequant_bwd(q, w, alpha, g, dw, da, grad_scale, stream)
    return dw, da
