"""The C-ABI library builds, loads and exports every entry point that
include/pq.h declares; host-side argument checks and pure host helpers
behave as documented. No CUDA work is launched (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from bit_quantization_aware_b200 import build as pqbuild
from oracle import pq_oracle

HEADER = os.path.join(pqbuild.INCLUDE, "pq.h")


@pytest.fixture(scope="module")
def L():
    path = pqbuild.build()
    from bit_quantization_aware_b200 import pq
    return pq.lib(path)


def declared():
    src = open(HEADER).read()
    return re.findall(r"^PQ_API\s+[\w\s\*]+?\b(pq_\w+)\s*\(", src, re.M)


def test_header_declares_entry_points():
    names = declared()
    for n in ("pq_fakequant_fwd", "pq_fakequant_bwd", "pq_pack_codes",
              "pq_fakequant_fwd_batch", "pq_fakequant_bwd_batch",
              "pq_scaled_weights", "pq_dequant_codes", "pq_dequant_codes_batch",
              "pq_fakequant_bwd_adamw", "pq_reduce_bwd_adamw",
              "pq_wq_gemm", "pq_wq_gemm_workspace_bytes", "pq_device_status",
              "pq_wq_gemm_noalloc", "pq_wq_gemm_batch", "pq_wq_gemm_batch_workspace_bytes", "pq_debug_abort_waits",
              "pq_status_string", "pq_default_grad_scale", "pq_code_bits",
              "pq_last_cuda_error", "pq_launch_count", "pq_ipc_export", "pq_ipc_open",
              "pq_ipc_close"):
        assert n in names


def test_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", pqbuild.LIB],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in declared():
        assert n in exported, n
        assert hasattr(L, n)
    # nothing but the declared C entry points is exported from our code
    ours = {s for s in exported if s.startswith("pq_")}
    assert ours == set(declared())


def test_sm100a_code_only():
    # the library carries sm_100a machine code (checked through the build
    # command, not by reading the binary)
    assert "arch=compute_100a,code=sm_100a" in " ".join(pqbuild.ARCH)


def test_host_helpers_match_oracle(L):
    from bit_quantization_aware_b200 import pq
    for q in pq_oracle.ALL_QUANTIZERS:
        assert pq.pq_code_bits(q) == pq_oracle.code_bits(q)
        for cols in (1, 1024, 4096, 14336):
            assert pq.pq_default_grad_scale(q, cols) == pytest.approx(
                pq_oracle.default_grad_scale(q, cols), rel=1e-7)
    assert pq.pq_code_bits(0) == 0 and pq.pq_code_bits(99) == 0
    assert pq.pq_default_grad_scale(pq.PQ_SEQ2, 0) == 0.0
    for s in range(6):
        assert pq.status_string(s)
    assert L.pq_last_cuda_error() == 0
    # argument checks that fail launch nothing, so the counter stays put
    n0 = pq.pq_launch_count()
    assert pq.pq_default_grad_scale(pq.PQ_SEQ2, 1024) > 0
    assert L.pq_fakequant_fwd(99, 4, 8, None, None, None, None, None) == pq.PQ_ERR_INVALID_ARG
    assert pq.pq_launch_count() == n0 >= 0


def test_argument_errors_launch_nothing(L):
    from bit_quantization_aware_b200 import pq
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: rejected on host
    f, b, k = L.pq_fakequant_fwd, L.pq_fakequant_bwd, L.pq_pack_codes
    E = pq.PQ_ERR_INVALID_ARG
    assert f(99, 4, 8, fake, fake, fake, None, None) == E       # bad enum
    assert f(pq.PQ_SEQ2, -1, 8, fake, fake, fake, None, None) == E
    assert f(pq.PQ_SEQ2, 4, -8, fake, fake, fake, None, None) == E
    assert f(pq.PQ_SEQ2, 4, 8, fake, fake, None, None, None) == E  # no wq
    assert f(pq.PQ_SEQ2, 4, 8, None, fake, fake, None, None) == E  # no w
    assert f(pq.PQ_SEQ2, 4, 8, fake, None, fake, None, None) == E  # no alpha
    assert f(pq.PQ_SEQ2, 4, 6, fake, fake, fake, fake, None) == E  # cols % 4
    assert f(pq.PQ_LSQ4, 4, 7, fake, fake, fake, fake, None) == E  # cols % 2
    assert k(pq.PQ_SEQ2, 4, 8, fake, fake, None, None) == E        # no packed
    assert b(0, 4, 8, fake, fake, fake, fake, fake, 1.0, None) == E
    assert b(pq.PQ_SEQ2, 4, 8, fake, fake, fake, fake, None, 1.0, None) == E
    assert b(pq.PQ_SEQ2, 4, 8, fake, fake, None, fake, fake, 1.0, None) == E
    # empty inputs are valid and launch nothing
    assert f(pq.PQ_SEQ2, 0, 8, None, None, fake, None, None) == pq.PQ_OK
    assert f(pq.PQ_SEQ2, 4, 0, None, None, fake, None, None) == pq.PQ_OK
    assert k(pq.PQ_LSQ3, 0, 0, None, None, fake, None) == pq.PQ_OK
    assert b(pq.PQ_SEQ2, 0, 8, None, None, None, None, None, 1.0, None) == pq.PQ_OK
    dq = L.pq_dequant_codes
    assert dq(99, 4, 8, fake, fake, fake, None) == E
    assert dq(pq.PQ_SEQ2, 4, 6, fake, fake, fake, None) == E      # cols % 4
    assert dq(pq.PQ_LSQ4, 4, 7, fake, fake, fake, None) == E      # cols % 2
    assert dq(pq.PQ_SEQ2, 4, 8, None, fake, fake, None) == E
    assert dq(pq.PQ_SEQ2, 4, 8, fake, fake, None, None) == E
    assert dq(pq.PQ_SEQ2, 0, 8, None, None, None, None) == pq.PQ_OK
    sw = L.pq_scaled_weights
    assert sw(-1, 8, fake, fake, fake, None) == E
    assert sw(4, 8, None, fake, fake, None) == E
    assert sw(4, 8, fake, fake, None, None) == E
    assert sw(0, 8, None, None, None, None) == pq.PQ_OK
    # empty shapes accept NULL arrays
    assert f(pq.PQ_SEQ2, 0, 8, None, None, None, None, None) == pq.PQ_OK
    assert k(pq.PQ_SEQ2, 3, 0, None, None, None, None) == pq.PQ_OK
    # but the backward of rows > 0, cols == 0 must write d(alpha)
    assert b(pq.PQ_SEQ2, 3, 0, None, None, None, None, None, 1.0, None) == E


def test_binding_fails_loudly_without_library(tmp_path):
    from bit_quantization_aware_b200 import pq
    saved = pq._lib
    pq._lib = None
    try:
        with pytest.raises(ImportError):
            pq.lib(os.path.join(tmp_path, "missing.so"))
    finally:
        pq._lib = saved


def test_batch_argument_errors_launch_nothing(L):
    from bit_quantization_aware_b200 import pq
    E = pq.PQ_ERR_INVALID_ARG
    fake = 0x10000
    good = dict(rows=4, cols=8, w=fake, alpha=fake, wq=fake, g=fake, dw=fake,
                dalpha=fake, grad_scale=1.0)
    arr = pq.matrix_array([good])
    assert L.pq_fakequant_fwd_batch(99, 1, arr, None) == E
    assert L.pq_fakequant_fwd_batch(pq.PQ_SEQ2, -1, arr, None) == E
    assert L.pq_fakequant_fwd_batch(pq.PQ_SEQ2, 1, None, None) == E
    assert L.pq_fakequant_bwd_batch(pq.PQ_SEQ2, 1, None, None) == E
    # one bad descriptor anywhere rejects the whole call before any launch
    for bad in (dict(good, rows=-1), dict(good, w=None), dict(good, wq=None),
                dict(good, cols=6, packed=fake)):
        arr = pq.matrix_array([dict(good, rows=0)] * 3 + [bad])
        assert L.pq_fakequant_fwd_batch(pq.PQ_SEQ2, 4, arr, None) == E
    for bad in (dict(good, dalpha=None), dict(good, g=None), dict(good, cols=-2)):
        arr = pq.matrix_array([dict(good, rows=0), bad])
        assert L.pq_fakequant_bwd_batch(pq.PQ_SEQ2, 2, arr, None) == E
    # empty batches and empty matrices launch nothing
    assert L.pq_fakequant_fwd_batch(pq.PQ_SEQ2, 0, None, None) == pq.PQ_OK
    arr = pq.matrix_array([dict(rows=0, cols=8), dict(rows=3, cols=0)])
    assert L.pq_fakequant_fwd_batch(pq.PQ_SEQ2, 2, arr, None) == pq.PQ_OK
    arr = pq.matrix_array([dict(rows=0, cols=8)])
    assert L.pq_fakequant_bwd_batch(pq.PQ_SEQ2, 1, arr, None) == pq.PQ_OK


def test_adamw_argument_errors(L):
    from bit_quantization_aware_b200 import pq
    E = pq.PQ_ERR_INVALID_ARG
    fake = 0x10000
    good = dict(rows=4, cols=8, w=fake, alpha=fake, g=fake, m_w=fake, v_w=fake,
                m_alpha=fake, v_alpha=fake, grad_scale=1.0)
    h = pq.adamw(1, 1e-3)
    f = pq.lib().pq_fakequant_bwd_adamw
    import ctypes
    arr = pq.adamw_matrix_array([good])
    assert f(pq.PQ_SEQ2, 1, arr, ctypes.byref(pq.adamw(0, 1e-3)), ctypes.byref(h), None) == E
    assert f(pq.PQ_SEQ2, 1, arr, ctypes.byref(h), ctypes.byref(pq.adamw(1, 1e-3, beta1=1.0)), None) == E
    assert f(pq.PQ_SEQ2, 1, arr, None, ctypes.byref(h), None) == E
    assert f(99, 1, arr, ctypes.byref(h), ctypes.byref(h), None) == E
    for bad in (dict(good, m_w=None), dict(good, alpha=None), dict(good, rows=-1),
                dict(good, v_alpha=None)):
        arr = pq.adamw_matrix_array([dict(good, rows=0), bad])
        assert f(pq.PQ_SEQ2, 2, arr, ctypes.byref(h), ctypes.byref(h), None) == E
    arr = pq.adamw_matrix_array([dict(rows=0, cols=8)])
    assert f(pq.PQ_SEQ2, 1, arr, ctypes.byref(h), ctypes.byref(h), None) == pq.PQ_OK


def _planes_bytes(m, k):
    """The integer mode's digit planes of one activation matrix plus its
    exponents: ten base-9 planes of packed e2m1 nibbles, mp = 8 or 16 rows
    each (k <= 2^20, fp4 MMAs), or four int8 planes of m rows (8-bit MMAs)."""
    r256 = lambda b: (b + 255) // 256 * 256
    if k <= 1 << 20:
        return r256(10 * (8 if m <= 8 else 16) * k // 2) + r256(4 * m)
    return r256(4 * m * k) + r256(4 * m)


def test_matmul_workspace_sizes(L):
    """Workspace sizing of the weight-only matmul (host arithmetic only): the
    one-row path needs one counter block, the integer mode (m <= 16) its
    activations' digit planes and exponents (plus split-K partial sums), a
    group one set per matrix; sizes are multiples of 256; bad shapes give
    -1; the no-alloc scratch holds every decode-sized problem of the
    Llama-3-8B shapes."""
    from bit_quantization_aware_b200 import pq
    q = pq.PQ_SEQ2
    assert L.pq_wq_gemm_workspace_bytes(q, 1, 16384, 16384) == 256
    for m in (2, 8, 9, 16):
        for n, k in ((16384, 16384), (127, 128), (130, (1 << 20) + 128)):
            b = L.pq_wq_gemm_workspace_bytes(q, m, n, k)
            assert b >= _planes_bytes(m, k) and b % 256 == 0, (m, n, k, b)
    # one row block, one chunk: no split-K scratch, the planes alone
    for m in (2, 8, 9, 16):
        assert L.pq_wq_gemm_workspace_bytes(q, m, 127, 512) == _planes_bytes(m, 512)
    assert L.pq_wq_gemm_workspace_bytes(q, 0, 128, 128) == -1
    assert L.pq_wq_gemm_workspace_bytes(q, 4, 128, 100) == -1
    assert L.pq_wq_gemm_workspace_bytes(pq.PQ_LSQ4, 4, 128, 128) == -1
    shapes = [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]
    xs = [ctypes.c_void_p(16 * (i + 1)) for i in range(len(shapes))]  # never dereferenced
    arr = (pq.PQGemmProblem * len(shapes))()
    for i, (n, k) in enumerate(shapes):
        arr[i].n, arr[i].k, arr[i].x_bf16 = n, k, xs[i].value
    for m in (1, 8, 16):
        b = L.pq_wq_gemm_batch_workspace_bytes(q, m, len(shapes), arr)
        assert b >= sum(_planes_bytes(m, k) for _, k in shapes) and b % 256 == 0
    cap = pq.WQ_GEMM_NOALLOC_SCRATCH_BYTES
    for m in range(1, 17):
        for n, k in shapes:
            assert L.pq_wq_gemm_workspace_bytes(q, m, n, k) <= cap
