"""CPU oracle for the FP4 quantized linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
never calls the CUDA library: the two share no code.

The arithmetic lives in ``qg_oracle.c`` (plain C, no fast-math, no FMA
contraction); this module compiles it with gcc on first use and wraps it with
ctypes over numpy arrays.  Each wrapper names the passage of the QbitAI
write-up of "Optimizing Large Language Model Training Using FP4 Quantization"
(news.movedaos.com/post/4103) whose definition it follows:

* ``e2m1_value`` / ``e2m1_encode``: the E2M1 paragraph (1 sign, 2 exponent,
  1 mantissa bit) and the ScaleShift paragraph (round to the nearest FP4 value
  by table lookup); ties go to the even code.
* ``threshold`` / ``clamp_compensate``: the outlier clamping and compensation
  paragraph (quantile search, A_clamped, sparse dA = A - A_clamped).
* ``quantize_rows`` / ``quantize_cols``: the granularity paragraph (token-wise
  for A, channel-wise for W) with the ScaleShift calibration.
* ``gemm_acc`` / ``linear_y`` / ``spmm``: Y = acc * s_i * t_j + dA * W, the
  layer output in double.
* ``mx_exponent`` / ``mx_quantize_rows`` / ``mx_quantize_cols`` / ``mx_gemm``:
  the MXFP4 block-scaled variant (the micro-scaling section of the lecture
  page "FP4量化训练的硬件挑战：NVIDIA Blackwell架构上的微缩放格式（Micro-scaling）实现",
  zyxy.net/?p=24232, and the micro-scaling paragraph of the low-precision
  training survey at 10100.com/article/123065115): blocks of 32 along K, each
  with the E8M0 scale 2^e, e the smallest exponent with 6 * 2^e >= block max.
* ``dgrad`` / ``wgrad``: the gradient GEMMs with FP4 operands (the write-up's
  paragraphs on the FP4 GEMM and on the differentiable gradient estimator say
  the training runs its matrix products in FP4; how gradients are quantized
  is not stated).  Reading: each operand is quantized with the forward's
  rule along the contraction dimension, one scale per outer index, no clamp.

Pins: every function here is checked in ``tests/test_oracle_pins.py``
against values fixed by the pages or the mathematics (worked examples,
brute force, library routines, closed forms and invariants); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qg_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall"]


def build(force: bool = False) -> str:
    """Compile qg_oracle.c into liboracle.so beside it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.orc_e2m1_value.restype = ctypes.c_double
    lib.orc_e2m1_value.argtypes = [ctypes.c_uint8]
    lib.orc_e2m1_encode.restype = ctypes.c_uint8
    lib.orc_e2m1_encode.argtypes = [ctypes.c_float]
    lib.orc_e2m1_encode_array.argtypes = [P, I64, P]
    lib.orc_e2m1_encode_bits_packed.argtypes = [ctypes.c_uint32, I64, P]
    lib.orc_quantile_rank.restype = I64
    lib.orc_quantile_rank.argtypes = [ctypes.c_double, I64]
    lib.orc_threshold.restype = ctypes.c_float
    lib.orc_threshold.argtypes = [P, I64, ctypes.c_double]
    lib.orc_clamp_compensate.restype = I64
    lib.orc_clamp_compensate.argtypes = [P, I64, I64, ctypes.c_float, P, P, P, P, I64]
    lib.orc_scale_factors.argtypes = [ctypes.c_float, P, P]
    lib.orc_quantize_rows.argtypes = [P, I64, I64, P, P]
    lib.orc_quantize_cols.argtypes = [P, I64, I64, P, P]
    lib.orc_quantize_act.restype = I64
    lib.orc_quantize_act.argtypes = [P, I64, I64, ctypes.c_double, P, P, P, P, P, I64, P]
    lib.orc_gemm_acc_rows.argtypes = [P, P, I64, I64, I64, P, I64, P]
    lib.orc_linear_y_rows.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_spmm.argtypes = [P, P, P, P, I64, I64, P]
    lib.orc_mx_exponent.restype = ctypes.c_int
    lib.orc_mx_exponent.argtypes = [ctypes.c_float]
    lib.orc_mx_quantize_rows.argtypes = [P, I64, I64, P, P]
    lib.orc_mx_quantize_cols.argtypes = [P, I64, I64, P, P]
    lib.orc_mx_gemm_rows.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def as_f32(x) -> np.ndarray:
    """Widen an input tensor to a contiguous float32 numpy array.

    Accepts numpy float32 arrays and torch float32/bfloat16 CPU tensors; the
    bf16 -> fp32 widening is exact, so the oracle sees the same values.
    """
    if isinstance(x, np.ndarray):
        assert x.dtype == np.float32
        return np.ascontiguousarray(x)
    import torch  # CPU-only use: dtype widening of an input tensor
    t = x.detach().to("cpu")
    if t.dtype != torch.float32:
        t = t.to(torch.float32)
    return np.ascontiguousarray(t.numpy())


def num_threads() -> int:
    return int(_load().orc_num_threads())


# -- E2M1 ---------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return float(_load().orc_e2m1_value(int(code)))


def e2m1_values() -> np.ndarray:
    """Value of each of the 16 codes (index = code)."""
    return np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e2m1_encode(x) -> np.ndarray:
    """One unpacked code per element of a float32 array."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32).reshape(-1))
    out = np.empty(x.size, dtype=np.uint8)
    _load().orc_e2m1_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e2m1_encode_bits_packed(start: int, n: int) -> np.ndarray:
    """Packed codes of the fp32 bit patterns start .. start+n-1 (NaN -> 0)."""
    assert n % 2 == 0
    out = np.empty(n // 2, dtype=np.uint8)
    _load().orc_e2m1_encode_bits_packed(ctypes.c_uint32(start & 0xFFFFFFFF), n, _ptr(out))
    return out


# -- threshold and clamp ----------------------------------------------------------
def quantile_rank(alpha: float, n: int) -> int:
    return int(_load().orc_quantile_rank(float(alpha), int(n)))


def threshold(A, alpha: float) -> float:
    a = as_f32(A).reshape(-1)
    return float(np.float32(_load().orc_threshold(_ptr(a), a.size, float(alpha))))


def nnz_capacity(n: int, alpha: float) -> int:
    """Upper bound on the clamped entries: n - ceil(alpha * n)."""
    return int(n - (quantile_rank(alpha, n) + 1))


def clamp_compensate(A, T: float):
    """Return (A_clamped float32, row_ptr int32, col int32, val float64)."""
    a = as_f32(A)
    M, K = a.shape
    a_c = np.empty_like(a)
    cap = M * K
    row_ptr = np.empty(M + 1, dtype=np.int32)
    col = np.empty(cap, dtype=np.int32)
    val = np.empty(cap, dtype=np.float64)
    nnz = _load().orc_clamp_compensate(_ptr(a), M, K, ctypes.c_float(T), _ptr(a_c),
                                       _ptr(row_ptr), _ptr(col), _ptr(val), cap)
    assert nnz >= 0
    return a_c, row_ptr, col[:nnz].copy(), val[:nnz].copy()


# -- quantizers -------------------------------------------------------------------
def scale_factors(amax: float):
    r = ctypes.c_float()
    s = ctypes.c_float()
    _load().orc_scale_factors(ctypes.c_float(amax), ctypes.byref(r), ctypes.byref(s))
    return np.float32(r.value), np.float32(s.value)


def quantize_rows(A):
    """Token-wise quantization: (codes uint8 M x K/2, scales float32 M)."""
    a = as_f32(A)
    M, K = a.shape
    assert K % 2 == 0
    codes = np.empty((M, K // 2), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    _load().orc_quantize_rows(_ptr(a), M, K, _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_cols(W):
    """Channel-wise quantization of W (K x N): (codesT uint8 N x K/2, scales N)."""
    w = as_f32(W)
    K, N = w.shape
    assert K % 2 == 0
    codesT = np.empty((N, K // 2), dtype=np.uint8)
    scales = np.empty(N, dtype=np.float32)
    _load().orc_quantize_cols(_ptr(w), K, N, _ptr(codesT), _ptr(scales))
    return codesT, scales


def quantize_act(A, alpha: float):
    """Threshold + clamp + dA + row quantization.

    Returns dict(codes, scales, row_ptr, col, val, T).
    """
    a = as_f32(A)
    M, K = a.shape
    cap = max(nnz_capacity(M * K, alpha), 1)
    codes = np.empty((M, K // 2), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    row_ptr = np.empty(M + 1, dtype=np.int32)
    col = np.empty(cap, dtype=np.int32)
    val = np.empty(cap, dtype=np.float64)
    T = ctypes.c_float()
    nnz = _load().orc_quantize_act(_ptr(a), M, K, float(alpha), _ptr(codes), _ptr(scales),
                                   _ptr(row_ptr), _ptr(col), _ptr(val), cap, ctypes.byref(T))
    assert nnz >= 0
    return dict(codes=codes, scales=scales, row_ptr=row_ptr, col=col[:nnz].copy(),
                val=val[:nnz].copy(), T=float(np.float32(T.value)))


# -- GEMM and layer output ------------------------------------------------------------
def _rows_arg(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size


def gemm_acc(codesA, codesWT, K: int, rows=None) -> np.ndarray:
    """acc (len(rows) or M) x N in double from packed codes."""
    cA = np.ascontiguousarray(codesA, dtype=np.uint8)
    cW = np.ascontiguousarray(codesWT, dtype=np.uint8)
    M, N = cA.shape[0], cW.shape[0]
    r, nr = _rows_arg(rows)
    R = nr if r is not None else M
    acc = np.empty((R, N), dtype=np.float64)
    _load().orc_gemm_acc_rows(_ptr(cA), _ptr(cW), M, N, K,
                              _ptr(r) if r is not None else None, nr, _ptr(acc))
    return acc


def linear_y(acc, sA, sW, row_ptr, col, val, W, rows=None) -> np.ndarray:
    """Y = acc * s_i * t_j + dA * W (double) for the listed rows (None: all)."""
    w = as_f32(W)
    K, N = w.shape
    sA = np.ascontiguousarray(sA, dtype=np.float32)
    sW = np.ascontiguousarray(sW, dtype=np.float32)
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    cl = np.ascontiguousarray(col, dtype=np.int32)
    vl = np.ascontiguousarray(val, dtype=np.float64)
    if cl.size == 0:
        cl = np.zeros(1, np.int32)
        vl = np.zeros(1, np.float64)
    M = rp.size - 1
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    r, nr = _rows_arg(rows)
    R = nr if r is not None else M
    Y = np.empty((R, N), dtype=np.float64)
    _load().orc_linear_y_rows(_ptr(acc), _ptr(sA), _ptr(sW), _ptr(rp), _ptr(cl), _ptr(vl),
                              _ptr(w), M, N, K, _ptr(r) if r is not None else None, nr, _ptr(Y))
    return Y


def spmm(row_ptr, col, val, W) -> np.ndarray:
    """dA * W in double (M x N)."""
    w = as_f32(W)
    K, N = w.shape
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    cl = np.ascontiguousarray(col, dtype=np.int32)
    vl = np.ascontiguousarray(val, dtype=np.float64)
    if cl.size == 0:
        cl = np.zeros(1, np.int32)
        vl = np.zeros(1, np.float64)
    M = rp.size - 1
    C = np.empty((M, N), dtype=np.float64)
    _load().orc_spmm(_ptr(rp), _ptr(cl), _ptr(vl), _ptr(w), M, N, _ptr(C))
    return C


def dequant_rows(codes, scales) -> np.ndarray:
    """Dequantized M x K matrix (double): grid value of each code times s_i."""
    vals = e2m1_values()
    c = np.asarray(codes, dtype=np.uint8)
    lo = vals[c & 15]
    hi = vals[c >> 4]
    M = c.shape[0]
    q = np.empty((M, 2 * c.shape[1]), dtype=np.float64)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    return q * np.asarray(scales, dtype=np.float64)[:, None]


# -- gradient GEMMs -------------------------------------------------------------------
def scaled_product(acc, s_rows, s_cols) -> np.ndarray:
    """acc[i, j] * s_rows[i] * s_cols[j] in double."""
    return (np.asarray(acc, dtype=np.float64)
            * np.asarray(s_rows, dtype=np.float32).astype(np.float64)[:, None]
            * np.asarray(s_cols, dtype=np.float32).astype(np.float64)[None, :])


def dgrad(dY, W, rows=None) -> np.ndarray:
    """dA = Q(dY) Q(W)^T (double) for the listed rows of dA (None: all).

    dY is M x N and W the forward weight, K x N; both are quantized per row,
    i.e. along N, the contraction dimension; dA is M x K.
    """
    cd, sd = quantize_rows(dY)
    cw, sw = quantize_rows(W)
    N = 2 * cd.shape[1]
    acc = gemm_acc(cd, cw, N, rows)
    return scaled_product(acc, sd if rows is None else sd[np.asarray(rows)], sw)


def wgrad(A, dY, rows=None) -> np.ndarray:
    """dW = Q(A)^T Q(dY) (double) for the listed rows of dW (None: all).

    A is M x K and dY is M x N; both are quantized per column, i.e. along the
    M tokens, the contraction dimension; dW is K x N.
    """
    ca, sa = quantize_cols(A)
    cd, sd = quantize_cols(dY)
    M = 2 * ca.shape[1]
    acc = gemm_acc(ca, cd, M, rows)
    return scaled_product(acc, sa if rows is None else sa[np.asarray(rows)], sd)


# -- MXFP4 block-scaled variant -------------------------------------------------------
def mx_exponent(amax: float) -> int:
    """Smallest e in [-127, 127] with 6 * 2^e >= amax (-127 for amax == 0)."""
    return int(_load().orc_mx_exponent(ctypes.c_float(amax)))


def mx_quantize_rows(A):
    """Rows of A (M x K) in blocks of 32: (codes uint8 M x K/2, E8M0 uint8 M x K/32)."""
    a = as_f32(A)
    M, K = a.shape
    assert K % 32 == 0
    codes = np.empty((M, K // 2), dtype=np.uint8)
    scales = np.empty((M, K // 32), dtype=np.uint8)
    _load().orc_mx_quantize_rows(_ptr(a), M, K, _ptr(codes), _ptr(scales))
    return codes, scales


def mx_quantize_cols(W):
    """Columns of W (K x N) in blocks of 32 along K, transposed:
    (codesT uint8 N x K/2, E8M0 uint8 N x K/32)."""
    w = as_f32(W)
    K, N = w.shape
    assert K % 32 == 0
    codesT = np.empty((N, K // 2), dtype=np.uint8)
    scalesT = np.empty((N, K // 32), dtype=np.uint8)
    _load().orc_mx_quantize_cols(_ptr(w), K, N, _ptr(codesT), _ptr(scalesT))
    return codesT, scalesT


def mx_gemm(codesA, sA, codesWT, sW, K: int, rows=None) -> np.ndarray:
    """Y = sum over blocks of 2^(eA + eW) * (block dot product of the codes),
    in double, for the listed rows (None: all)."""
    cA = np.ascontiguousarray(codesA, dtype=np.uint8)
    cW = np.ascontiguousarray(codesWT, dtype=np.uint8)
    sa = np.ascontiguousarray(sA, dtype=np.uint8)
    sw = np.ascontiguousarray(sW, dtype=np.uint8)
    M, N = cA.shape[0], cW.shape[0]
    r, nr = _rows_arg(rows)
    R = nr if r is not None else M
    Y = np.empty((R, N), dtype=np.float64)
    _load().orc_mx_gemm_rows(_ptr(cA), _ptr(sa), _ptr(cW), _ptr(sw), M, N, K,
                             _ptr(r) if r is not None else None, nr, _ptr(Y))
    return Y


def mx_dequant_rows(codes, scales) -> np.ndarray:
    """Dequantized M x K matrix (double): grid value of each code times its
    block's 2^e."""
    q = dequant_rows(codes, np.ones(np.asarray(codes).shape[0], dtype=np.float32))
    e = np.asarray(scales, dtype=np.int64) - 127
    return q * np.ldexp(1.0, np.repeat(e, 32, axis=1))
