"""Python binding of libqgemm.so, the B200 (sm_100a) FP4 quantized linear layer.

Argument marshalling only: every step of the layer runs in the CUDA kernels
behind the C ABI declared in ``include/qgemm.h``.  The functions named
``qg_*`` mirror the C entry points one to one and take torch tensors (device
memory and streams are torch's); the lower-case helpers below them allocate
outputs with torch and raise :class:`QGError` on a non-OK status.

There is no fallback: importing this package fails when ``lib/libqgemm.so``
is missing (build it with ``python quantize_gemm_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libqgemm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python quantize_gemm_b200/build.py, or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

QG_F32, QG_BF16 = 0, 1
QG_OK, QG_ERR_INVALID_ARG, QG_ERR_UNSUPPORTED_SHAPE, QG_ERR_WORKSPACE, QG_ERR_CUDA, \
    QG_ERR_NONFINITE, QG_ERR_TIMEOUT, QG_ERR_INTERNAL = range(8)
(QG_OP_QUANTIZE_ROWS, QG_OP_QUANTIZE_COLS, QG_OP_CLAMP_COMPENSATE, QG_OP_QUANTIZE_ACT,
 QG_OP_SPMM, QG_OP_FP4_GEMM, QG_OP_FP4_LINEAR, QG_OP_FP4_DGRAD, QG_OP_FP4_WGRAD,
 QG_OP_FP4_GEMM_COMPENSATED) = range(10)

# every symbol the header declares (checked by the CPU tests)
EXPORTED = (
    "qg_status_string", "qg_version", "qg_quantile_rank", "qg_nnz_capacity",
    "qg_workspace_size", "qg_workspace_init", "qg_sync_status", "qg_e2m1_encode",
    "qg_quantize_rows", "qg_quantize_cols", "qg_clamp_compensate", "qg_quantize_act",
    "qg_spmm_correction", "qg_fp4_gemm", "qg_fp4_linear", "qg_launch_count",
    "qg_quantize_cols_static", "qg_fp4_dgrad", "qg_fp4_wgrad", "qg_mx_scale_bytes",
    "qg_mx_quantize_rows", "qg_mx_quantize_cols", "qg_mx_gemm", "qg_fp4_mma_loop",
    "qg_fp4_linear_parts", "qg_fp4_gemm_compensated", "qg_spmm_accumulate",
    "qg_fp4_gemm_accumulate",
)


class _Csr(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col", ctypes.c_void_p),
                ("val", ctypes.c_void_p), ("nnz_capacity", ctypes.c_int64),
                ("nnz_out", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t
_D = ctypes.c_double


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("qg_status_string", ctypes.c_char_p, [_INT])
_sig("qg_version", ctypes.c_char_p, [])
_sig("qg_launch_count", ctypes.c_uint64, [])
_sig("qg_quantile_rank", _I64, [_D, _I64])
_sig("qg_nnz_capacity", _I64, [_I64, _D])
_sig("qg_workspace_size", _SZ, [_INT, _I64, _I64, _I64, _INT, _D])
_sig("qg_workspace_init", _INT, [_P, _SZ, _P])
_sig("qg_sync_status", _INT, [_P, _P])
_sig("qg_e2m1_encode", _INT, [_P, _I64, _P, _P, _SZ, _P])
_sig("qg_quantize_rows", _INT, [_P, _INT, _I64, _I64, _I64, _P, _P, _P, _SZ, _P])
_sig("qg_quantize_cols", _INT, [_P, _INT, _I64, _I64, _I64, _P, _P, _P, _SZ, _P])
_sig("qg_quantize_cols_static", _INT, [_P, _INT, _I64, _I64, _I64, _P, _P, _P])
_sig("qg_clamp_compensate", _INT,
     [_P, _INT, _I64, _I64, _I64, _D, _P, ctypes.POINTER(_Csr), _P, _P, _SZ, _P])
_sig("qg_quantize_act", _INT,
     [_P, _INT, _I64, _I64, _I64, _D, _P, _P, ctypes.POINTER(_Csr), _P, _P, _SZ, _P])
_sig("qg_spmm_correction", _INT,
     [ctypes.POINTER(_Csr), _I64, _P, _INT, _I64, _I64, _I64, _P, _P, _SZ, _P])
_sig("qg_spmm_accumulate", _INT,
     [ctypes.POINTER(_Csr), _I64, _P, _INT, _I64, _I64, _I64, _P, _P, _SZ, _P])
_sig("qg_fp4_gemm", _INT,
     [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _INT, _P, _P, _SZ, _P])
_sig("qg_fp4_gemm_accumulate", _INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P])
_sig("qg_fp4_gemm_compensated", _INT,
     [_P, _P, _P, _P, _I64, _I64, _I64, ctypes.POINTER(_Csr), _P, _INT, _I64, _P, _INT, _P, _SZ,
      _P])
_sig("qg_fp4_linear", _INT,
     [_P, _INT, _I64, _I64, _P, _P, _P, _I64, _D, _P, _INT, _P, _SZ, _P])
_sig("qg_fp4_linear_parts", _INT, [_I64, _I64, _I64, _INT, _D, ctypes.POINTER(_SZ)])
_sig("qg_mx_scale_bytes", _SZ, [_I64, _I64])
_sig("qg_mx_quantize_rows", _INT, [_P, _INT, _I64, _I64, _I64, _P, _P, _P, _SZ, _P])
_sig("qg_mx_quantize_cols", _INT, [_P, _INT, _I64, _I64, _I64, _P, _P, _P, _SZ, _P])
_sig("qg_mx_gemm", _INT, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _INT, _P, _P, _SZ, _P])
_sig("qg_fp4_mma_loop", _INT, [_I64, _INT, ctypes.POINTER(_D), _P, _P, _SZ, _P])
_sig("qg_fp4_dgrad", _INT, [_P, _INT, _I64, _I64, _P, _INT, _I64, _P, _INT, _P, _SZ, _P])
_sig("qg_fp4_wgrad", _INT, [_P, _INT, _I64, _I64, _P, _INT, _I64, _P, _INT, _P, _SZ, _P])


class QGError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        super().__init__(f"{where}: {qg_status_string(status)} (status {status})")


def qg_status_string(status: int) -> str:
    return _lib.qg_status_string(int(status)).decode()


def qg_version() -> str:
    return _lib.qg_version().decode()


def qg_launch_count() -> int:
    return int(_lib.qg_launch_count())


def qg_quantile_rank(alpha: float, n: int) -> int:
    return int(_lib.qg_quantile_rank(float(alpha), int(n)))


def qg_nnz_capacity(n: int, alpha: float) -> int:
    return int(_lib.qg_nnz_capacity(int(n), float(alpha)))


def qg_workspace_size(op: int, M: int, K: int, N: int, dtype: int, alpha: float = 1.0) -> int:
    return int(_lib.qg_workspace_size(int(op), int(M), int(K), int(N), int(dtype), float(alpha)))


# ------------------------------------------------------------------ marshalling
def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return QG_F32
    if t.dtype == torch.bfloat16:
        return QG_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (fp32 or bf16)")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str):
    if status != QG_OK:
        raise QGError(status, where)


@dataclass
class CSR:
    """dA in CSR form, device tensors (row_ptr int32 M+1, col int32, val f64)."""
    row_ptr: torch.Tensor
    col: torch.Tensor
    val: torch.Tensor
    nnz: torch.Tensor          # int64, 1 element (device)
    capacity: int

    @staticmethod
    def empty(M: int, capacity: int, device="cuda") -> "CSR":
        cap = max(int(capacity), 1)
        return CSR(torch.empty(M + 1, dtype=torch.int32, device=device),
                   torch.empty(cap, dtype=torch.int32, device=device),
                   torch.empty(cap, dtype=torch.float64, device=device),
                   torch.zeros(1, dtype=torch.int64, device=device), int(capacity))

    def c(self) -> _Csr:
        return _Csr(self.row_ptr.data_ptr(), self.col.data_ptr(), self.val.data_ptr(),
                    max(self.capacity, 1), self.nnz.data_ptr())

    def to_host(self):
        n = int(self.nnz.item())
        return (self.row_ptr.cpu().numpy(), self.col[:n].cpu().numpy(),
                self.val[:n].cpu().numpy())


class Workspace:
    """Device workspace for one call type: status word, counters, scratch."""

    def __init__(self, op: int, M: int, K: int, N: int = 1, dtype: int = QG_BF16,
                 alpha: float = 1.0, device="cuda", stream=None):
        self.nbytes = qg_workspace_size(op, M, K, N, dtype, alpha)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        _check(_lib.qg_workspace_init(_ptr(self.buf), self.nbytes, _stream(stream)),
               "qg_workspace_init")

    @property
    def ptr(self):
        return _ptr(self.buf)

    def sync_status(self, stream=None) -> int:
        return qg_sync_status(self, stream)


def qg_sync_status(ws: Workspace, stream=None) -> int:
    return int(_lib.qg_sync_status(ws.ptr, _stream(stream)))


# --------------------------------------------------------- the C entry points
def qg_e2m1_encode(x: torch.Tensor, packed: torch.Tensor, ws: Workspace, stream=None) -> int:
    return _lib.qg_e2m1_encode(_ptr(x), x.numel(), _ptr(packed), ws.ptr, ws.nbytes,
                               _stream(stream))


def qg_quantize_rows(A, codes, scales, ws: Workspace, lda=None, stream=None) -> int:
    M, K = A.shape
    return _lib.qg_quantize_rows(_ptr(A), _dt(A), M, K, A.stride(0) if lda is None else lda,
                                 _ptr(codes), _ptr(scales), ws.ptr, ws.nbytes, _stream(stream))


def qg_quantize_cols(W, codesT, scales, ws: Workspace, ldw=None, stream=None) -> int:
    K, N = W.shape
    return _lib.qg_quantize_cols(_ptr(W), _dt(W), K, N, W.stride(0) if ldw is None else ldw,
                                 _ptr(codesT), _ptr(scales), ws.ptr, ws.nbytes, _stream(stream))


def qg_quantize_cols_static(W, codesT, scales, ldw=None, stream=None) -> int:
    """qg_quantize_cols without a workspace (fixed in-library scratch, N <= 65536)."""
    K, N = W.shape
    return _lib.qg_quantize_cols_static(_ptr(W), _dt(W), K, N,
                                        W.stride(0) if ldw is None else ldw, _ptr(codesT),
                                        _ptr(scales), _stream(stream))


def qg_clamp_compensate(A, alpha, A_clamped, csr: CSR, T_out, ws: Workspace, stream=None) -> int:
    M, K = A.shape
    c = csr.c()
    return _lib.qg_clamp_compensate(_ptr(A), _dt(A), M, K, A.stride(0), float(alpha),
                                    _ptr(A_clamped), ctypes.byref(c), _ptr(T_out), ws.ptr,
                                    ws.nbytes, _stream(stream))


def qg_quantize_act(A, alpha, codes, scales, csr: CSR, T_out, ws: Workspace, stream=None) -> int:
    M, K = A.shape
    c = csr.c()
    return _lib.qg_quantize_act(_ptr(A), _dt(A), M, K, A.stride(0), float(alpha), _ptr(codes),
                                _ptr(scales), ctypes.byref(c), _ptr(T_out), ws.ptr, ws.nbytes,
                                _stream(stream))


def qg_spmm_correction(csr: CSR, M, W, C, ws: Workspace, stream=None) -> int:
    K, N = W.shape
    c = csr.c()
    return _lib.qg_spmm_correction(ctypes.byref(c), M, _ptr(W), _dt(W), K, N, W.stride(0),
                                   _ptr(C), ws.ptr, ws.nbytes, _stream(stream))


def qg_spmm_accumulate(csr: CSR, M, W, Y, ws: Workspace, stream=None) -> int:
    K, N = W.shape
    c = csr.c()
    return _lib.qg_spmm_accumulate(ctypes.byref(c), M, _ptr(W), _dt(W), K, N, W.stride(0),
                                   _ptr(Y), ws.ptr, ws.nbytes, _stream(stream))


ADD_ORDER_ENTRIES_PER_4096_K = 10   # the layer's order switch (see qg_fp4_linear)


def linear_adds_into_y(M: int, K: int, alpha: float) -> bool:
    """Whether qg_fp4_linear (fp32 Y) runs the GEMM first and adds the
    compensation into Y (True) or writes the compensation first and lets the
    GEMM add in place (False)."""
    return qg_nnz_capacity(M * K, alpha) * 4096 >= ADD_ORDER_ENTRIES_PER_4096_K * M * K


def qg_fp4_gemm(codesA, sA, codesWT, sW, M, N, K, C, Y, raw_acc, ws: Workspace,
                stream=None) -> int:
    y_dt = _dt(Y) if Y is not None else QG_F32
    return _lib.qg_fp4_gemm(_ptr(codesA), _ptr(sA), _ptr(codesWT), _ptr(sW), M, N, K, _ptr(C),
                            _ptr(Y), y_dt, _ptr(raw_acc), ws.ptr, ws.nbytes, _stream(stream))


def qg_fp4_gemm_compensated(codesA, sA, codesWT, sW, M, N, K, csr: CSR, W, Y, ws: Workspace,
                            ldw=None, stream=None) -> int:
    c = csr.c()
    return _lib.qg_fp4_gemm_compensated(_ptr(codesA), _ptr(sA), _ptr(codesWT), _ptr(sW), M, N, K,
                                        ctypes.byref(c), _ptr(W), _dt(W),
                                        W.stride(0) if ldw is None else ldw, _ptr(Y), _dt(Y),
                                        ws.ptr, ws.nbytes, _stream(stream))


def qg_fp4_gemm_accumulate(codesA, sA, codesWT, sW, M, N, K, Y, ws: Workspace,
                           stream=None) -> int:
    return _lib.qg_fp4_gemm_accumulate(_ptr(codesA), _ptr(sA), _ptr(codesWT), _ptr(sW), M, N, K,
                                       _ptr(Y), ws.ptr, ws.nbytes, _stream(stream))


def qg_fp4_linear(A, codesWT, sW, W, alpha, Y, ws: Workspace, stream=None) -> int:
    M, K = A.shape
    N = W.shape[1]
    return _lib.qg_fp4_linear(_ptr(A), _dt(A), M, K, _ptr(codesWT), _ptr(sW), _ptr(W), N,
                              float(alpha), _ptr(Y), _dt(Y), ws.ptr, ws.nbytes, _stream(stream))


def qg_fp4_linear_parts(M: int, K: int, N: int, dtype: int, alpha: float):
    """(status, the 7 byte offsets of qg_fp4_linear's intermediates in its workspace)."""
    arr = (_SZ * 7)()
    st = _lib.qg_fp4_linear_parts(int(M), int(K), int(N), int(dtype), float(alpha), arr)
    return st, [int(x) for x in arr]


def linear_parts(ws: Workspace, M: int, K: int, N: int, dtype: int, alpha: float) -> dict:
    """Views into `ws` of what qg_fp4_linear left there: activation codes and
    scales, dA (as a CSR) and T."""
    st, off = qg_fp4_linear_parts(M, K, N, dtype, alpha)
    _check(st, "qg_fp4_linear_parts")
    b = ws.buf

    def view(i, n, dt):
        item = torch.empty((), dtype=dt).element_size()
        return b[off[i]:off[i] + n * item].view(dt)

    nnz = view(5, 1, torch.int64)
    cap = max(qg_nnz_capacity(M * K, alpha), 1)
    return {"codes": view(0, M * (K // 2), torch.uint8).view(M, K // 2),
            "scales": view(1, M, torch.float32),
            "csr": CSR(view(2, M + 1, torch.int32), view(3, cap, torch.int32),
                       view(4, cap, torch.float64), nnz, cap),
            "T": view(6, 1, torch.float32)}


def _contig(*ts):
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("the backward entry points take row-major contiguous matrices")


def qg_fp4_dgrad(dY, W, dA, ws: Workspace, stream=None) -> int:
    _contig(dY, W, dA)
    M, N = dY.shape
    K = W.shape[0]
    return _lib.qg_fp4_dgrad(_ptr(dY), _dt(dY), M, N, _ptr(W), _dt(W), K, _ptr(dA), _dt(dA),
                             ws.ptr, ws.nbytes, _stream(stream))


def qg_fp4_wgrad(A, dY, dW, ws: Workspace, stream=None) -> int:
    _contig(A, dY, dW)
    M, K = A.shape
    N = dY.shape[1]
    return _lib.qg_fp4_wgrad(_ptr(A), _dt(A), M, K, _ptr(dY), _dt(dY), N, _ptr(dW), _dt(dW),
                             ws.ptr, ws.nbytes, _stream(stream))


def qg_mx_scale_bytes(rows: int, K: int) -> int:
    return int(_lib.qg_mx_scale_bytes(rows, K))


def qg_mx_quantize_rows(A, codes, scales, ws: Workspace, lda=None, stream=None) -> int:
    M, K = A.shape
    return _lib.qg_mx_quantize_rows(_ptr(A), _dt(A), M, K, A.stride(0) if lda is None else lda,
                                    _ptr(codes), _ptr(scales), ws.ptr, ws.nbytes, _stream(stream))


def qg_mx_quantize_cols(W, codesT, scalesT, ws: Workspace, ldw=None, stream=None) -> int:
    K, N = W.shape
    return _lib.qg_mx_quantize_cols(_ptr(W), _dt(W), K, N, W.stride(0) if ldw is None else ldw,
                                    _ptr(codesT), _ptr(scalesT), ws.ptr, ws.nbytes, _stream(stream))


def qg_mx_gemm(codesA, sA, codesWT, sW, M, N, K, C, Y, raw_acc, ws: Workspace, stream=None) -> int:
    y_dt = _dt(Y) if Y is not None else QG_F32
    return _lib.qg_mx_gemm(_ptr(codesA), _ptr(sA), _ptr(codesWT), _ptr(sW), M, N, K, _ptr(C),
                           _ptr(Y), y_dt, _ptr(raw_acc), ws.ptr, ws.nbytes, _stream(stream))


def qg_fp4_mma_loop(iters: int, pair: bool, ws: Workspace, stream=None, acc_out=None):
    """(status, MMA flops of the launch); acc_out (128 x 224 fp32, optional)
    receives CTA 0's accumulator."""
    flops = _D(0.0)
    st = _lib.qg_fp4_mma_loop(int(iters), 1 if pair else 0, ctypes.byref(flops), _ptr(acc_out),
                              ws.ptr, ws.nbytes, _stream(stream))
    return st, flops.value


def mx_scale_index(rows: int, K: int, device="cpu") -> torch.Tensor:
    """Byte offset, in the GEMM's scale-atom layout, of the scale of row r and
    32-block j, as a rows x K/32 int64 tensor (layout bookkeeping only)."""
    groups = 2 * ((K + 255) // 256)
    r = torch.arange(rows, device=device, dtype=torch.int64)[:, None]
    j = torch.arange(K // 32, device=device, dtype=torch.int64)[None, :]
    return (((r // 128) * groups + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4)


def mx_scales_to_rows(tiled: torch.Tensor, rows: int, K: int) -> torch.Tensor:
    """Atom layout -> plain rows x K/32 bytes."""
    return tiled.reshape(-1)[mx_scale_index(rows, K, tiled.device)]


def mx_scales_from_rows(plain: torch.Tensor, K: int) -> torch.Tensor:
    """Plain rows x K/32 bytes -> atom layout (padding bytes 127)."""
    rows = plain.shape[0]
    out = torch.full((qg_mx_scale_bytes(rows, K),), 127, dtype=torch.uint8, device=plain.device)
    out[mx_scale_index(rows, K, plain.device).reshape(-1)] = plain.reshape(-1).to(torch.uint8)
    return out


# ----------------------------------------------------------- allocating helpers
def e2m1_encode(x: torch.Tensor, ws: Optional[Workspace] = None) -> torch.Tensor:
    ws = ws or Workspace(QG_OP_QUANTIZE_ROWS, 1, 32, device=x.device)
    out = torch.empty(x.numel() // 2, dtype=torch.uint8, device=x.device)
    _check(qg_e2m1_encode(x, out, ws), "qg_e2m1_encode")
    return out


def quantize_rows(A: torch.Tensor, ws: Optional[Workspace] = None):
    M, K = A.shape
    ws = ws or Workspace(QG_OP_QUANTIZE_ROWS, M, K, 1, _dt(A), device=A.device)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=A.device)
    scales = torch.empty(M, dtype=torch.float32, device=A.device)
    _check(qg_quantize_rows(A, codes, scales, ws), "qg_quantize_rows")
    return codes, scales


def quantize_cols(W: torch.Tensor, ws: Optional[Workspace] = None):
    K, N = W.shape
    ws = ws or Workspace(QG_OP_QUANTIZE_COLS, 1, K, N, _dt(W), device=W.device)
    codesT = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(qg_quantize_cols(W, codesT, scales, ws), "qg_quantize_cols")
    return codesT, scales


def clamp_compensate(A: torch.Tensor, alpha: float, ws: Optional[Workspace] = None,
                     want_clamped: bool = True):
    M, K = A.shape
    ws = ws or Workspace(QG_OP_CLAMP_COMPENSATE, M, K, 1, _dt(A), alpha, device=A.device)
    csr = CSR.empty(M, qg_nnz_capacity(M * K, alpha), device=A.device)
    A_c = torch.empty_like(A) if want_clamped else None
    T = torch.empty(1, dtype=torch.float32, device=A.device)
    _check(qg_clamp_compensate(A, alpha, A_c, csr, T, ws), "qg_clamp_compensate")
    return A_c, csr, T


def quantize_act(A: torch.Tensor, alpha: float, ws: Optional[Workspace] = None):
    M, K = A.shape
    ws = ws or Workspace(QG_OP_QUANTIZE_ACT, M, K, 1, _dt(A), alpha, device=A.device)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=A.device)
    scales = torch.empty(M, dtype=torch.float32, device=A.device)
    csr = CSR.empty(M, qg_nnz_capacity(M * K, alpha), device=A.device)
    T = torch.empty(1, dtype=torch.float32, device=A.device)
    _check(qg_quantize_act(A, alpha, codes, scales, csr, T, ws), "qg_quantize_act")
    return codes, scales, csr, T


def spmm_correction(csr: CSR, M: int, W: torch.Tensor, ws: Optional[Workspace] = None):
    K, N = W.shape
    ws = ws or Workspace(QG_OP_SPMM, M, K, N, _dt(W), device=W.device)
    C = torch.empty((M, N), dtype=torch.float32, device=W.device)
    _check(qg_spmm_correction(csr, M, W, C, ws), "qg_spmm_correction")
    return C


def fp4_gemm(codesA, sA, codesWT, sW, K: int, C=None, out_dtype=torch.float32,
             raw: bool = False, ws: Optional[Workspace] = None):
    M, N = codesA.shape[0], codesWT.shape[0]
    ws = ws or Workspace(QG_OP_FP4_GEMM, M, K, N, QG_F32, device=codesA.device)
    Y = torch.empty((M, N), dtype=out_dtype, device=codesA.device)
    acc = torch.empty((M, N), dtype=torch.float32, device=codesA.device) if raw else None
    _check(qg_fp4_gemm(codesA, sA, codesWT, sW, M, N, K, C, Y, acc, ws), "qg_fp4_gemm")
    return (Y, acc) if raw else Y


def fp4_gemm_compensated(codesA, sA, codesWT, sW, K: int, csr: CSR, W, out_dtype=torch.float32,
                         ws: Optional[Workspace] = None):
    """Y = acc * sA_i * sW_j + dA . W in one kernel (dA as a CSR over the rows)."""
    M, N = codesA.shape[0], codesWT.shape[0]
    ws = ws or Workspace(QG_OP_FP4_GEMM_COMPENSATED, M, K, N, QG_F32, device=codesA.device)
    Y = torch.empty((M, N), dtype=out_dtype, device=codesA.device)
    _check(qg_fp4_gemm_compensated(codesA, sA, codesWT, sW, M, N, K, csr, W, Y, ws),
           "qg_fp4_gemm_compensated")
    return Y


def fp4_linear(A, codesWT, sW, W, alpha: float, out_dtype=torch.float32,
               ws: Optional[Workspace] = None):
    M, K = A.shape
    N = W.shape[1]
    ws = ws or Workspace(QG_OP_FP4_LINEAR, M, K, N, _dt(A), alpha, device=A.device)
    Y = torch.empty((M, N), dtype=out_dtype, device=A.device)
    _check(qg_fp4_linear(A, codesWT, sW, W, alpha, Y, ws), "qg_fp4_linear")
    return Y


def fp4_dgrad(dY, W, out_dtype=torch.float32, ws: Optional[Workspace] = None):
    """dA = Q(dY) Q(W)^T with dY (M x N) and W (K x N) quantized along N."""
    M, N = dY.shape
    K = W.shape[0]
    ws = ws or Workspace(QG_OP_FP4_DGRAD, M, K, N, QG_F32, device=dY.device)
    dA = torch.empty((M, K), dtype=out_dtype, device=dY.device)
    _check(qg_fp4_dgrad(dY, W, dA, ws), "qg_fp4_dgrad")
    return dA


def fp4_wgrad(A, dY, out_dtype=torch.float32, ws: Optional[Workspace] = None):
    """dW = Q(A)^T Q(dY) with A (M x K) and dY (M x N) quantized along the M tokens."""
    M, K = A.shape
    N = dY.shape[1]
    ws = ws or Workspace(QG_OP_FP4_WGRAD, M, K, N, QG_F32, device=A.device)
    dW = torch.empty((K, N), dtype=out_dtype, device=A.device)
    _check(qg_fp4_wgrad(A, dY, dW, ws), "qg_fp4_wgrad")
    return dW


def mx_quantize_rows(A: torch.Tensor, ws: Optional[Workspace] = None):
    """(codes M x K/2, scales in the atom layout) of the rows of A."""
    M, K = A.shape
    ws = ws or Workspace(QG_OP_QUANTIZE_ROWS, M, K, 1, _dt(A), device=A.device)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=A.device)
    scales = torch.empty(qg_mx_scale_bytes(M, K), dtype=torch.uint8, device=A.device)
    _check(qg_mx_quantize_rows(A, codes, scales, ws), "qg_mx_quantize_rows")
    return codes, scales


def mx_quantize_cols(W: torch.Tensor, ws: Optional[Workspace] = None):
    """(codesT N x K/2, scales in the atom layout) of the columns of W (K x N)."""
    K, N = W.shape
    ws = ws or Workspace(QG_OP_QUANTIZE_ROWS, 1, K, 1, _dt(W), device=W.device)
    codesT = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scalesT = torch.empty(qg_mx_scale_bytes(N, K), dtype=torch.uint8, device=W.device)
    _check(qg_mx_quantize_cols(W, codesT, scalesT, ws), "qg_mx_quantize_cols")
    return codesT, scalesT


def mx_gemm(codesA, sA, codesWT, sW, K: int, C=None, out_dtype=torch.float32, raw: bool = False,
            ws: Optional[Workspace] = None):
    M, N = codesA.shape[0], codesWT.shape[0]
    ws = ws or Workspace(QG_OP_FP4_GEMM, M, K, N, QG_F32, device=codesA.device)
    Y = torch.empty((M, N), dtype=out_dtype, device=codesA.device)
    acc = torch.empty((M, N), dtype=torch.float32, device=codesA.device) if raw else None
    _check(qg_mx_gemm(codesA, sA, codesWT, sW, M, N, K, C, Y, acc, ws), "qg_mx_gemm")
    return (Y, acc) if raw else Y


def fp4_mma_loop(iters: int, pair: bool = True, ws: Optional[Workspace] = None, stream=None,
                 acc_out: Optional[torch.Tensor] = None) -> float:
    """Enqueue the tensor-pipe E2M1 MMA loop; returns its flops (time it with
    CUDA events on `stream`).  acc_out (128 x 224 fp32) receives CTA 0's
    accumulator."""
    ws = ws or Workspace(QG_OP_FP4_GEMM, 1, 32, 1, QG_F32)
    st, flops = qg_fp4_mma_loop(iters, pair, ws, stream, acc_out)
    _check(st, "qg_fp4_mma_loop")
    return flops


def check_status(ws: Workspace, where: str = "device status", stream=None):
    _check(qg_sync_status(ws, stream), where)
