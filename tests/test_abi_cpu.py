"""The C-ABI library without a GPU: it loads, exports every symbol that
include/qgemm.h declares, and its host-only logic agrees with the oracle's
rank convention and with the header's contracts."""
import ctypes
import os
import re

import pytest
import torch

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemm.h")


def _header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qg_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def qg():
    import __graft_entry__
    __graft_entry__.build()
    import quantize_gemm_b200
    return quantize_gemm_b200


def test_header_declares_the_entry_points():
    funcs = _header_functions()
    for name in ("qg_quantize_rows", "qg_quantize_cols", "qg_clamp_compensate",
                 "qg_quantize_act", "qg_spmm_correction", "qg_fp4_gemm", "qg_fp4_linear",
                 "qg_sync_status", "qg_workspace_size", "qg_fp4_dgrad", "qg_fp4_wgrad",
                 "qg_mx_quantize_rows", "qg_mx_quantize_cols", "qg_mx_gemm", "qg_mx_scale_bytes"):
        assert name in funcs


def test_library_exports_every_declared_symbol(qg):
    lib = ctypes.CDLL(qg.LIB_PATH)
    for name in _header_functions():
        assert hasattr(lib, name), f"{name} declared in qgemm.h but not exported"
    assert set(_header_functions()) == set(qg.EXPORTED)


def test_rank_convention_matches_oracle(qg):
    for n in (1, 2, 10, 12, 131072, 4096 * 2048, 16384 * 11008):
        for alpha in (1e-12, 0.1, 0.5, 0.9, 0.95, 0.99, 0.999, 0.9999, 1.0):
            assert qg.qg_quantile_rank(alpha, n) == oracle.quantile_rank(alpha, n)
            assert qg.qg_nnz_capacity(n, alpha) == oracle.nnz_capacity(n, alpha)


def test_workspace_sizes(qg):
    for op in range(10):
        for (M, K, N, dt, a) in ((1, 32, 1, 0, 1.0), (256, 512, 512, 0, 0.99),
                                 (4096, 2048, 5504, 1, 0.99), (16384, 11008, 4096, 1, 0.999)):
            s = qg.qg_workspace_size(op, M, K, N, dt, a)
            assert s >= 256 and s % 256 == 0
    # the layer's workspace holds the activation codes, the CSR and one chunk
    # of fp32 compensation rows for bf16 Y: R rows x N with R a multiple of
    # 256 and R x N x 4 at most 128 MiB (or all of M when fewer rows; 256
    # rows when N is so wide that even those pass 128 MiB), so it does not
    # grow with M
    cap_bytes = 128 << 20

    def chunk_rows(M, N):
        r = max(256, cap_bytes // (4 * N) // 256 * 256)
        return min(r, M)

    for (M, K, N) in ((4096, 2048, 5504), (16384, 4096, 12288), (16384, 4096, 22016),
                      (16384, 11008, 4096), (65536, 4096, 4096), (300, 512, 1000),
                      (1024, 64, 200000)):
        cap = qg.qg_nnz_capacity(M * K, 0.99)
        s = qg.qg_workspace_size(qg.QG_OP_FP4_LINEAR, M, K, N, qg.QG_BF16, 0.99)
        R = chunk_rows(M, N)
        assert R == M or (R % 256 == 0 and R * N * 4 <= cap_bytes) or \
            (R == 256 and 256 * N * 4 > cap_bytes)
        assert s >= 4 * R * N + 12 * cap + M * K // 2
        # every other part is the same as without the chunk
        assert s - 4 * R * N < qg.qg_workspace_size(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, 0.99) \
            + M * K // 2 + 4 * M + 4 * (M + 1) + 12 * cap + 8192
    # at the 7B block's size the chunk is a fraction of M x N
    assert chunk_rows(16384, 12288) * 4 <= 16384
    scratch = 160 * 2 * 128 * 224 * 4
    g = qg.qg_workspace_size(qg.QG_OP_FP4_GEMM_COMPENSATED, 4096, 2048, 5504, qg.QG_F32, 1.0)
    assert scratch <= g < scratch + 4096
    # staging grows as alpha falls
    M, K = 4096, 2048
    a = qg.qg_workspace_size(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, 0.999)
    b = qg.qg_workspace_size(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, 0.99)
    assert b > a


def test_status_strings(qg):
    for s in range(8):
        assert qg.qg_status_string(s)
    assert qg.qg_status_string(99) == "unknown status"


def test_host_argument_checks_need_no_device(qg):
    """Argument errors come back before any CUDA call is made."""
    lib = qg._lib
    P = ctypes.c_void_p
    fake = P(1 << 20)   # never dereferenced: the checks reject the call first
    # K not a multiple of 32
    assert lib.qg_quantize_rows(fake, 1, 4, 48, 48, fake, fake, fake, 1 << 20, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    # K too large
    assert lib.qg_quantize_rows(fake, 1, 4, 16416, 16416, fake, fake, fake, 1 << 20, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    # bad dtype
    assert lib.qg_quantize_rows(fake, 7, 4, 64, 64, fake, fake, fake, 1 << 20, None) == \
        qg.QG_ERR_INVALID_ARG
    # misaligned A
    assert lib.qg_quantize_rows(P((1 << 20) + 4), 1, 4, 64, 64, fake, fake, fake, 1 << 20,
                                None) == qg.QG_ERR_INVALID_ARG
    # lda smaller than K
    assert lib.qg_quantize_rows(fake, 1, 4, 64, 32, fake, fake, fake, 1 << 20, None) == \
        qg.QG_ERR_INVALID_ARG
    # workspace too small
    assert lib.qg_quantize_rows(fake, 1, 4, 64, 64, fake, fake, fake, 16, None) == \
        qg.QG_ERR_WORKSPACE
    # alpha out of range
    csr = qg._Csr(1 << 20, 1 << 20, 1 << 20, 1000, 1 << 20)
    for alpha in (0.0, -0.5, 1.5, float("nan")):
        assert lib.qg_quantize_act(fake, 1, 4, 64, 64, alpha, fake, fake, ctypes.byref(csr),
                                   fake, fake, 1 << 30, None) == qg.QG_ERR_INVALID_ARG
    # CSR capacity below the bound n - ceil(alpha n)
    small = qg._Csr(1 << 20, 1 << 20, 1 << 20, 1, 1 << 20)
    assert lib.qg_quantize_act(fake, 1, 4, 64, 64, 0.5, fake, fake, ctypes.byref(small), fake,
                               fake, 1 << 30, None) == qg.QG_ERR_INVALID_ARG
    # GEMM with neither Y nor raw_acc
    assert lib.qg_fp4_gemm(fake, fake, fake, fake, 128, 128, 256, None, None, 0, None, fake,
                           1 << 20, None) == qg.QG_ERR_INVALID_ARG
    # gradient GEMMs: the contraction dimension (N for dgrad, M for wgrad)
    # must be a multiple of 32 and at most 16384; the outer ones are free
    big = 1 << 30
    assert lib.qg_fp4_dgrad(fake, 1, 64, 48, fake, 1, 64, fake, 0, fake, big, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    assert lib.qg_fp4_dgrad(fake, 1, 64, 16416, fake, 1, 64, fake, 0, fake, big, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    assert lib.qg_fp4_wgrad(fake, 1, 48, 64, fake, 1, 64, fake, 0, fake, big, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    assert lib.qg_fp4_wgrad(fake, 5, 64, 64, fake, 1, 64, fake, 0, fake, big, None) == \
        qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_dgrad(fake, 1, 64, 64, fake, 1, 64, P((1 << 20) + 8), 0, fake, big,
                            None) == qg.QG_ERR_INVALID_ARG
    need = qg.qg_workspace_size(qg.QG_OP_FP4_WGRAD, 64, 64, 64, 1, 1.0)
    assert lib.qg_fp4_wgrad(fake, 1, 64, 64, fake, 1, 64, fake, 0, fake, need - 256, None) == \
        qg.QG_ERR_WORKSPACE


def test_mx_scale_layout_host(qg):
    """The atom layout is a bijection between (row, 32-block) pairs of the
    padded matrix and the buffer's bytes; padding rows/blocks hold 127."""
    for rows, K in ((1, 32), (128, 256), (129, 288), (300, 5504), (40, 13824)):
        nbytes = qg.qg_mx_scale_bytes(rows, K)
        assert nbytes == -(-rows // 128) * -(-K // 256) * 1024
        rp = -(-rows // 128) * 128
        kp = 8 * -(-K // 256) * 32
        idx = qg.mx_scale_index(rp, kp)
        assert idx.numel() == nbytes and torch.unique(idx).numel() == nbytes
        plain = torch.randint(0, 255, (rows, K // 32), dtype=torch.uint8)
        tiled = qg.mx_scales_from_rows(plain, K)
        assert tiled.numel() == nbytes
        assert torch.equal(qg.mx_scales_to_rows(tiled, rows, K), plain)
        assert int((tiled == 127).sum()) >= nbytes - plain.numel()
    assert qg.qg_mx_scale_bytes(4, 48) == 0 and qg.qg_mx_scale_bytes(0, 64) == 0
    # host argument checks of the MX calls
    lib = qg._lib
    P = ctypes.c_void_p
    fake = P(1 << 20)
    assert lib.qg_mx_quantize_rows(fake, 1, 4, 48, 48, fake, fake, fake, 1 << 20, None) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    assert lib.qg_mx_quantize_rows(fake, 1, 4, 64, 64, fake, P((1 << 20) + 4), fake, 1 << 20,
                                   None) == qg.QG_ERR_INVALID_ARG
    assert lib.qg_mx_gemm(fake, fake, fake, fake, 128, 128, 256, None, None, 0, None, fake,
                          1 << 20, None) == qg.QG_ERR_INVALID_ARG



def test_mma_loop_host_checks(qg):
    """The tensor-pipe loop rejects out-of-range iteration counts, a missing
    flops pointer and a short workspace before anything is enqueued."""
    lib = qg._lib
    P = ctypes.c_void_p
    fake = P(1 << 20)
    flops = ctypes.c_double(-1.0)
    ws_need = qg.qg_workspace_size(qg.QG_OP_FP4_GEMM, 1, 32, 1, qg.QG_F32, 1.0)
    for iters in (0, -1, (1 << 20) + 1):
        assert lib.qg_fp4_mma_loop(iters, 1, ctypes.byref(flops), None, fake, ws_need, None) == \
            qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_mma_loop(16, 0, None, None, fake, ws_need, None) == qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_mma_loop(16, 0, ctypes.byref(flops), P((1 << 20) + 4), fake, ws_need,
                               None) == qg.QG_ERR_INVALID_ARG   # misaligned accumulator output
    assert lib.qg_fp4_mma_loop(16, 0, ctypes.byref(flops), None, fake, ws_need - 256, None) == \
        qg.QG_ERR_WORKSPACE
    assert flops.value == -1.0   # nothing written on a rejected call


C_CLIENT = r"""
#include <stdio.h>
#include "qgemm.h"
int main(void) {
    printf("%s\n", qg_status_string(QG_ERR_TIMEOUT));
    printf("%lld\n", (long long)qg_quantile_rank(0.99, 1000));
    printf("%zu\n", qg_workspace_size(QG_OP_FP4_LINEAR, 4096, 2048, 5504, QG_BF16, 0.99));
    printf("%zu\n", qg_mx_scale_bytes(300, 5504));
    /* rejected on the host before any CUDA call: K not a multiple of 32 */
    printf("%d\n", (int)qg_quantize_rows((const void*)0x100000, QG_BF16, 4, 48, 48,
                                         (uint8_t*)0x100000, (float*)0x100000,
                                         (void*)0x100000, 1 << 20, (cudaStream_t)0));
    return 0;
}
"""


def test_header_is_plain_c_and_links(qg, tmp_path):
    """include/qgemm.h compiles as C99 with warnings as errors, and a C
    program linked against libqgemm.so gets the same host-side answers as the
    Python binding (no device needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(qg.LIB_PATH)
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", inc, str(src),
                           "-o", str(exe), "-L", libdir, "-lqgemm", f"-Wl,-rpath,{libdir}"])
    out = subprocess.check_output([str(exe)], text=True).splitlines()
    assert out[0] == qg.qg_status_string(qg.QG_ERR_TIMEOUT)
    assert int(out[1]) == qg.qg_quantile_rank(0.99, 1000)
    assert int(out[2]) == qg.qg_workspace_size(qg.QG_OP_FP4_LINEAR, 4096, 2048, 5504, qg.QG_BF16, 0.99)
    assert int(out[3]) == qg.qg_mx_scale_bytes(300, 5504)
    assert int(out[4]) == qg.QG_ERR_UNSUPPORTED_SHAPE


def test_linear_parts_offsets(qg):
    """The intermediates of qg_fp4_linear sit at distinct 256-byte-aligned
    offsets inside the workspace, far enough apart for their sizes."""
    for (M, K, N, dt, alpha) in ((16384, 11008, 4096, qg.QG_BF16, 0.99),
                                 (256, 512, 512, qg.QG_F32, 0.99), (1, 32, 1, qg.QG_BF16, 1.0)):
        st, off = qg.qg_fp4_linear_parts(M, K, N, dt, alpha)
        assert st == qg.QG_OK
        total = qg.qg_workspace_size(qg.QG_OP_FP4_LINEAR, M, K, N, dt, alpha)
        cap = max(qg.qg_nnz_capacity(M * K, alpha), 1)
        sizes = [M * (K // 2), 4 * M, 4 * (M + 1), 4 * cap, 8 * cap, 8, 4]
        assert all(o % 256 == 0 for o in off)
        spans = sorted(zip(off, sizes))
        for (o1, s1), (o2, _) in zip(spans, spans[1:]):
            assert o1 + s1 <= o2
        assert spans[-1][0] + spans[-1][1] <= total
    assert qg.qg_fp4_linear_parts(64, 48, 64, qg.QG_BF16, 0.99)[0] == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert qg.qg_fp4_linear_parts(64, 64, 64, qg.QG_BF16, 0.0)[0] == qg.QG_ERR_INVALID_ARG
    assert qg._lib.qg_fp4_linear_parts(64, 64, 64, qg.QG_BF16, 0.99, None) == qg.QG_ERR_INVALID_ARG


def test_compensated_gemm_host_checks(qg):
    """The compensated GEMM rejects a missing CSR, a short weight pitch, a
    misaligned W and a short workspace before anything is enqueued."""
    lib = qg._lib
    P = ctypes.c_void_p
    fake = P(1 << 20)
    big = 1 << 30
    csr = qg._Csr(1 << 20, 1 << 20, 1 << 20, 1000, 1 << 20)
    nocol = qg._Csr(1 << 20, 0, 1 << 20, 1000, 1 << 20)
    M, N, K = 256, 512, 512
    args = lambda c, W, ldw, ws_bytes: (fake, fake, fake, fake, M, N, K, c, W, 1, ldw, fake, 0,
                                        fake, ws_bytes, None)
    need = qg.qg_workspace_size(qg.QG_OP_FP4_GEMM_COMPENSATED, M, K, N, qg.QG_F32, 1.0)
    before = qg.qg_launch_count()
    assert lib.qg_fp4_gemm_compensated(*args(None, fake, N, big)) == qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_gemm_compensated(*args(ctypes.byref(nocol), fake, N, big)) == \
        qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_gemm_compensated(*args(ctypes.byref(csr), fake, N - 1, big)) == \
        qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_gemm_compensated(*args(ctypes.byref(csr), P((1 << 20) + 2), N, big)) == \
        qg.QG_ERR_INVALID_ARG
    assert lib.qg_fp4_gemm_compensated(*args(ctypes.byref(csr), fake, N, need - 256)) == \
        qg.QG_ERR_WORKSPACE
    bad_k = (fake, fake, fake, fake, M, N, 48, ctypes.byref(csr), fake, 1, N, fake, 0, fake, big,
             None)
    assert lib.qg_fp4_gemm_compensated(*bad_k) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert qg.qg_launch_count() == before


def test_layer_order_switch(qg):
    """The layer's fp32 order depends only on the clamped entries possible per
    row against K: GEMM first from 10 per row for every 4096 of K up."""
    assert qg.linear_adds_into_y(16384, 4096, 0.99)         # 41 per row, switch at 10
    assert not qg.linear_adds_into_y(16384, 4096, 0.999)    # 4 per row
    assert qg.linear_adds_into_y(16384, 4096, 0.997)        # 12 per row
    assert not qg.linear_adds_into_y(16384, 4096, 0.998)    # 8 per row
    assert not qg.linear_adds_into_y(16384, 11008, 0.999)   # 11 per row, switch at 27
    assert qg.linear_adds_into_y(16384, 11008, 0.997)       # 33 per row
    assert qg.linear_adds_into_y(4096, 2048, 0.99)          # 20 per row, switch at 5
    assert qg.linear_adds_into_y(256, 512, 0.99)            # 5 per row, switch at 1.25
    assert not qg.linear_adds_into_y(256, 512, 0.999)       # 0.5 per row
    lib = qg._lib
    fake = ctypes.c_void_p(1 << 20)
    csr = qg._Csr(1 << 20, 1 << 20, 1 << 20, 1000, 1 << 20)
    assert lib.qg_spmm_accumulate(None, 64, fake, 1, 64, 64, 64, fake, fake, 1 << 30, None) == \
        qg.QG_ERR_INVALID_ARG
    assert lib.qg_spmm_accumulate(ctypes.byref(csr), 64, fake, 1, 64, 64, 32, fake, fake, 1 << 30,
                                  None) == qg.QG_ERR_INVALID_ARG   # ldw < N
    assert lib.qg_spmm_accumulate(ctypes.byref(csr), 64, fake, 1, 64, 64, 64, fake, fake, 16,
                                  None) == qg.QG_ERR_WORKSPACE
