"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Bars (from the layer's definition; see the header of include/qgemm.h):
* codes, scales, threshold T, the CSR of dA and the raw FP4 accumulator are
  bit-exact (integer / exactly representable results);
* the correction C = dA . W (fp32 FMA chain) is within (n + 2) * 2^-24 of the
  absolute sum |dA| . |W| per element, n = non-zeros in the row;
* Y (fp32) satisfies max |Y - Yo| / max(|Yo|, 1e-3 * rms(Yo)) <= 1e-3 against
  the oracle's fp64 evaluation of the same quantized operands;
* Y (bf16) is within one bf16 ulp of Yo.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle_pins import unpack
from workloads import WORKLOADS, make_layer_inputs, make_matrix

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qg():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import quantize_gemm_b200
    torch.cuda.set_device(0)
    return quantize_gemm_b200


def _np(t):
    return t.detach().cpu().numpy()


def y_rel_err(Y, Yo):
    Y = np.asarray(Y, dtype=np.float64)
    floor = 1e-3 * np.sqrt(np.mean(Yo ** 2)) if Yo.size else 0.0
    floor = max(floor, 1e-30)
    return float(np.max(np.abs(Y - Yo) / np.maximum(np.abs(Yo), floor))) if Yo.size else 0.0


def bf16_ulp(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


# ------------------------------------------------------------------ encoder
def test_e2m1_exhaustive_all_fp32_patterns(qg):
    """Every one of the 2^32 fp32 bit patterns (NaN patterns -> 0 on both
    sides, since NaN is rejected before encoding)."""
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ROWS, 1, 32, device="cuda")
    CH = 1 << 28
    for c in range(1 << 4):
        start = c * CH
        b = torch.arange(start, start + CH, dtype=torch.int64, device="cuda")
        b = torch.where(b >= (1 << 31), b - (1 << 32), b).to(torch.int32)
        x = b.view(torch.float32)
        x = torch.where(torch.isnan(x), torch.zeros_like(x), x)
        got = _np(qg.e2m1_encode(x, ws))
        del b, x
        want = oracle.e2m1_encode_bits_packed(start, CH)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (hex(start + 2 * int(bad[0])), got[bad[0]], want[bad[0]])
    qg.check_status(ws)


# ------------------------------------------------------------------ quantizers
def _special_rows(K, dtype):
    A = torch.zeros((6, K), dtype=torch.float32)
    A[1] = -0.0
    A[2, :] = 1e-45
    A[2, 3] = -3e-45
    A[3, :] = torch.linspace(-7, 7, K)
    A[4, :] = 1e30
    A[4, 1::2] = -2.5e30
    # exact ties after scaling by r = 1 (amax = 6)
    ties = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    A[5, :] = ties.repeat(K // 8) * torch.where(torch.arange(K) % 3 == 0, -1.0, 1.0)
    return A.to(dtype)


ROW_CASES = [
    (1, 32, torch.float32), (3, 64, torch.bfloat16), (257, 512, torch.float32),
    (100, 1056, torch.bfloat16), (64, 16384, torch.bfloat16), (32, 16384, torch.float32),
    (129, 2048, torch.bfloat16), (7, 4128, torch.float32),
    (50, 3072, torch.bfloat16), (77, 4096, torch.bfloat16), (5, 4064, torch.bfloat16),
    # bf16 rows split over 2 or 4 warps (4096 < K <= 16384), ragged last segments
    (33, 4128, torch.bfloat16), (19, 5504, torch.bfloat16), (70, 8192, torch.bfloat16),
    (17, 11008, torch.bfloat16), (9, 16384, torch.bfloat16), (1, 15360, torch.bfloat16),
    (300, 12320, torch.bfloat16),
]


@pytest.mark.parametrize("M,K,dtype", ROW_CASES)
def test_quantize_rows(qg, M, K, dtype):
    A = make_matrix((M, K), ("student_t", 3), seed=M * 7 + K, device="cuda", dtype=dtype,
                    scale=2.0)
    codes, scales = qg.quantize_rows(A)
    oc, os_ = oracle.quantize_rows(A.cpu())
    assert np.array_equal(_np(scales), os_)
    assert np.array_equal(_np(codes), oc)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_rows_special_values(qg, dtype):
    A = _special_rows(256, dtype).cuda()
    codes, scales = qg.quantize_rows(A)
    oc, os_ = oracle.quantize_rows(A.cpu())
    assert np.array_equal(_np(scales), os_)
    assert np.array_equal(_np(codes), oc)


@pytest.mark.parametrize("K,ld", [(512, 1024), (6144, 6152)])
def test_quantize_rows_strided(qg, K, ld):
    base = make_matrix((40, ld), seed=3, device="cuda", dtype=torch.bfloat16)
    A = base[:, :K]              # lda > K
    codes, scales = qg.quantize_rows(A)
    oc, os_ = oracle.quantize_rows(A.contiguous().cpu())
    assert np.array_equal(_np(codes), oc) and np.array_equal(_np(scales), os_)


COL_CASES = [
    (32, 1, torch.float32), (64, 7, torch.bfloat16), (512, 512, torch.float32),
    (2048, 5504, torch.bfloat16), (5504, 2048, torch.bfloat16), (16384, 40, torch.bfloat16),
    (96, 300, torch.float32),
]


@pytest.mark.parametrize("K,N,dtype", COL_CASES)
def test_quantize_cols(qg, K, N, dtype):
    W = make_matrix((K, N), seed=K + N, device="cuda", dtype=dtype, scale=0.02)
    codesT, t = qg.quantize_cols(W)
    oT, ot = oracle.quantize_cols(W.cpu())
    assert np.array_equal(_np(t), ot)
    assert np.array_equal(_np(codesT), oT)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_cols_special_values(qg, dtype):
    W = _special_rows(256, dtype).t().contiguous().cuda()   # columns = special rows
    codesT, t = qg.quantize_cols(W)
    oT, ot = oracle.quantize_cols(W.cpu())
    assert np.array_equal(_np(t), ot) and np.array_equal(_np(codesT), oT)


@pytest.mark.parametrize("width", [600, 604])
def test_quantize_cols_strided_bf16(qg, width):
    """A column block of a wider bf16 matrix: row pitch 600 (16-byte rows) and
    604 (rows not 16-byte multiples, element loads)."""
    Wide = make_matrix((288, width), seed=width, device="cuda", dtype=torch.bfloat16, scale=0.02)
    W = Wide[:, :300]
    codesT, t = qg.quantize_cols(W)
    oT, ot = oracle.quantize_cols(W.cpu().contiguous())
    assert np.array_equal(_np(t), ot) and np.array_equal(_np(codesT), oT)


# ------------------------------------------------------------------ threshold + clamp
def _act_inputs(name):
    if name == "tiny":
        return make_layer_inputs("tiny", 0, device="cuda")[0], 0.99
    if name == "llama1.3b_attn_m512":
        return make_layer_inputs("llama1.3b", 0, device="cuda", M=512)[0], 0.99
    if name == "llama7b_down_m256":
        return make_layer_inputs("llama7b", 4, device="cuda", M=256)[0], 0.99
    if name == "llama13b_qkv_m128":
        return make_layer_inputs("llama13b", 1, device="cuda", M=128)[0], 0.999
    if name == "ragged_k1056_fp32":
        return make_matrix((33, 1056), ("student_t", 3), seed=5, device="cuda"), 0.95
    if name == "no_clamp":
        return make_matrix((64, 512), seed=6, device="cuda", dtype=torch.bfloat16), 1.0
    if name == "clamp_almost_all":
        return make_matrix((16, 256), seed=7, device="cuda", dtype=torch.bfloat16), 1e-6
    if name == "ties_at_T":
        A = torch.ones((8, 64), device="cuda", dtype=torch.bfloat16)
        A[::2, ::3] = -2.0
        return A, 0.9
    if name == "single_row":
        return make_matrix((1, 8192), ("student_t", 4), seed=8, device="cuda",
                           dtype=torch.bfloat16), 0.99
    if name == "fp32_heavy_tail":
        return make_matrix((200, 640), ("student_t", 3), seed=9, device="cuda",
                           outliers=("random_entries", 0.002, 1e3)), 0.997
    if name == "bf16_ragged_k1056":
        return make_matrix((300, 1056), ("student_t", 4), seed=11, device="cuda",
                           dtype=torch.bfloat16), 0.99
    if name == "many_outliers_k2048":
        # alpha 0.3: about 70 % of the entries are clamped, so a 1024-column
        # step holds more outliers than a warp's list (512) and the clamp
        # pass stages them from its per-lane loop instead
        return make_matrix((64, 2048), ("student_t", 4), seed=13, device="cuda",
                           dtype=torch.bfloat16), 0.3
    if name in ("band_miss_low", "band_miss_high"):
        # M=512, K=256: the bf16 threshold pass samples rows 0, 8, 16, ...
        # only.  Here those rows are all zeros (every other row zero), or
        # 1000x larger than the rest (1/8 of the rows: the true quantile lies
        # well below the sampled one), so the band misses the order statistic
        # and the exact fallback has to produce the threshold.
        A = make_matrix((512, 256), ("student_t", 4), seed=12, device="cuda")
        if name == "band_miss_low":
            A[0::2] = 0.0
        else:
            A[0::8] *= 1000.0
        return A.to(torch.bfloat16), 0.99
    raise KeyError(name)


ACT_CASES = ["tiny", "llama1.3b_attn_m512", "llama7b_down_m256", "llama13b_qkv_m128",
             "ragged_k1056_fp32", "no_clamp", "clamp_almost_all", "ties_at_T", "single_row",
             "fp32_heavy_tail", "bf16_ragged_k1056", "band_miss_low", "band_miss_high",
             "many_outliers_k2048"]


def _check_act(qg, A, alpha, codes, scales, csr, T, exp):
    assert float(_np(T)[0]) == exp["T"]
    rp, col, val = csr.to_host()
    assert np.array_equal(rp, exp["row_ptr"])
    assert np.array_equal(col, exp["col"])
    assert np.array_equal(val, exp["val"])
    if codes is not None:
        assert np.array_equal(_np(scales), exp["scales"])
        assert np.array_equal(_np(codes), exp["codes"])


def test_quantize_act_workspace_shared_with_other_paths(qg):
    """One workspace used in turn by the cooperative bf16 kernel, the
    multi-kernel clamp_compensate sequence and the fp32 path: each call must
    start from its own state (the cooperative kernel's clean-counter
    shortcut must not trust counters another path left behind)."""
    A, alpha = _act_inputs("llama1.3b_attn_m512")
    Af = make_matrix(tuple(A.shape), ("student_t", 4), seed=99, device="cuda")
    M, K = A.shape
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_F32, alpha)
    exp = oracle.quantize_act(A.cpu(), alpha)
    exp_f = oracle.quantize_act(Af.cpu(), alpha)
    for step in range(3):
        out = qg.quantize_act(A, alpha, ws=ws)
        qg.check_status(ws, "fused")
        _check_act(qg, A, alpha, *out, exp)
        _, csr, T = qg.clamp_compensate(A, alpha, ws=ws, want_clamped=False)
        qg.check_status(ws, "clamp_compensate")
        _check_act(qg, A, alpha, None, None, csr, T, exp)
        out = qg.quantize_act(A, alpha, ws=ws)
        qg.check_status(ws, "fused after multi-kernel")
        _check_act(qg, A, alpha, *out, exp)
        out = qg.quantize_act(Af, alpha, ws=ws)
        qg.check_status(ws, "fp32")
        _check_act(qg, Af, alpha, *out, exp_f)


@pytest.mark.parametrize("case", ACT_CASES)
def test_quantize_act(qg, case):
    A, alpha = _act_inputs(case)
    M, K = A.shape
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg._dt(A), alpha)
    codes, scales, csr, T = qg.quantize_act(A, alpha, ws=ws)
    qg.check_status(ws, case)
    exp = oracle.quantize_act(A.cpu(), alpha)
    _check_act(qg, A, alpha, codes, scales, csr, T, exp)
    # same workspace again: identical bytes (canonical CSR, no stale state)
    codes2, scales2, csr2, T2 = qg.quantize_act(A, alpha, ws=ws)
    qg.check_status(ws, case)
    _check_act(qg, A, alpha, codes2, scales2, csr2, T2, exp)


@pytest.mark.parametrize("case", ["tiny", "llama7b_down_m256", "ragged_k1056_fp32", "ties_at_T"])
def test_clamp_compensate(qg, case):
    A, alpha = _act_inputs(case)
    M, K = A.shape
    ws = qg.Workspace(qg.QG_OP_CLAMP_COMPENSATE, M, K, 1, qg._dt(A), alpha)
    A_c, csr, T = qg.clamp_compensate(A, alpha, ws=ws)
    qg.check_status(ws, case)
    Th = oracle.threshold(A.cpu(), alpha)
    oa_c, orp, ocol, oval = oracle.clamp_compensate(A.cpu(), Th)
    assert float(_np(T)[0]) == Th
    assert np.array_equal(oracle.as_f32(A_c.cpu()), oa_c)
    rp, col, val = csr.to_host()
    assert np.array_equal(rp, orp) and np.array_equal(col, ocol) and np.array_equal(val, oval)
    # the CSR without the clamped copy
    _, csr2, _ = qg.clamp_compensate(A, alpha, ws=ws, want_clamped=False)
    qg.check_status(ws, case)
    rp2, col2, val2 = csr2.to_host()
    assert np.array_equal(rp2, orp) and np.array_equal(col2, ocol) and np.array_equal(val2, oval)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_nonfinite_input_reported(qg, bad, dtype):
    A = make_matrix((16, 256), seed=10, device="cuda", dtype=dtype)
    A[5, 17] = bad
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, 16, 256, 1, qg._dt(A), 0.99)
    qg.quantize_act(A, 0.99, ws=ws)
    assert ws.sync_status() == qg.QG_ERR_NONFINITE
    # the status is cleared by the read; a clean call on the same workspace is OK
    A[5, 17] = 1.0
    qg.quantize_act(A, 0.99, ws=ws)
    assert ws.sync_status() == qg.QG_OK


# ------------------------------------------------------------------ SpMM correction
@pytest.mark.parametrize("case,N,wdtype", [("tiny", 512, torch.float32),
                                            ("llama1.3b_attn_m512", 2048, torch.bfloat16),
                                            ("ragged_k1056_fp32", 100, torch.float32),
                                            ("clamp_almost_all", 264, torch.bfloat16)])
def test_spmm_correction(qg, case, N, wdtype):
    A, alpha = _act_inputs(case)
    M, K = A.shape
    W = make_matrix((K, N), seed=11, device="cuda", dtype=wdtype, scale=0.02)
    _, csr, _ = qg.clamp_compensate(A, alpha, want_clamped=False)
    C = _np(qg.spmm_correction(csr, M, W)).astype(np.float64)
    rp, col, val = csr.to_host()
    Co = oracle.spmm(rp, col, val, W.cpu())
    S = oracle.spmm(rp, col, np.abs(val), W.cpu().abs())
    n = np.diff(rp).astype(np.float64)[:, None]
    bound = (n + 2) * 2.0 ** -24 * S
    assert np.all(np.abs(C - Co) <= bound), float(np.max(np.abs(C - Co) - bound))


@pytest.mark.parametrize("case,N,wdtype", [("llama1.3b_attn_m512", 2048, torch.bfloat16),
                                            ("tiny", 512, torch.float32),
                                            ("bf16_ragged_k1056", 257, torch.bfloat16),
                                            ("no_clamp", 600, torch.bfloat16),
                                            ("clamp_almost_all", 264, torch.bfloat16)])
def test_spmm_accumulate(qg, case, N, wdtype):
    """Y += dA . W by the memory system's adds equals Y + (the stored
    compensation), element by element in fp32; rows without entries are left
    as they were."""
    A, alpha = _act_inputs(case)
    M, K = A.shape
    W = make_matrix((K, N), seed=13, device="cuda", dtype=wdtype, scale=0.02)
    _, csr, _ = qg.clamp_compensate(A, alpha, want_clamped=False)
    Y0 = make_matrix((M, N), seed=14, device="cuda")
    C = qg.spmm_correction(csr, M, W)
    Y = Y0.clone()
    ws = qg.Workspace(qg.QG_OP_SPMM, M, K, N, qg._dt(W))
    assert qg.qg_spmm_accumulate(csr, M, W, Y, ws) == qg.QG_OK
    qg.check_status(ws)
    assert torch.equal(Y, Y0 + C)
    rp = _np(csr.row_ptr)
    empty = np.nonzero(np.diff(rp) == 0)[0]
    if empty.size:
        idx = torch.from_numpy(empty).cuda()
        assert torch.equal(Y[idx], Y0[idx])


# ------------------------------------------------------------------ FP4 GEMM
GEMM_SHAPES = [(128, 256, 256), (1, 8, 32), (129, 257, 288), (300, 600, 1024),
               (1024, 1024, 4096), (256, 512, 16384), (4096, 2048, 2048), (513, 5504, 2048)]


def _rand_codes(rows, K, seed):
    g = np.random.default_rng(seed)
    return g.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_fp4_gemm_raw_accumulator_bit_exact(qg, M, N, K):
    cA = _rand_codes(M, K, M + K)
    cW = _rand_codes(N, K, N + 3 * K)
    sA = np.ones(M, np.float32)
    sW = np.ones(N, np.float32)
    Y, acc = qg.fp4_gemm(torch.from_numpy(cA).cuda(), torch.from_numpy(sA).cuda(),
                         torch.from_numpy(cW).cuda(), torch.from_numpy(sW).cuda(), K, raw=True)
    acc = _np(acc)
    rows = np.arange(M) if M * N * K <= (1 << 31) else \
        np.unique(np.concatenate([np.random.default_rng(1).integers(0, M, 48), [0, M - 1]]))
    want = oracle.gemm_acc(cA, cW, K, rows=rows)
    assert np.array_equal(acc[rows], want.astype(np.float32))
    assert np.array_equal(acc[rows].astype(np.float64), want)   # exact in fp32


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (129, 257, 288), (300, 600, 1024),
                                   (513, 5504, 2048)])
@pytest.mark.parametrize("with_c", [False, True])
def test_fp4_gemm_epilogue_fp32(qg, M, N, K, with_c):
    g = np.random.default_rng(M + N)
    cA, cW = _rand_codes(M, K, 5 + M), _rand_codes(N, K, 6 + N)
    sA = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    sW = (g.random(N) * 0.01 + 1e-4).astype(np.float32)
    C = (g.standard_normal((M, N)) * 0.5).astype(np.float32) if with_c else None
    Y = qg.fp4_gemm(torch.from_numpy(cA).cuda(), torch.from_numpy(sA).cuda(),
                    torch.from_numpy(cW).cuda(), torch.from_numpy(sW).cuda(), K,
                    C=torch.from_numpy(C).cuda() if with_c else None)
    acc = oracle.gemm_acc(cA, cW, K)
    Yo = acc * sA.astype(np.float64)[:, None] * sW.astype(np.float64)[None, :]
    if with_c:
        Yo = Yo + C.astype(np.float64)
    assert y_rel_err(_np(Y), Yo) <= 1e-3


@pytest.mark.parametrize("M,N,K", [(300, 600, 1024), (129, 257, 288), (256, 5504, 512)])
def test_fp4_gemm_direct_epilogue(qg, M, N, K):
    """Raw accumulator requested: the register-to-global epilogue writes Y too
    (16-byte stores for whole 32-column chunks when N % 8 == 0, scalar stores
    otherwise); Y with C must match like the TMA epilogue's."""
    g = np.random.default_rng(M + 7 * N)
    cA, cW = _rand_codes(M, K, 31 + M), _rand_codes(N, K, 32 + N)
    sA = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    sW = (g.random(N) * 0.01 + 1e-4).astype(np.float32)
    C = (g.standard_normal((M, N)) * 0.5).astype(np.float32)
    Y, acc = qg.fp4_gemm(torch.from_numpy(cA).cuda(), torch.from_numpy(sA).cuda(),
                         torch.from_numpy(cW).cuda(), torch.from_numpy(sW).cuda(), K,
                         C=torch.from_numpy(C).cuda(), raw=True)
    want = oracle.gemm_acc(cA, cW, K)
    assert np.array_equal(_np(acc).astype(np.float64), want)
    Yo = want * sA.astype(np.float64)[:, None] * sW.astype(np.float64)[None, :] + C.astype(np.float64)
    assert y_rel_err(_np(Y), Yo) <= 1e-3


@pytest.mark.parametrize("M,N,K", [(300, 600, 1024), (129, 257, 288), (513, 5504, 2048)])
def test_fp4_gemm_accumulates_in_place(qg, M, N, K):
    """C given as Y itself (fp32): Y += the scaled product, bit for bit what a
    separate C gives (TMA epilogue for N % 4 == 0, direct stores otherwise)."""
    g = np.random.default_rng(M + 3 * N)
    cA, cW = _rand_codes(M, K, 41 + M), _rand_codes(N, K, 42 + N)
    sA = torch.from_numpy((g.random(M) * 0.1 + 1e-3).astype(np.float32)).cuda()
    sW = torch.from_numpy((g.random(N) * 0.01 + 1e-4).astype(np.float32)).cuda()
    C = torch.from_numpy((g.standard_normal((M, N)) * 0.5).astype(np.float32)).cuda()
    cA, cW = torch.from_numpy(cA).cuda(), torch.from_numpy(cW).cuda()
    want = qg.fp4_gemm(cA, sA, cW, sW, K, C=C)
    Y = C.clone()
    ws = qg.Workspace(qg.QG_OP_FP4_GEMM, M, K, N, qg.QG_F32)
    assert qg.qg_fp4_gemm(cA, sA, cW, sW, M, N, K, Y, Y, None, ws) == qg.QG_OK
    qg.check_status(ws)
    assert torch.equal(Y, want)


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (300, 1000, 1024), (1024, 4096, 2048),
                                   (2048, 12288, 4096)])
def test_fp4_gemm_accumulate(qg, M, N, K):
    """qg_fp4_gemm_accumulate: Y += the scaled product by the memory system's
    bulk reduction, bit for bit the fp32 sum of Y and qg_fp4_gemm's own output
    (single-CTA and pair tiles, ragged tiles); N not a multiple of 4 is
    rejected before anything is enqueued."""
    g = np.random.default_rng(M + 5 * N)
    cA, cW = _rand_codes(M, K, 61 + M), _rand_codes(N, K, 62 + N)
    sA = torch.from_numpy((g.random(M) * 0.1 + 1e-3).astype(np.float32)).cuda()
    sW = torch.from_numpy((g.random(N) * 0.01 + 1e-4).astype(np.float32)).cuda()
    Y0 = torch.from_numpy((g.standard_normal((M, N)) * 0.5).astype(np.float32)).cuda()
    cA, cW = torch.from_numpy(cA).cuda(), torch.from_numpy(cW).cuda()
    G = qg.fp4_gemm(cA, sA, cW, sW, K)
    Y = Y0.clone()
    ws = qg.Workspace(qg.QG_OP_FP4_GEMM, M, K, N, qg.QG_F32)
    assert qg.qg_fp4_gemm_accumulate(cA, sA, cW, sW, M, N, K, Y, ws) == qg.QG_OK
    qg.check_status(ws)
    assert torch.equal(Y, Y0 + G)
    bad = torch.zeros((M, N - 2), dtype=torch.float32, device="cuda")
    assert qg.qg_fp4_gemm_accumulate(cA, sA, cW, sW, M, N - 2, K, bad, ws) == \
        qg.QG_ERR_UNSUPPORTED_SHAPE


def test_fp4_gemm_epilogue_bf16(qg):
    M, N, K = 300, 600, 1024
    g = np.random.default_rng(2)
    cA, cW = _rand_codes(M, K, 21), _rand_codes(N, K, 22)
    sA = (g.random(M) * 0.1 + 1e-3).astype(np.float32)
    sW = (g.random(N) * 0.01 + 1e-4).astype(np.float32)
    C = (g.standard_normal((M, N)) * 0.5).astype(np.float32)
    Y = qg.fp4_gemm(torch.from_numpy(cA).cuda(), torch.from_numpy(sA).cuda(),
                    torch.from_numpy(cW).cuda(), torch.from_numpy(sW).cuda(), K,
                    C=torch.from_numpy(C).cuda(), out_dtype=torch.bfloat16)
    acc = oracle.gemm_acc(cA, cW, K)
    Yo = acc * sA.astype(np.float64)[:, None] * sW.astype(np.float64)[None, :] + C
    err = np.abs(_np(Y.float()).astype(np.float64) - Yo)
    assert np.all(err <= bf16_ulp(Yo))


# ------------------------------------------------------------ compensated GEMM
COMP_CASES = [  # (activation case, N, W dtype, Y dtype)
    ("tiny", 512, torch.float32, torch.float32),
    ("llama1.3b_attn_m512", 2048, torch.bfloat16, torch.float32),
    ("llama1.3b_attn_m512", 2048, torch.bfloat16, torch.bfloat16),
    ("llama7b_down_m256", 4096, torch.bfloat16, torch.float32),
    ("ragged_k1056_fp32", 100, torch.float32, torch.float32),     # ragged last column group
    ("bf16_ragged_k1056", 257, torch.bfloat16, torch.float32),    # Y pitch not 16 B: direct stores
    ("bf16_ragged_k1056", 264, torch.bfloat16, torch.bfloat16),
    ("clamp_almost_all", 264, torch.bfloat16, torch.float32),     # every row full of entries
    ("no_clamp", 600, torch.bfloat16, torch.float32),             # no entries at all
    ("ties_at_T", 64, torch.bfloat16, torch.float32),             # 8 rows: one CTA, not a pair
    ("single_row", 1056, torch.bfloat16, torch.bfloat16),
]


@pytest.mark.parametrize("case,N,wdtype,ydtype", COMP_CASES)
def test_fp4_gemm_compensated(qg, case, N, wdtype, ydtype):
    """The GEMM with the compensation computed inside it equals, bit for bit,
    the two-kernel path (SpMM into C, then the GEMM adding C), and Y is within
    the layer's tolerance of the oracle."""
    A, alpha = _act_inputs(case)
    M, K = A.shape
    W = make_matrix((K, N), seed=K + 3 * N, device="cuda", dtype=wdtype, scale=0.02)
    codes, scales, csr, T = qg.quantize_act(A, alpha)
    codesT, t = qg.quantize_cols(W)
    ws = qg.Workspace(qg.QG_OP_FP4_GEMM_COMPENSATED, M, K, N, qg.QG_F32)
    Y = qg.fp4_gemm_compensated(codes, scales, codesT, t, K, csr, W, out_dtype=ydtype, ws=ws)
    qg.check_status(ws, case)
    C = qg.spmm_correction(csr, M, W)
    Y2 = qg.fp4_gemm(codes, scales, codesT, t, K, C=C, out_dtype=ydtype)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    # the same workspace again: the scratch slots keep the last call's rows
    Y3 = qg.fp4_gemm_compensated(codes, scales, codesT, t, K, csr, W, out_dtype=ydtype, ws=ws)
    qg.check_status(ws, case)
    assert torch.equal(Y3, Y)
    rp, col, val = csr.to_host()
    oT, ot = oracle.quantize_cols(W.cpu())
    acc = oracle.gemm_acc(_np(codes), oT, K)
    Yo = oracle.linear_y(acc, _np(scales), ot, rp, col, val, W.cpu())
    if ydtype == torch.float32:
        assert y_rel_err(_np(Y), Yo) <= 1e-3
    else:
        rms = np.sqrt(np.mean(Yo ** 2))
        assert np.all(np.abs(_np(Y.float()).astype(np.float64) - Yo) <= bf16_ulp(Yo) + 1e-6 * rms)


@pytest.mark.parametrize("M,K,N,alpha", [(700, 256, 65536, 0.99), (1000, 512, 40000, 0.999),
                                         (300, 1056, 8192, 0.99)])
def test_fp4_linear_bf16_chunks(qg, M, K, N, alpha):
    """The layer with bf16 Y goes through its rows in chunks (the SpMM writes a
    chunk's compensation into an fp32 scratch, the GEMM reads it while writing
    the chunk's Y).  With N this wide the chunks are 512, 768 or all rows, the
    last one ragged: Y equals, bit for bit, the compensated GEMM's single
    kernel on the same codes and CSR, and the oracle within a bf16 ulp on
    sampled rows."""
    A = make_matrix((M, K), ("student_t", 3), seed=M + K, device="cuda", dtype=torch.bfloat16)
    W = make_matrix((K, N), seed=N, device="cuda", dtype=torch.bfloat16, scale=0.02)
    codesT, t = qg.quantize_cols(W)
    ws = qg.Workspace(qg.QG_OP_FP4_LINEAR, M, K, N, qg.QG_BF16, alpha)
    Y = qg.fp4_linear(A, codesT, t, W, alpha, out_dtype=torch.bfloat16, ws=ws)
    qg.check_status(ws, "layer")
    # the layer's own codes and CSR, from its workspace
    st, off = qg.qg_fp4_linear_parts(M, K, N, qg.QG_BF16, alpha)
    assert st == qg.QG_OK
    buf = ws.buf
    codes = buf[off[0]:off[0] + M * (K // 2)].view(M, K // 2)
    scales = buf[off[1]:off[1] + 4 * M].view(torch.float32)
    cap = max(qg.qg_nnz_capacity(M * K, alpha), 1)
    csr = qg.CSR(buf[off[2]:off[2] + 4 * (M + 1)].view(torch.int32),
                 buf[off[3]:off[3] + 4 * cap].view(torch.int32),
                 buf[off[4]:off[4] + 8 * cap].view(torch.float64),
                 buf[off[5]:off[5] + 8].view(torch.int64), cap)
    wsc = qg.Workspace(qg.QG_OP_FP4_GEMM_COMPENSATED, M, K, N, qg.QG_F32)
    Y2 = qg.fp4_gemm_compensated(codes, scales, codesT, t, K, csr, W, out_dtype=torch.bfloat16,
                                 ws=wsc)
    qg.check_status(wsc, "compensated")
    assert torch.equal(Y, Y2)
    rows = np.arange(0, M, 97)
    Yo, _ = _linear_oracle(A, W, alpha, rows=rows)
    rms = np.sqrt(np.mean(Yo ** 2))
    got = _np(Y.float())[rows].astype(np.float64)
    assert np.all(np.abs(got - Yo) <= bf16_ulp(Yo) + 1e-6 * rms)


# ------------------------------------------------------------------ the layer
@pytest.mark.parametrize("M,K,N,dtype,alpha,gemm_first", [
    (300, 1024, 1002, torch.bfloat16, 0.99, True),     # N % 4 = 2: direct epilogue, 1-wide adds
    (300, 1024, 1002, torch.bfloat16, 0.999, False),   # N % 4 = 2: GEMM in place through C = Y
    (260, 512, 1000, torch.float32, 0.999, False),     # reducing GEMM, fp32 W (slice SpMM)
    (130, 2048, 516, torch.bfloat16, 0.995, True),     # N % 8 = 4: slice SpMM adding
    (520, 4096, 2048, torch.bfloat16, 0.998, False),   # 8 per row, switch at 10
    (520, 4096, 2048, torch.bfloat16, 0.997, True),    # 12 per row
])
def test_fp4_linear_fp32_orders(qg, M, K, N, dtype, alpha, gemm_first):
    """fp32 Y in the order the layer picks for the clamped entries per row
    against K, with widths that force each epilogue and SpMM form: Y equals
    bit for bit the separate calls on the layer's own codes and CSR (SpMM into
    a fresh C, then the GEMM reading C), and the oracle within 1e-3 on every
    fifth row."""
    assert qg.linear_adds_into_y(M, K, alpha) == gemm_first
    A = make_matrix((M, K), ("student_t", 3), seed=M + 7 * K, device="cuda", dtype=dtype)
    W = make_matrix((K, N), seed=N + 1, device="cuda", dtype=dtype, scale=0.02)
    codesT, t = qg.quantize_cols(W)
    dt = qg._dt(A)
    ws = qg.Workspace(qg.QG_OP_FP4_LINEAR, M, K, N, dt, alpha)
    Y = qg.fp4_linear(A, codesT, t, W, alpha, ws=ws)
    qg.check_status(ws, "layer")
    parts = qg.linear_parts(ws, M, K, N, dt, alpha)
    C = qg.spmm_correction(parts["csr"], M, W)
    Y2 = qg.fp4_gemm(parts["codes"], parts["scales"], codesT, t, K, C=C)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    rows = np.arange(0, M, 5)
    Yo, _ = _linear_oracle(A, W, alpha, rows=rows)
    assert y_rel_err(_np(Y)[rows], Yo) <= 1e-3


def _linear_oracle(A, W, alpha, rows=None):
    act = oracle.quantize_act(A.cpu(), alpha)
    oT, ot = oracle.quantize_cols(W.cpu())
    acc = oracle.gemm_acc(act["codes"], oT, A.shape[1], rows=rows)
    return oracle.linear_y(acc, act["scales"], ot, act["row_ptr"], act["col"], act["val"],
                           W.cpu(), rows=rows), act


LAYER_CASES = [("tiny", 0, None), ("llama1.3b", 0, 256), ("llama1.3b", 1, 256),
               ("llama1.3b", 2, 256), ("llama7b", 4, 128), ("llama13b", 1, 128)]


@pytest.mark.parametrize("wl,layer,M", LAYER_CASES)
def test_fp4_linear_small(qg, wl, layer, M):
    A, W = make_layer_inputs(wl, layer, device="cuda", M=M)
    alpha = WORKLOADS[wl].alphas[0]
    codesT, t = qg.quantize_cols(W)
    ws = qg.Workspace(qg.QG_OP_FP4_LINEAR, A.shape[0], A.shape[1], W.shape[1], qg._dt(A), alpha)
    Y = qg.fp4_linear(A, codesT, t, W, alpha, ws=ws)
    qg.check_status(ws)
    Yo, _ = _linear_oracle(A, W, alpha)
    assert y_rel_err(_np(Y), Yo) <= 1e-3
    Yb = qg.fp4_linear(A, codesT, t, W, alpha, out_dtype=torch.bfloat16, ws=ws)
    qg.check_status(ws)
    rms = np.sqrt(np.mean(Yo ** 2))
    assert np.all(np.abs(_np(Yb.float()).astype(np.float64) - Yo) <= bf16_ulp(Yo) + 1e-6 * rms)


@pytest.mark.parametrize("wl,layer", [("llama1.3b", 1), ("llama7b", 1), ("llama13b", 4)])
def test_fp4_linear_full_size_sampled(qg, wl, layer):
    """Full workload sizes, the launch configuration the benchmark times:
    T, codes, scales and dA, as the layer call left them in its workspace,
    checked exactly over the whole tensor, Y on a sample of rows computed by
    the oracle one by one."""
    A, W = make_layer_inputs(wl, layer, device="cuda")
    alpha = WORKLOADS[wl].alphas[0]
    M, K = A.shape
    N = W.shape[1]
    codesT, t = qg.quantize_cols(W)
    ws = qg.Workspace(qg.QG_OP_FP4_LINEAR, M, K, N, qg._dt(A), alpha)
    Y = qg.fp4_linear(A, codesT, t, W, alpha, ws=ws)
    qg.check_status(ws)
    parts = qg.linear_parts(ws, M, K, N, qg._dt(A), alpha)   # what the layer call used
    codes, scales, csr, T = parts["codes"], parts["scales"], parts["csr"], parts["T"]
    rows = np.unique(np.concatenate([np.random.default_rng(M + N).integers(0, M, 24), [0, M - 1]]))
    Yo, act = _linear_oracle(A, W, alpha, rows=rows)
    assert float(_np(T)[0]) == act["T"]
    assert np.array_equal(_np(codes), act["codes"]) and np.array_equal(_np(scales), act["scales"])
    rp, col, val = csr.to_host()
    assert np.array_equal(rp, act["row_ptr"]) and np.array_equal(col, act["col"])
    assert np.array_equal(val, act["val"])
    oT, ot = oracle.quantize_cols(W.cpu())
    assert np.array_equal(_np(codesT), oT) and np.array_equal(_np(t), ot)
    assert y_rel_err(_np(Y)[rows], Yo) <= 1e-3


# ------------------------------------------------------------ gradient GEMMs
GRAD_CASES = [  # (M, K, N, dtype): ragged outer sizes, warp-row and CTA-row quantizers
    (256, 512, 512, torch.float32), (300, 600, 1056, torch.bfloat16),
    (77, 1000, 4096, torch.bfloat16), (64, 200, 5504, torch.bfloat16),
    (1024, 96, 160, torch.bfloat16), (32, 33, 32, torch.float32),
]


def _grad_inputs(M, K, N, dtype, seed):
    A = make_matrix((M, K), ("student_t", 4), seed=seed, dtype=dtype)
    W = make_matrix((K, N), seed=seed + 1, dtype=dtype, scale=0.02)
    dY = make_matrix((M, N), seed=seed + 2, dtype=dtype, scale=1e-3)
    return A, W, dY


@pytest.mark.parametrize("M,K,N,dtype", GRAD_CASES)
def test_fp4_dgrad(qg, M, K, N, dtype):
    A, W, dY = _grad_inputs(M, K, N, dtype, seed=M + K)
    # forward Y = A W (M x N); backward dA = dY W^T with W (K x N): contraction over N
    ws = qg.Workspace(qg.QG_OP_FP4_DGRAD, M, K, N, qg.QG_F32)
    dA = qg.fp4_dgrad(dY.cuda(), W.cuda(), ws=ws)
    qg.check_status(ws)
    assert dA.shape == (M, K)
    Do = oracle.dgrad(dY, W)
    assert y_rel_err(_np(dA), Do) <= 1e-3
    dAb = qg.fp4_dgrad(dY.cuda(), W.cuda(), out_dtype=torch.bfloat16)
    rms = np.sqrt(np.mean(Do ** 2))
    assert np.all(np.abs(_np(dAb.float()).astype(np.float64) - Do) <= bf16_ulp(Do) + 1e-6 * rms)


@pytest.mark.parametrize("M,K,N,dtype", GRAD_CASES)
def test_fp4_wgrad(qg, M, K, N, dtype):
    if M % 32:
        pytest.skip("wgrad contracts over M")
    A, W, dY = _grad_inputs(M, K, N, dtype, seed=M + N)
    dW = qg.fp4_wgrad(A.cuda(), dY.cuda())
    assert dW.shape == (K, N)
    Wo = oracle.wgrad(A, dY)
    assert y_rel_err(_np(dW), Wo) <= 1e-3
    dWb = qg.fp4_wgrad(A.cuda(), dY.cuda(), out_dtype=torch.bfloat16)
    rms = np.sqrt(np.mean(Wo ** 2))
    assert np.all(np.abs(_np(dWb.float()).astype(np.float64) - Wo) <= bf16_ulp(Wo) + 1e-6 * rms)


def test_fp4_grads_exact_on_grid(qg):
    """Operands already on their scaled grids along the contraction dimension:
    both gradients equal the exact products (fp32 output, power-of-two
    scales, integer-valued accumulators)."""
    from oracle_pins import _on_grid_matrix
    g = np.random.default_rng(31)
    M, K, N = 96, 72, 160
    dY, *_ = _on_grid_matrix(g, M, N, g.integers(-4, 4, size=M).astype(np.float64))
    W, *_ = _on_grid_matrix(g, K, N, g.integers(-8, -2, size=K).astype(np.float64))
    dA = qg.fp4_dgrad(torch.from_numpy(dY).cuda(), torch.from_numpy(W).cuda())
    assert np.array_equal(_np(dA).astype(np.float64), dY.astype(np.float64) @ W.astype(np.float64).T)
    AT, *_ = _on_grid_matrix(g, K, M, g.integers(-3, 3, size=K).astype(np.float64))
    dYT, *_ = _on_grid_matrix(g, N, M, g.integers(-9, -5, size=N).astype(np.float64))
    A, dY2 = np.ascontiguousarray(AT.T), np.ascontiguousarray(dYT.T)
    dW = qg.fp4_wgrad(torch.from_numpy(A).cuda(), torch.from_numpy(dY2).cuda())
    assert np.array_equal(_np(dW).astype(np.float64), A.astype(np.float64).T @ dY2.astype(np.float64))


@pytest.mark.parametrize("wl,layer", [("llama1.3b", 1), ("llama7b", 4)])
def test_fp4_grads_full_size_sampled(qg, wl, layer):
    """A layer of the benchmark workloads at full size: dgrad and wgrad on a
    sample of output rows computed by the oracle one by one."""
    A, W = make_layer_inputs(wl, layer, device="cuda")
    M, K = A.shape
    N = W.shape[1]
    dY = make_matrix((M, N), seed=77, device="cuda", dtype=A.dtype, scale=1e-3)
    dA = qg.fp4_dgrad(dY, W)
    dW = qg.fp4_wgrad(A, dY)
    g = np.random.default_rng(M + K + N)
    rows = np.unique(np.concatenate([g.integers(0, M, 12), [0, M - 1]]))
    assert y_rel_err(_np(dA)[rows], oracle.dgrad(dY.cpu(), W.cpu(), rows=rows)) <= 1e-3
    rows = np.unique(np.concatenate([g.integers(0, K, 12), [0, K - 1]]))
    assert y_rel_err(_np(dW)[rows], oracle.wgrad(A.cpu(), dY.cpu(), rows=rows)) <= 1e-3


# ------------------------------------------------------------ MXFP4 variant
def _mx_plain(qg, tiled, rows, K):
    return _np(qg.mx_scales_to_rows(tiled, rows, K))


MX_ROW_CASES = [(1, 32, torch.float32), (5, 64, torch.bfloat16), (128, 256, torch.bfloat16),
                (129, 288, torch.float32), (300, 5504, torch.bfloat16), (77, 16384, torch.bfloat16),
                (256, 4096, torch.float32)]


@pytest.mark.parametrize("M,K,dtype", MX_ROW_CASES)
def test_mx_quantize_rows(qg, M, K, dtype):
    A = make_matrix((M, K), ("student_t", 3), seed=M + 3 * K, device="cuda", dtype=dtype,
                    scale=float(10.0 ** ((M % 7) - 3)))
    codes, tiled = qg.mx_quantize_rows(A)
    oc, os_ = oracle.mx_quantize_rows(A.cpu())
    assert np.array_equal(_np(codes), oc)
    assert np.array_equal(_mx_plain(qg, tiled, M, K), os_)
    # padding rows / blocks of the atoms hold 2^0
    idx = qg.mx_scale_index(M, K).reshape(-1).numpy()
    pad = np.ones(tiled.numel(), dtype=bool)
    pad[idx] = False
    assert np.all(_np(tiled)[pad] == 127)


def test_mx_quantize_rows_special_values(qg):
    K = 256
    A = np.zeros((6, K), dtype=np.float32)
    A[1, :] = -0.0
    A[2, :32] = 1e-42                       # subnormal block
    A[3, :] = np.float32(3.0e38) * np.sign(np.random.default_rng(1).standard_normal(K))
    A[4, ::3] = 6.0 * 2.0 ** -20            # block max exactly on 6 * 2^e
    A[5, :] = np.linspace(-7.0, 7.0, K, dtype=np.float32)
    for dt in (torch.float32, torch.bfloat16):
        At = torch.from_numpy(A).to(dt)
        codes, tiled = qg.mx_quantize_rows(At.cuda())
        oc, os_ = oracle.mx_quantize_rows(At)
        assert np.array_equal(_np(codes), oc)
        assert np.array_equal(_mx_plain(qg, tiled, 6, K), os_)


MX_COL_CASES = [(32, 1, torch.float32), (64, 200, torch.bfloat16), (288, 130, torch.bfloat16),
                (2048, 5504, torch.bfloat16), (512, 512, torch.float32)]


@pytest.mark.parametrize("K,N,dtype", MX_COL_CASES)
def test_mx_quantize_cols(qg, K, N, dtype):
    W = make_matrix((K, N), seed=K + N, device="cuda", dtype=dtype, scale=0.02)
    codesT, tiled = qg.mx_quantize_cols(W)
    oT, osT = oracle.mx_quantize_cols(W.cpu())
    assert np.array_equal(_np(codesT), oT)
    assert np.array_equal(_mx_plain(qg, tiled, N, K), osT)


MX_GEMM_CASES = [(128, 128, 256), (1, 8, 32), (300, 200, 288), (129, 640, 1024), (512, 384, 5504),
                 (256, 1000, 4096)]


@pytest.mark.parametrize("M,N,K", MX_GEMM_CASES)
def test_mx_gemm(qg, M, N, K):
    """Oracle codes and scales through the block-scaled MMA: fp32 Y within the
    layer tolerance of the oracle's double evaluation, bf16 within one ulp."""
    A = make_matrix((M, K), ("student_t", 4), seed=M + K, dtype=torch.float32)
    W = make_matrix((K, N), seed=N + K + 1, dtype=torch.float32, scale=0.02)
    qa, sa = oracle.mx_quantize_rows(A)
    qw, sw = oracle.mx_quantize_cols(W)
    Yo = oracle.mx_gemm(qa, sa, qw, sw, K)
    ta = qg.mx_scales_from_rows(torch.from_numpy(sa), K).cuda()
    tw = qg.mx_scales_from_rows(torch.from_numpy(sw), K).cuda()
    ca, cw = torch.from_numpy(qa).cuda(), torch.from_numpy(qw).cuda()
    Y = qg.mx_gemm(ca, ta, cw, tw, K)
    assert y_rel_err(_np(Y), Yo) <= 1e-3
    Yb = qg.mx_gemm(ca, ta, cw, tw, K, out_dtype=torch.bfloat16)
    rms = np.sqrt(np.mean(Yo ** 2))
    assert np.all(np.abs(_np(Yb.float()).astype(np.float64) - Yo) <= bf16_ulp(Yo) + 1e-6 * rms)
    C = torch.randn((M, N), device="cuda") * float(rms)
    Yc = qg.mx_gemm(ca, ta, cw, tw, K, C=C)
    assert y_rel_err(_np(Yc), Yo + _np(C).astype(np.float64)) <= 1e-3


def test_mx_gemm_exact_on_grid(qg):
    """Blocks on their scaled grids with exponents within +-2: every partial
    sum is exact in fp32, so the raw accumulator equals A @ W exactly."""
    from oracle_pins import _mx_on_grid_rows
    g = np.random.default_rng(41)
    M, N, K = 200, 136, 768
    A, *_ = _mx_on_grid_rows(g, M, K, espan=2)
    WT, *_ = _mx_on_grid_rows(g, N, K, espan=2)
    codes, ta = qg.mx_quantize_rows(torch.from_numpy(A).cuda())
    codesW, tw = qg.mx_quantize_rows(torch.from_numpy(WT).cuda())
    Y, acc = qg.mx_gemm(codes, ta, codesW, tw, K, raw=True)
    exact = A.astype(np.float64) @ WT.astype(np.float64).T
    assert np.array_equal(_np(acc).astype(np.float64), exact)
    assert np.array_equal(_np(Y).astype(np.float64), exact)


@pytest.mark.parametrize("wl,layer", [("llama1.3b", 1), ("llama7b", 1)])
def test_mx_pipeline_full_size_sampled(qg, wl, layer):
    """A layer of the benchmark workloads at full size through the MX path
    (GPU quantizers, GPU GEMM): codes and scales exact over the whole
    tensors, Y on sampled rows against the oracle."""
    A, W = make_layer_inputs(wl, layer, device="cuda")
    M, K = A.shape
    N = W.shape[1]
    codes, ta = qg.mx_quantize_rows(A)
    codesT, tw = qg.mx_quantize_cols(W)
    Y = qg.mx_gemm(codes, ta, codesT, tw, K)
    oc, os_ = oracle.mx_quantize_rows(A.cpu())
    oT, osT = oracle.mx_quantize_cols(W.cpu())
    assert np.array_equal(_np(codes), oc) and np.array_equal(_mx_plain(qg, ta, M, K), os_)
    assert np.array_equal(_np(codesT), oT) and np.array_equal(_mx_plain(qg, tw, N, K), osT)
    rows = np.unique(np.concatenate([np.random.default_rng(M + N).integers(0, M, 16), [0, M - 1]]))
    Yo = oracle.mx_gemm(oc, os_, oT, osT, K, rows=rows)
    assert y_rel_err(_np(Y)[rows], Yo) <= 1e-3


def test_mx_quantizers_flag_nonfinite(qg):
    """A NaN or Inf in a block sets the workspace status (reported as
    QG_ERR_NONFINITE) in both MX quantizers; finite inputs leave it clean."""
    A = make_matrix((64, 256), seed=5, device="cuda", dtype=torch.bfloat16)
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ROWS, 64, 256, 1, qg.QG_BF16)
    qg.mx_quantize_rows(A, ws=ws)
    assert qg.qg_sync_status(ws) == qg.QG_OK
    for bad in (float("nan"), float("inf")):
        B = A.clone()
        B[7, 100] = bad
        qg.mx_quantize_rows(B, ws=ws)
        assert qg.qg_sync_status(ws) == qg.QG_ERR_NONFINITE
        qg.mx_quantize_cols(B, ws=ws)
        assert qg.qg_sync_status(ws) == qg.QG_ERR_NONFINITE
    qg.mx_quantize_cols(A, ws=ws)
    assert qg.qg_sync_status(ws) == qg.QG_OK
