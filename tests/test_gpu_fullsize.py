"""Parity at the largest sizes: the 7B decoder block's four linears at
M = 16384 tokens (Student-t(3) activations, no planted outliers) for both of its
clamp quantiles, and the activation quantizer on the 256M-element end of the
quantizer sweep.

Each layer runs through qg_fp4_linear in the launch configuration the benchmark
times; T, the activation codes and scales and the CSR of dA are read back from
the workspace that call used (qg_fp4_linear_parts) and compared with the oracle
bit for bit over the whole tensor; Y is compared on rows sampled across M with
the oracle's fp64 evaluation (max |Y - Yo| / max(|Yo|, 1e-3 rms(Yo)) <= 1e-3).
The weight codes and scales are checked over the whole tensor as well.
"""
import numpy as np
import pytest
import torch

import oracle
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
    floor = max(1e-3 * np.sqrt(np.mean(Yo ** 2)), 1e-30)
    return float(np.max(np.abs(Y - Yo) / np.maximum(np.abs(Yo), floor)))


BLOCK = WORKLOADS["block16k"]
CASES = [(li, a) for a in BLOCK.alphas for li in range(len(BLOCK.layers))]


@pytest.mark.parametrize("layer,alpha", CASES,
                         ids=[f"{BLOCK.layers[li].name}-a{a}" for li, a in CASES])
def test_block16k_layer_full_size(qg, layer, alpha):
    A, W = make_layer_inputs(BLOCK, layer, device="cuda")
    M, K = A.shape
    N = W.shape[1]
    dt = qg._dt(A)
    codesT, t = qg.quantize_cols(W)
    ws = qg.Workspace(qg.QG_OP_FP4_LINEAR, M, K, N, dt, alpha)
    Y = qg.fp4_linear(A, codesT, t, W, alpha, ws=ws)
    qg.check_status(ws, "block16k layer")
    parts = qg.linear_parts(ws, M, K, N, dt, alpha)
    A_h, W_h = A.cpu(), W.cpu()
    del A
    act = oracle.quantize_act(A_h, alpha)
    assert float(_np(parts["T"])[0]) == act["T"]
    assert np.array_equal(_np(parts["scales"]), act["scales"])
    assert np.array_equal(_np(parts["codes"]), act["codes"])
    rp, col, val = parts["csr"].to_host()
    assert np.array_equal(rp, act["row_ptr"])
    assert np.array_equal(col, act["col"]) and np.array_equal(val, act["val"])
    oT, ot = oracle.quantize_cols(W_h)
    assert np.array_equal(_np(t), ot) and np.array_equal(_np(codesT), oT)
    rows = np.unique(np.concatenate([np.random.default_rng(M + N + layer).integers(0, M, 30),
                                     [0, M - 1]]))
    acc = oracle.gemm_acc(act["codes"], oT, K, rows=rows)
    Yo = oracle.linear_y(acc, act["scales"], ot, act["row_ptr"], act["col"], act["val"], W_h,
                         rows=rows)
    assert y_rel_err(_np(Y[torch.from_numpy(rows).cuda()]), Yo) <= 1e-3


def test_quantize_act_sweep_256m_elements(qg):
    """The largest quantizer-sweep size, A = 65536 x 4096 bf16 Student-t(3),
    alpha = 0.99: T, codes, scales and the CSR over the whole tensor."""
    M, K, alpha = 65536, 4096, 0.99
    A = make_matrix((M, K), ("student_t", 3), seed=5008, device="cuda", dtype=torch.bfloat16)
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, alpha)
    codes, scales, csr, T = qg.quantize_act(A, alpha, ws=ws)
    qg.check_status(ws, "sweep 256M")
    A_h = A.cpu()
    del A
    exp = oracle.quantize_act(A_h, alpha)
    assert float(_np(T)[0]) == exp["T"]
    assert np.array_equal(_np(scales), exp["scales"])
    assert np.array_equal(_np(codes), exp["codes"])
    rp, col, val = csr.to_host()
    assert np.array_equal(rp, exp["row_ptr"])
    assert np.array_equal(col, exp["col"]) and np.array_equal(val, exp["val"])
