"""GPU checks of the measurement and failure-handling paths.

* The tensor-pipe MMA loop (qg_fp4_mma_loop), whose rate is the FP4 GEMM's
  ceiling: its accumulator must equal `iters` times the product of the two
  operand tiles it keeps in shared memory, computed here on the CPU from the
  same word generator and the E2M1 value table, so a wrong descriptor or a
  dropped MMA cannot pass for a fast loop.
* A bounded device wait that runs out: the cooperative activation kernel's grid
  barrier is given a count that no CTA can complete (set from the host in the
  workspace), so every CTA's wait gives up after its limit (about a second),
  the call reports QG_ERR_TIMEOUT through qg_sync_status, and the next call on
  the same workspace is clean and exact.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import make_matrix

pytestmark = pytest.mark.gpu

BN = 224


@pytest.fixture(scope="module")
def qg():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import quantize_gemm_b200
    torch.cuda.set_device(0)
    return quantize_gemm_b200


def _loop_tiles(cta: int):
    """The loop's operand tiles of one CTA as logical rows of 128 bytes (the
    128-byte swizzle undone): A 128 rows, W^T 224 rows."""
    n_words = (128 * 128 + BN * 128) // 4
    i = np.arange(n_words, dtype=np.uint64)
    h = (i * np.uint64(2654435761) + np.uint64(cta)) & np.uint64(0xFFFFFFFF)
    h ^= h >> np.uint64(15)
    w = ((h * np.uint64(2246822519)) & np.uint64(0xFFFFFFFF)).astype("<u4")
    b = w.view(np.uint8)

    def unswizzle(t):
        out = np.empty_like(t)
        for r in range(t.shape[0]):
            for c in range(8):
                p = c ^ (r % 8)
                out[r, 16 * c:16 * c + 16] = t[r, 16 * p:16 * p + 16]
        return out

    return unswizzle(b[:128 * 128].reshape(128, 128)), unswizzle(b[128 * 128:].reshape(BN, 128))


def _decode(tile):
    vals = oracle.e2m1_values()
    lo, hi = tile & 0x0F, tile >> 4
    out = np.empty((tile.shape[0], 2 * tile.shape[1]), dtype=np.float64)
    out[:, 0::2] = vals[lo]
    out[:, 1::2] = vals[hi]
    return out


@pytest.mark.parametrize("pair", [False, True])
@pytest.mark.parametrize("iters", [1, 64])
def test_mma_loop_accumulator_matches_cpu_product(qg, pair, iters):
    ws = qg.Workspace(qg.QG_OP_FP4_GEMM, 1, 32, 1, qg.QG_F32)
    acc = torch.full((128, BN), -1.0, dtype=torch.float32, device="cuda")
    flops = qg.fp4_mma_loop(iters, pair, ws, acc_out=acc)
    qg.check_status(ws, "mma loop")
    A0, B0 = _loop_tiles(0)
    if pair:
        _, B1 = _loop_tiles(1)
        B = np.concatenate([B0[:BN // 2], B1[:BN // 2]])
    else:
        B = B0
    want = iters * (_decode(A0) @ _decode(B).T)
    got = acc.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, want)
    ctas = flops / (2.0 * 128 * BN * 64 * 4 * iters)
    assert ctas >= 2 and ctas == int(ctas)


def test_grid_barrier_wait_times_out_and_recovers(qg):
    A = make_matrix((2048, 1024), ("student_t", 4), seed=21, device="cuda", dtype=torch.bfloat16)
    alpha = 0.99
    M, K = A.shape
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, alpha)
    exp = oracle.quantize_act(A.cpu(), alpha)
    codes, scales, csr, T = qg.quantize_act(A, alpha, ws=ws)
    assert ws.sync_status() == qg.QG_OK
    # grid barrier words at bytes 16..23 of the workspace: a count that the
    # CTAs' arrivals can never bring to "last"
    stuck = torch.tensor([1 << 30, 0], dtype=torch.int32).view(torch.uint8).cuda()
    ws.buf[16:24].copy_(stuck)
    st = qg.qg_quantize_act(A, alpha, codes, scales, csr, T, ws)
    assert st == qg.QG_OK                       # the launch itself is fine
    assert ws.sync_status() == qg.QG_ERR_TIMEOUT
    assert int(ws.buf[16:24].view(torch.int32)[0].item()) == 0   # barrier words reset
    codes, scales, csr, T = qg.quantize_act(A, alpha, ws=ws)
    assert ws.sync_status() == qg.QG_OK
    assert float(T.item()) == exp["T"]
    assert np.array_equal(codes.cpu().numpy(), exp["codes"])
    assert np.array_equal(scales.cpu().numpy(), exp["scales"])
    rp, col, val = csr.to_host()
    assert np.array_equal(rp, exp["row_ptr"]) and np.array_equal(col, exp["col"])
    assert np.array_equal(val, exp["val"])
