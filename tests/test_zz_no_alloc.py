"""qg_quantize_cols_static: the column quantizer for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

It must give exactly what the workspace-based qg_quantize_cols gives, on
consecutive calls (the array keeps the previous call's contents, so a stale
column maximum would show up in the second call), and reject sizes beyond its
fixed capacity.  This file is collected last on purpose: when it fails, a run
that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from workloads import make_matrix

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


CASES = [(2048, 5504, torch.bfloat16, 1.0), (512, 512, torch.float32, 0.5),
         (64, 7, torch.bfloat16, 0.25), (4096, 65536, torch.bfloat16, 0.02)]


def test_static_scratch_matches_workspace_version_on_consecutive_calls(qg):
    for call in range(2):
        for i, (K, N, dtype, scale) in enumerate(CASES):
            # second round: smaller magnitudes, so leftover maxima would be wrong
            W = make_matrix((K, N), seed=100 * call + i, device="cuda", dtype=dtype,
                            scale=scale / (1 + 9 * call))
            ref_codes, ref_t = qg.quantize_cols(W)
            codes = torch.full_like(ref_codes, 0xAA)
            t = torch.full_like(ref_t, -1.0)
            st = qg.qg_quantize_cols_static(W, codes, t)
            assert st == qg.QG_OK, qg.qg_status_string(st)
            torch.cuda.synchronize()
            assert torch.equal(t, ref_t), (call, K, N)
            assert torch.equal(codes, ref_codes), (call, K, N)


def test_static_scratch_rejects_too_many_columns(qg):
    W = torch.zeros((32, 65537), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((65537, 16), dtype=torch.uint8, device="cuda")
    t = torch.empty(65537, dtype=torch.float32, device="cuda")
    before = qg.qg_launch_count()
    assert qg.qg_quantize_cols_static(W, codes, t) == qg.QG_ERR_UNSUPPORTED_SHAPE
    assert qg.qg_launch_count() == before      # nothing was enqueued
