"""The multi-kernel sequences of the bf16 activation and column quantizers
(used when a device has no cooperative launch) against the oracle, bit-exact.

On a B200 the library takes the single cooperative kernels, so these paths
are reached by starting a fresh process with QGEMM_NO_COOPERATIVE=1 (read once,
when the library sets up the device)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import json, sys
sys.path.insert(0, ROOT)
import numpy as np
import torch
import quantize_gemm_b200 as qg
import oracle
from workloads import make_matrix
out = {}
cases = [("tiny", (64, 512), 0.99), ("ragged_k1056", (300, 1056), 0.99),
         ("many_outliers_k2048", (64, 2048), 0.3), ("rows_k4096", (128, 4096), 0.999)]
for name, shape, alpha in cases:
    A = make_matrix(shape, ("student_t", 4), seed=21, device="cuda", dtype=torch.bfloat16)
    M, K = A.shape
    ws = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, alpha)
    before = qg.qg_launch_count()
    codes, scales, csr, T = qg.quantize_act(A, alpha, ws=ws)
    qg.check_status(ws, name)
    launches = qg.qg_launch_count() - before
    exp = oracle.quantize_act(A.cpu(), alpha)
    rp, col, val = csr.to_host()
    ok = (float(T.cpu()[0]) == exp["T"] and np.array_equal(rp, exp["row_ptr"])
          and np.array_equal(col, exp["col"]) and np.array_equal(val, exp["val"])
          and np.array_equal(scales.cpu().numpy(), exp["scales"])
          and np.array_equal(codes.cpu().numpy(), exp["codes"]))
    out["act_" + name] = {"ok": bool(ok), "launches": int(launches)}
W = make_matrix((1024, 768), ("student_t", 4), seed=22, device="cuda", dtype=torch.bfloat16)
before = qg.qg_launch_count()
codesT, s = qg.quantize_cols(W)
torch.cuda.synchronize()
launches = qg.qg_launch_count() - before
exp_codes, exp_scales = oracle.quantize_cols(W.cpu())
ok = (np.array_equal(codesT.cpu().numpy(), exp_codes) and np.array_equal(s.cpu().numpy(), exp_scales))
out["cols"] = {"ok": bool(ok), "launches": int(launches)}
print(json.dumps(out))
'''


@pytest.mark.gpu
def test_multi_kernel_quantizers_match_the_oracle():
    env = dict(os.environ, QGEMM_NO_COOPERATIVE="1")
    r = subprocess.run([sys.executable, "-c", SCRIPT.replace("ROOT", repr(ROOT))], env=env,
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    for name, v in res.items():
        assert v["ok"], (name, v)
        # the multi-kernel sequences launch more than one kernel
        assert v["launches"] > 1, (name, v)
