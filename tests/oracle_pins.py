"""Pins for the CPU oracle: checks against values fixed by the pages or by
mathematics, never by the oracle itself.

Each ``pin_*`` function takes the oracle module (the real one, or a variant
built from a source with a planted mistake) and raises AssertionError when the
oracle disagrees with the pin.  ``tests/test_oracle_pins.py`` runs them on the
real oracle; ``tests/test_oracle_mutants.py`` checks that every planted mistake
fails at least one of them.

Independent references used here (none calls the oracle's arithmetic):
* the E2M1 magnitudes from the format's bit fields (1 sign, 2 exponent bits
  with bias 1, 1 mantissa bit);
* nearest-value search over that grid in double, ties to the even code;
* ``numpy.quantile(..., method="inverted_cdf")``, ``numpy.sort`` and a brute
  force count for the threshold;
* ``scipy.sparse`` for the CSR of dA and for dA * W;
* integer matrix products (numpy int64) for the FP4 accumulator;
* closed forms: matrices already on the scaled grid quantize to themselves;
* invariants: A_clamped + dA == A, |A_clamped| <= T, the nnz bound, each
  non-zero row carries a code of magnitude 6, the rounding error bound.
"""
from __future__ import annotations

import json
import os

import numpy as np
import scipy.sparse as sp

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "worked_examples.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- references
def format_grid() -> np.ndarray:
    """Value of each 4-bit code from the E2M1 bit fields (bias 1)."""
    out = np.empty(16)
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)
        out[c] = -mag if s else mag
    return out


def ref_encode(x) -> np.ndarray:
    """Nearest grid value by exhaustive distance search, ties to the even code."""
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    grid = format_grid()[:8]
    mag = np.abs(x.astype(np.float64))
    d = np.abs(mag[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    is_best = d == best
    # prefer even codes among equally near neighbours
    pref = np.where(is_best, np.where(np.arange(8) % 2 == 0, 2, 1), 0)
    code = np.argmax(pref, axis=1).astype(np.uint8)
    # above the largest grid value the nearest one is 6 (distances of huge
    # magnitudes all round to the same double, so decide these directly)
    code = np.where(mag > grid[-1], np.uint8(7), code).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 3
    return code | sign


def pack(codes_unpacked) -> np.ndarray:
    c = np.asarray(codes_unpacked, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def encoder_probe_inputs(rng) -> np.ndarray:
    """Every bf16 value, dense fp32 neighbourhoods of grid points and
    midpoints, special values and random fp32 bit patterns (no NaN)."""
    bf = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    grid = format_grid()[:8]
    mids = 0.5 * (grid[:-1] + grid[1:])
    centres = np.concatenate([grid, mids]).astype(np.float32)
    neigh = [centres]
    up = centres.copy()
    dn = centres.copy()
    for _ in range(64):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(-np.inf))
        neigh += [up.copy(), dn.copy()]
    neigh = np.concatenate(neigh)
    specials = np.array([0.0, np.inf, np.finfo(np.float32).max, np.finfo(np.float32).tiny,
                         1e-45, 6.0, 6.5, 7.0, 12.0, 1e38], dtype=np.float32)
    rnd = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32).view(
        np.float32)
    xs = np.concatenate([bf, neigh, -neigh, specials, -specials, rnd])
    return xs[~np.isnan(xs)]


# ------------------------------------------------------------------- pins
def pin_grid(orc):
    g = golden()["e2m1_grid"]
    vals = orc.e2m1_values()
    assert np.array_equal(vals, format_grid())
    assert np.array_equal(vals, np.array(g["values"]))
    assert np.array_equal(np.signbit(vals), np.signbit(np.array(g["values"])))


def pin_encoder_ties(orc):
    g = golden()["e2m1_ties"]
    got = orc.e2m1_encode(np.array(g["inputs"], dtype=np.float32))
    assert got.tolist() == g["codes"], (got.tolist(), g["codes"])


def pin_encoder_nearest_search(orc, seed=1):
    xs = encoder_probe_inputs(np.random.default_rng(seed))
    got = orc.e2m1_encode(xs)
    want = ref_encode(xs)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (xs[bad[:8]], got[bad[:8]], want[bad[:8]])


def pin_encode_bits_packed(orc, seed=15):
    """The packed sweep over consecutive fp32 bit patterns (the exhaustive GPU
    encoder test's reference) equals the independent nearest-value search on
    the same patterns, packed two per byte with the even pattern in the low
    nibble, NaN patterns mapped to code 0: ranges around zero, 1, the top grid
    value, the largest finite values into Inf and NaN (both signs), and random
    starts (odd ones included)."""
    rng = np.random.default_rng(seed)
    starts = [0x00000000, 0x3F7FFF00, 0x40BFFF01, 0x7F7FFF80, 0x7FBFFFF0, 0x807FFF00,
              0xBF7FFFF1, 0xFF7FFF80, 0xFFFFFE00]
    starts += [int(s) for s in rng.integers(0, (1 << 32) - 4096, size=6)]
    for start in starts:
        n = 2048
        bits = (np.arange(n, dtype=np.uint64) + np.uint64(start)).astype(np.uint32)
        x = bits.view(np.float32)
        want_codes = ref_encode(np.where(np.isnan(x), np.float32(0.0), x))
        want = pack(want_codes)
        got = orc.e2m1_encode_bits_packed(start, n)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (hex(start), int(bad[0]), got[bad[0]], want[bad[0]])


def pin_row_worked_example(orc):
    g = golden()["row_quantization"]
    codes, s = orc.quantize_rows(np.array([g["row"]], dtype=np.float32))
    assert codes[0].tolist() == g["codes_packed"]
    assert unpack(codes)[0].tolist() == g["codes_unpacked"]
    assert float(s[0]) == g["scale"]
    dq = orc.dequant_rows(codes, s)[0]
    assert dq.tolist() == g["dequant"]


def pin_col_worked_example(orc):
    g = golden()["column_quantization"]
    W = np.array(g["W"], dtype=np.float32)
    codesT, t = orc.quantize_cols(W)
    assert codesT.tolist() == g["codesT_packed"]
    assert t.tolist() == g["scales"]


def pin_threshold_worked_example(orc):
    g = golden()["threshold_clamp"]
    A = np.array(g["A"], dtype=np.float32)
    for case in g["cases"]:
        assert orc.quantile_rank(case["alpha"], A.size) == case["k"]
        T = orc.threshold(A, case["alpha"])
        assert T == case["T"]
        a_c, rp, col, val = orc.clamp_compensate(A, T)
        assert rp.tolist() == case["row_ptr"]
        assert col.tolist() == case["col"]
        assert val.tolist() == case["val"]
        assert a_c.tolist() == case["A_clamped"]


def pin_act_worked_example(orc):
    g = golden()["act_quantization"]
    out = orc.quantize_act(np.array(g["A"], dtype=np.float32), g["alpha"])
    assert out["T"] == g["T"]
    assert out["codes"].tolist() == g["codes_packed"]
    assert unpack(out["codes"]).tolist() == g["codes_unpacked"]
    assert out["scales"].tolist() == g["scales"]
    assert out["row_ptr"].tolist() == g["row_ptr"]
    assert out["col"].tolist() == g["col"]
    assert out["val"].tolist() == g["val"]


def pin_gemm_worked_example(orc):
    g = golden()["gemm"]
    acc = orc.gemm_acc(np.array(g["codesA_packed"], np.uint8),
                       np.array(g["codesWT_packed"], np.uint8), g["K"])
    assert acc.tolist() == g["acc"]


def _threshold_cases(rng):
    cases = []
    for n in (1, 2, 3, 7, 10, 64, 1000, 4097):
        cases.append(rng.standard_normal(n).astype(np.float32))
    # heavy tail with many ties (values rounded to 8 mantissa bits, like bf16)
    t = rng.standard_t(3, size=20000).astype(np.float32)
    cases.append((t.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32))
    cases.append(np.zeros(50, np.float32))
    cases.append(np.array([3.0, -3.0, 3.0, 0.0, -0.0], np.float32))
    return cases


def pin_threshold_vs_sort_and_quantile(orc, seed=2):
    rng = np.random.default_rng(seed)
    for a in _threshold_cases(rng):
        mag = np.sort(np.abs(a.astype(np.float64)))
        n = a.size
        for alpha in (1e-9, 0.1, 0.5, 0.9, 0.99, 0.999, 0.9999, 1.0):
            T = orc.threshold(a.reshape(1, -1), alpha)
            # brute force over the definition: the smallest |a| such that at
            # least ceil(alpha * n) entries are <= it
            need = int(np.ceil(alpha * n))
            need = min(max(need, 1), n)
            if n <= 1000:
                cands = [v for v in np.unique(mag) if np.count_nonzero(mag <= v) >= need]
                assert T == min(cands), (n, alpha, T, min(cands))
            assert T == mag[need - 1]
            q = np.quantile(np.abs(a.astype(np.float64)), alpha, method="inverted_cdf")
            assert T == q, (n, alpha, T, q)


def pin_clamp_invariants(orc, seed=3):
    rng = np.random.default_rng(seed)
    for (M, K, alpha) in ((7, 33, 0.9), (16, 64, 0.99), (40, 128, 0.999), (5, 8, 0.5)):
        A = (rng.standard_t(3, size=(M, K)) * 2).astype(np.float32)
        T = orc.threshold(A, alpha)
        a_c, rp, col, val = orc.clamp_compensate(A, T)
        # A_c + dA == A exactly (fp64)
        dA = sp.csr_matrix((val, col, rp), shape=(M, K)).toarray()
        assert np.array_equal(a_c.astype(np.float64) + dA, A.astype(np.float64))
        assert np.all(np.abs(a_c) <= T)
        # dA is non-zero exactly where |a| > T, in canonical CSR order
        mask = np.abs(A) > T
        ref = sp.csr_matrix(np.where(mask, A.astype(np.float64) - np.sign(A) * T, 0.0))
        ref.sort_indices()
        assert rp.tolist() == ref.indptr.tolist()
        assert col.tolist() == ref.indices.tolist()
        assert np.array_equal(val, ref.data)
        n = A.size
        assert col.size <= n - int(np.ceil(alpha * n))
        assert np.count_nonzero(np.abs(A) <= T) >= int(np.ceil(alpha * n))


def _on_grid_matrix(rng, M, K, exps):
    """Rows that are exactly on grid * 2^e with max magnitude 6 * 2^e."""
    grid = format_grid()[:8]
    codes = rng.integers(0, 8, size=(M, K))
    codes[np.arange(M), rng.integers(0, K, size=M)] = 7
    sign = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    A = sign * grid[codes] * (2.0 ** exps)[:, None]
    return A.astype(np.float32), codes, sign, exps


def pin_quantize_rows_identity(orc, seed=4):
    rng = np.random.default_rng(seed)
    M, K = 33, 64
    exps = rng.integers(-20, 20, size=M).astype(np.float64)
    A, codes, sign, exps = _on_grid_matrix(rng, M, K, exps)
    q, s = orc.quantize_rows(A)
    want = (codes | np.where(sign < 0, 8, 0)).astype(np.uint8)
    assert np.array_equal(unpack(q), want)
    assert np.array_equal(s.astype(np.float64), 2.0 ** exps)


def pin_quantize_rows_properties(orc, seed=5):
    rng = np.random.default_rng(seed)
    grid = format_grid()[:8]
    for (M, K, scale) in ((9, 32, 1.0), (20, 256, 1e-3), (3, 1024, 1e4)):
        A = (rng.standard_t(3, size=(M, K)) * scale).astype(np.float32)
        q, s = orc.quantize_rows(A)
        u = unpack(q)
        amax = np.abs(A).max(axis=1)
        assert np.array_equal(s, (amax / np.float32(6)).astype(np.float32))
        # every non-zero row has a code of magnitude 6
        assert np.all(np.any((u & 7) == 7, axis=1))
        # the dequantized value is the nearest grid point of a*r, so the
        # error is at most half the local grid gap times s (gap 2 above 4)
        r = (np.float32(6) / amax).astype(np.float32)
        x = (A * r[:, None]).astype(np.float32).astype(np.float64)
        dq = orc.dequant_rows(q, s) / s.astype(np.float64)[:, None]
        err = np.abs(np.abs(x) - np.abs(dq))
        gap = np.where(np.abs(x) > 4, 1.0, np.where(np.abs(x) > 2, 0.5, 0.25))
        assert np.all(err <= gap + 1e-6)
        # monotone in a within each row, odd symmetric in sign
        for i in range(M):
            order = np.argsort(A[i], kind="stable")
            v = orc.dequant_rows(q[i:i + 1], s[i:i + 1])[0][order]
            assert np.all(np.diff(v) >= 0)
        qn, sn = orc.quantize_rows(-A)
        assert np.array_equal(qn, q ^ np.uint8(0x88)) and np.array_equal(sn, s)
        assert set(np.unique(np.abs(orc.dequant_rows(q, s) / s[:, None]))) <= set(grid)


def pin_quantize_degenerate_rows(orc):
    A = np.zeros((4, 8), np.float32)
    A[1, :] = -0.0
    A[2, 3] = np.float32(1e-45)     # 6 / amax overflows fp32
    A[3, :] = np.float32(-1e-45)
    q, s = orc.quantize_rows(A)
    assert s.tolist() == [0.0, 0.0, 0.0, 0.0]
    assert unpack(q)[0].tolist() == [0] * 8
    assert unpack(q)[1].tolist() == [8] * 8
    assert unpack(q)[2].tolist() == [0] * 8
    assert unpack(q)[3].tolist() == [8] * 8


def pin_quantize_cols_transpose(orc, seed=6):
    rng = np.random.default_rng(seed)
    K, N = 64, 24
    exps = rng.integers(-10, 10, size=N).astype(np.float64)
    WT, codes, sign, exps = _on_grid_matrix(rng, N, K, exps)
    qT, t = orc.quantize_cols(np.ascontiguousarray(WT.T))
    want = (codes | np.where(sign < 0, 8, 0)).astype(np.uint8)
    assert np.array_equal(unpack(qT), want)
    assert np.array_equal(t.astype(np.float64), 2.0 ** exps)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    qT, t = orc.quantize_cols(W)
    assert np.array_equal(t, (np.abs(W).max(axis=0) / np.float32(6)).astype(np.float32))
    assert np.all(np.any((unpack(qT) & 7) == 7, axis=1))


def pin_gemm_vs_integer_matmul(orc, seed=7):
    rng = np.random.default_rng(seed)
    twice = (2 * format_grid()).astype(np.int64)   # integers
    for (M, N, K) in ((5, 7, 32), (33, 17, 256), (8, 8, 4096)):
        cA = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
        cW = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
        acc = orc.gemm_acc(cA, cW, K)
        ia = twice[unpack(cA)]
        iw = twice[unpack(cW)]
        ref = (ia @ iw.T).astype(np.float64) / 4.0
        assert np.array_equal(acc, ref)
        rows = np.array([M - 1, 0, M // 2])
        assert np.array_equal(orc.gemm_acc(cA, cW, K, rows=rows), ref[rows])


def pin_spmm_vs_scipy(orc, seed=8):
    rng = np.random.default_rng(seed)
    M, K, N = 30, 64, 40
    A = (rng.standard_t(3, size=(M, K))).astype(np.float32)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    T = orc.threshold(A, 0.9)
    _, rp, col, val = orc.clamp_compensate(A, T)
    C = orc.spmm(rp, col, val, W)
    ref = sp.csr_matrix((val, col, rp), shape=(M, K)) @ W.astype(np.float64)
    assert np.allclose(C, ref, rtol=1e-13, atol=1e-15)


def pin_linear_no_clamp_is_dequant_matmul(orc, seed=9):
    rng = np.random.default_rng(seed)
    M, K, N = 17, 128, 23
    A = rng.standard_normal((M, K)).astype(np.float32)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    act = orc.quantize_act(A, 1.0)
    assert act["col"].size == 0
    qT, t = orc.quantize_cols(W)
    acc = orc.gemm_acc(act["codes"], qT, K)
    Y = orc.linear_y(acc, act["scales"], t, act["row_ptr"], act["col"], act["val"], W)
    ref = orc.dequant_rows(act["codes"], act["scales"]) @ orc.dequant_rows(qT, t).T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-14)


def pin_linear_exact_on_grid(orc, seed=10):
    """A and W already on the scaled grid, no clamp: Y == A @ W exactly, and
    with a clamp Y == A @ W up to rounding (the correction restores A)."""
    rng = np.random.default_rng(seed)
    M, K, N = 12, 64, 10
    A, *_ = _on_grid_matrix(rng, M, K, rng.integers(-3, 3, size=M).astype(np.float64))
    WT, *_ = _on_grid_matrix(rng, N, K, rng.integers(-6, -2, size=N).astype(np.float64))
    W = np.ascontiguousarray(WT.T)
    exact = A.astype(np.float64) @ W.astype(np.float64)
    act = orc.quantize_act(A, 1.0)
    qT, t = orc.quantize_cols(W)
    acc = orc.gemm_acc(act["codes"], qT, K)
    Y = orc.linear_y(acc, act["scales"], t, act["row_ptr"], act["col"], act["val"], W)
    assert np.array_equal(Y, exact)
    # clamp on: Y = dq(A_c) W_q + dA W with W_q == W here; dq(A_c) differs
    # from A_c, so compare with the pieces: dA W exactly restores A - A_c
    act = orc.quantize_act(A, 0.9)
    assert act["col"].size > 0
    acc = orc.gemm_acc(act["codes"], qT, K)
    Y = orc.linear_y(acc, act["scales"], t, act["row_ptr"], act["col"], act["val"], W)
    dA = sp.csr_matrix((act["val"], act["col"], act["row_ptr"]), shape=(M, K)).toarray()
    ref = orc.dequant_rows(act["codes"], act["scales"]) @ W.astype(np.float64) + dA @ W
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


def pin_quantize_act_composition(orc, seed=11):
    rng = np.random.default_rng(seed)
    M, K = 24, 96
    A = (rng.standard_t(4, size=(M, K))).astype(np.float32)
    A[:, 5] *= 30
    out = orc.quantize_act(A, 0.99)
    n = A.size
    mag = np.sort(np.abs(A.astype(np.float64)).ravel())
    assert out["T"] == mag[int(np.ceil(0.99 * n)) - 1]
    T = np.float32(out["T"])
    A_c = np.where(np.abs(A) > T, np.sign(A) * T, A).astype(np.float32)
    q, s = orc.quantize_rows(A_c)
    assert np.array_equal(out["codes"], q) and np.array_equal(out["scales"], s)
    # amax_i = min(rowmax_i, T)
    amax = np.minimum(np.abs(A).max(axis=1), T)
    assert np.array_equal(out["scales"], (amax / np.float32(6)).astype(np.float32))


def pin_dgrad_exact_on_grid(orc, seed=12):
    """dY rows and W rows on their own scaled grids (spread exponents): the
    quantization along N is exact, so dA == dY @ W^T exactly.  Quantizing
    along the wrong dimension, a transposed operand or a lost scale breaks it
    (M, N, K all differ)."""
    rng = np.random.default_rng(seed)
    M, N, K = 12, 64, 20
    dY, *_ = _on_grid_matrix(rng, M, N, rng.integers(-4, 5, size=M).astype(np.float64))
    W, *_ = _on_grid_matrix(rng, K, N, rng.integers(-9, -1, size=K).astype(np.float64))
    exact = dY.astype(np.float64) @ W.astype(np.float64).T
    got = orc.dgrad(dY, W)
    assert got.shape == (M, K) and np.array_equal(got, exact)
    rows = [11, 0, 5]
    assert np.array_equal(orc.dgrad(dY, W, rows=rows), exact[rows])


def pin_wgrad_exact_on_grid(orc, seed=13):
    """A columns and dY columns on their own scaled grids: the quantization
    along the M tokens is exact, so dW == A^T @ dY exactly."""
    rng = np.random.default_rng(seed)
    M, K, N = 64, 18, 26
    AT, *_ = _on_grid_matrix(rng, K, M, rng.integers(-5, 4, size=K).astype(np.float64))
    dYT, *_ = _on_grid_matrix(rng, N, M, rng.integers(-12, -3, size=N).astype(np.float64))
    A, dY = np.ascontiguousarray(AT.T), np.ascontiguousarray(dYT.T)
    exact = A.astype(np.float64).T @ dY.astype(np.float64)
    got = orc.wgrad(A, dY)
    assert got.shape == (K, N) and np.array_equal(got, exact)
    rows = [17, 3]
    assert np.array_equal(orc.wgrad(A, dY, rows=rows), exact[rows])


def pin_grads_within_rounding_bound(orc, seed=14):
    """Off-grid inputs: |Q(x) - x| <= s for every element (the widest grid
    gap, 4 to 6, is 2 in units of s), so each gradient lies within
    sum(s_x |y| + |x| s_y + s_x s_y) of the exact product."""
    rng = np.random.default_rng(seed)
    M, K, N = 96, 40, 32
    A = rng.standard_t(4, size=(M, K)).astype(np.float32)
    W = (rng.standard_normal((K, N)) * 0.05).astype(np.float32)
    dY = (rng.standard_normal((M, N)) * 1e-3).astype(np.float32)
    a64, w64, d64 = (x.astype(np.float64) for x in (A, W, dY))
    # dgrad: scales per row of dY and per row of W (along N)
    sd = np.abs(d64).max(axis=1) / 6
    sw = np.abs(w64).max(axis=1) / 6
    bound = (sd[:, None] * (np.abs(w64).sum(axis=1))[None, :]
             + (np.abs(d64).sum(axis=1))[:, None] * sw[None, :]
             + N * sd[:, None] * sw[None, :])
    got = orc.dgrad(dY, W)
    err = np.abs(got - d64 @ w64.T)
    assert np.all(err <= bound * (1 + 1e-6)) and err.max() > 0
    # wgrad: scales per column of A and per column of dY (along M)
    sa = np.abs(a64).max(axis=0) / 6
    sy = np.abs(d64).max(axis=0) / 6
    bound = (sa[:, None] * (np.abs(d64).sum(axis=0))[None, :]
             + (np.abs(a64).sum(axis=0))[:, None] * sy[None, :]
             + M * sa[:, None] * sy[None, :])
    got = orc.wgrad(A, dY)
    err = np.abs(got - a64.T @ d64)
    assert np.all(err <= bound * (1 + 1e-6)) and err.max() > 0


# ------------------------------------------------------------ MXFP4 variant
def _mx_exponent_by_bits(amax: float) -> int:
    """The block exponent from the fp32 fields alone: with amax = m * 2^E,
    m in [1, 2), 6 * 2^e >= amax holds first at e = E - 2 when m <= 1.5 and
    at e = E - 1 when m > 1.5; clamped to [-127, 127]; -127 for zero."""
    a = np.float32(amax)
    if a == 0:
        return -127
    bits = int(np.array([a], dtype=np.float32).view(np.uint32)[0])
    ex, man = (bits >> 23) & 0xFF, bits & 0x7FFFFF
    if ex == 0:                       # subnormal: far below 6 * 2^-127
        return -127
    E = ex - 127
    e = E - 2 if man <= 0x400000 else E - 1
    return max(-127, min(127, e))


def pin_mx_worked_example(orc):
    g = golden()["mx_block_quantization"]
    codes, scales = orc.mx_quantize_rows(np.array(g["rows"], dtype=np.float32))
    assert np.array_equal(unpack(codes), np.array(g["codes_unpacked"], dtype=np.uint8))
    assert np.array_equal(scales, np.array(g["scales_e8m0"], dtype=np.uint8))
    dq = orc.mx_dequant_rows(codes, scales)
    for r, want in enumerate(g["dequant_first"]):
        assert np.array_equal(dq[r, :len(want)], np.array(want))
    for k, e in g["exponents"].items():
        assert orc.mx_exponent(float(k)) == e


def pin_mx_exponent_vs_bit_fields(orc, seed=20):
    rng = np.random.default_rng(seed)
    vals = [0.0, 1e-45, 1e-40, 2.0 ** -126, 3.4e38, 6.0, 3.0, 1.5, 0.75]
    for e in range(-125, 126, 7):
        for m in (1.0, 1.25, 1.5, 1.75, 1.9999999):
            vals.append(m * 2.0 ** e)
            vals.append(np.nextafter(np.float32(m * 2.0 ** e), np.float32(np.inf)))
            vals.append(np.nextafter(np.float32(m * 2.0 ** e), np.float32(0)))
    vals += list((rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000)).astype(np.float32))
    for v in vals:
        v = abs(float(np.float32(v)))
        assert orc.mx_exponent(v) == _mx_exponent_by_bits(v), v


def _mx_on_grid_rows(rng, M, K, espan=30):
    """Rows of 32-blocks, each block on grid * 2^e_b with its max 4 or 6 * 2^e_b,
    e_b in [-espan, espan)."""
    grid = format_grid()[:8]
    nb = K // 32
    codes = rng.integers(0, 8, size=(M, K))
    top = np.where(rng.random((M, nb)) < 0.5, 6, 7)            # grid 4 or 6
    codes = np.minimum(codes, np.repeat(top, 32, axis=1))
    pos = rng.integers(0, 32, size=(M, nb)) + 32 * np.arange(nb)
    codes[np.arange(M)[:, None], pos] = top
    sign = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    eb = rng.integers(-espan, espan, size=(M, nb))
    A = sign * grid[codes] * np.ldexp(1.0, np.repeat(eb, 32, axis=1))
    return A.astype(np.float32), codes, sign, eb


def pin_mx_rows_on_grid_identity(orc, seed=21):
    rng = np.random.default_rng(seed)
    A, codes, sign, eb = _mx_on_grid_rows(rng, 9, 128)
    q, s = orc.mx_quantize_rows(A)
    assert np.array_equal(s.astype(np.int64) - 127, eb)
    want = (codes | np.where(sign < 0, 8, 0)).astype(np.uint8)
    assert np.array_equal(unpack(q), want)
    assert np.array_equal(orc.mx_dequant_rows(q, s), A.astype(np.float64))


def pin_mx_rows_properties(orc, seed=22):
    """Off-grid rows: the exponent is minimal, nothing clips, and every value
    is within one block unit 2^e of its dequantized value (the widest grid
    gap, 4 to 6, is 2 units); a block of zeros keeps only sign bits."""
    rng = np.random.default_rng(seed)
    A = (rng.standard_t(3, size=(17, 256)) * 10.0 ** rng.integers(-5, 5, size=(17, 1))).astype(np.float32)
    A[3, 32:64] = 0.0
    A[4, 64:96] = -0.0
    q, s = orc.mx_quantize_rows(A)
    e = s.astype(np.int64) - 127
    amax = np.abs(A.astype(np.float64)).reshape(17, 8, 32).max(axis=2)
    nz = amax > 0
    assert np.all(np.ldexp(6.0, e)[nz] >= amax[nz])
    assert np.all((np.ldexp(6.0, e - 1) < amax)[nz & (e > -127)])
    assert np.all(e[~nz] == -127)
    dq = orc.mx_dequant_rows(q, s)
    unit = np.ldexp(1.0, np.repeat(e, 32, axis=1))
    assert np.all(np.abs(dq - A) <= unit)
    u = unpack(q)
    assert np.all(u[3, 32:64] == 0) and np.all(u[4, 64:96] == 8)


def pin_mx_cols_are_rows_of_transpose(orc, seed=23):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((96, 40)) * 0.02).astype(np.float32)
    qT, sT = orc.mx_quantize_cols(W)
    qr, sr = orc.mx_quantize_rows(np.ascontiguousarray(W.T))
    assert np.array_equal(qT, qr) and np.array_equal(sT, sr)


def pin_mx_gemm(orc, seed=24):
    """On-grid operands (block exponents within +-4, so every sum is exact in
    double): the block-scaled product is A @ W exactly; off-grid: it equals
    the product of the dequantized operands (numpy matmul)."""
    rng = np.random.default_rng(seed)
    M, N, K = 7, 11, 96
    A, *_ = _mx_on_grid_rows(rng, M, K, espan=4)
    WT, *_ = _mx_on_grid_rows(rng, N, K, espan=4)
    qa, sa = orc.mx_quantize_rows(A)
    qw, sw = orc.mx_quantize_rows(WT)
    Y = orc.mx_gemm(qa, sa, qw, sw, K)
    assert np.array_equal(Y, A.astype(np.float64) @ WT.astype(np.float64).T)
    B = rng.standard_t(4, size=(M, K)).astype(np.float32)
    W = rng.standard_normal((K, N)).astype(np.float32)
    qb, sb = orc.mx_quantize_rows(B)
    qwt, swt = orc.mx_quantize_cols(W)
    Y = orc.mx_gemm(qb, sb, qwt, swt, K)
    ref = orc.mx_dequant_rows(qb, sb) @ orc.mx_dequant_rows(qwt, swt).T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-300)
    assert np.array_equal(orc.mx_gemm(qb, sb, qwt, swt, K, rows=[6, 2]), Y[[6, 2]])


ALL_PINS = [
    pin_grid, pin_encoder_ties, pin_encoder_nearest_search, pin_encode_bits_packed,
    pin_row_worked_example,
    pin_col_worked_example, pin_threshold_worked_example, pin_act_worked_example,
    pin_gemm_worked_example, pin_threshold_vs_sort_and_quantile, pin_clamp_invariants,
    pin_quantize_rows_identity, pin_quantize_rows_properties, pin_quantize_degenerate_rows,
    pin_quantize_cols_transpose, pin_gemm_vs_integer_matmul, pin_spmm_vs_scipy,
    pin_linear_no_clamp_is_dequant_matmul, pin_linear_exact_on_grid,
    pin_quantize_act_composition, pin_dgrad_exact_on_grid, pin_wgrad_exact_on_grid,
    pin_grads_within_rounding_bound, pin_mx_worked_example, pin_mx_exponent_vs_bit_fields,
    pin_mx_rows_on_grid_identity, pin_mx_rows_properties, pin_mx_cols_are_rows_of_transpose,
    pin_mx_gemm,
]
