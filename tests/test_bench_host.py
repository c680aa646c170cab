"""Host-side logic of bench.py that the multi-GPU runs rely on, on CPU:
max-over-ranks timing with a world_size-2 gloo group, the weak-scaling
aggregate, and the seeded workload generator."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from workloads import WORKLOADS, make_layer_inputs, seed_for


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        m = bench.max_over_ranks(ms, world)
        v = bench.weak_scaling_value(100.0, 4, m, world)
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        m, v = out[r]
        assert m == 15.0                              # the slowest rank's time
        assert v == pytest.approx(2 * 100.0 * 4 / 15e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(10.0, 2, 4.0, 1) == pytest.approx(5000.0)


def test_workload_generator_is_seeded_and_shaped():
    A1, W1 = make_layer_inputs("tiny", 0, device="cpu")
    A2, W2 = make_layer_inputs("tiny", 0, device="cpu")
    assert torch.equal(A1, A2) and torch.equal(W1, W2)
    wl = WORKLOADS["tiny"]
    assert A1.shape == (wl.M, wl.layers[0].K) and W1.shape == (wl.layers[0].K, wl.layers[0].N)
    assert A1.dtype == torch.float32
    # the 8-channel outliers: 0.5% of entries scaled by 50 lie in 8 columns
    big = (A1.abs() > 10).nonzero()
    assert 0 < big.shape[0] <= round(0.005 * A1.numel())
    assert len(set(big[:, 1].tolist())) <= 8
    A3, _ = make_layer_inputs("llama1.3b", 0, device="cpu", M=64)
    assert A3.dtype == torch.bfloat16 and A3.shape == (64, 2048)
    assert seed_for(WORKLOADS["llama7b"], 3) == 2003


def _ref_args(steps, warmup):
    import argparse
    return argparse.Namespace(workload="tiny", layer=None, steps=steps, warmup=warmup, alpha=None)


@pytest.mark.parametrize("budget", [bench.REFERENCE_BUDGET_S, 1e-3])
def test_reference_arm_line_and_bounded_sample(monkeypatch, budget):
    """The reference arm (the oracle on the host) prints the contract's fields;
    with a tiny time budget every step falls back to the smallest sample (32-row
    and 32-column slices, one Y row per layer) and still reports the metric."""
    monkeypatch.setattr(bench, "REFERENCE_BUDGET_S", budget)
    line = bench.reference_arm(_ref_args(steps=4, warmup=3), 0, 1)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in line
    assert line["impl"] == "reference" and line["steps"] == 4 and line["warmup"] == 3
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    # the same workload description as the GPU arm's line
    args = _ref_args(steps=4, warmup=3)
    wl = WORKLOADS[args.workload]
    shared = bench.workload_config(wl, list(wl.layers), wl.alphas[0])
    assert {k: line["config"][k] for k in shared} == shared
    sample = line["cpu_baseline"]["sample"]
    if budget < 1:
        assert "fraction" in sample
    else:
        assert "full tensors" in sample


def test_cpu_baseline_is_bounded_and_labelled(monkeypatch):
    """The GPU arm's cpu_baseline times the oracle on a bounded sample: with a
    tiny budget it falls back to the smallest slices and says so."""
    import types
    wl = WORKLOADS["tiny"]
    A, W = make_layer_inputs("tiny", 0, device="cpu")
    L = types.SimpleNamespace(A=A, W=W, alpha=0.99, flops=2 * A.shape[0] * A.shape[1] * W.shape[1])
    monkeypatch.setattr(bench, "CPU_BASELINE_BUDGET_S", 1e-3)
    out = bench.cpu_baseline(None, wl, [L])
    assert out["kind"] == "oracle" and out["cores"] >= 1 and out["value"] > 0
    assert 0 < out["sample_fraction"] < 1 and "fraction" in out["sample"]
    assert out["sample_wall_s"] < 60


def test_layer_order_follows_the_library_switch():
    """The bench times each layer's two kernels in the order qg_fp4_linear
    picks: at the 7B block's size, GEMM first at alpha 0.99 (41 and 110
    clamped entries per row possible) and SpMM first at 0.999 (4 and 11, below
    the switch of 10 per 4096 of K) on every layer."""
    from types import SimpleNamespace
    import quantize_gemm_b200 as qg
    wl = WORKLOADS["block16k"]
    for a in wl.alphas:
        for lay in wl.layers:
            L = SimpleNamespace(M=wl.M, K=lay.K, N=lay.N, alpha=a)
            order = bench.layer_order(qg, L)
            assert order[:2] == ("quantize_cols", "quantize_act")
            assert sorted(order[2:]) == ["fp4_gemm", "spmm"]
            assert (order[2] == "fp4_gemm") == qg.linear_adds_into_y(wl.M, lay.K, a)
            assert (order[2] == "fp4_gemm") == (a == 0.99)
