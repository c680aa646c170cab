"""The benchmark's step as one CUDA graph: capturing the library calls
(cooperative, cluster and plain launches) and replaying them gives the same
bytes as launching them eagerly, and the workspaces stay clean."""
import pytest
import torch

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


@pytest.mark.parametrize("workload", ["tiny", "llama1.3b"])
def test_graph_replay_matches_eager(qg, workload):
    import bench
    from workloads import WORKLOADS
    dev = torch.device("cuda", 0)
    wl = WORKLOADS[workload]
    layers = [bench.Layer(qg, wl, i, dev) for i in range(len(wl.layers))]
    bench.run_step(qg, layers)
    torch.cuda.synchronize()
    want = [(L.Y.clone(), L.codes.clone(), L.s.clone(), L.codesT.clone(), L.T.clone(),
             L.csr.nnz.clone()) for L in layers]
    graph, per_step = bench.capture_step(qg, layers)
    assert graph is not None and per_step >= 4 * len(layers)
    for L in layers:
        L.Y.zero_()
        L.codes.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    for L, w in zip(layers, want):
        for ws in L.workspaces():
            qg.check_status(ws, "replay")
        got = (L.Y, L.codes, L.s, L.codesT, L.T, L.csr.nnz)
        for g, e in zip(got, w):
            assert torch.equal(g, e)
