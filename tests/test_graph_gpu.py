"""The deferred decode runs inside a CUDA graph (GPU).

Every entry point only enqueues kernels on the caller's stream (programmatic
dependent launches included), so a caller can capture a whole decode loop once
and replay it. This test captures 16 steps of the fused deferred schedule
(append-reads, the fused merge-read and a final flush) on a side stream and
checks that replaying the graph gives bit-identical outputs and state to the
same calls made directly.
"""
import numpy as np
import pytest

import workloads as W
from tests.gpu_util import device_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("decay", [W.CHANNEL, W.RWKV6])
def test_captured_decode_matches_direct_calls(decay):
    import torch

    import gated_delta_rule_104_b200 as g

    w = W.Workload("graph", decay, 4, 8, 128, 128, 16, "bf16", "f32", 0.1, (8,), seed=11)
    d = device_inputs(w, W.generate(w))
    rw = decay == W.RWKV6
    B, H = w.B, w.H

    def run(S, log, outs, stream):
        dec = g.DeferredDecoder(S, log, fused_merge=True)
        for t in range(w.T):
            beta = None if rw else d["beta"][t]
            dec.step(d["q"][t], d["k"][t], d["v"][t], beta, d["a"][t], outs[t], stream)
        dec.flush(stream)

    # direct calls
    S_d = d["S0"].clone()
    log_d = g.Log.allocate(B, H, 128, 128, 8, torch.bfloat16, True, rwkv6=rw)
    o_d = [torch.empty(B, H, 128, device="cuda") for _ in range(w.T)]
    run(S_d, log_d, o_d, torch.cuda.current_stream())
    torch.cuda.synchronize()

    # captured once, replayed twice from the same starting state
    S_g = d["S0"].clone()
    log_g = g.Log.allocate(B, H, 128, 128, 8, torch.bfloat16, True, rwkv6=rw)
    o_g = [torch.empty(B, H, 128, device="cuda") for _ in range(w.T)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        run(S_g, log_g, o_g, side)
    for _ in range(2):
        S_g.copy_(d["S0"])
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(S_g, S_d)
    for t in range(w.T):
        assert torch.equal(o_g[t], o_d[t]), t
    assert np.isfinite(S_g.cpu().numpy()).all()
    del graph
