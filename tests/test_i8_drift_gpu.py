"""How far the int8 base drifts from the exact recurrence over a full run.

The int8 deferred base (DL_I8: int8 codes with one fp32 scale per state row,
max|row| / 127) is re-rounded at every merge. test_i8_gpu.py checks the
kernels against an oracle that rounds at the same points; this test measures
what a user of the int8 base gets against the exact recurrence O1 (the fp64
eager oracle, no rounding): the benchmarked workload (KDA, B=256, H=32,
d=128, bf16 inputs, 512 steps, L=16, fused merges, so 32 merges), on sampled
heads, over every step's output and the final state.

Bound. A merge rounds every element of a row to the nearest code step, so it
moves the element by at most half a step, max|row| / 254 <= max|S| / 254.
The transitions between merges do not amplify an error (decays a <= 1; the
delta rule's I - beta k k^T is a contraction for beta |k|^2 <= 2), so the
drift of the state after m merges (and the rounding of the initial state) is
at most the sum of the half steps, (m + 1) / 254 of max|S|; the output
o = S q inherits the same relative bound. The
rounding errors are independent and of either sign, so the observed drift is
far smaller: it grows like the square root of the number of merges, which is
checked too (the drift at the end against the drift after the first merges).
The numbers are printed (pytest -s) for the record.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.test_fullsize_gpu import sample_heads

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.timeout(900)
def test_int8_base_drift_from_the_exact_recurrence():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_104_b200 as g

    w = W.WORKLOADS["kda_b256_h32_d128_t512"]
    L = w.L[0]
    heads = sample_heads(w, n=8)
    d = W.device_inputs_chunked(w, workers=W.default_workers())
    o_ref, S_ref = oracle.run_workload_heads(w, W.generate(w, heads=heads), "eager")

    B, H = w.B, w.H
    S8 = g.I8State.allocate(B, H, w.d_k, w.d_v)
    g.dl_state_to_i8(d["S0"].float().contiguous(), S8)
    log = g.Log.allocate(B, H, w.d_k, w.d_v, L, d["q"].dtype, True)
    dec = g.DeferredDecoder(S8, log, fused_merge=True)
    o = torch.empty(B, H, w.d_v, device="cuda")
    idx = torch.tensor(heads, device="cuda")
    outs = []
    for t in range(w.T):
        dec.step(d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["a"][t], o)
        outs.append(o.view(-1, w.d_v)[idx].clone())
    dec.flush()
    S = torch.empty(B, H, w.d_v, w.d_k, device="cuda")
    g.dl_state_from_i8(S8, S)
    torch.cuda.synchronize()
    got_o = torch.stack(outs).cpu().numpy().astype(np.float64)
    got_S = S.view(-1, w.d_v, w.d_k)[idx].cpu().numpy().astype(np.float64)
    assert g.dl_device_faults() == 0

    scale_o = np.abs(o_ref).max()
    drift_o = np.abs(got_o - o_ref).max(axis=(1, 2)) / scale_o  # per step
    drift_S = float(np.abs(got_S - S_ref).max() / np.abs(S_ref).max())
    merges = w.T // L
    bound = (merges + 1) / 254.0
    early = float(drift_o[: 4 * L].max())  # the first four merges
    late = float(drift_o.max())
    print(f"\nint8 base vs exact recurrence, {w.name}, L={L}, {merges} merges, heads {heads}:")
    for t in (L, 4 * L, 8 * L, 16 * L, w.T):
        print(f"  o drift up to step {t}: {drift_o[:t].max():.3e}")
    print(f"  final state drift: {drift_S:.3e}; linear bound {bound:.3e}")
    assert np.isfinite(got_o).all() and np.isfinite(got_S).all()
    assert late <= bound and drift_S <= bound
    # independent roundings: far below the linear bound, and growing no faster
    # than the square root of the merge count (with a factor 2 of slack)
    assert late <= 2.0 * early * np.sqrt(merges / 4.0) + 1e-12
