"""Full-size parity: every workload at its full size, run in the launch
configuration bench.py times (all T steps through the C ABI; deferred on the
fused schedule with the workload's log capacity, plus the unfused schedule
for the benchmarked workload), checked against the fp64 oracle on sampled
heads (each head's whole history is generated alone and replayed by the
oracle), and, on every head, by properties that hold at any size: the eager
and deferred final states agree and every output is finite.

Tolerances as in test_parity_gpu: max|delta| / max|ref| <= 1e-4 (fp32 state)
or 2e-2 (bf16 state), over all steps of o and over the final state.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import rel_err, run_cuda, state_to_f64, tolerance


@pytest.fixture
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def sample_heads(w, n=6, seed=1):
    n = min(n, w.heads)
    rng = np.random.default_rng(seed)
    picks = {h for h in (0, w.heads - 1, w.H, w.heads // 2) if h < w.heads}
    while len(picks) < n:
        picks.add(int(rng.integers(w.heads)))
    return sorted(picks)


def schedules(w):
    out = [("eager", 0, True)]
    for L in w.L:
        out.append(("deferred", L, True))
    if w.name == "kda_b256_h32_d128_t512":
        out.append(("deferred", w.L[0], False))
    return out


def test_sampled_heads_are_valid():
    for w in W.WORKLOADS.values():
        hs = sample_heads(w)
        assert len(hs) == min(6, w.heads) and all(0 <= h < w.heads for h in hs)


@pytest.mark.gpu
@pytest.mark.slow
@pytest.mark.timeout(900)
@pytest.mark.parametrize("name", W.WORKLOAD_ORDER)
def test_full_size(name, _cuda):
    import torch

    w = W.WORKLOADS[name]
    heads = sample_heads(w)
    d = W.device_inputs_chunked(w, workers=W.default_workers())
    ref = W.generate(w, heads=heads)
    o_ref, S_ref = oracle.run_workload_heads(w, ref, "eager")
    tol = tolerance(w)
    idx = torch.tensor(heads, device="cuda")
    finals = {}
    for path, L, fused in schedules(w):
        o, S = run_cuda(w, d, path, L, fused, o_heads=idx)
        assert np.isfinite(o).all()
        S_all = S.view(w.heads, w.d_v, w.d_k)
        assert bool(torch.isfinite(S_all).all())
        S_s = state_to_f64(S_all[idx])
        eo, es = rel_err(o, o_ref), rel_err(S_s, S_ref)
        assert eo <= tol and es <= tol, f"{name} {path} L={L} fused={fused}: o {eo:.3e} S {es:.3e}"
        finals[(path, L, fused)] = S_all.float()
        del S
    # every head: the deferred schedules end where the eager one does
    S_e = finals[("eager", 0, True)]
    scale = float(S_e.abs().max())
    for key, S_d in finals.items():
        if key[0] == "deferred":
            diff = float((S_d - S_e).abs().max()) / scale
            assert diff <= 2 * tol, (name, key, diff)
