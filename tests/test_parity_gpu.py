"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bar (per workload, over all steps): max|o - o_ref| / max|o_ref| and, after the
last step (deferred: after the final merge), max|S - S_ref| / max|S_ref| are
at most 1e-4 for an fp32 state and 2e-2 for a bf16 state. The oracle reads
the same rounded inputs; its fp64 result is the reference for both schedules
(DeltaLog reproduces the eager recurrence exactly up to rounding: Technical
Summary, "Methodology").
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import device_inputs, rel_err, run_cuda, state_to_f64, tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_104_b200 as g

    g.load()


def check(w, path, L=0, fused=True, x=None):
    x = x if x is not None else W.generate(w)
    o_ref, S_ref = oracle.run_workload_heads(w, x, "eager")
    d = device_inputs(w, x)
    o, S = run_cuda(w, d, path, L, fused)
    S = state_to_f64(S).reshape(S_ref.shape)
    eo, es = rel_err(o, o_ref), rel_err(S, S_ref)
    tol = tolerance(w)
    assert eo <= tol and es <= tol, f"{w.name} {path} L={L} fused={fused}: o {eo:.3e} S {es:.3e} (tol {tol})"
    return eo, es


# --------------------------------------------------------------- small case, whole

@pytest.mark.parametrize("path,L,fused", [("eager", 0, True), ("deferred", 4, True), ("deferred", 4, False),
                                          ("deferred", 16, True), ("deferred", 16, False),
                                          ("deferred", 1, True), ("deferred", 5, False)])
def test_gdn_small_fp32(path, L, fused):
    check(W.WORKLOADS["gdn_b1_h2_d64_t16"], path, L, fused)


@pytest.mark.parametrize("path,L,fused", [("eager", 0, True), ("deferred", 4, True), ("deferred", 4, False),
                                          ("deferred", 16, True), ("deferred", 1, True), ("deferred", 5, False)])
def test_rwkv6_small_fp32(path, L, fused):
    check(W.scaled(W.WORKLOADS["gdn_b1_h2_d64_t16"], name="rwkv6_b1_h2_d64_t16", decay=W.RWKV6), path, L, fused)


# --------------------------------------------------------------- reduced sizes of each workload

REDUCED = [
    (W.scaled(W.WORKLOADS["gdn_b64_h16_d128_t1024"], B=3, H=4, T=45), 8),
    (W.scaled(W.WORKLOADS["kda_b256_h32_d128_t512"], B=3, H=5, T=40), 16),
    (W.scaled(W.WORKLOADS["gdn_b1024_h32_dk128_dv256_t256"], B=2, H=3, T=29), 8),
    (W.scaled(W.WORKLOADS["rwkv6_b256_h32_d128_t512"], B=3, H=5, T=40), 16),
]


@pytest.mark.parametrize("w,L", REDUCED, ids=[w.name for w, _ in REDUCED])
@pytest.mark.parametrize("sched", ["eager", "fused", "unfused"])
def test_reduced_workloads(w, L, sched):
    x = W.generate(w)
    if sched == "eager":
        check(w, "eager", x=x)
    else:
        check(w, "deferred", L, sched == "fused", x=x)


@pytest.mark.parametrize("L", [1, 4, 8, 16, 32, 64])
def test_kda_log_length_sweep_reduced(L):
    w = W.scaled(W.WORKLOADS["kda_b128_h16_d128_t2048"], B=2, H=2, T=150)
    x = _SWEEP_INPUTS.setdefault(w, W.generate(w))
    check(w, "deferred", L, True, x=x)
    check(w, "deferred", L, False, x=x)


_SWEEP_INPUTS = {}


# --------------------------------------------------------------- every supported shape and dtype

COMBOS = [(dk, dv, sd, idt, dec) for dk in (64, 128) for dv in (64, 128, 256) for sd in ("f32", "bf16")
          for idt in ("f32", "bf16") for dec in (W.HEAD, W.CHANNEL, W.RWKV6)]


@pytest.mark.parametrize("dk,dv,sd,idt,dec", COMBOS)
def test_every_shape_and_dtype(dk, dv, sd, idt, dec):
    w = W.Workload(f"combo_{dk}_{dv}_{sd}_{idt}_{dec}", dec, 2, 2, dk, dv, 11, idt, sd, 0.3, (4,), seed=3)
    x = W.generate(w)
    check(w, "eager", x=x)
    check(w, "deferred", 4, True, x=x)
    check(w, "deferred", 4, False, x=x)


# --------------------------------------------------------------- degenerate cases

def _custom(w, **over):
    x = W.generate(w)
    for k, val in over.items():
        x[k] = val(x[k]) if callable(val) else val
    return x


def test_zero_decay_resets_state():
    """a = 0 forgets everything: S_t = beta_t v_t k_t^T each step."""
    w = W.Workload("zero_decay", W.CHANNEL, 2, 3, 128, 128, 9, "f32", "f32", 0.1, (4,))
    x = _custom(w, a=lambda a: np.zeros_like(a))
    for path, L, fused in (("eager", 0, True), ("deferred", 4, True), ("deferred", 4, False)):
        check(w, path, L, fused, x=x)


def test_rwkv6_zero_decay_keeps_last_outer_product():
    """RWKV6 with a = 0: S_t = v_t k_t^T each step; with a = 1 it is plain
    linear attention, S_t = S_0 + sum v k^T (both against the oracle)."""
    w = W.Workload("rwkv6_decays", W.RWKV6, 2, 3, 128, 64, 9, "f32", "f32", 0.1, (4,))
    for fill in (np.zeros_like, np.ones_like):
        x = _custom(w, a=lambda a: fill(a))
        for path, L, fused in (("eager", 0, True), ("deferred", 4, True), ("deferred", 4, False)):
            check(w, path, L, fused, x=x)


def test_beta_zero_and_unit_decay_keep_state():
    w = W.Workload("identity", W.HEAD, 2, 2, 64, 128, 7, "f32", "f32", 0.1, (3,))
    x = _custom(w, beta=lambda b: np.zeros_like(b), a=lambda a: np.ones_like(a))
    for path, L, fused in (("eager", 0, True), ("deferred", 3, True), ("deferred", 3, False)):
        check(w, path, L, fused, x=x)


def test_single_head_minimum():
    w = W.Workload("one_head", W.CHANNEL, 1, 1, 64, 64, 5, "bf16", "f32", 0.1, (64,))
    x = W.generate(w)
    check(w, "eager", x=x)
    check(w, "deferred", 64, True, x=x)   # log never fills: only the final flush merges


def test_deferred_L1_close_to_eager():
    """With L = 1 every step merges; the result matches eager to fp32 rounding."""
    import torch

    w = W.Workload("l1", W.CHANNEL, 2, 4, 128, 128, 12, "bf16", "f32", 0.1, (1,))
    x = W.generate(w)
    d = device_inputs(w, x)
    o_e, S_e = run_cuda(w, d, "eager")
    o_d, S_d = run_cuda(w, d, "deferred", 1, True)
    assert rel_err(o_d, o_e.astype(np.float64)) < 1e-5
    assert rel_err(state_to_f64(S_d), state_to_f64(S_e)) < 1e-5
    assert torch.cuda.is_available()


def test_append_leaves_base_unwritten_and_logs_inputs():
    """dl_log_append_read writes only log slot n and o: the base is bit-identical
    afterwards and the slot holds the step's inputs unchanged."""
    import torch

    import gated_delta_rule_104_b200 as g

    w = W.Workload("append", W.CHANNEL, 2, 3, 128, 128, 3, "bf16", "f32", 0.1, (4,))
    d = device_inputs(w, W.generate(w))
    S = d["S0"].clone()
    before = S.clone()
    log = g.Log.allocate(2, 3, 128, 128, 4, torch.bfloat16, True)
    o = torch.empty(2, 3, 128, device="cuda")
    for t in range(3):
        g.dl_log_append_read(S, log, t, d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["a"][t], o)
    torch.cuda.synchronize()
    assert torch.equal(S, before)
    for t in range(3):
        assert torch.equal(log.k[:, :, t], d["k"][t]) and torch.equal(log.v[:, :, t], d["v"][t])
        assert torch.equal(log.beta[:, :, t], d["beta"][t]) and torch.equal(log.a[:, :, t], d["a"][t])
    with pytest.raises(g.DeltaLogError):
        g.dl_log_append_read(S, log, 4, d["q"][0], d["k"][0], d["v"][0], d["beta"][0], d["a"][0], o)


def test_rwkv6_log_has_no_beta_or_metadata():
    """An RWKV6 log is allocated without beta and x (null pointers through the
    ABI); appends store k, v, a unchanged and leave the base unwritten."""
    import torch

    import gated_delta_rule_104_b200 as g

    w = W.Workload("append_rwkv6", W.RWKV6, 2, 3, 128, 128, 3, "bf16", "f32", 0.1, (4,))
    d = device_inputs(w, W.generate(w))
    S = d["S0"].clone()
    before = S.clone()
    log = g.Log.allocate(2, 3, 128, 128, 4, torch.bfloat16, True, rwkv6=True)
    assert log.beta is None and log.x is None and log.kind == g.DL_RWKV6
    o = torch.empty(2, 3, 128, device="cuda")
    for t in range(3):
        g.dl_log_append_read(S, log, t, d["q"][t], d["k"][t], d["v"][t], None, d["a"][t], o)
    torch.cuda.synchronize()
    assert torch.equal(S, before)
    for t in range(3):
        assert torch.equal(log.k[:, :, t], d["k"][t]) and torch.equal(log.v[:, :, t], d["v"][t])
        assert torch.equal(log.a[:, :, t], d["a"][t])
