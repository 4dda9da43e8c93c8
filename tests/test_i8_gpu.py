"""GPU parity of the int8 deferred base (DL_I8) against the fp64 oracle that
rounds its base at the same points (oracle.deferred(..., base_i8=True)).

The base holds int8 codes with one scale per state row (max|row| / 127,
nearest, ties to even) and is re-rounded by every merge. Both sides take the
rounding in fp32, so a conversion of the same fp32 state gives the same codes
and scales exactly. The kernels merge in about fp32 precision, the oracle in
fp64, so a merged value that lands within that difference of a rounding
boundary can round to the neighbouring code: one step, max|row| / 127, in
that element. Such flips are rare (an fp32-level
perturbation hits a boundary with probability ~1e-4 per element and merge).
The bar is therefore: max|delta| / max|ref| <= 2/127 over all outputs and the
final state, and at most 1% of the elements off by more than 1e-4 * max|ref|
(the rest agree to fp32 accumulation). Shapes, kinds and log lengths as in
test_parity_gpu; the initial base is rounded by dl_state_to_i8.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import device_inputs

pytestmark = pytest.mark.gpu

STEP_BOUND = 2.0 / 127.0
CLOSE = 1e-4
FRACTION = 0.01


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_104_b200 as g

    g.load()


def assert_i8_close(got, ref, what):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    scale = max(np.abs(ref).max(), 1e-300)
    err = np.abs(got - ref) / scale
    far = float((err > CLOSE).mean())
    assert err.max() <= STEP_BOUND and far <= FRACTION, f"{what}: max {err.max():.3e}, far fraction {far:.2e}"


def run_i8(w, x, L, fused=True):
    import torch

    import gated_delta_rule_104_b200 as g

    d = device_inputs(w, x)
    B, H = w.B, w.H
    chan, rw = w.decay != W.HEAD, w.decay == W.RWKV6
    S8 = g.I8State.allocate(B, H, w.d_k, w.d_v)
    g.dl_state_to_i8(d["S0"].float().contiguous(), S8)
    log = g.Log.allocate(B, H, w.d_k, w.d_v, L, d["q"].dtype, chan, rwkv6=rw)
    dec = g.DeferredDecoder(S8, log, fused_merge=fused)
    o = torch.empty(B, H, w.d_v, device="cuda")
    outs = []
    for t in range(w.T):
        dec.step(d["q"][t], d["k"][t], d["v"][t], None if rw else d["beta"][t], d["a"][t], o)
        outs.append(o.cpu().numpy().copy())
    dec.flush()
    S = torch.empty(B, H, w.d_v, w.d_k, device="cuda")
    g.dl_state_from_i8(S8, S)
    torch.cuda.synchronize()
    return np.stack(outs).reshape(w.T, B * H, w.d_v), S.cpu().numpy().astype(np.float64).reshape(B * H, w.d_v,
                                                                                                   w.d_k)


def oracle_i8(w, x, L):
    f = W.as_f64(w, x)
    chan, rw = w.decay != W.HEAD, w.decay == W.RWKV6
    return oracle.deferred(f["S0"], f["q"], f["k"], f["v"], f["beta"], f["a"], chan, L, rw, base_i8=True)


def test_conversion_matches_the_oracle_rounding():
    import torch

    import gated_delta_rule_104_b200 as g

    rng = np.random.default_rng(31)
    for dk, dv in ((64, 64), (128, 256)):
        S = (rng.standard_normal((3, 2, dv, dk)) * rng.uniform(0.01, 3.0, (3, 2, dv, 1))).astype(np.float32)
        S[0, 0, 5] = 0.0  # an all-zero row
        Sd = torch.from_numpy(S).cuda()
        S8 = g.I8State.allocate(3, 2, dk, dv)
        g.dl_state_to_i8(Sd, S8)
        back = torch.empty_like(Sd)
        g.dl_state_from_i8(S8, back)
        torch.cuda.synchronize()
        ref = oracle.quantize_i8(S.reshape(6, dv, dk).astype(np.float64)).reshape(S.shape)
        # integer work, decided in fp32 on both sides: the same codes, bit for bit
        assert np.array_equal(back.cpu().numpy().astype(np.float64), ref), f"round trip {dk}x{dv}"
        codes = S8.codes.cpu().numpy().astype(np.int32)
        assert np.abs(codes).max() <= 127 and (codes[0, 0, 5] == 0).all()
        sc = S8.scales.cpu().numpy()
        assert np.array_equal(sc, np.abs(S).max(axis=-1) / np.float32(127))
        # the codes reproduce the values exactly: value = code * scale in fp32
        assert np.array_equal(back.cpu().numpy(), (codes * sc[..., None]).astype(np.float32))


CASES = [(dk, dv, dec, idt) for dk, dv in ((64, 64), (128, 128), (128, 256), (64, 256))
         for dec in (W.HEAD, W.CHANNEL, W.RWKV6) for idt in ("f32", "bf16")]


@pytest.mark.parametrize("dk,dv,dec,idt", CASES)
def test_deferred_int8_base(dk, dv, dec, idt):
    w = W.Workload(f"i8_{dk}_{dv}_{dec}_{idt}", dec, 2, 2, dk, dv, 21, idt, "f32", 0.3, (4,), seed=5)
    x = W.generate(w)
    o_ref, S_ref = oracle_i8(w, x, 4)
    for fused in (True, False):
        o, S = run_i8(w, x, 4, fused)
        assert_i8_close(o, o_ref, f"{w.name} fused={fused} o")
        assert_i8_close(S, S_ref, f"{w.name} fused={fused} S")


@pytest.mark.parametrize("L", [1, 16, 32])
def test_int8_log_lengths(L):
    """L = 32 runs each merge as two 16-entry sub-merges through the on-chip tile."""
    w = W.Workload(f"i8_L{L}", W.CHANNEL, 2, 3, 128, 128, 70, "bf16", "f32", 0.1, (L,), seed=6)
    x = W.generate(w)
    o_ref, S_ref = oracle_i8(w, x, L)
    o, S = run_i8(w, x, L)
    assert_i8_close(o, o_ref, f"L={L} o")
    assert_i8_close(S, S_ref, f"L={L} S")


def test_int8_pool_matches_the_deferred_schedule():
    """An int8 pool whose rows are all listed every step follows the same
    deferred schedule per sequence as the plain int8 base."""
    import torch

    import gated_delta_rule_104_b200 as g

    w = W.Workload("i8_pool", W.CHANNEL, 3, 2, 64, 64, 19, "f32", "f32", 0.3, (4,), seed=8)
    x = W.generate(w)
    d = device_inputs(w, x)
    o_ref, S_ref = oracle_i8(w, x, 4)
    pool = g.Pool.allocate(w.B, w.H, w.d_k, w.d_v, 4, torch.int8, torch.float32, True)
    for b in range(w.B):
        pool.reset(b, d["S0"][b].float())
    slot = torch.arange(w.B, dtype=torch.int32, device="cuda")
    o = torch.empty(w.B, w.H, w.d_v, device="cuda")
    outs = []
    for t in range(w.T):
        g.dl_pool_step(pool, slot, d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["a"][t], o)
        outs.append(o.cpu().numpy().copy())
    g.dl_pool_flush(pool, slot)
    S = torch.empty(w.B, w.H, w.d_v, w.d_k, device="cuda")
    g.dl_state_from_i8(pool.S, S)
    torch.cuda.synchronize()
    assert int(pool.status.item()) == 0
    assert_i8_close(np.stack(outs).reshape(o_ref.shape), o_ref, "pool o")
    assert_i8_close(S.cpu().numpy().reshape(S_ref.shape), S_ref, "pool S")


def test_eager_rejects_an_int8_state():
    import torch

    import gated_delta_rule_104_b200 as g

    S8 = g.I8State.allocate(1, 1, 64, 64)
    x = torch.zeros(1, 1, 64, device="cuda")
    with pytest.raises(TypeError):
        g.dl_gdn_decode_step(S8, x, x, x, torch.zeros(1, 1, device="cuda"), torch.zeros(1, 1, device="cuda"), x)
