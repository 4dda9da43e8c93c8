"""GPU checks of the one-kernel deferred read.

dl_log_append_read runs as one persistent kernel (prep warps a few heads
ahead of decode warps, the key-side results handed over in shared memory)
when the base is fp32 or bf16, L <= 16, d_v <= 128 and there are at least 32
heads per SM, and as two kernels (replay_prep, then append_decode through a
workspace) otherwise. dl_log_append_read_noalloc always takes the two-kernel
form, so it serves here as the reference: both forms evaluate the same
products and sums in the same order, and must agree bit for bit at every log
fill n = 0 .. L-1, in o and in the log slot and X row each call appends,
while the base stays unwritten. Every case has 32 heads per SM plus a ragged
37 (so blocks hold different head counts and the slot ring wraps), and the
cases cover every decay rule, both input and base dtypes, and every d_k x d_v
tiling of the decode unit. Some are also held to the fp64 oracle's eager
outputs at the parity bar. Afterwards no bounded wait may have run out (the
fault word is 0).
"""
import numpy as np
import pytest

import gated_delta_rule_104_b200._binding as b
import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    b.load()
    b.dl_device_faults(clear=True)


CASES = [
    # (decay, input dtype, state dtype, d_k, d_v, H, L, oracle check)
    (W.CHANNEL, "bf16", "f32", 128, 128, 32, 16, False),
    (W.HEAD, "bf16", "bf16", 128, 128, 16, 8, True),
    (W.RWKV6, "bf16", "f32", 128, 64, 8, 16, False),
    (W.CHANNEL, "f32", "f32", 64, 128, 5, 12, True),
    (W.HEAD, "f32", "bf16", 64, 64, 3, 5, True),
    (W.RWKV6, "f32", "f32", 64, 64, 1, 1, True),
    (W.CHANNEL, "bf16", "bf16", 128, 64, 7, 16, False),
]


def _batch(H):
    """Batch size giving 32 heads per SM plus a ragged 37."""
    import torch

    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return -(-(32 * sms + 37) // H)


def _rel(x, ref):
    x = np.asarray(x, np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-300))


@pytest.mark.parametrize("decay,in_dtype,s_dtype,d_k,d_v,H,L,check_oracle", CASES)
def test_fused_read_matches_two_kernel_form(decay, in_dtype, s_dtype, d_k, d_v, H, L, check_oracle):
    import torch

    B = _batch(H)
    w = W.Workload(f"fused_{decay}_{in_dtype}_{s_dtype}_{d_k}x{d_v}", decay, B, H, d_k, d_v, L, in_dtype, s_dtype,
                   0.1, (L,), seed=H * 7 + L)
    x = W.generate(w)
    d = W.device_inputs(w, x)
    rw = decay == W.RWKV6
    chan = decay != W.HEAD
    tdt = d["q"].dtype
    S = d["S0"]
    S_keep = S.clone()
    log_f = b.Log.allocate(B, H, d_k, d_v, L, tdt, chan, rwkv6=rw)
    log_s = b.Log.allocate(B, H, d_k, d_v, L, tdt, chan, rwkv6=rw)
    log_s.work = None
    o_f = torch.empty(B, H, d_v, device="cuda")
    o_s = torch.empty_like(o_f)
    o_ref = None
    if check_oracle:
        o_ref, _ = oracle.run_workload_heads(w, x, "eager")
        o_ref = np.asarray(o_ref).reshape(L, w.heads, d_v)
    tol = 2e-2 if s_dtype == "bf16" else 1e-4
    names = ("k", "v", "a") if rw else ("k", "v", "beta", "a", "x")
    for n in range(L):
        beta_n = None if rw else d["beta"][n]
        args = (d["q"][n], d["k"][n], d["v"][n], beta_n, d["a"][n])
        b.dl_log_append_read(S, log_f, n, *args, o_f)
        b.dl_log_append_read_noalloc(S, log_s, n, *args, o_s)
        torch.cuda.synchronize()
        assert torch.equal(o_f, o_s), (n, float((o_f - o_s).abs().max()))
        for name in names:
            assert torch.equal(getattr(log_f, name)[:, :, n], getattr(log_s, name)[:, :, n]), (name, n)
        if o_ref is not None:
            got = o_f.double().cpu().numpy().reshape(w.heads, d_v)
            assert _rel(got, o_ref[n]) <= tol, (n, _rel(got, o_ref[n]))
    assert torch.equal(S, S_keep), "the read wrote the base"
    assert b.dl_device_faults() == 0
