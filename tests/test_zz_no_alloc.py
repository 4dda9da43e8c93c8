"""The no-allocation deferred step (dl_log_append_read_noalloc).

Some callers cannot allocate device memory: a serving engine whose caching
allocator already holds the device's memory for its state pool, a plugin
host that passes a kernel only its input and output buffers, or a decode loop
that must not risk the device-wide synchronisation of a cudaMalloc. For them
the library offers a variant of dl_log_append_read whose scratch lives in a
fixed array inside the library instead of a caller-provided workspace.

These tests call it through the C ABI:
  * on a host-only check, sizes beyond the array are refused;
  * on the GPU, calls in a row fill a whole log (n = 0 .. L-1). Every output
    is compared with the fp64 oracle and with dl_log_append_read (with a
    workspace) within the 1e-4 relative bound of the parity tests, and the
    log slot and the row of the log's X matrix each call writes must equal
    the workspace variant's bit for bit. A merge of the log written by the
    no-allocation calls must then give the oracle's state;
  * the same at the array's limit (16384 heads at d_k = d_v = 128: exactly
    16 MiB of scratch) and on a GDN shape with d_v = 256 and a bf16 state.
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import gated_delta_rule_104_b200._binding as b
import workloads as W


def test_noalloc_refuses_sizes_beyond_its_array():
    """Host-side check only (no launch): B*H*(d_k+d_v)*4 above 16 MiB. The
    call goes through the prototype the binding's load() sets."""
    lib = b.load()
    fn = lib.dl_log_append_read_noalloc
    A = 0x7f0000000000
    B, H = 1024, 32  # 32768 heads * 384 floats * 4 bytes = 48 MiB of scratch
    log = b.dl_log(A + (1 << 40), A + (2 << 40), A + (3 << 40), A + (4 << 40), A + (5 << 40), b.DL_BF16, 8,
                   None, 0)
    big = 1 << 36
    rc = fn(A, b.DL_BF16, b.DL_DECAY_HEAD, ctypes.byref(log), 0, A + big, A + 2 * big, A + 3 * big,
            A + 4 * big, A + 5 * big, b.DL_BF16, A + 6 * big, B, H, 128, 256, None)
    assert rc == b.DL_ERR_UNSUPPORTED
    assert "DL_NOALLOC_WORK_BYTES" in lib.dl_last_error().decode()


def _rel(x, ref):
    x = np.asarray(x, np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-300))


def _fill_and_merge(w, L, oracle_mod):
    """L no-allocation appends (n = 0 .. L-1), each beside the workspace
    variant on its own log, then dl_log_merge of the no-allocation log."""
    import torch

    x = W.generate(w)
    d = W.device_inputs(w, x)
    o_ref, S_ref = oracle_mod.run_workload_heads(w, x, "eager")
    o_ref = np.asarray(o_ref).reshape(w.T, w.heads, w.d_v)
    tol = 2e-2 if w.state_dtype == "bf16" else 1e-4
    chan = w.decay != W.HEAD
    tdt = d["q"].dtype
    S = d["S0"].clone()
    S_keep = S.clone()
    log_ref = b.Log.allocate(w.B, w.H, w.d_k, w.d_v, L, tdt, chan)
    log_na = b.Log.allocate(w.B, w.H, w.d_k, w.d_v, L, tdt, chan)
    log_na.work = None  # the no-allocation call takes no workspace
    o_ws = torch.empty(w.B, w.H, w.d_v, device="cuda")
    o_na = torch.empty_like(o_ws)
    for n in range(L):
        args = (d["q"][n], d["k"][n], d["v"][n], d["beta"][n], d["a"][n])
        b.dl_log_append_read(S, log_ref, n, *args, o_ws)
        b.dl_log_append_read_noalloc(S, log_na, n, *args, o_na)
        torch.cuda.synchronize()
        got = o_na.double().cpu().numpy().reshape(w.heads, w.d_v)
        assert _rel(got, o_ws.double().cpu().numpy().reshape(w.heads, w.d_v)) <= 1e-4, n
        assert _rel(got, o_ref[n]) <= tol, (n, _rel(got, o_ref[n]))
        for name in ("k", "v", "beta", "a"):
            assert torch.equal(getattr(log_na, name)[:, :, n], getattr(log_ref, name)[:, :, n]), (name, n)
        assert torch.equal(log_na.x[:, :, n], log_ref.x[:, :, n]), ("x", n)
    assert torch.equal(S, S_keep), "the read wrote the base"
    b.dl_log_merge(S, log_na, L)
    torch.cuda.synchronize()
    got_S = S.double().cpu().numpy()
    err = _rel(got_S.reshape(np.asarray(S_ref).shape), np.asarray(S_ref))
    assert err <= tol, err


@pytest.mark.gpu
def test_noalloc_fills_a_log_that_merges_to_the_oracle(oracle_mod):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.Workload("noalloc_kda", W.CHANNEL, 8, 16, 128, 128, 8, "bf16", "f32", 0.1, (8,), seed=7)
    _fill_and_merge(w, 8, oracle_mod)


@pytest.mark.gpu
def test_noalloc_at_the_array_limit(oracle_mod):
    """16384 heads at d_k = d_v = 128: the scratch fills DL_NOALLOC_WORK_BYTES."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.Workload("noalloc_limit", W.CHANNEL, 512, 32, 128, 128, 3, "bf16", "f32", 0.1, (3,), seed=11)
    assert w.heads * (w.d_k + w.d_v) * 4 == b.DL_NOALLOC_WORK_BYTES
    _fill_and_merge(w, 3, oracle_mod)


@pytest.mark.gpu
def test_noalloc_gdn_dv256_bf16_state(oracle_mod):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.Workload("noalloc_gdn", W.HEAD, 4, 8, 128, 256, 5, "bf16", "bf16", 1.0, (5,), seed=3)
    _fill_and_merge(w, 5, oracle_mod)
