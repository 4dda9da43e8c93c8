"""The no-allocation deferred step (dl_log_append_read_noalloc).

Some callers cannot allocate device memory: a serving engine whose caching
allocator already holds the device's memory for its state pool, a plugin
host that passes a kernel only its input and output buffers, or a decode loop
that must not risk the device-wide synchronisation of a cudaMalloc. For them
the library offers a variant of dl_log_append_read whose scratch lives in a
fixed array inside the library instead of a caller-provided workspace.

These tests call it through the C ABI and check, on two calls in a row (log
fills n = 0 and n = 1), that its outputs and log writes equal those of
dl_log_append_read with a workspace, within the 1e-4 relative bound the
parity tests use, and that sizes beyond the array are refused. The file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import gated_delta_rule_104_b200._binding as b
import workloads as W


def test_noalloc_refuses_sizes_beyond_its_array():
    """Host-side check only (no launch): B*H*(d_k+d_v)*4 above 16 MiB."""
    lib = b.load()
    fn = lib.dl_log_append_read_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, i, i, ctypes.POINTER(b.dl_log), i, vp, vp, vp, vp, vp, i, vp, i, i, i, i, vp]
    fn.restype = ctypes.c_int
    A = 0x7f0000000000
    B, H = 1024, 32  # 32768 heads * 384 floats * 4 bytes = 48 MiB of scratch
    log = b.dl_log(A + (1 << 40), A + (2 << 40), A + (3 << 40), A + (4 << 40), A + (5 << 40), b.DL_BF16, 8,
                   None, 0)
    big = 1 << 36
    rc = fn(A, b.DL_BF16, b.DL_DECAY_HEAD, ctypes.byref(log), 0, A + big, A + 2 * big, A + 3 * big,
            A + 4 * big, A + 5 * big, b.DL_BF16, A + 6 * big, B, H, 128, 256, None)
    assert rc == b.DL_ERR_UNSUPPORTED
    assert "DL_NOALLOC_WORK_BYTES" in lib.dl_last_error().decode()


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_variant_on_two_calls():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.Workload("noalloc", W.CHANNEL, 8, 16, 128, 128, 2, "bf16", "f32", 0.1, (4,), seed=7)
    x = W.generate(w)
    d = W.device_inputs(w, x)
    S = d["S0"].contiguous()
    log_ref = b.Log.allocate(w.B, w.H, w.d_k, w.d_v, 4, torch.bfloat16, True)
    log_na = b.Log.allocate(w.B, w.H, w.d_k, w.d_v, 4, torch.bfloat16, True)
    log_na.work = None  # the no-allocation call takes no workspace
    o_ref = torch.empty(w.B, w.H, w.d_v, device="cuda")
    o_na = torch.empty_like(o_ref)
    for n in range(2):
        args = (d["q"][n], d["k"][n], d["v"][n], d["beta"][n], d["a"][n])
        b.dl_log_append_read(S, log_ref, n, *args, o_ref)
        b.dl_log_append_read_noalloc(S, log_na, n, *args, o_na)
        torch.cuda.synchronize()
        ref = o_ref.double().cpu().numpy()
        got = o_na.double().cpu().numpy()
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err <= 1e-4, (n, err)
        for name in ("k", "v", "beta", "a"):
            assert torch.equal(getattr(log_na, name)[:, :, n], getattr(log_ref, name)[:, :, n]), name
