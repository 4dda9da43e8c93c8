"""GPU parity of the tensor-core merge (merge_tc.cu) through its pipeline.

The tcgen05 kernel takes every merge of an fp32 base with d_k = 128, d_v a
multiple of 128 and at most 16 entries. It runs one CTA per SM over units
(head, 128-row tile), two pipeline stages deep, so a case needs several units
per CTA (here 4 to 7) to reuse both stages and carry tensor memory and the
operand tiles from one unit to the next. Each case runs the deferred schedule
(fused or unfused merges) over T steps against the fp64 oracle's eager
recurrence, at the parity bar of 1e-4 (max|delta| / max|ref|, outputs over
all steps and the final state), and then checks that no bounded wait of the
kernel ran out (the library's fault word is 0).
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_util import device_inputs, rel_err, run_cuda, state_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_104_b200 as g

    g.load()
    g.dl_device_faults(clear=True)


def _case(decay, in_dtype, d_v, B, H, T, seed):
    return W.Workload(f"tc_{decay}_{in_dtype}_dv{d_v}", decay, B, H, 128, d_v, T, in_dtype, "f32", 0.1, (16,),
                      seed=seed)


CASES = [
    # (decay, input dtype, d_v, B, H, T, L, fused)
    (W.CHANNEL, "bf16", 128, 24, 32, 34, 16, True),
    (W.CHANNEL, "bf16", 128, 24, 32, 34, 16, False),
    (W.HEAD, "bf16", 128, 24, 32, 21, 8, True),
    (W.HEAD, "f32", 256, 12, 32, 21, 8, False),
    (W.CHANNEL, "f32", 256, 12, 32, 19, 4, True),
    (W.RWKV6, "bf16", 128, 24, 32, 34, 16, True),
    (W.RWKV6, "f32", 256, 12, 32, 17, 5, False),
    (W.CHANNEL, "bf16", 128, 24, 32, 9, 1, True),
]


@pytest.mark.parametrize("decay,in_dtype,d_v,B,H,T,L,fused", CASES)
def test_tensor_core_merge_pipeline(decay, in_dtype, d_v, B, H, T, L, fused):
    import gated_delta_rule_104_b200 as g

    w = _case(decay, in_dtype, d_v, B, H, T, seed=B * 131 + T)
    x = W.generate(w)
    o_ref, S_ref = oracle.run_workload_heads(w, x, "eager")
    d = device_inputs(w, x)
    o, S = run_cuda(w, d, "deferred", L, fused)
    S = state_to_f64(S).reshape(S_ref.shape)
    eo, es = rel_err(o, o_ref), rel_err(S, S_ref)
    assert eo <= 1e-4 and es <= 1e-4, f"{w.name} L={L} fused={fused}: o {eo:.3e} S {es:.3e}"
    assert np.isfinite(o).all()
    assert g.dl_device_faults() == 0
