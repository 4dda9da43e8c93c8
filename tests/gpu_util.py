"""Helpers shared by the GPU tests: move seeded inputs to the device, run the
CUDA path (through the C ABI) over all T steps, compare with the oracle."""
from __future__ import annotations

import numpy as np

import workloads as W


to_torch = W.to_torch
device_inputs = W.device_inputs


def state_to_f64(S) -> np.ndarray:
    import torch

    return S.detach().to(torch.float64).cpu().numpy()


def run_cuda(w: W.Workload, d, path: str, L: int = 0, fused: bool = True, keep_o: bool = True,
             o_heads=None):
    """Run all T steps through the library. Returns (o, S): o [T, nh, d_v]
    float32 numpy (only ``o_heads`` columns if given), S the final state."""
    import torch

    import gated_delta_rule_104_b200 as g

    S = d["S0"].clone()
    B, H = S.shape[0], S.shape[1]
    T = w.T
    chan = w.decay != W.HEAD
    rw = w.decay == W.RWKV6
    o_step = torch.empty(B, H, w.d_v, dtype=torch.float32, device=S.device)
    keep = []
    if path == "eager":
        fn = g.dl_kda_decode_step if chan else g.dl_gdn_decode_step
        for t in range(T):
            if rw:
                g.dl_rwkv6_decode_step(S, d["q"][t], d["k"][t], d["v"][t], d["a"][t], o_step)
            else:
                fn(S, d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["a"][t], o_step)
            if keep_o:
                keep.append(_pick(o_step, o_heads))
    else:
        tdt = d["q"].dtype
        log = g.Log.allocate(B, H, w.d_k, w.d_v, L, tdt, chan, device=S.device, rwkv6=rw)
        dec = g.DeferredDecoder(S, log, fused_merge=fused)
        for t in range(T):
            beta_t = None if rw else d["beta"][t]
            dec.step(d["q"][t], d["k"][t], d["v"][t], beta_t, d["a"][t], o_step)
            if keep_o:
                keep.append(_pick(o_step, o_heads))
        dec.flush()
    torch.cuda.synchronize()
    o = torch.stack(keep).cpu().numpy() if keep_o else None
    return o, S


def _pick(o_step, heads):
    flat = o_step.view(-1, o_step.shape[-1])
    if heads is None:
        return flat.clone()
    return flat[heads].clone()


def rel_err(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.abs(np.asarray(x, np.float64) - ref).max() / max(np.abs(ref).max(), 1e-300))


def tolerance(w: W.Workload) -> float:
    """max|delta| / max|ref| bound: 1e-4 for an fp32 state, 2e-2 for bf16."""
    return 2e-2 if w.state_dtype == "bf16" else 1e-4
