"""Seeded synthetic inputs for the gated delta-rule decode step.

This module is shared by the CUDA path's tests/benchmark and by the CPU
oracle. It holds the five workload definitions and the seeded generators of
their inputs, and none of the method's arithmetic: it draws random numbers,
applies the input distributions (L2 normalisation of q and k, sigmoid for
beta, exp(-c*softplus) for the decay gate) and rounds to the storage dtype.

Input recipe (per workload, per (b, h) head):
  * every head has its own PCG64 stream seeded by SeedSequence([seed, b, h]),
    so any subset of heads can be generated alone (the oracle checks sampled
    heads of the full-size workloads this way);
  * draw order inside a head, all float32 standard normals:
    S0 [d_v, d_k], q [T, d_k], k [T, d_k], v [T, d_v], beta [T],
    a [T] (head-wise decay, GDN) or [T, d_k] (channel-wise decay, KDA);
  * S0 <- 0.02 * N(0, 1)   (standard deviation 0.02);
  * q, k <- x / ||x||_2 per (t, b, h) over d_k, in float32, no epsilon;
  * v <- N(0, 1);  beta <- sigmoid(N(0, 1));
  * a <- exp(-c * softplus(N(0, 1))), c = 0.1 (mild decay) or 1.0 (strong);
  * then every tensor is rounded (round-to-nearest-even) to its storage
    dtype; both the GPU path and the oracle read the rounded values.

Layouts (row-major, contiguous):
  S0 [B, H, d_v, d_k];  q, k [T, B, H, d_k];  v [T, B, H, d_v];
  beta [T, B, H];  a [T, B, H] (GDN) or [T, B, H, d_k] (KDA).
bf16 tensors are returned as numpy uint16 arrays holding the bf16 bit
patterns (``bf16_to_f32`` widens them exactly).

The shapes and distributions follow the workloads in which the DeltaLog page
("DeltaLog: Deferred Materialization of Recurrent States for Linear Attention
Decoding", Technical Summary, "Problem" and "Kernel Implementation") places
the state-update tax: a [B, H] batch of d_k x d_v states, GDN with head-wise
and KDA with channel-wise decay.
"""
from __future__ import annotations

import dataclasses
import math
import multiprocessing as _mp
import os
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import shared_memory
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

HEAD = "head"        # one scalar decay per head and step (Gated DeltaNet)
CHANNEL = "channel"  # one decay per key channel and step (Kimi Delta Attention)
RWKV6 = "rwkv6"      # one decay per key channel, raw-value update, no beta (RWKV6)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    decay: str           # HEAD, CHANNEL or RWKV6
    B: int
    H: int
    d_k: int
    d_v: int
    T: int
    in_dtype: str        # "f32" or "bf16": q, k, v, beta, a (and the log)
    state_dtype: str     # "f32" or "bf16": S
    decay_scale: float   # c in a = exp(-c * softplus(N(0,1)))
    L: Tuple[int, ...]   # log capacities run on the deferred schedule
    seed: int = 0
    note: str = ""

    @property
    def heads(self) -> int:
        return self.B * self.H

    def state_bytes(self) -> int:
        if self.state_dtype == "i8":  # int8 codes and a float scale per row
            return self.heads * self.d_v * (self.d_k + 4)
        return self.heads * self.d_v * self.d_k * (4 if self.state_dtype == "f32" else 2)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("gdn_b1_h2_d64_t16", HEAD, 1, 2, 64, 64, 16, "f32", "f32", 0.1, (4, 16),
                 note="small GDN case, fp32 everything"),
        Workload("gdn_b64_h16_d128_t1024", HEAD, 64, 16, 128, 128, 1024, "bf16", "f32", 0.1, (8,),
                 note="GDN, bf16 inputs, fp32 state, eager vs deferred L=8"),
        Workload("kda_b256_h32_d128_t512", CHANNEL, 256, 32, 128, 128, 512, "bf16", "f32", 0.1, (16,),
                 note="KDA, bf16 inputs, fp32 state (512 MiB), eager vs deferred L=16"),
        Workload("kda_b128_h16_d128_t2048", CHANNEL, 128, 16, 128, 128, 2048, "bf16", "f32", 0.1,
                 (1, 4, 8, 16, 32, 64), note="KDA log-length sweep"),
        Workload("gdn_b1024_h32_dk128_dv256_t256", HEAD, 1024, 32, 128, 256, 256, "bf16", "bf16", 1.0,
                 (8,), note="large-batch GDN, bf16 state, strong decay, deferred L=8"),
        Workload("rwkv6_b256_h32_d128_t512", RWKV6, 256, 32, 128, 128, 512, "bf16", "f32", 0.1, (16,),
                 note="RWKV6 at the KDA target's shapes: channel decay, raw-value update"),
    ]
}
WORKLOAD_ORDER: List[str] = list(WORKLOADS)


def scaled(w: Workload, **changes) -> Workload:
    """A copy of ``w`` with some sizes changed (smaller test cases of a workload)."""
    return dataclasses.replace(w, **changes)


# ---------------------------------------------------------------- bf16 bits

def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored values (float32 array or bf16 bits) widened exactly to float64."""
    if dtype == "bf16":
        return bf16_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16(x) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _np_dtype(dtype: str):
    return np.uint16 if dtype == "bf16" else np.float32


# ---------------------------------------------------------------- generation

def _head_draws(w: Workload, b: int, h: int):
    """Draw one head's raw inputs in the fixed order, transformed, float32."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, b, h])))
    f32 = np.float32
    S0 = f32(0.02) * rng.standard_normal((w.d_v, w.d_k), dtype=f32)
    q = rng.standard_normal((w.T, w.d_k), dtype=f32)
    k = rng.standard_normal((w.T, w.d_k), dtype=f32)
    v = rng.standard_normal((w.T, w.d_v), dtype=f32)
    beta_raw = rng.standard_normal((w.T,), dtype=f32)
    a_shape = (w.T,) if w.decay == HEAD else (w.T, w.d_k)
    a_raw = rng.standard_normal(a_shape, dtype=f32)
    q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True, dtype=f32))
    k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True, dtype=f32))
    beta = f32(1) / (f32(1) + np.exp(-beta_raw))
    softplus = np.log1p(np.exp(a_raw))
    a = np.exp(-f32(w.decay_scale) * softplus)
    return S0, q.astype(f32), k.astype(f32), v, beta.astype(f32), a.astype(f32)


def _alloc(w: Workload, nh: int, buffers=None) -> Dict[str, np.ndarray]:
    shapes = shapes_for(w, nh)
    out = {}
    for key, (shape, dt) in shapes.items():
        if buffers is not None:
            out[key] = np.ndarray(shape, dtype=dt, buffer=buffers[key].buf)
        else:
            out[key] = np.empty(shape, dtype=dt)
    return out


def shapes_for(w: Workload, nh: int) -> Dict[str, Tuple[tuple, type]]:
    """Storage shapes with the [B, H] head axes flattened to ``nh`` heads."""
    it, st = _np_dtype(w.in_dtype), _np_dtype(w.state_dtype)
    a_shape = (w.T, nh) if w.decay == HEAD else (w.T, nh, w.d_k)
    return {
        "S0": ((nh, w.d_v, w.d_k), st),
        "q": ((w.T, nh, w.d_k), it),
        "k": ((w.T, nh, w.d_k), it),
        "v": ((w.T, nh, w.d_v), it),
        "beta": ((w.T, nh), it),
        "a": (a_shape, it),
    }


def _fill(w: Workload, heads: Sequence[int], out: Dict[str, np.ndarray], offset: int = 0):
    for j, hid in enumerate(heads):
        b, h = divmod(int(hid), w.H)
        S0, q, k, v, beta, a = _head_draws(w, b, h)
        col = offset + j
        out["S0"][col] = _store(S0, w.state_dtype)
        out["q"][:, col] = _store(q, w.in_dtype)
        out["k"][:, col] = _store(k, w.in_dtype)
        out["v"][:, col] = _store(v, w.in_dtype)
        out["beta"][:, col] = _store(beta, w.in_dtype)
        out["a"][:, col] = _store(a, w.in_dtype)


def _worker(args):
    w, heads, offset, nh, names = args
    shms = {key: shared_memory.SharedMemory(name=nm) for key, nm in names.items()}
    try:
        out = _alloc(w, nh, shms)
        _fill(w, heads, out, offset)
        del out
    finally:
        for s in shms.values():
            s.close()
    return len(heads)


def generate(w: Workload, heads: Optional[Sequence[int]] = None, workers: int = 1) -> Dict[str, np.ndarray]:
    """Inputs of workload ``w`` for the given flat head ids (default: all).

    Returns a dict with S0 [nh, d_v, d_k], q/k [T, nh, d_k], v [T, nh, d_v],
    beta [T, nh], a [T, nh] or [T, nh, d_k]; ``nh = len(heads)``; with all heads
    the nh axis is the row-major [B, H] pair. ``workers > 1`` spreads heads over
    spawned processes (start them before any CUDA call in this process).
    """
    if heads is None:
        heads = range(w.heads)
    heads = [int(x) for x in heads]
    nh = len(heads)
    if workers <= 1 or nh < 64:
        out = _alloc(w, nh)
        _fill(w, heads, out)
        return out
    shapes = shapes_for(w, nh)
    shms = {}
    try:
        for key, (shape, dt) in shapes.items():
            nbytes = int(np.prod(shape)) * np.dtype(dt).itemsize
            shms[key] = shared_memory.SharedMemory(create=True, size=max(nbytes, 1))
        names = {key: s.name for key, s in shms.items()}
        chunk = int(math.ceil(nh / (workers * 4)))
        jobs = [(w, heads[i:i + chunk], i, nh, names) for i in range(0, nh, chunk)]
        ctx = _mp.get_context("spawn")
        with ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as ex:
            done = sum(ex.map(_worker, jobs))
        assert done == nh
        view = _alloc(w, nh, shms)
        out = {key: arr.copy() for key, arr in view.items()}
        del view
        return out
    finally:
        for s in shms.values():
            s.close()
            s.unlink()


def default_workers() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 32))


def as_f64(w: Workload, inputs: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """All stored inputs widened exactly to float64 (what the oracle reads)."""
    out = {}
    for key, arr in inputs.items():
        dt = w.state_dtype if key == "S0" else w.in_dtype
        out[key] = to_f64(arr, dt)
    return out


# ---------------------------------------------------------------- device copies

def to_torch(arr: np.ndarray, dtype: str, device="cuda"):
    """A stored array (float32, or bf16 bits as uint16) as a torch tensor."""
    import torch

    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


def device_inputs(w: Workload, x: Dict[str, np.ndarray], device="cuda"):
    """Generated inputs as device tensors with the [B, H] head axes restored
    (a subset of heads becomes B = 1, H = number of heads)."""
    nh = x["S0"].shape[0]
    B, H = (w.B, w.H) if nh == w.heads else (1, nh)
    d = {
        "S0": to_torch(x["S0"], w.state_dtype, device).view(B, H, w.d_v, w.d_k),
        "q": to_torch(x["q"], w.in_dtype, device).view(w.T, B, H, w.d_k),
        "k": to_torch(x["k"], w.in_dtype, device).view(w.T, B, H, w.d_k),
        "v": to_torch(x["v"], w.in_dtype, device).view(w.T, B, H, w.d_v),
        "beta": to_torch(x["beta"], w.in_dtype, device).view(w.T, B, H),
    }
    a_shape = (w.T, B, H) if w.decay == HEAD else (w.T, B, H, w.d_k)
    d["a"] = to_torch(x["a"], w.in_dtype, device).view(*a_shape)
    return d


def device_inputs_chunked(w: Workload, device="cuda", workers: int = 1, chunk_heads: int = 2048):
    """Like ``device_inputs(w, generate(w))`` for all heads, but generated
    ``chunk_heads`` heads at a time and copied straight into the device
    tensors, so the host never holds the whole workload."""
    import torch

    it = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    st = torch.bfloat16 if w.state_dtype == "bf16" else torch.float32
    nh = w.heads
    d = {
        "S0": torch.empty(nh, w.d_v, w.d_k, dtype=st, device=device),
        "q": torch.empty(w.T, nh, w.d_k, dtype=it, device=device),
        "k": torch.empty(w.T, nh, w.d_k, dtype=it, device=device),
        "v": torch.empty(w.T, nh, w.d_v, dtype=it, device=device),
        "beta": torch.empty(w.T, nh, dtype=it, device=device),
        "a": torch.empty(*((w.T, nh) if w.decay == HEAD else (w.T, nh, w.d_k)), dtype=it, device=device),
    }
    for h0 in range(0, nh, chunk_heads):
        heads = list(range(h0, min(nh, h0 + chunk_heads)))
        x = generate(w, heads=heads, workers=workers)
        for key, arr in x.items():
            dt = w.state_dtype if key == "S0" else w.in_dtype
            t = to_torch(arr, dt, device)
            if key == "S0":
                d[key][h0:h0 + len(heads)] = t
            else:
                d[key][:, h0:h0 + len(heads)] = t
        del x
    B, H = w.B, w.H
    d["S0"] = d["S0"].view(B, H, w.d_v, w.d_k)
    d["q"] = d["q"].view(w.T, B, H, w.d_k)
    d["k"] = d["k"].view(w.T, B, H, w.d_k)
    d["v"] = d["v"].view(w.T, B, H, w.d_v)
    d["beta"] = d["beta"].view(w.T, B, H)
    d["a"] = d["a"].view(*((w.T, B, H) if w.decay == HEAD else (w.T, B, H, w.d_k)))
    return d
