"""fp64 CPU oracle of the gated delta-rule decode step (eager and DeltaLog).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by ``bench.py``'s CPU-baseline leg (and its ``--impl reference`` arm),
nowhere else. It shares no code with the CUDA library in
``gated_delta_rule_104_b200`` and neither imports the other.

Forms (all fp64, following "DeltaLog: Deferred Materialization of Recurrent
States for Linear Attention Decoding", Technical Summary):
  * ``eager``       -- the recurrence step by step (C, deltalog_oracle.c);
  * ``deferred``    -- base + bounded log with merges every L steps (C);
  * ``brute_force`` -- dense d_k x d_k factor matrices multiplied with numpy,
                       for tiny shapes only;
  * ``pool_eager``  -- a pool of per-sequence states, each listed slot
                       advanced one eager step (the slot-pool entry points).

Definition used (the pages describe the update only in words -- decay, then a
delta-rule correction that subtracts the current read before writing, with a
head-wise scalar decay for Gated DeltaNet and a per-key decay for Kimi Delta
Attention, "Kernel Implementation"): per head, S is d_v x d_k and

    S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t.

RWKV6 (``rwkv6=True``), the page's third model ("per-key decay; raw-value
updates, no delta-rule correction", "Kernel Implementation"), is read as
S_t = S_{t-1} Diag(a_t) + v_t k_t^T, o_t = S_t q_t: no beta, and no "bonus"
term (the pages do not define one).

Every function's parity with the pages is pinned by tests/test_oracle_pins.py
(invariants, closed forms, hand-worked exact examples, brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "deltalog_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libdeltalog_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, strict IEEE fp64)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c99", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class CLib:
    """ctypes handle on one build of the C oracle (``path``)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        for name, extra in (("oracle_eager", []), ("oracle_deferred", [ctypes.c_int]),
                            ("oracle_deferred_i8", [ctypes.c_int])):
            fn = getattr(lib, name)
            fn.restype = None
            fn.argtypes = ([ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
                           + extra + [dp] * 7)
        lib.oracle_quantize_i8.restype = None
        lib.oracle_quantize_i8.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int, dp]
        lib.oracle_abi_version.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def eager(self, S0, q, k, v, beta, a, channel_decay: bool, rwkv6: bool = False):
        """Eager recurrence over T steps. Shapes: S0 [NH,d_v,d_k]; q,k [T,NH,d_k];
        v [T,NH,d_v]; beta [T,NH] (unused, may be None, for RWKV6); a [T,NH] or
        [T,NH,d_k]. Returns (o [T,NH,d_v], S_T)."""
        S, q, k, v, beta, a, NH, T, dk, dv = _prep(S0, q, k, v, beta, a, channel_decay or rwkv6)
        o = np.zeros((T, NH, dv), dtype=np.float64)
        self.lib.oracle_eager(NH, T, dk, dv, _kind(channel_decay, rwkv6),
                              _c(S), _c(q), _c(k), _c(v), _c(beta), _c(a), _c(o))
        return o, S

    def deferred(self, S0, q, k, v, beta, a, channel_decay: bool, L: int, rwkv6: bool = False,
                 base_i8: bool = False):
        """DeltaLog schedule with log capacity L (merge when full and at the end).
        ``base_i8``: the base is held in int8 with a scale per row, quantised at
        the start and after every merge. Returns (o [T,NH,d_v], S_T)."""
        if L < 1:
            raise ValueError("log capacity L must be >= 1")
        S, q, k, v, beta, a, NH, T, dk, dv = _prep(S0, q, k, v, beta, a, channel_decay or rwkv6)
        o = np.zeros((T, NH, dv), dtype=np.float64)
        fn = self.lib.oracle_deferred_i8 if base_i8 else self.lib.oracle_deferred
        fn(NH, T, dk, dv, _kind(channel_decay, rwkv6), int(L),
           _c(S), _c(q), _c(k), _c(v), _c(beta), _c(a), _c(o))
        return o, S

    def quantize_i8(self, S):
        """The int8 base's rounding of states [NH, d_v, d_k] (a copy)."""
        S = np.array(S, dtype=np.float64, order="C", copy=True)
        NH, dv, dk = S.shape
        self.lib.oracle_quantize_i8(NH, dk, dv, _c(S))
        return S


def _kind(channel_decay: bool, rwkv6: bool) -> int:
    """The C oracle's rule code: 0 head-wise decay, 1 channel-wise, 2 RWKV6."""
    return 2 if rwkv6 else int(bool(channel_decay))


def _load() -> CLib:
    global _lib
    with _lock:
        if _lib is None:
            _lib = CLib(build())
    return _lib


def _c(arr: np.ndarray):
    return arr.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(S0, q, k, v, beta, a, channel_decay):
    S = np.array(S0, dtype=np.float64, order="C", copy=True)
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    if beta is None:  # RWKV6 has no beta; the C side does not read it
        beta = np.zeros(q.shape[:2], dtype=np.float64)
    beta = np.ascontiguousarray(beta, dtype=np.float64)
    a = np.ascontiguousarray(a, dtype=np.float64)
    NH, dv, dk = S.shape
    T = q.shape[0]
    assert q.shape == (T, NH, dk) and k.shape == (T, NH, dk), (q.shape, k.shape)
    assert v.shape == (T, NH, dv) and beta.shape == (T, NH)
    assert a.shape == ((T, NH, dk) if channel_decay else (T, NH)), a.shape
    return S, q, k, v, beta, a, NH, T, dk, dv


def eager(S0, q, k, v, beta, a, channel_decay: bool, rwkv6: bool = False):
    """Eager recurrence (see ``CLib.eager``) with the default build."""
    return _load().eager(S0, q, k, v, beta, a, channel_decay, rwkv6)


def deferred(S0, q, k, v, beta, a, channel_decay: bool, L: int, rwkv6: bool = False, base_i8: bool = False):
    """DeltaLog schedule (see ``CLib.deferred``) with the default build."""
    return _load().deferred(S0, q, k, v, beta, a, channel_decay, L, rwkv6, base_i8)


def quantize_i8(S):
    """The int8 base's per-row rounding (see ``CLib.quantize_i8``)."""
    return _load().quantize_i8(S)


def brute_force(S0, q, k, v, beta, a, channel_decay: bool, rwkv6: bool = False):
    """Tiny shapes only: build A_t = Diag(a_t)(I - beta_t k_t k_t^T) as dense
    matrices and apply S_t = S_{t-1} A_t + beta_t v_t k_t^T, o_t = S_t q_t with
    numpy matrix products (RWKV6: A_t = Diag(a_t), S_t = S_{t-1} A_t + v_t k_t^T).
    Returns (o [T,NH,d_v], S_T)."""
    S = np.array(S0, dtype=np.float64, copy=True)
    NH, dv, dk = S.shape
    T = q.shape[0]
    assert dk <= 16 and dv <= 16, "brute force is for tiny shapes"
    o = np.zeros((T, NH, dv))
    eye = np.eye(dk)
    for h in range(NH):
        for t in range(T):
            kt = np.asarray(k[t, h], dtype=np.float64).reshape(dk, 1)
            vt = np.asarray(v[t, h], dtype=np.float64).reshape(dv, 1)
            at = np.asarray(a[t, h], dtype=np.float64)
            Da = np.diag(at if (channel_decay or rwkv6) else np.full(dk, float(at)))
            if rwkv6:
                S[h] = S[h] @ Da + vt @ kt.T
            else:
                A = Da @ (eye - float(beta[t, h]) * (kt @ kt.T))
                S[h] = S[h] @ A + float(beta[t, h]) * (vt @ kt.T)
            o[t, h] = S[h] @ np.asarray(q[t, h], dtype=np.float64)
    return o, S


def pool_eager(S_pool0, steps, channel_decay: bool, rwkv6: bool = False, resets=None):
    """A pool of per-sequence states advanced by the recurrence, for the slot
    pool entry points: ``S_pool0`` [P, H, d_v, d_k]; ``steps`` a list of
    (slot [B], q [B,H,d_k], k, v [B,H,d_v], beta [B,H], a [B,H] or [B,H,d_k]) in
    which every listed slot takes one eager step with its row's inputs;
    ``resets`` maps a step index to {slot: new state [H, d_v, d_k]} applied
    before that step (a new sequence taking the slot). Returns (list of o
    [B,H,d_v] per step, final S_pool)."""
    S = np.array(S_pool0, dtype=np.float64, copy=True)
    P, H, dv, dk = S.shape
    flat = S.reshape(P * H, dv, dk)
    outs = []
    for t, (slot, q, k, v, beta, a) in enumerate(steps):
        for s_, S0 in (resets or {}).get(t, {}).items():
            flat[s_ * H:(s_ + 1) * H] = np.asarray(S0, dtype=np.float64)
        slot = np.asarray(slot, dtype=np.int64)
        B = slot.size
        heads = (slot[:, None] * H + np.arange(H)[None, :]).reshape(-1)
        chan = channel_decay or rwkv6
        a_ = np.asarray(a, np.float64).reshape((1, B * H, dk) if chan else (1, B * H))
        beta_ = None if beta is None else np.asarray(beta, np.float64).reshape(1, B * H)
        o, Snew = eager(flat[heads], np.asarray(q, np.float64).reshape(1, B * H, dk),
                        np.asarray(k, np.float64).reshape(1, B * H, dk), np.asarray(v, np.float64).reshape(1, B * H, dv),
                        beta_, a_, channel_decay, rwkv6)
        flat[heads] = Snew
        outs.append(o[0].reshape(B, H, dv))
    return outs, flat.reshape(P, H, dv, dk)


def brute_force_window(Sbar, ks, vs, betas, As_diag):
    """The closed form the deferred schedule rests on, for tiny shapes:
    S_n = Sbar A_1...A_n + sum_i beta_i v_i k_i^T A_{i+1}...A_n, each A_i a
    dense matrix. ``As_diag[i]`` is the decay vector of entry i."""
    dk = Sbar.shape[1]
    n = len(ks)
    mats = []
    for i in range(n):
        ki = np.asarray(ks[i], dtype=np.float64).reshape(dk, 1)
        mats.append(np.diag(np.asarray(As_diag[i], dtype=np.float64)) @ (np.eye(dk) - betas[i] * (ki @ ki.T)))

    def prod(lo, hi):  # A_lo ... A_hi (1-based, inclusive); identity if empty
        P = np.eye(dk)
        for i in range(lo, hi + 1):
            P = P @ mats[i - 1]
        return P

    S = Sbar @ prod(1, n)
    for i in range(1, n + 1):
        ki = np.asarray(ks[i - 1], dtype=np.float64).reshape(1, dk)
        vi = np.asarray(vs[i - 1], dtype=np.float64).reshape(-1, 1)
        S = S + betas[i - 1] * (vi @ ki) @ prod(i + 1, n)
    return S


def run_workload_heads(w, inputs: Dict[str, np.ndarray], path: str = "eager", L: Optional[int] = None):
    """Run the oracle on generated inputs (``workloads.generate`` output for
    some heads). ``path`` is "eager" or "deferred" (then ``L`` is required)."""
    import workloads  # the shared seeded-input module, no method arithmetic

    f = workloads.as_f64(w, inputs)
    chan = w.decay != workloads.HEAD
    rw = w.decay == workloads.RWKV6
    if path == "eager":
        return eager(f["S0"], f["q"], f["k"], f["v"], f["beta"], f["a"], chan, rw)
    return deferred(f["S0"], f["q"], f["k"], f["v"], f["beta"], f["a"], chan, int(L), rw)


def omp_threads() -> int:
    """Threads the OpenMP runtime will use (OMP_NUM_THREADS, else the CPUs
    this process may run on)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        try:
            return int(env.split(",")[0])
        except ValueError:
            pass
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1
