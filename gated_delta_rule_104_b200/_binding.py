"""ctypes binding of libdeltalog.so (include/deltalog.h).

Argument marshalling only: every function here checks that the tensors are
CUDA, contiguous and of a supported dtype, reads their shapes, and passes raw
device pointers, sizes and the stream to the C ABI. All arithmetic runs in the
library's CUDA kernels. There is no fallback: a missing library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
# the library a process loads: libdeltalog.so, or the file DELTALOG_LIBRARY
# names (e.g. the index-guard debug build, libdeltalog_guard.so)
LIB_PATH = os.environ.get("DELTALOG_LIBRARY") or os.path.join(HERE, "libdeltalog.so")
GUARD_LIB_PATH = os.path.join(HERE, "libdeltalog_guard.so")

DL_OK, DL_ERR_INVALID_ARG, DL_ERR_UNSUPPORTED, DL_ERR_LOG_FULL, DL_ERR_CUDA = range(5)
DL_F32, DL_BF16, DL_I8 = 0, 1, 2
DL_DECAY_HEAD, DL_DECAY_CHANNEL, DL_RWKV6 = 0, 1, 2
DL_MAX_LOG = 64
ABI_VERSION = 9

EXPORTS = ("dl_gdn_decode_step", "dl_kda_decode_step", "dl_rwkv6_decode_step", "dl_log_append_read", "dl_log_merge",
           "dl_log_merge_read", "dl_log_work_bytes", "dl_log_append_read_noalloc", "dl_pool_step",
           "dl_pool_flush", "dl_state_bytes", "dl_state_to_i8", "dl_state_from_i8", "dl_status_string",
           "dl_last_error", "dl_abi_version", "dl_device_faults", "dl_index_guard_build")
DL_NOALLOC_WORK_BYTES = 16 << 20


class DeltaLogError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn}: status {status} ({_status_name(status)}): {message}")
        self.status = status


class dl_log(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("a", ctypes.c_void_p), ("x", ctypes.c_void_p), ("dtype", ctypes.c_int), ("L", ctypes.c_int),
                ("work", ctypes.c_void_p), ("work_bytes", ctypes.c_size_t)]


class dl_pool(ctypes.Structure):
    _fields_ = [("S", ctypes.c_void_p), ("s_dtype", ctypes.c_int), ("P", ctypes.c_int), ("n", ctypes.c_void_p),
                ("status", ctypes.c_void_p), ("log", dl_log)]


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libdeltalog.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libdeltalog.so not found at {p}: build it with "
                           "`python -m gated_delta_rule_104_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(p)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
    step = [vp, i, vp, vp, vp, vp, vp, i, f, i, i, i, i, vp]
    lib.dl_gdn_decode_step.argtypes = step
    lib.dl_kda_decode_step.argtypes = step
    lib.dl_rwkv6_decode_step.argtypes = [vp, i, vp, vp, vp, vp, i, f, i, i, i, i, vp]
    lp = ctypes.POINTER(dl_log)
    lib.dl_log_append_read.argtypes = [vp, i, i, lp, i, vp, vp, vp, vp, vp, i, f, i, i, i, i, vp]
    lib.dl_log_merge_read.argtypes = [vp, i, i, lp, i, vp, vp, vp, vp, vp, i, f, i, i, i, i, vp]
    lib.dl_log_append_read_noalloc.argtypes = [vp, i, i, lp, i, vp, vp, vp, vp, vp, i, f, i, i, i, i, vp]
    pp = ctypes.POINTER(dl_pool)
    lib.dl_pool_step.argtypes = [pp, i, vp, vp, vp, vp, vp, vp, i, f, i, i, i, i, vp]
    lib.dl_pool_flush.argtypes = [pp, i, vp, i, i, i, i, vp]
    lib.dl_state_bytes.argtypes = [i, i, i, i, i]
    lib.dl_state_bytes.restype = ctypes.c_size_t
    lib.dl_state_to_i8.argtypes = [vp, i, vp, i, i, i, i, vp]
    lib.dl_state_from_i8.argtypes = [vp, vp, i, i, i, i, i, vp]
    lib.dl_log_merge.argtypes = [vp, i, i, lp, i, i, i, i, i, vp]
    for name in ("dl_gdn_decode_step", "dl_kda_decode_step", "dl_rwkv6_decode_step", "dl_log_append_read",
                 "dl_log_merge", "dl_log_merge_read", "dl_log_append_read_noalloc", "dl_pool_step",
                 "dl_pool_flush", "dl_state_to_i8", "dl_state_from_i8"):
        getattr(lib, name).restype = ctypes.c_int
    lib.dl_status_string.argtypes = [ctypes.c_int]
    lib.dl_status_string.restype = ctypes.c_char_p
    lib.dl_last_error.argtypes = []
    lib.dl_last_error.restype = ctypes.c_char_p
    lib.dl_log_work_bytes.argtypes = [i, i, i, i]
    lib.dl_log_work_bytes.restype = ctypes.c_size_t
    lib.dl_abi_version.argtypes = []
    lib.dl_abi_version.restype = ctypes.c_int
    lib.dl_device_faults.argtypes = [ctypes.POINTER(ctypes.c_uint), ctypes.c_int]
    lib.dl_device_faults.restype = ctypes.c_int
    lib.dl_index_guard_build.argtypes = []
    lib.dl_index_guard_build.restype = ctypes.c_int
    if lib.dl_abi_version() != ABI_VERSION:
        raise RuntimeError(f"libdeltalog.so ABI {lib.dl_abi_version()} != binding ABI {ABI_VERSION}: rebuild")
    if path is None:
        _lib = lib
    return lib


def _status_name(s: int) -> str:
    return {0: "DL_OK", 1: "DL_ERR_INVALID_ARG", 2: "DL_ERR_UNSUPPORTED", 3: "DL_ERR_LOG_FULL",
            4: "DL_ERR_CUDA"}.get(s, "?")


def check(fn: str, status: int) -> None:
    if status != DL_OK:
        msg = load().dl_last_error().decode(errors="replace")
        raise DeltaLogError(fn, status, msg)


# ------------------------------------------------------------------ tensors

def _torch():
    import torch  # device memory and streams only

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return DL_F32
    if t.dtype == torch.bfloat16:
        return DL_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t, name: str, optional: bool = False) -> Optional[int]:
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class I8State:
    """A deferred base in the int8 layout (DL_I8): one device buffer of
    B*H*d_v*d_k int8 codes followed by B*H*d_v float32 row scales; an element's
    value is code * scale. ``codes`` and ``scales`` are views of the buffer."""

    def __init__(self, buf, B: int, H: int, d_k: int, d_v: int):
        self.buf, self.B, self.H, self.d_k, self.d_v = buf, int(B), int(H), int(d_k), int(d_v)
        self.shape = (self.B, self.H, self.d_v, self.d_k)

    @classmethod
    def allocate(cls, B, H, d_k, d_v, device="cuda"):
        torch = _torch()
        n = B * H * d_v * d_k
        return cls(torch.zeros(n + 4 * B * H * d_v, dtype=torch.uint8, device=device), B, H, d_k, d_v)

    @property
    def codes(self):
        torch = _torch()
        n = self.B * self.H * self.d_v * self.d_k
        return self.buf[:n].view(torch.int8).view(self.shape)

    @property
    def scales(self):
        torch = _torch()
        n = self.B * self.H * self.d_v * self.d_k
        return self.buf[n:].view(torch.float32).view(self.B, self.H, self.d_v)

    def data_ptr(self) -> int:
        return self.buf.data_ptr()


def dl_state_to_i8(S, out: "I8State", stream=None) -> None:
    """Round a float32 / bfloat16 state [B,H,d_v,d_k] into ``out``."""
    B, H, dk, dv = _dims(S)
    check("dl_state_to_i8", load().dl_state_to_i8(_ptr(S, "S"), _dtype_code(S), out.data_ptr(), B, H, dk, dv,
                                                  _stream(stream)))


def dl_state_from_i8(S8: "I8State", out, stream=None) -> None:
    """The values of an int8 state into ``out`` (float32 or bfloat16 [B,H,d_v,d_k])."""
    check("dl_state_from_i8", load().dl_state_from_i8(S8.data_ptr(), _ptr(out, "S"), _dtype_code(out), S8.B, S8.H,
                                                      S8.d_k, S8.d_v, _stream(stream)))


def _dims(S):
    if isinstance(S, I8State):
        return S.B, S.H, S.d_k, S.d_v
    if S.dim() != 4:
        raise ValueError("state must be [B, H, d_v, d_k]")
    B, H, dv, dk = S.shape
    return int(B), int(H), int(dk), int(dv)


def _state_code(S) -> int:
    return DL_I8 if isinstance(S, I8State) else _dtype_code(S)


def _state_ptr(S, name: str) -> int:
    if isinstance(S, I8State):
        return _ptr(S.buf, name)
    return _ptr(S, name)


def _in_dtype(*ts) -> int:
    codes = {_dtype_code(t) for t in ts if t is not None}
    if len(codes) != 1:
        raise TypeError("q, k, v, beta and a must share one dtype")
    return codes.pop()


def _check_shapes(B, H, dk, dv, q, k, v, beta, a, o, chan):
    exp = {"q": (q, B * H * dk), "k": (k, B * H * dk), "v": (v, B * H * dv), "beta": (beta, B * H),
           "a": (a, B * H * (dk if chan else 1)), "o": (o, B * H * dv)}
    for name, (t, n) in exp.items():
        if t is None and name == "beta":
            continue
        if t.numel() != n:
            raise ValueError(f"{name} has {t.numel()} elements, expected {n}")
    if o.dtype != _torch().float32:
        raise TypeError("o must be float32")


def dl_gdn_decode_step(S, q, k, v, beta, a, o, stream=None) -> None:
    """Eager GDN step in place on S [B,H,d_v,d_k]; o [B,H,d_v] float32."""
    _eager("dl_gdn_decode_step", S, q, k, v, beta, a, o, stream, chan=False)


def dl_kda_decode_step(S, q, k, v, beta, a, o, stream=None) -> None:
    """Eager KDA step (a [B,H,d_k]) in place on S; o [B,H,d_v] float32."""
    _eager("dl_kda_decode_step", S, q, k, v, beta, a, o, stream, chan=True)


def dl_rwkv6_decode_step(S, q, k, v, a, o, stream=None) -> None:
    """Eager RWKV6 step (a [B,H,d_k]; raw-value update, no beta) in place on S."""
    B, H, dk, dv = _dims(S)
    _check_shapes(B, H, dk, dv, q, k, v, None, a, o, True)
    st = _stream(stream)
    status = load().dl_rwkv6_decode_step(_ptr(S, "S"), _dtype_code(S), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                         _ptr(a, "a"), _in_dtype(q, k, v, a), _ptr(o, "o"), B, H, dk, dv, st)
    check("dl_rwkv6_decode_step", status)


def _eager(fn, S, q, k, v, beta, a, o, stream, chan):
    if isinstance(S, I8State):
        raise TypeError("the eager step takes a float32 or bfloat16 state")
    B, H, dk, dv = _dims(S)
    _check_shapes(B, H, dk, dv, q, k, v, beta, a, o, chan)
    st = _stream(stream)
    status = getattr(load(), fn)(_ptr(S, "S"), _dtype_code(S), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                 _ptr(beta, "beta"), _ptr(a, "a"), _in_dtype(q, k, v, beta, a),
                                 _ptr(o, "o"), B, H, dk, dv, st)
    check(fn, status)


class Log:
    """Caller-owned bounded log buffers of a deferred state (device tensors):
    k [B,H,L,d_k], v [B,H,L,d_v], beta [B,H,L], a [B,H,L] or [B,H,L,d_k],
    x [B,H,L,L] float32 (the log's triangular solve matrix), work (fp32 workspace).
    An RWKV6 log (``rwkv6=True``: channel decay, no delta correction) has no
    beta and no x (None)."""

    def __init__(self, k, v, beta, a, x, L: int, channel_decay: bool, work=None, rwkv6: bool = False):
        self.k, self.v, self.beta, self.a, self.x = k, v, beta, a, x
        self.L = int(L)
        self.rwkv6 = bool(rwkv6)
        self.channel_decay = bool(channel_decay) or self.rwkv6
        self.dtype = _in_dtype(k, v, beta, a)
        self.work = work

    @classmethod
    def allocate(cls, B, H, d_k, d_v, L, dtype, channel_decay, device="cuda", rwkv6: bool = False):
        torch = _torch()
        z = lambda *s: torch.zeros(*s, dtype=dtype, device=device)  # noqa: E731
        chan = channel_decay or rwkv6
        a = z(B, H, L, d_k) if chan else z(B, H, L)
        work = torch.empty(B * H * (d_k + d_v), dtype=torch.float32, device=device)
        x = None if rwkv6 else torch.zeros(B, H, L, L, dtype=torch.float32, device=device)
        beta = None if rwkv6 else z(B, H, L)
        return cls(z(B, H, L, d_k), z(B, H, L, d_v), beta, a, x, L, chan, work, rwkv6)

    def struct(self) -> dl_log:
        wp = _ptr(self.work, "log.work") if self.work is not None else None
        wb = self.work.numel() * self.work.element_size() if self.work is not None else 0
        return dl_log(_ptr(self.k, "log.k"), _ptr(self.v, "log.v"), _ptr(self.beta, "log.beta", self.rwkv6),
                      _ptr(self.a, "log.a"), _ptr(self.x, "log.x", self.rwkv6), self.dtype, self.L, wp, wb)

    @property
    def kind(self) -> int:
        if self.rwkv6:
            return DL_RWKV6
        return DL_DECAY_CHANNEL if self.channel_decay else DL_DECAY_HEAD


def dl_log_append_read(S_base, log: Log, n: int, q, k, v, beta, a, o, stream=None) -> None:
    """Append entry n and read o from base + log (base not written)."""
    _log_step("dl_log_append_read", S_base, log, n, q, k, v, beta, a, o, stream)


def dl_log_merge_read(S_base, log: Log, n: int, q, k, v, beta, a, o, stream=None) -> None:
    """Merge log entries 0..n-1 plus this step into the base; o = new base q."""
    _log_step("dl_log_merge_read", S_base, log, n, q, k, v, beta, a, o, stream)


def _log_step(fn, S, log, n, q, k, v, beta, a, o, stream):
    B, H, dk, dv = _dims(S)
    _check_shapes(B, H, dk, dv, q, k, v, beta, a, o, log.channel_decay)
    st = _stream(stream)
    ls = log.struct()
    status = getattr(load(), fn)(_state_ptr(S, "S_base"), _state_code(S), log.kind, ctypes.byref(ls), int(n),
                                 _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(beta, "beta", log.rwkv6),
                                 _ptr(a, "a"),
                                 _in_dtype(q, k, v, beta, a), _ptr(o, "o"), B, H, dk, dv, st)
    check(fn, status)


def dl_log_merge(S_base, log: Log, n: int, stream=None) -> None:
    """Merge log entries 0..n-1 into the base in place."""
    B, H, dk, dv = _dims(S_base)
    st = _stream(stream)
    ls = log.struct()
    status = load().dl_log_merge(_state_ptr(S_base, "S_base"), _state_code(S_base), log.kind, ctypes.byref(ls),
                                 int(n), B, H, dk, dv, st)
    check("dl_log_merge", status)


def dl_device_faults(clear: bool = False) -> int:
    """The kernels' fault word on the current device (0: no bounded wait ran
    out and, in the index-guard build, no shared-memory write was out of
    bounds). Synchronises the device."""
    w = ctypes.c_uint(0)
    check("dl_device_faults", load().dl_device_faults(ctypes.byref(w), 1 if clear else 0))
    return int(w.value)


def dl_index_guard_build() -> bool:
    """Whether the loaded library is the index-guard debug build."""
    return bool(load().dl_index_guard_build())


def dl_status_string(status: int) -> str:
    return load().dl_status_string(int(status)).decode()


def dl_log_append_read_noalloc(S_base, log: Log, n: int, q, k, v, beta, a, o, stream=None) -> None:
    """As dl_log_append_read, with the scratch in the library's fixed device
    array instead of ``log.work``: for callers that cannot allocate device
    memory. Calls that overlap on the GPU race on that array."""
    _log_step("dl_log_append_read_noalloc", S_base, log, n, q, k, v, beta, a, o, stream)


# ------------------------------------------------------------------ slot pool

class Pool:
    """A pool of P per-sequence deferred states (device tensors): S [P,H,d_v,d_k],
    ``log`` a Log over the P slots (its workspace covers a batch of up to P
    rows), n [P] int32 log counts, status [1] int32 error word. A new sequence
    taking slot s needs S[s] = its initial state and n[s] = 0 (``reset``)."""

    def __init__(self, S, log: Log, n, status=None):
        self.S, self.log, self.n, self.status = S, log, n, status
        self.P = int(S.shape[0])  # (S may be an I8State: an int8 pool)

    @classmethod
    def allocate(cls, P, H, d_k, d_v, L, s_dtype, in_dtype, channel_decay, rwkv6: bool = False, device="cuda"):
        """``s_dtype``: torch.float32, torch.bfloat16, or torch.int8 for an int8 pool (DL_I8)."""
        torch = _torch()
        if s_dtype == torch.int8:
            S = I8State.allocate(P, H, d_k, d_v, device=device)
        else:
            S = torch.zeros(P, H, d_v, d_k, dtype=s_dtype, device=device)
        log = Log.allocate(P, H, d_k, d_v, L, in_dtype, channel_decay, device=device, rwkv6=rwkv6)
        n = torch.zeros(P, dtype=torch.int32, device=device)
        status = torch.zeros(1, dtype=torch.int32, device=device)
        return cls(S, log, n, status)

    def reset(self, slot: int, S0) -> None:
        """Start a new sequence in ``slot`` from state S0 [H, d_v, d_k] (stream-ordered copies;
        an int8 pool takes S0 rounded to its layout)."""
        if isinstance(self.S, I8State):
            tmp = I8State.allocate(1, self.S.H, self.S.d_k, self.S.d_v, device=self.S.buf.device)
            dl_state_to_i8(S0.reshape(1, *S0.shape).contiguous(), tmp)
            self.S.codes[slot].copy_(tmp.codes[0])
            self.S.scales[slot].copy_(tmp.scales[0])
        else:
            self.S[slot].copy_(S0)
        self.n[slot] = 0

    def struct(self) -> dl_pool:
        if self.n.dtype != _torch().int32:
            raise TypeError("pool.n must be int32")
        return dl_pool(_state_ptr(self.S, "pool.S"), _state_code(self.S), self.P, _ptr(self.n, "pool.n"),
                       _ptr(self.status, "pool.status", True), self.log.struct())


def _slots(slot, B: int) -> int:
    torch = _torch()
    if slot.dtype != torch.int32 or slot.numel() != B:
        raise ValueError(f"slot must be int32 with {B} entries")
    return _ptr(slot, "slot")


def dl_pool_step(pool: Pool, slot, q, k, v, beta, a, o, stream=None) -> None:
    """One decode step of the batch rows ``slot`` [B] int32 of the pool
    (inputs and o are [B,H,...]); each row appends or, on its L-th entry,
    merges, following its own log count."""
    B, H, dk = int(q.shape[0]), int(q.shape[1]), int(q.shape[2])
    dv = int(pool.S.shape[2])  # (an I8State has .shape too)
    _check_shapes(B, H, dk, dv, q, k, v, beta, a, o, pool.log.channel_decay)
    ps = pool.struct()
    status = load().dl_pool_step(ctypes.byref(ps), pool.log.kind, _slots(slot, B), _ptr(q, "q"), _ptr(k, "k"),
                                 _ptr(v, "v"), _ptr(beta, "beta", pool.log.rwkv6), _ptr(a, "a"),
                                 _in_dtype(q, k, v, beta, a), _ptr(o, "o"), B, H, dk, dv, _stream(stream))
    check("dl_pool_step", status)


def dl_pool_flush(pool: Pool, slot, stream=None) -> None:
    """Merge the listed slots' logs into their bases and zero their counts."""
    B = int(slot.numel())
    _, H, dv, dk = (int(x) for x in pool.S.shape)
    ps = pool.struct()
    status = load().dl_pool_flush(ctypes.byref(ps), pool.log.kind, _slots(slot, B), B, H, dk, dv, _stream(stream))
    check("dl_pool_flush", status)
