"""Host-side driver of the DeltaLog schedule for one batch of states.

DeltaLog page, Technical Summary, "Core Mechanism: Base + Log": the live
state is a dense base plus a bounded log; each step appends its factors and
reads from base + log, and every L steps the log is merged into the base.

``DeferredDecoder`` keeps the host count n of valid log entries (the same for
every sequence of the batch) and issues, per step:
  * n < L-1, or fused merging off:  dl_log_append_read(n), n += 1, and (fused
    off) dl_log_merge(L) when the log becomes full;
  * n == L-1 with fused merging:    dl_log_merge_read(n) -- the step that
    fills the log merges it in the same pass over the base -- then n = 0.
``flush()`` merges what is left so the base holds the current state.
The backend (``ops``) is the ctypes binding by default; tests substitute a
recording fake to check the schedule on the CPU.
"""
from __future__ import annotations

from typing import Optional


class DeferredDecoder:
    def __init__(self, S_base, log, fused_merge: bool = True, ops=None):
        if ops is None:
            from . import _binding as ops
        self.ops = ops
        self.S = S_base
        self.log = log
        self.L = int(log.L)
        self.fused = bool(fused_merge)
        self.n = 0
        self.steps = 0

    def step(self, q, k, v, beta, a, o, stream: Optional[object] = None) -> None:
        if self.fused and self.n == self.L - 1:
            self.ops.dl_log_merge_read(self.S, self.log, self.n, q, k, v, beta, a, o, stream)
            self.n = 0
        else:
            self.ops.dl_log_append_read(self.S, self.log, self.n, q, k, v, beta, a, o, stream)
            self.n += 1
            if self.n == self.L:
                self.ops.dl_log_merge(self.S, self.log, self.n, stream)
                self.n = 0
        self.steps += 1

    def flush(self, stream: Optional[object] = None) -> None:
        if self.n:
            self.ops.dl_log_merge(self.S, self.log, self.n, stream)
            self.n = 0
