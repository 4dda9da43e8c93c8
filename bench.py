"""Decode-step benchmark: gated delta-rule state updates on B200.

One bench step = one full decode of the workload's T tokens for all B
sequences (every head of every layer-slice in the batch), through the C ABI:
  * deferred (the headline, DeltaLog schedule): dl_log_append_read on the
    steps that append, dl_log_merge_read on the step that fills the log
    (merge fused with that step's read), i.e. every row of the path: append,
    key-side recursion, base read, merge;
  * eager, timed the same way, reported beside it;
  * e2e: the deferred decode from pinned host buffers -- initial state and
    each token's q, k, v, beta, a copied in, each token's o and the final
    state copied out, all inside the timed region.
Metric: decode tokens/s = B * T / time (state updates/s = B * H * T / time)
and achieved HBM GB/s of the dominant kernel against the measured peak.

Timing: W untimed warm-up steps, then K steps between a barrier +
cuda.synchronize on both sides, CUDA events on the launching stream, max
over ranks. Inputs (a 512 MiB fp32 state) are larger than L2, so no flush.
Multi-GPU (torchrun, one rank per GPU): every rank decodes its own batch
(weak scaling; sequences are independent, no collective on the data path).

--impl reference times the fp64 CPU oracle (the only other implementation
of this path) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402  (seeded inputs; no method arithmetic)

METRIC = "decode tokens/sec (B×H state updates/s) and achieved HBM GB/s vs peak, 1 B200"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "kda_b256_h32_d128_t512"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
# ncu DRAM traffic per launch, recorded per (kernel, workload, L) with a hash of
# the kernel sources it was captured on (profiles/dram_traffic.json)
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")


# ---------------------------------------------------------------- byte model

def entry_bytes(w: W.Workload) -> int:
    """Bytes of one log entry / one step's (k, v, beta, a); RWKV6 has no beta."""
    s_in = 2 if w.in_dtype == "bf16" else 4
    beta = 0 if w.decay == W.RWKV6 else 1
    return (w.d_k + w.d_v + beta + (1 if w.decay == W.HEAD else w.d_k)) * s_in


def state_bytes_head(w: W.Workload) -> int:
    if w.state_dtype == "i8":  # int8 codes and a float scale per row
        return w.d_v * w.d_k + 4 * w.d_v
    return w.d_v * w.d_k * (2 if w.state_dtype == "bf16" else 4)


def alg_bytes(w: W.Workload, kind: str, n: int) -> int:
    """Algorithmic HBM bytes of one launch over all B*H heads.

    eager:        state read + write, this step's inputs, o
    append_read:  state read (no write), n log entries read, one entry
                  written, this step's inputs, o, and the log metadata: the
                  older entries' C rows read (n(n-1)/2 floats), the new row
                  written (n floats); RWKV6 keeps no such rows
    merge_read:   state read + write, n log entries and their C rows, this
                  step's inputs, o
    merge:        state read + write, n log entries and their C rows
    pool:         one slot-pool step of the whole batch with staggered fills
                  (sequence b holds (b + step) mod L entries, n = L): the
                  rows at L - 1 merge (merge_read), the others append_read
    """
    if kind == "pool":
        L = n
        tot = 0
        for c in range(L):
            nseq = len(range(c, w.B, L))
            sub = "merge_read" if c == L - 1 else "append_read"
            tot += nseq * alg_bytes(w, sub, c) // w.B
        return tot
    e, S = entry_bytes(w), state_bytes_head(w)
    s_in = 2 if w.in_dtype == "bf16" else 4
    q, o = w.d_k * s_in, 4 * w.d_v
    delta = w.decay != W.RWKV6
    crows = 4 * n * (n - 1) // 2 if delta else 0
    per_head = {
        "eager": 2 * S + e + q + o,
        "append_read": S + n * e + e + e + q + o + crows + (4 * n if delta else 0),
        "merge_read": 2 * S + n * e + e + q + o + crows,
        "merge": 2 * S + n * e + crows,
    }[kind]
    return per_head * w.heads


KERNELS_PER_CALL = {"eager": 1, "append_read": 2, "merge_read": 1, "merge": 1, "pool": 4}  # see Launcher.kernels


# ---------------------------------------------------------------- helpers

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def reduce_max(x: float) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def code_tokens(src: str) -> str:
    """C/C++/CUDA source with its comments removed and whitespace runs folded
    to one space: what the compiler sees, so that a comment edit does not
    count as a kernel change. String and character literals are kept whole."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(sources) -> str:
    """Hash of a kernel's code (comments and layout excluded); a recorded DRAM
    traffic figure is used only while its sources still hash to the value
    recorded with it."""
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_key(kind: str, workload: str, L: int) -> str:
    return f"{kind}/{workload}/L{L}"


def profiled_traffic(kind: str, workload: str, L: int, record: str = TRAFFIC_RECORD):
    """DRAM bytes per launch of ``kind`` from the committed ncu record, if one
    was taken for this workload and L on the current kernel sources (else None)."""
    try:
        with open(record, encoding="utf-8") as f:
            rec = json.load(f).get(traffic_key(kind, workload, L))
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha256_16") != kernel_source_hash(rec.get("sources", [])):
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms (read only)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle leg

REFERENCE_RUN_S = 120.0  # oracle seconds for all timed steps of `--impl reference`
REFERENCE_MAX_HEADS = 2048  # bound on its sample (about 1 MB of inputs per head)


def oracle_sample(w: W.Workload, L: int, budget_s: float, first_head: int = 0):
    """Time the fp64 oracle (deferred schedule, log capacity L) on heads of the
    workload until about ``budget_s`` seconds of CPU work; returns
    (tokens/s-equivalent, heads, seconds, threads)."""
    import oracle  # test infrastructure: CPU baseline only

    oracle.build()
    threads = oracle.omp_threads()
    chunk = max(1, threads)
    heads_done, secs, h0 = 0, 0.0, first_head
    while secs < budget_s and heads_done < w.heads:
        heads = [(h0 + i) % w.heads for i in range(min(chunk, w.heads - heads_done))]
        x = W.generate(w, heads=heads)
        t0 = time.perf_counter()
        oracle.run_workload_heads(w, x, "deferred", L)
        secs += time.perf_counter() - t0
        heads_done += len(heads)
        h0 += len(heads)
        # next chunk: double, but no more than the measured rate fits in what is
        # left of the budget (a multiple of the threads, at least one round)
        fit = int((budget_s - secs) / (max(secs, 1e-9) / heads_done)) // threads * threads
        chunk = max(threads, min(chunk * 2, 4096, fit))
    tokens = heads_done * w.T / w.H  # one token = one sequence step across its H heads
    return tokens / secs, heads_done, secs, threads


def run_reference(args, w, L):
    rank, _, ws = dist_env()
    if rank != 0:
        return 0
    import oracle  # the reference arm is the oracle itself

    oracle.build()
    threads = oracle.omp_threads()
    # Each timed step runs the oracle's deferred schedule over one fixed sample
    # of heads (all T steps of each), sized by a short probe so that a step is
    # about `budget` seconds and the whole run about REFERENCE_RUN_S; the
    # sample's inputs are generated once and reused by every step.
    budget = min(args.cpu_seconds_per_step, max(1.0, REFERENCE_RUN_S / max(1, args.steps)))
    n_probe = min(threads, w.heads)
    probe = W.generate(w, heads=range(n_probe))
    t0 = time.perf_counter()
    oracle.run_workload_heads(w, probe, "deferred", L)
    per_head = max(time.perf_counter() - t0, 1e-9) / n_probe
    nh = int(budget / per_head) // threads * threads
    nh = max(n_probe, min(nh, w.heads, REFERENCE_MAX_HEADS))
    stride = 997  # spread the sample over the batch (coprime with every B*H used)
    x = W.generate(w, heads=[(i * stride) % w.heads for i in range(nh)])
    for _ in range(args.warmup):
        oracle.run_workload_heads(w, probe, "deferred", L)
    secs_all = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.run_workload_heads(w, x, "deferred", L)
        secs_all += time.perf_counter() - t0
    heads_all = nh * args.steps
    value = heads_all * w.T / w.H / secs_all
    sample = (f"the same {nh} of {w.heads} (b,h) heads x all {w.T} steps in each of {args.steps} steps "
              f"({secs_all / max(1, args.steps):.1f} s of oracle work each), deferred schedule L={L}, fp64")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * w.B * w.T / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(w, L, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_block(w, L, args):
    decay = {W.CHANNEL: "channel (KDA)", W.HEAD: "head (GDN)",
             W.RWKV6: "channel, raw-value update without delta correction (RWKV6)"}[w.decay]
    return {"workload": w.name, "decay": decay,
            "B": w.B, "H": w.H, "d_k": w.d_k, "d_v": w.d_v, "T": w.T, "L": L,
            "state_dtype": ("deferred base int8 (row scales), eager " + w.state_dtype)
            if getattr(args, "base_i8", False) else w.state_dtype, "in_dtype": w.in_dtype,
            "schedule": {"fused": "DeltaLog deferred, merge fused into the L-th step",
                         "unfused": "DeltaLog deferred, separate merge every L steps",
                         "pool": "slot pool, staggered log fills (each step 1/L of the rows merge)"}[args.schedule],
            "global_batch": w.B * max(1, dist_env()[2]), "seq_len": w.T,
            # (the reference arm prints the same block as this arm; its own timing,
            # host wall time of the oracle, is stated in its cpu_baseline)
            "timing": ("launches issued directly, CUDA events around the decode"
                       if getattr(args, "no_graph", False)
                       else "one decode captured as a CUDA graph, replayed once per step between CUDA events; "
                            "per-kernel split from one more decode with events around each launch"),
            "l2": "inputs larger than L2 (state %d MiB per GPU), no flush" % (w.state_bytes() >> 20)}


# ---------------------------------------------------------------- GPU legs

class Launcher:
    """Issues the T steps of one decode and (optionally) brackets every launch
    with CUDA events on the launching stream."""

    def __init__(self, g, w, d, S, log, o_all, schedule, stream, pool=None):
        self.g, self.w, self.d, self.S, self.log, self.o_all = g, w, d, S, log, o_all
        self.schedule, self.stream, self.pool = schedule, stream, pool
        self.chan = w.decay != W.HEAD
        self.rwkv6 = w.decay == W.RWKV6
        self.L = log.L if log is not None else 0

    def kernels(self, kind):
        """Kernels one call of `kind` launches: the deferred read runs as one
        kernel on an fp32 or bf16 base with L <= 16, d_v <= 128 and at least
        32 heads per SM, else as two."""
        import torch

        if kind == "append_read":
            if not isinstance(self.S, torch.Tensor) or self.S.dtype not in (torch.float32, torch.bfloat16):
                return 2  # an int8 base
            sms = torch.cuda.get_device_properties(self.S.device).multi_processor_count
            one = self.L <= 16 and self.w.d_v <= 128 and self.w.heads >= 32 * sms
            return 1 if one else 2
        return KERNELS_PER_CALL[kind]

    def plan(self):
        """(kind, n) of each launch of one decode, in order."""
        out, n = [], 0
        if self.schedule == "pool":
            return [("pool", self.L)] * self.w.T
        for _ in range(self.w.T):
            if self.schedule == "eager":
                out.append(("eager", 0))
            elif self.schedule == "fused" and n == self.L - 1:
                out.append(("merge_read", n))
                n = 0
            else:
                out.append(("append_read", n))
                n += 1
                if n == self.L:
                    out.append(("merge", n))
                    n = 0
        if n:
            out.append(("merge", n))  # flush so that S holds the final state
        return out

    def pool_join(self):
        """Untimed: sequence b joins at step (L-1) - (b mod L), so after L-1
        steps it holds b mod L entries and the fills are staggered."""
        import torch

        g, d, L = self.g, self.d, self.L
        B = self.w.B
        for j in range(L - 1):
            rows = [b for b in range(B) if j >= (L - 1) - (b % L)]
            if not rows:
                continue
            idx = torch.tensor(rows, dtype=torch.long, device="cuda")
            slot = idx.to(torch.int32)
            pick = lambda key: d[key][j].index_select(0, idx).contiguous()  # noqa: E731
            beta = None if self.rwkv6 else pick("beta")
            o = torch.empty(len(rows), self.w.H, self.w.d_v, device="cuda")
            g.dl_pool_step(self.pool, slot, pick("q"), pick("k"), pick("v"), beta, pick("a"), o, self.stream)

    def run(self, events=None):
        g, d, S, o, st = self.g, self.d, self.S, self.o_all, self.stream
        if self.schedule == "pool":
            slots = self.pool_slots
            for t in range(self.w.T):
                if events is not None:
                    events.append(self._ev())
                beta = None if self.rwkv6 else d["beta"][t]
                g.dl_pool_step(self.pool, slots, d["q"][t], d["k"][t], d["v"][t], beta, d["a"][t], o[t], st)
            if events is not None:
                events.append(self._ev())
            return
        t = 0
        for kind, n in self.plan():
            if events is not None:
                events.append(self._ev())
            beta = None if self.rwkv6 else d["beta"][t]
            if kind == "eager":
                if self.rwkv6:
                    g.dl_rwkv6_decode_step(S, d["q"][t], d["k"][t], d["v"][t], d["a"][t], o[t], st)
                else:
                    fn = g.dl_kda_decode_step if self.chan else g.dl_gdn_decode_step
                    fn(S, d["q"][t], d["k"][t], d["v"][t], beta, d["a"][t], o[t], st)
                t += 1
            elif kind == "append_read":
                g.dl_log_append_read(S, self.log, n, d["q"][t], d["k"][t], d["v"][t], beta, d["a"][t], o[t], st)
                t += 1
            elif kind == "merge_read":
                g.dl_log_merge_read(S, self.log, n, d["q"][t], d["k"][t], d["v"][t], beta, d["a"][t], o[t], st)
                t += 1
            else:
                g.dl_log_merge(S, self.log, n, st)
        if events is not None:
            events.append(self._ev())

    def _ev(self):
        import torch

        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e


def timed(launcher, steps, warmup, use_graph=True):
    """Returns (ms per step (max over ranks), per-kind {durations}, launches).

    The step time: with ``use_graph`` one decode (all T steps' launches) is
    captured once in a CUDA graph after the warm-up and replayed ``steps``
    times between CUDA events, so that host launch overhead does not enter
    (a serving loop replays its decode graph the same way); otherwise the
    launches are issued directly. The per-kind split always comes from one
    more decode issued directly with events around every launch (for short
    kernels those times include launch gaps: an upper bound)."""
    import torch
    import torch.distributed as dist

    for _ in range(warmup):
        launcher.run()
    torch.cuda.synchronize()
    if dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    plan = launcher.plan()
    graph = None
    if use_graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        home = launcher.stream
        launcher.stream = side
        try:
            with torch.cuda.graph(graph, stream=side):
                launcher.run()
        finally:
            launcher.stream = home
        torch.cuda.synchronize()
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        if dist.is_initialized():
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(launcher.stream)
        for _ in range(steps):
            graph.replay()
        e1.record(launcher.stream)
        torch.cuda.synchronize()
        if dist.is_initialized():
            dist.barrier()
        total_ms = e0.elapsed_time(e1)
        ev = []
        launcher.run(ev)  # the per-kind split
        torch.cuda.synchronize()
        all_events = [ev]
    else:
        all_events = []
        for _ in range(steps):
            ev = []
            launcher.run(ev)
            all_events.append(ev)
        torch.cuda.synchronize()
        if dist.is_initialized():
            dist.barrier()
        total_ms = sum(ev[0].elapsed_time(ev[-1]) for ev in all_events)
    per_kind = {}
    for ev in all_events:
        for i, (kind, n) in enumerate(plan):
            per_kind.setdefault(kind, []).append((n, ev[i].elapsed_time(ev[i + 1])))
    del graph
    ms = reduce_max(total_ms / steps)
    return ms, per_kind, steps * sum(launcher.kernels(kind) for kind, _ in plan)


def roofline_for(w, per_kind, kind, peak, peak_note, traffic):
    rec = per_kind.get(kind, [])
    if not rec:
        return None
    total_bytes = sum(alg_bytes(w, kind, n) for n, _ in rec)
    total_s = sum(ms for _, ms in rec) / 1000.0
    achieved = total_bytes / total_s / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": kind, "launches": len(rec), "avg_us": round(1e6 * total_s / len(rec), 2),
            "alg_bytes_per_launch": round(total_bytes / len(rec)), "peak_source": peak_note,
            "frac_of_8tbs_spec": round(achieved / SPEC_HBM_GBS, 4)}


def run_e2e(g, w, host, L, schedule, steps, warmup, stream):
    """Deferred decode from pinned host buffers through the public API:
    per step, S0 and every token's inputs H2D, every token's o and the final
    state D2H (copy streams overlap the kernels)."""
    import torch

    dev = torch.device("cuda")
    chan = w.decay != W.HEAD
    rw = w.decay == W.RWKV6
    tdt = torch.bfloat16 if w.in_dtype == "bf16" else torch.float32
    B, H = w.B, w.H
    S = torch.empty(B, H, w.d_v, w.d_k, dtype=host["S0"].dtype, device=dev)
    log = g.Log.allocate(B, H, w.d_k, w.d_v, L, tdt, chan, device=dev, rwkv6=rw)
    names = ("q", "k", "v", "a") if rw else ("q", "k", "v", "beta", "a")
    # Each token's inputs sit in one pinned staging row (every field 16-byte
    # aligned), as a caller's input buffer would hold them, so that one copy per
    # token moves them; the device slots are views of one buffer the same way.
    fields, row = [], 0
    for n in names:
        t0 = host[n][0]
        nb = t0.numel() * t0.element_size()
        fields.append((n, row, nb, t0.dtype, tuple(t0.shape)))
        row += (nb + 15) // 16 * 16
    packed = torch.empty(w.T, row, dtype=torch.uint8, pin_memory=True)
    for t in range(w.T):
        for n, off, nb, dt, shp in fields:
            packed[t, off:off + nb].view(dt).view(shp).copy_(host[n][t])
    nslot = 3
    slot_buf = [torch.empty(row, dtype=torch.uint8, device=dev) for _ in range(nslot)]
    slots = [{n: slot_buf[j][off:off + nb].view(dt).view(shp) for n, off, nb, dt, shp in fields}
             for j in range(nslot)]
    o_dev = [torch.empty(B, H, w.d_v, dtype=torch.float32, device=dev) for _ in range(nslot)]
    o_host = torch.empty(w.T, B, H, w.d_v, dtype=torch.float32, pin_memory=True)
    S_host = torch.empty_like(host["S0"], pin_memory=True)
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_bytes = host["S0"].numel() * host["S0"].element_size() + w.T * row
    d2h_bytes = o_host.numel() * 4 + S_host.numel() * S_host.element_size()

    def one():
        ev_in = [torch.cuda.Event() for _ in range(nslot)]
        ev_used = [None] * nslot
        ev_out = [None] * nslot
        with torch.cuda.stream(h2d):
            S.copy_(host["S0"], non_blocking=True)
        s_ready = torch.cuda.Event()
        s_ready.record(h2d)
        stream.wait_event(s_ready)
        dec = g.DeferredDecoder(S, log, fused_merge=(schedule == "fused"))
        for t in range(w.T):
            j = t % nslot
            with torch.cuda.stream(h2d):
                if ev_used[j] is not None:
                    h2d.wait_event(ev_used[j])
                slot_buf[j].copy_(packed[t], non_blocking=True)
                ev_in[j].record(h2d)
            stream.wait_event(ev_in[j])
            if ev_out[j] is not None:
                stream.wait_event(ev_out[j])  # o slot drained
            sl = slots[j]
            dec.step(sl["q"], sl["k"], sl["v"], sl.get("beta"), sl["a"], o_dev[j], stream)
            ev_used[j] = torch.cuda.Event()
            ev_used[j].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_used[j])
                o_host[t].copy_(o_dev[j], non_blocking=True)
                ev_out[j] = torch.cuda.Event()
                ev_out[j].record(d2h)
        dec.flush(stream)
        done = torch.cuda.Event()
        done.record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(done)
            S_host.copy_(S, non_blocking=True)

    import torch.distributed as dist

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    if dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    start_events = []
    for _ in range(steps):
        one()
    # the last D2H copy ends the step: join it into the timing stream
    end_d2h = torch.cuda.Event()
    end_d2h.record(d2h)
    stream.wait_event(end_d2h)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist.is_initialized():
        dist.barrier()
    ms = reduce_max(e0.elapsed_time(e1) / steps)
    del start_events
    return ms, h2d_bytes, d2h_bytes


def decode_bytes(w, plan):
    """Algorithmic bytes of one whole decode (every launch of the plan)."""
    return sum(alg_bytes(w, kind, n) for kind, n in plan)


def run_sweep(args, w, Ls):
    """Log-capacity sweep on one workload (the page's trade-off between replay
    traffic and saved dense writes): per L, the fused deferred decode's
    tokens/s, its read/merge time split and its bytes per token, beside the
    eager decode's."""
    workers = args.workers or W.default_workers()
    x = W.generate(w, workers=workers)

    import torch

    import gated_delta_rule_104_b200 as g

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA library is the only compute path)")
    torch.cuda.set_device(0)
    g.load()
    d = W.device_inputs(w, x)
    del x
    stream = torch.cuda.current_stream()
    chan, rw = w.decay != W.HEAD, w.decay == W.RWKV6
    o_all = torch.empty(w.T, w.B, w.H, w.d_v, dtype=torch.float32, device="cuda")
    peak, peak_note = measured_peaks()
    tokens = w.B * w.T
    S_e = d["S0"].clone()
    lau_e = Launcher(g, w, d, S_e, None, o_all, "eager", stream)
    with ClockSampler(0) as smp:
        ms_e, kinds_e, _ = timed(lau_e, args.steps, args.warmup, not args.no_graph)
    del S_e
    eager_bpt = decode_bytes(w, lau_e.plan()) / tokens
    eager_val = tokens / (ms_e / 1000.0)
    print(json.dumps({"sweep": "eager", "workload": w.name, "value": eager_val, "unit": UNIT,
                      "ms_per_step": round(ms_e, 3), "alg_bytes_per_token": round(eager_bpt),
                      "roofline": roofline_for(w, kinds_e, "eager", peak, peak_note, None),
                      "clocks": smp.summary()}), flush=True)
    for L in Ls:
        S = d["S0"].clone()
        log = g.Log.allocate(w.B, w.H, w.d_k, w.d_v, L, d["q"].dtype, chan, rwkv6=rw)
        lau = Launcher(g, w, d, S, log, o_all, "fused", stream)
        with ClockSampler(0) as smp:
            ms, kinds, launches = timed(lau, args.steps, args.warmup, not args.no_graph)
        split = {k: round(sum(ms_ for _, ms_ in v) / (args.steps if args.no_graph else 1), 3) for k, v in kinds.items()}
        bpt = decode_bytes(w, lau.plan()) / tokens
        value = tokens / (ms / 1000.0)
        print(json.dumps({
            "sweep": "L", "workload": w.name, "L": L, "value": value, "unit": UNIT, "ms_per_step": round(ms, 3),
            "eager_value": eager_val, "deferred_over_eager": value / eager_val,
            "ms_per_step_by_kernel": split,
            "read_share": round(split.get("append_read", 0.0) / max(ms, 1e-9), 4),
            "alg_bytes_per_token": round(bpt), "eager_alg_bytes_per_token": round(eager_bpt),
            "eager_over_deferred_bytes": round(eager_bpt / bpt, 4),
            "roofline": {k: roofline_for(w, kinds, k, peak, peak_note, profiled_traffic(k, w.name, L))
                         for k in kinds},
            "gpu_launches": launches, "clocks": smp.summary()}), flush=True)
        del S, log
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--L", type=int, default=0, help="log capacity (default: the workload's)")
    ap.add_argument("--schedule", choices=["fused", "unfused", "pool"], default="fused",
                    help="pool: the slot-pool step over the whole batch at staggered log fills")
    ap.add_argument("--workers", type=int, default=0, help="input-generation processes (0: auto)")
    ap.add_argument("--cpu-seconds-per-step", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--base-i8", action="store_true",
                    help="the deferred legs on an int8 base (DL_I8, rounded from S0 before timing); eager stays fp32")
    ap.add_argument("--no-eager", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="decode only this many tokens per step (small profiling runs; default: the workload's T)")
    ap.add_argument("--no-graph", action="store_true",
                    help="issue every launch directly in the timed steps (default: replay a CUDA graph of one decode)")
    ap.add_argument("--sweep-L", default="",
                    help="comma list of log capacities: one JSON line per L (fused deferred schedule, with the "
                         "read/merge split and bytes per token) after one eager line, inputs generated once")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = W.WORKLOADS[args.workload]
    if args.tokens:
        w = W.scaled(w, T=args.tokens)
    L = args.L or max(w.L)
    rank, local_rank, ws = dist_env()
    if args.gpus != ws and ws > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={ws}", file=sys.stderr)

    if args.impl == "reference":
        return run_reference(args, w, L)
    if args.sweep_L:
        return run_sweep(args, w, [int(x) for x in args.sweep_L.split(",") if x.strip()])

    # Inputs first (spawned generator processes start before any CUDA call).
    workers = args.workers or W.default_workers()
    t0 = time.time()
    x = W.generate(w, workers=workers)
    gen_s = time.time() - t0

    import torch
    import torch.distributed as dist

    import gated_delta_rule_104_b200 as g

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA library is the only compute path)")
    torch.cuda.set_device(local_rank)
    if ws > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    g.load()
    d = W.device_inputs(w, x)
    stream = torch.cuda.current_stream()
    chan = w.decay != W.HEAD
    tdt = d["q"].dtype
    o_all = torch.empty(w.T, w.B, w.H, w.d_v, dtype=torch.float32, device="cuda")
    peak, peak_note = measured_peaks()

    sampler = ClockSampler(local_rank)
    with sampler:
        rw = w.decay == W.RWKV6
        if args.base_i8 and args.schedule != "pool":
            S8 = g.I8State.allocate(w.B, w.H, w.d_k, w.d_v)
            g.dl_state_to_i8(d["S0"].float().contiguous(), S8)
            log = g.Log.allocate(w.B, w.H, w.d_k, w.d_v, L, tdt, chan, rwkv6=rw)
            w_def = W.scaled(w, state_dtype="i8")  # byte model of the deferred kernels
            lau = Launcher(g, w_def, d, S8, log, o_all, args.schedule, stream)
            S_def = S8
        elif args.schedule == "pool":
            pool = g.Pool.allocate(w.B, w.H, w.d_k, w.d_v, L, d["S0"].dtype, tdt, chan, rwkv6=rw)
            pool.S.copy_(d["S0"])
            S_def, log = pool.S, pool.log
            lau = Launcher(g, w, d, S_def, log, o_all, "pool", stream, pool=pool)
            lau.pool_slots = torch.arange(w.B, dtype=torch.int32, device="cuda")
            lau.pool_join()
        else:
            S_def = d["S0"].clone()
            log = g.Log.allocate(w.B, w.H, w.d_k, w.d_v, L, tdt, chan, rwkv6=rw)
            lau = Launcher(g, w, d, S_def, log, o_all, args.schedule, stream)
        ms_def, kinds_def, launches = timed(lau, args.steps, args.warmup, not args.no_graph)
        eager = None
        if not args.no_eager:
            S_e = d["S0"].clone()
            lau_e = Launcher(g, w, d, S_e, None, o_all, "eager", stream)
            ms_e, kinds_e, _ = timed(lau_e, args.steps, args.warmup, not args.no_graph)
            eager = {"value": w.B * w.T / (ms_e / 1000.0) * ws, "unit": UNIT, "ms_per_step": round(ms_e, 3),
                     "state_updates_per_s": w.heads * w.T / (ms_e / 1000.0) * ws,
                     "roofline": roofline_for(w, kinds_e, "eager", peak, peak_note, None)}
            del S_e
    clocks = sampler.summary()

    value = w.B * w.T / (ms_def / 1000.0) * ws
    main_kind = "pool" if args.schedule == "pool" else "append_read"
    wb = W.scaled(w, state_dtype="i8") if args.base_i8 else w
    def traffic(kind):  # the ncu record is of the fp32/bf16 base on the fused schedule
        if args.base_i8 or args.tokens or args.schedule == "unfused":
            return None
        return profiled_traffic(kind, w.name, L)

    rf = roofline_for(wb, kinds_def, main_kind, peak, peak_note, traffic(main_kind))
    other = {k: roofline_for(wb, kinds_def, k, peak, peak_note, traffic(k)) for k in kinds_def if k != main_kind}
    split_steps = 1 if not args.no_graph else args.steps
    step_time = {k: round(sum(ms for _, ms in v) / split_steps, 3) for k, v in kinds_def.items()}

    e2e = None
    if not args.no_e2e and args.schedule != "pool" and not args.base_i8:
        host = {}
        for n in ("S0", "q", "k", "v", "beta", "a"):
            if n == "beta" and w.decay == W.RWKV6:
                continue
            host[n] = d[n].cpu().pin_memory()
        ms_e2e, h2d_b, d2h_b = run_e2e(g, w, host, L, args.schedule, max(2, args.steps // 4), args.warmup, stream)
        e2e = {"value": w.B * w.T / (ms_e2e / 1000.0) * ws, "unit": UNIT, "ms_per_step": round(ms_e2e, 3),
               "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
               "what": "deferred decode from pinned host memory: S0 and per-token inputs in, per-token o "
                       "and the final state out, inside the timed region"}
        del host

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, heads, secs, threads = oracle_sample(w, L, args.cpu_seconds_per_step)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{heads} of {w.heads} (b,h) heads x all {w.T} steps, fp64 deferred schedule L={L}, "
                         f"{secs:.1f} s on {threads} OpenMP threads; tokens = heads x T / H"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_def, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "config": config_block(w, L, args),
        "state_updates_per_s": w.heads * w.T / (ms_def / 1000.0) * ws,
        "roofline": rf, "roofline_other_kernels": other, "ms_per_step_by_kernel": step_time,
        "eager": eager, "deferred_over_eager": (value / eager["value"]) if eager else None,
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": launches, "clocks": clocks,
        "input_generation_s": round(gen_s, 1),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
