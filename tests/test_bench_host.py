"""Host-side pieces of bench.py and of the schedule driver (CPU only)."""
import os
import subprocess
import sys

import pytest

import bench
import workloads as W
from gated_delta_rule_104_b200.schedule import DeferredDecoder


class FakeOps:
    def __init__(self):
        self.calls = []

    def dl_log_append_read(self, S, log, n, *a):
        assert 0 <= n < log.L
        self.calls.append(("append_read", n))

    def dl_log_merge_read(self, S, log, n, *a):
        assert 0 <= n < log.L
        self.calls.append(("merge_read", n))

    def dl_log_merge(self, S, log, n, *a):
        assert 1 <= n <= log.L
        self.calls.append(("merge", n))


class FakeLog:
    def __init__(self, L):
        self.L = L


def run_schedule(L, T, fused):
    ops = FakeOps()
    dec = DeferredDecoder(None, FakeLog(L), fused_merge=fused, ops=ops)
    for _ in range(T):
        dec.step(None, None, None, None, None, None)
    dec.flush()
    return ops.calls


def test_unfused_schedule_appends_then_merges_full_log():
    calls = run_schedule(4, 10, False)
    assert calls == [("append_read", 0), ("append_read", 1), ("append_read", 2), ("append_read", 3), ("merge", 4),
                     ("append_read", 0), ("append_read", 1), ("append_read", 2), ("append_read", 3), ("merge", 4),
                     ("append_read", 0), ("append_read", 1), ("merge", 2)]


def test_fused_schedule_merges_on_the_filling_step():
    calls = run_schedule(4, 10, True)
    assert calls == [("append_read", 0), ("append_read", 1), ("append_read", 2), ("merge_read", 3),
                     ("append_read", 0), ("append_read", 1), ("append_read", 2), ("merge_read", 3),
                     ("append_read", 0), ("append_read", 1), ("merge", 2)]


@pytest.mark.parametrize("L", [1, 2, 16, 64])
@pytest.mark.parametrize("fused", [True, False])
def test_every_step_reads_once_and_log_never_overflows(L, fused):
    T = 131
    calls = run_schedule(L, T, fused)
    assert sum(1 for k, _ in calls if k in ("append_read", "merge_read")) == T
    n = 0
    for kind, m in calls:
        assert m == n if kind != "merge" else m == n
        n = 0 if kind in ("merge", "merge_read") else n + 1
        assert n <= L
    assert n == 0  # flushed


def test_bench_plan_matches_the_driver():
    w = W.scaled(W.WORKLOADS["kda_b256_h32_d128_t512"], T=40)
    for sched in ("fused", "unfused"):
        lau = bench.Launcher(None, w, None, None, FakeLog(16), None, sched, None)
        assert lau.plan() == run_schedule(16, 40, sched == "fused")
    lau = bench.Launcher(None, w, None, None, None, None, "eager", None)
    assert lau.plan() == [("eager", 0)] * 40


def test_byte_model_matches_the_state_sizes():
    w = W.WORKLOADS["kda_b256_h32_d128_t512"]
    assert w.state_bytes() == 512 << 20
    assert bench.entry_bytes(w) == (128 + 128 + 1 + 128) * 2 == 770
    # eager moves the state twice, the deferred read once
    assert bench.alg_bytes(w, "eager", 0) - 2 * w.state_bytes() == w.heads * (770 + 256 + 512)
    assert bench.alg_bytes(w, "append_read", 3) - w.state_bytes() == w.heads * (5 * 770 + 256 + 512 + 4 * 3 + 4 * 3)
    w4 = W.WORKLOADS["gdn_b1024_h32_dk128_dv256_t256"]
    assert w4.state_bytes() == 2 << 30 and bench.entry_bytes(w4) == (128 + 256 + 2) * 2
    # a pool step at staggered fills: 1/L of the rows at each count, the last one merging
    assert bench.alg_bytes(w, "pool", 16) == (sum(bench.alg_bytes(w, "append_read", c) for c in range(15))
                                              + bench.alg_bytes(w, "merge_read", 15)) // 16
    lau = bench.Launcher(None, w, None, None, type("FakeLog", (), {"L": 16})(), None, "pool", None)
    assert lau.plan() == [("pool", 16)] * w.T
    # RWKV6: no beta in an entry and no triangular-solve rows in the log
    w6 = W.WORKLOADS["rwkv6_b256_h32_d128_t512"]
    assert bench.entry_bytes(w6) == (128 + 128 + 128) * 2
    assert bench.alg_bytes(w6, "append_read", 3) - w6.state_bytes() == w6.heads * (5 * 768 + 256 + 512)


def test_reduce_max_without_process_group():
    assert bench.reduce_max(3.5) == 3.5


GLOO_SCRIPT = r"""
import os, sys
sys.path.insert(0, os.environ["REPO"])
import torch.distributed as dist
import bench
dist.init_process_group("gloo", init_method="env://")
r = dist.get_rank()
m = bench.reduce_max(10.0 + r)            # per-rank device times -> the max
assert m == 11.0, m
open(os.path.join(os.environ["OUT"], f"rank{r}.txt"), "w").write(f"ok {m}")
dist.destroy_process_group()
"""


def test_max_over_ranks_gloo_world2(tmp_path):
    script = tmp_path / "gloo_max.py"
    script.write_text(GLOO_SCRIPT)
    env = dict(os.environ, REPO=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), OUT=str(tmp_path))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", "--master-port=29613", str(script)]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stdout + r.stderr
    for rank in (0, 1):  # every rank sees the max of the per-rank times
        assert (tmp_path / f"rank{rank}.txt").read_text() == "ok 11.0"


def test_kernel_hash_ignores_comments_and_layout_only():
    """The profiled traffic stays tied to the kernel's code: a comment or a
    re-wrapped line keeps the hash, any change of code or literal moves it."""
    src = 'int f(int x) {  // the count\n  /* scaled */ return x * 2 + "a//b"[0]; }\n'
    same = 'int f(int x) {\n    return x * 2 + "a//b"[0];  /* other words */ }'
    assert bench.code_tokens(src) == bench.code_tokens(same)
    assert bench.code_tokens(src) != bench.code_tokens(src.replace("x * 2", "x * 3"))
    assert bench.code_tokens(src) != bench.code_tokens(src.replace('"a//b"', '"a/ /b"'))
    assert "/*" in bench.code_tokens('s = "/*"; t = 1;') and bench.code_tokens("a /* b */ c") == "a c"
    assert bench.code_tokens("x = '\\'' ; // y") == "x = '\\'' ;"


def test_reference_arm_prints_one_oracle_line():
    """`--impl reference` times the oracle on host cores and prints the
    contract's line (smallest workload, so that it runs in seconds)."""
    import json

    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
                          "--workload", "gdn_b1_h2_d64_t16"], cwd=os.path.dirname(bench.__file__),
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s" and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "the same 2 of 2 (b,h) heads" in d["cpu_baseline"]["sample"]


def test_traffic_record_is_used_only_on_the_sources_it_was_taken_on(tmp_path):
    """roofline.traffic comes from the committed JSON record of ncu DRAM bytes,
    keyed by kernel, workload and L, and only while the kernel sources still
    hash to the value recorded with them."""
    import json

    srcs = ["gated_delta_rule_104_b200/csrc/deferred_read.cu", "gated_delta_rule_104_b200/csrc/common.cuh"]
    rec = {bench.traffic_key("append_read", "w", 16): {"dram_bytes_per_launch": 123.0, "sources": srcs,
                                                      "source_sha256_16": bench.kernel_source_hash(srcs)},
           bench.traffic_key("merge_read", "w", 16): {"dram_bytes_per_launch": 9.0, "sources": srcs,
                                                     "source_sha256_16": "0" * 16}}
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(rec))
    assert bench.profiled_traffic("append_read", "w", 16, str(p)) == 123.0
    assert bench.profiled_traffic("merge_read", "w", 16, str(p)) is None  # stale hash
    assert bench.profiled_traffic("append_read", "w", 8, str(p)) is None  # no record for this L
    assert bench.profiled_traffic("append_read", "w", 16, str(tmp_path / "missing.json")) is None
    # the committed record parses and names existing sources
    committed = json.load(open(bench.TRAFFIC_RECORD))
    for key, r in committed.items():
        assert key.count("/") == 2 and r["dram_bytes_per_launch"] > 0
        for s in r["sources"]:
            assert os.path.exists(os.path.join(os.path.dirname(bench.__file__), s)), s


def test_sweep_plan_bytes_per_token():
    """The sweep's bytes per token: eager is 2 states + inputs per head-step;
    the fused deferred plan at L = 1 is one merge-read per step (the same bytes
    as eager); at larger L it is below eager."""
    w = W.WORKLOADS["kda_b128_h16_d128_t2048"]
    w = W.scaled(w, T=64)

    def plan(schedule, L):
        lau = bench.Launcher(None, w, None, None, None, None, schedule, None)
        lau.L = L
        return lau.plan()

    eager = bench.decode_bytes(w, plan("eager", 0))
    assert eager == w.T * bench.alg_bytes(w, "eager", 0)
    assert bench.decode_bytes(w, plan("fused", 1)) == w.T * bench.alg_bytes(w, "merge_read", 0)
    assert bench.alg_bytes(w, "merge_read", 0) == bench.alg_bytes(w, "eager", 0)
    for L in (4, 8, 16):
        assert bench.decode_bytes(w, plan("fused", L)) < eager
