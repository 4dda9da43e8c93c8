"""GPU parity of the slot pool (dl_pool_step / dl_pool_flush) against the fp64
oracle's per-sequence recurrence (oracle.pool_eager).

Schedule: P slots; each step lists a random subset of the slots in random
order (a ragged batch), so the sequences sit at different log fills and merge
on different steps; now and then a slot is handed to a new sequence (its
state replaced, its count zeroed). After the last step every slot is flushed
and the pool must hold each sequence's dense state.

Inputs follow the workloads' recipe (unit q and k, v ~ N(0, 1), beta =
sigmoid(N(0, 1)), a = exp(-c softplus(N(0, 1)))), rounded to the input dtype;
the oracle reads the rounded values. Bar as in test_parity_gpu: max|delta| /
max|ref| <= 1e-4 (fp32 state) or 2e-2 (bf16 state), over every output row
and the final pool.
"""
import numpy as np
import pytest

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_104_b200 as g

    g.load()


def _round(x, dt):
    x = np.asarray(x, np.float32)
    return W.bf16_to_f32(W.f32_to_bf16(x)) if dt == "bf16" else x


def _step_inputs(rng, B, H, dk, dv, chan, dt, c=0.3):
    q = rng.standard_normal((B, H, dk)).astype(np.float32)
    k = rng.standard_normal((B, H, dk)).astype(np.float32)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, dv)).astype(np.float32)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H)))).astype(np.float32)
    a = np.exp(-c * np.log1p(np.exp(rng.standard_normal((B, H, dk) if chan else (B, H))))).astype(np.float32)
    return [_round(x, dt) for x in (q, k, v, beta, a)]


def run_pool(P, H, dk, dv, L, T, sdt, idt, decay, seed, resets_every=7):
    import torch

    import gated_delta_rule_104_b200 as g

    rng = np.random.default_rng(seed)
    chan, rw = decay != W.HEAD, decay == W.RWKV6
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}
    pool = g.Pool.allocate(P, H, dk, dv, L, tdt[sdt], tdt[idt], chan, rwkv6=rw)
    S0 = _round(0.02 * rng.standard_normal((P, H, dv, dk)), sdt)
    pool.S.copy_(torch.from_numpy(S0).to(tdt[sdt]))
    steps, resets, outs = [], {}, []
    for t in range(T):
        if t and t % resets_every == 0:  # a new sequence takes a random slot
            s_new = int(rng.integers(P))
            S_new = _round(0.02 * rng.standard_normal((H, dv, dk)), sdt)
            resets[t] = {s_new: S_new}
            pool.reset(s_new, torch.from_numpy(S_new).to(tdt[sdt]))
        B = int(rng.integers(1, P + 1))
        slot = rng.permutation(P)[:B]
        q, k, v, beta, a = _step_inputs(rng, B, H, dk, dv, chan, idt)
        steps.append((slot, q, k, v, None if rw else beta, a))
        dev = [torch.from_numpy(x).to(tdt[idt]).cuda() for x in (q, k, v, beta, a)]
        o = torch.full((B, H, dv), float("nan"), device="cuda")
        g.dl_pool_step(pool, torch.from_numpy(slot.astype(np.int32)).cuda(), dev[0], dev[1], dev[2],
                       None if rw else dev[3], dev[4], o)
        outs.append(o)
    g.dl_pool_flush(pool, torch.arange(P, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert int(pool.status.item()) == 0
    assert int(pool.n.abs().sum().item()) == 0  # every slot flushed
    o_ref, S_ref = oracle.pool_eager(S0.astype(np.float64), steps, chan, rw, resets)
    o_gpu = np.concatenate([x.cpu().numpy().reshape(-1) for x in outs])
    o_exp = np.concatenate([x.reshape(-1) for x in o_ref])
    S_gpu = pool.S.float().cpu().numpy().astype(np.float64)
    tol = 2e-2 if sdt == "bf16" else 1e-4
    eo = np.abs(o_gpu - o_exp).max() / np.abs(o_exp).max()
    es = np.abs(S_gpu - S_ref).max() / np.abs(S_ref).max()
    assert eo <= tol and es <= tol, f"pool {decay} L={L} {sdt}/{idt}: o {eo:.3e} S {es:.3e}"
    return pool


@pytest.mark.parametrize("decay", [W.HEAD, W.CHANNEL, W.RWKV6])
@pytest.mark.parametrize("L", [1, 4, 16])
def test_pool_ragged_batches(decay, L):
    run_pool(P=6, H=3, dk=128, dv=128, L=L, T=41, sdt="f32", idt="bf16", decay=decay, seed=L)


@pytest.mark.parametrize("dk,dv,sdt,idt", [(64, 64, "f32", "f32"), (64, 256, "bf16", "bf16"),
                                           (128, 64, "bf16", "f32")])
def test_pool_shapes_and_dtypes(dk, dv, sdt, idt):
    run_pool(P=5, H=2, dk=dk, dv=dv, L=8, T=30, sdt=sdt, idt=idt, decay=W.CHANNEL, seed=dk + dv)


def test_pool_out_of_range_rows_are_skipped_and_flagged():
    """A row whose slot is outside [0, P) is skipped (its o untouched) and the
    status word flags it; the other rows are computed as usual."""
    import torch

    import gated_delta_rule_104_b200 as g

    P, H, dk, dv, L = 3, 2, 64, 64, 4
    pool = g.Pool.allocate(P, H, dk, dv, L, torch.float32, torch.float32, True)
    rng = np.random.default_rng(5)
    S0 = 0.02 * rng.standard_normal((P, H, dv, dk))
    pool.S.copy_(torch.from_numpy(S0).float())
    q, k, v, beta, a = _step_inputs(rng, 2, H, dk, dv, True, "f32")
    dev = [torch.from_numpy(x).cuda() for x in (q, k, v, beta, a)]
    o = torch.full((2, H, dv), -7.0, device="cuda")
    slot = torch.tensor([1, P], dtype=torch.int32, device="cuda")  # row 1 names a slot that does not exist
    g.dl_pool_step(pool, slot, *dev, o)
    torch.cuda.synchronize()
    assert int(pool.status.item()) == 1
    assert bool((o[1] == -7.0).all())
    o_ref, _ = oracle.pool_eager(S0, [(np.array([1]), q[:1], k[:1], v[:1], beta[:1], a[:1])], True)
    assert np.abs(o[0].cpu().numpy() - o_ref[0][0]).max() <= 1e-4 * np.abs(o_ref[0]).max()
    assert pool.n.tolist() == [0, 1, 0]
