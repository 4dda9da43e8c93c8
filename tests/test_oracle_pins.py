"""Pins of the fp64 oracle to things other than itself (CPU only).

The update rule (decay, then the delta-rule correction; head-wise decay for
Gated DeltaNet, per-key decay for Kimi Delta Attention -- DeltaLog page,
Technical Summary, "Kernel Implementation") is

    S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,

and the deferred schedule must reproduce it exactly: the method changes only
when the state is written back, never what it computes (Technical Summary,
"Methodology").

Pins:
  P0 hand-worked exact examples (tests/golden/hand_worked_steps.json);
  P1 beta = 0, a = 1 leaves S unchanged and o = S_0 q;
  P2 unit-norm k with beta = 1 stores v exactly: S_t k_t = v_t;
  P3 beta = 0 gives S_T = S_0 Diag(prod_t a_t);
  P4 a = 1, beta = 1, orthonormal k_1..k_n: S_n = S_0 (I - sum k k^T) + sum v k^T;
  P5 channel decay with all channels equal = head-wise decay;
  P6 deferred schedule = eager for every log capacity (merge cadence, flush);
  P7 dense brute-force matrix products = eager = deferred on tiny shapes;
  P8 the deferred window identity S_n = S_bar A_1..A_n + sum beta v k^T A_{i+1}..A_n;
  P9 RWKV6 (per-key decay, raw-value update, no correction: S_t = S_{t-1} Diag(a_t)
     + v_t k_t^T) -- dense brute force = eager = deferred at every log capacity;
  P10 RWKV6 closed form S_T = S_0 Diag(prod_t a_t) + sum_t v_t (k_t o prod_{m>t} a_m)^T,
     with its special cases a = 1 (plain linear attention) and a = 0;
  P11 the slot pool (per-sequence states in slots, ragged batches): a
     sequence's outputs and state are those of its own recurrence, whatever
     the other slots do; slots not listed in a step are left unchanged;
  P12 the int8 base (a scale per state row, max|row| / 127, codes rounded to
     the nearest integer, ties to even): a hand-worked row; rounding a rounded
     state changes nothing; with no merge before the end the outputs are the
     eager ones from the rounded initial state and the final state is that
     state rounded; with merges every L steps the base is the exact schedule's
     rounded once per window.
The mutation test builds copies of the C oracle with planted mistakes and
checks that these pins reject each of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_steps.json")


def rand_case(rng, NH, T, dk, dv, chan, unit_k=True, beta=None, a=None):
    S0 = rng.standard_normal((NH, dv, dk)) * 0.3
    q = rng.standard_normal((T, NH, dk))
    k = rng.standard_normal((T, NH, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, NH, dv))
    if beta is None:
        beta = rng.uniform(0.05, 0.95, (T, NH))
    if a is None:
        a = rng.uniform(0.6, 1.0, (T, NH, dk) if chan else (T, NH))
    return S0, q, k, v, beta, a


def rel(x, y):
    return np.abs(x - y).max() / max(np.abs(y).max(), 1e-300)


# ------------------------------------------------------------------ P0

def _frac(x):
    return float(Fraction(x))


@pytest.mark.parametrize("form", ["eager", "deferred1", "deferred2", "deferred3", "brute"])
def test_p0_hand_worked_examples(form, oracle_mod):
    run_golden(form, oracle_mod)


def run_golden(form, impl):
    g = json.load(open(GOLDEN))
    for case in g["cases"]:
        rw = case["decay"] == "rwkv6"
        chan = case["decay"] in ("channel", "rwkv6")
        S0 = np.array([[[_frac(x) for x in r] for r in case["S0"]]])
        steps = case["steps"]
        T = len(steps)
        dv, dk = S0.shape[1:]
        q = np.array([[[_frac(x) for x in s["q"]]] for s in steps])
        k = np.array([[[_frac(x) for x in s["k"]]] for s in steps])
        v = np.array([[[_frac(x) for x in s["v"]]] for s in steps])
        beta = np.array([[_frac(s["beta"])] for s in steps])
        if chan:
            a = np.array([[[_frac(x) for x in s["a"]]] for s in steps])
        else:
            a = np.array([[_frac(s["a"])] for s in steps])
        o_exp = np.array([[[_frac(x) for x in s["o"]]] for s in steps])
        S_exp = np.array([[[_frac(x) for x in r] for r in steps[-1]["S"]]])
        if form == "eager":
            o, S = impl.eager(S0, q, k, v, beta, a, chan, rw)
        elif form.startswith("deferred"):
            o, S = impl.deferred(S0, q, k, v, beta, a, chan, int(form[-1]), rw)
        else:
            o, S = oracle.brute_force(S0, q, k, v, beta, a, chan, rw)
        assert np.allclose(o, o_exp, rtol=0, atol=1e-14), (case["name"], form, o, o_exp)
        assert np.allclose(S, S_exp, rtol=0, atol=1e-14), (case["name"], form, S, S_exp)
        # every intermediate state as well (eager, one step at a time)
        if form == "eager":
            Sc = S0
            for t, s in enumerate(steps):
                _, Sc = impl.eager(Sc, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1], a[t:t + 1], chan, rw)
                exp = np.array([[[_frac(x) for x in r] for r in s["S"]]])
                assert np.allclose(Sc, exp, rtol=0, atol=1e-14), (case["name"], t)


# ------------------------------------------------------------------ P1

def check_p1(impl):
    rng = np.random.default_rng(11)
    for chan in (False, True):
        S0, q, k, v, _, _ = rand_case(rng, 3, 7, 8, 6, chan)
        beta = np.zeros((7, 3))
        a = np.ones((7, 3, 8)) if chan else np.ones((7, 3))
        for form in ("eager", 1, 3, 7):
            if form == "eager":
                o, S = impl.eager(S0, q, k, v, beta, a, chan)
            else:
                o, S = impl.deferred(S0, q, k, v, beta, a, chan, form)
            assert np.array_equal(S, S0)
            o_exp = np.einsum("hvk,thk->thv", S0, q)
            assert rel(o, o_exp) < 1e-14


def test_p1_identity_step(oracle_mod):
    check_p1(oracle_mod)


# ------------------------------------------------------------------ P2

def check_p2(impl):
    rng = np.random.default_rng(12)
    for chan in (False, True):
        NH, T, dk, dv = 2, 6, 16, 12
        S0, q, k, v, _, a = rand_case(rng, NH, T, dk, dv, chan)
        beta = np.ones((T, NH))
        S = S0
        for t in range(T):  # after every step S_t k_t = v_t
            _, S = impl.eager(S, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1], a[t:t + 1], chan)
            Sk = np.einsum("hvk,hk->hv", S, k[t])
            assert np.abs(Sk - v[t]).max() < 1e-13
        # the deferred read sees the same: with q_t = k_t the output is v_t
        for L in (1, 2, 4, 6):
            o, _ = impl.deferred(S0, k, k, v, beta, a, chan, L)
            assert np.abs(o - v).max() < 1e-13, L


def test_p2_unit_key_stores_value(oracle_mod):
    check_p2(oracle_mod)


# ------------------------------------------------------------------ P3

def check_p3(impl):
    rng = np.random.default_rng(13)
    for chan in (False, True):
        NH, T, dk, dv = 2, 9, 8, 5
        S0, q, k, v, _, a = rand_case(rng, NH, T, dk, dv, chan)
        beta = np.zeros((T, NH))
        decay = a if chan else np.repeat(a[:, :, None], dk, axis=2)
        cum = np.cumprod(decay, axis=0)  # [T, NH, dk]
        o_exp = np.einsum("hvk,thk,thk->thv", S0, cum, q)
        S_exp = S0 * cum[-1][:, None, :]
        for form in ("eager", 2, 4, 9):
            o, S = (impl.eager(S0, q, k, v, beta, a, chan) if form == "eager"
                    else impl.deferred(S0, q, k, v, beta, a, chan, form))
            assert rel(S, S_exp) < 1e-14 and rel(o, o_exp) < 1e-14, form


def test_p3_pure_decay_closed_form(oracle_mod):
    check_p3(oracle_mod)


# ------------------------------------------------------------------ P4

def check_p4(impl):
    rng = np.random.default_rng(14)
    for chan in (False, True):
        NH, n, dk, dv = 2, 5, 8, 6
        S0 = rng.standard_normal((NH, dv, dk))
        k = np.empty((n, NH, dk))
        for h in range(NH):
            Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
            k[:, h] = Q[:, :n].T
        q = rng.standard_normal((n, NH, dk))
        v = rng.standard_normal((n, NH, dv))
        beta = np.ones((n, NH))
        a = np.ones((n, NH, dk)) if chan else np.ones((n, NH))
        P = np.einsum("thk,thj->hkj", k, k)  # sum_i k_i k_i^T
        S_exp = np.einsum("hvk,hkj->hvj", S0, np.eye(dk)[None] - P) + np.einsum("thv,thk->hvk", v, k)
        for form in ("eager", 1, 2, 5):
            _, S = (impl.eager(S0, q, k, v, beta, a, chan) if form == "eager"
                    else impl.deferred(S0, q, k, v, beta, a, chan, form))
            assert rel(S, S_exp) < 1e-13, form


def test_p4_orthonormal_projection_closed_form(oracle_mod):
    check_p4(oracle_mod)


# ------------------------------------------------------------------ P5

def check_p5(impl):
    rng = np.random.default_rng(15)
    NH, T, dk, dv = 3, 8, 8, 4
    S0, q, k, v, beta, a = rand_case(rng, NH, T, dk, dv, False)
    a_vec = np.repeat(a[:, :, None], dk, axis=2)
    for form in ("eager", 3):
        r_head = (impl.eager(S0, q, k, v, beta, a, False) if form == "eager"
                  else impl.deferred(S0, q, k, v, beta, a, False, form))
        r_chan = (impl.eager(S0, q, k, v, beta, a_vec, True) if form == "eager"
                  else impl.deferred(S0, q, k, v, beta, a_vec, True, form))
        assert np.array_equal(r_head[0], r_chan[0]) and np.array_equal(r_head[1], r_chan[1])


def test_p5_channel_decay_with_equal_channels_is_head_decay(oracle_mod):
    check_p5(oracle_mod)


# ------------------------------------------------------------------ P6

def check_p6(impl):
    rng = np.random.default_rng(16)
    for chan in (False, True):
        NH, T, dk, dv = 3, 23, 16, 24
        S0, q, k, v, beta, a = rand_case(rng, NH, T, dk, dv, chan)
        o_e, S_e = impl.eager(S0, q, k, v, beta, a, chan)
        for L in (1, 2, 5, 8, 23, 40):
            o_d, S_d = impl.deferred(S0, q, k, v, beta, a, chan, L)
            tol = 1e-15 if L == 1 else 1e-12
            assert rel(o_d, o_e) < tol and rel(S_d, S_e) < tol, (chan, L, rel(o_d, o_e), rel(S_d, S_e))


def test_p6_deferred_equals_eager(oracle_mod):
    check_p6(oracle_mod)


def test_p6_generated_small_workload(oracle_mod):
    w = W.WORKLOADS["gdn_b1_h2_d64_t16"]
    x = W.generate(w)
    o_e, S_e = oracle.run_workload_heads(w, x, "eager")
    for L in w.L + (1, 5):
        o_d, S_d = oracle.run_workload_heads(w, x, "deferred", L)
        assert rel(o_d, o_e) < 1e-12 and rel(S_d, S_e) < 1e-12


# ------------------------------------------------------------------ P7

def check_p7(impl):
    rng = np.random.default_rng(17)
    for chan in (False, True):
        for (dk, dv) in ((4, 4), (5, 3), (3, 7), (8, 8)):
            NH, T = 2, 6
            S0, q, k, v, beta, a = rand_case(rng, NH, T, dk, dv, chan, unit_k=False)
            o_b, S_b = oracle.brute_force(S0, q, k, v, beta, a, chan)
            o_e, S_e = impl.eager(S0, q, k, v, beta, a, chan)
            assert rel(o_e, o_b) < 1e-13 and rel(S_e, S_b) < 1e-13, (chan, dk, dv)
            for L in (1, 2, 4, 6):
                o_d, S_d = impl.deferred(S0, q, k, v, beta, a, chan, L)
                assert rel(o_d, o_b) < 1e-12 and rel(S_d, S_b) < 1e-12, (chan, dk, dv, L)


def test_p7_brute_force_products(oracle_mod):
    check_p7(oracle_mod)


def test_p7_zero_decay_resets_state(oracle_mod):
    """a = 0 (full forgetting) makes S_t = beta v k^T regardless of history."""
    rng = np.random.default_rng(18)
    for chan in (False, True):
        S0, q, k, v, beta, _ = rand_case(rng, 2, 4, 6, 5, chan)
        a = np.zeros((4, 2, 6)) if chan else np.zeros((4, 2))
        o_b, S_b = oracle.brute_force(S0, q, k, v, beta, a, chan)
        assert np.allclose(S_b[1], beta[-1, 1] * np.outer(v[-1, 1], k[-1, 1]))
        for form in ("eager", 1, 3, 4):
            o, S = (oracle_mod.eager(S0, q, k, v, beta, a, chan) if form == "eager"
                    else oracle_mod.deferred(S0, q, k, v, beta, a, chan, form))
            assert np.abs(o - o_b).max() < 1e-13 and np.abs(S - S_b).max() < 1e-13


# ------------------------------------------------------------------ P8

def test_p8_window_identity():
    """The deferred closed form equals stepping the recurrence (dense products)."""
    rng = np.random.default_rng(19)
    dk, dv, n = 6, 4, 5
    Sbar = rng.standard_normal((dv, dk))
    ks = [rng.standard_normal(dk) for _ in range(n)]
    vs = [rng.standard_normal(dv) for _ in range(n)]
    betas = list(rng.uniform(0.1, 0.9, n))
    As = [rng.uniform(0.5, 1.0, dk) for _ in range(n)]
    S = Sbar.copy()
    for i in range(n):
        S = S @ np.diag(As[i]) @ (np.eye(dk) - betas[i] * np.outer(ks[i], ks[i])) + betas[i] * np.outer(vs[i], ks[i])
    assert rel(oracle.brute_force_window(Sbar, ks, vs, betas, As), S) < 1e-13


# ------------------------------------------------------------------ P9, P10 (RWKV6)

def check_p9(impl):
    rng = np.random.default_rng(20)
    for (dk, dv) in ((4, 4), (5, 3), (3, 7), (8, 8)):
        NH, T = 2, 7
        S0, q, k, v, _, a = rand_case(rng, NH, T, dk, dv, True, unit_k=False)
        o_b, S_b = oracle.brute_force(S0, q, k, v, None, a, True, rwkv6=True)
        o_e, S_e = impl.eager(S0, q, k, v, None, a, True, rwkv6=True)
        assert rel(o_e, o_b) < 1e-13 and rel(S_e, S_b) < 1e-13, (dk, dv)
        for L in (1, 2, 3, 7, 9):
            o_d, S_d = impl.deferred(S0, q, k, v, None, a, True, L, rwkv6=True)
            assert rel(o_d, o_b) < 1e-12 and rel(S_d, S_b) < 1e-12, (dk, dv, L)


def test_p9_rwkv6_brute_force(oracle_mod):
    check_p9(oracle_mod)


def rwkv6_closed_form(S0, q, k, v, a):
    """o_t and S_T from the unrolled sum (no step recursion):
    S_t = S_0 Diag(prod_{m<=t} a_m) + sum_{i<=t} v_i (k_i o prod_{i<m<=t} a_m)^T."""
    T = q.shape[0]
    o = np.zeros(v.shape)
    for t in range(T):
        cum = np.prod(a[:t + 1], axis=0)  # [NH, dk]
        S = S0 * cum[:, None, :]
        for i in range(t + 1):
            tail = np.prod(a[i + 1:t + 1], axis=0) if i < t else np.ones_like(cum)
            S = S + np.einsum("hv,hk->hvk", v[i], k[i] * tail)
        o[t] = np.einsum("hvk,hk->hv", S, q[t])
    return o, S


def check_p10(impl):
    rng = np.random.default_rng(21)
    NH, T, dk, dv = 2, 8, 6, 5
    S0, q, k, v, _, a = rand_case(rng, NH, T, dk, dv, True, unit_k=False)
    for aa in (a, np.ones_like(a), np.zeros_like(a)):
        o_c, S_c = rwkv6_closed_form(S0, q, k, v, aa)
        if aa is not a and aa.max() == 1.0:  # a = 1: plain linear attention
            assert rel(S_c, S0 + np.einsum("thv,thk->hvk", v, k)) < 1e-14
        if aa.max() == 0.0:  # a = 0: only the last outer product survives
            assert rel(S_c, np.einsum("hv,hk->hvk", v[-1], k[-1])) < 1e-14
        for form in ("eager", 1, 3, 8):
            o, S = (impl.eager(S0, q, k, v, None, aa, True, rwkv6=True) if form == "eager"
                    else impl.deferred(S0, q, k, v, None, aa, True, form, rwkv6=True))
            assert rel(o, o_c) < 1e-13 and rel(S, S_c) < 1e-13, form


def test_p10_rwkv6_closed_form(oracle_mod):
    check_p10(oracle_mod)


# ------------------------------------------------------------------ P11 (slot pool)

def check_p11():
    rng = np.random.default_rng(22)
    P, H, dk, dv, T = 4, 2, 6, 5, 9
    for chan, rw in ((False, False), (True, False), (True, True)):
        S_pool0 = rng.standard_normal((P, H, dv, dk))
        # two sequences: A lives in slot 2 for all steps; B in slot 0 for steps
        # 0..3, then a new sequence C takes slot 0 from its own initial state.
        S_C = rng.standard_normal((H, dv, dk))
        per_seq = {name: rand_case(rng, H, T, dk, dv, chan or rw) for name in "ABC"}
        steps, resets, rows = [], {5: {0: S_C}}, []
        for t in range(T):
            listed = [(2, "A")] + ([(0, "B")] if t < 4 else [(0, "C")] if t >= 5 else [])
            if t % 2:
                listed = listed[::-1]
            slot = np.array([s_ for s_, _ in listed])
            idx = {"q": 1, "k": 2, "v": 3, "beta": 4, "a": 5}
            steps.append((slot, *(np.stack([per_seq[n_][idx[key]][t] for _, n_ in listed])
                                  for key in ("q", "k", "v", "beta", "a"))))
            rows.append([n_ for _, n_ in listed])
        outs, S_fin = oracle.pool_eager(S_pool0, steps, chan, rw, resets)
        # each sequence alone
        def alone(S0, name, t0, t1):
            c = per_seq[name]
            sl = slice(t0, t1)
            return oracle.eager(S0, c[1][sl], c[2][sl], c[3][sl], c[4][sl], c[5][sl], chan, rw)
        oA, SA = alone(S_pool0[2], "A", 0, T)
        oB, SB = alone(S_pool0[0], "B", 0, 4)
        oC, SC = alone(S_C, "C", 5, T)
        for t in range(T):
            for j, name in enumerate(rows[t]):
                ref = {"A": lambda: oA[t], "B": lambda: oB[t], "C": lambda: oC[t - 5]}[name]()
                assert np.array_equal(outs[t][j], ref), (chan, rw, t, name)
        assert np.array_equal(S_fin[2], SA) and np.array_equal(S_fin[0], SC)
        assert np.array_equal(S_fin[1], S_pool0[1]) and np.array_equal(S_fin[3], S_pool0[3])  # never listed


def test_p11_slot_pool_is_per_sequence_recurrence(oracle_mod):
    check_p11()


# ------------------------------------------------------------------ P12 (int8 base)

def check_p12(impl):
    # Hand-worked rows whose fp32 arithmetic is exact, so that the expected
    # values can be checked by eye:
    # - max 127, scale 1: 62.5 -> 62 and -3.5 -> -4 (ties to even), 0.4 -> 0;
    # - an all-zero row stays zero;
    # - max 63.5, scale 0.5: 31.75 / 0.5 = 63.5 -> 64 (even), 15.875 -> 31.75 -> 32,
    #   0.25 -> 0.5 -> 0 (even);
    # - the code is decided in fp32, the kernel's precision: 62.50000001 is
    #   62.5 in fp32, a tie that goes to the even 62 (an fp64 decision gives 63).
    S = np.array([[[127.0, 62.5, -3.5, 0.4], [0.0, 0.0, 0.0, 0.0], [-63.5, 31.75, 15.875, 0.25],
                   [127.0, 62.50000001, 0.0, 0.0]]])
    exp = np.array([[[127.0, 62.0, -4.0, 0.0], [0.0, 0.0, 0.0, 0.0], [-63.5, 32.0, 16.0, 0.0],
                     [127.0, 62.0, 0.0, 0.0]]])
    got = impl.quantize_i8(S)
    assert np.array_equal(got, exp), got
    rng = np.random.default_rng(23)
    R = rng.standard_normal((3, 6, 8))
    once = impl.quantize_i8(R)
    # every value is code * scale with an integer code in [-127, 127] and the
    # row's fp32 scale max|row| / 127
    R32 = R.astype(np.float32)
    scale = np.abs(R32).max(axis=-1, keepdims=True) / np.float32(127)
    codes = once / scale.astype(np.float64)
    assert np.allclose(codes, np.round(codes), rtol=0, atol=1e-4) and np.abs(np.round(codes)).max() <= 127
    assert np.array_equal(once, (np.round(codes).astype(np.float32) * scale).astype(np.float64))
    # and it is the nearest such value to each fp32 input (at most half a step away)
    assert (np.abs(once - R32.astype(np.float64)) <= 0.5 * scale * (1 + 1e-6)).all()
    # rounding again moves a value by at most an fp32 rounding of its scale
    assert np.allclose(impl.quantize_i8(once), once, rtol=1e-6, atol=0)
    for chan, rw in ((False, False), (True, False), (True, True)):
        NH, T, dk, dv = 2, 9, 8, 6
        S0, q, k, v, beta, a = rand_case(rng, NH, T, dk, dv, chan or rw)
        # no merge before the end: eager from the rounded start, final state rounded
        o_e, S_e = impl.eager(impl.quantize_i8(S0), q, k, v, beta, a, chan, rw)
        o_d, S_d = impl.deferred(S0, q, k, v, beta, a, chan, T + 1, rw, base_i8=True)
        assert rel(o_d, o_e) < 1e-12 and rel(S_d, impl.quantize_i8(S_e)) < 1e-12, (chan, rw)
        # merges every L steps: window by window, the exact schedule then a rounding
        L = 3
        o_d, S_d = impl.deferred(S0, q, k, v, beta, a, chan, L, rw, base_i8=True)
        Sw = impl.quantize_i8(S0)
        for w0 in range(0, T, L):
            sl = slice(w0, w0 + L)
            ow, Sw = impl.deferred(Sw, q[sl], k[sl], v[sl], beta[sl], a[sl], chan, L, rw)
            assert rel(o_d[sl], ow) < 1e-12, (chan, rw, w0)
            Sw = impl.quantize_i8(Sw)
        assert rel(S_d, Sw) < 1e-12, (chan, rw)


def test_p12_int8_base(oracle_mod):
    check_p12(oracle_mod)


# ------------------------------------------------------------------ inputs

def test_generator_distributions():
    w = W.scaled(W.WORKLOADS["kda_b256_h32_d128_t512"], T=32)
    x = W.generate(w, heads=[0, 1, 8191])
    f = W.as_f64(w, x)
    assert np.allclose(np.linalg.norm(f["q"], axis=-1), 1, atol=1e-2)  # bf16-rounded unit vectors
    assert (f["a"] > 0).all() and (f["a"] <= 1).all()  # bf16 can round a to 1
    assert (f["beta"] > 0).all() and (f["beta"] < 1).all()
    assert 0.01 < f["S0"].std() < 0.03
    # a head generated alone equals the same head generated with others
    y = W.generate(w, heads=[8191])
    assert np.array_equal(y["k"][:, 0], x["k"][:, 2])


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -7 + 2 ** -9, -2.5], dtype=np.float32)
    back = W.bf16_to_f32(W.f32_to_bf16(vals))
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == np.float32(1 + 2 ** -6) and back[4] == -2.5
    assert back[3] == np.float32(1 + 2 ** -7)  # below the halfway point rounds down
