"""Pins for the CPU oracle: checks against what the mathematics fixes.

Each ``pin_*`` function runs the oracle (optionally a different build of it,
given by ``library``) and raises AssertionError when its result contradicts
a hand-worked example, a closed form, an invariant or a special case of the
gated delta rule.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on deliberately broken copies of the
oracle source to show that each plausible mistake is caught.

The update being pinned (fused sigmoid-gating delta-rule decode step, vLLM PR
35777 summary, 实现拆解; sglang PR 18271):
    decay = exp(-exp(A_log) softplus(a + dt_bias)), beta = sigmoid(b)
    S <- decay S;  S <- S + k^ (beta (v - S^T k^))^T;  o = S^T q^
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

import oracle
from helpers import (BF16_NEG_INF, BF16_POS_INF, bf16, bf16_bits_to_f32, golden_arrays,
                     load_golden, random_problem)

L2 = oracle.L2NORM_QK
INTER = oracle.WRITE_INTERMEDIATE
NOFINAL = oracle.NO_FINAL_WRITEBACK


def _run(p, library=None, **kw):
    return oracle.update(p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"],
                         p["state_pool"], p["state_indices"], p.get("cu_seqlens"),
                         library=library, **kw)


# --------------------------------------------------------------------------
# Hand-worked examples (tests/golden)
# --------------------------------------------------------------------------

def _pin_golden(name, library):
    case = load_golden(name)
    p = golden_arrays(case)
    flags = INTER | (L2 if case["l2norm"] else 0)
    scale = None if case["l2norm"] else case["scale"]  # l2 case pins the default 1/sqrt(K)
    status, out, st, inter = _run(p, library, scale=scale, flags=flags)
    tol = case["tolerance_abs"]
    assert status == 0
    exp_out = np.array(case["expected_out"], dtype=np.float64)
    exp_inter = np.array(case["expected_inter"], dtype=np.float64)
    T = len(case["tokens"])
    np.testing.assert_allclose(out.reshape(T, -1), exp_out, rtol=0, atol=tol)
    np.testing.assert_allclose(inter.reshape(T, case["K"], case["V"]), exp_inter, rtol=0, atol=tol)
    np.testing.assert_allclose(st.reshape(case["K"], case["V"]), exp_inter[-1], rtol=0, atol=tol)


def pin_golden_decay_quarter(library=None):
    _pin_golden("k4v4_two_tokens_decay_quarter.json", library)


def pin_golden_l2norm_no_decay(library=None):
    _pin_golden("k4v4_l2norm_no_decay.json", library)


def golden_exact_rational(name):
    """Brute force of a golden case in exact rational arithmetic, with decay
    and beta taken as the exact values the case derives (1/4, 1/2).  Only
    used for the L2-off golden, whose every quantity is rational."""
    case = load_golden(name)
    assert not case["l2norm"]
    decay, beta, scale = Fraction(1, 4), Fraction(1, 2), Fraction(case["scale"])
    S = [[Fraction(x) for x in row] for row in case["state_in"]]
    outs, states = [], []
    for tok in case["tokens"]:
        k = [Fraction(x) for x in tok["k"]]
        q = [Fraction(x) * scale for x in tok["q"]]
        v = [Fraction(x) for x in tok["v"]]
        S = [[decay * x for x in row] for row in S]
        Stk = [sum(S[r][c] * k[r] for r in range(4)) for c in range(4)]
        d = [beta * (v[c] - Stk[c]) for c in range(4)]
        S = [[S[r][c] + k[r] * d[c] for c in range(4)] for r in range(4)]
        outs.append([sum(S[r][c] * q[r] for r in range(4)) for c in range(4)])
        states.append([row[:] for row in S])
    return outs, states


# --------------------------------------------------------------------------
# Special cases and closed forms
# --------------------------------------------------------------------------

def pin_gating_pattern(library=None):
    """Known gate values placed per (sequence, value head):
    a = -inf  -> softplus = 0 -> decay = 1;
    a = 1, dt_bias = -1 -> softplus(0) = ln 2 -> decay = 2^-exp(A_log):
        A_log = 0 -> 1/2, A_log = ln 2 -> 1/4;
    b = -inf -> beta = 0 (S' = decay S);  b = +inf -> beta = 1.
    With L2 off, k = e_j and q = e_m (one-hot), beta = 1 gives S'[j] = v and
    every other row decay*S[r]; o = scale * S'[m]."""
    rng = np.random.default_rng(11)
    N, H, HV, K, V = 6, 2, 4, 8, 8
    p = random_problem(rng, N=N, T=1, H=H, HV=HV, K=K, V=V)
    A_log = np.array([0.0, np.log(2.0), 0.0, np.log(2.0)], dtype=np.float32)
    p["A_log"] = A_log
    p["dt_bias"] = np.full(HV, -1.0, dtype=np.float32)
    a_is_one = (np.arange(N)[:, None] + np.arange(HV)[None, :]) % 2 == 0
    p["a"] = np.where(a_is_one, bf16(1.0), BF16_NEG_INF).astype(np.uint16)
    b_is_pos = (np.arange(N)[:, None] * 3 + np.arange(HV)[None, :]) % 3 == 0
    p["b"] = np.where(b_is_pos, BF16_POS_INF, BF16_NEG_INF).astype(np.uint16)
    jk = rng.integers(0, K, size=(N, H))
    jq = rng.integers(0, K, size=(N, H))
    q = np.zeros((N, H, K), dtype=np.float32)
    k = np.zeros((N, H, K), dtype=np.float32)
    for i in range(N):
        for h in range(H):
            k[i, h, jk[i, h]] = 1.0
            q[i, h, jq[i, h]] = 1.0
    p["q"], p["k"] = bf16(q), bf16(k)
    scale = 0.25
    status, out, st, _ = _run(p, library, scale=scale, flags=0)
    assert status == 0
    vals = {0.0: 0.5, float(np.float32(np.log(2.0))): 0.25}
    G = HV // H
    v = bf16_bits_to_f32(p["v"]).astype(np.float64)
    for i in range(N):
        slot = p["state_indices"][i]
        for hv in range(HV):
            h = hv // G
            c = vals[float(A_log[hv])] if a_is_one[i, hv] else 1.0
            S0 = p["state_pool"][slot, hv].astype(np.float64)
            S1 = st[slot, hv]
            expect = c * S0
            if b_is_pos[i, hv]:
                expect[jk[i, h]] = v[i, hv]
            # rtol covers ln 2 rounded to fp32 (decay off by 3e-9 relative)
            np.testing.assert_allclose(S1, expect, rtol=1e-8, atol=1e-14)
            np.testing.assert_allclose(out[i, hv], scale * expect[jq[i, h]], rtol=1e-8, atol=1e-14)


def pin_unit_k_recall(library=None):
    """g = 0 (A_log = -inf), beta = 1 (b = +inf), unit k: S'^T k = v.
    L2 off with k = e_j: exact up to one rounding; L2 on with k = 2 e_j:
    k^ = e_j / sqrt(1 + eps/4), so S'^T k^ = v within ~1e-6."""
    rng = np.random.default_rng(12)
    for l2, kval, tol in ((False, 1.0, 1e-14), (True, 2.0, 1e-5)):
        N, H, HV, K, V = 4, 1, 2, 8, 8
        p = random_problem(rng, N=N, T=1, H=H, HV=HV, K=K, V=V, state_scale=1.0)
        p["A_log"] = np.full(HV, -np.inf, dtype=np.float32)
        p["b"] = np.full((N, HV), BF16_POS_INF, dtype=np.uint16)
        j = rng.integers(0, K, size=N)
        k = np.zeros((N, H, K), dtype=np.float32)
        k[np.arange(N), 0, j] = kval
        p["k"] = bf16(k)
        status, out, st, _ = _run(p, library, flags=L2 if l2 else 0)
        assert status == 0
        v = bf16_bits_to_f32(p["v"]).astype(np.float64)
        for i in range(N):
            slot = p["state_indices"][i]
            khat = k[i, 0] / kval
            for hv in range(HV):
                recall = st[slot, hv].T @ khat
                np.testing.assert_allclose(recall, v[i, hv], rtol=tol, atol=tol)


def pin_no_decay_rows(library=None):
    """A_log = -inf gives decay 1: with L2 off and k = e_j only row j moves,
    every other row is bit-identical; b = 0 (beta = 1/2) gives row j =
    (S[j] + v) / 2."""
    rng = np.random.default_rng(13)
    N, H, HV, K, V = 5, 1, 2, 8, 8
    p = random_problem(rng, N=N, T=1, H=H, HV=HV, K=K, V=V, state_scale=1.0)
    p["A_log"] = np.full(HV, -np.inf, dtype=np.float32)
    p["b"] = np.zeros((N, HV), dtype=np.uint16)
    j = rng.integers(0, K, size=N)
    k = np.zeros((N, H, K), dtype=np.float32)
    k[np.arange(N), 0, j] = 1.0
    p["k"] = bf16(k)
    status, _, st, _ = _run(p, library, flags=0)
    assert status == 0
    v = bf16_bits_to_f32(p["v"]).astype(np.float64)
    for i in range(N):
        slot = p["state_indices"][i]
        for hv in range(HV):
            S0 = p["state_pool"][slot, hv].astype(np.float64)
            S1 = st[slot, hv]
            others = [r for r in range(K) if r != j[i]]
            assert np.array_equal(S1[others], S0[others])
            np.testing.assert_allclose(S1[j[i]], (S0[j[i]] + v[i, hv]) / 2, rtol=1e-14, atol=1e-14)


def pin_zero_state_one_token(library=None):
    """From S = 0, one token with L2 off and b = 0 (beta = 1/2):
    S' = (1/2) k v^T and o = (1/2) scale (k . q) v, whatever the decay."""
    rng = np.random.default_rng(14)
    N, H, HV, K, V = 3, 2, 4, 8, 8
    p = random_problem(rng, N=N, T=1, H=H, HV=HV, K=K, V=V)
    p["state_pool"][:] = 0
    p["b"] = np.zeros((N, HV), dtype=np.uint16)
    scale = 0.375
    status, out, st, _ = _run(p, library, scale=scale, flags=0)
    assert status == 0
    q = bf16_bits_to_f32(p["q"]).astype(np.float64)
    k = bf16_bits_to_f32(p["k"]).astype(np.float64)
    v = bf16_bits_to_f32(p["v"]).astype(np.float64)
    for i in range(N):
        slot = p["state_indices"][i]
        for hv in range(HV):
            h = hv // (HV // H)
            np.testing.assert_allclose(st[slot, hv], 0.5 * np.outer(k[i, h], v[i, hv]), rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(out[i, hv], 0.5 * scale * (k[i, h] @ q[i, h]) * v[i, hv], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

def pin_chain_equals_multi_token(library=None):
    """A T-token call equals T single-token calls that carry the state.
    In the fp32 twin the carried state is fp32 on both sides, so the two are
    bit-identical; in fp64 the single calls round the state to fp32 between
    tokens, so they agree to ~1e-7."""
    rng = np.random.default_rng(15)
    T, H, HV, K, V = 5, 2, 4, 8, 8
    p = random_problem(rng, N=3, T=T, H=H, HV=HV, K=K, V=V)
    for precision, tol in (("f32", 0.0), ("f64", 1e-6)):
        status, out_all, st_all, _ = _run(p, library, precision=precision)
        assert status == 0
        pool = p["state_pool"].copy()
        cu = p["cu_seqlens"]
        N = len(cu) - 1
        outs = []
        for t in range(T):
            tok = cu[:-1] + t
            step = dict(q=p["q"][tok], k=p["k"][tok], v=p["v"][tok], a=p["a"][tok], b=p["b"][tok],
                        A_log=p["A_log"], dt_bias=p["dt_bias"], state_pool=pool,
                        state_indices=p["state_indices"], cu_seqlens=np.arange(N + 1, dtype=np.int32))
            s, o, st, _ = _run(step, library, precision=precision)
            assert s == 0
            outs.append(o)
            pool = st.astype(np.float32)
        chained = np.stack(outs, axis=1).reshape(out_all.shape)
        if tol == 0.0:
            assert np.array_equal(chained, out_all)
            assert np.array_equal(pool, st_all)
        else:
            np.testing.assert_allclose(chained, out_all, rtol=tol, atol=tol)
            np.testing.assert_allclose(pool, st_all, rtol=0, atol=tol)


def pin_intermediate_prefix(library=None):
    """inter[bos_i + t] is the state after the first t+1 tokens of sequence i,
    i.e. the final state of the same call truncated to those tokens."""
    rng = np.random.default_rng(16)
    lens = [3, 1, 4, 2]
    p = random_problem(rng, lens=lens, H=2, HV=4, K=8, V=8, pad=(1,))
    status, out, st, inter = _run(p, library, flags=L2 | INTER)
    assert status == 0
    cu = p["cu_seqlens"]
    for i, L in enumerate(lens):
        slot = p["state_indices"][i]
        for t in range(L):
            rows = np.arange(cu[i], cu[i] + t + 1)
            sub = dict(q=p["q"][rows], k=p["k"][rows], v=p["v"][rows], a=p["a"][rows], b=p["b"][rows],
                       A_log=p["A_log"], dt_bias=p["dt_bias"], state_pool=p["state_pool"],
                       state_indices=np.array([slot], dtype=np.int32),
                       cu_seqlens=np.array([0, t + 1], dtype=np.int32))
            s, o, st_t, _ = _run(sub, library, flags=L2)
            assert s == 0
            if slot < 0:
                assert np.all(np.isnan(inter[cu[i] + t]))
                assert np.all(o == 0)
            else:
                assert np.array_equal(inter[cu[i] + t], st_t[slot])
                assert np.array_equal(out[cu[i] + t], o[t])


def pin_gqa_decomposition(library=None):
    """Value head hv reads key head hv // (HV/H) (value heads grouped
    contiguously under key heads, the `ba` reshape of vLLM PR 37975):
    a GQA call equals one single-head call per value head."""
    rng = np.random.default_rng(17)
    H, HV = 2, 6
    p = random_problem(rng, lens=[2, 3], H=H, HV=HV, K=8, V=8)
    status, out, st, _ = _run(p, library)
    assert status == 0
    G = HV // H
    for hv in range(HV):
        h = hv // G
        sub = dict(q=p["q"][:, h:h + 1], k=p["k"][:, h:h + 1], v=p["v"][:, hv:hv + 1],
                   a=p["a"][:, hv:hv + 1], b=p["b"][:, hv:hv + 1], A_log=p["A_log"][hv:hv + 1],
                   dt_bias=p["dt_bias"][hv:hv + 1],
                   state_pool=np.ascontiguousarray(p["state_pool"][:, hv:hv + 1]),
                   state_indices=p["state_indices"], cu_seqlens=p["cu_seqlens"])
        s, o, st1, _ = _run(sub, library)
        assert s == 0
        assert np.array_equal(o[:, 0], out[:, hv])
        assert np.array_equal(st1[:, 0], st[:, hv])


def pin_heads_independent(library=None):
    """Changing the inputs of one value head leaves every other head's output
    and state bit-identical."""
    rng = np.random.default_rng(18)
    p = random_problem(rng, lens=[2, 1, 3], H=2, HV=4, K=8, V=8)
    _, out0, st0, _ = _run(p, library)
    p2 = dict(p)
    p2["v"] = p["v"].copy()
    p2["v"][:, 3] ^= np.uint16(0x0040)
    p2["b"] = p["b"].copy()
    p2["b"][:, 3] ^= np.uint16(0x0020)
    _, out1, st1, _ = _run(p2, library)
    assert np.array_equal(out0[:, :3], out1[:, :3])
    assert np.array_equal(st0[:, :3], st1[:, :3])
    assert not np.array_equal(out0[:, 3], out1[:, 3])


def pin_slot_permutation(library=None):
    """Moving the states to other pool slots (and the indices with them)
    moves the results the same way, bit for bit."""
    rng = np.random.default_rng(19)
    p = random_problem(rng, lens=[1, 2, 2, 1], H=2, HV=4, K=8, V=8, num_slots=9, pad=(2,))
    _, out0, st0, _ = _run(p, library)
    perm = rng.permutation(9)            # new slot of old slot s is perm[s]
    pool = np.empty_like(p["state_pool"])
    pool[perm] = p["state_pool"]
    idx = np.where(p["state_indices"] >= 0, perm[np.maximum(p["state_indices"], 0)], -1).astype(np.int32)
    p2 = dict(p, state_pool=pool, state_indices=idx)
    _, out1, st1, _ = _run(p2, library)
    assert np.array_equal(out0, out1)
    assert np.array_equal(st1[perm], st0)


def pin_padding_and_untouched(library=None):
    """slot -1: output rows are exactly 0, no intermediate rows are written,
    and no pool slot changes; slots no index names are bit-identical."""
    rng = np.random.default_rng(20)
    p = random_problem(rng, lens=[2, 3, 1, 2], H=2, HV=4, K=8, V=8, num_slots=10, pad=(0, 2))
    status, out, st, inter = _run(p, library, flags=L2 | INTER)
    assert status == 0
    cu = p["cu_seqlens"]
    for i in (0, 2):
        rows = slice(cu[i], cu[i + 1])
        assert np.all(out[rows] == 0) and not np.any(np.signbit(out[rows]))
        assert np.all(np.isnan(inter[rows]))
    used = set(int(s) for s in p["state_indices"] if s >= 0)
    for s in range(10):
        if s not in used:
            assert np.array_equal(st[s], p["state_pool"][s].astype(np.float64))
    for i in (1, 3):
        rows = slice(cu[i], cu[i + 1])
        assert np.all(np.isfinite(out[rows])) and np.all(np.isfinite(inter[rows]))


def pin_invalid_and_empty(library=None):
    """A slot index >= num_slots or < -1 sets the bad-slot bit; a
    non-monotone cu_seqlens sets the bad-seqlens bit; either sequence is
    skipped whole.  A zero-length sequence touches nothing."""
    rng = np.random.default_rng(21)
    p = random_problem(rng, lens=[2, 0, 1, 2], H=1, HV=2, K=8, V=8, num_slots=8)
    status, out, st, _ = _run(p, library)
    assert status == 0
    assert np.array_equal(st[p["state_indices"][1]], p["state_pool"][p["state_indices"][1]].astype(np.float64))
    p2 = dict(p, state_indices=p["state_indices"].copy())
    p2["state_indices"][2] = 8
    p2["state_indices"][3] = -5
    status2, out2, st2, _ = _run(p2, library)
    assert status2 == oracle.BAD_SLOT
    cu = p["cu_seqlens"]
    assert np.all(np.isnan(out2[cu[2]:cu[4]]))
    assert np.array_equal(out2[cu[0]:cu[1]], out[cu[0]:cu[1]])
    p3 = dict(p, cu_seqlens=np.array([0, 2, 1, 3, 5], dtype=np.int32))
    status3, out3, _, _ = _run(p3, library)
    assert status3 & oracle.BAD_SEQLENS


def pin_no_final_writeback(library=None):
    """NO_FINAL_WRITEBACK leaves the pool as it was and changes no output."""
    rng = np.random.default_rng(22)
    p = random_problem(rng, lens=[3, 2], H=2, HV=4, K=8, V=8)
    _, out0, _, inter0 = _run(p, library, flags=L2 | INTER)
    _, out1, st1, inter1 = _run(p, library, flags=L2 | INTER | NOFINAL)
    assert np.array_equal(out0, out1) and np.array_equal(inter0, inter1)
    assert np.array_equal(st1, p["state_pool"].astype(np.float64))


def pin_softplus_large_argument(library=None):
    """Above x = 20 softplus returns x: a = 24, dt_bias = 1, A_log = 0 give
    decay = e^-25 exactly as exp(-25) rounds; b = -inf keeps only the decay."""
    rng = np.random.default_rng(23)
    p = random_problem(rng, N=2, T=1, H=1, HV=2, K=8, V=8)
    p["a"] = np.full((2, 2), bf16(24.0), dtype=np.uint16)
    p["dt_bias"] = np.ones(2, dtype=np.float32)
    p["A_log"] = np.zeros(2, dtype=np.float32)
    p["b"] = np.full((2, 2), BF16_NEG_INF, dtype=np.uint16)
    _, _, st, _ = _run(p, library)
    for i in range(2):
        s = p["state_indices"][i]
        np.testing.assert_allclose(st[s], np.exp(-25.0) * p["state_pool"][s].astype(np.float64), rtol=1e-15)


# --------------------------------------------------------------------------
# The unfused pair (gating alone; recurrence with given g, beta) and fp32 inputs
# --------------------------------------------------------------------------

def _pin_golden_given(name, g_value, library):
    """A golden case through the given-gates recurrence: g and beta passed
    as arrays with the values the case derives."""
    case = load_golden(name)
    p = golden_arrays(case)
    T = len(case["tokens"])
    g = np.full((T, 1), g_value, dtype=np.float32)
    beta = np.full((T, 1), 0.5, dtype=np.float32)
    flags = INTER | (L2 if case["l2norm"] else 0)
    scale = None if case["l2norm"] else case["scale"]
    status, out, st, inter = oracle.update(p["q"], p["k"], p["v"], None, None, None, None, p["state_pool"],
                                           p["state_indices"], None, scale=scale, flags=flags, g=g, beta=beta,
                                           library=library)
    assert status == 0
    tol = case["tolerance_abs"]
    np.testing.assert_allclose(out.reshape(T, -1), np.array(case["expected_out"]), rtol=0, atol=tol)
    np.testing.assert_allclose(inter.reshape(T, case["K"], case["V"]), np.array(case["expected_inter"]),
                               rtol=0, atol=tol)


def pin_given_gates_golden(library=None):
    """decay 1/4 is g = ln(1/4) (rounded to fp32: 4e-9 relative), beta 1/2;
    no decay is g = 0."""
    _pin_golden_given("k4v4_two_tokens_decay_quarter.json", np.log(0.25), library)
    _pin_golden_given("k4v4_l2norm_no_decay.json", 0.0, library)


def pin_gating_closed_forms(library=None):
    """softplus(0) = ln 2 (a = -dt_bias), softplus(2) = ln(1 + e^2),
    softplus(-inf) = 0, the threshold branch (x = 25), sigmoid(0) = 1/2,
    sigmoid(+-inf) = 1 / 0."""
    a = np.stack([bf16([1.0, 1.0, 24.0]), np.array([BF16_NEG_INF, bf16(1.0), bf16(1.0)], dtype=np.uint16)])
    b = np.stack([np.array([0, BF16_POS_INF, BF16_NEG_INF], dtype=np.uint16), bf16([0.0, 0.0, 0.0])])
    A_log = np.array([0.0, np.log(2.0), 0.0], dtype=np.float32)
    dt_bias = np.array([-1.0, -1.0, 1.0], dtype=np.float32)
    g, beta = oracle.gating(a, b, A_log, dt_bias, library=library)
    e2 = float(np.exp(np.float64(np.float32(np.log(2.0)))))
    np.testing.assert_allclose(g[0], [-np.log(2.0), -e2 * np.log(2.0), -25.0], rtol=1e-15)
    assert g[1, 0] == 0.0
    np.testing.assert_allclose(g[1, 1:], [-e2 * np.log(2.0), -np.log(1.0 + np.e ** 2)], rtol=1e-15)
    assert list(beta[0]) == [0.5, 1.0, 0.0] and list(beta[1]) == [0.5, 0.5, 0.5]


def pin_fused_equals_gating_then_given(library=None):
    """The fused update equals the unfused pair: gates from the gating step
    (rounded to fp32, as the pair stores them), then the recurrence with
    given gates."""
    rng = np.random.default_rng(24)
    p = random_problem(rng, lens=[3, 1, 4], H=2, HV=4, K=8, V=8, pad=(1,))
    _, o_f, s_f, i_f = _run(p, library, flags=L2 | INTER)
    g, beta = oracle.gating(p["a"], p["b"], p["A_log"], p["dt_bias"], library=library)
    status, o_u, s_u, i_u = oracle.update(p["q"], p["k"], p["v"], None, None, None, None, p["state_pool"],
                                          p["state_indices"], p["cu_seqlens"], flags=L2 | INTER,
                                          g=g.astype(np.float32), beta=beta.astype(np.float32), library=library)
    assert status == 0
    np.testing.assert_allclose(o_u, o_f, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(s_u, s_f, rtol=1e-5, atol=1e-6)
    assert np.array_equal(np.isnan(i_u), np.isnan(i_f))


def pin_fp32_inputs_equal_bf16_inputs(library=None):
    """The same values given as fp32 instead of bf16 patterns give the same
    bits (the arithmetic is fp64 either way)."""
    rng = np.random.default_rng(25)
    p = random_problem(rng, lens=[2, 3], H=2, HV=4, K=8, V=8)
    ref = _run(p, library, flags=L2 | INTER)
    pf = dict(p)
    for n in ("q", "k", "v", "a", "b"):
        pf[n] = bf16_bits_to_f32(p[n])
    got = _run(pf, library, flags=L2 | INTER)
    for x, y in zip(ref[1:], got[1:]):
        assert np.array_equal(x, y, equal_nan=True)
    g1, b1 = oracle.gating(p["a"], p["b"], p["A_log"], p["dt_bias"], library=library)
    g2, b2 = oracle.gating(pf["a"], pf["b"], p["A_log"], p["dt_bias"], library=library)
    assert np.array_equal(g1, g2) and np.array_equal(b1, b2)
    # fp32 values that are not bf16 values go through unrounded
    pf["v"] = pf["v"] + np.float32(1.0 / 3.0)
    _, o3, _, _ = _run(pf, library, flags=L2 | INTER)
    assert not np.array_equal(o3, got[1])


ALL_PINS = [
    pin_golden_decay_quarter, pin_golden_l2norm_no_decay, pin_gating_pattern,
    pin_unit_k_recall, pin_no_decay_rows, pin_zero_state_one_token,
    pin_chain_equals_multi_token, pin_intermediate_prefix, pin_gqa_decomposition,
    pin_heads_independent, pin_slot_permutation, pin_padding_and_untouched,
    pin_invalid_and_empty, pin_no_final_writeback, pin_softplus_large_argument,
    pin_given_gates_golden, pin_gating_closed_forms, pin_fused_equals_gating_then_given,
    pin_fp32_inputs_equal_bf16_inputs,
]
