"""Pins for the fp64 CPU oracle, against facts that do not come from the oracle.

Each test fixes the oracle to something other than itself: a brute-force
matrix-form recomputation with an explicit boolean mask, closed forms (row 0,
window 1, uniform scores), a hand-worked example, invariants of the softmax
(row sums, causality, shift invariance, gradient identities) and central
finite differences of L = sum(O * dO).

The definition being pinned: "NanoGPT Speedrun baseline", section "El
Mecanismo de Atencion" (softmax(QK^T / sqrt(d_k)) V, Attn_ij = 0 for j > i),
the boolean triu(diagonal=1) mask of "Un GPT desde cero + nanoGPT",
Laboratorio L2.1 (True = blocked), and the sliding-window item of the
modded-nanogpt README's technique list.
"""
import json
import math
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rng_inputs(NH, T, D, seed, n=4):
    r = np.random.default_rng(seed)
    return [r.standard_normal((NH, T, D)) for _ in range(n)]


# --------------------------------------------------------------------------
# Brute force: explicit T x T scores, explicit boolean mask, explicit softmax.
# --------------------------------------------------------------------------
def blocked_mask(T, window):
    """True = blocked: future keys (triu, diagonal=1) and, with a window W,
    keys at or before i - W."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    m = j > i
    if window > 0:
        m = m | (j <= i - window)
    return m


def brute_fwd(q, k, v, scale, window):
    T = q.shape[-2]
    S = scale * np.einsum("hid,hjd->hij", q, k)
    S = np.where(blocked_mask(T, window)[None], -np.inf, S)
    m = S.max(axis=-1, keepdims=True)
    e = np.exp(S - m)
    P = e / e.sum(axis=-1, keepdims=True)
    lse = (m + np.log(e.sum(axis=-1, keepdims=True)))[..., 0]
    return P @ v, lse, P


def brute_bwd(q, k, v, dO, scale, window):
    _, _, P = brute_fwd(q, k, v, scale, window)
    dV = np.swapaxes(P, -1, -2) @ dO
    dP = dO @ np.swapaxes(v, -1, -2)
    delta = (P * dP).sum(-1)
    dS = P * (dP - delta[..., None])
    dQ = scale * dS @ k
    dK = scale * np.swapaxes(dS, -1, -2) @ q
    return dQ, dK, dV, delta


CASES = [(T, D, W) for T in (1, 2, 5, 17, 64) for D in (4, 64) for W in (0, 1, 3, 8)]


@pytest.mark.parametrize("T,D,W", CASES)
def test_fwd_matches_bruteforce(oracle_mod, T, D, W):
    q, k, v, _ = rng_inputs(2, T, D, seed=T * 100 + D + W)
    o, lse = oracle_mod.attn_fwd(q, k, v, 1 / math.sqrt(D), W)
    ob, lseb, _ = brute_fwd(q, k, v, 1 / math.sqrt(D), W)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lseb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,D,W", CASES)
def test_bwd_matches_bruteforce(oracle_mod, T, D, W):
    q, k, v, do = rng_inputs(2, T, D, seed=T * 100 + D + W + 7)
    s = 1 / math.sqrt(D)
    got = oracle_mod.attn_bwd(q, k, v, do, s, W)
    ref = brute_bwd(q, k, v, do, s, W)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-11)


# --------------------------------------------------------------------------
# Probabilities read out with V = identity (T <= D makes O equal to P).
# --------------------------------------------------------------------------
@pytest.mark.parametrize("W", [0, 1, 3, 8])
def test_rows_are_probabilities(oracle_mod, W):
    T, D = 24, 32
    q, k, _, _ = rng_inputs(3, T, D, seed=11 + W)
    v = np.zeros((3, T, D))
    v[:, np.arange(T), np.arange(T)] = 1.0     # V_j = e_j  =>  O_ij = P_ij
    P, _ = oracle_mod.attn_fwd(q, k, v, 0.3, W)
    P = P[..., :T]
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (P >= 0).all()
    blocked = blocked_mask(T, W)
    assert (P[:, blocked] == 0.0).all(), "a blocked key received probability"
    assert (P[:, ~blocked] > 0.0).all(), "a visible key received no probability"


# --------------------------------------------------------------------------
# Closed forms.
# --------------------------------------------------------------------------
def test_row0_is_v0(oracle_mod):
    q, k, v, _ = rng_inputs(4, 33, 16, seed=5)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.125, 0)
    assert np.array_equal(o[:, 0], v[:, 0]), "query 0 sees only key 0, so O_0 = V_0 exactly"
    np.testing.assert_allclose(lse[:, 0], 0.125 * (q[:, 0] * k[:, 0]).sum(-1), rtol=0, atol=1e-13)


def test_window_one_is_identity(oracle_mod):
    q, k, v, _ = rng_inputs(2, 40, 8, seed=6)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.7, 1)
    assert np.array_equal(o, v), "with window 1 each query sees only itself"
    np.testing.assert_allclose(lse, 0.7 * (q * k).sum(-1), rtol=0, atol=1e-13)


@pytest.mark.parametrize("W", [0, 1, 5, 100])
def test_zero_query_gives_prefix_means(oracle_mod, W):
    T, D = 50, 8
    _, k, v, _ = rng_inputs(2, T, D, seed=7)
    q = np.zeros_like(k)               # every visible score is 0: uniform weights
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.125, W)
    for i in range(T):
        lo = 0 if W <= 0 else max(0, i - W + 1)
        np.testing.assert_allclose(o[:, i], v[:, lo:i + 1].mean(axis=1), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, i], math.log(i + 1 - lo), rtol=0, atol=1e-13)


def test_equal_keys_give_prefix_means(oracle_mod):
    T, D = 30, 8
    q, k, v, _ = rng_inputs(1, T, D, seed=8)
    k[:] = k[:, :1]                    # all key rows equal: scores constant along each row
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.125, 0)
    for i in range(T):
        np.testing.assert_allclose(o[0, i], v[0, :i + 1].mean(axis=0), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, i], 0.125 * q[0, i] @ k[0, 0] + math.log(i + 1),
                                   rtol=0, atol=1e-13)


def test_worked_example(oracle_mod):
    """Hand-worked 3-token example (tests/golden/worked_example.json)."""
    with open(os.path.join(HERE, "golden", "worked_example.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        q, k, v = (np.array(c[n], dtype=np.float64)[None] for n in ("q", "k", "v"))
        o, lse = oracle_mod.attn_fwd(q, k, v, c["scale"], c["window"])
        np.testing.assert_allclose(o[0], np.array(c["o"]), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0], np.array(c["lse"]), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Invariants.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("W", [0, 4])
def test_causality(oracle_mod, W):
    T, D, i0 = 20, 8, 11
    q, k, v, do = rng_inputs(2, T, D, seed=9)
    s = 0.35
    o, lse = oracle_mod.attn_fwd(q, k, v, s, W)
    dq, dk, dv, _ = oracle_mod.attn_bwd(q, k, v, do, s, W)
    k2, v2 = k.copy(), v.copy()
    k2[:, i0 + 1:] += 3.0
    v2[:, i0 + 1:] -= 2.0
    o2, lse2 = oracle_mod.attn_fwd(q, k2, v2, s, W)
    dq2, _, _, _ = oracle_mod.attn_bwd(q, k2, v2, do, s, W)
    assert np.array_equal(o[:, :i0 + 1], o2[:, :i0 + 1])
    assert np.array_equal(lse[:, :i0 + 1], lse2[:, :i0 + 1])
    assert np.array_equal(dq[:, :i0 + 1], dq2[:, :i0 + 1])
    # the last key is seen by the last query alone
    _, _, P = brute_fwd(q, k, v, s, W)
    np.testing.assert_allclose(dv[:, -1], P[:, -1, -1, None] * do[:, -1], rtol=0, atol=1e-13)
    assert np.abs(dk[:, -1]).max() > 0


@pytest.mark.parametrize("W", [0, 3])
def test_gradient_identities(oracle_mod, W):
    T, D = 33, 16
    q, k, v, do = rng_inputs(3, T, D, seed=10)
    s = 0.25
    o, _ = oracle_mod.attn_fwd(q, k, v, s, W)
    dq, dk, dv, delta = oracle_mod.attn_bwd(q, k, v, do, s, W)
    # softmax is invariant to a common shift of all keys: the key gradients sum to 0
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, rtol=0, atol=1e-12)
    # rows of P sum to one: the value gradients sum to the output gradients
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), rtol=0, atol=1e-12)
    # Delta computed as sum_j P_ij dP_ij equals the row dot dO_i . O_i
    np.testing.assert_allclose(delta, (do * o).sum(-1), rtol=0, atol=1e-12)


def test_shift_invariance(oracle_mod):
    T, D = 26, 8
    q, k, v, do = rng_inputs(2, T, D, seed=12)
    s = 0.4
    c = np.random.default_rng(1).standard_normal(D)
    o, lse = oracle_mod.attn_fwd(q, k, v, s, 0)
    g = oracle_mod.attn_bwd(q, k, v, do, s, 0)
    o2, lse2 = oracle_mod.attn_fwd(q, k + c, v, s, 0)
    g2 = oracle_mod.attn_bwd(q, k + c, v, do, s, 0)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2 - lse, s * (q @ c), rtol=0, atol=1e-12)
    for a, b in zip(g[:3], g2[:3]):
        np.testing.assert_allclose(b, a, rtol=0, atol=1e-11)


def test_thread_count_does_not_change_results(oracle_mod):
    q, k, v, do = rng_inputs(7, 40, 16, seed=13)
    a = oracle_mod.attn_bwd(q, k, v, do, 0.25, 0, nthreads=1)
    b = oracle_mod.attn_bwd(q, k, v, do, 0.25, 0, nthreads=4)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# --------------------------------------------------------------------------
# Central finite differences of L = sum(O * dO).
# --------------------------------------------------------------------------
@pytest.mark.parametrize("D", [4, 8, 64])
@pytest.mark.parametrize("W", [0, 3])
def test_finite_differences(oracle_mod, D, W):
    NH, T = 2, (16 if D < 64 else 9)
    q, k, v, do = rng_inputs(NH, T, D, seed=100 + D + W)
    s = 1 / math.sqrt(D)
    dq, dk, dv, _ = oracle_mod.attn_bwd(q, k, v, do, s, W)
    h = 1e-6

    def loss(qq, kk, vv):
        o, _ = oracle_mod.attn_fwd(qq, kk, vv, s, W)
        return float((o * do).sum())

    for which, ana in ((0, dq), (1, dk), (2, dv)):
        num = np.zeros_like(ana)
        args = [q, k, v]
        for idx in np.ndindex(*ana.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            num[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        rel = np.linalg.norm(num - ana) / np.linalg.norm(ana)
        assert rel <= 1e-6, f"operand {which}: relative error {rel:.3e}"
        assert np.abs(num - ana).max() <= 1e-6 * max(1.0, np.abs(ana).max())


def test_bad_arguments_rejected(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.attn_fwd(np.zeros((2, 3)), np.zeros((2, 4)), np.zeros((2, 3)), 1.0)


def test_empty_inputs(oracle_mod):
    z = np.zeros((2, 0, 8))
    o, lse = oracle_mod.attn_fwd(z, z, z, 1.0)
    assert o.shape == (2, 0, 8) and lse.shape == (2, 0)
