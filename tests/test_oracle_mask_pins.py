"""Pins for the oracle's per-head windows and document boundaries.

The masked oracle (oracle_attn_fwd_masked / oracle_attn_bwd_masked) follows two items of the
modded-nanogpt README's technique list: the long/short sliding-window pattern (here a window per
head) and training batches aligned to document ends with a maximum document length (here: a
token attends only inside its own document).  These tests fix it to facts from outside the code
under test: a brute-force recomputation with an explicit combined boolean mask, the fact that a
row packed with documents is exactly the separate causal attentions of those documents, closed
forms for one-token documents, and central finite differences of L = sum(O * dO).
"""
import numpy as np
import pytest

import workloads


def rng(shape, seed, n=4):
    r = np.random.default_rng(seed)
    return [r.standard_normal(shape) for _ in range(n)]


def combined_blocked(T, window, first):
    """True = blocked: future keys, keys at or before i - window, keys before the document start."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    m = j > i
    if window > 0:
        m = m | (j <= i - window)
    return m | (j < np.asarray(first)[:, None])


def brute(q, k, v, dO, scale, windows, doc_start):
    B, H, T, D = q.shape
    O = np.zeros_like(q); L = np.zeros((B, H, T)); dQ = np.zeros_like(q); dK = np.zeros_like(q)
    dV = np.zeros_like(q)
    for b in range(B):
        first = doc_start[b] if doc_start is not None else np.zeros(T, dtype=int)
        for h in range(H):
            S = scale * q[b, h] @ k[b, h].T
            S = np.where(combined_blocked(T, windows[h], first), -np.inf, S)
            m = S.max(-1, keepdims=True)
            e = np.exp(S - m)
            P = e / e.sum(-1, keepdims=True)
            O[b, h] = P @ v[b, h]
            L[b, h] = (m + np.log(e.sum(-1, keepdims=True)))[:, 0]
            dP = dO[b, h] @ v[b, h].T
            dS = P * (dP - (P * dP).sum(-1, keepdims=True))
            dV[b, h] = P.T @ dO[b, h]
            dQ[b, h] = scale * dS @ k[b, h]
            dK[b, h] = scale * dS.T @ q[b, h]
    return O, L, dQ, dK, dV


DOCS = [
    [[5, 9, 1, 30, 3], [40]],                 # row 0 packed, row 1 one document
    [[1] * 40, [2, 2, 36]],                   # one-token documents
    [[17, 23], [39, 1]],
]


@pytest.mark.parametrize("docs", DOCS)
@pytest.mark.parametrize("windows", [[0, 0, 0], [1, 4, 0], [7, 40, 3]])
def test_brute_force_with_combined_mask(oracle_mod, docs, windows):
    T, D, s = 40, 8, 0.4
    ds = np.stack([workloads.doc_starts_from_lengths(d, T) for d in docs])
    q, k, v, dO = rng((2, 3, T, D), seed=len(docs[0]) + sum(windows))
    o, lse = oracle_mod.attn_fwd_masked(q, k, v, s, windows, 0, ds)
    dq, dk, dv, _ = oracle_mod.attn_bwd_masked(q, k, v, dO, s, windows, 0, ds)
    O, L, dQ, dK, dV = brute(q, k, v, dO, s, windows, ds)
    for got, ref in ((o, O), (lse, L), (dq, dQ), (dk, dK), (dv, dV)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [0, 3, 11])
def test_packed_row_equals_separate_documents(oracle_mod, window):
    """A row of documents laid end to end is the concatenation of each document's own attention."""
    lengths, D, s = [7, 1, 19, 12, 25], 16, 0.25
    T = sum(lengths)
    ds = workloads.doc_starts_from_lengths(lengths, T)[None]
    q, k, v, dO = rng((1, 2, T, D), seed=window)
    o, lse = oracle_mod.attn_fwd_masked(q, k, v, s, None, window, ds)
    dq, dk, dv, _ = oracle_mod.attn_bwd_masked(q, k, v, dO, s, None, window, ds)
    pos = 0
    for n in lengths:
        sl = slice(pos, pos + n)
        ro, rl = oracle_mod.attn_fwd(q[:, :, sl], k[:, :, sl], v[:, :, sl], s, window)
        rq, rk, rv, _ = oracle_mod.attn_bwd(q[:, :, sl], k[:, :, sl], v[:, :, sl], dO[:, :, sl], s, window)
        np.testing.assert_allclose(o[:, :, sl], ro, atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[:, :, sl], rl, atol=1e-13, rtol=0)
        for a, b in ((dq, rq), (dk, rk), (dv, rv)):
            np.testing.assert_allclose(a[:, :, sl], b, atol=1e-13, rtol=0)
        pos += n


def test_per_head_windows_equal_one_call_per_head(oracle_mod):
    T, D, s, windows = 50, 8, 0.3, [1, 9, 0, 64]
    q, k, v, dO = rng((2, 4, T, D), seed=7)
    o, lse = oracle_mod.attn_fwd_masked(q, k, v, s, windows)
    dq, dk, dv, _ = oracle_mod.attn_bwd_masked(q, k, v, dO, s, windows)
    for h, w in enumerate(windows):
        ro, rl = oracle_mod.attn_fwd(q[:, h], k[:, h], v[:, h], s, w)
        rq, rk, rv, _ = oracle_mod.attn_bwd(q[:, h], k[:, h], v[:, h], dO[:, h], s, w)
        np.testing.assert_array_equal(o[:, h], ro)
        np.testing.assert_array_equal(lse[:, h], rl)
        np.testing.assert_array_equal(dq[:, h], rq)
        np.testing.assert_array_equal(dk[:, h], rk)
        np.testing.assert_array_equal(dv[:, h], rv)


def test_one_token_documents_copy_v(oracle_mod):
    """A token that is a document of its own sees only itself: O_i = V_i, lse_i = s q_i.k_i,
    and its dQ and dK vanish."""
    T, D, s = 30, 8, 0.5
    ds = np.arange(T)[None]
    q, k, v, dO = rng((1, 2, T, D), seed=3)
    o, lse = oracle_mod.attn_fwd_masked(q, k, v, s, None, 0, ds)
    dq, dk, dv, _ = oracle_mod.attn_bwd_masked(q, k, v, dO, s, None, 0, ds)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_allclose(lse, s * (q * k).sum(-1), atol=1e-14)
    np.testing.assert_array_equal(dv, dO)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0


def test_finite_differences_under_mask(oracle_mod):
    T, D, s, windows = 12, 4, 0.7, [3, 0]
    ds = workloads.doc_starts_from_lengths([5, 4, 3], T)[None]
    q, k, v, dO = rng((1, 2, T, D), seed=11)

    def loss(q_, k_, v_):
        o, _ = oracle_mod.attn_fwd_masked(q_, k_, v_, s, windows, 0, ds)
        return float((o * dO).sum())

    dq, dk, dv, _ = oracle_mod.attn_bwd_masked(q, k, v, dO, s, windows, 0, ds)
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        args = [q, k, v]
        num = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            num[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        err = np.linalg.norm(num - grad) / max(np.linalg.norm(grad), 1e-30)
        assert err <= 1e-6, (which, err)


def test_bad_document_starts_are_rejected(oracle_mod):
    q, k, v, _ = rng((1, 1, 6, 4), seed=1)
    with pytest.raises(RuntimeError):
        oracle_mod.attn_fwd_masked(q, k, v, 0.5, None, 0, np.array([[0, 0, 3, 3, 4, 4]]))   # 3 > 2
    with pytest.raises(RuntimeError):
        oracle_mod.attn_fwd_masked(q, k, v, 0.5, None, 0, np.array([[0, 0, 0, -1, 0, 0]]))


def test_document_start_recipe():
    ds = workloads.doc_starts_from_lengths([3, 1, 4], 10)
    assert ds.tolist() == [0, 0, 0, 3, 4, 4, 4, 4, 8, 8]
    rows = workloads.make_doc_starts(3, 500, seed=5, max_doc_len=64)
    assert rows.shape == (3, 500)
    for r in rows:
        i = np.arange(500)
        assert (r <= i).all() and (np.diff(r) >= 0).all()
        assert ((r == i) | (np.r_[0, r[:-1]] == r)).all()             # a document starts or continues
        starts = np.unique(r)
        assert (np.diff(np.r_[starts, 500]) <= 64).all()
