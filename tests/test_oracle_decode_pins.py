"""Pins for the oracle's decode function (one new query against a key/value cache, the inner
step of the generation loop of "Un GPT desde cero + nanoGPT", Laboratorio L2.1).

Decode must equal the last row of the full causal forward over the sequence so far: the
generation loop reruns the model on the whole prefix and keeps the last position.  The tests
check exactly that against the already pinned forward oracle, plus closed forms (one cached
token gives O = V_0; equal keys give the mean of the visible values), the window rule, and
lengths past the cache or at zero."""
import numpy as np
import pytest


def rng(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("window", [0, 1, 5, 100])
def test_decode_is_last_row_of_causal_forward(oracle_mod, window):
    B, H, T, D, s = 3, 2, 40, 16, 0.3
    lens = [40, 17, 1]
    k, v = rng((B, H, T, D), 1), rng((B, H, T, D), 2)
    q = rng((B, H, D), 3)
    o, lse = oracle_mod.attn_decode(q, k, v, lens, s, window)
    for b, L in enumerate(lens):
        qf = np.zeros((1, H, L, D))
        qf[0, :, L - 1] = q[b]
        fo, fl = oracle_mod.attn_fwd(qf, k[b:b + 1, :, :L], v[b:b + 1, :, :L], s, window)
        np.testing.assert_allclose(o[b], fo[0, :, L - 1], atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[b], fl[0, :, L - 1], atol=1e-13, rtol=0)


def test_decode_closed_forms(oracle_mod):
    B, H, T, D = 2, 3, 10, 8
    k, v, q = rng((B, H, T, D), 4), rng((B, H, T, D), 5), rng((B, H, D), 6)
    o, lse = oracle_mod.attn_decode(q, k, v, [1, 1], 0.5)
    np.testing.assert_array_equal(o, v[:, :, 0])
    np.testing.assert_allclose(lse, 0.5 * (q * k[:, :, 0]).sum(-1), atol=1e-14)
    k_eq = np.repeat(k[:, :, :1], T, axis=2)            # every key the same: uniform weights
    o, lse = oracle_mod.attn_decode(q, k_eq, v, [10, 6], 0.5, window=4)
    np.testing.assert_allclose(o[0], v[0, :, 6:10].mean(axis=1), atol=1e-13)
    np.testing.assert_allclose(o[1], v[1, :, 2:6].mean(axis=1), atol=1e-13)
    np.testing.assert_allclose(lse[0], 0.5 * (q[0] * k[0, :, 0]).sum(-1) + np.log(4), atol=1e-13)


def test_decode_length_limits(oracle_mod):
    B, H, T, D = 2, 1, 6, 4
    k, v, q = rng((B, H, T, D), 7), rng((B, H, T, D), 8), rng((B, H, D), 9)
    o, lse = oracle_mod.attn_decode(q, k, v, [0, 99], 1.0)
    assert (o[0] == 0).all() and np.isneginf(lse[0]).all()                 # nothing cached
    o_full, l_full = oracle_mod.attn_decode(q, k, v, [0, 6], 1.0)           # lengths clamp to the cache
    np.testing.assert_array_equal(o[1], o_full[1])
    np.testing.assert_array_equal(lse[1], l_full[1])
