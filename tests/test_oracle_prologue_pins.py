"""Pins for the oracle's QK-Norm + rotary prologue (the step before attention in the modded-nanogpt
README's "modernised architecture" item, and the RoPE exercise of "Un GPT desde cero + nanoGPT").

Fixed against facts from outside the code: a rotation is a complex multiplication, so each
half-split pair (n_i, n_{i+D/2}) read as n_i + 1j n_{i+D/2} must come out multiplied by
exp(1j t base^(-2i/D)) (numpy's complex arithmetic, an independent routine); rows come out with
unit norm; token 0 is not rotated; scores of rotated rows depend only on the distance between
positions; a positive rescaling of the input changes nothing; and the gradient matches central
finite differences and is orthogonal to the input row."""
import numpy as np
import pytest


def rng(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("D", [8, 64, 128])
def test_prologue_is_normalise_then_complex_rotation(oracle_mod, D):
    T, base = 50, 10000.0
    x = rng((2, T, D), D)
    y = oracle_mod.qk_prologue_fwd(x, True, base)
    n = x / np.linalg.norm(x, axis=-1, keepdims=True)
    z = n[..., :D // 2] + 1j * n[..., D // 2:]
    ang = np.arange(T)[:, None] * base ** (-2.0 * np.arange(D // 2) / D)[None, :]
    w = z * np.exp(1j * ang)
    np.testing.assert_allclose(y, np.concatenate([w.real, w.imag], axis=-1), atol=1e-13)


def test_prologue_invariants(oracle_mod):
    T, D = 64, 64
    x = rng((3, T, D), 1)
    y = oracle_mod.qk_prologue_fwd(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-13)          # unit rows
    np.testing.assert_allclose(y[:, 0], x[:, 0] / np.linalg.norm(x[:, 0], axis=-1, keepdims=True),
                               atol=1e-14)                                              # token 0
    np.testing.assert_allclose(oracle_mod.qk_prologue_fwd(3.7 * x), y, atol=1e-13)      # scale-free
    np.testing.assert_allclose(oracle_mod.qk_prologue_fwd(x, norm=False, rope_base=0), x, atol=0)
    # relative position: the same raw q, k at positions (t, s) and (t + d, s + d) give one score
    q, k = rng((D,), 2), rng((D,), 3)
    xs = np.zeros((1, T, D))
    xs[0, 5], xs[0, 9], xs[0, 25], xs[0, 29] = q, k, q, k
    yy = oracle_mod.qk_prologue_fwd(xs)
    assert abs(yy[0, 9] @ yy[0, 5] - yy[0, 29] @ yy[0, 25]) < 1e-12


@pytest.mark.parametrize("norm,base", [(True, 10000.0), (False, 10000.0), (True, 0.0)])
def test_prologue_gradient_matches_finite_differences(oracle_mod, norm, base):
    T, D = 6, 8
    x, dy = rng((2, T, D), 4), rng((2, T, D), 5)
    dx = oracle_mod.qk_prologue_bwd(x, dy, norm, base)
    h = 1e-6
    num = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        num[idx] = ((oracle_mod.qk_prologue_fwd(xp, norm, base) - oracle_mod.qk_prologue_fwd(xm, norm, base)) * dy
                    ).sum() / (2 * h)
    assert np.linalg.norm(num - dx) / np.linalg.norm(dx) <= 1e-7
    if norm:
        np.testing.assert_allclose((dx * x).sum(-1), 0.0, atol=1e-12)                  # orthogonal to x
