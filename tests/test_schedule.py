"""Host checks of the kernels' work decomposition (csrc/schedule.h), compiled for the CPU.

The header decides which K/V tiles each query tile visits (forward), which query tiles each
key tile visits (backward), the forward kernel's persistent item order and the backward
kernel's work units.  A tile the schedule skipped would silently drop terms of the softmax
sums or of the gradients, so these tests compare the decomposition with brute force over
every (query, key) position of small problems, and check that the persistent orders cover
each work item exactly once."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "causal_attention_sdpa_b200", "csrc")


@pytest.fixture(scope="module")
def S(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("sched") / "libschedule_host.so")
    subprocess.run([cxx, "-std=c++17", "-O1", "-shared", "-fPIC", "-I", CSRC,
                    os.path.join(ROOT, "tests", "schedule_host.cpp"), "-o", out], check=True)
    return ctypes.CDLL(out)


def key_range(S, qt, window):
    lo, hi = ctypes.c_int(), ctypes.c_int()
    S.sch_fwd_key_range(qt, window, ctypes.byref(lo), ctypes.byref(hi))
    return lo.value, hi.value


def visible(T, window):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    v = j <= i
    if window > 0:
        v &= j > i - window
    return v


CASES = [(T, W) for T in (1, 5, 127, 128, 129, 255, 256, 300, 640, 1024)
         for W in (0, 1, 2, 127, 128, 129, 200, 256, 1000, 5000)]


@pytest.mark.parametrize("T,W", CASES)
def test_forward_key_ranges_match_brute_force(S, T, W):
    K = S.sch_tile()
    n_tiles = -(-T // K)
    vis = visible(T, W)
    for qt in range(n_tiles):
        rows = vis[qt * K:(qt + 1) * K]
        needed = sorted({j // K for j in np.nonzero(rows.any(axis=0))[0]})
        lo, hi = key_range(S, qt, W)
        # every needed key tile is visited, and none outside [first needed, diagonal]
        assert needed and needed[0] == lo and needed[-1] == hi, (qt, lo, hi, needed)
        assert needed == list(range(lo, hi + 1))


@pytest.mark.parametrize("T,W", CASES)
def test_backward_query_ranges_match_brute_force(S, T, W):
    K = S.sch_tile()
    n_tiles = -(-T // K)
    vis = visible(T, W)
    for kt in range(n_tiles):
        cols = vis[:, kt * K:(kt + 1) * K]
        needed = sorted({i // K for i in np.nonzero(cols.any(axis=1))[0]})
        last = S.sch_bwd_last_query_tile(kt, n_tiles, W)
        assert needed == list(range(kt, last + 1)), (kt, last, needed)


@pytest.mark.parametrize("T,W,BH", [(1024, 0, 7), (1000, 0, 3), (8192, 1024, 5), (300, 129, 4)])
def test_backward_units_cover_every_visible_tile_pair_once(S, T, W, BH):
    K = S.sch_tile()
    n_tiles = -(-T // K)
    vis = visible(T, W)
    want = {(kt, qt) for kt in range(n_tiles) for qt in range(n_tiles)
            if vis[qt * K:(qt + 1) * K, kt * K:(kt + 1) * K].any()}
    seen = {}
    bh, kt, nq = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    for u in range(BH * n_tiles):
        S.sch_bwd_unit(u, n_tiles, W, ctypes.byref(bh), ctypes.byref(kt), ctypes.byref(nq))
        assert 0 <= bh.value < BH and 0 <= kt.value < n_tiles and nq.value >= 1
        for qt in range(kt.value, kt.value + nq.value):
            key = (bh.value, kt.value, qt)
            assert key not in seen
            seen[key] = u
    assert set(seen) == {(b, k, q) for b in range(BH) for (k, q) in want}


def fwd_schedule(S, sms, n_blocks, BH, persistent):
    hpw, waves = ctypes.c_int(), ctypes.c_int()
    S.sch_fwd_grid(sms, n_blocks, BH, int(persistent), ctypes.byref(hpw), ctypes.byref(waves))
    G = hpw.value * n_blocks
    items = {}
    per_cta = [[] for _ in range(G)]
    bh, qb = ctypes.c_int(), ctypes.c_int()
    for cta in range(G):
        for k in range(waves.value):
            S.sch_fwd_item(hpw.value, n_blocks, BH, cta, k, ctypes.byref(bh), ctypes.byref(qb))
            if bh.value < 0:
                continue
            key = (bh.value, qb.value)
            assert key not in items, f"item {key} scheduled twice"
            items[key] = (cta, k)
            per_cta[cta].append(qb.value)
    return G, items, per_cta


@pytest.mark.parametrize("sms,T,BH,persistent", [
    (148, 1024, 768, True), (148, 1024, 96, True), (148, 1024, 320, True), (148, 256, 6, True),
    (148, 8192, 24, False), (148, 8192, 24, True), (132, 2048, 50, True), (16, 40000, 3, True),
    (148, 1000, 1, True)])
def test_forward_items_scheduled_exactly_once(S, sms, T, BH, persistent):
    n_blocks = -(-(-(-T // 128)) // 2)
    G, items, per_cta = fwd_schedule(S, sms, n_blocks, BH, persistent)
    assert set(items) == {(b, q) for b in range(BH) for q in range(n_blocks)}
    if persistent:
        # at most one CTA per SM unless one head alone has more blocks than the GPU has SMs
        assert G <= max(sms, n_blocks)
    else:
        # one item per CTA
        assert G == BH * n_blocks and all(len(c) == 1 for c in per_cta)


def test_forward_persistent_order_balances_the_causal_triangle(S):
    # GPT-2 124M shape: 768 heads x 4 blocks on 148 SMs.  Block qb costs 4 qb + 3 tile-rounds;
    # the busiest CTA stays within one longest block of the mean.
    G, items, per_cta = fwd_schedule(S, 148, 4, 768, True)
    work = [sum(4 * qb + 3 for qb in c) for c in per_cta]
    mean = sum(work) / len(work)
    assert max(work) <= mean + 4 * 3 + 3
    # the blocks of one head run in the same wave (shared K/V tiles through L2)
    for b in range(768):
        assert len({items[(b, q)][1] for q in range(4)}) == 1


# ---------------------------------------------------------------------------------------------
# Per-head windows and document starts: the kernels derive tile ranges and mask decisions from
# each row's lower key bound (row_lower).  Brute force over every (query, key) pair of rows packed
# with random documents.
# ---------------------------------------------------------------------------------------------
def doc_visible(T, window, ds):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    v = (j <= i) & (j >= np.asarray(ds)[:, None])
    if window > 0:
        v &= j > i - window
    return v


def random_doc_starts(T, seed, max_len):
    import workloads
    return workloads.make_doc_starts(1, T, seed, max_len)[0]


DOC_CASES = [(T, W, L, seed) for T in (1, 100, 128, 300, 1000) for W in (0, 1, 64, 200)
             for L, seed in ((1, 0), (7, 1), (150, 2), (5000, 3))]


@pytest.mark.parametrize("T,W,L,seed", DOC_CASES)
def test_doc_masks_match_brute_force(S, T, W, L, seed):
    K = S.sch_tile()
    n_tiles = -(-T // K)
    ds = random_doc_starts(T, seed, L).astype(np.int32)
    vis = doc_visible(T, W, ds)
    lower = np.array([S.sch_row_lower(i, W, int(ds[i])) for i in range(T)])
    # each row's lower bound is exactly its first visible key
    assert (lower == vis.argmax(axis=1)).all()
    for qt in range(n_tiles):
        rows = vis[qt * K:(qt + 1) * K]
        needed = sorted({j // K for j in np.nonzero(rows.any(axis=0))[0]})
        lo, hi = ctypes.c_int(), ctypes.c_int()
        S.sch_fwd_key_range_lb(qt, int(lower[qt * K]), ctypes.byref(lo), ctypes.byref(hi))
        # the forward visits every needed key tile (extra tiles are masked to zero)
        assert set(needed) <= set(range(lo.value, hi.value + 1)), (qt, lo.value, hi.value, needed)
        last_lo = lower[min(qt * K + K - 1, T - 1)]
        for j in range(lo.value, hi.value + 1):
            full = rows[:, j * K:(j + 1) * K]
            cols = min(K, T - j * K)
            unmasked = not (j == qt or j * K < last_lo)
            if unmasked:   # a tile the kernels do not mask must be fully visible to every row
                assert full[:, :cols].all(), (qt, j)
    ptr = ds.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    for kt in range(n_tiles):
        cols = vis[:, kt * K:(kt + 1) * K]
        needed = sorted({i // K for i in np.nonzero(cols.any(axis=1))[0]})
        last = S.sch_bwd_last_query_tile_lb(kt, n_tiles, T, W, ptr)
        assert set(needed) <= set(range(kt, last + 1)), (kt, last, needed)
        assert not needed or needed[-1] == last, (kt, last, needed)
