"""Host checks of the kernels' work decomposition (csrc/schedule.h), compiled for the CPU.

The header decides which K/V tiles each query tile visits (forward), which query tiles each
key tile visits (backward), and the list order in which the work items of both passes go to
the SMs.  A tile the schedule skipped would silently drop terms of the softmax sums or of the
gradients, so these tests compare the decomposition with brute force over every (query, key)
position of small problems, and check that the list orders hold each work item exactly once."""
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


@pytest.mark.parametrize("T,W,BH,tail", [(1024, 0, 7, 0), (1000, 0, 3, 2), (8192, 1024, 5, 5), (300, 129, 4, 3),
                                          (1024, 0, 13, 4)])
def test_backward_units_cover_every_visible_tile_pair_once(S, T, W, BH, tail):
    K = S.sch_tile()
    n_tiles = -(-T // K)
    vis = visible(T, W)
    want = {(kt, qt) for kt in range(n_tiles) for qt in range(n_tiles)
            if vis[qt * K:(qt + 1) * K, kt * K:(kt + 1) * K].any()}
    seen = {}
    bh, kt, nq = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    for u in range(BH * n_tiles):
        S.sch_bwd_unit(u, BH, n_tiles, tail, W, ctypes.byref(bh), ctypes.byref(kt), ctypes.byref(nq))
        assert 0 <= bh.value < BH and 0 <= kt.value < n_tiles and nq.value >= 1
        for qt in range(kt.value, kt.value + nq.value):
            key = (bh.value, kt.value, qt)
            assert key not in seen
            seen[key] = u
    assert set(seen) == {(b, k, q) for b in range(BH) for (k, q) in want}


def list_order(S, BH, n_cls, tail):
    bh, cls = ctypes.c_int(), ctypes.c_int()
    out = []
    for i in range(BH * n_cls):
        S.sch_list_item(i, BH, n_cls, tail, ctypes.byref(bh), ctypes.byref(cls))
        out.append((bh.value, cls.value))
    return out


@pytest.mark.parametrize("BH,n_cls,tail", [(1, 1, 0), (1, 8, 1), (7, 4, 0), (7, 4, 2), (7, 4, 7), (768, 4, 74),
                                           (192, 8, 37), (24, 32, 10), (5, 3, 4), (100, 1, 100)])
def test_list_order(S, BH, n_cls, tail):
    items = list_order(S, BH, n_cls, tail)
    # every (head, class) exactly once
    assert sorted(items) == [(b, c) for b in range(BH) for c in range(n_cls)]
    # head-major (each head's classes in order, longest first) up to the last `tail` heads, which
    # go class-major
    head = BH - tail
    assert items[:head * n_cls] == [(b, c) for b in range(head) for c in range(n_cls)]
    assert items[head * n_cls:] == [(b, c) for c in range(n_cls) for b in range(head, BH)]


def test_tail_holds_two_items_per_sm(S):
    for sms in (148, 132, 16):
        for BH in (1, 7, 96, 768, 5000):
            for n_cls in (1, 4, 8, 32, 300):
                t = S.sch_tail_heads(BH, n_cls, sms)
                assert 0 <= t <= BH
                assert t == BH or (t * n_cls >= 2 * sms and (t - 1) * n_cls < 2 * sms)


def list_makespan(sizes, sms=148):
    """Greedy list scheduling: each SM takes the next item of the list when it is free."""
    import heapq
    free = [0.0] * sms
    for w in sizes:
        t = heapq.heappop(free)
        heapq.heappush(free, t + w)
    return max(free)


@pytest.mark.parametrize("B,H,T", [(64, 12, 1024), (16, 12, 1024), (4, 16, 4096), (2, 32, 8192)])
def test_list_order_balances_the_causal_triangle(S, B, H, T):
    # Causal forward: block qb of a head costs 2 qb + 2 key-tile steps; backward: key tile kt
    # is seen by n_tiles - kt query tiles.  Taken greedily, the list ends within a few percent of
    # the mean load, where plain head-major order leaves a tail of long items.
    BH, n_tiles = B * H, T // 128
    n_blocks = n_tiles // 2
    tail = S.sch_tail_heads(BH, n_blocks, 148)
    bh, qb = ctypes.c_int(), ctypes.c_int()
    fwd = []
    for i in range(BH * n_blocks):
        S.sch_fwd_item(i, BH, n_blocks, tail, ctypes.byref(bh), ctypes.byref(qb))
        fwd.append(2 * qb.value + 2)
    assert list_makespan(fwd) <= 1.03 * sum(fwd) / 148 + 2
    assert list_makespan(fwd) <= list_makespan([2 * q + 2 for _ in range(BH) for q in reversed(range(n_blocks))])
    tail = S.sch_tail_heads(BH, n_tiles, 148)
    kt, nq = ctypes.c_int(), ctypes.c_int()
    bwd = []
    for u in range(BH * n_tiles):
        S.sch_bwd_unit(u, BH, n_tiles, tail, 0, ctypes.byref(bh), ctypes.byref(kt), ctypes.byref(nq))
        bwd.append(nq.value)
    assert list_makespan(bwd) <= 1.03 * sum(bwd) / 148 + 1
    assert list_makespan(bwd) <= list_makespan([n_tiles - k for _ in range(BH) for k in range(n_tiles)])


def static_schedule(S, sms, n_blocks, BH):
    hpw, waves = ctypes.c_int(), ctypes.c_int()
    use = S.sch_fwd_static_grid(sms, n_blocks, BH, ctypes.byref(hpw), ctypes.byref(waves))
    G = hpw.value * n_blocks
    items, per_cta = {}, [[] for _ in range(G)]
    bh, qb = ctypes.c_int(), ctypes.c_int()
    for cta in range(G):
        for k in range(waves.value):
            S.sch_fwd_static_item(hpw.value, n_blocks, BH, cta, k, ctypes.byref(bh), ctypes.byref(qb))
            if bh.value < 0:
                continue
            key = (bh.value, qb.value)
            assert key not in items, f"item {key} scheduled twice"
            items[key] = (cta, k)
            per_cta[cta].append(qb.value)
    return bool(use), hpw.value, waves.value, G, items, per_cta


@pytest.mark.parametrize("sms,T,BH", [(148, 1024, 768), (148, 1024, 96), (148, 1024, 320), (148, 256, 6),
                                      (148, 8192, 24), (132, 2048, 50), (148, 4096, 600), (16, 40000, 3),
                                      (148, 1000, 1)])
def test_static_forward_order(S, sms, T, BH):
    n_blocks = -(-(-(-T // 128)) // 2)
    use, hpw, waves, G, items, per_cta = static_schedule(S, sms, n_blocks, BH)
    # every item exactly once, at most one block per SM
    assert set(items) == {(b, q) for b in range(BH) for q in range(n_blocks)}
    # chosen only for at least four full rotations of the block classes, one block per SM
    assert use == (G <= sms and waves >= 4 * n_blocks)
    # the blocks of one head run in the same wave (shared K/V tiles through L2)
    for b in range(BH):
        assert len({items[(b, q)][1] for q in range(n_blocks)}) == 1


def test_static_forward_order_balances_the_gpt2_shape(S):
    # 768 heads x 4 blocks on 148 SMs, block qb costing 2 qb + 2 key-tile steps: the busiest block
    # stays within one longest item of the mean.
    use, hpw, waves, G, items, per_cta = static_schedule(S, 148, 4, 768)
    assert use
    work = [sum(2 * qb + 2 for qb in c) for c in per_cta]
    assert max(work) <= sum(work) / len(work) + 8


@pytest.mark.parametrize("T,BH", [(1024, 768), (1024, 96), (256, 6), (8192, 24), (2048, 50), (40000, 3),
                                  (1000, 1), (100, 2)])
def test_forward_items_listed_exactly_once(S, T, BH):
    n_blocks = -(-(-(-T // 128)) // 2)
    tail = S.sch_tail_heads(BH, n_blocks, 148)
    bh, qb = ctypes.c_int(), ctypes.c_int()
    seen = []
    for i in range(BH * n_blocks):
        S.sch_fwd_item(i, BH, n_blocks, tail, ctypes.byref(bh), ctypes.byref(qb))
        seen.append((bh.value, qb.value))
    assert sorted(seen) == [(b, q) for b in range(BH) for q in range(n_blocks)]
    # the list starts with the last, longest query block
    assert seen[0][1] == n_blocks - 1


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
