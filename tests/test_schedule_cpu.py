"""The persistent kernels' work schedules, restated in Python from their definitions
(csrc/fa_ptx.cuh item_position, csrc/fa_bwd.cuh bwd_item, csrc/fa_bwd_fused.cuh FusedWalk,
csrc/fa_api.cu launch_fused, csrc/fa_fwd.cuh fwd_item / causal_klast / FwdSched) and checked
for the properties the kernels rely on: every (batch*head, tile) item is visited by exactly
one CTA, paired causal items all cost the same, the launcher pairs only when the pairs fill
the last round of CTAs, and the forward visits every key tile that holds a visible
(query, key) pair."""
import itertools

import numpy as np
import pytest


def item_position(n_items, k, grid, cta):
    # round k deals positions k*G .. k*G + G - 1, in alternating direction
    pos = k * grid + ((grid - 1 - cta) if (k & 1) else cta)
    return pos if pos < n_items else -1


def bwd_item(causal, n, bh_count, k, grid, cta):
    pos = item_position(n * bh_count, k, grid, cta)
    if pos < 0:
        return None
    if causal:  # costliest first across heads: tile 0 (the most query tiles) first
        return (pos % bh_count, pos // bh_count)
    return (pos // n, pos % n)  # head-major


def paired_walk(n, bh_count, grid, cta):
    """Items of one CTA when causal key tiles are dealt as pairs (j, n - 1 - j)."""
    n_pairs = (n + 1) // 2
    out, k = [], 0
    while True:
        pos = item_position(n_pairs * bh_count, k, grid, cta)
        if pos < 0:
            return out
        bh, pr = pos // n_pairs, pos % n_pairs
        out.append((bh, pr))
        if n - 1 - pr != pr:
            out.append((bh, n - 1 - pr))
        k += 1


def launcher_pairs(n, bh_count, sms):
    """The fused launcher's rule: pair when the last round of CTAs is at least 95% full."""
    pairs = (n + 1) // 2 * bh_count
    slots = (pairs + sms - 1) // sms * sms
    return 20 * (slots - pairs) <= slots


@pytest.mark.parametrize("causal", [False, True])
def test_single_items_cover_every_tile_once(causal):
    for n, bh_count, sms in itertools.product((1, 2, 5, 16, 64), (1, 3, 32), (7, 148)):
        grid = min(n * bh_count, sms)
        seen = []
        for cta in range(grid):
            k = 0
            while (it := bwd_item(causal, n, bh_count, k, grid, cta)) is not None:
                seen.append(it)
                k += 1
        assert sorted(seen) == sorted(itertools.product(range(bh_count), range(n))), (n, bh_count, sms)


def test_paired_items_cover_every_tile_once_and_cost_the_same():
    for n, bh_count, sms in itertools.product((1, 2, 3, 5, 16, 63, 64), (1, 3, 32), (7, 148)):
        n_pairs = (n + 1) // 2
        grid = min(n_pairs * bh_count, sms)
        seen = []
        for cta in range(grid):
            items = paired_walk(n, bh_count, grid, cta)
            seen += items
        assert sorted(seen) == sorted(itertools.product(range(bh_count), range(n))), (n, bh_count, sms)
    # with the causal mask key tile j has n - j query tiles: a pair (j, n - 1 - j) has n + 1
    for n in (2, 16, 64):
        assert {(n - j) + (n - (n - 1 - j)) for j in range(n // 2)} == {n + 1}


def test_pairs_fill_the_rounds_at_the_bench_shape():
    # B=2 H=16 N=8192: 64 key tiles, 32 pairs per head, 1024 pairs over 148 SMs (7 rounds,
    # 12 empty slots in the last): paired. B=1 H=16 N=4096: 256 pairs, the second of two
    # rounds 73% full: single items.
    assert launcher_pairs(64, 32, 148)
    assert not launcher_pairs(32, 16, 148)
    # one head per SM always fills the rounds (the parity test that forces pairing)
    assert launcher_pairs(3, 148, 148) and launcher_pairs(8, 148, 148)


# ------------------------------------------------------------------ forward


def fwd_item(causal, n_qblocks, bh_count, k, grid, cta):
    """(bh, qb) of a CTA's k-th forward item; an item is Q tiles 2 qb and 2 qb + 1."""
    pos = item_position(n_qblocks * bh_count, k, grid, cta)
    if pos < 0:
        return None
    if causal:  # block-major, the costliest (last) query block first
        return (pos % bh_count, n_qblocks - 1 - pos // bh_count)
    return (pos // n_qblocks, n_qblocks - 1 - pos % n_qblocks)  # head-major


def causal_klast(t, off, n_ktiles):
    """Last key tile Q tile t visits with the causal mask (bottom-right aligned, off = Nk - Nq)."""
    x = 128 * t + 127 + off
    last = -1 if x < 0 else x >> 7
    return min(last, n_ktiles - 1)


def fwd_visits(t, causal, n_ktiles, off):
    last = causal_klast(t, off, n_ktiles) if causal else n_ktiles - 1
    return set(range(last + 1))


@pytest.mark.parametrize("causal", [False, True])
def test_forward_items_cover_every_query_tile_once(causal):
    for n_tiles, bh_count, sms in itertools.product((1, 2, 3, 5, 16, 63, 64), (1, 3, 32), (7, 148)):
        n_qblocks = (n_tiles + 1) // 2
        grid = min(n_qblocks * bh_count, sms)
        tiles = []
        for cta in range(grid):
            k, qbs = 0, []
            while (it := fwd_item(causal, n_qblocks, bh_count, k, grid, cta)) is not None:
                bh, qb = it
                tiles += [(bh, t) for t in (2 * qb, 2 * qb + 1) if t < n_tiles]
                qbs.append(qb)
                k += 1
            if causal:  # each CTA's items get no costlier: the deal stays balanced
                assert qbs == sorted(qbs, reverse=True), (n_tiles, bh_count, sms, cta)
        assert sorted(tiles) == sorted(itertools.product(range(bh_count), range(n_tiles)))


@pytest.mark.parametrize("nq,nk", [(128, 128), (300, 300), (1000, 1000), (200, 700), (700, 200),
                                   (129, 1), (1, 129), (384, 256), (256, 384)])
def test_causal_forward_visits_every_visible_key_tile(nq, nk):
    """Brute force over (query, key) pairs: key j is visible to query i iff j <= i + Nk - Nq.
    Every key tile holding a visible pair of one of a Q tile's real rows is visited; a tile
    whose rows see nothing visits nothing (those rows get O = 0, lse = -inf); a visited tile
    that no real row sees occurs only in the last, partial Q tile (its element mask zeroes it)."""
    off = nk - nq
    n_tiles, n_ktiles = -(-nq // 128), -(-nk // 128)
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    vis = j <= i + off
    for t in range(n_tiles):
        rows = vis[128 * t:128 * (t + 1)]
        needed = {jt for jt in range(n_ktiles) if rows[:, 128 * jt:128 * (jt + 1)].any()}
        got = fwd_visits(t, True, n_ktiles, off)
        assert needed <= got, (nq, nk, t, sorted(needed - got))
        if not needed:
            assert not got, (nq, nk, t)
        if got - needed:
            assert t == n_tiles - 1 and nq % 128, (nq, nk, t, sorted(got - needed))
        if nq == nk:  # the square case: the diagonal tile is the last one
            assert max(got) == t


# ------------------------------------------------------------------ backward visibility


def causal_qfirst(j, off):
    """First query tile that sees key tile j (dK/dV and fused kernels)."""
    x = 128 * j - 127 - off
    return 0 if x <= 0 else (x + 127) >> 7


@pytest.mark.parametrize("nq,nk", [(128, 128), (300, 300), (1000, 1000), (200, 700), (700, 200),
                                   (129, 1), (1, 129), (384, 256), (256, 384), (640, 1000)])
def test_causal_backward_pairs(nq, nk):
    """The dK/dV side (query tiles t >= qfirst(j) of key tile j) and the dQ side (key tiles
    j <= klast(t) of query tile t) visit the same (query tile, key tile) pairs, and these
    hold every visible (query, key) pair of real rows and keys."""
    off = nk - nq
    n_tiles, n_ktiles = -(-nq // 128), -(-nk // 128)
    by_key = {(t, j) for j in range(n_ktiles) for t in range(causal_qfirst(j, off), n_tiles)}
    by_query = {(t, j) for t in range(n_tiles) for j in range(causal_klast(t, off, n_ktiles) + 1)}
    assert by_key == by_query, (nq, nk, sorted(by_key ^ by_query))
    vis = np.arange(nk)[None, :] <= np.arange(nq)[:, None] + off
    needed = {(t, j) for t in range(n_tiles) for j in range(n_ktiles)
              if vis[128 * t:128 * (t + 1), 128 * j:128 * (j + 1)].any()}
    assert needed <= by_key, (nq, nk, sorted(needed - by_key))
    extra = by_key - needed  # pairs no real row sees: only in the last, partial query tile
    assert all(t == n_tiles - 1 and nq % 128 for t, _ in extra), (nq, nk, sorted(extra))
