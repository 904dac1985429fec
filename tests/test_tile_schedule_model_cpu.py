"""The work decomposition of the attention kernels, checked on the CPU against
brute-force definitions.

A Python model of the kernels' index arithmetic (stacked Q tiles of
T = floor(128 / g) tokens and g heads, forward items of two Q tiles with their
key-tile counts, backward items of one 128-key tile with their first Q tile,
the per-tile masking flag, the persistent snake order) is compared with what
causal or bidirectional attention needs: every visible (query, key) pair lies
in a visited tile pair, no visited tile pair is fully masked, every tile pair
that holds a hidden pair is flagged for masking, and every work item is taken
by exactly one CTA.  The GPU parity tests check the arithmetic on the tiles;
this checks that the schedule visits the right tiles for every shape,
including group sizes that do not divide 128 and ragged sequence ends.
"""
import itertools
import random

import pytest

BM, NK_FWD, NK_BWD = 128, 64, 128


def _visible(i, j, N, causal):
    return i < N and j < N and (not causal or j <= i)


def fwd_items(B, N, Hkv, g, causal):
    """The forward's work items as the kernel decodes them: (b, kvh, qt0, nkv0, nkv1)."""
    T = BM // g
    n_qt = -(-N // T)
    n_pairs = -(-n_qt // 2)
    n_bh = B * Hkv
    out = []
    for item in range(n_pairs * n_bh):
        pair = n_pairs - 1 - item // n_bh  # latest tokens first
        bh = item % n_bh
        qt0 = 2 * pair
        has1 = qt0 + 1 < n_qt
        end0 = min(N, (qt0 + 1) * T) if causal else N
        end1 = min(N, (qt0 + 2) * T) if causal else N
        out.append((bh // Hkv, bh % Hkv, qt0, -(-end0 // NK_FWD), -(-end1 // NK_FWD) if has1 else 0))
    return out


def fwd_masked(k0, qt, T, N, causal):
    return (k0 + NK_FWD > N) or (causal and k0 + NK_FWD - 1 > qt * T)


def bwd_items(B, N, Hkv, g, causal):
    """The backward's work items: (b, kvh, k0, qt_first, nq)."""
    T = BM // g
    n_qt = -(-N // T)
    n_kt = -(-N // NK_BWD)
    n_bh = B * Hkv
    out = []
    for item in range(n_kt * n_bh):
        kt, bh = divmod(item, n_bh)
        k0 = kt * NK_BWD
        qt_first = k0 // T if causal else 0
        out.append((bh // Hkv, bh % Hkv, k0, qt_first, n_qt - qt_first))
    return out


def bwd_masked(k0, qt, T, causal):
    return causal and k0 + NK_BWD - 1 > qt * T


def snake(n_items, grid):
    """Items of each CTA of a persistent grid, in the kernels' snake order."""
    per_cta = {c: [] for c in range(grid)}
    for c in range(grid):
        r = 0
        while True:
            item = r * grid + ((grid - 1 - c) if r & 1 else c)
            if item >= n_items:
                break
            per_cta[c].append(item)
            r += 1
    return per_cta


def _tile_pairs_needed(N, T, NK, causal):
    n_qt, n_kt = -(-N // T), -(-N // NK)
    need = set()
    for qt, kt in itertools.product(range(n_qt), range(n_kt)):
        if any(_visible(i, j, N, causal) for i in range(qt * T, qt * T + T) for j in range(kt * NK, kt * NK + NK)):
            need.add((qt, kt))
    return need


def _hidden(qt, kt, T, NK, N, causal):
    """A (query, key) pair of the tile pair with a valid query whose key must not count."""
    return any(i < N and not _visible(i, j, N, causal)
               for i in range(qt * T, qt * T + T) for j in range(kt * NK, kt * NK + NK))


SHAPES = [(1, 200, 1, 8), (2, 130, 2, 1), (1, 1000, 1, 3), (1, 517, 2, 6), (1, 64, 1, 16), (1, 1, 1, 4),
          (1, 300, 1, 128), (2, 129, 3, 5), (1, 700, 1, 100)]


@pytest.mark.parametrize("B,N,Hkv,g", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_forward_visits_exactly_the_needed_key_tiles(B, N, Hkv, g, causal):
    T = BM // g
    need = _tile_pairs_needed(N, T, NK_FWD, causal)
    seen = {}
    for b, kvh, qt0, nkv0, nkv1 in fwd_items(B, N, Hkv, g, causal):
        for qt, nkv in ((qt0, nkv0), (qt0 + 1, nkv1)):
            for kt in range(nkv):
                seen[(b, kvh, qt, kt)] = seen.get((b, kvh, qt, kt), 0) + 1
                assert (qt, kt) in need, f"fully masked tile pair visited: q tile {qt}, k tile {kt}"
                if _hidden(qt, kt, T, NK_FWD, N, causal):
                    assert fwd_masked(kt * NK_FWD, qt, T, N, causal), f"unflagged tile pair {qt}, {kt}"
    for b, kvh in itertools.product(range(B), range(Hkv)):
        for qt, kt in need:
            assert seen.get((b, kvh, qt, kt)) == 1, f"tile pair {qt}, {kt} of ({b}, {kvh}) visited {seen.get((b, kvh, qt, kt))} times"


@pytest.mark.parametrize("B,N,Hkv,g", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_backward_visits_exactly_the_needed_query_tiles(B, N, Hkv, g, causal):
    T = BM // g
    need = _tile_pairs_needed(N, T, NK_BWD, causal)
    seen = {}
    for b, kvh, k0, qt_first, nq in bwd_items(B, N, Hkv, g, causal):
        kt = k0 // NK_BWD
        for qt in range(qt_first, qt_first + nq):
            seen[(b, kvh, qt, kt)] = seen.get((b, kvh, qt, kt), 0) + 1
            assert (qt, kt) in need, f"fully masked tile pair visited: q tile {qt}, k tile {kt}"
            if causal and any(i < N and j < N and j > i for i in range(qt * T, qt * T + T)
                              for j in range(k0, k0 + NK_BWD)):
                assert bwd_masked(k0, qt, T, causal), f"unflagged tile pair {qt}, {kt}"
    for b, kvh in itertools.product(range(B), range(Hkv)):
        for qt, kt in need:
            assert seen.get((b, kvh, qt, kt)) == 1


@pytest.mark.parametrize("g", [1, 2, 3, 5, 8, 16, 100, 128])
def test_stacked_rows_cover_every_token_and_head_once(g):
    N, T = 1000, BM // g
    rows = T * g
    assert rows <= BM
    cover = {}
    for qt in range(-(-N // T)):
        for r in range(rows):
            tok, head = qt * T + r // g, r % g
            if tok < N:
                cover[(tok, head)] = cover.get((tok, head), 0) + 1
    assert len(cover) == N * g and set(cover.values()) == {1}


@pytest.mark.parametrize("n_items,grid", [(1, 148), (148, 148), (149, 148), (1000, 148), (7, 3), (64, 8)])
def test_snake_order_gives_every_item_to_one_cta(n_items, grid):
    per_cta = snake(n_items, min(n_items, grid))
    taken = sorted(i for items in per_cta.values() for i in items)
    assert taken == list(range(n_items))
    counts = [len(v) for v in per_cta.values()]
    assert max(counts) - min(counts) <= 1


@pytest.mark.parametrize("B,N,Hkv,g", [(32, 1024, 4, 2), (32, 1024, 1, 16), (2, 8192, 4, 2)])
@pytest.mark.parametrize("kind", ["fwd", "bwd"])
def test_snake_order_evens_out_causal_work(B, N, Hkv, g, kind):
    """Causal items are listed heaviest first.  Dealing them in a snake (each
    round reversing the direction) keeps every CTA's total within half of the
    largest item's cost of every other CTA's, and its busiest CTA has less work
    than round-robin dealing would give it."""
    if kind == "fwd":
        costs = [n0 + n1 for (_, _, _, n0, n1) in fwd_items(B, N, Hkv, g, True)]
    else:
        costs = [nq for (*_, nq) in bwd_items(B, N, Hkv, g, True)]
    grid = 148
    assert len(costs) > grid  # at least two rounds
    snake_totals = [sum(costs[i] for i in items) for items in snake(len(costs), grid).values()]
    rr_totals = [sum(costs[i::grid]) for i in range(grid)]
    assert max(snake_totals) - min(snake_totals) <= max(costs) / 2
    assert max(snake_totals) < max(rr_totals)


def fwd_split_items(B, N, Hkv, g, causal):
    """The forward's split-mode items (small problems): one Q tile each, slot
    t taking the key tiles t, t + 2, ...: (b, kvh, qt, [key tiles of slot 0],
    [key tiles of slot 1])."""
    T = BM // g
    n_qt = -(-N // T)
    n_bh = B * Hkv
    out = []
    for item in range(n_qt * n_bh):
        qt = n_qt - 1 - item // n_bh
        bh = item % n_bh
        end = min(N, (qt + 1) * T) if causal else N
        nkv = -(-end // NK_FWD)
        n0, n1 = (nkv + 1) // 2, nkv // 2
        out.append((bh // Hkv, bh % Hkv, qt, [2 * j for j in range(n0)], [2 * j + 1 for j in range(n1)]))
    return out


@pytest.mark.parametrize("B,N,Hkv,g", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_forward_split_mode_visits_exactly_the_needed_key_tiles(B, N, Hkv, g, causal):
    T = BM // g
    need = _tile_pairs_needed(N, T, NK_FWD, causal)
    seen = {}
    for b, kvh, qt, tiles0, tiles1 in fwd_split_items(B, N, Hkv, g, causal):
        assert len(tiles0) >= len(tiles1) and not set(tiles0) & set(tiles1)
        for kt in tiles0 + tiles1:
            seen[(b, kvh, qt, kt)] = seen.get((b, kvh, qt, kt), 0) + 1
            assert (qt, kt) in need, f"fully masked tile pair visited: q tile {qt}, k tile {kt}"
            if _hidden(qt, kt, T, NK_FWD, N, causal):
                assert fwd_masked(kt * NK_FWD, qt, T, N, causal), f"unflagged tile pair {qt}, {kt}"
    for b, kvh in itertools.product(range(B), range(Hkv)):
        for qt, kt in need:
            assert seen.get((b, kvh, qt, kt)) == 1


def fwd_range_plan(B, N, Hkv, g, causal, sms=148):
    """The host's choice of key ranges for small problems (split mode with a
    workspace): None when every Q tile stays one item, else (chunk, number of
    items).  Chunk: the smallest even number of key tiles (at least 2) whose
    items do not outnumber the SMs; ranges only if they shorten the longest Q
    tile's walk by at least 6 key tiles per slot."""
    T = BM // g
    n_qt = -(-N // T)
    n_bh = B * Hkv
    if not (-(-n_qt // 2) * n_bh < sms // 2 and n_qt * n_bh < sms // 2):
        return None
    nkv = [-(-(min(N, (qt + 1) * T) if causal else N) // NK_FWD) for qt in range(n_qt)]
    chunk = 2
    while chunk < nkv[-1] and n_bh * sum(-(-n // chunk) for n in nkv) > sms:
        chunk += 2
    if -(-nkv[-1] // 2) - chunk // 2 < 6:
        return None
    return chunk, n_bh * sum(-(-n // chunk) for n in nkv)


def fwd_range_items(B, N, Hkv, g, causal, chunk, n_items):
    """The items as the kernel decodes them: the k-th range of a (batch, KV
    head), Q tiles from the last, ranges in key order: (b, kvh, qt, c, nch,
    [key tiles of slot 0], [key tiles of slot 1])."""
    T = BM // g
    n_qt = -(-N // T)
    n_bh = B * Hkv

    def nkv_of(qt):
        return -(-(min(N, (qt + 1) * T) if causal else N) // NK_FWD)

    out = []
    for item in range(n_items):
        k, bh = item // n_bh, item % n_bh
        qt = n_qt - 1
        nkv = nkv_of(qt)
        nch = -(-nkv // chunk)
        while k >= nch and qt > 0:
            k -= nch
            qt -= 1
            nkv = nkv_of(qt)
            nch = -(-nkv // chunk)
        kt0 = k * chunk
        n = max(0, min(nkv - kt0, chunk))
        n0, n1 = (n + 1) // 2, n // 2
        out.append((bh // Hkv, bh % Hkv, qt, k, nch, [kt0 + 2 * j for j in range(n0)],
                    [kt0 + 2 * j + 1 for j in range(n1)]))
    return out


RANGE_SHAPES = [(1, 2000, 1, 2), (1, 4096, 1, 2), (1, 2500, 1, 3), (1, 1500, 1, 6), (1, 2300, 1, 4), (1, 3000, 1, 1),
                (1, 1000, 2, 1), (2, 1500, 1, 2)]


@pytest.mark.parametrize("B,N,Hkv,g", RANGE_SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_forward_key_ranges_visit_exactly_the_needed_key_tiles(B, N, Hkv, g, causal):
    """Split mode with key ranges over several CTAs: every needed (Q tile, key
    tile) pair is computed by exactly one slot of one range, the ranges of a Q
    tile are consecutive and disjoint and their count is the one the merge
    waits for, and tiles holding hidden pairs are flagged for masking."""
    plan = fwd_range_plan(B, N, Hkv, g, causal)
    if plan is None:
        pytest.skip("no key ranges for this shape")
    chunk, n_items = plan
    T = BM // g
    need = _tile_pairs_needed(N, T, NK_FWD, causal)
    seen, ranges = {}, {}
    for b, kvh, qt, c, nch, tiles0, tiles1 in fwd_range_items(B, N, Hkv, g, causal, chunk, n_items):
        assert 0 <= c < nch and tiles0, "empty range"
        assert len(tiles0) >= len(tiles1) and not set(tiles0) & set(tiles1)
        assert all(c * chunk <= kt < (c + 1) * chunk for kt in tiles0 + tiles1)
        ranges.setdefault((b, kvh, qt), []).append((c, nch))
        for kt in tiles0 + tiles1:
            seen[(b, kvh, qt, kt)] = seen.get((b, kvh, qt, kt), 0) + 1
            assert (qt, kt) in need, f"fully masked tile pair visited: q tile {qt}, k tile {kt}"
            if _hidden(qt, kt, T, NK_FWD, N, causal):
                assert fwd_masked(kt * NK_FWD, qt, T, N, causal), f"unflagged tile pair {qt}, {kt}"
    for b, kvh in itertools.product(range(B), range(Hkv)):
        for qt, kt in need:
            assert seen.get((b, kvh, qt, kt)) == 1
    for key, rs in ranges.items():
        nch = rs[0][1]
        assert sorted(c for c, _ in rs) == list(range(nch)) and all(n == nch for _, n in rs), key


def test_forward_key_ranges_choice():
    """One long sequence with a single KV head (B=1, N=4096, 2/1, causal): 64
    Q tiles, ranges of 16 key tiles would make 160 items for 148 SMs, so 18:
    148 items (one Q tile per CTA walked up to 32 key tiles per slot, now 9).
    The SQAT-m layer-sized forward (B=1, N=1024, 8/4) would go from 8 key
    tiles per slot to 3, too little to pay for the merge: no ranges."""
    assert fwd_range_plan(1, 4096, 1, 2, True) == (18, 148)
    assert fwd_range_plan(1, 4096, 1, 2, False) == (32, 128)
    assert fwd_range_plan(1, 1024, 4, 2, True) is None
    assert fwd_range_plan(32, 1024, 4, 2, True) is None
    assert fwd_range_plan(1, 256, 4, 2, True) is None
