"""A model of the synchronisation of the persistent forward kernel
(``sqa_fwd_kernel``), run on the CPU under random schedules.

Roles, in the kernel's program order: the TMA producer (a pair of Q tiles per
work item into one of QBUF buffers, K/V tiles into a ring of STAGES), one MMA
issuer per Q tile (S = Q K^T into two TMEM buffers per tile, O += P V), and
the four softmax warps of each tile (P written over S in place, an occasional
rescale of O, the epilogue).  Barrier arrival counts are the kernel's.

Buffers checked by stage (see ``sync_model``): the Q buffers (producer writes,
both issuers read), the K/V stages (producer writes, both issuers read until
their release), and each tile's two S/P buffers (issuer's S MMA writes, the
4 warps rewrite P, the P V MMA reads).  The O accumulator of each tile is
shared by interleaved users and gets its own checker: no P V MMA, rescale or
epilogue read overlaps another user, a rescale at step G comes after P V of
step G - 1 completed and before P V of step G starts, the epilogue comes after
the item's last P V, and the next item's first P V after all 4 warps have read
O.  Whether a warp rescales O at a step depends on the data, so each step
draws it at random.

Work lists mirror the kernel's items: per item, nkv0 key tiles for Q tile 0,
nkv1 for Q tile 1 (0 when the item has one tile; one more than nkv0 under a
causal mask when the tiles straddle a key-tile boundary) and nkv = max of the
two loaded.  The kernel's buffer configurations are run: QBUF 2 with 8 stages
(dh <= 32), QBUF 2 with 4 stages (dh 64), each with two S buffers per tile,
and QBUF 1 with 2 stages and one S buffer per tile (dh 128, 128-key tiles);
QBUF 1 with 3 stages and two S buffers is kept as a further case.

With one S buffer per tile the two tiles' softmax warpgroups also pass a token
(mbarriers tok0 / tok1) around their exponentials, within each item: slot 0's
step j after slot 1's step j - 1, slot 1's step j after slot 0's step j, where
the other slot has such a step (an order across items deadlocks: the next
item's Q load waits for the Q buffer this item's last steps hold).  A custom
checker asserts that the two tiles' exponential phases never overlap within
an item.
"""
import random

import pytest
import sync_model

WARPS_PER_TILE = 4

STAGES = {
    "q": [("producer writes the Q pair", 1), ("both issuers read", 2)],
    "kv": [("producer writes K, V", 1), ("both issuers read", 2)],
    "S0": [("issuer 0 writes S", 1), ("tile 0 warps write P", WARPS_PER_TILE), ("issuer 0 reads P (P V)", 1)],
    "S1": [("issuer 1 writes S", 1), ("tile 1 warps write P", WARPS_PER_TILE), ("issuer 1 reads P (P V)", 1)],
}


class Accumulator:
    """Users of one tile's O accumulator in TMEM."""

    def __init__(self):
        self.pv_started = self.pv_done = 0  # P V steps (across items)
        self.active = {}                    # kind -> active users
        self.epi_ended = {}                 # item -> warps that finished the epilogue

    def _alone(self, kind):
        others = {k: n for k, n in self.active.items() if k != kind and n}
        assert not others, f"hazard on O: {kind} overlaps {others}"

    def begin(self, slot, info):
        kind = info[0]
        self._alone(kind)
        if kind == "pv":
            _, step, item, first = info
            assert self.active.get("pv", 0) == 0 and self.pv_started == step == self.pv_done, \
                f"hazard on O: P V step {step} out of order"
            if first and item > 0:
                assert self.epi_ended.get(item - 1, 0) == WARPS_PER_TILE, \
                    f"hazard on O: item {item} overwrites O before its epilogue read item {item - 1}"
            self.pv_started += 1
        elif kind == "rescale":
            _, step = info
            assert self.pv_done == step and self.pv_started == step, \
                f"hazard on O: rescale at step {step} with {self.pv_done} P V done, {self.pv_started} started"
        else:  # epilogue
            _, item, steps_end = info
            assert self.pv_done == steps_end, f"hazard on O: epilogue of item {item} before its last P V"
        self.active[kind] = self.active.get(kind, 0) + 1

    def end(self, slot, info):
        kind = info[0]
        self.active[kind] -= 1
        if kind == "pv":
            self.pv_done += 1
        elif kind == "epi":
            self.epi_ended[info[1]] = self.epi_ended.get(info[1], 0) + 1


def _roles(items, QB, ST, rnd, NSB=2, split=False):
    """items: [(nkv0, nkv1)] per work item of one CTA.  split: both slots on one
    Q tile, slot t taking the item's key tiles t, t + 2, ... (nkv0 = ceil(n / 2),
    nkv1 = floor(n / 2)), slot 1's O read by slot 0's warps in the combine."""
    cnt = {"split_ready": 32 * WARPS_PER_TILE, "split_done": 32 * WARPS_PER_TILE}
    for qb in range(QB):
        cnt[f"q_full{qb}"] = 1
        cnt[f"q_empty{qb}"] = 2
    for s in range(ST):
        cnt[f"kv_full{s}"] = 1
        cnt[f"kv_empty{s}"] = 2
    cnt["tok0"] = cnt["tok1"] = 32 * WARPS_PER_TILE
    for t in range(2):
        for buf in range(2):
            cnt[f"s_full{t}{buf}"] = 1
            cnt[f"p_full{t}{buf}"] = 32 * WARPS_PER_TILE
        cnt[f"o_done{t}"] = 1
        cnt[f"o_final{t}"] = 1
        cnt[f"o_free{t}"] = 32 * WARPS_PER_TILE

    def W(b, k):
        return ("wait", b, k)

    def A(b, m=1):
        return ("arrive", b, m)

    def B(res, slot, v, stage=None):
        return ("begin", (res, slot), v, stage)

    def E(res, slot, v, stage=None):
        return ("end", (res, slot), v, stage)

    def nkv_of(n0, n1):
        return n0 + n1 if split else max(n0, n1)

    prod, g = [], 0
    for r, (n0, n1) in enumerate(items):
        qb, nkv = r % QB, nkv_of(n0, n1)
        if r >= QB:
            prod.append(W(f"q_empty{qb}", r // QB - 1))
        prod += [B("q", qb, r, 0), E("q", qb, r, 0), A(f"q_full{qb}")]
        for j in range(nkv):
            s = (g + j) % ST
            if g + j >= ST:
                prod.append(W(f"kv_empty{s}", (g + j) // ST - 1))
            prod += [B("kv", s, g + j, 0), E("kv", s, g + j, 0), A(f"kv_full{s}")]
        g += nkv

    def issuer(t):
        ops, g, G, nd, loaded = [], [0], 0, 0, [0]
        S = f"S{t}"

        def own(j):
            return 2 * j + t if split else j

        def ensure(gj):
            out = []
            while loaded[0] <= gj:
                i = loaded[0]
                out.append(W(f"kv_full{i % ST}", i // ST))
                if split and (i - g[0]) % 2 != t:  # the other slot's tile: released at once
                    out += [B("kv", i % ST, i, 1), E("kv", i % ST, i, 1), A(f"kv_empty{i % ST}")]
                loaded[0] += 1
            return out

        def qk(qb, gj, step):  # S of key tile gj into buffer step % NSB; the MMA reads Q and K
            return [B(S, step % NSB, step, 0), E(S, step % NSB, step, 0), A(f"s_full{t}{step % NSB}")]

        for r, (n0, n1) in enumerate(items):
            nkv_t, nkv, qb = (n1 if t else n0), nkv_of(n0, n1), r % QB
            base = g[0]
            ops += [W(f"q_full{qb}", r // QB), B("q", qb, r, 1)]
            for j in range(min(NSB, nkv_t)):
                gi = base + own(j)
                ops += ensure(gi) + [B("kv", gi % ST, gi, 1)] + qk(qb, gi, G + j)
            for j in range(nkv_t):
                step, gi = G + j, base + own(j)
                ops.append(W(f"p_full{t}{step % NSB}", step // NSB))
                if j == 0 and nd > 0:
                    ops.append(W(f"o_free{t}", nd - 1))
                # P V: reads P from the S buffer and V, accumulates into O; MMAs of one
                # issuer run in order, so its read of P ends before the next S MMA.
                ops += [B(S, step % NSB, step, 2), B("O", t, ("pv", step, nd, j == 0)),
                        E(S, step % NSB, step, 2), E("O", t, ("pv",)), A(f"o_done{t}")]
                if j + 1 == nkv_t:
                    ops.append(A(f"o_final{t}"))
                # the stage is released (after the P V just issued) before a later one is awaited
                ops += [E("kv", gi % ST, gi, 1), A(f"kv_empty{gi % ST}")]
                if j + NSB < nkv_t:
                    gn = base + own(j + NSB)
                    ops += ensure(gn) + [B("kv", gn % ST, gn, 1)] + qk(qb, gn, step + NSB)
            if split:
                if nkv > 0:
                    ops += ensure(base + nkv - 1)
            else:
                for j in range(nkv_t, nkv):  # tiles the other Q tile needs: released once loaded
                    ops += ensure(base + j) + [B("kv", (base + j) % ST, base + j, 1),
                                               E("kv", (base + j) % ST, base + j, 1),
                                               A(f"kv_empty{(base + j) % ST}")]
            ops += [E("q", qb, r, 1), A(f"q_empty{qb}")]
            G += nkv_t
            nd += 1 if nkv_t else 0
            g[0] = base + nkv
        return ops

    token = NSB == 1

    def softmax_warp(t):
        ops, G, nd, G1, nd1, nc = [], 0, 0, 0, 0, 0
        S = f"S{t}"
        G_other = 0
        for r, (n0, n1) in enumerate(items):
            nkv_t, nkv_o = (n1, n0) if t else (n0, n1)
            G_o, G_other = G_other, G_other + nkv_o
            combine = split and n1 > 0
            if nkv_t == 0:
                continue
            for j in range(nkv_t):
                step = G + j
                ops += [W(f"s_full{t}{step % NSB}", step // NSB), B(S, step % NSB, step, 1)]
                if j > 0 and rnd.random() < 0.5:  # the running maximum rose: rescale O
                    ops += [W(f"o_done{t}", step - 1), B("O", t, ("rescale", step)), E("O", t, ("rescale",))]
                if token:
                    k_other = j if t else j - 1
                    if 0 <= k_other < nkv_o:
                        ops.append(W(f"tok{1 - t}", G_o + k_other))
                ops += [B("X", t, ("exp", r)), E("X", t, ("exp", r))]
                ops.append(E(S, step % NSB, step, 1))
                if token:  # the turn before P (the Q buffer is released after the last P V)
                    ops.append(A(f"tok{t}", 32))
                ops.append(A(f"p_full{t}{step % NSB}", 32))
            ops.append(W(f"o_final{t}", nd))
            if combine and t == 1:
                # hand m, l to slot 0; O_1 stays until slot 0 has read it
                ops += [A("split_ready", 32), W("split_done", nc), A(f"o_free{t}", 32)]
            else:
                if combine:  # slot 0 reads O_1 as well
                    ops += [W("split_ready", nc), B("O", 1, ("epi", nd1, G1 + n1)), E("O", 1, ("epi", nd1))]
                ops += [B("O", t, ("epi", nd, G + nkv_t)), E("O", t, ("epi", nd)), A(f"o_free{t}", 32)]
                if combine:
                    ops.append(A("split_done", 32))
            G += nkv_t
            nd += 1
            if combine:
                nc += 1
            if split and n1 > 0:
                G1 += n1
                nd1 += 1
        return ops

    roles = {"producer": prod, "issuer0": issuer(0), "issuer1": issuer(1)}
    for w in range(2 * WARPS_PER_TILE):
        roles[f"warp{w}"] = softmax_warp(w // WARPS_PER_TILE)
    return roles, cnt


def _items(rnd):
    out = []
    for _ in range(rnd.randint(1, 5)):
        kind = rnd.random()
        n0 = rnd.randint(1, 6)
        if kind < 0.15:
            out.append((n0, 0))        # last, single-tile item
        elif kind < 0.6:
            out.append((n0, n0 + 1))   # causal: tile 1 needs one more key tile
        else:
            out.append((n0, n0))       # bidirectional, or both tiles in one key tile
    return out


def run(items, QB, ST, seed, drop=None, NSB=2, split=False):
    rnd = random.Random(seed)
    roles, cnt = _roles(items, QB, ST, rnd, NSB, split)
    if drop is not None:
        roles = {r: [op for op in ops if not drop(r, op)] for r, ops in roles.items()}
    sync_model.run(roles, cnt, STAGES, seed, custom={"O": _OCheck(), "X": _ExpCheck(NSB == 1)},
                   skewed=seed % 2 == 1)


class _ExpCheck:
    """With the token (one S buffer per tile), the two tiles' exponential
    phases of one item never overlap."""

    def __init__(self, exclusive):
        self.exclusive = exclusive
        self.active = {0: {}, 1: {}}  # slot -> item -> warps in their exponentials

    def begin(self, slot, info):
        item = info[1]
        if self.exclusive:
            assert self.active[1 - slot].get(item, 0) == 0, "both tiles in their exponentials at once"
        self.active[slot][item] = self.active[slot].get(item, 0) + 1

    def end(self, slot, info):
        self.active[slot][info[1]] -= 1


class _OCheck:
    """One Accumulator per Q tile."""

    def __init__(self):
        self.acc = {0: Accumulator(), 1: Accumulator()}

    def begin(self, slot, info):
        self.acc[slot].begin(slot, info)

    def end(self, slot, info):
        self.acc[slot].end(slot, info)


@pytest.mark.parametrize("QB,ST,NSB", [(2, 8, 2), (2, 4, 2), (1, 3, 2), (1, 2, 1)])
def test_forward_protocol_has_no_deadlock_aliasing_or_hazard(QB, ST, NSB):
    rnd = random.Random(QB * 10 + ST)
    for trial in range(150):
        items = _items(rnd)
        for seed in range(3):
            run(items, QB, ST, trial * 100 + seed, NSB=NSB)


def _drop(role_prefix, barrier):
    return lambda r, op: r.startswith(role_prefix) and op[0] == "wait" and op[1].startswith(barrier)


# Waits whose removal the model must notice.  (The issuers' o_free wait is
# implied by the rest of the protocol: the first P V of the next item also
# waits for p_full of that step, which every warp signals only after its
# epilogue has read O.  The kernel keeps it as a second guard.)
DROPS = {
    # the warps would rescale O while a P V MMA still accumulates into it
    "warps: o_done": _drop("warp", "o_done"),
    # P V would read P before the warps wrote it
    "issuer: p_full": _drop("issuer", "p_full"),
    # the warps would read S before the MMA wrote it
    "warps: s_full": _drop("warp", "s_full"),
    # the epilogue would read O before the last P V
    "warps: o_final": _drop("warp", "o_final"),
    # the producer would overwrite a K/V stage or a Q buffer still in use
    "producer: kv_empty": _drop("producer", "kv_empty"),
    "producer: q_empty": _drop("producer", "q_empty"),
    # an issuer would read K/V or Q before they landed
    "issuer: kv_full": _drop("issuer", "kv_full"),
    "issuer: q_full": _drop("issuer", "q_full"),
    # with one S buffer per tile: both tiles would run their exponentials at once
    "warps: tok": _drop("warp", "tok"),
}


# With one S buffer per tile (dh 128) the next S MMA of a tile comes after its
# P V MMA in the issuer's order, so the warps' s_full wait also implies the
# P V of the previous step completed: there the o_done wait is implied.
IMPLIED = {("warps: o_done", 1), ("warps: tok", 2)}  # no token with two S buffers


def test_turn_after_p_would_let_a_wait_pass_early():
    # why each slot arrives on its turn barrier before p_full: with the turn
    # last, the Q buffer can be released (and the next item started) while a
    # thread of the other slot has not yet passed its last turn of this item, so
    # a slot that skipped those turns finds a phase of the same parity open
    rnd = random.Random(7)
    failures = 0
    for trial in range(200):
        items = _items(rnd)
        roles, cnt = _roles(items, 1, 2, random.Random(trial), 1)
        for r, ops in roles.items():
            for n in range(len(ops) - 1):  # swap each (turn, p_full) arrival pair back
                if ops[n][0] == ops[n + 1][0] == "arrive" and ops[n][1].startswith("tok") \
                        and ops[n + 1][1].startswith("p_full"):
                    ops[n], ops[n + 1] = ops[n + 1], ops[n]
        try:
            sync_model.run(roles, cnt, STAGES, trial, custom={"O": _OCheck(), "X": _ExpCheck(True)},
                           skewed=trial % 2 == 1)
        except AssertionError as e:
            failures += "passes early" in str(e)
    assert failures > 0


def test_turns_with_two_q_buffers_would_alias_their_phases():
    # why the kernel keeps turns to one Q buffer: with two, a slot runs a whole
    # item ahead through an item the other slot has no tile in
    rnd = random.Random(5)
    failures = 0
    for trial in range(100):
        items = _items(rnd)
        rnd2 = random.Random(trial)
        roles, cnt = _roles(items, 2, 4, rnd2, 1)
        try:
            sync_model.run(roles, cnt, STAGES, trial, custom={"O": _OCheck(), "X": _ExpCheck(True)},
                           skewed=trial % 2 == 1)
        except AssertionError as e:
            failures += "aliasing" in str(e)
    assert failures > 0


@pytest.mark.parametrize("name,NSB", [(n, b) for n in DROPS for b in (2, 1) if (n, b) not in IMPLIED])
def test_model_detects_a_dropped_wait(name, NSB):
    rnd = random.Random(17)
    failures = 0
    for trial in range(150):
        items = _items(rnd)
        try:
            run(items, 2 if NSB == 2 else 1, 4 if NSB == 2 else 2, trial, drop=DROPS[name], NSB=NSB)
        except AssertionError:
            failures += 1
    assert failures > 0, name


def _split_items(rnd):
    out = []
    for _ in range(rnd.randint(1, 5)):
        n = rnd.randint(1, 9)
        out.append(((n + 1) // 2, n // 2))
    return out


@pytest.mark.parametrize("QB,ST", [(2, 8), (2, 4)])
def test_split_mode_has_no_deadlock_aliasing_or_hazard(QB, ST):
    """One Q tile per item, the two slots on alternate key tiles, slot 1's
    results combined into slot 0's (dh <= 64)."""
    rnd = random.Random(QB * 100 + ST)
    for trial in range(200):
        items = _split_items(rnd)
        for seed in range(3):
            run(items, QB, ST, trial * 100 + seed, split=True)


SPLIT_DROPS = dict({n: d for n, d in DROPS.items() if n != "warps: tok"}, **{  # split mode: dh <= 64, no token
    # slot 0 would read slot 1's O, m, l before they are final
    "warps: split_ready": _drop("warp", "split_ready"),
    # slot 1 would free O_1 for the next item while slot 0 still reads it
    "warps: split_done": _drop("warp", "split_done"),
})


@pytest.mark.parametrize("name", list(SPLIT_DROPS))
def test_split_model_detects_a_dropped_wait(name):
    rnd = random.Random(31)
    failures = 0
    for trial in range(200):
        items = _split_items(rnd)
        try:
            run(items, 2, 4, trial, drop=SPLIT_DROPS[name], split=True)
        except AssertionError:
            failures += 1
    assert failures > 0, name
