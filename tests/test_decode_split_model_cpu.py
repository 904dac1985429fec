"""Python models of the decoding split paths' index arithmetic, run on the
CPU against the fp64 oracle: the register-resident path (below) and the
shared-memory path (at the end of the file, with the rule that picks a path).

The model follows the CUDA kernel's work split step by step: the range of
positions per CTA chosen from the SM count and the CTAs resident per SM, the
cache rows of all K/V heads of a range as one run, thread slot t taking rows
t, t + STEP, ... (always K/V head t mod H_kv), its private online softmax, the
warp butterfly over slots of the same head, the per-slot records and the
holders that merge them, the partial layout and the combine over
ceil(len / span) ranges.  Arithmetic is fp64, so any mistake in the mapping
shows as a mismatch far above rounding.  The grid size is a free parameter here
(any SM count and occupancy), which the GPU tests cannot vary.
"""
import itertools
import math

import numpy as np
import pytest

import oracle

THREADS = 256


def rows_step(dh):
    return THREADS * 8 // dh


def rows_min_span(dh, hkv):
    return 16 * rows_step(dh) // hkv


def rows_path(g, hkv, dh):
    return 1 <= g <= 4 and hkv >= 1 and (hkv & (hkv - 1)) == 0 and hkv <= rows_step(dh)


def span_for(B, N, Hkv, dh, sms, occ):
    want = (4 * sms * occ + B - 1) // B
    unit = rows_step(dh) // Hkv
    span = (N + want - 1) // want
    span = (span + unit - 1) // unit * unit
    return max(span, rows_min_span(dh, Hkv))


def _merge(m1, l1, o1, m2, l2, o2):
    mn = np.maximum(m1, m2)
    with np.errstate(invalid="ignore"):
        a = np.where(m1 == -np.inf, 0.0, np.exp2(m1 - mn))
        c = np.where(m2 == -np.inf, 0.0, np.exp2(m2 - mn))
    return mn, l1 * a + l2 * c, o1 * a[:, None] + o2 * c[:, None]


def model(q, k, v, lens, scale, sms, occ):
    B, Hq, dh = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    assert rows_path(g, Hkv, dh)
    L, STEP = dh // 8, rows_step(dh)
    P = 32 // L
    assert STEP == (THREADS // 32) * P
    span = span_for(B, N, Hkv, dh, sms, occ)
    n_split = (N + span - 1) // span
    assert n_split <= -(-N // rows_min_span(dh, Hkv))  # within the workspace bound
    part = np.full((B, Hkv, n_split, g, dh + 2), np.nan)
    sl2 = scale * math.log2(math.e)
    for b in range(B):
        ln = N if lens is None else min(max(lens[b], 0), N)
        for split in range(n_split):
            j0 = split * span
            j1 = min(ln, j0 + span)
            n_rows = max(j1 - j0, 0) * Hkv
            n_steps = (n_rows + STEP - 1) // STEP
            m = np.full((STEP, g), -np.inf)
            l = np.zeros((STEP, g))
            o = np.zeros((STEP, g, dh))
            for t in range(STEP):
                kvh = t & (Hkv - 1)
                qs = q[b, kvh * g : (kvh + 1) * g] * sl2
                for st in range(n_steps):
                    r = t + st * STEP
                    if r >= n_rows:
                        continue
                    j, hk = j0 + r // Hkv, r % Hkv
                    assert hk == kvh and j0 <= j < j1
                    sc = qs @ k[b, j, hk]
                    mn = np.maximum(m[t], sc)
                    with np.errstate(invalid="ignore"):
                        a = np.where(m[t] == -np.inf, 0.0, np.exp2(m[t] - mn))
                    w = np.exp2(sc - mn)
                    l[t] = l[t] * a + w
                    o[t] = o[t] * a[:, None] + w[:, None] * v[b, j, hk]
                    m[t] = mn
            off = Hkv * L  # butterfly over lane offsets that keep the head and the columns
            while off < 32:
                so = off // L
                new = [None] * STEP
                for t in range(STEP):
                    w_, sl = divmod(t, P)
                    pt = w_ * P + (sl ^ so)
                    assert (pt & (Hkv - 1)) == (t & (Hkv - 1))
                    new[t] = _merge(m[t], l[t], o[t], m[pt], l[pt], o[pt])
                for t in range(STEP):
                    m[t], l[t], o[t] = new[t]
                off <<= 1
            held = min(Hkv, P)
            rec = {t: (m[t], l[t], o[t]) for t in range(STEP) if t % P < held}
            n_hold = THREADS // 32 if Hkv <= P else STEP // Hkv
            for hk in range(Hkv):
                hs = [(i * P + hk) if Hkv <= P else (hk + i * Hkv) for i in range(n_hold)]
                assert all(x in rec and (x & (Hkv - 1)) == hk for x in hs)
                M = np.max([rec[x][0] for x in hs], axis=0)
                acc_l, acc_o = np.zeros(g), np.zeros((g, dh))
                for x in hs:
                    mx, lx, ox = rec[x]
                    with np.errstate(invalid="ignore"):
                        w = np.where(mx == -np.inf, 0.0, np.exp2(mx - M))
                    acc_l += lx * w
                    acc_o += ox * w[:, None]
                part[b, hk, split, :, :dh] = acc_o
                part[b, hk, split, :, dh] = M
                part[b, hk, split, :, dh + 1] = acc_l
    out, lse = np.zeros((B, Hq, dh)), np.zeros((B, Hq))
    for b in range(B):
        ln = N if lens is None else min(max(lens[b], 0), N)
        n_used = (ln + span - 1) // span
        for hq in range(Hq):
            kvh, hg = divmod(hq, g)
            ps = part[b, kvh, :n_used, hg]
            assert not np.isnan(ps).any()  # every range the combine reads was written
            if n_used == 0:
                out[b, hq], lse[b, hq] = 0.0, -np.inf
                continue
            M = ps[:, dh].max()
            w = np.exp2(ps[:, dh] - M)
            Ls = (ps[:, dh + 1] * w).sum()
            out[b, hq] = (ps[:, :dh] * w[:, None]).sum(0) / Ls
            lse[b, hq] = (M + math.log2(Ls)) * math.log(2)
    return out, lse


CASES = [
    ((3, 300, 8, 4, 16), [1, 128, 300]),
    ((2, 1000, 2, 1, 16), [999, 257]),
    ((2, 129, 4, 4, 128), None),
    ((4, 200, 12, 4, 64), [200, 129, 128, 5]),
    ((2, 300, 16, 16, 128), [300, 17]),
    ((1, 400, 32, 8, 64), None),
    ((2, 90, 16, 16, 64), [0, 90]),
    ((1, 3000, 8, 2, 128), [2999]),
]


@pytest.mark.parametrize("shape,lens", CASES, ids=lambda c: "x".join(map(str, c)) if isinstance(c, tuple) else str(c))
@pytest.mark.parametrize("sms,occ", [(148, 2), (148, 1), (2, 1)])
def test_register_resident_split_model_matches_oracle(shape, lens, sms, occ):
    B, N, Hq, Hkv, dh = shape
    rng = np.random.default_rng(B * 1000 + N + dh)
    q = rng.standard_normal((B, Hq, dh))
    k = rng.standard_normal((B, N, Hkv, dh))
    v = rng.standard_normal((B, N, Hkv, dh))
    out, lse = model(q, k, v, lens, 1 / math.sqrt(dh), sms, occ)
    keep = [i for i in range(B) if lens is None or lens[i] > 0]
    for i in set(range(B)) - set(keep):
        assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
    ref_out, ref_lse = oracle.sqa_decode(q[keep], k[keep], v[keep], None if lens is None else [lens[i] for i in keep])
    np.testing.assert_allclose(out[keep], ref_out, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse[keep], ref_lse, rtol=0, atol=1e-10)


@pytest.mark.parametrize("B,N,Hkv,dh", [(32, 32768, 4, 16), (8, 65536, 4, 128)])
def test_grid_of_the_decoding_workloads(B, N, Hkv, dh):
    # two resident CTAs per SM on 148 SMs give four full waves
    span = span_for(B, N, Hkv, dh, 148, 2)
    assert B * -(-N // span) == 4 * 148 * 2


# ----------------------------------------------------------------------------- general path


def decode_chunk(dh):
    return 256 if dh <= 32 else (128 if dh == 64 else 64)


def model_general(q, k, v, lens, scale):
    """The shared-memory split path: one CTA per (range of 4 chunks, K/V head,
    sequence); per chunk, all g heads' scores, block-wide online softmax."""
    B, Hq, dh = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    CH = decode_chunk(dh)
    span = 4 * CH
    n_split = -(-N // span)
    part = np.full((B, Hkv, n_split, g, dh + 2), np.nan)
    sl2 = scale * math.log2(math.e)
    for b, kvh, split in itertools.product(range(B), range(Hkv), range(n_split)):
        ln = N if lens is None else min(max(lens[b], 0), N)
        c_first = split * 4
        n_chunks = max(0, min(4, -(-ln // CH) - c_first))
        if n_chunks == 0:
            part[b, kvh, split, :, :dh] = 0.0
            part[b, kvh, split, :, dh] = -np.inf
            part[b, kvh, split, :, dh + 1] = 0.0
            continue
        qs = q[b, kvh * g : (kvh + 1) * g] * sl2
        m, l, o = np.full(g, -np.inf), np.zeros(g), np.zeros((g, dh))
        for c in range(n_chunks):
            j0 = (c_first + c) * CH
            cnt = min(CH, ln - j0)
            assert cnt > 0 and j0 + cnt <= ln
            s = np.full((g, CH), -np.inf)
            s[:, :cnt] = qs @ k[b, j0 : j0 + cnt, kvh].T
            mn = np.maximum(m, s.max(axis=1))
            w = np.exp2(s - mn[:, None])
            with np.errstate(invalid="ignore"):
                a = np.where(m == -np.inf, 0.0, np.exp2(m - mn))
            l = l * a + w.sum(axis=1)
            o = o * a[:, None] + w[:, :cnt] @ v[b, j0 : j0 + cnt, kvh]
            m = mn
        part[b, kvh, split, :, :dh] = o
        part[b, kvh, split, :, dh] = m
        part[b, kvh, split, :, dh + 1] = l
    out, lse = np.zeros((B, Hq, dh)), np.zeros((B, Hq))
    for b in range(B):
        ln = N if lens is None else min(max(lens[b], 0), N)
        n_used = -(-ln // span)
        for hq in range(Hq):
            kvh, hg = divmod(hq, g)
            ps = part[b, kvh, :n_used, hg]
            if n_used == 0:
                out[b, hq], lse[b, hq] = 0.0, -np.inf
                continue
            M = ps[:, dh].max()
            w = np.exp2(ps[:, dh] - M)
            Ls = (ps[:, dh + 1] * w).sum()
            out[b, hq] = (ps[:, :dh] * w[:, None]).sum(0) / Ls
            lse[b, hq] = (M + math.log2(Ls)) * math.log(2)
    return out, lse


GENERAL_CASES = [
    ((2, 1000, 16, 1, 16), [999, 257]),
    ((2, 3000, 128, 1, 16), [2999, 3]),
    ((2, 520, 16, 2, 128), [520, 131]),
    ((2, 500, 6, 3, 32), [500, 250]),
    ((2, 1100, 8, 1, 64), [0, 1100]),
    ((1, 256, 32, 4, 16), None),  # exactly one chunk
    ((1, 1025, 16, 2, 16), None),  # one position into the second range
]


@pytest.mark.parametrize("shape,lens", GENERAL_CASES, ids=lambda c: "x".join(map(str, c)) if isinstance(c, tuple) else str(c))
def test_shared_memory_split_model_matches_oracle(shape, lens):
    B, N, Hq, Hkv, dh = shape
    rng = np.random.default_rng(N + Hq)
    q = rng.standard_normal((B, Hq, dh))
    k = rng.standard_normal((B, N, Hkv, dh))
    v = rng.standard_normal((B, N, Hkv, dh))
    out, lse = model_general(q, k, v, lens, 1 / math.sqrt(dh))
    keep = [i for i in range(B) if lens is None or lens[i] > 0]
    for i in set(range(B)) - set(keep):
        assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
    ref_out, ref_lse = oracle.sqa_decode(q[keep], k[keep], v[keep], None if lens is None else [lens[i] for i in keep])
    np.testing.assert_allclose(out[keep], ref_out, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse[keep], ref_lse, rtol=0, atol=1e-10)


@pytest.mark.parametrize("g,hkv,dh,rows_path_expected", [(2, 4, 16, True), (4, 8, 128, True), (1, 16, 128, True),
                                                         (5, 1, 16, False), (16, 1, 16, False), (2, 3, 32, False),
                                                         (2, 32, 128, False), (4, 128, 16, True)])
def test_path_selection(g, hkv, dh, rows_path_expected):
    # the register-resident path takes groups of at most 4 heads whose K/V head
    # count is a power of two no larger than the rows a CTA takes per step
    assert rows_path(g, hkv, dh) == rows_path_expected
