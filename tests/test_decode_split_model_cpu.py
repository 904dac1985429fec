"""Python models of the decoding split paths' index arithmetic, run on the
CPU against the fp64 oracle: the register-resident path (below), the
shared-memory path (with the rule that picks a path) and the tensor-core path
(at the end of the file, at the level of mma.sync and ldmatrix fragments).

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


# ----------------------------------------------------------------------------- tensor-core path
#
# Fragment layouts of mma.sync.m16n8k16 (bf16 operands, fp32 accumulators) and
# ldmatrix, as the PTX ISA defines them, for lane t with r = t // 4, c = t % 4:
#   A (16 x 16, row-major):  a0 = A[r][2c:2c+2], a1 = A[r+8][2c:2c+2],
#                            a2 = A[r][2c+8:2c+10], a3 = A[r+8][2c+8:2c+10]
#   B (16 x 8, "col"):       b0 = B[2c:2c+2][r], b1 = B[2c+8:2c+10][r]
#   C/D (16 x 8):            d0, d1 = D[r][2c], D[r][2c+1]; d2, d3 = D[r+8][2c], D[r+8][2c+1]
#   ldmatrix .x4: lanes 8i..8i+7 give the row addresses of matrix i; lane t
#   receives M_i[r][2c:2c+2] (.trans: M_i[2c][r], M_i[2c+1][r]).
# The model holds registers as per-lane arrays and shared memory as 16-byte
# pieces, and runs the kernel's index arithmetic through these definitions.

MMA_STAGES = 3
LANES = np.arange(32)
FR, FC = LANES // 4, LANES % 4


def mma_path(g):
    return 5 <= g <= 16


def mma_chunk(dh):
    return 64 if dh == 128 else 128


def mma_piece(dh, row, j):
    p = dh // 8
    if p >= 8:
        return row * p + (j ^ (row & 7))
    sh = 1 if p == 4 else 2
    return row * p + (j ^ ((row >> sh) & (p - 1)))


def ldmatrix_x4(pieces, addr, trans=False):
    """pieces: [n][8] shared-memory pieces; addr[lane] = piece index.  Returns
    regs[4][32][2]."""
    regs = np.zeros((4, 32, 2))
    for i in range(4):
        m = pieces[addr[8 * i : 8 * i + 8]]  # 8 x 8, rows as addressed
        if trans:
            regs[i, :, 0] = m[2 * FC, FR]
            regs[i, :, 1] = m[2 * FC + 1, FR]
        else:
            regs[i, :, 0] = m[FR, 2 * FC]
            regs[i, :, 1] = m[FR, 2 * FC + 1]
    return regs


def mma16816(d, a, b0, b1):
    """d[32][4] += A B, A from a[4][32][2], B from b0, b1 [32][2]."""
    A = np.zeros((16, 16))
    B = np.zeros((16, 8))
    for h in range(2):
        A[FR, 2 * FC + h] = a[0][:, h]
        A[FR + 8, 2 * FC + h] = a[1][:, h]
        A[FR, 2 * FC + 8 + h] = a[2][:, h]
        A[FR + 8, 2 * FC + 8 + h] = a[3][:, h]
        B[2 * FC + h, FR] = b0[:, h]
        B[2 * FC + 8 + h, FR] = b1[:, h]
    D = A @ B
    d[:, 0] += D[FR, 2 * FC]
    d[:, 1] += D[FR, 2 * FC + 1]
    d[:, 2] += D[FR + 8, 2 * FC]
    d[:, 3] += D[FR + 8, 2 * FC + 1]


def shfl_xor(x, m):
    return x[LANES ^ m]


def model_mma(q, k, v, lens, scale):
    B, Hq, dh = q.shape
    N, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    assert mma_path(g)
    CH, P = mma_chunk(dh), dh // 8
    KS, NB = dh // 16, dh // 8
    span = 4 * decode_chunk(dh)  # the shared-memory path's span: the same workspace
    n_split = -(-N // span)
    part = np.full((B, Hkv, n_split, g, dh + 2), np.nan)
    sl2 = scale * math.log2(math.e)
    for b, kvh, split in itertools.product(range(B), range(Hkv), range(n_split)):
        ln = N if lens is None else min(max(lens[b], 0), N)
        r0, r1 = split * span, min(ln, split * span + span)
        rec = part[b, kvh, split]
        if r1 <= r0:
            rec[:, :dh], rec[:, dh], rec[:, dh + 1] = 0.0, -np.inf, 0.0
            continue
        n_chunks = -(-(r1 - r0) // CH)
        ring_k = np.full((MMA_STAGES, CH * P, 8), np.nan)
        ring_v = np.full((MMA_STAGES, CH * P, 8), np.nan)

        def load_chunk(ci):
            st = ci % MMA_STAGES
            for i in range(CH * P):
                row, j = divmod(i, P)
                pos = min(r0 + ci * CH + row, ln - 1)
                at = mma_piece(dh, row, j)
                ring_k[st, at] = k[b, pos, kvh, 8 * j : 8 * j + 8]
                ring_v[st, at] = v[b, pos, kvh, 8 * j : 8 * j + 8]

        qh = q[b, kvh * g : (kvh + 1) * g]
        qa = np.zeros((KS, 4, 32, 2))
        for ks in range(KS):
            k0 = ks * 16 + 2 * FC
            for slot, (rows, cols) in enumerate([(FR, k0), (FR + 8, k0), (FR, k0 + 8), (FR + 8, k0 + 8)]):
                for h in range(2):
                    qa[ks, slot, :, h] = np.where(rows < g, qh[np.minimum(rows, g - 1), cols + h], 0.0)
        for ci in range(min(n_chunks, MMA_STAGES - 1)):
            load_chunk(ci)
        warps = []
        for w in range(4):
            warps.append(dict(m0=np.full(32, -np.inf), m1=np.full(32, -np.inf), l0=np.zeros(32), l1=np.zeros(32),
                              o=np.zeros((NB, 32, 4))))
        KW = CH // 4
        NKB = KW // 8
        for ci in range(n_chunks):
            if ci + MMA_STAGES - 1 < n_chunks:
                load_chunk(ci + MMA_STAGES - 1)
            kbuf, vbuf = ring_k[ci % MMA_STAGES], ring_v[ci % MMA_STAGES]
            chunk_pos = r0 + ci * CH
            for w, st in enumerate(warps):
                key0 = w * KW
                s_ = [np.zeros((32, 4)) for _ in range(NKB)]
                for ks in range(KS):
                    for h in range(NKB // 2):
                        krow = key0 + 16 * h + (LANES & 7) + ((LANES >> 4) << 3)
                        kb = ldmatrix_x4(kbuf, mma_piece(dh, krow, 2 * ks + ((LANES >> 3) & 1)))
                        mma16816(s_[2 * h], qa[ks], kb[0], kb[1])
                        mma16816(s_[2 * h + 1], qa[ks], kb[2], kb[3])
                if chunk_pos + CH > r1:  # the range ends in this chunk
                    for nb in range(NKB):
                        kp = chunk_pos + key0 + 8 * nb + 2 * FC
                        s_[nb][kp >= r1, 0] = -np.inf
                        s_[nb][kp >= r1, 2] = -np.inf
                        s_[nb][kp + 1 >= r1, 1] = -np.inf
                        s_[nb][kp + 1 >= r1, 3] = -np.inf
                mx0 = np.max([np.maximum(x[:, 0], x[:, 1]) for x in s_], axis=0)
                mx1 = np.max([np.maximum(x[:, 2], x[:, 3]) for x in s_], axis=0)
                for sh in (1, 2):
                    mx0 = np.maximum(mx0, shfl_xor(mx0, sh))
                    mx1 = np.maximum(mx1, shfl_xor(mx1, sh))
                t0, t1 = mx0 * sl2, mx1 * sl2
                up0, up1 = t0 > st["m0"] + 8.0, t1 > st["m1"] + 8.0
                if (up0 | up1).any():  # warp vote
                    with np.errstate(invalid="ignore"):
                        a0 = np.where(up0 & (st["m0"] != -np.inf), np.exp2(st["m0"] - t0), 1.0)
                        a1 = np.where(up1 & (st["m1"] != -np.inf), np.exp2(st["m1"] - t1), 1.0)
                    st["m0"] = np.where(up0, t0, st["m0"])
                    st["m1"] = np.where(up1, t1, st["m1"])
                    st["l0"], st["l1"] = st["l0"] * a0, st["l1"] * a1
                    st["o"][:, :, 0:2] *= a0[None, :, None]
                    st["o"][:, :, 2:4] *= a1[None, :, None]
                nm0 = np.where(st["m0"] == -np.inf, 0.0, -st["m0"])
                nm1 = np.where(st["m1"] == -np.inf, 0.0, -st["m1"])
                pa = np.zeros((NKB // 2, 4, 32, 2))
                for nb in range(NKB):
                    p01 = np.exp2(s_[nb][:, 0:2] * sl2 + nm0[:, None])
                    p23 = np.exp2(s_[nb][:, 2:4] * sl2 + nm1[:, None])
                    st["l0"] = st["l0"] + p01.sum(1)
                    st["l1"] = st["l1"] + p23.sum(1)
                    pa[nb >> 1, (nb & 1) * 2 + 0] = p01
                    pa[nb >> 1, (nb & 1) * 2 + 1] = p23
                for h in range(NKB // 2):
                    for nb in range(0, NB, 2):
                        vrow = key0 + 16 * h + (LANES & 7) + (((LANES >> 3) & 1) << 3)
                        vb = ldmatrix_x4(vbuf, mma_piece(dh, vrow, nb + (LANES >> 4)), trans=True)
                        mma16816(st["o"][nb], pa[h], vb[0], vb[1])
                        mma16816(st["o"][nb + 1], pa[h], vb[2], vb[3])
        # merge the four warps into the record
        ms = np.zeros((4, 16))
        ls = np.zeros((4, 16))
        os_ = np.full((4, 16, dh), np.nan)
        for w, st in enumerate(warps):
            for nm in ("l0", "l1"):
                for sh in (1, 2):
                    st[nm] = st[nm] + shfl_xor(st[nm], sh)
            ms[w, FR], ms[w, FR + 8] = st["m0"], st["m1"]
        M = ms.max(0)
        for w, st in enumerate(warps):
            with np.errstate(invalid="ignore"):
                f0 = np.where(st["m0"] == -np.inf, 0.0, np.exp2(st["m0"] - M[FR]))
                f1 = np.where(st["m1"] == -np.inf, 0.0, np.exp2(st["m1"] - M[FR + 8]))
            ls[w, FR], ls[w, FR + 8] = st["l0"] * f0, st["l1"] * f1
            for nb in range(NB):
                col = nb * 8 + 2 * FC
                os_[w, FR, col] = st["o"][nb][:, 0] * f0
                os_[w, FR, col + 1] = st["o"][nb][:, 1] * f0
                os_[w, FR + 8, col] = st["o"][nb][:, 2] * f1
                os_[w, FR + 8, col + 1] = st["o"][nb][:, 3] * f1
        rec[:, :dh] = os_.sum(0)[:g]
        rec[:, dh] = M[:g]
        rec[:, dh + 1] = ls.sum(0)[:g]
    out, lse = np.zeros((B, Hq, dh)), np.zeros((B, Hq))
    for b in range(B):
        ln = N if lens is None else min(max(lens[b], 0), N)
        n_used = -(-ln // span)
        for hq in range(Hq):
            kvh, hg = divmod(hq, g)
            ps = part[b, kvh, :n_used, hg]
            assert not np.isnan(ps).any()
            if n_used == 0:
                out[b, hq], lse[b, hq] = 0.0, -np.inf
                continue
            M = ps[:, dh].max()
            w = np.exp2(ps[:, dh] - M)
            Ls = (ps[:, dh + 1] * w).sum()
            out[b, hq] = (ps[:, :dh] * w[:, None]).sum(0) / Ls
            lse[b, hq] = (M + math.log2(Ls)) * math.log(2)
    return out, lse


MMA_CASES = [
    ((2, 1100, 16, 1, 16), [1100, 257]),
    ((2, 300, 5, 1, 32), [300, 1]),
    ((1, 600, 24, 2, 64), [600]),
    ((2, 280, 8, 1, 128), [280, 65]),
    ((2, 200, 21, 3, 16), [0, 129]),
]


@pytest.mark.parametrize("shape,lens", MMA_CASES, ids=lambda c: "x".join(map(str, c)) if isinstance(c, tuple) else str(c))
def test_tensor_core_split_model_matches_oracle(shape, lens):
    B, N, Hq, Hkv, dh = shape
    rng = np.random.default_rng(N * 7 + Hq)
    q = rng.standard_normal((B, Hq, dh))
    k = rng.standard_normal((B, N, Hkv, dh))
    v = rng.standard_normal((B, N, Hkv, dh))
    out, lse = model_mma(q, k, v, lens, 1 / math.sqrt(dh))
    keep = [i for i in range(B) if lens is None or lens[i] > 0]
    for i in set(range(B)) - set(keep):
        assert np.all(out[i] == 0) and np.all(np.isneginf(lse[i]))
    ref_out, ref_lse = oracle.sqa_decode(q[keep], k[keep], v[keep], None if lens is None else [lens[i] for i in keep])
    np.testing.assert_allclose(out[keep], ref_out, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse[keep], ref_lse, rtol=0, atol=1e-10)


@pytest.mark.parametrize("dh", [16, 32, 64, 128])
def test_tensor_core_path_swizzle_is_conflict_free(dh):
    # every ldmatrix phase (8 consecutive rows, one 16-byte piece each) hits 8
    # different 16-byte bank groups, and the swizzle permutes each row's pieces
    p = dh // 8
    for row in range(mma_chunk(dh)):
        assert sorted(mma_piece(dh, row, j) for j in range(p)) == list(range(row * p, row * p + p))
    for row0 in range(0, mma_chunk(dh), 8):
        for j in range(p):
            groups = {mma_piece(dh, row0 + i, j) % 8 for i in range(8)}
            assert len(groups) == 8


@pytest.mark.parametrize("g,hkv,dh,path", [(4, 4, 16, "rows"), (5, 1, 16, "mma"), (16, 1, 16, "mma"),
                                           (8, 2, 128, "mma"), (17, 1, 64, "general"), (2, 3, 32, "general"),
                                           (3, 32, 128, "general"), (128, 1, 16, "general")])
def test_three_way_path_selection(g, hkv, dh, path):
    # register-resident first, then tensor cores for 5-16 heads, else shared memory
    got = "rows" if rows_path(g, hkv, dh) else ("mma" if mma_path(g) else "general")
    assert got == path


@pytest.mark.parametrize("dh", [16, 128])
def test_tensor_core_model_raises_the_reference_maximum(dh):
    # scores that grow along the cache (keys scaled up with their position) make
    # later steps exceed the reference maximum by more than 8 (log2 units), so
    # the rescale of O and l runs, mid-range and across warps
    B, N, Hq, Hkv = 1, 700, 10, 1
    rng = np.random.default_rng(dh)
    q = rng.standard_normal((B, Hq, dh))
    k = rng.standard_normal((B, N, Hkv, dh)) * (1.0 + np.arange(N) / 40.0)[None, :, None, None]
    v = rng.standard_normal((B, N, Hkv, dh))
    out, lse = model_mma(q, k, v, [N], 1 / math.sqrt(dh))
    ref_out, ref_lse = oracle.sqa_decode(q, k, v, [N])
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-9)
