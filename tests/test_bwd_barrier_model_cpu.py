"""A model of the synchronisation of the persistent dh 16/32 backward kernel
(``sqa_bwd_tf32_kernel``), run on the CPU under random schedules.

Each role of the kernel is a list of what it does, in the kernel's order: the
mbarrier waits and arrives, and the windows in which it uses a buffer.  The
roles are the TMA producer, issuer A (S^T / dP^T halves into three TMEM
buffers, then dQ), the DV and DK issuers, and the eight softmax warps (two
warpgroups; warpgroup w takes half w of every Q tile).  Every barrier has the kernel's arrival count; a use window of an
asynchronous copy or MMA ends where its completion arrives on a barrier.

The model fails on
* phase aliasing: a wait on phase k of a barrier finds it k + 2 completions
  ahead, so a parity wait would pass on the wrong phase;
* over-arrival, or deadlock (no role can move while some have not finished);
* a data hazard: every buffer version goes through its stages in order (for
  example an S^T buffer: written by issuer A's MMAs, rewritten in place by the
  4 warps of its half's warpgroup, read by the DV and DK MMAs), each stage with its number of
  users; a use that starts before every user of the previous stage (or of the
  previous version) has finished is a hazard.

The checker is ``sync_model.run``.  Random schedules over random work lists
(items of 1-6 Q tiles, several items per CTA) and both Q/dO stage counts the kernel uses (4 at dh 16, 2 at dh 32)
cover the interleavings a GPU may produce.
"""
import random

import pytest
import sync_model

NBUF = 3  # S^T / dP^T TMEM buffers
NWG = 2   # softmax warpgroups
WARPS = 4 * NWG

# Stages of every version of each buffer: (who, number of users).
STAGES = {
    "kv": [("producer writes K, V", 1), ("issuer A reads", 1)],
    "stage": [("producer writes Q, dO, stats", 1), ("issuer A, DV, DK and the warps read", 3 + WARPS)],
    # the fp32 image of a stage's dO (Q): built by the DV (DK) warp from the
    # bf16 tile, read by that warp's MMAs
    "img_acc_dv": [("DV converts dO", 1), ("DV MMAs read", 1)],
    "img_acc_dk": [("DK converts Q", 1), ("DK MMAs read", 1)],
    "S": [("issuer A writes S^T, dP^T", 1), ("the half's warpgroup rewrites P^T, dS^T", 4), ("DV and DK read", 2)],
    "dsbuf": [("warps write dS", WARPS), ("issuer A reads (dQ)", 1)],
    "dqtm": [("issuer A writes dQ", 1), ("warps read dQ", WARPS)],
    "acc_dv": [("DV accumulates dV", 1), ("warps read dV", WARPS)],
    "acc_dk": [("DK accumulates dK", 1), ("warps read dK", WARPS)],
}


def _roles(nqs, QS):
    cnt = {}

    def bar(name, n):
        cnt[name] = n

    for kb in range(2):
        bar(f"kv_full{kb}", 1)
        bar(f"kv_empty{kb}", 1)
    for s in range(QS):
        bar(f"qd_full{s}", 1)
        bar(f"qd_empty{s}", 3)  # issuer A (after dQ), DV and DK
    for x in range(NBUF):
        bar(f"s_full{x}", 1)
        bar(f"ds_ready{x}", 128)  # the warpgroup that owns the half
        bar(f"kvmma_done{x}", 2)
    for w in range(NWG):
        bar(f"dsq_ready{w}", 128)
    for x in range(2):
        bar(f"dq_full{x}", 1)
        bar(f"dq_empty{x}", 32 * WARPS)
    bar("dkv_final", 2)
    bar("dkv_free", 32 * WARPS)

    def W(b, k):
        return ("wait", b, k)

    def A(b, m=1):
        return ("arrive", b, m)

    def B(res, slot, v, stage):  # begin using version v of buffer res[slot] in the given stage
        return ("begin", (res, slot), v, stage)

    def E(res, slot, v, stage):
        return ("end", (res, slot), v, stage)

    prod, gt = [], 0
    for r, nq in enumerate(nqs):
        kb = r & 1
        if r >= 2:
            prod.append(W(f"kv_empty{kb}", (r >> 1) - 1))
        prod += [B("kv", kb, r, 0), E("kv", kb, r, 0), A(f"kv_full{kb}")]
        for i in range(nq):
            G = gt + i
            s = G % QS
            if G >= QS:
                prod.append(W(f"qd_empty{s}", G // QS - 1))
            prod += [B("stage", s, G, 0), E("stage", s, G, 0), A(f"qd_full{s}")]
        gt += nq

    issuer_a, gt = [], 0
    for r, nq in enumerate(nqs):
        kb, nh = r & 1, 2 * nq
        issuer_a += [W(f"kv_full{kb}", r >> 1), B("kv", kb, r, 1)]

        def half(hl, gt=gt):
            G, H = gt + (hl >> 1), 2 * gt + hl
            s, x = G % QS, H % NBUF
            ops = []
            if hl % 2 == 0:
                ops += [W(f"qd_full{s}", G // QS), B("stage", s, G, 1)]
            if H >= NBUF:
                ops.append(W(f"kvmma_done{x}", H // NBUF - 1))
            ops += [B("S", x, H, 0), E("S", x, H, 0), A(f"s_full{x}")]
            if hl % 2 == 1:
                ops.append(E("stage", s, G, 1))  # both halves' MMAs have read Q and dO
            return ops

        for hl in range(min(NBUF, nh)):
            issuer_a += half(hl)
        for i in range(nq):
            G = gt + i
            if 2 * i + 3 < nh:  # the next tile's second half goes ahead of this tile's dQ
                issuer_a += half(2 * i + 3)
            issuer_a += [W(f"dsq_ready{w}", G) for w in range(NWG)]
            issuer_a.append(B("dsbuf", G & 1, G, 1))
            if G >= 2:
                issuer_a.append(W(f"dq_empty{G & 1}", (G >> 1) - 1))
            issuer_a += [B("dqtm", G & 1, G, 0), E("dsbuf", G & 1, G, 1), E("dqtm", G & 1, G, 0)]
            issuer_a += [A(f"dq_full{G & 1}"), A(f"qd_empty{G % QS}")]
            if 2 * i + 4 < nh:
                issuer_a += half(2 * i + 4)
        issuer_a += [E("kv", kb, r, 1), A(f"kv_empty{kb}")]
        gt += nq

    def kv_issuer(acc):  # DV and DK issuers: the same sequence on their own accumulator
        ops, gt = [], 0
        for r, nq in enumerate(nqs):
            img = "img_" + acc
            for hl in range(2 * nq):
                G, H = gt + (hl >> 1), 2 * gt + hl
                s, x = G % QS, H % NBUF
                if hl % 2 == 0:  # the tile's fp32 image, from the bf16 tile
                    ops += [W(f"qd_full{s}", G // QS), B("stage", s, G, 1), B(img, s, G, 0), E(img, s, G, 0),
                            E("stage", s, G, 1)]
                ops.append(W(f"ds_ready{x}", H // NBUF))
                if hl == 0 and r > 0:
                    ops.append(W("dkv_free", r - 1))
                if hl == 0:
                    ops.append(B(acc, 0, r, 0))
                if hl % 2 == 0:
                    ops.append(B(img, s, G, 1))
                ops += [B("S", x, H, 2), E("S", x, H, 2), A(f"kvmma_done{x}")]
                if hl % 2 == 1:
                    ops += [E(img, s, G, 1), A(f"qd_empty{s}")]
            ops += [E(acc, 0, r, 0), A("dkv_final")]
            gt += nq
        return ops

    def softmax_warp(w):  # one warp (32 arrivals) of warpgroup w
        ops, gt = [], 0
        for r, nq in enumerate(nqs):
            for i in range(nq):
                G = gt + i
                s = G % QS
                ops += [W(f"qd_full{s}", G // QS), B("stage", s, G, 1)]
                if G >= 2:  # the dQ MMA of tile G - 2 has read this dS buffer
                    ops.append(W(f"dq_full{G & 1}", (G >> 1) - 1))
                ops.append(B("dsbuf", G & 1, G, 0))
                H = 2 * G + w  # warpgroup w owns half w of every tile
                x = H % NBUF
                ops += [W(f"s_full{x}", H // NBUF), B("S", x, H, 1), E("S", x, H, 1), A(f"ds_ready{x}", 32)]
                ops.append(E("dsbuf", G & 1, G, 0))
                if G > 0:
                    ops.append(W(f"dq_full{(G - 1) & 1}", (G - 1) >> 1))
                ops += [E("stage", s, G, 1), A(f"dsq_ready{w}", 32)]
                if i > 0:
                    P = G - 1
                    ops += [B("dqtm", P & 1, P, 1), E("dqtm", P & 1, P, 1), A(f"dq_empty{P & 1}", 32)]
            G = gt + nq - 1
            ops += [W(f"dq_full{G & 1}", G >> 1), B("dqtm", G & 1, G, 1), E("dqtm", G & 1, G, 1),
                    A(f"dq_empty{G & 1}", 32)]
            ops += [W("dkv_final", r), B("acc_dv", 0, r, 1), B("acc_dk", 0, r, 1), E("acc_dv", 0, r, 1),
                    E("acc_dk", 0, r, 1), A("dkv_free", 32)]
            gt += nq
        return ops

    roles = {"producer": prod, "issuer_a": issuer_a, "dv": kv_issuer("acc_dv"), "dk": kv_issuer("acc_dk")}
    for k in range(WARPS):
        roles[f"warp{k}"] = softmax_warp(k // 4)
    return roles, cnt


def run(nqs, QS, seed, drop=None):
    """One random schedule.  drop(role, op) -> True removes that op (used only
    to show that the model notices a missing wait)."""
    roles, cnt = _roles(nqs, QS)
    if drop is not None:
        roles = {r: [op for op in ops if not drop(r, op)] for r, ops in roles.items()}
    sync_model.run(roles, cnt, STAGES, seed)


@pytest.mark.parametrize("QS", [2, 4])
def test_backward_protocol_has_no_deadlock_aliasing_or_hazard(QS):
    rnd = random.Random(QS)
    for trial in range(120):
        nqs = [rnd.randint(1, 6) for _ in range(rnd.randint(1, 5))]
        for seed in range(4):
            run(nqs, QS, seed * 1000 + trial)


def _drop_wait(role_prefix, barrier):
    def drop(r, op):
        return r.startswith(role_prefix) and op[0] == "wait" and op[1].startswith(barrier)
    return drop


# Waits whose removal the model must notice.  (Two other waits of the kernel
# are implied by the rest of the protocol and the model shows no failure
# without them: the DV/DK issuers' dkv_free wait, because their next ds_ready
# wait already follows every warp's dV/dK epilogue, and issuer A's dq_empty
# wait, because its dsq_ready wait already follows every warp's dQ epilogue of
# tile G - 2.  The kernel keeps them as a second guard.)
DROPS = {
    # issuer A would refill an S^T / dP^T buffer that DV and DK still read
    "issuer A: kvmma_done": _drop_wait("issuer_a", "kvmma_done"),
    # the producer would overwrite a Q / dO stage still being read
    "producer: qd_empty": _drop_wait("producer", "qd_empty"),
    # the producer would overwrite a K / V buffer issuer A still reads
    "producer: kv_empty": _drop_wait("producer", "kv_empty"),
    # DV / DK would read P^T, dS^T before the warps wrote them
    "dv: ds_ready": _drop_wait("dv", "ds_ready"),
    "dk: ds_ready": _drop_wait("dk", "ds_ready"),
    # the warps would read S^T before issuer A's MMAs wrote it
    "warps: s_full": _drop_wait("warp", "s_full"),
    # issuer A's dQ MMA would read dS before every warp wrote it
    "issuer A: dsq_ready": _drop_wait("issuer_a", "dsq_ready"),
    # DV / DK would build an fp32 image from a bf16 tile that has not landed,
    # over the image their MMAs of tile G - QS may still read
    "dv: qd_full": _drop_wait("dv", "qd_full"),
    "dk: qd_full": _drop_wait("dk", "qd_full"),
}


@pytest.mark.parametrize("name", list(DROPS))
def test_model_detects_a_dropped_wait(name):
    failures = 0
    rnd = random.Random(11)
    for trial in range(150):
        nqs = [rnd.randint(1, 6) for _ in range(rnd.randint(2, 5))]
        try:
            run(nqs, 2, trial, drop=DROPS[name])
        except AssertionError:
            failures += 1
    assert failures > 0, name


def test_model_detects_the_wait_before_the_dq_epilogue_missing():
    """The warps' wait for the dQ MMA of tile G - 1 (just before they signal
    their dS of tile G) also guards their read of that dQ from TMEM: without it
    the read can start before the MMA has written it."""
    rnd = random.Random(3)
    failures = 0
    for trial in range(150):
        nqs = [rnd.randint(2, 6) for _ in range(rnd.randint(1, 4))]
        ops = _roles(nqs, 2)[0]["warp0"]
        before_signal = {ops[i] for i in range(len(ops) - 1)
                         if ops[i][0] == "wait" and ops[i][1].startswith("dq_full")
                         and ops[i + 1][0] == "end" and ops[i + 1][1][0] == "stage"}
        try:
            run(nqs, 2, trial, drop=lambda r, op: r.startswith("warp") and op in before_signal)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_detects_the_hoisted_dq_wait_missing():
    """Without the warps' wait for the dQ MMA of tile G - 2 before writing dS
    of tile G into the same shared-memory buffer (the wait just before the
    buffer's use begins), some schedule overwrites dS that the dQ MMA still
    reads."""
    rnd = random.Random(5)
    failures = 0
    for trial in range(150):
        nqs = [rnd.randint(2, 6) for _ in range(rnd.randint(1, 4))]
        ops = _roles(nqs, 2)[0]["warp0"]
        hoisted = {ops[i] for i in range(len(ops) - 1)
                   if ops[i][0] == "wait" and ops[i][1].startswith("dq_full")
                   and ops[i + 1][0] == "begin" and ops[i + 1][1][0] == "dsbuf"}
        try:
            run(nqs, 2, trial, drop=lambda r, op: r.startswith("warp") and op in hoisted)
        except AssertionError:
            failures += 1
    assert failures > 0
