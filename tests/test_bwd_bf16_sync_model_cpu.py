"""A model of the synchronisation of the dh 64/128 backward kernel
(``sqa_bwd_kernel``: one CTA per 128-key tile), run on the CPU under random
schedules with the checker in ``sync_model``.

Roles, in the kernel's program order: the TMA producer (K and V once, then the
Q/dO stages with their statistics), the MMA-issuing warp (S^T and dP^T, then
dV += P^T dO and dK += dS^T Q, then dQ = dS K) and the eight softmax warps
(P^T and dS^T rewritten in TMEM, dS into shared memory, the dQ epilogue, the
dV/dK epilogue).  At dh 128 the dQ accumulator reuses S^T's TMEM columns, so
one buffer version goes through S written, P^T rewritten, P^T read by the dV
MMA, dQ written, dQ read; the S^T MMA of the next tile must wait until the
warps have read dQ.  At dh 64 dQ has its own columns.  Barrier arrival counts
are the kernel's.
"""
import random

import pytest
import sync_model

WARPS = 8


def _stages(shared):
    st = [("S^T write", 1), ("warps rewrite P^T", WARPS), ("dV MMA reads P^T", 1)]
    if shared:
        st += [("dQ write (same columns)", 1), ("warps read dQ", WARPS)]
    return {
        "kv": [("producer writes K, V", 1), ("issuer reads", 1)],
        "stage": [("producer writes Q, dO, stats", 1), ("issuer and warps read", 1 + WARPS)],
        "ST": st,
        "DPT": [("dP^T write", 1), ("warps rewrite dS^T", WARPS), ("dK MMA reads dS^T", 1)],
        "DQ": [("dQ write", 1), ("warps read dQ", WARPS)],
        "dsbuf": [("warps write dS", WARPS), ("dQ MMA reads dS", 1)],
        "acc_dv": [("issuer accumulates dV", 1), ("warps read dV", WARPS)],
        "acc_dk": [("issuer accumulates dK", 1), ("warps read dK", WARPS)],
    }


def _roles(nq, QS, shared):
    cnt = {"kv_full": 1, "s_full": 1, "ds_ready": 32 * WARPS, "dq_full": 1, "dq_empty": 32 * WARPS, "dkv_final": 1}
    for s in range(QS):
        cnt[f"qd_full{s}"] = 1
        cnt[f"qd_empty{s}"] = 1

    def W(b, k):
        return ("wait", b, k)

    def A(b, m=1):
        return ("arrive", b, m)

    def B(res, v, stage, slot=0):
        return ("begin", (res, slot), v, stage)

    def E(res, v, stage, slot=0):
        return ("end", (res, slot), v, stage)

    prod = [B("kv", 0, 0), E("kv", 0, 0), A("kv_full")]
    for i in range(nq):
        s = i % QS
        if i >= QS:
            prod.append(W(f"qd_empty{s}", i // QS - 1))
        prod += [B("stage", i, 0, s), E("stage", i, 0, s), A(f"qd_full{s}")]

    dq_res, dq_w, dq_r = ("ST", 3, 4) if shared else ("DQ", 0, 1)
    iss = [W("kv_full", 0), B("kv", 0, 1)]
    for i in range(nq):
        s = i % QS
        iss += [W(f"qd_full{s}", i // QS), B("stage", i, 1, s)]
        if shared and i > 0:  # S^T overwrites the columns of dQ (i - 1)
            iss.append(W("dq_empty", i - 1))
        iss += [B("ST", i, 0), B("DPT", i, 0), E("ST", i, 0), E("DPT", i, 0), A("s_full")]
        iss.append(W("ds_ready", i))
        if i == 0:
            iss += [B("acc_dv", 0, 0), B("acc_dk", 0, 0)]
        # MMAs of one issuer run in order: the dV/dK reads end before dQ writes
        iss += [B("ST", i, 2), B("DPT", i, 2), E("ST", i, 2), E("DPT", i, 2), E("stage", i, 1, s)]
        if not shared and i > 0:
            iss.append(W("dq_empty", i - 1))
        iss += [B("dsbuf", i, 1), B(dq_res, i, dq_w), E("dsbuf", i, 1), E(dq_res, i, dq_w)]
        iss += [A("dq_full"), A(f"qd_empty{s}")]
    iss += [E("acc_dv", 0, 0), E("acc_dk", 0, 0), A("dkv_final"), E("kv", 0, 1)]

    def warp():
        ops = []
        for i in range(nq):
            s = i % QS
            ops += [W(f"qd_full{s}", i // QS), W("s_full", i), B("stage", i, 1, s), B("ST", i, 1), B("DPT", i, 1),
                    B("dsbuf", i, 0), E("ST", i, 1), E("DPT", i, 1), E("dsbuf", i, 0), E("stage", i, 1, s),
                    A("ds_ready", 32)]
            ops += [W("dq_full", i), B(dq_res, i, dq_r), E(dq_res, i, dq_r), A("dq_empty", 32)]
        ops += [W("dkv_final", 0), B("acc_dv", 0, 1), B("acc_dk", 0, 1), E("acc_dv", 0, 1), E("acc_dk", 0, 1)]
        return ops

    roles = {"producer": prod, "issuer": iss}
    for w in range(WARPS):
        roles[f"warp{w}"] = warp()
    return roles, cnt


def run(nq, dh, seed, drop=None):
    QS, shared = (1, True) if dh == 128 else (2, False)
    roles, cnt = _roles(nq, QS, shared)
    if drop is not None:
        roles = {r: [op for op in ops if not drop(r, op)] for r, ops in roles.items()}
    sync_model.run(roles, cnt, _stages(shared), seed)


@pytest.mark.parametrize("dh", [64, 128])
def test_protocol_has_no_deadlock_aliasing_or_hazard(dh):
    rnd = random.Random(dh)
    for trial in range(200):
        run(rnd.randint(1, 12), dh, trial)


def _drop(role_prefix, barrier):
    return lambda r, op: r.startswith(role_prefix) and op[0] == "wait" and op[1].startswith(barrier)


DROPS = {
    # the issuer's next S^T (dh 128) or dQ (dh 64) would overwrite dQ the warps still read
    "issuer: dq_empty": _drop("issuer", "dq_empty"),
    # dV / dK / dQ MMAs would read P^T, dS^T, dS before the warps wrote them
    "issuer: ds_ready": _drop("issuer", "ds_ready"),
    # the warps would read S^T before the MMA wrote it
    "warps: s_full": _drop("warp", "s_full"),
    # the warps would read dQ before the MMA wrote it
    "warps: dq_full": _drop("warp", "dq_full"),
    # the epilogue would read dV / dK before the last MMA
    "warps: dkv_final": _drop("warp", "dkv_final"),
    # the producer would overwrite a Q/dO stage still in use
    "producer: qd_empty": _drop("producer", "qd_empty"),
}


# At dh 64 the issuer's dq_empty wait is implied: its dQ MMA of tile i also
# waits for ds_ready of tile i, which every warp signals only after reading dQ
# of tile i - 1.  At dh 128 the S^T MMA, which comes before that wait, reuses
# dQ's columns, so there the wait is needed.
IMPLIED = {("issuer: dq_empty", 64)}


@pytest.mark.parametrize("name,dh", [(n, d) for n in DROPS for d in (64, 128) if (n, d) not in IMPLIED])
def test_model_detects_a_dropped_wait(name, dh):
    rnd = random.Random(23)
    failures = 0
    for trial in range(200):
        try:
            run(rnd.randint(2, 10), dh, trial, drop=DROPS[name])
        except AssertionError:
            failures += 1
    assert failures > 0, (name, dh)
