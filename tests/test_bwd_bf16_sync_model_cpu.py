"""A model of the synchronisation of the dh 64/128 backward kernel
(``sqa_bwd_kernel`` in sqa_bwd_bf16.cuh: one CTA per 128-key tile), run on
the CPU under random schedules with the checker in ``sync_model``.

Roles, in the kernel's program order:
* the TMA producer: K and V once; the first two Q/dO stages; then, per tile,
  the next tile's -lse2 once the warps have finished P^T (p_ready of the second
  half), its -D once they have finished dS (ds_ready), and the Q/dO tile two
  ahead once the stage is free (qd_empty);
* the MMA-issuing warp: S^T, dP^T (after the dQ of the previous tile was read
  out), dV per half of 64 query rows (after that half's p_ready), dK and dQ
  (after ds_ready); MMAs of one issuer run in order, so they are modelled at
  their place in its program, and everything the other roles learn about them
  comes through commits that follow them;
* the eight softmax warps: P^T of both halves (rewriting S^T's columns), dS^T
  (rewriting dP^T's columns) and dS into shared memory, the dQ read-out, the
  dV/dK epilogue.

TMEM columns [128, 256) go through dP^T written, dS^T rewritten, dS^T read by
the dK MMA, dQ written and dQ read out before the next tile's dP^T.  Barrier
arrival counts are the kernel's.
"""
import random

import pytest
import sync_model

WARPS = 8
QS = 2


def _stages():
    return {
        "kv": [("producer writes K, V", 1), ("issuer reads", 1)],
        "stage": [("producer writes Q, dO", 1), ("MMAs read Q, dO", 1)],
        "lse": [("producer writes -lse2", 1), ("warps read -lse2", WARPS)],
        "dbuf": [("producer writes -D", 1), ("warps read -D", WARPS)],
        "ST": [("S^T write", 1), ("warps rewrite P^T", WARPS), ("dV MMA reads P^T", 1)],
        "DPT": [("dP^T write", 1), ("warps rewrite dS^T", WARPS), ("dK MMA reads dS^T", 1),
                ("dQ write (same columns)", 1), ("warps read dQ", WARPS)],
        "dsbuf": [("warps write dS", WARPS), ("dQ MMA reads dS", 1)],
        "acc_dv": [("issuer accumulates dV", 1), ("warps read dV", WARPS)],
        "acc_dk": [("issuer accumulates dK", 1), ("warps read dK", WARPS)],
    }


def _roles(nq):
    cnt = {"kv_full": 1, "lse_full": 1, "d_full": 1, "s_full": 1, "dp_full": 1, "p_ready0": 32 * WARPS,
           "p_ready1": 32 * WARPS, "ds_ready": 32 * WARPS, "dq_full": 1, "dq_empty": 32 * WARPS, "dkv_final": 1}
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

    def write(res, v, stage, slot=0):
        return [B(res, v, stage, slot), E(res, v, stage, slot)]

    prod = write("kv", 0, 0) + [A("kv_full")]
    prod += write("lse", 0, 0) + [A("lse_full")] + write("dbuf", 0, 0) + [A("d_full")]
    for i in range(min(QS, nq)):
        prod += write("stage", i, 0, i % QS) + [A(f"qd_full{i % QS}")]
    for i in range(nq - 1):
        prod += [W("p_ready1", i)] + write("lse", i + 1, 0) + [A("lse_full")]
        prod += [W("ds_ready", i)] + write("dbuf", i + 1, 0) + [A("d_full")]
        if i + QS < nq:
            s = i % QS
            prod += [W(f"qd_empty{s}", i // QS)] + write("stage", i + QS, 0, s) + [A(f"qd_full{s}")]

    iss = [W("kv_full", 0), B("kv", 0, 1), B("acc_dv", 0, 0), B("acc_dk", 0, 0)]
    for i in range(nq):
        s = i % QS
        iss += [W(f"qd_full{s}", i // QS), B("stage", i, 1, s)]
        iss += [B("ST", i, 0, 0), B("ST", i, 0, 1), E("ST", i, 0, 0), E("ST", i, 0, 1), A("s_full")]
        if i > 0:
            iss.append(W("dq_empty", i - 1))
        iss += write("DPT", i, 0) + [A("dp_full")]
        for hh in range(2):
            iss += [W(f"p_ready{hh}", i)] + write("ST", i, 2, hh)
        iss += [W("ds_ready", i)] + write("DPT", i, 2) + [E("stage", i, 1, s), A(f"qd_empty{s}")]
        iss += [B("dsbuf", i, 1), B("DPT", i, 3), E("dsbuf", i, 1), E("DPT", i, 3), A("dq_full")]
    iss += [E("acc_dv", 0, 0), E("acc_dk", 0, 0), A("dkv_final"), E("kv", 0, 1)]

    def warp():
        ops = []
        for i in range(nq):
            ops += [W("s_full", i), W("lse_full", i), B("lse", i, 1)]
            for hh in range(2):
                ops += write("ST", i, 1, hh)
                if hh == 1:
                    ops.append(E("lse", i, 1))
                ops.append(A(f"p_ready{hh}", 32))
            ops += [W("dp_full", i), W("d_full", i), B("dbuf", i, 1), B("DPT", i, 1), B("dsbuf", i, 0),
                    E("DPT", i, 1), E("dsbuf", i, 0), E("dbuf", i, 1), A("ds_ready", 32)]
            ops += [W("dq_full", i)] + write("DPT", i, 4) + [A("dq_empty", 32)]
        ops += [W("dkv_final", 0), B("acc_dv", 0, 1), B("acc_dk", 0, 1), E("acc_dv", 0, 1), E("acc_dk", 0, 1)]
        return ops

    roles = {"producer": prod, "issuer": iss}
    for w in range(WARPS):
        roles[f"warp{w}"] = warp()
    return roles, cnt


def run(nq, seed, drop=None):
    roles, cnt = _roles(nq)
    if drop is not None:
        roles = {r: [op for op in ops if not drop(r, op)] for r, ops in roles.items()}
    sync_model.run(roles, cnt, _stages(), seed, skewed=seed % 2 == 1)


def test_protocol_has_no_deadlock_aliasing_or_hazard():
    rnd = random.Random(128)
    for trial in range(300):
        run(rnd.randint(1, 12), trial)


def _drop(role_prefix, barrier):
    return lambda r, op: r.startswith(role_prefix) and op[0] == "wait" and op[1].startswith(barrier)


DROPS = {
    # dP^T of the next tile would overwrite dQ the warps still read
    "issuer: dq_empty": _drop("issuer", "dq_empty"),
    # dV would read P^T before the warps wrote it
    "issuer: p_ready": _drop("issuer", "p_ready"),
    # dK / dQ would read dS^T / dS before the warps wrote them
    "issuer: ds_ready": _drop("issuer", "ds_ready"),
    # the MMAs would read a Q/dO stage before it landed
    "issuer: qd_full": _drop("issuer", "qd_full"),
    # the warps would read S^T, dP^T or dQ before the MMA wrote it
    "warps: s_full": _drop("warp", "s_full"),
    "warps: dp_full": _drop("warp", "dp_full"),
    "warps: dq_full": _drop("warp", "dq_full"),
    # the warps would read statistics before they landed
    "warps: lse_full": _drop("warp", "lse_full"),
    "warps: d_full": _drop("warp", "d_full"),
    # the epilogue would read dV / dK before the last MMA
    "warps: dkv_final": _drop("warp", "dkv_final"),
    # the producer would overwrite statistics or a Q/dO stage still in use
    "producer: p_ready": _drop("producer", "p_ready"),
    "producer: ds_ready": _drop("producer", "ds_ready"),
    "producer: qd_empty": _drop("producer", "qd_empty"),
}


@pytest.mark.parametrize("name", list(DROPS))
def test_model_detects_a_dropped_wait(name):
    rnd = random.Random(23)
    failures = 0
    for trial in range(300):
        try:
            run(rnd.randint(2, 10), trial, drop=DROPS[name])
        except AssertionError:
            failures += 1
    assert failures > 0, name
