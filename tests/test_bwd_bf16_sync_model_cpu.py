"""Models of the synchronisation of the dh 64/128 backward kernels, run on the
CPU under random schedules with the checker in ``sync_model``.

``sqa_bwd_kernel`` (dK and dV, one CTA per 128-key tile), in program order:
* the TMA producer: K and V once; the first two Q/dO stages; then, per tile,
  the next tile's -lse2 once the warps have finished P^T (p_ready of the second
  half), its -D once they have finished dS^T (ds_ready), and the Q/dO tile two
  ahead once the stage is free (qd_empty);
* the MMA-issuing warp: S^T and dP^T of the first tile, then per tile dV per
  half of 64 query rows (after that half's p_ready), S^T of the next tile,
  dK (after ds_ready) and dP^T of the next tile; MMAs of one issuer run in
  order, so they are modelled at their place in its program, and everything the
  other roles learn about them comes through commits that follow them;
* the eight softmax warps: P^T of both halves (rewriting S^T's columns), dS^T
  (rewriting dP^T's columns), the dV/dK epilogue.

``sqa_bwd_q_kernel`` (dQ, one CTA per stacked Q tile): the producer streams
K/V through a ring; the warps put Q and dO into TMEM; two issuers run S_j and
dP_j into buffer j % 2, a third dQ of j once dS_j is ready; the warps turn S_j and dP_j into
dS_j in place; the epilogue reads dQ.  Barrier arrival counts are the kernels'.
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
        "DPT": [("dP^T write", 1), ("warps rewrite dS^T", WARPS), ("dK MMA reads dS^T", 1)],
        "acc_dv": [("issuer accumulates dV", 1), ("warps read dV", WARPS)],
        "acc_dk": [("issuer accumulates dK", 1), ("warps read dK", WARPS)],
    }


def _roles(nq):
    cnt = {"kv_full": 1, "lse_full": 1, "d_full": 1, "s_full": 1, "dp_full": 1, "p_ready0": 32 * WARPS,
           "p_ready1": 32 * WARPS, "ds_ready": 32 * WARPS, "dkv_final": 1}
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
    iss += [W("qd_full0", 0), B("stage", 0, 1, 0)]
    iss += [B("ST", 0, 0, 0), B("ST", 0, 0, 1), E("ST", 0, 0, 0), E("ST", 0, 0, 1), A("s_full")]
    iss += write("DPT", 0, 0) + [A("dp_full")]
    for i in range(nq):
        s, s1 = i % QS, (i + 1) % QS
        for hh in range(2):
            iss += [W(f"p_ready{hh}", i)] + write("ST", i, 2, hh)
        if i + 1 < nq:
            iss += [W(f"qd_full{s1}", (i + 1) // QS), B("stage", i + 1, 1, s1)]
            iss += [B("ST", i + 1, 0, 0), B("ST", i + 1, 0, 1), E("ST", i + 1, 0, 0), E("ST", i + 1, 0, 1),
                    A("s_full")]
        iss += [W("ds_ready", i)] + write("DPT", i, 2) + [E("stage", i, 1, s), A(f"qd_empty{s}")]
        if i + 1 < nq:
            iss += write("DPT", i + 1, 0) + [A("dp_full")]
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
            ops += [W("dp_full", i), W("d_full", i), B("dbuf", i, 1), B("DPT", i, 1), E("DPT", i, 1),
                    E("dbuf", i, 1), A("ds_ready", 32)]
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
    # dV would read P^T before the warps wrote it
    "issuer: p_ready": _drop("issuer", "p_ready"),
    # dK would read dS^T before the warps wrote it; S^T / dP^T of the next tile
    # would overwrite P^T / dS^T still in use
    "issuer: ds_ready": _drop("issuer", "ds_ready"),
    # the MMAs would read a Q/dO stage before it landed
    "issuer: qd_full": _drop("issuer", "qd_full"),
    # the warps would read S^T or dP^T before the MMA wrote it
    "warps: s_full": _drop("warp", "s_full"),
    "warps: dp_full": _drop("warp", "dp_full"),
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


def test_p_ready_is_needed_per_half():
    """p_ready exists per half of 64 query rows, each completing once per tile.
    With one barrier completing twice per tile the producer, which waits only
    for the second half (phase 2 i + 1), finds phase 2 i - 1 of the same parity
    completed as soon as tile i - 1 is done and would refill the statistics
    while tile i still reads them, and the issuer can find the barrier two
    phases ahead of its wait; the checker must report one or the other."""
    def merge(op):
        if op[0] in ("wait", "arrive") and op[1] in ("p_ready0", "p_ready1"):
            if op[0] == "arrive":
                return ("arrive", "p_ready", op[2])
            return ("wait", "p_ready", 2 * op[2] + (op[1] == "p_ready1"))
        return op

    rnd = random.Random(5)
    failures = 0
    for trial in range(300):
        roles, cnt = _roles(rnd.randint(2, 8))
        roles = {r: [merge(op) for op in ops] for r, ops in roles.items()}
        cnt["p_ready"] = cnt.pop("p_ready0")
        del cnt["p_ready1"]
        try:
            sync_model.run(roles, cnt, _stages(), trial, skewed=trial % 2 == 1)
        except AssertionError as e:
            assert any(w in str(e) for w in ("passes early", "aliasing", "hazard")), e
            failures += 1
    assert failures > 0


# --------------------------------------------------------------------------- sqa_bwd_q_kernel


def _q_stages():
    return {
        "kv": [("producer writes K, V", 1), ("S, dP and dQ MMAs read", 3)],
        "QD": [("warps write Q, dO into TMEM", WARPS), ("S, dP MMAs read", 2)],
        "SB": [("S and dP MMAs write", 2), ("warps rewrite dS", WARPS), ("dQ MMA reads dS", 1)],
        "acc_dq": [("dQ issuer accumulates dQ", 1), ("warps read dQ", WARPS)],
    }


def _q_roles(nkv, ST):
    """Three issuers: S and dP (one each) of tile j into buffer j % 2 once the
    dQ of j - 2 has read that buffer (dq_done), and dQ of j once the warps made
    dS_j."""
    cnt = {"qd_ready": 32 * WARPS, "dq_final": 1}
    for s in range(ST):
        cnt[f"kv_full{s}"] = 1
        cnt[f"kv_empty{s}"] = 1
    for x in range(2):
        cnt[f"sd_full{x}"] = 2  # the S and the dP issuer
        cnt[f"ds_ready{x}"] = 32 * WARPS
        cnt[f"dq_done{x}"] = 1

    def W(b, k):
        return ("wait", b, k)

    def A(b, m=1):
        return ("arrive", b, m)

    def B(res, v, stage, slot=0):
        return ("begin", (res, slot), v, stage)

    def E(res, v, stage, slot=0):
        return ("end", (res, slot), v, stage)

    prod = []
    for j in range(nkv):
        s = j % ST
        if j >= ST:
            prod.append(W(f"kv_empty{s}", j // ST - 1))
        prod += [B("kv", j, 0, s), E("kv", j, 0, s), A(f"kv_full{s}")]

    def sd_issuer():
        ops = [W("qd_ready", 0), B("QD", 0, 1)]
        for j in range(nkv):
            x = j & 1
            ops.append(W(f"kv_full{j % ST}", j // ST))
            if j >= 2:
                ops.append(W(f"dq_done{x}", (j - 2) >> 1))
            # the MMAs read K_j or V_j and write buffer x; done when sd_full arrives
            ops += [B("kv", j, 1, j % ST), B("SB", j, 0, x), E("SB", j, 0, x), E("kv", j, 1, j % ST),
                    A(f"sd_full{x}")]
        ops.append(E("QD", 0, 1))
        return ops

    iss_q = [B("acc_dq", 0, 0)]
    for j in range(nkv):
        x = j & 1
        iss_q += [W(f"ds_ready{x}", j >> 1), B("SB", j, 2, x), B("kv", j, 1, j % ST), E("SB", j, 2, x),
                  E("kv", j, 1, j % ST), A(f"dq_done{x}"), A(f"kv_empty{j % ST}")]
    iss_q += [E("acc_dq", 0, 0), A("dq_final")]

    def warp():
        ops = [B("QD", 0, 0), E("QD", 0, 0), A("qd_ready", 32)]
        for j in range(nkv):
            x = j & 1
            ops += [W(f"sd_full{x}", j >> 1), B("SB", j, 1, x), E("SB", j, 1, x), A(f"ds_ready{x}", 32)]
        ops += [W("dq_final", 0), B("acc_dq", 0, 1), E("acc_dq", 0, 1)]
        return ops

    roles = {"producer": prod, "issuer_s": sd_issuer(), "issuer_dp": sd_issuer(), "issuer_q": iss_q}
    for w in range(WARPS):
        roles[f"warp{w}"] = warp()
    return roles, cnt


def run_q(nkv, ST, seed, drop=None):
    roles, cnt = _q_roles(nkv, ST)
    if drop is not None:
        roles = {r: [op for op in ops if not drop(r, op)] for r, ops in roles.items()}
    sync_model.run(roles, cnt, _q_stages(), seed, skewed=seed % 2 == 1)


@pytest.mark.parametrize("ST", [6, 8, 2])
def test_q_kernel_protocol_has_no_deadlock_aliasing_or_hazard(ST):
    rnd = random.Random(ST)
    for trial in range(300):
        run_q(rnd.randint(1, 14), ST, trial)


Q_DROPS = {
    # S / dP would read Q, dO before the warps put them into TMEM
    "issuer: qd_ready": _drop("issuer_s", "qd_ready"),
    "dP issuer: qd_ready": _drop("issuer_dp", "qd_ready"),
    # dQ would read dS before the warps wrote it
    "issuer: ds_ready": _drop("issuer_q", "ds_ready"),
    # S of j + 2 would overwrite dS_j before the dQ MMA read it
    "issuer: dq_done": _drop("issuer_s", "dq_done"),
    "dP issuer: dq_done": _drop("issuer_dp", "dq_done"),
    # the MMAs would read a K/V stage before it landed
    "issuer: kv_full": _drop("issuer_s", "kv_full"),
    # the warps would read S / dP before the MMA wrote them, or dQ before the last MMA
    "warps: sd_full": _drop("warp", "sd_full"),
    "warps: dq_final": _drop("warp", "dq_final"),
    # the producer would overwrite a K/V stage still in use
    "producer: kv_empty": _drop("producer", "kv_empty"),
}


@pytest.mark.parametrize("name", list(Q_DROPS))
def test_q_model_detects_a_dropped_wait(name):
    rnd = random.Random(29)
    failures = 0
    for trial in range(300):
        # with two stages the K/V ring alone keeps S_{j+2} behind the dQ of j
        # (its load waits for the stage that dQ releases): six stages too
        try:
            run_q(rnd.randint(3, 12), 2 if trial % 2 else 6, trial, drop=Q_DROPS[name])
        except AssertionError:
            failures += 1
    assert failures > 0, name
