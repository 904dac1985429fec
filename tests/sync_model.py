"""Random-schedule checker for models of a kernel's synchronisation (test
helper, CPU only).

A model is a dict role -> list of operations, in the role's program order:

* ("wait", barrier, k): wait for phase k of an mbarrier, i.e. its (k + 1)-th
  completion;
* ("arrive", barrier, m): m arrivals (an asynchronous copy or MMA's completion
  is an arrival);
* ("begin" | "end", (buffer, slot), version, stage): the window in which the
  role uses one version of a buffer in one stage of that version's life (for
  example 0 = written by an MMA, 1 = rewritten by the softmax warps, 2 = read
  by another MMA); each stage has a number of users;
* ("begin" | "end", (name, slot), info, None) on a buffer handled by a custom
  checker object (``custom``), for accumulators whose users interleave.

``run`` executes one random interleaving and raises AssertionError on phase
aliasing (a wait finds the barrier k + 2 completions ahead, so a parity wait
would pass on the wrong phase, or only k - 1 completions in, so a parity wait
would pass before phase k has completed), over-arrival, deadlock, or a buffer hazard (a
use starts before every user of the previous stage or version has finished).
"""
import random


class Buffer:
    """Version and stage of one buffer, and its users."""

    def __init__(self, stages):
        self.stages = stages  # [(description, number of users)]
        self.version, self.stage, self.ended, self.active = None, None, 0, 0

    def begin(self, v, k):
        n = len(self.stages)
        if (v, k) == (self.version, self.stage):
            assert self.ended + self.active < self.stages[k][1], "more users than the stage has"
        else:
            if self.version is not None:
                assert self.active == 0 and self.ended == self.stages[self.stage][1], \
                    f"hazard: '{self.stages[k][0]}' v{v} starts while '{self.stages[self.stage][0]}' " \
                    f"v{self.version} has {self.active} active and {self.ended} finished users"
            nxt = (self.version, self.stage + 1) if self.version is not None and self.stage + 1 < n else None
            first = k == 0 and (self.version is None or (self.stage == n - 1 and v > self.version))
            assert (v, k) == nxt or first, \
                f"hazard: '{self.stages[k][0]}' v{v} out of order (at v{self.version} stage {self.stage})"
            self.version, self.stage, self.ended = v, k, 0
        self.active += 1

    def end(self, v, k):
        assert (v, k) == (self.version, self.stage) and self.active > 0
        self.active -= 1
        self.ended += 1


def run(roles, counts, stages, seed, custom=None, skewed=False):
    """One random interleaving of ``roles``; ``counts``: barrier -> arrivals per
    phase; ``stages``: buffer kind -> [(description, users)]; ``custom``:
    buffer name -> object with begin(slot, info) and end(slot, info).
    ``skewed``: give each role a random speed for the whole run (a role may then
    lag far behind the others), instead of picking ready roles uniformly."""
    done = {b: 0 for b in counts}
    arrived = {b: 0 for b in counts}
    bufs = {}
    pc = {r: 0 for r in roles}
    rnd = random.Random(seed)
    speed = {r: (10.0 ** rnd.uniform(-3, 0) if skewed else 1.0) for r in roles}
    while True:
        ready = []
        for r, ops in roles.items():
            if pc[r] == len(ops):
                continue
            op = ops[pc[r]]
            if op[0] != "wait":
                ready.append(r)
            else:
                _, b, k = op
                assert done[b] < k + 2, f"phase aliasing: {r} waits on {b} phase {k} after {done[b]} completions"
                assert done[b] != k - 1, f"parity wait passes early: {r} waits on {b} phase {k} " \
                    f"after {done[b]} completions (phase {k - 1}, same parity, still open)"
                if done[b] == k + 1:
                    ready.append(r)
        if not ready:
            break
        r = rnd.choices(ready, weights=[speed[x] for x in ready])[0] if skewed else rnd.choice(ready)
        op = roles[r][pc[r]]
        pc[r] += 1
        if op[0] == "arrive":
            _, b, m = op
            arrived[b] += m
            assert arrived[b] <= counts[b], f"over-arrival on {b}"
            if arrived[b] == counts[b]:
                arrived[b] = 0
                done[b] += 1
        elif op[0] in ("begin", "end"):
            _, (name, slot), v, k = op
            if custom and name in custom:
                getattr(custom[name], op[0])(slot, v)
            else:
                buf = bufs.setdefault((name, slot), Buffer(stages[name]))
                (buf.begin if op[0] == "begin" else buf.end)(v, k)
    stuck = {r: roles[r][pc[r]] for r in roles if pc[r] < len(roles[r])}
    assert not stuck, f"deadlock: {stuck}"
    assert all(a == 0 for a in arrived.values())  # every phase that was started was completed
