"""Model check of the backward kernel's barrier protocol (CPU only).

bsa_bwd_kernel (csrc/bsa_bwd_sm100.cu) coordinates its roles -- TMA producer,
score issuer, accumulate issuer, eight compute warps -- with mbarriers waited on
by phase parity.  A parity wait is only sound when the waiter can never fall a
whole phase behind: otherwise a later phase of the same parity satisfies it, or
it waits for a phase that already went by.  This test replays each role's
sequence of waits, arrivals and asynchronous completions (TMA loads and MMA
commits, completing in any order) under random interleavings for random tile
lists, and asserts that every wait is met by exactly the phase it targets and
that no schedule deadlocks.  The sequences mirror the kernel's loops: tile
stage k % 2, entry stage g % 4, score stage g % 2, accumulator stage k % 2, and
the compute warps' epilogue deferred to the first entry of the next tile.
"""

import random

import pytest

E_STAGES = 4
COMPUTE_WARPS = 8


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrivals, self.done = name, count, 0, 0

    def arrive(self):
        self.arrivals += 1
        assert self.arrivals <= self.count, self.name
        if self.arrivals == self.count:
            self.arrivals = 0
            self.done += 1


def _roles(dkv, counts):
    bars = {}

    def bar(name, count=1):
        bars[name] = _Bar(name, count)

    for i in range(2):
        for n in ("TileFull", "TileEmpty", "ScoreFull", "ScoreFree", "AccFull"):
            bar(f"{n}{i}")
        bar(f"DsFull{i}", COMPUTE_WARPS)
        bar(f"AccEmpty{i}", COMPUTE_WARPS)
    for i in range(E_STAGES):
        bar(f"EntFull{i}")
        bar(f"EntEmpty{i}")

    def wait(name, phase):  # wait for the completion of phase `phase` (no-op if < 0)
        return ("wait", name, phase) if phase >= 0 else None

    prod, score, acc = [], [], []
    g = 0
    for k, cnt in enumerate(counts):
        ts = k & 1
        prod += [wait(f"TileEmpty{ts}", (k >> 1) - 1), ("async", f"TileFull{ts}")]
        score += [wait(f"TileFull{ts}", k >> 1)]
        acc += [wait(f"AccEmpty{ts}", (k >> 1) - 1)]
        for _ in range(cnt):
            es, ss = g % E_STAGES, g & 1
            prod += [wait(f"EntEmpty{es}", g // E_STAGES - 1), ("async", f"EntFull{es}")]
            score += [wait(f"EntFull{es}", g // E_STAGES), wait(f"ScoreFree{ss}", (g >> 1) - 1),
                      ("async", f"ScoreFull{ss}")]
            acc += [wait(f"DsFull{ss}", g >> 1), ("async", f"ScoreFree{ss}"), ("async", f"EntEmpty{es}")]
            g += 1
        score += [("async", f"TileEmpty{ts}")]
        acc += [("async", f"AccFull{ts}")]
    roles = {"producer": prod, "score": score, "acc": acc}
    for w in range(COMPUTE_WARPS):
        ops, g, pend = [], 0, None
        for k, cnt in enumerate(counts):
            for n in range(cnt):
                es, ss = g % E_STAGES, g & 1
                ops.append(wait(f"ScoreFull{ss}", g >> 1))
                if dkv:
                    ops.append(wait(f"EntFull{es}", g // E_STAGES))
                ops.append(("arrive", f"DsFull{ss}"))
                if n == 0 and pend is not None:
                    ops += [wait(f"AccFull{pend & 1}", pend >> 1), ("arrive", f"AccEmpty{pend & 1}")]
                    pend = None
                g += 1
            pend = k
        if pend is not None:
            ops += [wait(f"AccFull{pend & 1}", pend >> 1), ("arrive", f"AccEmpty{pend & 1}")]
        roles[f"compute{w}"] = ops
    return bars, {r: [o for o in ops if o is not None] for r, ops in roles.items()}


def _run(dkv, counts, seed):
    rnd = random.Random(seed)
    bars, roles = _roles(dkv, counts)
    pc = {r: 0 for r in roles}
    inflight = []
    while True:
        runnable = []
        for r, ops in roles.items():
            if pc[r] == len(ops):
                continue
            op = ops[pc[r]]
            if op[0] == "wait":
                b, t = bars[op[1]], op[2]
                if (b.done & 1) != (t & 1):  # try_wait.parity: the phase of t's parity completed
                    assert b.done == t + 1, f"{r}: {op} satisfied by a later phase (done={b.done})"
                    runnable.append(r)
                else:
                    assert b.done <= t, f"{r}: {op} waits for a phase already gone (done={b.done})"
            else:
                runnable.append(r)
        choices = runnable + (["async"] if inflight else [])
        if not choices:
            stuck = [(r, roles[r][pc[r]]) for r in roles if pc[r] < len(roles[r])]
            assert not stuck, f"deadlock: {stuck}"
            return
        c = rnd.choice(choices)
        if c == "async":
            bars[inflight.pop(rnd.randrange(len(inflight)))].arrive()
            continue
        op = roles[c][pc[c]]
        pc[c] += 1
        if op[0] == "arrive":
            bars[op[1]].arrive()
        elif op[0] == "async":
            inflight.append(op[1])


@pytest.mark.parametrize("dkv", [False, True], ids=["dq", "dkv"])
def test_random_schedules_never_alias_or_deadlock(dkv):
    for seed in range(250):
        rnd = random.Random(seed)
        counts = [rnd.randint(1, 6) for _ in range(rnd.randint(1, 6))]
        _run(dkv, counts, seed)


def test_the_model_catches_a_missing_release():
    # planting a mistake in the model: a score issuer that does not wait for the
    # score stage to be freed lets S of entry g + 2 overwrite stage g % 2 while
    # entry g is still being read -- the check must flag it as an aliased phase
    import tests.test_bwd_protocol as m
    orig = m._roles

    def broken(dkv, counts):
        bars, roles = orig(dkv, counts)
        roles["score"] = [o for o in roles["score"] if not (o[0] == "wait" and o[1].startswith("ScoreFree"))]
        return bars, roles

    m._roles = broken
    try:
        with pytest.raises(AssertionError):
            for seed in range(200):
                m._run(False, [6, 6, 6], seed)
    finally:
        m._roles = orig
