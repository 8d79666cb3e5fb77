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
stage k % 2, entry stage g % 4, score stage g % 3, accumulator stage k % 2
(dQ; one accumulator stage for dK/dV), and
the compute warps' epilogue deferred to the first entry of the next tile.
"""

import random

import pytest

from protocol_model import Bar, replay, wait

E_STAGES = 4
COMPUTE_WARPS = 8


def _roles(dkv, counts):
    bars = {}

    def bar(name, count=1):
        bars[name] = Bar(name, count)

    S = 3  # score stages
    A = 1 if dkv else 2  # accumulator stages: one for dK/dV (128 columns), two for dQ
    for i in range(2):
        for n in ("TileFull", "TileEmpty"):
            bar(f"{n}{i}")
    for i in range(A):
        bar(f"AccFull{i}")
        bar(f"AccEmpty{i}", COMPUTE_WARPS)
    for i in range(S):
        bar(f"ScoreFull{i}")
        bar(f"ScoreFree{i}")
        bar(f"DsFull{i}", COMPUTE_WARPS)
    for i in range(E_STAGES):
        bar(f"EntFull{i}")
        bar(f"EntEmpty{i}")

    prod, score, acc = [], [], []
    g = 0
    for k, cnt in enumerate(counts):
        ts = k & 1
        prod += [wait(f"TileEmpty{ts}", (k >> 1) - 1), ("async", f"TileFull{ts}")]
        score += [wait(f"TileFull{ts}", k >> 1)]
        acc += [wait(f"AccEmpty{k % A}", k // A - 1)]
        for _ in range(cnt):
            es, ss = g % E_STAGES, g % S
            prod += [wait(f"EntEmpty{es}", g // E_STAGES - 1), ("async", f"EntFull{es}")]
            score += [wait(f"EntFull{es}", g // E_STAGES), wait(f"ScoreFree{ss}", g // S - 1),
                      ("async", f"ScoreFull{ss}")]
            acc += [wait(f"DsFull{ss}", g // S), ("async", f"ScoreFree{ss}"), ("async", f"EntEmpty{es}")]
            g += 1
        score += [("async", f"TileEmpty{ts}")]
        acc += [("async", f"AccFull{k % A}")]
    roles = {"producer": prod, "score": score, "acc": acc}
    for w in range(COMPUTE_WARPS):
        ops, g, pend = [], 0, None
        for k, cnt in enumerate(counts):
            for n in range(cnt):
                es, ss = g % E_STAGES, g % S
                ops.append(wait(f"ScoreFull{ss}", g // S))
                if dkv:
                    ops.append(wait(f"EntFull{es}", g // E_STAGES))
                ops.append(("arrive", f"DsFull{ss}"))
                if n == 0 and pend is not None:
                    ops += [wait(f"AccFull{pend % A}", pend // A), ("arrive", f"AccEmpty{pend % A}")]
                    pend = None
                g += 1
            pend = k
        if pend is not None:
            ops += [wait(f"AccFull{pend % A}", pend // A), ("arrive", f"AccEmpty{pend % A}")]
        roles[f"compute{w}"] = ops
    return bars, roles


def _run(dkv, counts, seed):
    bars, roles = _roles(dkv, counts)
    replay(bars, roles, seed)


@pytest.mark.parametrize("dkv", [False, True], ids=["dq", "dkv"])
def test_random_schedules_never_alias_or_deadlock(dkv):
    for seed in range(250):
        rnd = random.Random(seed)
        counts = [rnd.randint(1, 6) for _ in range(rnd.randint(1, 6))]
        _run(dkv, counts, seed)


def test_the_model_catches_a_missing_release():
    # planting a mistake in the model: a score issuer that does not wait for the
    # score stage to be freed lets S of entry g + 3 overwrite stage g % 3 while
    # entry g is still being read -- the check must flag it as an aliased phase
    import tests.test_bwd_protocol as m
    orig = m._roles

    def broken(dkv, counts):
        bars, roles = orig(dkv, counts)
        roles["score"] = [o for o in roles["score"] if not (o and o[0] == "wait" and o[1].startswith("ScoreFree"))]
        return bars, roles

    m._roles = broken
    try:
        with pytest.raises(AssertionError):
            for seed in range(200):
                m._run(False, [6, 6, 6], seed)
    finally:
        m._roles = orig
