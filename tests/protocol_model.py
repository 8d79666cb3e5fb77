"""Replays the barrier protocol of a kernel's roles under random interleavings.

Helper of the protocol tests (tests/test_fwd_protocol.py,
tests/test_bwd_protocol.py).  A role is a list of operations on named mbarriers:
  ("wait", bar, t)   wait, by phase parity, for the completion of phase t of bar
  ("arrive", bar)    one arrival by the role itself
  ("async", bar)     one arrival that happens later, in any order with the other
                     pending ones (a TMA load's completion or an MMA commit)
  ("async", bar, f)  the same, calling f() when the operation lands (before the
                     arrival): the moment an asynchronous copy or MMA has finished
                     reading and writing its buffers
  ("do", f)          calls f() when the role reaches it: a read or a write of a
                     buffer, whose assertions check that the buffer holds what the
                     role expects
The replay asserts that each wait is met by exactly the phase it targets (a
parity wait cannot tell phase t from phase t + 2), that every "do" and landing
check holds, and that no schedule deadlocks.
"""

import random


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrivals, self.done = name, count, 0, 0

    def arrive(self):
        self.arrivals += 1
        assert self.arrivals <= self.count, self.name
        if self.arrivals == self.count:
            self.arrivals = 0
            self.done += 1


def wait(name, phase):
    """A wait for phase `phase` (None when the phase is negative: no wait needed)."""
    return ("wait", name, phase) if phase >= 0 else None


def replay(bars, roles, seed):
    rnd = random.Random(seed)
    roles = {r: [o for o in ops if o is not None] for r, ops in roles.items()}
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
            landed = inflight.pop(rnd.randrange(len(inflight)))
            if len(landed) > 1:
                landed[1]()
            bars[landed[0]].arrive()
            continue
        op = roles[c][pc[c]]
        pc[c] += 1
        if op[0] == "arrive":
            bars[op[1]].arrive()
        elif op[0] == "async":
            inflight.append(op[1:])
        elif op[0] == "do":
            op[1]()
