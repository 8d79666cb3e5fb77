"""Model check of the forward kernel's barrier protocol (CPU only).

One slot of bsa_fwd_kernel (csrc/bsa_fwd_sm100.cu) coordinates a TMA producer,
an S issuer, a PV issuer and four softmax warps through mbarriers waited on by
phase parity: a 4-entry item ring (6 readers), two Q stages, a 3-stage K ring
released by the S commits, a 4-stage V ring released by the PV commits, three S
buffers (P written over S, 4 warp arrivals in this model for the 128 threads),
and O, released by the epilogue that runs one chunk into the next tile.  A
softmax warp that raises a row's running max waits for the previous chunk's PV
before rescaling O.  This test replays the roles' sequences under random
interleavings for random work lists (each chunk's rescale decided at random
per warp) and asserts that every wait is met by exactly the phase it targets
and that no schedule deadlocks.
"""

import random

import pytest

from protocol_model import Bar, replay, wait

ITEMS, KST, VST, SBUF, WARPS = 4, 3, 4, 3, 4


def _roles(counts, rescale_seed):
    rnd = random.Random(rescale_seed)
    bars = {}

    def bar(name, count=1):
        bars[name] = Bar(name, count)

    for i in range(2):
        bar(f"QFull{i}")
        bar(f"QEmpty{i}")
    for i in range(KST):
        bar(f"KFull{i}")
    for i in range(VST):
        bar(f"VFull{i}")
        bar(f"VFree{i}")
    for i in range(SBUF):
        bar(f"SFull{i}")
        bar(f"PFull{i}", WARPS)
    bar("OFree", WARPS)
    for i in range(ITEMS):
        bar(f"ItemFull{i}")
        bar(f"ItemEmpty{i}", 2 + WARPS)

    n_items = len(counts)
    # producer: stages each item (and a final sentinel), then its loads
    prod, g = [], 0
    for k in range(n_items + 1):
        ii = k % ITEMS
        prod += [wait(f"ItemEmpty{ii}", k // ITEMS - 1), ("arrive", f"ItemFull{ii}")]
        if k == n_items:
            break
        qs = k & 1
        prod += [wait(f"QEmpty{qs}", (k >> 1) - 1), ("async", f"QFull{qs}")]
        for _ in range(counts[k]):
            prod += [wait(f"SFull{g % KST}", g // KST - 1), ("async", f"KFull{g % KST}")]
            prod += [wait(f"VFree{g % VST}", g // VST - 1), ("async", f"VFull{g % VST}")]
            g += 1
    # S issuer
    s_iss, g = [], 0
    for k in range(n_items + 1):
        ii = k % ITEMS
        s_iss += [wait(f"ItemFull{ii}", k // ITEMS), ("arrive", f"ItemEmpty{ii}")]
        if k == n_items:
            break
        s_iss += [wait(f"QFull{k & 1}", k >> 1)]
        for n in range(counts[k]):
            s_iss += [wait(f"KFull{g % KST}", g // KST)]
            if g >= SBUF:
                s_iss += [wait(f"VFree{(g - SBUF) % VST}", (g - SBUF) // VST)]
            s_iss += [("async", f"SFull{g % SBUF}")]
            if n == counts[k] - 1:
                s_iss += [("async", f"QEmpty{k & 1}")]
            g += 1
    # PV issuer
    pv, g = [], 0
    for k in range(n_items + 1):
        ii = k % ITEMS
        pv += [wait(f"ItemFull{ii}", k // ITEMS), ("arrive", f"ItemEmpty{ii}")]
        if k == n_items:
            break
        for n in range(counts[k]):
            if n == 0:
                pv += [wait("OFree", k - 1)]
            pv += [wait(f"VFull{g % VST}", g // VST), wait(f"PFull{g % SBUF}", g // SBUF),
                   ("async", f"VFree{g % VST}")]
            g += 1
    roles = {"producer": prod, "s_issuer": s_iss, "pv_issuer": pv}
    # softmax warps, epilogue one chunk late
    for w in range(WARPS):
        ops, g, pend = [], 0, None
        for k in range(n_items + 1):
            ops.append(wait(f"ItemFull{k % ITEMS}", k // ITEMS))
            if k == n_items:
                break
            for n in range(counts[k]):
                ops.append(wait(f"SFull{g % SBUF}", g // SBUF))
                if n > 0 and rnd.random() < 0.3:  # the running max grew: rescale O after PV(g - 1)
                    ops.append(wait(f"VFree{(g - 1) % VST}", (g - 1) // VST))
                ops.append(("arrive", f"PFull{g % SBUF}"))
                if n == 0 and pend is not None:
                    pk, g_last = pend
                    ops += [wait(f"VFree{g_last % VST}", g_last // VST), ("arrive", "OFree"),
                            ("arrive", f"ItemEmpty{pk % ITEMS}")]
                    pend = None
                g += 1
            pend = (k, g - 1)
        if pend is not None:
            pk, g_last = pend
            ops += [wait(f"VFree{g_last % VST}", g_last // VST), ("arrive", "OFree"),
                    ("arrive", f"ItemEmpty{pk % ITEMS}")]
        roles[f"softmax{w}"] = ops
    return bars, roles


def test_random_schedules_never_alias_or_deadlock():
    for seed in range(300):
        rnd = random.Random(seed)
        counts = [rnd.randint(1, 7) for _ in range(rnd.randint(1, 9))]
        bars, roles = _roles(counts, seed)
        replay(bars, roles, seed)


def test_the_model_catches_a_missing_release():
    # planting a mistake in the model: an S issuer that does not wait for
    # PV(g - 3) lets S(g) overwrite the buffer P(g - 3) still occupies
    rnd = random.Random(1)
    with pytest.raises(AssertionError):
        for seed in range(300):
            counts = [rnd.randint(4, 7) for _ in range(4)]
            bars, roles = _roles(counts, seed)
            roles["s_issuer"] = [o for o in roles["s_issuer"]
                                 if not (o and o[0] == "wait" and o[1].startswith("VFree"))]
            replay(bars, roles, seed)
