"""Model check of the forward kernel's barrier protocol (CPU only).

One slot of bsa_fwd_kernel (csrc/bsa_fwd_sm100.cu) runs seven roles -- a K
producer (stages each work item in a 4-entry ring, loads Q and K), a V producer,
an S issuer, a PV issuer and four softmax warps -- coordinated by mbarriers
waited on by phase parity: the item ring (7 readers), two Q buffers, two K and
two V stages of one 128-key chunk each, one set of S columns (SFull / SFree),
one set of P columns (PFull, released with the V stage by the PV commit), and O,
whose epilogue runs in the first chunk of the next tile and stages its rows in
the finished tile's Q buffer.

SFree and PFull take one arrival from every softmax thread; a warp's 32 arrivals
follow its own TMEM accesses in program order, so the model counts one arrival
per warp.

At head dim 128 the slot has two PV issuers, one per 64-column half of O; both
commit to the V stage's barrier, which then takes two arrivals, and both read
the item ring.  The model runs with one PV issuer (d = 64) and with two.

The test replays the roles' sequences under random interleavings, for random
work lists, with every asynchronous copy and MMA landing at a random later
moment, and asserts
  * that every parity wait is met by exactly the phase it targets and that no
    schedule deadlocks;
  * that every buffer holds what its reader expects when it reads it, and that
    nothing is overwritten while an earlier copy or MMA may still read it (the
    checks below run when a role reads or writes a buffer, when it issues an
    asynchronous operation, and when that operation lands).
"""

import random

import pytest

from protocol_model import Bar, replay, wait

RING, KST, VST, WARPS = 4, 2, 2, 4


def readers(n_pv):
    return 2 + n_pv + WARPS  # V producer, S issuer, PV issuers, softmax warps


class Slot:
    """Contents of one slot's buffers as the replay moves on."""

    def __init__(self, counts, n_pv=1):
        self.counts = counts
        self.n_pv = n_pv
        self.readers = readers(n_pv)
        self.first = [sum(counts[:k]) for k in range(len(counts) + 1)]  # first chunk of tile k
        self.staged = [None] * RING           # item in each ring stage
        self.readers_done = [0] * (len(counts) + 1)
        self.q_issued = [None, None]          # tile whose Q load was issued into each buffer
        self.q_landed = [None, None]
        self.q_released = [set() for _ in counts]
        self.k_issued, self.k_landed = [None] * KST, [None] * KST
        self.v_issued, self.v_landed = [None] * VST, [None] * VST
        self.s_issued, self.s_done = -1, set()
        self.s_loaded = [-1] * WARPS
        self.p_written = [-1] * WARPS
        self.pv_issued = [0] * n_pv            # per column half of O
        self.pv_done = [set() for _ in range(n_pv)]

    def s_complete(self, k):
        return all(x in self.s_done for x in range(self.first[k], self.first[k + 1]))

    def pv_complete_to(self, g):
        return all(x in done for done in self.pv_done for x in range(g))

    def pv_all_done(self, x):
        return all(x in done for done in self.pv_done)

    def pv_issued_to(self, g):
        return all(n == g for n in self.pv_issued)


def _k_producer(st, n_items, drop=()):
    """Stages item k (and a final sentinel), then loads Q of tile k into buffer
    k % 2 once tile k - 2 released it, and K of chunk g into stage g % 2 once
    S(g - 2) is done."""
    ops, g = [], 0
    for k in range(n_items + 1):
        ii = k % RING

        def stage(k=k, ii=ii):
            assert k < RING or st.readers_done[k - RING] == st.readers, f"item {k} staged over a read stage"
            st.staged[ii] = k

        ops += [wait(f"ItemEmpty{ii}", k // RING - 1), ("do", stage), ("arrive", f"ItemFull{ii}")]
        if k == n_items:
            break
        qs = k & 1

        def issue_q(k=k, qs=qs):
            if k >= 2:
                assert len(st.q_released[k - 2]) == WARPS, f"Q of tile {k} over tile {k - 2}'s staged O"
                assert st.s_complete(k - 2), f"Q of tile {k} over a buffer an S MMA reads"
            st.q_issued[qs] = k

        def land_q(k=k, qs=qs):
            assert st.q_issued[qs] == k
            st.q_landed[qs] = k

        if "QEmpty" not in drop:
            ops.append(wait(f"QEmpty{qs}", (k >> 1) - 1))
        ops += [("do", issue_q), ("async", f"QFull{qs}", land_q)]
        for _ in range(st.counts[k]):
            ks = g % KST

            def issue_k(g=g, ks=ks):
                assert g < KST or (g - KST) in st.s_done, f"K({g}) over the stage S({g - KST}) reads"
                st.k_issued[ks] = g

            def land_k(g=g, ks=ks):
                assert st.k_issued[ks] == g
                st.k_landed[ks] = g

            ops += [wait(f"KFree{ks}", g // KST - 1), ("do", issue_k), ("async", f"KFull{ks}", land_k)]
            g += 1
    return ops


def _v_producer(st, n_items):
    """Follows the item ring; loads V of chunk g into stage g % 2 once PV(g - 2)
    is done and releases each item after its last load."""
    ops, g = [], 0
    for k in range(n_items + 1):
        ii = k % RING
        ops.append(wait(f"ItemFull{ii}", k // RING))
        if k == n_items:
            break
        for _ in range(st.counts[k]):
            vs = g % VST

            def issue_v(k=k, g=g, vs=vs):
                assert st.staged[k % RING] == k, "V producer reads a restaged item"
                assert g < VST or st.pv_all_done(g - VST), f"V({g}) over the stage PV({g - VST}) reads"
                st.v_issued[vs] = g

            def land_v(g=g, vs=vs):
                assert st.v_issued[vs] == g
                st.v_landed[vs] = g

            ops += [wait(f"VFree{vs}", g // VST - 1), ("do", issue_v), ("async", f"VFull{vs}", land_v)]
            g += 1

        def release(k=k):
            st.readers_done[k] += 1

        ops += [("do", release), ("arrive", f"ItemEmpty{ii}")]
    return ops


def _take(st, k):
    def f():
        assert st.staged[k % RING] == k, f"item {k} read from a restaged stage"
        st.readers_done[k] += 1
    return f


def _s_issuer(st, n_items, drop=()):
    """Per chunk g: S(g) = Q K_g^T into the S columns once K(g) landed and the
    four softmax warps loaded S(g - 1); one commit signals S full, another frees
    the K stage (both land when the MMAs are done)."""
    ops, g = [], 0
    for k in range(n_items + 1):
        ii = k % RING
        ops += [wait(f"ItemFull{ii}", k // RING), ("do", _take(st, k)), ("arrive", f"ItemEmpty{ii}")]
        if k == n_items:
            break
        qs = k & 1
        ops.append(wait(f"QFull{qs}", k >> 1))
        for _ in range(st.counts[k]):
            ks = g % KST

            def issue_s(k=k, g=g, ks=ks, qs=qs):
                assert st.k_landed[ks] == g and st.k_issued[ks] == g, f"S({g}) reads a K stage not holding K({g})"
                assert st.q_landed[qs] == k and st.q_issued[qs] == k, f"S({g}) reads a Q buffer not holding tile {k}"
                assert all(x >= g - 1 for x in st.s_loaded), f"S({g}) overwrites S({g - 1}) before it was loaded"
                st.s_issued = g

            def land_s(k=k, g=g, ks=ks, qs=qs):
                if g in st.s_done:  # the other commit of the same MMAs landed first
                    return
                assert st.k_issued[ks] == g, f"K stage reloaded while S({g}) read it"
                assert st.q_issued[qs] == k, f"Q buffer reloaded while S({g}) read it"
                assert st.s_issued == g
                st.s_done.add(g)

            ops.append(wait(f"KFull{ks}", g // KST))
            if "SFree" not in drop:
                ops.append(wait("SFree", g - 1))
            ops += [("do", issue_s), ("async", "SFull", land_s), ("async", f"KFree{ks}", land_s)]
            g += 1
    return ops


def _pv_issuer(st, n_items, half=0):
    """Per chunk g: O (+)= P(g) V_g (this issuer's column half of O) once V(g)
    landed and the four softmax warps wrote P(g); its commit (with the other
    half's, at d = 128) frees the V stage and the P columns."""
    ops, g = [], 0
    for k in range(n_items + 1):
        ii = k % RING
        ops += [wait(f"ItemFull{ii}", k // RING), ("do", _take(st, k)), ("arrive", f"ItemEmpty{ii}")]
        if k == n_items:
            break
        for _ in range(st.counts[k]):
            vs = g % VST

            def issue_pv(g=g, vs=vs):
                assert st.v_landed[vs] == g and st.v_issued[vs] == g, f"PV({g}) reads a V stage not holding V({g})"
                assert all(x == g for x in st.p_written), f"PV({g}) before every warp wrote P({g})"
                assert st.pv_issued[half] == g
                st.pv_issued[half] = g + 1

            def land_pv(g=g, vs=vs):
                assert st.v_issued[vs] == g, f"V stage reloaded while PV({g}) read it"
                assert all(x == g for x in st.p_written), f"P columns rewritten while PV({g}) read them"
                st.pv_done[half].add(g)

            ops += [wait(f"VFull{vs}", g // VST), wait("PFull", g), ("do", issue_pv),
                    ("async", f"VFree{vs}", land_pv)]
            g += 1
    return ops


def _softmax_warp(st, n_items, w, drop=()):
    """Per chunk g: load S(g) and release the S columns; wait for PV(g - 1) (the P
    columns are free and O holds chunk g - 1); in the first chunk of a tile run
    the previous tile's epilogue (O read from TMEM, staged in that tile's Q buffer,
    item released); rescale O if needed; write P(g).  The Q buffer of the last
    epilogue is released one chunk later, or at the end of a one-chunk tile."""
    ops, g = [], 0
    pend, q_pending = None, None

    def release_q(kq):
        def f():
            st.q_released[kq].add(w)
        return [("do", f), ("arrive", f"QEmpty{kq & 1}")]

    def epilogue(kp, g_now):
        def f():
            assert st.staged[kp % RING] == kp, f"epilogue of tile {kp} reads a restaged item"
            assert st.pv_complete_to(g_now) and st.pv_issued_to(g_now), f"O of tile {kp} read with a PV pending"
            assert st.s_complete(kp), f"O of tile {kp} staged over Q while an S MMA reads it"
            assert st.q_issued[kp & 1] == kp, f"O of tile {kp} staged in a reloaded Q buffer"
            st.readers_done[kp] += 1
        return [("do", f), ("arrive", f"ItemEmpty{kp % RING}")]

    def pv_wait(x):
        return None if "VFree" in drop else wait(f"VFree{x % VST}", x // VST)

    for k in range(n_items + 1):
        ops.append(wait(f"ItemFull{k % RING}", k // RING))
        if k == n_items:
            break
        for n in range(st.counts[k]):
            if q_pending is not None and n > 0:
                ops += release_q(q_pending)
                q_pending = None

            def load_s(k=k, g=g):
                assert g in st.s_done and st.s_issued == g, f"S({g}) loaded while not (or no longer) in TMEM"
                assert st.staged[k % RING] == k
                st.s_loaded[w] = g

            ops += [wait("SFull", g), ("do", load_s), ("arrive", "SFree")]
            if g > 0:
                ops.append(pv_wait(g - 1))
            if n == 0 and pend is not None:
                ops += epilogue(pend, g)
                q_pending, pend = pend, None

            def write_p(g=g):
                assert st.pv_complete_to(g) and st.pv_issued_to(g), f"P({g}) / O rescale with a PV pending"
                st.p_written[w] = g

            ops += [("do", write_p), ("arrive", "PFull")]
            g += 1
        if q_pending is not None:
            ops += release_q(q_pending)
            q_pending = None
        pend = k
    if pend is not None:
        ops += [pv_wait(g - 1)] + epilogue(pend, g)
    return ops


def _roles(counts, drop=(), n_pv=1):
    n_items = len(counts)
    st = Slot(counts, n_pv)
    vfree = 1 if "VFreeCount" in drop else n_pv
    bars = {}
    for name, count in ([(f"QFull{i}", 1) for i in range(2)] + [(f"QEmpty{i}", WARPS) for i in range(2)] +
                        [(f"KFull{i}", 1) for i in range(KST)] + [(f"KFree{i}", 1) for i in range(KST)] +
                        [(f"VFull{i}", 1) for i in range(VST)] + [(f"VFree{i}", vfree) for i in range(VST)] +
                        [("SFull", 1), ("SFree", WARPS), ("PFull", WARPS)] +
                        [(f"ItemFull{i}", 1) for i in range(RING)] +
                        [(f"ItemEmpty{i}", st.readers) for i in range(RING)]):
        bars[name] = Bar(name, count)
    roles = {"k_producer": _k_producer(st, n_items, drop), "v_producer": _v_producer(st, n_items),
             "s_issuer": _s_issuer(st, n_items, drop)}
    for h in range(n_pv):
        roles[f"pv_issuer{h}"] = _pv_issuer(st, n_items, h)
    for w in range(WARPS):
        roles[f"softmax{w}"] = _softmax_warp(st, n_items, w, drop)
    return bars, roles, st


def _work(rnd):
    # chunks per tile: 1 (a one-chunk tile releases its Q buffer at its end) to 6
    return [rnd.randint(1, 6) for _ in range(rnd.randint(1, 10))]


@pytest.mark.parametrize("n_pv", [1, 2])
def test_random_schedules_keep_every_buffer_consistent(n_pv):
    for seed in range(400):
        rnd = random.Random(seed)
        counts = _work(rnd)
        bars, roles, st = _roles(counts, n_pv=n_pv)
        replay(bars, roles, seed)
        total = sum(counts)
        assert all(done == set(range(total)) for done in st.pv_done) and st.s_done == set(range(total))
        assert st.readers_done[:len(counts)] == [readers(n_pv)] * len(counts)


@pytest.mark.parametrize("missing", ["VFree", "SFree", "QEmpty"])
def test_the_model_catches_a_missing_wait(missing):
    # planting a mistake in the model: without the softmax's wait for PV(g - 1), P(g)
    # is written over columns PV(g - 1) reads; without the S issuer's wait for SFree,
    # S(g) overwrites S(g - 1) before it was loaded; without the K producer's wait for
    # QEmpty, Q of tile k lands over tile k - 2's staged O
    caught = 0
    for seed in range(200):
        rnd = random.Random(seed)
        bars, roles, _ = _roles(_work(rnd), drop=(missing,))
        try:
            replay(bars, roles, seed)
        except AssertionError:
            caught += 1
    assert caught > 0


def test_the_model_catches_a_v_barrier_counting_one_of_two_pv_issuers():
    # planting a mistake: at d = 128 the V stage's barrier initialised for one
    # arrival lets V(g + 2) or P(g + 1) in while the other half's PV(g) still reads
    caught = 0
    for seed in range(200):
        rnd = random.Random(seed)
        bars, roles, _ = _roles(_work(rnd), drop=("VFreeCount",), n_pv=2)
        try:
            replay(bars, roles, seed)
        except AssertionError:
            caught += 1
    assert caught > 0
