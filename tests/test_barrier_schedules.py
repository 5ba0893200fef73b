"""The barrier schedules of the dK/dV kernel and the forward, checked on a model under
random interleavings.

The kernel's warps meet on mbarriers: the MMA warp's commits complete a phase when the
tensor cores finish, and the dS warps arrive on ``p_ready`` / ``ds_ready`` without
waiting on them.  A wait asks for the phase of one parity, so it can only tell the
current phase from the one before.  The model below replays the schedule of
``attn_bwd_kv_kernel`` (csrc/bwd.cuh) step by step -- which MMA is issued after which
wait, which buffer each product reads and writes, which barrier each warp arrives on --
and explores random interleavings of the MMA warp, the tensor pipe (in-order completion)
and the dS warps, checking that every product reads what the schedule says it reads
(S^T(g), P^T(g) of every warp, dS^T(g)) and that no schedule deadlocks.

Two S^T buffers with one shared ``p_ready`` barrier is the schedule that let dV(g)
read a slow warp's P^T columns before it wrote them: the model finds that interleaving.
The schedules the kernel uses (one buffer with the split dV issue at d = 128; two
buffers with one ``p_ready`` per buffer at d = 64) pass, and so does the forward's
(two teams on one MMA warp, PV in two halves, S(j+1) behind PV(j)).
"""
import random

import pytest


class Barrier:
    """An mbarrier: ``count`` arrivals complete a phase; a parity wait passes once the
    phase of that parity is the last completed one."""

    def __init__(self, count):
        self.count, self.pending, self.completed = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.completed & 1) != parity


class Violation(Exception):
    pass


def run(steps, warps, two_buffers, p_ready_per_buffer, split_dv, seed, s_early=None):
    """One random interleaving.  ``s_early``: issue S^T(g+1) before dV(g) (the default
    with two buffers) rather than behind it."""
    s_early = two_buffers if s_early is None else s_early
    rnd = random.Random(seed)
    nb = 2 if two_buffers else 1
    bars = {"s_full": [Barrier(1) for _ in range(nb)], "dp_full": Barrier(1), "ds_ready": Barrier(warps),
            "p_ready": [Barrier(warps) for _ in range(2 if p_ready_per_buffer else 1)], "p_half": Barrier(warps)}
    sbuf = [[None] * warps for _ in range(nb)]     # per buffer, per warp's columns: ("S"|"P", step)
    dpbuf = [None] * warps                          # per warp's columns: ("dP"|"dS", step)
    pipe = []                                       # issued products, performed in order

    def p_bar(g):
        return bars["p_ready"][g % nb if p_ready_per_buffer else 0]

    def p_par(g):
        return (g // nb if p_ready_per_buffer else g) & 1

    def perform(op):
        kind, g = op[0], op[1]
        if kind == "S":
            for w in range(warps):
                sbuf[g % nb][w] = ("S", g)
            bars["s_full"][g % nb].arrive()
        elif kind == "dP":
            for w in range(warps):
                dpbuf[w] = ("dP", g)
            bars["dp_full"].arrive()
        elif kind == "dV":                          # reads the half (or all) of P^T(g) it was issued for
            for w in range(warps):
                if sbuf[g % nb][w] != ("P", g):
                    raise Violation(f"dV({g}) read warp {w}'s columns holding {sbuf[g % nb][w]}")
        elif kind == "dK":
            for w in range(warps):
                if dpbuf[w] != ("dS", g):
                    raise Violation(f"dK({g}) read warp {w}'s columns holding {dpbuf[w]}")

    def mma():                                      # the MMA warp's program
        yield ("issue", ("S", 0))
        yield ("issue", ("dP", 0))
        for g in range(steps):
            if s_early and g + 1 < steps:
                yield ("issue", ("S", g + 1))
            if split_dv:
                yield ("wait", bars["p_half"], g & 1)
                yield ("issue", ("dVhalf", g))
            yield ("wait", p_bar(g), p_par(g))
            yield ("issue", ("dV", g))
            if not s_early and g + 1 < steps:
                yield ("issue", ("S", g + 1))
            yield ("wait", bars["ds_ready"], g & 1)
            yield ("issue", ("dK", g))
            if g + 1 < steps:
                yield ("issue", ("dP", g + 1))

    def ds_warp(w):                                 # one dS warp's program
        for g in range(steps):
            yield ("wait", bars["s_full"][g % nb], (g // nb) & 1)
            yield ("check", lambda g=g: sbuf[g % nb][w] == ("S", g), f"warp {w} phase A({g}) read S^T")
            yield ("do", lambda g=g: sbuf[g % nb].__setitem__(w, ("P", g)))
            if split_dv:
                yield ("arrive", bars["p_half"])
            yield ("arrive", p_bar(g))
            yield ("wait", bars["dp_full"], g & 1)
            yield ("check", lambda g=g: dpbuf[w] == ("dP", g), f"warp {w} phase B({g}) read dP^T")
            yield ("do", lambda g=g: dpbuf.__setitem__(w, ("dS", g)))
            yield ("arrive", bars["ds_ready"])

    agents = {"mma": mma(), **{f"w{w}": ds_warp(w) for w in range(warps)}}
    nxt = {name: next(gen) for name, gen in agents.items()}
    while nxt or pipe:
        ready = [n for n, op in nxt.items() if op[0] != "wait" or op[1].passed(op[2])]
        choices = ready + (["pipe"] if pipe else [])
        if not choices:
            raise Violation("deadlock")
        who = rnd.choice(choices)
        if who == "pipe":
            op = pipe.pop(0)
            if op[0] != "dVhalf":                   # the first half reads what p_half guarantees
                perform(op)
            continue
        op = nxt[who]
        if op[0] == "issue":
            pipe.append(op[1])
        elif op[0] == "arrive":
            op[1].arrive()
        elif op[0] == "check" and not op[1]():
            raise Violation(op[2])
        elif op[0] == "do":
            op[1]()
        try:
            nxt[who] = next(agents[who])
        except StopIteration:
            del nxt[who]


def explore(seeds=400, **kw):
    for seed in range(seeds):
        try:
            run(seed=seed, **kw)
        except Violation as e:
            return str(e)
    return None


def test_two_buffers_with_one_shared_p_ready_lets_dv_read_unwritten_columns():
    found = explore(steps=6, warps=4, two_buffers=True, p_ready_per_buffer=False, split_dv=False)
    assert found is not None and found.startswith("dV(")


def test_one_buffer_with_s_issued_before_dv_overwrites_p():
    """The model also catches the ordering mistake the in-order issue rule prevents."""
    found = explore(steps=4, warps=2, two_buffers=False, p_ready_per_buffer=True, split_dv=False, s_early=True)
    assert found is not None


@pytest.mark.parametrize("steps", [1, 2, 7])
def test_two_buffers_with_a_p_ready_per_buffer_is_safe(steps):
    """The d = 64 schedule of the kernel."""
    assert explore(steps=steps, warps=4, two_buffers=True, p_ready_per_buffer=True, split_dv=False) is None


@pytest.mark.parametrize("steps", [1, 2, 7])
def test_one_buffer_with_the_split_dv_issue_is_safe(steps):
    """The d = 128 schedule of the kernel (p_ready per buffer, one buffer: one barrier)."""
    assert explore(steps=steps, warps=4, two_buffers=False, p_ready_per_buffer=True, split_dv=True) is None


def run_forward(steps, warps, split_pv, seed, s_before_pv=False):
    """One random interleaving of the forward's schedule (fwd_pp.cuh): two teams, each
    with its S/P buffer in TMEM, served by one MMA warp in the order PV_A(j), S_A(j+1),
    PV_B(j), S_B(j+1); a team's warps post partial maxima (arrive and wait on xbar, one
    barrier per step parity), write P in two halves (p_half after the first) and arrive
    on p_ready.  ``s_before_pv`` issues S_X(j+1) ahead of PV_X(j) (a mistake)."""
    rnd = random.Random(seed)
    teams = (0, 1)
    bars = {x: {"s_full": Barrier(1), "p_half": Barrier(warps), "p_ready": Barrier(warps),
                "xbar": [Barrier(warps), Barrier(warps)]} for x in teams}
    buf = {x: [[None, None] for _ in range(warps)] for x in teams}   # [warp][half] of P, or S
    pipe = []

    def perform(op):
        kind, x, j, half = op
        if kind == "S":
            for w in range(warps):
                buf[x][w] = [("S", j), ("S", j)]
            bars[x]["s_full"].arrive()
        else:                                        # PV half reads P(j) of every warp
            for w in range(warps):
                for h in ((half,) if half is not None else (0, 1)):
                    if buf[x][w][h] != ("P", j):
                        raise Violation(f"PV_{x}({j}) half {h} read warp {w}'s {buf[x][w][h]}")

    def mma():
        for x in teams:
            yield ("issue", ("S", x, 0, None))
        for j in range(steps):
            for x in teams:
                if s_before_pv and j + 1 < steps:
                    yield ("issue", ("S", x, j + 1, None))
                if split_pv:
                    yield ("wait", bars[x]["p_half"], j & 1)
                    yield ("issue", ("PV", x, j, 0))
                    yield ("wait", bars[x]["p_ready"], j & 1)
                    yield ("issue", ("PV", x, j, 1))
                else:
                    yield ("wait", bars[x]["p_ready"], j & 1)
                    yield ("issue", ("PV", x, j, None))
                if not s_before_pv and j + 1 < steps:
                    yield ("issue", ("S", x, j + 1, None))

    def warp(x, w):
        for j in range(steps):
            yield ("wait", bars[x]["s_full"], j & 1)
            yield ("check", lambda j=j: buf[x][w] == [("S", j), ("S", j)], f"team {x} warp {w} read S({j})")
            xb = bars[x]["xbar"][j & 1]
            yield ("arrive", xb)
            yield ("wait", xb, (j >> 1) & 1)
            for h in (0, 1):
                yield ("do", lambda h=h, j=j: buf[x][w].__setitem__(h, ("P", j)))
                if h == 0 and split_pv:
                    yield ("arrive", bars[x]["p_half"])
            yield ("arrive", bars[x]["p_ready"])

    agents = {"mma": mma(), **{f"t{x}w{w}": warp(x, w) for x in teams for w in range(warps)}}
    nxt = {name: next(gen) for name, gen in agents.items()}
    while nxt or pipe:
        ready = [n for n, op in nxt.items() if op[0] != "wait" or op[1].passed(op[2])]
        choices = ready + (["pipe"] if pipe else [])
        if not choices:
            raise Violation("deadlock")
        who = rnd.choice(choices)
        if who == "pipe":
            perform(pipe.pop(0))
            continue
        op = nxt[who]
        if op[0] == "issue":
            pipe.append(op[1])
        elif op[0] == "arrive":
            op[1].arrive()
        elif op[0] == "check" and not op[1]():
            raise Violation(op[2])
        elif op[0] == "do":
            op[1]()
        try:
            nxt[who] = next(agents[who])
        except StopIteration:
            del nxt[who]


def explore_forward(seeds=300, **kw):
    for seed in range(seeds):
        try:
            run_forward(seed=seed, **kw)
        except Violation as e:
            return str(e)
    return None


@pytest.mark.parametrize("split_pv", [False, True])
def test_forward_schedule_is_safe(split_pv):
    """The forward's schedule, with PV issued whole or in the two halves the kernel uses."""
    assert explore_forward(steps=5, warps=4, split_pv=split_pv) is None


def test_forward_with_s_ahead_of_pv_overwrites_p():
    assert explore_forward(steps=4, warps=2, split_pv=True, s_before_pv=True) is not None


def run_dq(steps, warps, seed, dp_early=False, dp_free_wait=True):
    """One random interleaving of the dQ kernel's schedule: S(j+1) into the other of two
    buffers before dQ(j); the dS warps read S(j) (phase A), then dP(j), arrive on
    dp_free, write dS(j) over S(j) and arrive on ds_ready; dQ(j) reads dS(j); dP(j+1)
    waits for dp_free(j).  ``dp_early`` issues dP(j+1) ahead of the wait for ds_ready(j)
    (a variant that was measured); ``dp_free_wait`` False drops the dp_free wait."""
    rnd = random.Random(seed)
    bars = {"s_full": [Barrier(1), Barrier(1)], "dp_full": Barrier(1), "dp_free": Barrier(warps),
            "ds_ready": Barrier(warps)}
    sbuf = [[None] * warps for _ in range(2)]
    dpbuf = [None] * warps
    pipe = []

    def perform(op):
        kind, j = op
        if kind == "S":
            for w in range(warps):
                sbuf[j % 2][w] = ("S", j)
            bars["s_full"][j % 2].arrive()
        elif kind == "dP":
            for w in range(warps):
                dpbuf[w] = ("dP", j)
            bars["dp_full"].arrive()
        else:
            for w in range(warps):
                if sbuf[j % 2][w] != ("dS", j):
                    raise Violation(f"dQ({j}) read warp {w}'s {sbuf[j % 2][w]}")

    def mma():
        yield ("issue", ("S", 0))
        yield ("issue", ("dP", 0))
        def dp_next(j):
            if dp_free_wait:
                yield ("wait", bars["dp_free"], j & 1)
            yield ("issue", ("dP", j + 1))

        for j in range(steps):
            if j + 1 < steps:
                yield ("issue", ("S", j + 1))
            if dp_early and j + 1 < steps:
                yield from dp_next(j)
            yield ("wait", bars["ds_ready"], j & 1)
            yield ("issue", ("dQ", j))
            if not dp_early and j + 1 < steps:
                yield from dp_next(j)

    def warp(w):
        for j in range(steps):
            yield ("wait", bars["s_full"][j % 2], (j >> 1) & 1)
            yield ("check", lambda j=j: sbuf[j % 2][w] == ("S", j), f"warp {w} read S({j})")
            yield ("wait", bars["dp_full"], j & 1)
            yield ("check", lambda j=j: dpbuf[w] == ("dP", j), f"warp {w} read dP({j})")
            yield ("arrive", bars["dp_free"])
            yield ("do", lambda j=j: sbuf[j % 2].__setitem__(w, ("dS", j)))
            yield ("arrive", bars["ds_ready"])

    agents = {"mma": mma(), **{f"w{w}": warp(w) for w in range(warps)}}
    nxt = {name: next(gen) for name, gen in agents.items()}
    while nxt or pipe:
        ready = [n for n, op in nxt.items() if op[0] != "wait" or op[1].passed(op[2])]
        choices = ready + (["pipe"] if pipe else [])
        if not choices:
            raise Violation("deadlock")
        who = rnd.choice(choices)
        if who == "pipe":
            perform(pipe.pop(0))
            continue
        op = nxt[who]
        if op[0] == "issue":
            pipe.append(op[1])
        elif op[0] == "arrive":
            op[1].arrive()
        elif op[0] == "check" and not op[1]():
            raise Violation(op[2])
        elif op[0] == "do":
            op[1]()
        try:
            nxt[who] = next(agents[who])
        except StopIteration:
            del nxt[who]


def first_dq_violation(**kw):
    for seed in range(300):
        try:
            run_dq(seed=seed, **kw)
        except Violation as e:
            return str(e)
    return None


def test_dq_schedule_is_safe():
    """The kernel's order: dP(j+1) behind dQ(j), which waited for every warp's dS(j)."""
    assert first_dq_violation(steps=6, warps=4) is None


def test_dq_with_dp_ahead_of_dq_lets_ds_ready_complete_early():
    """dP(j+1) ahead of dQ(j) (a measured variant, not kept) lets a fast warp reach
    step j+1's dS and arrive on ds_ready before a slow warp's step-j arrival, even with
    the dp_free wait: the same run-ahead as the old d = 64 dK/dV schedule.  Depending on
    the interleaving dQ(j) reads unwritten dS, or the MMA warp's parity wait sees the
    barrier two phases on and waits for good."""
    outcomes = set()
    for seed in range(300):
        try:
            run_dq(steps=4, warps=4, seed=seed, dp_early=True)
            outcomes.add("ok")
        except Violation as e:
            outcomes.add("deadlock" if str(e) == "deadlock" else str(e).split("(")[0])
    assert "dQ" in outcomes                     # a read of unwritten dS is reachable


def test_dq_with_dp_ahead_and_no_dp_free_wait_overwrites_dp():
    assert first_dq_violation(steps=4, warps=2, dp_early=True, dp_free_wait=False) is not None
