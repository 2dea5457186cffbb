"""The mbarrier protocols of the forward and backward kernels, checked on the
CPU for deadlock and phase aliasing under random schedules.

Each kernel role (TMA producer, MMA issuer, each softmax / elementwise /
dQ-drain warp) is modelled as its own agent: the sequence of barrier waits
and arrivals it performs, transcribed from the kernel source.  A TMA load and
an MMA commit are modelled as arrivals made when the role issues them (the
hardware makes them later, which only removes schedules, never adds one).

An mbarrier is waited on by phase parity, so a wait for phase k that begins
after phases k and k+1 have both completed sees the parity of the running
phase and hangs: "phase aliasing".  The checker tracks the intended phase
index of every wait and fails on aliasing as well as on deadlock (no agent
can move while some have not finished).  A mutant that drops one wait from
a protocol variant that needs it must be caught, which shows that the
checker has teeth.
"""
import random

import pytest


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0   # completed phases

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


class Aliased(Exception):
    pass


def run_schedule(barriers, agents, seed):
    """Runs the agents (generators of ("wait", name, k) / ("arrive", name))
    under a random schedule.  Returns the agents left unfinished."""
    rng = random.Random(seed)
    cur = [next(a, None) for a in agents]
    while True:
        ready = []
        for i, op in enumerate(cur):
            if op is None:
                continue
            if op[0] == "wait":
                b = barriers[op[1]]
                if b.phase > op[2] + 1:
                    raise Aliased("%r waits for phase %d of %r, already at %d"
                                  % (i, op[2], op[1], b.phase))
                if b.phase < op[2] + 1:
                    continue
            ready.append(i)
        if not ready:
            break
        i = rng.choice(ready)
        if cur[i][0] == "arrive":
            barriers[cur[i][1]].arrive()
        cur[i] = next(agents[i], None)
    return [i for i, op in enumerate(cur) if op is not None]


# --------------------------------------------------------------- forward
def forward_protocol(n_t, p_smem, ns, warps_per_tile=4, drop_p_free_wait=False):
    """fwd_kernel: producer (warp 8), MMA issuer (warp 9), softmax warps of
    Q tiles 0 and 1.  n_t = K/V tiles of each Q tile; p_smem selects the
    d = 64 order (P in shared memory), else the d = 128 order (P in TMEM)."""
    nmax = max(n_t)
    W = warps_per_tile
    bars = {}
    for t in range(2):
        bars[("q_full", t)] = Barrier(1)
        bars[("s_full", t)] = Barrier(1)
        bars[("s_free", t)] = Barrier(W)
        bars[("p_full", t)] = Barrier(W)
        bars[("p_free", t)] = Barrier(1)
    for s in range(ns):
        bars[("kv_full", s)] = Barrier(1)
        bars[("kv_empty", s)] = Barrier(1)

    def producer():
        for t in range(2):
            if n_t[t]:
                yield ("arrive", ("q_full", t))
        for n in range(2 * nmax):
            if n >= ns:
                yield ("wait", ("kv_empty", n % ns), n // ns - 1)
            yield ("arrive", ("kv_full", n % ns))

    def issuer():
        if nmax == 0:
            return
        for t in range(2):
            if n_t[t]:
                yield ("wait", ("q_full", t), 0)
        yield ("wait", ("kv_full", 0), 0)
        for t in range(2):
            if n_t[t]:
                yield ("arrive", ("s_full", t))
        yield ("arrive", ("kv_empty", 0))
        for j in range(nmax):
            nv, nk = 2 * j + 1, 2 * j + 2
            has_next = j + 1 < nmax
            if p_smem:
                if has_next:
                    yield ("wait", ("kv_full", nk % ns), nk // ns)
                yield ("wait", ("kv_full", nv % ns), nv // ns)
                for t in range(2):
                    if has_next and j + 1 < n_t[t]:
                        yield ("wait", ("s_free", t), j)
                        yield ("arrive", ("s_full", t))
                    if j < n_t[t]:
                        yield ("wait", ("p_full", t), j)
                        yield ("arrive", ("p_free", t))
                if has_next:
                    yield ("arrive", ("kv_empty", nk % ns))
                yield ("arrive", ("kv_empty", nv % ns))
            else:
                yield ("wait", ("kv_full", nv % ns), nv // ns)
                if j < n_t[0]:
                    yield ("wait", ("p_full", 0), j)
                    yield ("arrive", ("p_free", 0))
                if has_next:
                    yield ("wait", ("kv_full", nk % ns), nk // ns)
                    if j + 1 < n_t[0]:
                        yield ("arrive", ("s_full", 0))
                if j < n_t[1]:
                    yield ("wait", ("p_full", 1), j)
                    yield ("arrive", ("p_free", 1))
                yield ("arrive", ("kv_empty", nv % ns))
                if has_next:
                    if j + 1 < n_t[1]:
                        yield ("arrive", ("s_full", 1))
                    yield ("arrive", ("kv_empty", nk % ns))

    def softmax_warp(t):
        n = n_t[t]
        for j in range(n):
            yield ("wait", ("s_full", t), j)
            yield ("arrive", ("s_free", t))
            if p_smem and j > 0 and not drop_p_free_wait:
                yield ("wait", ("p_free", t), j - 1)
            yield ("arrive", ("p_full", t))
        if n:
            yield ("wait", ("p_free", t), n - 1)

    agents = [producer(), issuer()]
    for t in range(2):
        agents += [softmax_warp(t) for _ in range(W)]
    return bars, agents


FWD_CASES = [(1, 2), (3, 4), (7, 8), (4, 4), (1, 0), (3, 0), (15, 16)]


@pytest.mark.parametrize("p_smem,ns", [(True, 6), (False, 3)], ids=["d64", "d128"])
@pytest.mark.parametrize("n_t", FWD_CASES)
def test_forward_protocol(p_smem, ns, n_t):
    for seed in range(150):
        bars, agents = forward_protocol(n_t, p_smem, ns)
        assert run_schedule(bars, agents, seed) == [], (n_t, seed)


def test_forward_mutant_is_caught():
    # without the wait for the previous P V, a d = 64 softmax warpgroup can
    # arrive on p_full for two tiles before the issuer has taken the first
    caught = 0
    for seed in range(150):
        bars, agents = forward_protocol((3, 4), True, 6, drop_p_free_wait=True)
        try:
            if run_schedule(bars, agents, seed):
                caught += 1
        except Aliased:
            caught += 1
    assert caught > 0


# -------------------------------------------------------------- backward
def backward_protocol(T, d, do_stages=2, warps=8, drain_warps=4):
    """bwd_main_kernel: producer (warp 12), MMA issuer (warp 13), the eight
    elementwise warps and the four dQ-drain warps, over T (query head,
    query tile) iterations."""
    bars = {("kv_full",): Barrier(1), ("s_full",): Barrier(1), ("dp_full",): Barrier(1),
            ("p_full",): Barrier(warps), ("ds_full",): Barrier(warps),
            ("ds_empty",): Barrier(1), ("dq_full",): Barrier(1),
            ("dq_empty",): Barrier(drain_warps), ("dkv_done",): Barrier(1)}
    for s in range(2):
        bars[("q_full", s)] = Barrier(1)
        bars[("q_empty", s)] = Barrier(1)
        bars[("st_full", s)] = Barrier(1)
    for s in range(do_stages):
        bars[("do_full", s)] = Barrier(1)
        bars[("do_empty", s)] = Barrier(1)

    def producer():
        yield ("arrive", ("kv_full",))
        for n in range(T):
            s = n & 1
            if n >= 2:
                yield ("wait", ("q_empty", s), n // 2 - 1)
            yield ("arrive", ("q_full", s))
            sd = n % do_stages
            if n >= do_stages:
                yield ("wait", ("do_empty", sd), n // do_stages - 1)
            yield ("arrive", ("do_full", sd))
            yield ("arrive", ("st_full", s))

    def issuer():
        yield ("wait", ("kv_full",), 0)
        yield ("wait", ("q_full", 0), 0)
        yield ("arrive", ("s_full",))
        yield ("wait", ("do_full", 0), 0)
        yield ("arrive", ("dp_full",))
        for n in range(T):
            s = n & 1
            has_next = n + 1 < T
            yield ("wait", ("p_full",), n)
            yield ("arrive", ("do_empty", n % do_stages))
            if has_next:
                yield ("wait", ("q_full", (n + 1) & 1), (n + 1) >> 1)
                yield ("arrive", ("s_full",))
            yield ("wait", ("ds_full",), n)
            if d != 128 and n > 0:
                yield ("wait", ("dq_empty",), n - 1)
            yield ("arrive", ("dq_full",))
            yield ("arrive", ("q_empty", s))
            yield ("arrive", ("ds_empty",))
            if has_next:
                yield ("wait", ("do_full", (n + 1) % do_stages), (n + 1) // do_stages)
                if d == 128:
                    yield ("wait", ("dq_empty",), n)
                yield ("arrive", ("dp_full",))
        yield ("arrive", ("dkv_done",))

    def drain_warp():
        for n in range(T):
            yield ("wait", ("dq_full",), n)
            yield ("arrive", ("dq_empty",))

    def elementwise_warp():
        for n in range(T):
            yield ("wait", ("s_full",), n)
            yield ("wait", ("st_full", n & 1), n >> 1)
            yield ("arrive", ("p_full",))
            yield ("wait", ("dp_full",), n)
            if n > 0:
                yield ("wait", ("ds_empty",), n - 1)
            yield ("arrive", ("ds_full",))
        yield ("wait", ("dkv_done",), 0)

    agents = [producer(), issuer()]
    agents += [drain_warp() for _ in range(drain_warps)]
    agents += [elementwise_warp() for _ in range(warps)]
    return bars, agents


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 2, 3, 5, 12])
def test_backward_protocol(d, T):
    for seed in range(100):
        bars, agents = backward_protocol(T, d)
        assert run_schedule(bars, agents, seed) == [], (T, d, seed)


def test_checker_catches_a_stalled_consumer():
    # a protocol that lets a producer run two phases ahead of its consumer
    # must be reported, not silently accepted
    bars = {("x",): Barrier(1), ("y",): Barrier(1)}

    def fast():
        yield ("arrive", ("x",))
        yield ("arrive", ("x",))
        yield ("arrive", ("y",))

    def slow():
        yield ("wait", ("y",), 0)
        yield ("wait", ("x",), 0)

    with pytest.raises(Aliased):
        run_schedule(bars, [fast(), slow()], 0)
