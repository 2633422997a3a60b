"""Model of the decode-attention kernel's shared-memory pipeline (CPU only).

The kernel streams blocks through NS shared-memory stages: a producer warp
waits on the stage's "empty" mbarrier, arms the "full" mbarrier with the
expected bytes and issues the bulk copies; unit k lands in stage k % NS and
is consumed by warp k % NCW, which waits on "full" by phase parity and then
arrives on "empty".  Consumer warps also meet at a named barrier at the end
of every head piece.  Parity waits only distinguish a phase from the one
before it, so a stage must always be consumed by the same warp, i.e. NS must
be a multiple of NCW.  This model replays the protocol under random
interleavings and out-of-order copy completion and checks that no warp ever
reads a stage before its copy landed and that no barrier receives an extra
arrival.  It also shows that a shared-stage layout (NS=6, NCW=4, the layout
that faulted on the 128K-context workload) breaks.
"""
import random

import pytest

# (stages, consumer warps) of each kernel variant: bf16 D=128, bf16 D=64,
# FP8 D=128, 4-bit D=128, fp32 D=64, fp32 D=128
KERNEL_LAYOUTS = [(6, 6), (8, 8), (12, 6), (14, 7), (4, 4), (3, 3)]


class MBarrier:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def arrive(self, tx=0):
        assert self.pending > 0, "arrival on a barrier with no pending arrivals"
        self.pending -= 1
        self.tx += tx
        self._complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def parity_done(self, parity):
        return (self.phase & 1) != parity


def replay(n_units, piece_ends, NS, NCW, seed):
    rnd = random.Random(seed)
    full = [MBarrier(1) for _ in range(NS)]
    empty = [MBarrier(1) for _ in range(NS)]
    holds = [None] * NS          # ("loading", k, copies left) | ("ready", k)
    inflight = []
    issued = 0
    cons = [{"u": 0, "st": "walk"} for _ in range(NCW)]
    at_barrier = set()
    for _ in range(60 * n_units + 1000):
        order = ["P", "T"] + list(range(NCW))
        rnd.shuffle(order)
        for a in order:
            if a == "P" and issued < n_units:
                s, ph = issued % NS, (issued // NS) & 1
                if empty[s].parity_done(ph ^ 1):
                    assert holds[s] is None, "copy issued into a stage still in use"
                    full[s].arrive(tx=3)                      # K tile, V tile, query rows
                    inflight += [(s, issued)] * 3
                    holds[s] = ("loading", issued, 3)
                    issued += 1
            elif a == "T" and inflight:
                s, k = inflight.pop(rnd.randrange(len(inflight)))
                left = holds[s][2] - 1
                holds[s] = ("loading", k, left) if left else ("ready", k)
                full[s].complete_tx(1)
            elif a not in ("P", "T"):
                c = cons[a]
                u = c["u"]
                if u >= n_units:
                    continue
                if c["st"] == "walk":
                    if u % NCW == a:
                        s, ph = u % NS, (u // NS) & 1
                        if not full[s].parity_done(ph):
                            continue
                        assert holds[s] == ("ready", u), f"unit {u} read before its copy landed"
                        holds[s] = None
                        empty[s].arrive()
                    c["st"] = "bar" if u in piece_ends else "next"
                    if c["st"] == "bar":
                        at_barrier.add(a)
                if c["st"] == "bar" and len(at_barrier) == NCW:
                    for cc in cons:
                        if cc["st"] == "bar":
                            cc["st"] = "next"
                    at_barrier.clear()
                if c["st"] == "next":
                    c["u"] += 1
                    c["st"] = "walk"
        if issued >= n_units and not inflight and all(c["u"] >= n_units for c in cons):
            return
    raise AssertionError("no progress: deadlock")


def _cases(rng, n):
    for trial in range(n):
        U = rng.choice([3, 17, 53, 300, 1500])
        ends = set(rng.randrange(U) for _ in range(max(1, U // 40))) | {U - 1}
        yield U, ends, trial


@pytest.mark.parametrize("NS,NCW", sorted(set(KERNEL_LAYOUTS)))
def test_kernel_stage_layouts_never_break_the_protocol(NS, NCW):
    assert NS % NCW == 0
    for U, ends, trial in _cases(random.Random(NS * 10 + NCW), 40):
        replay(U, ends, NS, NCW, seed=trial)


def test_shared_stages_break_the_protocol():
    broken = 0
    for U, ends, trial in _cases(random.Random(5), 40):
        try:
            replay(U, ends, 6, 4, seed=trial)
        except AssertionError:
            broken += 1
    assert broken > 0

