"""Model of the compaction planner's arrival tickets (CPU only).

The plan kernel runs one CTA per (256-token chunk, sequence).  Each CTA
writes its chunk's kept counts, fences, and takes a ticket from its
sequence's counter; the CTA that draws the last ticket scans that sequence's
counts, resets the counter, fences and takes a ticket from the layer counter;
the CTA that draws the last of those plans the layer (reading every
sequence's totals) and resets that counter.  With one sequence the second
ticket is skipped.  No CTA ever waits, so any interleaving must give exactly
one scan per sequence and one plan, each reading only values already
written, and leave every counter at zero for the next call.  This model runs
the protocol under random interleavings of the CTAs' steps (memory is
sequentially consistent at the fences, which is what the kernel's
__threadfence before every ticket provides) and checks those properties over
several consecutive calls that share the counters.
"""
import random

import pytest


def run_call(n_chunks, batch, tickets, rng, refused=False):
    """One plan-kernel launch; returns (scans per sequence, plans, values seen)."""
    counts = [[None] * n_chunks for _ in range(batch)]
    totals = [None] * batch
    scans = [0] * batch
    plans = []
    seen = []

    def cta(b, c):
        counts[b][c] = (b, c)                 # chunk counts
        yield                                 # fence, then the sequence ticket
        t = tickets[b]
        tickets[b] = t + 1
        if t != n_chunks - 1:
            return
        yield
        assert all(x is not None for x in counts[b]), "scan before every chunk count was written"
        scans[b] += 1
        totals[b] = b
        tickets[b] = 0
        if batch > 1:
            yield                             # fence, then the layer ticket
            t2 = tickets[-1]
            tickets[-1] = t2 + 1
            if t2 != batch - 1:
                return
            yield
            tickets[-1] = 0
        assert all(x is not None for x in totals), "plan before every sequence total was written"
        seen.append(list(totals))
        plans.append("refused" if refused else "planned")

    live = [cta(b, c) for b in range(batch) for c in range(n_chunks)]
    while live:
        g = rng.choice(live)
        try:
            next(g)
        except StopIteration:
            live.remove(g)
    return scans, plans, seen


@pytest.mark.parametrize("n_chunks,batch", [(1, 1), (32, 1), (4, 3), (7, 8), (2, 16)])
def test_one_scan_per_sequence_one_plan_counters_reset(n_chunks, batch):
    rng = random.Random(1000 * n_chunks + batch)
    tickets = [0] * (batch + 1)             # per-sequence counters, then the layer counter
    for call in range(30):
        scans, plans, seen = run_call(n_chunks, batch, tickets, rng, refused=call % 7 == 3)
        assert scans == [1] * batch
        assert len(plans) == 1 and seen == [list(range(batch))]
        assert tickets == [0] * (batch + 1), "a counter was left set for the next call"


def test_a_counter_left_set_breaks_the_next_call():
    """Why the counters must be reset by the CTAs that consume them: a counter
    left one ahead makes the next call scan before its last chunk is counted."""
    rng = random.Random(7)
    with pytest.raises(AssertionError):
        for _ in range(50):
            tickets = [1, 0]                # sequence 0's counter one ahead
            run_call(4, 1, tickets, rng)
