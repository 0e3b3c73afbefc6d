"""Model check of the full-grid phase timer protocol (CPU).

The protocol is the notify timer of the DeepEP PR #720 page ("Notify
full-kernel duration"), as the library's phase timers carry it out: thread 0
of each block publishes its start as ~t through atomicMax (the largest
complement is the earliest start); at its end each block adds one to a
completion count, and the block that brings the count to the grid size adds
end - start to the cumulative sum, counts the launch and clears the two
working words for the next launch.  A block's start is performed before its
count (in the kernels: the start is taken in an earlier kernel of the stream,
or thread 0 consumes the start's returned value before it counts).

Under every interleaving of the blocks' steps that keeps that order, each
launch must add exactly (last end - earliest start) and leave the working
words at zero.  A planted reordering -- a start performed after the block's
count -- must break it, which shows that the ordering is what the kernels
need.  The model restates the protocol in ep_common.cuh; the GPU tests check
the kernels themselves."""
import itertools
import random

import pytest

MASK = (1 << 64) - 1


class Timer:
    def __init__(self):
        self.start_c = 0
        self.done = 0
        self.sum_ns = 0
        self.launches = 0


def block(t, b, blocks, start, end, reorder=False):
    """Generator: the block's atomic steps, one per yield."""
    def begin():
        t.start_c = max(t.start_c, ~start & MASK)

    def count():
        t.done += 1
        if t.done == blocks:  # the last block closes the launch
            s = ~t.start_c & MASK
            t.start_c = 0
            t.sum_ns += end_of_launch[0] - s if end_of_launch else 0
            t.launches += 1
            t.done = 0

    if not reorder:
        begin()
        yield
        count()
    else:  # the start lands after the count
        count()
        yield
        begin()
    yield


end_of_launch = []  # the last block's clock when it closes (set per launch)


def run_launch(t, starts, ends, order, reorder_block=None):
    """One launch of len(starts) blocks; `order` lists which block steps
    next.  The clock of the closing block is the latest end."""
    end_of_launch.clear()
    end_of_launch.append(max(ends))
    gens = {b: block(t, b, len(starts), starts[b], ends[b], reorder=(b == reorder_block))
            for b in range(len(starts))}
    for b in order:
        try:
            next(gens[b])
        except StopIteration:
            pass
    for g in gens.values():  # drain
        for _ in g:
            pass


def interleavings(blocks, steps=2):
    """Every order of `steps` steps per block that keeps each block's steps in order."""
    seq = [b for b in range(blocks) for _ in range(steps)]
    seen = set()
    for p in itertools.permutations(seq):
        if p not in seen:
            seen.add(p)
            yield p


@pytest.mark.parametrize("blocks", [1, 2, 3])
def test_every_interleaving_adds_the_launch_span_and_clears(blocks):
    rng = random.Random(blocks)
    t = Timer()
    total = 0
    for order in interleavings(blocks):
        starts = [rng.randint(1_000, 2_000) for _ in range(blocks)]
        ends = [s + rng.randint(10, 500) for s in starts]
        run_launch(t, starts, ends, order)
        total += max(ends) - min(starts)
        assert t.start_c == 0 and t.done == 0
    assert t.sum_ns == total
    assert t.launches == sum(1 for _ in interleavings(blocks))


@pytest.mark.parametrize("seed", range(20))
def test_random_grids_over_many_launches(seed):
    rng = random.Random(100 + seed)
    t = Timer()
    total = 0
    for _ in range(rng.randint(1, 6)):
        blocks = rng.randint(1, 12)
        starts = [rng.randint(0, 10_000) for _ in range(blocks)]
        ends = [s + rng.randint(1, 5_000) for s in starts]
        order = [b for b in range(blocks) for _ in range(2)]
        rng.shuffle(order)
        # keep each block's steps in order: the k-th occurrence of b is its k-th step
        run_launch(t, starts, ends, order)
        total += max(ends) - min(starts)
        assert t.start_c == 0 and t.done == 0
    assert t.sum_ns == total


def test_a_start_performed_after_its_count_breaks_the_launch():
    """Planted mistake: block 1's start lands after the last count.  The
    launch loses its earliest start, and the stray start is left in the
    working word, where it corrupts the next launch."""
    t = Timer()
    starts, ends = [1_000, 500], [1_200, 900]
    # block 0 begins, block 1 counts (early), block 0 counts (closes), block 1 begins late
    run_launch(t, starts, ends, order=[0, 1, 0, 1], reorder_block=1)
    assert t.sum_ns != max(ends) - min(starts)
    assert t.start_c != 0  # the next launch would start from a stale stamp
