"""Model check of the LL dispatch kernel's token-claim protocol (CPU).

Each CTA b takes token b first, then claims tokens from a shared counter
(value + grid size), keeping S stages plus one claim ahead; a stage that
receives -1 ends the CTA's loop.  Under any interleaving of the CTAs' steps,
every token must be processed exactly once and every CTA must stop.  The
model restates the protocol described in ep_ll.cu; the GPU parity tests check
the kernel itself."""
import random

import pytest

S = 2  # input stages of the kernel


class Counter:
    def __init__(self, grid, num_tok):
        self.v = 0
        self.grid = grid
        self.num_tok = num_tok

    def take(self):
        c = self.v + self.grid
        self.v += 1
        return c if c < self.num_tok else -1


def cta(b, counter, processed):
    """Generator: one step per yield, in the kernel's order of claims."""
    stages = [b] + [None] * (S - 1)
    for i in range(1, S):
        stages[i] = counter.take()
        yield
    ahead = counter.take()
    yield
    i = 0
    while True:
        u = stages[i % S]
        if u < 0:
            return
        processed.append(u)
        yield
        nxt = ahead
        ahead = counter.take() if nxt >= 0 else -1
        stages[i % S] = nxt
        i += 1
        yield


@pytest.mark.parametrize("seed", range(40))
def test_every_token_exactly_once_under_random_interleavings(seed):
    rng = random.Random(seed)
    num_tok = rng.choice([1, 2, 3, 7, 64, 300, 1000])
    grid = rng.randint(1, min(num_tok, 40))   # the kernel's grid is at most num_tok
    counter = Counter(grid, num_tok)
    processed = []
    live = {b: cta(b, counter, processed) for b in range(grid)}
    steps = 0
    while live:
        b = rng.choice(list(live))
        try:
            next(live[b])
        except StopIteration:
            del live[b]
        steps += 1
        assert steps < 100 * (num_tok + grid) + 1000, "a CTA did not stop"
    assert sorted(processed) == list(range(num_tok))
