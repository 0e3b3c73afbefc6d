"""Model check of the single-pass scan's decoupled look-back (CPU).

Tiles draw tickets in order; each publishes its own count (flag 1, or the
inclusive prefix, flag 2, for tile 0), then reads windows of W predecessor
descriptors: it adds every value from the nearest predecessor back to and
including the first inclusive prefix, moves W further back if the window
holds none, and re-reads the window while a descriptor it needs is still
unpublished; finally it publishes its own inclusive prefix.  Under any
interleaving, each tile's result must be the exact exclusive prefix of the
counts.  The model restates the procedure in ep_scan.cuh; the GPU parity
tests check the kernels themselves."""
import random

import pytest


def tile(j, counts, desc, result, W):
    agg = counts[j]
    if j == 0:
        desc[0] = (2, agg)
        result[0] = 0
        return
    desc[j] = (1, agg)
    yield
    excl = 0
    base = j - 1
    while True:
        window = [desc[base - u] if base - u >= 0 else (2, 0) for u in range(W)]
        pstar = next((u for u, (f, _) in enumerate(window) if f == 2), W)
        if any(window[u][0] == 0 for u in range(min(pstar + 1, W))):
            yield          # a predecessor has not published yet: read again later
            continue
        excl += sum(window[u][1] for u in range(min(pstar + 1, W)))
        if pstar < W:
            break
        base -= W
        yield
    desc[j] = (2, excl + agg)
    result[j] = excl


@pytest.mark.parametrize("seed", range(40))
def test_exclusive_prefix_under_random_interleavings(seed):
    rng = random.Random(seed)
    n = rng.choice([1, 2, 5, 17, 64, 200])
    W = rng.choice([1, 4, 16, 32, 64])
    counts = [rng.randint(0, 9) for _ in range(n)]
    desc = [(0, 0)] * n
    result = [None] * n
    started, live = 0, {}
    steps = 0
    while started < n or live:
        # a tile only starts after every lower ticket has started (ticket order)
        if started < n and (not live or rng.random() < 0.3):
            live[started] = tile(started, counts, desc, result, W)
            started += 1
            continue
        j = rng.choice(list(live))
        try:
            next(live[j])
        except StopIteration:
            del live[j]
        steps += 1
        assert steps < 200 * n * n + 1000, "a tile never finished"
    expect = [sum(counts[:j]) for j in range(n)]
    assert result == expect
