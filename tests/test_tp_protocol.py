"""The head split's cross-rank ordering, as a model run on CPU.

The fused o-projection reduction (include/mla_tp.h) orders the ranks through two
arrival counters per rank. Its kernels run on one GPU here (every rank inside one
launch), where the ranks' steps never interleave the way separate GPUs can. This
test replays the protocol's steps per rank, in the order the kernels take them, under
many random interleavings of the ranks, and checks each rank's output every step:

  projection (per rank, per step): for each block of K, add the rank's partial
      sums of every owner's columns into that owner's accumulator, then count the
      block at every owner's counter 0;
  finish (per rank): wait until counter 0 reaches step x ranks x blocks; read and
      zero its accumulator; write the rounded columns into every rank's output;
      count itself at every rank's counter 1; wait until its counter 1 reaches
      step x ranks;
  consumer (per rank): read its output, before that rank's next projection.

A wrong order (zeroing after the count, counting before the adds, a missing wait)
shows up as a wrong sum, a lost contribution or a wait that never ends.
"""
import random

import numpy as np
import pytest


def _run(world, steps, blocks, seed, zero_after_count=False, skip_second_wait=False):
    rng = random.Random(seed)
    cols = 3                                 # columns each rank owns
    acc = [np.zeros(cols) for _ in range(world)]
    out = [np.full(cols * world, np.nan) for _ in range(world)]
    cnt0 = [0] * world
    cnt1 = [0] * world
    partial = {(r, e): np.random.default_rng(1000 * e + r).integers(-8, 9, (world, cols)).astype(float)
               for r in range(world) for e in range(1, steps + 1)}
    want = {e: np.concatenate([sum(partial[(r, e)][c] for r in range(world)) for c in range(world)])
            for e in range(1, steps + 1)}

    def rank_program(r):
        for e in range(1, steps + 1):
            # projection: blocks of K, each reduced into every owner, then counted there
            for b in range(blocks):
                for c in range(world):
                    acc[c] += partial[(r, e)][c] / blocks
                    yield
                for c in range(world):
                    cnt0[c] += 1
                yield
            # finish
            while cnt0[r] < e * world * blocks:
                yield "wait"
            v = acc[r].copy()
            if not zero_after_count:
                acc[r][:] = 0
            for c in range(world):
                out[c][r * cols:(r + 1) * cols] = v
                yield
            for c in range(world):
                cnt1[c] += 1
            if zero_after_count:
                yield
                acc[r][:] = 0
            if not skip_second_wait:
                while cnt1[r] < e * world:
                    yield "wait"
            # consumer of this step's output
            got = out[r].copy()
            results.append((r, e, got))
            yield

    results = []
    progs = {r: rank_program(r) for r in range(world)}
    stalled = 0
    while progs:
        r = rng.choice(sorted(progs))
        try:
            state = next(progs[r])
        except StopIteration:
            del progs[r]
            continue
        stalled = stalled + 1 if state == "wait" else 0
        if stalled > 10000:
            raise RuntimeError("no rank can move")
    return results, want


@pytest.mark.parametrize("world,blocks", [(2, 1), (2, 3), (4, 2), (8, 1)])
def test_every_interleaving_sums_every_rank(world, blocks):
    for seed in range(60):
        results, want = _run(world, steps=4, blocks=blocks, seed=seed)
        assert len(results) == world * 4
        for r, e, got in results:
            np.testing.assert_allclose(got, want[e], rtol=0, atol=1e-12, err_msg=f"rank {r} step {e} seed {seed}")


def test_the_model_sees_a_broken_order():
    # Pins the model itself: a rank that skips the second wait may read its output
    # before every owner has written its columns for this step.
    bad = 0
    for seed in range(60):
        results, want = _run(4, steps=3, blocks=1, seed=seed, skip_second_wait=True)
        bad += any(not np.allclose(got, want[e]) for _, e, got in results)
    assert bad > 0
    # Zeroing the accumulator after counting lets a fast peer's next-step sums be wiped.
    bad = 0
    for seed in range(200):
        results, want = _run(4, steps=3, blocks=2, seed=seed, zero_after_count=True)
        bad += any(not np.allclose(got, want[e]) for _, e, got in results)
    assert bad > 0
