"""The pipelined denoising window with a KV range per denoising stage (host side): the
slice lists of a stage schedule with a transition, checked pair by pair against the
definition, and plan reuse as the window slides (MAGI-1 research notes, "Inference
tricks > KV Cache": a limited KV range, and a range of 1 at chosen denoising stages for
controllable transitions)."""
import numpy as np

import oracle
from block_causal_attention_b200.streaming import PipelinedWindow


def _expected_mask(first, window, cache_chunks, C, rng_of):
    """Visible (query, key) pairs from the definition: the chunk at absolute index c sees
    the chunks [c - R, c]; cache key k belongs to absolute chunk first - cache_chunks + k // C
    and window key n to chunk first + n // C."""
    nq, nc = window * C, cache_chunks * C
    m = np.zeros((nq, nc + nq), bool)
    for i in range(nq):
        c = first + i // C
        R = rng_of(i // C, c)
        for k in range(nc + nq):
            a = first - cache_chunks + k // C if k < nc else first + (k - nc) // C
            m[i, k] = c - R <= a <= c
    return m


def test_stage_schedule_slices_match_the_definition():
    C, W_, NC, R = 6, 4, 5, 3
    win = PipelinedWindow(4, 2, 24, 1, 2, 3, W_, NC, R, host_only=True)
    win.add_transition(9, stages=(2, 3), kv_range=1)      # shot change: range 1 at the two noisiest stages
    win.add_transition(12, stages=(0,), kv_range=0)       # detail change: the chunk alone at the last stage

    def rng_of(p, c):
        if c == 9 and p in (2, 3):
            r = 1
        elif c == 12 and p == 0:
            r = 0
        else:
            r = R
        return min(r, NC + p, c)

    for first in range(0, 14):
        rg = win.ranges(first)
        assert rg == tuple(rng_of(p, first + p) for p in range(W_))
        got = oracle.mask_dense(win.slices(rg), W_ * C, (NC + W_) * C)
        assert np.array_equal(got, _expected_mask(first, W_, NC, C, rng_of)), first


def test_plans_are_compiled_once_per_layout_and_moved_otherwise():
    win = PipelinedWindow(4, 2, 24, 2, 3, 4, 4, 8, 4, host_only=True)
    win.add_transition(10, stages=(2, 3), kv_range=1)
    layouts = set()
    for first in range(4, 16):
        p = win.plan(first)
        layouts.add(win.ranges(first))
        assert p.info()["num_q"] == 4 * 24
    assert win.compiles == len(layouts) < 12
    win.close()
