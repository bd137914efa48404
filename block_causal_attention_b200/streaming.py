"""The pipelined denoising window with a KV range per denoising stage.

MAGI-1 generates a video chunk by chunk: a window of consecutive chunks is denoised
together, the oldest chunk (least noise) at the front and the newest (most noise) at the
back, and each step the window slides by one chunk; fully denoised chunks leave the window
and their keys and values stay in a KV cache (MAGI-1 research notes, "Inference tricks >
KV Cache"; the pipelined denoising of the "Magi-1 开源&刷屏" article).  The KV range limits
how many earlier chunks a chunk attends to (a range of 8: each new chunk depends on the 8
chunks before it), and changing the range at chosen denoising stages gives controllable
transitions: a range of 1 at the high-noise stages changes the shot while keeping the
subject, a range of 1 at the low-noise stages keeps the layout and changes the details
(same page).

Readings taken here (the pages give the idea, not the indexing):
  * a window of W chunks; window position p = 0 .. W-1 from the least to the most noisy
    chunk, so a chunk's denoising stage is its window position and it moves to p - 1 each
    step;
  * KV range R: the chunk at absolute index c sees chunks [c - R, c] (fully), taken from the
    cache for chunks before the window and from the window itself (block-causal);
  * the cache holds the `cache_chunks` chunks just before the window, oldest first;
  * a transition at chunk X with stages S: while chunk X sits at a window position in S, its
    range is `transition_range` instead of the normal one.

The slice list of a step depends only on the ranges of the W window positions, so plans are
compiled once per distinct range tuple and reused: each step only moves the plan's start
frame (``Plan.update_positions``), which rewrites the RoPE tables and nothing else.
"""
from __future__ import annotations

import time
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

from . import Plan


class PipelinedWindow:
    """Plans for the W-chunk denoising window of one video, one per distinct KV-range
    layout, moved to each step's frames on demand."""

    def __init__(self, hq: int, hkv: int, d: int, frames: int, height: int, width: int, window: int,
                 cache_chunks: int, kv_range: int, rope_base=(1e4, 1e4, 1e4), eps: float = 1e-6,
                 o_fp32: bool = False, host_only: bool = False):
        if window < 1 or cache_chunks < 0 or kv_range < 0:
            raise ValueError("window >= 1, cache_chunks >= 0 and kv_range >= 0 are required")
        self.hq, self.hkv, self.d = hq, hkv, d
        self.frames, self.height, self.width = frames, height, width
        self.window, self.cache_chunks, self.kv_range = window, cache_chunks, kv_range
        self.rope_base, self.eps, self.o_fp32, self.host_only = tuple(rope_base), eps, o_fp32, host_only
        self.chunk_tokens = frames * height * width
        self.transitions: Dict[int, Tuple[frozenset, int]] = {}
        self._plans: Dict[Tuple[int, ...], Plan] = {}
        self.compiles = 0                 # plans compiled so far (one per distinct layout)
        self.last_host_ms = 0.0           # host time of the last plan() call

    # ------------------------------------------------------------------ schedule
    def add_transition(self, chunk: int, stages: Iterable[int], kv_range: int = 1) -> None:
        """While `chunk` is at one of the window positions `stages`, it sees only the
        `kv_range` chunks before it."""
        self.transitions[int(chunk)] = (frozenset(int(s) for s in stages), int(kv_range))

    def ranges(self, first_chunk: int) -> Tuple[int, ...]:
        """KV range of each window position when the window starts at absolute chunk
        `first_chunk`, clipped to the chunks that exist (the cache and the window)."""
        out = []
        for p in range(self.window):
            c = first_chunk + p
            r = self.kv_range
            tr = self.transitions.get(c)
            if tr is not None and p in tr[0]:
                r = tr[1]
            out.append(min(r, self.cache_chunks + p, c))
        return tuple(out)

    def slices(self, ranges: Sequence[int]) -> np.ndarray:
        """One FULL slice per window chunk: position p sees keys of chunks
        [cache + p - R_p, cache + p] of the [cache | window] key space."""
        C, nc = self.chunk_tokens, self.cache_chunks
        out = [(p * C, (p + 1) * C, (nc + p - int(r)) * C, (nc + p + 1) * C, 0) for p, r in enumerate(ranges)]
        return np.asarray(out, np.int64)

    def videos(self, first_chunk: int) -> np.ndarray:
        return np.asarray([[self.window, self.frames, self.height, self.width, first_chunk * self.frames]], np.int32)

    # ------------------------------------------------------------------ plans
    def plan(self, first_chunk: int, stream=None) -> Plan:
        """The plan of the step whose window starts at absolute chunk `first_chunk`: the
        cached plan of its range layout, moved to the window's frames (compiled the first
        time the layout appears).  The cache given to the plan's fwd must hold the
        `cache_chunks` chunks before the window ([Nc, Hkv, D], Nc = cache_chunks * C)."""
        t = time.perf_counter()
        rg = self.ranges(first_chunk)
        vids = self.videos(first_chunk)
        p = self._plans.get(rg)
        if p is None:
            p = Plan(self.hq, self.hkv, self.d, vids, self.cache_chunks * self.chunk_tokens, self.slices(rg),
                     self.rope_base, self.eps, self.o_fp32, host_only=self.host_only)
            self._plans[rg] = p
            self.compiles += 1
        else:
            p.update_positions(vids, stream=stream)
        self.last_host_ms = (time.perf_counter() - t) * 1e3
        return p

    def close(self) -> None:
        for p in self._plans.values():
            p.close()
        self._plans.clear()
