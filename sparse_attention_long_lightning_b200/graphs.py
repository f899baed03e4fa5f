"""CUDA-graph capture of a step built from libsala calls.

A decode step of the hybrid stack is many small launches (per Lightning layer one,
per sparse layer four: block scores, top-k, split attention, combine).  Every libsala
call launches asynchronously on the caller's stream, allocates nothing when its output
and scratch buffers are passed in, and synchronises nowhere, so a whole step can be
captured once as a CUDA graph and replayed with one launch.  The caller keeps the
step's inputs in static tensors and writes the next step's values into them
(``copy_``) before each replay; in-place state updates (the Lightning state, the
block-mean cache) happen inside the graph exactly as in eager execution.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch


def capture_step(step_fn: Callable[[], None], *, warmup: int = 1, pool=None,
                 restore: Optional[Callable[[], None]] = None) -> "torch.cuda.CUDAGraph":
    """Run ``step_fn`` ``warmup`` times eagerly on a side stream (this fills libsala's
    per-device caches and kernel attributes, and applies the step's in-place updates:
    ``restore``, when given, puts the state back after the warm-up and after the
    capture), then capture one call of it into a CUDA graph.  Replay with
    ``graph.replay()`` on the stream that should run it."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):
            step_fn()
    torch.cuda.current_stream().wait_stream(side)
    if restore is not None:
        restore()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, pool=pool):
        step_fn()
    if restore is not None:
        restore()
    return graph


class StaticStep:
    """A captured step with named static inputs: ``set(name=tensor, ...)`` copies the
    next values in, ``replay()`` runs the graph.  ``inputs`` maps names to the static
    tensors that ``step_fn`` reads."""

    def __init__(self, step_fn: Callable[[], None], inputs: dict, *, warmup: int = 1,
                 restore: Optional[Callable[[], None]] = None):
        self.inputs = inputs
        self.graph = capture_step(step_fn, warmup=warmup, restore=restore)

    def set(self, **values):
        for name, value in values.items():
            self.inputs[name].copy_(value, non_blocking=True)

    def replay(self):
        self.graph.replay()
