"""One CUDA graph over a fixed sequence of decode-step calls.

A model with many linear-attention layers runs one ``damp_decode_step`` per
layer for every generated token; each call is a single kernel launch on the
pools' stream.  ``DecodeGraph`` captures such a sequence once, on static
argument buffers, and replays it with one ``cudaGraphLaunch`` per token, so the
per-layer host launch cost leaves the critical path.  The caller refreshes the
static buffers in place (for instance ``graph.args[i]["q"].copy_(...)``)
between replays; the graph reads whatever they hold when it runs.

Every kernel in the graph is a libdamp kernel: this module only records and
replays launches.  Kernel attributes are set when a pool is created, so the
captured calls perform no set-up of their own.
"""
from __future__ import annotations

import torch

from . import damp_decode_step

_KEYS = ("slot_idx", "q", "k", "v", "alpha", "beta", "out")


class DecodeGraph:
    """Capture ``damp_decode_step(pool_i, **args_i)`` for i = 0..L-1, in order.

    ``calls`` is a list of ``(pool, args)`` where ``pool`` is a
    :class:`DampPool` (or a raw handle) and ``args`` a dict holding the device
    tensors ``slot_idx, q, k, v, alpha, beta, out``.  Those tensors stay owned
    by the caller and must outlive the graph.  Capturing does not run the
    steps: no pool is modified until the first :meth:`replay`.
    """

    def __init__(self, calls, device=None):
        self.calls = []
        for pool, args in calls:
            missing = [k for k in _KEYS if k not in args]
            if missing:
                raise ValueError(f"decode call lacks {missing}")
            handle = getattr(pool, "handle", pool)
            self.calls.append((handle, {k: args[k] for k in _KEYS}))
        if not self.calls:
            raise ValueError("DecodeGraph needs at least one call")
        self.device = device or self.calls[0][1]["q"].device
        self.graph = torch.cuda.CUDAGraph()
        self.stream = torch.cuda.Stream(self.device)
        # Capture on a side stream that first waits for the work already queued.
        self.stream.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(self.stream):
            self.graph.capture_begin()
            try:
                for handle, a in self.calls:
                    damp_decode_step(handle, a["slot_idx"], a["q"], a["k"], a["v"],
                                     a["alpha"], a["beta"], a["out"], stream=self.stream)
            finally:
                self.graph.capture_end()
        torch.cuda.current_stream(self.device).wait_stream(self.stream)

    @property
    def args(self):
        return [a for _, a in self.calls]

    def replay(self):
        """Run every captured step once, in capture order, on the current stream."""
        self.graph.replay()

    def reset(self):
        self.graph.reset()
