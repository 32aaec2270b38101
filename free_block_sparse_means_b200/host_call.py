"""SparsePR calls on host (pinned) buffers with the transfers overlapped.

The (batch, head) pairs of a call are independent [paperlayer §4: every step
is per head], so a call over host tensors can run in chunks of heads: the
inputs of chunk c are copied in while chunk c - 1 computes, and the output of
chunk c - 1 is copied out while chunk c computes (three CUDA streams,
double-buffered device tensors, one workspace).  Each chunk is an ordinary
sparsepr_call through the C ABI with head0 set to the chunk's first flattened
head, so every head draws the same k-means initial rows as in one call over
all heads and the output is the same.

This module only schedules copies and calls; all arithmetic runs in the
library's kernels.
"""
from __future__ import annotations

import torch

from . import _binding as spr


class HostPipeline:
    """Device buffers, workspace and streams for repeated calls on host
    tensors of one shape [B, H, N, d] (bf16, contiguous, pinned)."""

    def __init__(self, shape, heads_per_chunk: int, device=None, **params):
        B, H, N, d = shape
        self.BH, self.N, self.d = B * H, N, d
        self.hc = max(1, min(int(heads_per_chunk), self.BH))
        self.device = torch.device(device or "cuda")
        self.params = dict(params)
        shp = (1, self.hc, N, d)
        mk = lambda: torch.empty(shp, dtype=torch.bfloat16, device=self.device)  # noqa: E731
        self.qkv = [[mk(), mk(), mk()] for _ in range(2)]
        self.out = [mk(), mk()]
        self._prm = {}
        self.ws = spr.alloc_workspace(self._params(self.hc, 0), device=self.device)
        self.s_in = torch.cuda.Stream(self.device)
        self.s_comp = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)

    def chunks(self):
        return [(h0, min(self.BH, h0 + self.hc)) for h0 in range(0, self.BH, self.hc)]

    def _params(self, n: int, head0: int, b: int = 0):
        key = (n, head0, b)
        if key not in self._prm:
            Q, K, V = (t[:, :n] for t in self.qkv[b])
            self._prm[key] = spr.make_params(Q, K, V, self.out[b][:, :n], head0=head0,
                                             **self.params)
        return self._prm[key]

    def __call__(self, Qh, Kh, Vh, Oh, stream=None):
        """Enqueue the whole call; `stream` (default: the current stream) is
        ordered before the first copy and after the last one."""
        stream = stream or torch.cuda.current_stream(self.device)
        flat = [t.view(self.BH, self.N, self.d) for t in (Qh, Kh, Vh, Oh)]
        start = torch.cuda.Event()
        start.record(stream)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)
        ev_in, ev_comp, ev_out = [], [], []
        for c, (h0, h1) in enumerate(self.chunks()):
            b, n = c % 2, h1 - h0
            # inputs: buffer b was last read by the computation of chunk c - 2
            if c >= 2:
                self.s_in.wait_event(ev_comp[c - 2])
            with torch.cuda.stream(self.s_in):
                for dev, host in zip(self.qkv[b], flat[:3]):
                    dev[0, :n].copy_(host[h0:h1], non_blocking=True)
            ev_in.append(torch.cuda.Event())
            ev_in[c].record(self.s_in)
            # compute: its output buffer was last copied out for chunk c - 2
            self.s_comp.wait_event(ev_in[c])
            if c >= 2:
                self.s_comp.wait_event(ev_out[c - 2])
            Q, K, V = (t[:, :n] for t in self.qkv[b])
            spr.sparsepr_call(self._params(n, h0, b), Q, K, V, self.out[b][:, :n], self.ws,
                              self.s_comp)
            ev_comp.append(torch.cuda.Event())
            ev_comp[c].record(self.s_comp)
            # output
            self.s_out.wait_event(ev_comp[c])
            with torch.cuda.stream(self.s_out):
                flat[3][h0:h1].copy_(self.out[b][0, :n], non_blocking=True)
            ev_out.append(torch.cuda.Event())
            ev_out[c].record(self.s_out)
        stream.wait_event(ev_out[-1])
        stream.wait_event(ev_comp[-1])
        return self
