"""Graph-captured decode step: the indexer as a serving loop calls it.

A decode step of the lightning indexer takes the new query token of every
request (q, w), scores every cached key and keeps the top-k positions.  In
serving, that step runs inside a CUDA graph (the pages' systems capture the
decode step in SGLang's decode graph).  ``DecodeIndexer`` does the same with
the li kernels: at construction it allocates device buffers and pinned host
buffers once and captures

    H2D copy of (q, w)  ->  li_decode_select (score + top-k)  ->  D2H copy of the indices

as one CUDA graph; each ``step()`` writes the host inputs and replays it.

With ``zero_copy`` the transfers are done by the li kernels themselves instead
of DMA copies: a copy kernel reads the page-locked inputs through their mapped
device address, and the top-k writes the selected positions straight into the
page-locked output buffer.  On the B200 boxes measured it was slower than the
DMA copies (PCIe reads from a kernel are latency-bound), so it is off by
default.  Every
kernel in the graph is an li kernel; torch only provides the buffers and the
stream.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import api


class DecodeIndexer:
    """Decode-step indexer over a resident FP8 key cache.

    k8: uint8 [B, L, d] e4m3 cache bytes, ks: fp32 [B, L] per-token scales (device
    tensors, owned by the caller and read in place at every step); H heads; k
    positions kept per request.  ``lens`` (int32 [B], device) optionally limits
    the visible length per request.
    """

    def __init__(self, k8: torch.Tensor, ks: torch.Tensor, heads: int, k: int, lens: Optional[torch.Tensor] = None,
                 zero_copy: bool = False):
        if not (k8.is_cuda and ks.is_cuda):
            raise ValueError("the key cache must be resident on a CUDA device")
        self.k8, self.ks, self.lens = k8, ks, lens
        self.zero_copy = zero_copy
        B, L, d = k8.shape
        self.B, self.L, self.d, self.H, self.k = B, L, d, heads, k
        dev = k8.device
        # q and w travel in one staging buffer: [q bf16 (B*H*d) | w fp32 (B*H)], one copy per step
        qbytes = B * heads * d * 2
        nbytes = qbytes + B * heads * 4
        self.in_dev = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.in_host = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
        self.q_dev = self.in_dev[:qbytes].view(torch.bfloat16).view(B, heads, d)
        self.w_dev = self.in_dev[qbytes:].view(torch.float32).view(B, heads)
        self.q_host = self.in_host[:qbytes].view(torch.bfloat16).view(B, heads, d)
        self.w_host = self.in_host[qbytes:].view(torch.float32).view(B, heads)
        self.scores = torch.empty((B, (L + 3) // 4 * 4), dtype=torch.float32, device=dev)
        self.idx_dev = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.ws = api.li_decode_select_workspace(B, dev, L)
        self.idx_host = torch.empty((B, k), dtype=torch.int32).pin_memory()
        self._launch()  # warm-up: loads the module, sets kernel attributes, checks arguments
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._launch()

    def _launch(self):
        if self.zero_copy:
            api.li_copy_from_host(self.in_dev, self.in_host)
            api.li_decode_select(self.q_dev, self.w_dev, self.k8, self.ks, self.k, lens=self.lens,
                                 scores=self.scores, workspace=self.ws, idx=self.idx_host)
            return
        self.in_dev.copy_(self.in_host, non_blocking=True)
        api.li_decode_select(self.q_dev, self.w_dev, self.k8, self.ks, self.k, lens=self.lens, scores=self.scores,
                             workspace=self.ws, idx=self.idx_dev)
        self.idx_host.copy_(self.idx_dev, non_blocking=True)

    def step(self, q: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None, sync: bool = True):
        """Run one decode step.  q: bf16 [B,H,d] and w: fp32 [B,H] on the host (copied
        into the pinned staging buffers; pass None to use what is already staged).
        Returns the pinned int32 [B, k] host tensor of selected positions (valid
        after the step completes: ``sync=True`` waits for it)."""
        if q is not None:
            self.q_host.copy_(q)
        if w is not None:
            self.w_host.copy_(w)
        self.graph.replay()
        if sync:
            torch.cuda.current_stream().synchronize()
        return self.idx_host

    @property
    def h2d_bytes(self) -> int:
        return self.in_host.numel()

    @property
    def d2h_bytes(self) -> int:
        return self.idx_host.numel() * 4


class DecodePipeline:
    """Independent decode-indexer steps back to back, with their transfers overlapped.

    A serving engine that runs the indexer of many independent steps (other
    request batches, micro-batches in flight together) does not need step i's
    selection before step i+1's inputs can move.  Here ``steps`` such steps
    form one CUDA graph:

        copy stream 1:  H2D(i)   H2D(i+1)   H2D(i+2) ...
        compute:              select(i)  select(i+1)  select(i+2) ...
        copy stream 2:                 D2H(i)     D2H(i+1) ...

    Step i's inputs come from its own page-locked host buffer into device
    slot i % 2 while step i-1's kernels run; its selected positions go from
    device slot i % 2 to its own page-locked host buffer while step i+1's
    kernels run.  Every step still copies its own inputs in and its own result
    out; only the waiting is overlapped.  The slots are reused two steps later,
    after their previous step's kernels (inputs) and result copy (outputs)
    have finished.  Every kernel in the graph is an li kernel.

    ``streams`` compute streams take the steps in turn (step i on stream
    i % streams), each with its own scores and workspace.  With one, the
    steps' kernels run one after another.  With two, step i's top-k (a chain
    of short, latency-bound phases on a few dozen SMs) overlaps step i+1's
    scorer, which streams the cache at HBM bandwidth.

    caches: a list of ``steps`` (k8, ks) key caches, one per step (a cache may
    repeat); heads, k, lens as for ``DecodeIndexer``.  The host inputs are
    ``q_host[i]`` (bf16 [B,H,d]) and ``w_host[i]`` (fp32 [B,H]); ``run()``
    replays the graph and returns the list of pinned int32 [B, k] results.
    """

    def __init__(self, caches, heads: int, k: int, lens: Optional[torch.Tensor] = None, streams: int = 2):
        self.caches = list(caches)
        k8, ks = self.caches[0]
        if not (k8.is_cuda and ks.is_cuda):
            raise ValueError("the key caches must be resident on a CUDA device")
        B, L, d = k8.shape
        self.B, self.L, self.d, self.H, self.k, self.lens = B, L, d, heads, k, lens
        self.steps = S = len(self.caches)
        if streams not in (1, 2):
            raise ValueError("streams must be 1 or 2")
        self.nstreams = streams
        dev = k8.device
        qbytes = B * heads * d * 2
        self.nbytes = nbytes = qbytes + B * heads * 4
        self.in_host = [torch.zeros(nbytes, dtype=torch.uint8).pin_memory() for _ in range(S)]
        self.q_host = [t[:qbytes].view(torch.bfloat16).view(B, heads, d) for t in self.in_host]
        self.w_host = [t[qbytes:].view(torch.float32).view(B, heads) for t in self.in_host]
        self.idx_host = [torch.empty((B, k), dtype=torch.int32).pin_memory() for _ in range(S)]
        self.in_dev = [torch.zeros(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.q_dev = [t[:qbytes].view(torch.bfloat16).view(B, heads, d) for t in self.in_dev]
        self.w_dev = [t[qbytes:].view(torch.float32).view(B, heads) for t in self.in_dev]
        self.idx_dev = [torch.empty((B, k), dtype=torch.int32, device=dev) for _ in range(2)]
        self.scores = [torch.empty((B, (L + 3) // 4 * 4), dtype=torch.float32, device=dev) for _ in range(streams)]
        self.ws = [api.li_decode_select_workspace(B, dev, L) for _ in range(streams)]
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.s_comp = [torch.cuda.Stream(device=dev) for _ in range(streams)] if streams > 1 else []
        self._select(0, torch.cuda.current_stream(dev))  # warm-up: module, kernel attributes, argument checks
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._capture(torch.cuda.current_stream(dev))

    def _select(self, i, stream):
        j, c = i % 2, i % self.nstreams
        k8, ks = self.caches[i]
        api.li_decode_select(self.q_dev[j], self.w_dev[j], k8, ks, self.k, lens=self.lens, scores=self.scores[c],
                             workspace=self.ws[c], idx=self.idx_dev[j], stream=stream)

    def _capture(self, main):
        fork = torch.cuda.Event()
        fork.record(main)
        self.s_in.wait_event(fork)
        self.s_out.wait_event(fork)
        for s in self.s_comp:
            s.wait_event(fork)
        done_sel, done_out = [], []
        for i in range(self.steps):
            j = i % 2
            comp = self.s_comp[i % self.nstreams] if self.s_comp else main
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(done_sel[i - 2])  # slot j's inputs were read by step i - 2
                self.in_dev[j].copy_(self.in_host[i], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(self.s_in)
            comp.wait_event(arrived)
            if i >= 2:
                comp.wait_event(done_out[i - 2])  # slot j's result of step i - 2 has been copied out
            # step i - streams, on the same compute stream, used this stream's scores and workspace
            self._select(i, comp)
            ev = torch.cuda.Event()
            ev.record(comp)
            done_sel.append(ev)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(ev)
                self.idx_host[i].copy_(self.idx_dev[j], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(self.s_out)
                done_out.append(ev_o)
        main.wait_event(done_out[-1])
        for s in [self.s_in] + self.s_comp:
            joined = torch.cuda.Event()
            joined.record(s)
            main.wait_event(joined)

    def run(self, sync: bool = True):
        """Replay the ``steps`` steps; returns the pinned host results (valid once the stream has
        been synchronised: ``sync=True`` waits)."""
        self.graph.replay()
        if sync:
            torch.cuda.current_stream().synchronize()
        return self.idx_host

    @property
    def h2d_bytes_per_step(self) -> int:
        return self.nbytes

    @property
    def d2h_bytes_per_step(self) -> int:
        return self.B * self.k * 4
