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
        self.ws = api.li_decode_select_workspace(B, dev)
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
