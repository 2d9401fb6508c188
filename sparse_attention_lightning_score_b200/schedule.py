"""Which selection each layer attends, and the two-stream decode step that follows from it.

Two schedules from the pages, both host-side (no kernel of their own):

- IndexCache (IndexCache explainer, "Full and Shared layers"): F layers run
  their indexer and write the selection into a buffer; each S layer skips its
  indexer and attends the buffer as the latest F layer left it.  Layer 0 is
  always F.
- Multi-layer Indexer (long-version transcript): a layer with an indexer
  attends the selection of the indexer layer `lag` indexer layers back instead
  of its own, so its own scan runs on a second stream beside attention and is
  joined only where a later layer first needs it.  The first indexer layer has
  nothing to borrow and stays serial.  Stacked on IndexCache, the layers
  without an indexer copy what their nearest indexer layer attends.  The last
  `lag` indexer layers feed no later layer within the step, so they do not run.

A plan is a list of LayerPlan; lag 0 with every layer retained is plain DSA.  The step runs on a
high-priority main stream and a low-priority side stream (`priority_streams`), captured into a graph
that keeps those priorities (`StepGraph`): with equal priorities the side stream's indexer blocks take
SMs from the main stream's critical path, and overlap then costs more than it saves.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Sequence


@dataclass(frozen=True)
class LayerPlan:
    runs_indexer: bool   # this layer scores its cache and writes a selection
    attends: int         # the layer whose selection this layer's attention reads


def _retained_layers(n_layers: int, retention: float = 1.0, retained: Optional[Sequence[int]] = None,
                     independent: Sequence[int] = (0,)) -> List[int]:
    if n_layers <= 0:
        raise ValueError("n_layers must be positive")
    if retained is None:
        if not (0.0 < retention <= 1.0):
            raise ValueError("retention must lie in (0, 1]")
        stride = 1.0 / retention
        retained = sorted({min(n_layers - 1, int(round(i * stride))) for i in range(max(1, round(n_layers * retention)))})
    keep = sorted(set(int(x) for x in retained) | set(int(x) for x in independent) | {0})
    if keep[0] < 0 or keep[-1] >= n_layers:
        raise ValueError("retained layer out of range")
    return keep


def indexcache_plan(n_layers: int, retention: float = 1.0, retained: Optional[Sequence[int]] = None,
                    independent: Sequence[int] = (0,)) -> List[LayerPlan]:
    """F layers (layer 0, the `independent` ones and the retained set) attend their own fresh
    selection; every other layer attends the latest F layer's."""
    return mli_plan(n_layers, lag=0, retention=retention, retained=retained, independent=independent)


def mli_plan(n_layers: int, lag: int = 1, retention: float = 1.0, retained: Optional[Sequence[int]] = None,
             independent: Sequence[int] = (0,)) -> List[LayerPlan]:
    """Indexer layers R[0] < R[1] < ... (layer 0, the `independent` layers and the retained set).
    Layers from R[i] up to R[i+1]-1 attend the selection of R[max(i - lag, 0)], except that an
    independent layer attends its own (serial).  lag = 0 is IndexCache (or DSA with every layer kept)."""
    if lag < 0:
        raise ValueError("lag must be >= 0")
    keep = _retained_layers(n_layers, retention, retained, independent)
    indep = set(int(x) for x in independent) | {0}
    attends = []
    i = -1
    for layer in range(n_layers):
        if i + 1 < len(keep) and keep[i + 1] == layer:
            i += 1
        own = keep[i]
        # a layer between indexer layers copies what its indexer layer attends
        attends.append(own if own in indep else keep[max(i - lag, 0)])
    # an indexer whose selection no layer attends (the last `lag` ones) is not run
    used = set(attends)
    return [LayerPlan(runs_indexer=(layer in used), attends=attends[layer]) for layer in range(n_layers)]


def check_plan(plan: Sequence[LayerPlan]) -> None:
    """Every attended selection comes from a layer that runs its indexer, at or before the
    attending layer; layer 0 runs its own."""
    if not plan or not plan[0].runs_indexer or plan[0].attends != 0:
        raise ValueError("layer 0 must run its indexer and attend its own selection")
    for layer, p in enumerate(plan):
        if not (0 <= p.attends <= layer) or not plan[p.attends].runs_indexer:
            raise ValueError(f"layer {layer} attends a selection that does not exist yet")


def selection_buffers(plan: Sequence[LayerPlan]) -> Dict[int, int]:
    """Buffer slot per indexer layer: a slot is reused only once every layer attending its previous
    writer has come earlier in layer order (IndexCache with lag 0 needs one slot; lag d needs d + 1
    when every layer keeps its indexer)."""
    last_use: Dict[int, int] = {}
    for layer, p in enumerate(plan):
        last_use[p.attends] = layer
    slot_of: Dict[int, int] = {}
    free_after: List[int] = []  # per slot: the last layer that reads its current contents
    for layer, p in enumerate(plan):
        if not p.runs_indexer:
            continue
        # the writer at `layer` may reuse a slot whose readers are all before this layer in the main
        # stream order (their attention is enqueued before this layer's indexer is allowed to write)
        for s, until in enumerate(free_after):
            if until < layer:
                slot_of[layer] = s
                free_after[s] = last_use.get(layer, layer)
                break
        else:
            slot_of[layer] = len(free_after)
            free_after.append(last_use.get(layer, layer))
    return slot_of


class TwoStreamStep:
    """One decode step over the layers of a plan, on a main and a side CUDA stream.

    `indexer(layer, out_slot, stream)` launches layer `layer`'s indexer writing selection buffer
    `out_slot`; `attention(layer, in_slot, stream)` launches the layer's attention reading buffer
    `in_slot`; `rest(layer, stream)` (optional) launches the rest of the layer (projection, MLP).
    In the overlapped form an indexer whose selection is attended by a later layer runs on the side
    stream, released by an event at its layer's start (the layer input exists then) and by the last
    reader of the buffer it overwrites; the main stream waits for it where the selection is first
    attended.  An indexer whose own layer attends its selection runs serially on the main stream.
    With overlap=False everything runs on the main stream in layer order.
    """

    def __init__(self, plan: Sequence[LayerPlan], indexer: Callable, attention: Callable,
                 rest: Optional[Callable] = None, overlap: bool = True):
        check_plan(plan)
        self.plan = list(plan)
        self.slots = selection_buffers(self.plan)
        self.n_slots = max(self.slots.values()) + 1
        self.indexer, self.attention, self.rest = indexer, attention, rest
        self.overlap = overlap

    def run(self, main, side):
        """Enqueue the step on `main` (and `side`); both are torch.cuda.Stream objects.  Returns after
        enqueueing; if the side stream was used it is joined back into the main stream at the end."""
        import torch
        plan = self.plan
        first_reader = {}
        for layer, p in enumerate(plan):
            first_reader.setdefault(p.attends, layer)
        done = {}            # indexer layer -> event after its selection is written
        last_read = {}       # slot -> event after the latest attention that read it
        forked = False       # the side stream holds work of this step
        for layer, p in enumerate(plan):
            if p.runs_indexer:
                slot = self.slots[layer]
                serial = (not self.overlap) or first_reader.get(layer, layer) == layer
                if serial:
                    self.indexer(layer, slot, main)
                else:
                    start = torch.cuda.Event()
                    start.record(main)                     # this layer's input exists
                    side.wait_event(start)
                    if slot in last_read:                  # the buffer's previous readers are done
                        side.wait_event(last_read[slot])
                    self.indexer(layer, slot, side)
                    forked = True
                    ev = torch.cuda.Event()
                    ev.record(side)
                    done[layer] = ev
            src = p.attends
            if src in done and first_reader[src] == layer:
                main.wait_event(done.pop(src))             # join where the selection is first needed
            slot = self.slots[src]
            self.attention(layer, slot, main)
            ev = torch.cuda.Event()
            ev.record(main)
            last_read[slot] = ev
            if self.rest is not None:
                self.rest(layer, main)
        for ev in done.values():                           # selections nobody attends this step
            main.wait_event(ev)
        if forked:                                         # (a graph capture needs the side stream joined)
            join = torch.cuda.Event()
            join.record(side)
            main.wait_event(join)


def priority_streams():
    """(main, side): a main stream at the highest priority and a side stream at the lowest, so that
    blocks of the layer's critical path are scheduled before the side stream's indexer blocks."""
    import torch
    return torch.cuda.Stream(priority=-32), torch.cuda.Stream(priority=0)


class StepGraph:
    """One TwoStreamStep captured into a CUDA graph instantiated with node priorities: each kernel
    keeps the priority of the stream it was captured from (the indexers on a low-priority side
    stream fill SMs the main stream leaves idle instead of taking them from it)."""

    def __init__(self, step: TwoStreamStep, main, side, node_priority: bool = True):
        import ctypes
        import torch
        from . import _lib
        self._lib = _lib.load()
        self.main = main
        self.graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(self.graph, stream=main):
            step.run(main, side)
        exec_ = ctypes.c_void_p()
        st = self._lib.li_graph_instantiate(ctypes.c_void_p(self.graph.raw_cuda_graph()), int(node_priority),
                                            ctypes.byref(exec_))
        _lib.check("li_graph_instantiate", st)
        self.exec = exec_

    def replay(self):
        import ctypes
        from . import _lib
        _lib.check("li_graph_launch", self._lib.li_graph_launch(self.exec, ctypes.c_void_p(self.main.cuda_stream)))

    def close(self):
        if self.exec:
            self._lib.li_graph_destroy(self.exec)
            self.exec = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class DecodeLayerStack:
    """A synthetic stack of DSA decode layers to drive TwoStreamStep with the library's kernels.

    Per layer: the indexer's bf16 query [B,H,128], weights [B,H] and FP8 key cache [B,L,128] with
    per-row scales (li_decode_select -> selection [B,k]); the attention's bf16 query [B,Ha,576] and
    latent cache [B,L,576] (li_sparse_attention -> out [B,Ha,512] fp32); optionally a dense block
    standing in for the rest of the layer (x [B,dm] @ W [dm,dn], cuBLAS via torch).  Inputs are seeded
    and synthetic; caches are distinct per layer so that no layer reads another's from L2.
    """

    def __init__(self, n_layers: int, B: int, L: int, k: int = 2048, heads: int = 64, att_heads: int = 128,
                 dense: Optional[tuple] = None, device="cuda", seed: int = 0):
        import torch
        from . import api, synth
        self.api = api
        self.n, self.B, self.L, self.k = n_layers, B, L, k
        case = synth.dsa_decode(B=B, L=L, H=heads, k_top=k, seed=seed)
        g = torch.Generator(device=device).manual_seed(seed)
        self.k8 = [case.k8.to(device)] + [case.k8.to(device).clone() for _ in range(n_layers - 1)]
        self.ks = [case.ks.to(device)] + [case.ks.to(device).clone() for _ in range(n_layers - 1)]
        self.q = [(torch.randn(B, heads, 128, device=device, generator=g)).to(torch.bfloat16) for _ in range(n_layers)]
        self.w = [torch.randn(B, heads, device=device, generator=g) * 0.1 for _ in range(n_layers)]
        self.qa = [torch.randn(B, att_heads, 576, device=device, generator=g).to(torch.bfloat16)
                   for _ in range(n_layers)]
        self.kv = [torch.randn(B, L, 576, device=device, generator=g).to(torch.bfloat16) for _ in range(n_layers)]
        self.out = torch.empty(n_layers, B, att_heads, 512, device=device)
        self.scale = 1.0 / 192 ** 0.5
        self.dense = None
        if dense is not None:
            dm, dn = dense
            self.x = torch.randn(B, dm, device=device, generator=g).to(torch.bfloat16)
            self.W = [torch.randn(dm, dn, device=device, generator=g).to(torch.bfloat16) * dm ** -0.5
                      for _ in range(n_layers)]
            self.y = torch.empty(B, dn, device=device, dtype=torch.bfloat16)
            self.dense = dense
        self.sel = None
        self._ws = {}

    def bind(self, plan: Sequence[LayerPlan], overlap: bool = True, with_rest: bool = True) -> TwoStreamStep:
        """A TwoStreamStep over this stack for `plan` (selection buffers sized for it); the dense block
        runs after each layer's attention when the stack has one and `with_rest` is set."""
        import torch
        step = TwoStreamStep(plan, self._indexer, self._attention,
                             self._rest if (self.dense and with_rest) else None, overlap=overlap)
        self.sel = torch.empty(step.n_slots, self.B, self.k, dtype=torch.int32, device=self.out.device)
        self.scores = torch.empty(step.n_slots, self.B, (self.L + 3) // 4 * 4, dtype=torch.float32,
                                  device=self.out.device)
        self.hist = [self.api.li_decode_select_workspace(self.B, self.out.device, self.L) for _ in range(step.n_slots)]
        self.att_ws = self.api.li_sparse_attention_workspace(self.B, self.qa[0].shape[1], self.k, self.out.device)
        return step

    def _indexer(self, layer, slot, stream):
        self.api.li_decode_select(self.q[layer], self.w[layer], self.k8[layer], self.ks[layer], self.k,
                                  scores=self.scores[slot], workspace=self.hist[slot], idx=self.sel[slot],
                                  stream=stream)

    def _attention(self, layer, slot, stream):
        self.api.li_sparse_attention(self.qa[layer], self.kv[layer], self.sel[slot], self.scale,
                                     out=self.out[layer], workspace=self.att_ws, stream=stream)

    def _rest(self, layer, stream):
        import torch
        with torch.cuda.stream(stream):
            torch.matmul(self.x, self.W[layer], out=self.y)
