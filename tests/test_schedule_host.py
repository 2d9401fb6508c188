"""Host logic of the IndexCache / Multi-layer Indexer schedules (no GPU).

Plans are checked against hand-derived layer maps; the two-stream executor is
run on fake streams and events that record a happens-before graph, and every
attention must follow the indexer that wrote its selection, while every
overwrite of a selection buffer must follow that buffer's last reader.
"""
import itertools

import pytest
import torch

from sparse_attention_lightning_score_b200.schedule import (LayerPlan, TwoStreamStep, check_plan, indexcache_plan,
                                                            mli_plan, selection_buffers)


def _flags(plan):
    return "".join("I" if p.runs_indexer else "." for p in plan), [p.attends for p in plan]


def test_plans_match_hand_derivation():
    # DSA: every layer scores and attends its own selection
    assert _flags(mli_plan(6, lag=0)) == ("IIIIII", [0, 1, 2, 3, 4, 5])
    # MLI, lag 1: layer 0 is serial; layer l attends layer l-1's; the last indexer feeds nobody
    assert _flags(mli_plan(6, lag=1)) == ("IIIII.", [0, 0, 1, 2, 3, 4])
    # lag 2: two indexer layers back, clamped to the first
    assert _flags(mli_plan(6, lag=2)) == ("IIII..", [0, 0, 0, 1, 2, 3])
    # IndexCache, half the layers: S layers copy the latest F layer
    assert _flags(indexcache_plan(8, retention=0.5)) == ("I.I.I.I.", [0, 0, 2, 2, 4, 4, 6, 6])
    # both: F layers attend the previous F layer's selection; S layers copy their F layer
    assert _flags(mli_plan(8, lag=1, retention=0.5)) == ("I.I.I...", [0, 0, 0, 0, 2, 2, 4, 4])
    # GLM-5: layers 0 and 1 are independent (own indexer, own selection)
    assert _flags(mli_plan(8, lag=1, retention=0.25, independent=(0, 1))) == ("II......", [0, 1, 1, 1, 1, 1, 1, 1])


def test_explicit_retained_layers():
    plan = mli_plan(5, lag=1, retained=[0, 2, 3])
    assert _flags(plan) == ("I.I..", [0, 0, 0, 2, 2])
    plan = indexcache_plan(5, retained=[0, 2, 3])
    assert _flags(plan) == ("I.II.", [0, 0, 2, 3, 3])


@pytest.mark.parametrize("n,lag,ret", list(itertools.product([1, 2, 5, 8, 13], [0, 1, 2, 3], [1.0, 0.5, 0.34, 0.25])))
def test_plan_invariants(n, lag, ret):
    plan = mli_plan(n, lag=lag, retention=ret)
    check_plan(plan)
    assert plan[0] == LayerPlan(True, 0)
    for layer, p in enumerate(plan):
        assert p.attends <= layer
        if lag == 0:
            # without lag a layer attends the newest selection at or before it
            assert p.attends == max(q for q in range(layer + 1) if plan[q].runs_indexer)
    slots = selection_buffers(plan)
    assert set(slots) == {l for l, p in enumerate(plan) if p.runs_indexer}
    if lag == 0:
        assert max(slots.values()) == 0          # IndexCache: one buffer
    elif ret == 1.0 and n >= 2 * lag + 1:
        assert max(slots.values()) == lag        # lag d: d + 1 buffers once lag + 1 indexers are in use
    # a slot is never rewritten while a layer that attends its previous contents is still to come
    for w, s in slots.items():
        for w2, s2 in slots.items():
            if s2 == s and w2 > w:
                readers = [l for l, p in enumerate(plan) if p.attends == w]
                assert all(r < w2 for r in readers)


def test_bad_plans_rejected():
    with pytest.raises(ValueError):
        check_plan([LayerPlan(True, 0), LayerPlan(False, 2), LayerPlan(True, 2)])
    with pytest.raises(ValueError):
        check_plan([LayerPlan(False, 0)])
    with pytest.raises(ValueError):
        mli_plan(4, lag=-1)
    with pytest.raises(ValueError):
        mli_plan(4, retention=0.0)


# ---------------------------------------------------------------------------
# the executor on fake streams: happens-before over recorded operations
# ---------------------------------------------------------------------------
class _Graph:
    def __init__(self):
        self.nodes = []          # (kind, detail)
        self.edges = {}          # node -> set of predecessors

    def add(self, stream, kind, detail=None, extra_pred=()):
        i = len(self.nodes)
        self.nodes.append((kind, detail))
        preds = set(extra_pred)
        if stream.last is not None:
            preds.add(stream.last)
        preds |= stream.pending_waits
        stream.pending_waits = set()
        self.edges[i] = preds
        stream.last = i
        return i

    def before(self, a, b):
        """a happens before b."""
        seen, todo = set(), [b]
        while todo:
            x = todo.pop()
            for p in self.edges[x]:
                if p == a:
                    return True
                if p not in seen:
                    seen.add(p)
                    todo.append(p)
        return False


class _Stream:
    def __init__(self, g, name):
        self.g, self.name, self.last, self.pending_waits = g, name, None, set()

    def wait_event(self, ev):
        if ev.node is not None:
            self.pending_waits.add(ev.node)


class _Event:
    graph = None

    def __init__(self, *a, **k):
        self.node = None

    def record(self, stream):
        self.node = stream.g.add(stream, "record")


def _run_fake(plan, overlap):
    g = _Graph()
    main, side = _Stream(g, "main"), _Stream(g, "side")
    ops = []

    def indexer(layer, slot, st):
        ops.append(("idx", layer, slot, g.add(st, "idx", (layer, slot))))

    def attention(layer, slot, st):
        ops.append(("att", layer, slot, g.add(st, "att", (layer, slot))))

    step = TwoStreamStep(plan, indexer, attention, overlap=overlap)
    orig = torch.cuda.Event
    torch.cuda.Event = _Event
    try:
        step.run(main, side)
    finally:
        torch.cuda.Event = orig
    end = g.add(main, "end")
    return g, ops, step, end


@pytest.mark.parametrize("plan", [mli_plan(8, lag=0), mli_plan(8, lag=1), mli_plan(9, lag=2),
                                  indexcache_plan(8, retention=0.5), mli_plan(12, lag=1, retention=0.5),
                                  mli_plan(10, lag=3, retention=0.5), mli_plan(8, lag=1, retention=0.25,
                                                                               independent=(0, 1))])
@pytest.mark.parametrize("overlap", [True, False])
def test_two_stream_step_orders_every_dependency(plan, overlap):
    g, ops, step, end = _run_fake(plan, overlap)
    writes = {(o[1]): o for o in ops if o[0] == "idx"}
    atts = [o for o in ops if o[0] == "att"]
    assert [o[1] for o in atts] == list(range(len(plan)))            # every layer attends once, in order
    assert sorted(writes) == [l for l, p in enumerate(plan) if p.runs_indexer]
    for _, layer, slot, node in atts:
        src = plan[layer].attends
        w = writes[src]
        assert slot == w[2] == step.slots[src]
        assert g.before(w[3], node), (layer, src)                    # the selection exists
        # no later writer of the same slot may land before this reader
        for other, o in writes.items():
            if o[2] == slot and other > src:
                assert g.before(node, o[3]), (layer, other)
    for o in writes.values():
        assert g.before(o[3], end)                                   # the step ends after every indexer
    # an indexer runs after its own layer's input exists: after the previous layer's attention
    for layer, o in writes.items():
        if layer > 0:
            prev_att = atts[layer - 1][3]
            assert g.before(prev_att, o[3])
    if overlap and any(p.attends < l for l, p in enumerate(plan) if p.runs_indexer):
        # something really runs on the side stream, unordered with the main stream's attention
        side_idx = [o for o in writes.values() if not g.before(o[3], atts[o[1]][3]) and o[1] > 0]
        assert side_idx
