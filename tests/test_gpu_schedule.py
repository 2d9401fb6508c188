"""The two-stream decode step (IndexCache / Multi-layer Indexer schedules) on the GPU.

For every plan, the overlapped step (indexers on a side stream, attention on
the main stream, eager and as a replayed CUDA graph) must give exactly the
attention outputs of a serial reference that scores each indexer layer, then
runs each layer's attention on the selection its plan names.
"""
import pytest
import torch

from sparse_attention_lightning_score_b200 import api
from sparse_attention_lightning_score_b200._lib import LI_OK
from sparse_attention_lightning_score_b200.schedule import DecodeLayerStack, indexcache_plan, mli_plan

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _reference(stack, plan):
    sels = {}
    for layer, p in enumerate(plan):
        if p.runs_indexer:
            _, idx = api.li_decode_select(stack.q[layer], stack.w[layer], stack.k8[layer], stack.ks[layer], stack.k)
            sels[layer] = idx
    out = torch.empty_like(stack.out)
    for layer, p in enumerate(plan):
        api.li_sparse_attention(stack.qa[layer], stack.kv[layer], sels[p.attends], stack.scale, out=out[layer])
    torch.cuda.synchronize()
    return out


@pytest.fixture(scope="module")
def stack():
    return DecodeLayerStack(n_layers=6, B=2, L=5000, k=512, device=DEV, seed=3)


@pytest.mark.parametrize("plan", [mli_plan(6, lag=0), mli_plan(6, lag=1), mli_plan(6, lag=2),
                                  indexcache_plan(6, retention=0.5), mli_plan(6, lag=1, retention=0.5),
                                  mli_plan(6, lag=1, retention=0.34, independent=(0, 1))],
                         ids=["dsa", "mli1", "mli2", "ic_half", "ic_half_mli1", "glm5_like"])
def test_overlapped_step_matches_serial_reference(stack, plan):
    ref = _reference(stack, plan)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    for overlap in (True, False):
        step = stack.bind(plan, overlap=overlap)
        stack.out.zero_()
        step.run(main, side)
        torch.cuda.synchronize()
        assert torch.equal(stack.out, ref), overlap
    # the same step captured once and replayed
    step = stack.bind(plan, overlap=True)
    step.run(main, side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step.run(torch.cuda.current_stream(), side)
    stack.out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(stack.out, ref)
    assert api.li_get_last_error() == LI_OK


def test_step_with_dense_block(stack):
    dense = DecodeLayerStack(n_layers=4, B=2, L=3000, k=256, dense=(1024, 2048), device=DEV, seed=4)
    plan = mli_plan(4, lag=1)
    ref = _reference(dense, plan)
    step = dense.bind(plan)
    step.run(torch.cuda.current_stream(), torch.cuda.Stream())
    torch.cuda.synchronize()
    assert torch.equal(dense.out, ref)
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("plan", [mli_plan(6, lag=1), mli_plan(6, lag=2, retention=0.5)], ids=["mli1", "ic_half_mli2"])
def test_priority_graph_matches_serial_reference(stack, plan):
    # high-priority main stream, low-priority side stream, graph instantiated with node priorities
    from sparse_attention_lightning_score_b200.schedule import StepGraph, priority_streams
    ref = _reference(stack, plan)
    main, side = priority_streams()
    step = stack.bind(plan, overlap=True)
    with torch.cuda.stream(main):
        step.run(main, side)
    torch.cuda.synchronize()
    g = StepGraph(step, main, side)
    stack.out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    g.close()
    assert torch.equal(stack.out, ref)
    assert api.li_get_last_error() == LI_OK
