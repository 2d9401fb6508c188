"""GPU parity of the consumer: sparse attention over the indexer's selection
(li_sparse_attention) against the fp64 oracle.

Tolerance: |o - o_ref| <= 1e-2 * sum_i p_i |v_i| + 1e-6.  The kernel takes
q . k in fp32 from bf16 operands (exact products), rounds the softmax weights
to bf16 for the value product (relative 2^-9 each) and sums in fp32, so its
error is a few 1e-3 of that scale; 1e-2 is the bf16 tolerance used for the
other bf16 paths.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_lightning_score_b200 import api
from sparse_attention_lightning_score_b200._lib import LI_ERR_BOUNDS, LI_OK

pytestmark = pytest.mark.gpu
DEV = "cuda"
RTOL = 1e-2


def _np(t):
    return t.detach().cpu().numpy()


def _case(B, H, L, k, seed, shared=False, pad_rows=()):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, 576, generator=g).to(torch.bfloat16)
    kv = torch.randn(L if shared else B * L, 576, generator=g).to(torch.bfloat16)
    if not shared:
        kv = kv.view(B, L, 576)
    rng = np.random.default_rng(seed)
    sel = np.stack([np.sort(rng.choice(L, min(k, L), replace=False)) for _ in range(B)]).astype(np.int32)
    if sel.shape[1] < k:
        sel = np.concatenate([sel, np.full((B, k - sel.shape[1]), -1, np.int32)], axis=1)
    for b, n in pad_rows:  # the last n selections of request b are top-k pads
        if n:
            sel[b, -n:] = -1
    return q, kv, sel


def _check(q, kv, sel, scale, out):
    ref, mag = oracle.sparse_attention(q, kv, sel, scale, with_mag=True)
    got = _np(out)
    err = np.abs(got - ref)
    bound = RTOL * mag + 1e-6
    assert np.all(err <= bound), (float((err / (mag + 1e-30)).max()), np.argwhere(err > bound)[:5])


@pytest.mark.parametrize("B,H,L,k,shared,pads", [
    (2, 128, 5000, 2048, False, ()),                 # the decode shape: 2048 selections, 128 heads
    (3, 64, 3000, 300, False, ((1, 45),)),          # ragged last split, pads in one request
    (2, 128, 700, 129, True, ()),                    # one shared cache, one position in the last split
    (1, 64, 100, 128, False, ((0, 128),)),           # nothing selected: o = 0
])
def test_sparse_attention_against_oracle(B, H, L, k, shared, pads):
    q, kv, sel = _case(B, H, L, k, seed=B * 10 + k, shared=shared, pad_rows=pads)
    scale = 1.0 / math.sqrt(576)
    out = api.li_sparse_attention(q.to(DEV), kv.to(DEV), torch.from_numpy(sel).to(DEV), scale)
    _check(q, kv, sel, scale, out)
    assert api.li_get_last_error() == LI_OK
    if pads and pads[0][1] == k:
        assert np.all(_np(out) == 0.0)


def test_sparse_attention_sharp_softmax():
    # large logits: the per-split maxima and the merge's rescaling carry the result
    q, kv, sel = _case(2, 64, 4000, 1000, seed=5)
    out = api.li_sparse_attention(q.to(DEV), kv.to(DEV), torch.from_numpy(sel).to(DEV), 0.5)
    _check(q, kv, sel, 0.5, out)


def test_sparse_attention_full_size():
    # B = 8 requests of 32768 cached rows, 128 heads, the indexer's 2048 selections
    q, kv, sel = _case(8, 128, 32768, 2048, seed=8)
    scale = 1.0 / math.sqrt(192)
    out = api.li_sparse_attention(q.to(DEV), kv.to(DEV), torch.from_numpy(sel).to(DEV), scale)
    _check(q, kv, sel, scale, out)
    assert api.li_get_last_error() == LI_OK


def test_sparse_attention_out_of_range_selection_reported():
    q, kv, sel = _case(2, 64, 500, 256, seed=9)
    bad = sel.copy()
    bad[1, 3] = 500          # one past the cache
    out = api.li_sparse_attention(q.to(DEV), kv.to(DEV), torch.from_numpy(bad).to(DEV), 0.1)
    assert api.li_get_last_error() == LI_ERR_BOUNDS
    bad[1, 3] = -1           # the oracle's reading: skipped
    _check(q, kv, bad, 0.1, out)
    assert api.li_get_last_error() == LI_OK


def test_sparse_attention_order_of_selection_irrelevant():
    q, kv, sel = _case(2, 128, 3000, 640, seed=11)
    qd, kvd = q.to(DEV), kv.to(DEV)
    a = api.li_sparse_attention(qd, kvd, torch.from_numpy(sel).to(DEV), 0.05)
    rev = np.ascontiguousarray(sel[:, ::-1])
    b = api.li_sparse_attention(qd, kvd, torch.from_numpy(rev).to(DEV), 0.05)
    # a different order puts other positions in each split: the bf16 rounding of the weights is taken
    # against another split maximum, so the two results differ at that level; both meet the oracle
    _check(q, kv, sel, 0.05, a)
    _check(q, kv, rev, 0.05, b)
