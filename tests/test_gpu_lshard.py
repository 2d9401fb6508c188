"""GPU parity of the L-sharded decode step, emulated on one GPU: the cache of
every request is cut into P slices, each slice selects its own top-k with
li_decode_select (as each rank would), the P selections are stacked in shard
order (as the all-gather delivers them) and li_merge_shards merges them.  The
result must equal, bit for bit, li_decode_select over the whole cache: the same
global positions and the same scores.  No rank waits on another here: the
shards run one after another on the same GPU.
"""
import numpy as np
import pytest
import torch

from sparse_attention_lightning_score_b200 import api, synth
from sparse_attention_lightning_score_b200._lib import LI_ERR_BOUNDS, LI_OK
from sparse_attention_lightning_score_b200.dist import shard_lens

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("B,L,P,k,lens", [
    (4, 32768, 4, 2048, [32768, 20000, 9000, 2100]),   # full, partial and empty shards
    (2, 12000, 2, 2048, [12000, 7000]),                # a last-reached shard holding fewer than k
    (3, 40000, 8, 512, None),
    (2, 6000, 3, 100, [6000, 1]),
])
def test_lshard_merge_equals_full_selection(B, L, P, k, lens):
    case = synth.dsa_decode(B=B, L=L, seed=70 + P, lens=lens)
    q, w = case.q.to(DEV), case.w.to(DEV)
    k8, ks, ln = case.k8.to(DEV), case.ks.to(DEV), case.lens.to(DEV)
    _, full_idx, full_vals = api.li_decode_select(q, w, k8, ks, k, lens=ln, with_values=True)
    sl = -(-L // P)
    vals, idx = [], []
    for p in range(P):
        lo, hi = p * sl, min((p + 1) * sl, L)
        k8p = torch.zeros(B, sl, 128, dtype=torch.uint8, device=DEV)
        ksp = torch.ones(B, sl, device=DEV)
        if hi > lo:
            k8p[:, :hi - lo] = k8[:, lo:hi]
            ksp[:, :hi - lo] = ks[:, lo:hi]
        _, ip, vp = api.li_decode_select(q, w, k8p, ksp, k, lens=shard_lens(ln, p, sl), with_values=True)
        vals.append(vp)
        idx.append(ip)
    out_idx, out_vals = api.li_merge_shards(torch.stack(vals), torch.stack(idx), sl, k, with_values=True)
    assert np.array_equal(_np(out_idx), _np(full_idx))
    assert np.array_equal(_np(out_vals).view(np.uint32), _np(full_vals).view(np.uint32))
    assert api.li_get_last_error() == LI_OK


def test_lshard_merge_reports_a_list_with_a_gap():
    # shard 0 claims fewer than k positions but shard 1 has some: not a split of one context
    vals = torch.tensor([[[3.0, 1.0, -float("inf")]], [[2.0, 0.5, -float("inf")]]], device=DEV)
    idx = torch.tensor([[[0, 1, -1]], [[0, 2, -1]]], dtype=torch.int32, device=DEV)
    out = api.li_merge_shards(vals, idx, 100, 3)
    assert api.li_get_last_error() == LI_ERR_BOUNDS
    assert _np(out).tolist() == [[0, 1, -1]]  # only the valid prefix is merged
    assert api.li_get_last_error() == LI_OK


def test_lshard_merge_dirty_workspace_gives_the_same_selection():
    # the merge counts the candidates' first digits into the workspace's histograms for the row
    # top-k; histograms that are not zero give the same result through the plain passes, are
    # reported, and are left zero
    case = synth.dsa_decode(B=2, L=16000, seed=81)
    q, w, k8, ks = case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV)
    P, k, sl = 4, 1024, 4000
    vals, idx = [], []
    for p in range(P):
        _, ip, vp = api.li_decode_select(q, w, k8[:, p * sl:(p + 1) * sl].contiguous(),
                                         ks[:, p * sl:(p + 1) * sl].contiguous(), k, with_values=True)
        vals.append(vp)
        idx.append(ip)
    vals, idx = torch.stack(vals), torch.stack(idx)
    from sparse_attention_lightning_score_b200 import _lib
    ws = torch.zeros(_lib.load().li_merge_shards_workspace(P, 2, k), dtype=torch.uint8, device=DEV)
    tail = ws[ws.numel() - 2 * 2048 * 4:]
    clean = api.li_merge_shards(vals, idx, sl, k, workspace=ws)
    torch.cuda.synchronize()
    assert api.li_get_last_error() == LI_OK and int(tail.count_nonzero()) == 0
    tail.view(torch.int32)[::3] = 2
    dirty = api.li_merge_shards(vals, idx, sl, k, workspace=ws)
    torch.cuda.synchronize()
    assert api.li_get_last_error() == LI_ERR_BOUNDS and int(tail.count_nonzero()) == 0
    assert torch.equal(clean, dirty)
    _, full = api.li_decode_select(q, w, k8, ks, k)
    assert torch.equal(clean, full)
