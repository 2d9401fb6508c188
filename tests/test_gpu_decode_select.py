"""GPU parity of the one-call decode step (li_decode_select).

The call must return exactly what li_index_score followed by li_topk returns
on the same inputs: scores bit for bit, selections and their values bit for
bit.  Those two calls are pinned to the oracle elsewhere; one case here also
goes to the oracle directly.  The histogram workspace must be all zero again
after every call, and a workspace that was not zero must still give the exact
result and raise LI_ERR_BOUNDS.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_lightning_score_b200 import api, synth
from sparse_attention_lightning_score_b200._lib import LI_ERR_BOUNDS, LI_OK
from tests._checks import assert_scores_close, assert_topk_equivalent

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().cpu().numpy()


def _dev(case):
    return case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV), case.lens.to(DEV)


def _two_calls(q, w, k8, ks, lens, k_top):
    L = k8.shape[-2]
    sc = api.li_index_score(q, w, k8, ks, lens=lens)
    idx, vals = api.li_topk(sc, k_top, lens=lens, max_len=L, with_values=True)
    return sc, idx, vals


def _hist_zero(ws, rows):
    return int(ws[:api.li_decode_select_hist_bytes(rows)].count_nonzero()) == 0


def _assert_same(got, want, lens):
    sc, idx, vals = got
    sc_r, idx_r, vals_r = want
    for b, n in enumerate(_np(lens).tolist()):
        assert np.array_equal(_np(sc[b, :n]).view(np.uint32), _np(sc_r[b, :n]).view(np.uint32)), b
    assert np.array_equal(_np(idx), _np(idx_r))
    assert np.array_equal(_np(vals).view(np.uint32), _np(vals_r).view(np.uint32))


@pytest.mark.parametrize("B,L,lens,k_top", [
    (3, 1000, [1000, 517, 129], 64),
    (5, 300, [0, 1, 127, 128, 300], 100),       # empty, single and ragged rows
    (4, 5000, [5000, 2048, 2049, 0], 2048),     # rows at and just above k
    (8, 32768, None, 2048),                     # the benchmarked decode step
    (2, 131072, None, 2048),
    (1, 262144, None, 2048),                    # longest row: more candidates than a CTA keeps
    (3, 20000, None, 1),
])
def test_decode_select_matches_score_then_topk(B, L, lens, k_top):
    case = synth.dsa_decode(B=B, L=L, seed=40 + B, lens=lens)
    q, w, k8, ks, ln = _dev(case)
    ws = api.li_decode_select_workspace(B, DEV, L)
    got = api.li_decode_select(q, w, k8, ks, k_top, lens=ln, workspace=ws, with_values=True)
    _assert_same(got, _two_calls(q, w, k8, ks, ln, k_top), ln)
    assert api.li_get_last_error() == LI_OK
    assert _hist_zero(ws, B)


def test_decode_select_halves_equal_the_call():
    case = synth.dsa_decode(B=4, L=20000, seed=31, lens=[20000, 15000, 2049, 300])
    q, w, k8, ks, ln = _dev(case)
    ws = api.li_decode_select_workspace(4, DEV, 20000)
    sc = api.li_decode_select_score(q, w, k8, ks, ws, lens=ln)
    idx, vals = api.li_decode_select_finish(sc, 2048, ws, max_len=20000, lens=ln, with_values=True)
    _assert_same((sc, idx, vals), _two_calls(q, w, k8, ks, ln, 2048), ln)
    assert api.li_get_last_error() == LI_OK
    assert _hist_zero(ws, 4)


def test_decode_select_many_long_rows():
    # 300 rows of 70,000 positions over one shared cache: more rows than SMs, one scorer CTA and one
    # top-k CTA per row, slices far above the cluster top-k's 4K
    case = synth.dsa_decode(B=1, L=70000, seed=33)
    g = torch.Generator().manual_seed(33)
    q = torch.randn(300, 64, 128, generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn(300, 64, generator=g) * 0.1).to(DEV)
    k8, ks = case.k8[0].to(DEV), case.ks[0].to(DEV)
    lens = torch.randint(60000, 70001, (300,), generator=g, dtype=torch.int32).to(DEV)
    got = api.li_decode_select(q, w, k8, ks, 2048, lens=lens, with_values=True)
    _assert_same(got, _two_calls(q, w, k8, ks, lens, 2048), lens)
    assert api.li_get_last_error() == LI_OK


def test_decode_select_against_oracle():
    case = synth.dsa_decode(B=4, L=3000, seed=23, lens=[3000, 2500, 100, 2049])
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    L = 3000
    ref, mag = oracle.index_score(q8, oracle.E4M3, case.w, case.k8, oracle.E4M3, q_scale=sq, k_scale=case.ks,
                                  k_batch_rows=L, L=L, lens=case.lens.numpy(), with_mag=True)
    q, w, k8, ks, ln = _dev(case)
    sc, idx = api.li_decode_select(q, w, k8, ks, 512, lens=ln)
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-2)
    ridx, _ = oracle.topk(ref, 512, lens=case.lens.numpy())
    assert_topk_equivalent(_np(idx), ridx, ref, 1e-2, n_valid=case.lens.numpy())
    assert api.li_get_last_error() == LI_OK


def test_decode_select_workspace_reused_across_steps():
    ws = api.li_decode_select_workspace(4, DEV, 9000)
    for seed in (1, 2, 3):
        case = synth.dsa_decode(B=4, L=9000, seed=seed, lens=[9000, 7000, 3000, 2100])
        q, w, k8, ks, ln = _dev(case)
        got = api.li_decode_select(q, w, k8, ks, 2048, lens=ln, workspace=ws, with_values=True)
        _assert_same(got, _two_calls(q, w, k8, ks, ln, 2048), ln)
    assert api.li_get_last_error() == LI_OK
    assert _hist_zero(ws, 4)


def test_decode_select_shared_cache_and_many_rows():
    # 160 rows (more rows than SMs: one CTA per row) over one shared cache
    case = synth.dsa_decode(B=1, L=6000, seed=9)
    g = torch.Generator().manual_seed(9)
    q = torch.randn(160, 64, 128, generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn(160, 64, generator=g) * 0.1).to(DEV)
    k8, ks = case.k8[0].to(DEV), case.ks[0].to(DEV)
    lens = torch.randint(0, 6001, (160,), generator=g, dtype=torch.int32).to(DEV)
    got = api.li_decode_select(q, w, k8, ks, 1024, lens=lens, with_values=True)
    _assert_same(got, _two_calls(q, w, k8, ks, lens, 1024), lens)
    assert api.li_get_last_error() == LI_OK


def test_decode_select_all_scores_equal():
    # zero weights: every score is 0, one bin holds the whole row, ties go to the lowest positions
    case = synth.dsa_decode(B=2, L=40000, seed=5)
    q, _, k8, ks, ln = _dev(case)
    w = torch.zeros(2, 64, device=DEV)
    ws = api.li_decode_select_workspace(2, DEV, 40000)
    sc, idx = api.li_decode_select(q, w, k8, ks, 2048, lens=ln, workspace=ws)
    assert np.array_equal(_np(idx), np.tile(np.arange(2048, dtype=np.int32), (2, 1)))
    assert api.li_get_last_error() == LI_OK
    assert _hist_zero(ws, 2)


def test_decode_select_dirty_workspace_is_reported_and_healed():
    case = synth.dsa_decode(B=3, L=12000, seed=6)
    q, w, k8, ks, ln = _dev(case)
    ws = api.li_decode_select_workspace(3, DEV, 12000)
    ws.view(torch.int32)[::7] = 3  # counts that describe no row
    got = api.li_decode_select(q, w, k8, ks, 2048, lens=ln, workspace=ws, with_values=True)
    _assert_same(got, _two_calls(q, w, k8, ks, ln, 2048), ln)
    assert api.li_get_last_error() == LI_ERR_BOUNDS
    assert _hist_zero(ws, 3)
    got = api.li_decode_select(q, w, k8, ks, 2048, lens=ln, workspace=ws, with_values=True)
    _assert_same(got, _two_calls(q, w, k8, ks, ln, 2048), ln)
    assert api.li_get_last_error() == LI_OK


# ---------------------------------------------------------------------------
# multi-token decode: T query tokens per request share the request's cache
# ---------------------------------------------------------------------------
def _mtp_case(B, T, L, lens, seed):
    case = synth.dsa_decode(B=B, L=L, seed=seed, lens=lens)
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B * T, 64, 128, generator=g).to(torch.bfloat16)
    w = torch.randn(B * T, 64, generator=g) * 0.1
    return case, q, w


@pytest.mark.parametrize("B,T,L,lens", [(4, 2, 5000, [5000, 3000, 2, 1]), (2, 4, 32768, None),
                                        (3, 3, 2100, [2100, 2049, 2050])])
def test_multi_token_decode_matches_per_token_calls(B, T, L, lens):
    case, q, w = _mtp_case(B, T, L, lens, seed=60 + T)
    k8, ks, ln = case.k8.to(DEV), case.ks.to(DEV), case.lens.to(DEV)
    qd, wd = q.to(DEV), w.to(DEV)
    sc, idx, vals = api.li_decode_select(qd, wd, k8, ks, 2048, lens=ln, tokens_per_request=T, with_values=True)
    sc2 = api.li_index_score(qd, wd, k8, ks, lens=ln, tokens_per_request=T)
    for t in range(T):
        rows = [b * T + t for b in range(B)]
        lt = torch.clamp(case.lens - (T - 1 - t), min=0).to(DEV)
        sc_t, idx_t, vals_t = api.li_decode_select(qd[rows].contiguous(), wd[rows].contiguous(), k8, ks, 2048,
                                                   lens=lt, with_values=True)
        for i, b in enumerate(rows):
            n = int(lt[i])
            assert np.array_equal(_np(sc[b, :n]).view(np.uint32), _np(sc_t[i, :n]).view(np.uint32)), (t, b)
            assert np.array_equal(_np(sc2[b, :n]).view(np.uint32), _np(sc_t[i, :n]).view(np.uint32)), (t, b)
        assert np.array_equal(_np(idx[rows]), _np(idx_t)), t
        assert np.array_equal(_np(vals[rows]).view(np.uint32), _np(vals_t).view(np.uint32)), t
    assert api.li_get_last_error() == LI_OK


def test_multi_token_decode_against_oracle():
    B, T, L = 2, 3, 4000
    case, q, w = _mtp_case(B, T, L, [4000, 2500], seed=66)
    sc, idx = api.li_decode_select(q.to(DEV), w.to(DEV), case.k8.to(DEV), case.ks.to(DEV), 512,
                                   lens=case.lens.to(DEV), tokens_per_request=T)
    q8, sq, _ = oracle.quantize_query(q, w.numpy())
    for t in range(T):
        rows = [b * T + t for b in range(B)]
        lt = np.maximum(case.lens.numpy() - (T - 1 - t), 0)
        ref, mag = oracle.index_score(q8[rows], oracle.E4M3, w[rows], case.k8, oracle.E4M3, q_scale=sq[rows],
                                      k_scale=case.ks, k_batch_rows=L, L=L, lens=lt, with_mag=True)
        assert_scores_close(_np(sc)[rows, :L], ref, mag, 1e-2, visible=np.isfinite(ref))
        ridx, _ = oracle.topk(ref, 512, lens=lt)
        assert_topk_equivalent(_np(idx)[rows], ridx, ref, 1e-2, n_valid=lt)
    assert api.li_get_last_error() == LI_OK
