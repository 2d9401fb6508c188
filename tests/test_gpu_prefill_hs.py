"""GPU parity for the causal prefill scorer and hierarchical selection."""
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


def _oracle_prefill(case, rows=None, causal_offset=0):
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    return oracle.index_score(q8, oracle.E4M3, case.w, case.k8, oracle.E4M3, q_scale=sq, k_scale=case.ks,
                              causal=True, causal_offset=causal_offset, rows=rows, with_mag=True)


# ---------------------------------------------------------------------------
# causal prefill
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,L,off", [(1003, 1003, 0), (500, 537, 37), (3, 300, 150), (130, 130, 0)])
def test_prefill_scores_all_rows(T, L, off):
    case = synth.dsa_prefill(T=T, L=L, seed=50 + T)
    ref, mag = _oracle_prefill(case, causal_offset=off)
    sc = api.li_index_score(case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV), causal=True,
                            causal_offset=off)
    got = _np(sc)[:, :L]
    vis = np.isfinite(ref)
    assert_scores_close(np.where(vis, got, 0.0), ref, mag, 1e-2, visible=vis)
    k = 64
    idx = api.li_topk(sc, k, causal=True, causal_offset=off, max_len=L)
    ridx, _ = oracle.topk(ref, k, causal=True, causal_offset=off, max_len=L)
    assert_topk_equivalent(_np(idx), ridx, ref, 1e-2)
    assert api.li_get_last_error() == LI_OK


def test_prefill_full_size_sampled_rows():
    """The causal prefill configuration at full size (T = L = 8192, k = 2048): all
    scores and selections of a row sample, boundary rows included."""
    case = synth.dsa_prefill()
    T = L = 8192
    rows = sorted(set([0, 1, 127, 128, 2046, 2047, 2048, 4095, 4096, 8190, 8191] +
                      np.random.default_rng(0).integers(0, T, 24).tolist()))
    ref, mag = _oracle_prefill(case, rows=rows)
    sc = api.li_index_score(case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV), causal=True)
    idx = api.li_topk(sc, 2048, causal=True, max_len=L)
    got = _np(sc)[rows, :L]
    vis = np.isfinite(ref)
    assert_scores_close(np.where(vis, got, 0.0), ref, mag, 1e-2, visible=vis)
    ridx = np.stack([oracle.topk(ref[i:i + 1], 2048, lens=[r + 1])[0][0] for i, r in enumerate(rows)])
    assert_topk_equivalent(_np(idx)[rows], ridx, ref, 1e-2)
    # rows with a prefix shorter than k select their whole prefix
    assert np.array_equal(_np(idx)[100, :101], np.arange(101)) and np.all(_np(idx)[100, 101:] == -1)
    assert api.li_get_last_error() == LI_OK


# ---------------------------------------------------------------------------
# hierarchical selection
# ---------------------------------------------------------------------------
def _gpu_anchor_and_followers(case, n_cand, c):
    F = case.q.shape[0] - 1
    qts = [api.li_absorb_query(case.q[l].to(DEV), case.w_dec[l].to(DEV)) for l in range(1 + F)]
    L = case.c.shape[1]
    sc = api.li_latent_score(qts[0], case.w[0].to(DEV), c, lens=case.lens.to(DEV))
    cand = api.li_topk(sc, n_cand, lens=case.lens.to(DEV), max_len=L)
    qt_f = torch.stack(qts[1:]).contiguous()
    return qts, sc, cand, qt_f


@pytest.mark.parametrize("B,L,C,k,lens", [(2, 3000, 512, 128, None), (3, 2000, 640, 100, [2000, 500, 77]),
                                          (1, 1000, 130, 130, None)])
def test_hs_refine_matches_oracle(B, L, C, k, lens):
    case = synth.latent_hs(B=B, L=L, n_cand=C, k_top=k, seed=60 + B, lens=lens)
    c = case.c.to(DEV)
    qts, sc, cand, qt_f = _gpu_anchor_and_followers(case, C, c)
    out = api.li_hs_refine(c, cand, qt_f, case.w[1:].contiguous().to(DEV), k)
    ref = oracle.hs_refine(qt_f.cpu(), oracle.BF16, case.w[1:], case.c, _np(cand), k)
    # same candidates and the same bf16 queries: only fp32-vs-fp64 rounding differs
    _, cs = oracle.hs_refine(qt_f.cpu(), oracle.BF16, case.w[1:], case.c, _np(cand), k, with_scores=True)
    g = _np(out)
    for f in range(qt_f.shape[0]):
        for b in range(B):
            cb = _np(cand)[b]
            assert set(g[f, b][g[f, b] >= 0].tolist()) <= set(cb[cb >= 0].tolist())
            # compare in candidate-slot space
            pos = {int(p): i for i, p in enumerate(cb) if p >= 0}
            gi = np.array([[pos[int(p)] for p in g[f, b] if p >= 0] + [-1] * int((g[f, b] < 0).sum())])
            ri = np.array([[pos[int(p)] for p in ref[f, b] if p >= 0] + [-1] * int((ref[f, b] < 0).sum())])
            assert_topk_equivalent(gi, ri, cs[f, b:b + 1], 1e-2)
    assert api.li_get_last_error() == LI_OK


def test_hs_all_positions_equal_full_selection():
    case = synth.latent_hs(B=2, L=1024, n_cand=1024, k_top=200, seed=70)
    c = case.c.to(DEV)
    qts = [api.li_absorb_query(case.q[l].to(DEV), case.w_dec[l].to(DEV)) for l in range(4)]
    cand = torch.arange(1024, dtype=torch.int32, device=DEV).repeat(2, 1).contiguous()
    qt_f = torch.stack(qts[1:]).contiguous()
    out = api.li_hs_refine(c, cand, qt_f, case.w[1:].contiguous().to(DEV), 200)
    for f in range(3):
        sc = api.li_latent_score(qts[1 + f], case.w[1 + f].to(DEV), c)
        full = api.li_topk(sc, 200, max_len=1024)
        assert np.array_equal(_np(out[f]), _np(full))


def test_hs_out_of_range_candidate_reported():
    case = synth.latent_hs(B=1, L=256, n_cand=128, k_top=16, seed=71)
    c = case.c.to(DEV)
    cand = torch.arange(128, dtype=torch.int32).reshape(1, 128)
    cand[0, 5] = 10 ** 6
    qts = [api.li_absorb_query(case.q[l].to(DEV), case.w_dec[l].to(DEV)) for l in range(4)]
    api.li_hs_refine(c, cand.to(DEV), torch.stack(qts[1:]).contiguous(), case.w[1:].contiguous().to(DEV), 16)
    assert api.li_get_last_error() == LI_ERR_BOUNDS
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("C,k", [(8192, 2048), (640, 100)])
def test_hs_histogram_path_equals_plain_passes(C, k):
    # the rescoring kernel counts each follower row's first-digit histogram for the top-k; a
    # workspace whose histograms are dirty must give the same selection (plain passes), be
    # reported, and be left zero
    case = synth.latent_hs(B=2, L=20000, n_cand=C, k_top=k, seed=90)
    c = case.c.to(DEV)
    qts, sc, cand, qt_f = _gpu_anchor_and_followers(case, C, c)
    w = case.w[1:].contiguous().to(DEV)
    F = qt_f.shape[0]
    ws = api.li_hs_refine_workspace(2, C, F, DEV)
    tail = ws[ws.numel() - F * 2 * 2048 * 4:]
    out = api.li_hs_refine(c, cand, qt_f, w, k, workspace=ws)
    torch.cuda.synchronize()
    assert api.li_get_last_error() == LI_OK and int(tail.count_nonzero()) == 0
    tail.view(torch.int32)[::7] = 3
    dirty = api.li_hs_refine(c, cand, qt_f, w, k, workspace=ws)
    torch.cuda.synchronize()
    assert api.li_get_last_error() == LI_ERR_BOUNDS and int(tail.count_nonzero()) == 0
    assert torch.equal(out, dirty)
    again = api.li_hs_refine(c, cand, qt_f, w, k, workspace=ws)
    assert torch.equal(out, again) and api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("B", [1, 16])
def test_hs_full_size(B):
    """The HS configuration at full size (L = 131072, C = 8192, 3 followers, k = 2048)."""
    case = synth.latent_hs(B=B, L=131072, seed=4)
    c = case.c.to(DEV)
    qts, sc, cand, qt_f = _gpu_anchor_and_followers(case, 8192, c)
    # anchor scan and candidate selection against the oracle (same bf16 absorbed query)
    rows = list(range(B)) if B == 1 else [0, 7, 15]
    ref, mag = oracle.latent_score(qts[0].cpu(), oracle.BF16, case.w[0], case.c, rows=rows, with_mag=True)
    assert_scores_close(_np(sc)[rows, :131072], ref, mag, 1e-2)
    ridx, _ = oracle.topk(ref, 8192)
    assert_topk_equivalent(_np(cand)[rows], ridx, ref, 1e-2)
    out = api.li_hs_refine(c, cand, qt_f, case.w[1:].contiguous().to(DEV), 2048)
    cd = _np(cand)[rows]
    ro, cs = oracle.hs_refine(qt_f[:, rows].cpu(), oracle.BF16, case.w[1:, rows], case.c[rows], cd, 2048,
                              with_scores=True)
    g = _np(out)[:, rows]
    for f in range(3):
        for i in range(len(rows)):
            pos = {int(p): j for j, p in enumerate(cd[i])}
            gi = np.array([[pos[int(p)] for p in g[f, i]]])
            ri = np.array([[pos[int(p)] for p in ro[f, i]]])
            assert_topk_equivalent(gi, ri, cs[f, i:i + 1], 1e-2)
    assert api.li_get_last_error() == LI_OK


# ---------------------------------------------------------------------------
# one-launch absorption of a layer group; latent scan with the first-digit histogram
# ---------------------------------------------------------------------------
def test_absorb_layers_matches_per_layer_calls():
    case = synth.latent_hs(B=5, L=64, seed=81)
    q = case.q.to(DEV).contiguous()          # [4, B, H, d]
    wd = case.w_dec.to(DEV).contiguous()     # [4, H, d, dc]
    got = api.li_absorb_query_layers(q, wd)
    for l in range(4):
        one = api.li_absorb_query(q[l], wd[l])
        assert torch.equal(got[l].view(torch.int16), one.view(torch.int16)), l
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("B,L,k,lens", [(1, 131072, 8192, None), (16, 32768, 8192, None),
                                        (3, 20000, 2048, [20000, 2048, 0]), (2, 5000, 100, [4999, 1])])
def test_latent_score_hist_then_topk_hist(B, L, k, lens):
    """The anchor's scan with the histogram, then li_topk_hist: bit for bit what li_latent_score
    followed by li_topk gives, and the histogram left zero."""
    case = synth.latent_hs(B=B, L=L, seed=82 + B, lens=lens)
    c = case.c.to(DEV)
    qt = api.li_absorb_query(case.q[0].to(DEV), case.w_dec[0].to(DEV))
    w = case.w[0].to(DEV)
    ln = case.lens.to(DEV)
    hist = api.li_decode_select_workspace(B, DEV).view(torch.int32)[:B * 2048]
    sc = api.li_latent_score_hist(qt, w, c, hist, lens=ln)
    idx, vals = api.li_topk_hist(sc, k, hist, lens=ln, max_len=L, with_values=True)
    sc_r = api.li_latent_score(qt, w, c, lens=ln)
    idx_r, vals_r = api.li_topk(sc_r, k, lens=ln, max_len=L, with_values=True)
    for b, n in enumerate(case.lens.tolist()):
        assert np.array_equal(_np(sc[b, :n]).view(np.uint32), _np(sc_r[b, :n]).view(np.uint32)), b
    assert np.array_equal(_np(idx), _np(idx_r))
    assert np.array_equal(_np(vals).view(np.uint32), _np(vals_r).view(np.uint32))
    assert api.li_get_last_error() == LI_OK
    assert int(hist.count_nonzero()) == 0
