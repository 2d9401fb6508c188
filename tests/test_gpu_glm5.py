"""GPU parity for GLM-5's indexer shape: 32 indexer heads instead of DeepSeek-V3.2's 64
(Multi-layer Indexer, Appendix settings table), on the decode scan, the one-call decode step,
multi-token decode, the latent scan (d_c = 256) and hierarchical selection."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_lightning_score_b200 import api, synth
from sparse_attention_lightning_score_b200._lib import LI_OK
from tests._checks import assert_scores_close, assert_topk_equivalent

pytestmark = pytest.mark.gpu
DEV = "cuda"
H = 32


def _np(t):
    return t.detach().cpu().numpy()


def _oracle_decode(case, rows=None):
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    L = case.k8.shape[1]
    return oracle.index_score(q8, oracle.E4M3, case.w, case.k8, oracle.E4M3, q_scale=sq, k_scale=case.ks,
                              k_batch_rows=L, L=L, lens=case.lens.numpy(), rows=rows, with_mag=True)


@pytest.mark.parametrize("B,L,lens,k_top", [(3, 5000, [5000, 2100, 129], 512), (4, 300, [0, 1, 255, 300], 64)])
def test_decode_32_heads_against_oracle(B, L, lens, k_top):
    case = synth.dsa_decode(B=B, L=L, H=H, seed=90 + B, lens=lens)
    ref, mag = _oracle_decode(case)
    q, w, k8, ks, ln = (case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV), case.lens.to(DEV))
    sc = api.li_index_score(q, w, k8, ks, lens=ln)
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-2, visible=np.isfinite(ref))
    sc2, idx, vals = api.li_decode_select(q, w, k8, ks, k_top, lens=ln, with_values=True)
    for b, n in enumerate(case.lens.tolist()):
        assert np.array_equal(_np(sc2[b, :n]).view(np.uint32), _np(sc[b, :n]).view(np.uint32)), b
    idx_r, vals_r = api.li_topk(sc, k_top, lens=ln, max_len=L, with_values=True)
    assert np.array_equal(_np(idx), _np(idx_r))
    assert np.array_equal(_np(vals).view(np.uint32), _np(vals_r).view(np.uint32))
    ridx, _ = oracle.topk(ref, k_top, lens=case.lens.numpy())
    assert_topk_equivalent(_np(idx), ridx, ref, 1e-2, n_valid=case.lens.numpy())
    assert api.li_get_last_error() == LI_OK


def test_decode_32_heads_full_size_sampled_rows():
    # the decode step at B = 8, L = 32768 with GLM-5's head count; rows 0 and 5 against the oracle
    case = synth.dsa_decode(B=8, L=32768, H=H, seed=94)
    q, w, k8, ks = case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV)
    sc, idx = api.li_decode_select(q, w, k8, ks, 2048)
    rows = [0, 5]
    ref, mag = _oracle_decode(case, rows=rows)
    assert_scores_close(_np(sc)[rows, :32768], ref, mag, 1e-2)
    ridx, _ = oracle.topk(ref, 2048)
    assert_topk_equivalent(_np(idx)[rows], ridx, ref, 1e-2)
    assert api.li_get_last_error() == LI_OK


def test_multi_token_decode_32_heads():
    B, T, L = 3, 2, 6000
    case = synth.dsa_decode(B=B, L=L, H=H, seed=95, lens=[6000, 3000, 2049])
    g = torch.Generator().manual_seed(95)
    q = torch.randn(B * T, H, 128, generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn(B * T, H, generator=g) * 0.1).to(DEV)
    k8, ks, ln = case.k8.to(DEV), case.ks.to(DEV), case.lens.to(DEV)
    sc, idx = api.li_decode_select(q, w, k8, ks, 2048, lens=ln, tokens_per_request=T)
    for t in range(T):
        rows = [b * T + t for b in range(B)]
        lt = torch.clamp(case.lens - (T - 1 - t), min=0).to(DEV)
        sc_t, idx_t = api.li_decode_select(q[rows].contiguous(), w[rows].contiguous(), k8, ks, 2048, lens=lt)
        for i, r in enumerate(rows):
            n = int(lt[i])
            assert np.array_equal(_np(sc[r, :n]).view(np.uint32), _np(sc_t[i, :n]).view(np.uint32)), (t, r)
        assert np.array_equal(_np(idx[rows]), _np(idx_t)), t
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("B,L,lens,shared", [(2, 3000, [3000, 1234], False), (3, 700, None, True)])
def test_latent_32_heads_against_oracle(B, L, lens, shared):
    case = synth.latent_group(B=B, L=L, H=H, G=1, seed=96 + B, lens=lens)
    c = case.c[0:1] if shared else case.c
    cd = c.to(DEV)
    qt = api.li_absorb_query(case.q[0].to(DEV), case.w_dec[0].to(DEV))
    ln = case.lens.to(DEV)
    sc = api.li_latent_score(qt, case.w[0].to(DEV), cd[0] if shared else cd, lens=ln)
    ref, mag = oracle.latent_score(qt.cpu(), oracle.BF16, case.w[0], c[0] if shared else c, lens=case.lens.numpy(),
                                   c_batch_rows=0 if shared else None, with_mag=True)
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-2, visible=np.isfinite(ref))
    hist = api.li_decode_select_workspace(B, DEV).view(torch.int32)[:B * 2048]
    sc_h = api.li_latent_score_hist(qt, case.w[0].to(DEV), cd[0] if shared else cd, hist, lens=ln)
    idx, vals = api.li_topk_hist(sc_h, 256, hist, lens=ln, max_len=L, with_values=True)
    idx_r, vals_r = api.li_topk(sc, 256, lens=ln, max_len=L, with_values=True)
    for b, n in enumerate(case.lens.tolist()):
        assert np.array_equal(_np(sc_h[b, :n]).view(np.uint32), _np(sc[b, :n]).view(np.uint32)), b
    assert np.array_equal(_np(idx), _np(idx_r))
    assert np.array_equal(_np(vals).view(np.uint32), _np(vals_r).view(np.uint32))
    assert int(hist.count_nonzero()) == 0
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("F", [1, 3, 4])
def test_hs_refine_32_heads_against_oracle(F):
    B, L, C, k = 2, 4000, 640, 200
    case = synth.latent_hs(B=B, L=L, H=H, F=F, n_cand=C, k_top=k, seed=97 + F, lens=[4000, 1500])
    c = case.c.to(DEV)
    qts = [api.li_absorb_query(case.q[l].to(DEV), case.w_dec[l].to(DEV)) for l in range(1 + F)]
    sc = api.li_latent_score(qts[0], case.w[0].to(DEV), c, lens=case.lens.to(DEV))
    cand = api.li_topk(sc, C, lens=case.lens.to(DEV), max_len=L)
    qt_f = torch.stack(qts[1:]).contiguous()
    out = api.li_hs_refine(c, cand, qt_f, case.w[1:].contiguous().to(DEV), k)
    ref, cs = oracle.hs_refine(qt_f.cpu(), oracle.BF16, case.w[1:], case.c, _np(cand), k, with_scores=True)
    g = _np(out)
    for f in range(F):
        for b in range(B):
            cb = _np(cand)[b]
            assert set(g[f, b][g[f, b] >= 0].tolist()) <= set(cb[cb >= 0].tolist())
            pos = {int(p): i for i, p in enumerate(cb) if p >= 0}
            gi = np.array([[pos[int(p)] for p in g[f, b] if p >= 0] + [-1] * int((g[f, b] < 0).sum())])
            ri = np.array([[pos[int(p)] for p in ref[f, b] if p >= 0] + [-1] * int((ref[f, b] < 0).sum())])
            assert_topk_equivalent(gi, ri, cs[f, b:b + 1], 1e-2)
    assert api.li_get_last_error() == LI_OK
