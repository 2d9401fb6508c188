"""GPU parity of the FP8 latent scan (li_latent_score_fp8): DeepSeek-V3.2's shared
latent of 64 RoPE + 128 NoPE dimensions stored as an e4m3 cache with per-row
scales (LatentIndex appendix, Table 5).

The kernel quantises the absorbed bf16 query per (request, head) as
li_quantize_query does; the oracle quantises the same bf16 query itself and
scores the same cache bytes in fp64.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_lightning_score_b200 import api, synth
from sparse_attention_lightning_score_b200._lib import LI_OK
from tests._checks import assert_scores_close, assert_topk_equivalent

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().cpu().numpy()


def _absorbed(case, layer=0):
    return api.li_absorb_query(case.q[layer].to(DEV), case.w_dec[layer].to(DEV))


def _oracle_scores(case, qt, layer=0, rows=None):
    q8, sq, _ = oracle.quantize_query(qt.cpu(), case.w[layer].numpy())
    L = case.c8.shape[1]
    return oracle.index_score(q8, oracle.E4M3, case.w[layer], case.c8, oracle.E4M3, q_scale=sq, k_scale=case.cs,
                              k_batch_rows=L, L=L, lens=case.lens.numpy(), rows=rows, with_mag=True)


@pytest.mark.parametrize("B,L,lens", [(2, 3000, None), (3, 1000, [1000, 129, 0]), (1, 300, None)])
def test_latent8_scores_match_oracle(B, L, lens):
    case = synth.latent_rope_nope(B=B, L=L, G=1, seed=90 + B, lens=lens)
    qt = _absorbed(case)
    sc = api.li_latent_score_fp8(qt, case.w[0].to(DEV), case.c8.to(DEV), case.cs.to(DEV), lens=case.lens.to(DEV))
    ref, mag = _oracle_scores(case, qt)
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-2)
    k = min(256, L)
    idx = api.li_topk(sc, k, lens=case.lens.to(DEV), max_len=L)
    ridx, _ = oracle.topk(ref, k, lens=case.lens.numpy())
    assert_topk_equivalent(_np(idx), ridx, ref, 1e-2, n_valid=case.lens.numpy())
    assert api.li_get_last_error() == LI_OK


def test_latent8_rope_part_passes_through_absorption():
    # the RoPE block of the decoder is the identity: q~[:, :, :64] is the query's own RoPE part
    case = synth.latent_rope_nope(B=2, L=64, G=1, seed=95)
    qt = _absorbed(case)
    assert torch.equal(qt[:, :, :64].cpu(), case.q[0, :, :, :64])


def test_latent8_shared_cache():
    case = synth.latent_rope_nope(B=1, L=2000, G=1, seed=96)
    g = torch.Generator().manual_seed(96)
    q = torch.randn(4, 64, 128, generator=g).to(torch.bfloat16)
    w = torch.randn(4, 64, generator=g) * 0.1
    qt = api.li_absorb_query(q.to(DEV), case.w_dec[0].to(DEV))
    sc = api.li_latent_score_fp8(qt, w.to(DEV), case.c8[0].to(DEV), case.cs[0].to(DEV))
    q8, sq, _ = oracle.quantize_query(qt.cpu(), w.numpy())
    ref, mag = oracle.index_score(q8, oracle.E4M3, w, case.c8[0], oracle.E4M3, q_scale=sq, k_scale=case.cs[0],
                                  k_batch_rows=0, L=2000, with_mag=True)
    assert_scores_close(_np(sc)[:, :2000], ref, mag, 1e-2)
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("B,L,k", [(4, 65536, 2048), (2, 9000, 100)])
def test_latent8_hist_then_topk_hist(B, L, k):
    """With the histogram: scores bit for bit those of the plain call, the same selection as
    li_topk on them, and the histogram left zero."""
    case = synth.latent_rope_nope(B=B, L=L, G=1, seed=97)
    qt = _absorbed(case)
    w, c8, cs = case.w[0].to(DEV), case.c8.to(DEV), case.cs.to(DEV)
    hist = api.li_decode_select_workspace(B, DEV).view(torch.int32)[:B * 2048]
    sc = api.li_latent_score_fp8(qt, w, c8, cs, hist=hist)
    idx = api.li_topk_hist(sc, k, hist, max_len=L)
    sc_r = api.li_latent_score_fp8(qt, w, c8, cs)
    assert np.array_equal(_np(sc[:, :L]).view(np.uint32), _np(sc_r[:, :L]).view(np.uint32))
    assert np.array_equal(_np(idx), _np(api.li_topk(sc_r, k, max_len=L)))
    assert api.li_get_last_error() == LI_OK
    assert int(hist.count_nonzero()) == 0


def test_latent8_full_size_sampled_rows():
    """B = 4, L = 65536 (the latent workload's shape): sampled requests against the oracle."""
    case = synth.latent_rope_nope(B=4, L=65536, G=1, seed=98)
    qt = _absorbed(case)
    sc = api.li_latent_score_fp8(qt, case.w[0].to(DEV), case.c8.to(DEV), case.cs.to(DEV))
    rows = [0, 3]
    ref, mag = _oracle_scores(case, qt, rows=rows)
    assert_scores_close(_np(sc)[rows, :65536], ref, mag, 1e-2)
    idx = api.li_topk(sc, 2048, max_len=65536)
    ridx, _ = oracle.topk(ref, 2048)
    assert_topk_equivalent(_np(idx)[rows], ridx, ref, 1e-2)
    assert api.li_get_last_error() == LI_OK


# ---------------------------------------------------------------------------
# hierarchical selection over the FP8 latent (li_hs_refine_fp8)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,L,C,k,F,lens", [(2, 3000, 512, 128, 3, None), (3, 2000, 640, 100, 2, [2000, 500, 77]),
                                            (1, 1000, 130, 130, 1, None), (2, 20000, 8192, 2048, 4, None)])
def test_hs_fp8_matches_oracle(B, L, C, k, F, lens):
    case = synth.latent_rope_nope(B=B, L=L, G=1 + F, seed=70 + F, lens=lens)
    qts = [_absorbed(case, l) for l in range(1 + F)]
    c8, cs, ln = case.c8.to(DEV), case.cs.to(DEV), case.lens.to(DEV)
    sc = api.li_latent_score_fp8(qts[0], case.w[0].to(DEV), c8, cs, lens=ln)
    cand = api.li_topk(sc, C, lens=ln, max_len=L)
    qt_f = torch.stack(qts[1:]).contiguous()
    wf = case.w[1:].contiguous()
    out = api.li_hs_refine_fp8(c8, cs, cand, qt_f, wf.to(DEV), k)
    ref, cscores = oracle.hs_refine_fp8(qt_f.cpu(), wf, case.c8, case.cs, _np(cand), k, with_scores=True)
    g = _np(out)
    for f in range(F):
        for b in range(B):
            cb = _np(cand)[b]
            assert set(g[f, b][g[f, b] >= 0].tolist()) <= set(cb[cb >= 0].tolist())
            pos = {int(p): i for i, p in enumerate(cb) if p >= 0}
            gi = np.array([[pos[int(p)] for p in g[f, b] if p >= 0] + [-1] * int((g[f, b] < 0).sum())])
            ri = np.array([[pos[int(p)] for p in ref[f, b] if p >= 0] + [-1] * int((ref[f, b] < 0).sum())])
            assert_topk_equivalent(gi, ri, cscores[f, b:b + 1], 1e-2)
    assert api.li_get_last_error() == LI_OK


def test_hs_fp8_histogram_path_equals_plain_passes():
    # as for the bf16 latent: dirty histograms give the same selection, are reported and healed
    from sparse_attention_lightning_score_b200._lib import LI_ERR_BOUNDS
    F, C, k = 3, 8192, 2048
    case = synth.latent_rope_nope(B=2, L=20000, G=1 + F, seed=91)
    qts = [_absorbed(case, l) for l in range(1 + F)]
    c8, cs = case.c8.to(DEV), case.cs.to(DEV)
    sc = api.li_latent_score_fp8(qts[0], case.w[0].to(DEV), c8, cs)
    cand = api.li_topk(sc, C, max_len=20000)
    qt_f = torch.stack(qts[1:]).contiguous()
    wf = case.w[1:].contiguous().to(DEV)
    ws = api.li_hs_refine_workspace(2, C, F, DEV)
    tail = ws[ws.numel() - F * 2 * 2048 * 4:]
    out = api.li_hs_refine_fp8(c8, cs, cand, qt_f, wf, k, workspace=ws)
    torch.cuda.synchronize()
    assert api.li_get_last_error() == LI_OK and int(tail.count_nonzero()) == 0
    tail.view(torch.int32)[::5] = 1
    dirty = api.li_hs_refine_fp8(c8, cs, cand, qt_f, wf, k, workspace=ws)
    torch.cuda.synchronize()
    assert api.li_get_last_error() == LI_ERR_BOUNDS and int(tail.count_nonzero()) == 0
    assert torch.equal(out, dirty)


def test_hs_fp8_out_of_range_candidate_reported():
    case = synth.latent_rope_nope(B=1, L=500, G=2, seed=77)
    qt = _absorbed(case, 1)
    cand = torch.tensor([[3, 7, 499, 500]], dtype=torch.int32, device=DEV)  # 500: one past the cache
    api.li_hs_refine_fp8(case.c8.to(DEV), case.cs.to(DEV), cand, qt[None].contiguous(),
                         case.w[1:2].contiguous().to(DEV), 2)
    from sparse_attention_lightning_score_b200._lib import LI_ERR_BOUNDS
    assert api.li_get_last_error() == LI_ERR_BOUNDS
