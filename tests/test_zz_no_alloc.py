"""li_hs_refine_noalloc, the allocation-free variant of li_hs_refine.

Callers inside an engine that owns all device memory (or a plugin handed only
its inputs and outputs) cannot give li_hs_refine a workspace; this entry point
keeps the followers' candidate scores in a fixed device array instead.  It must
select exactly what the allocating entry point selects, call after call, even
though every call reuses the same array.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_lightning_score_b200 import _lib, api, synth

DEV = "cuda"


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(c, cand, qt, w, k, out):
    F, B, H, dc = qt.shape
    st = _lib.load().li_hs_refine_noalloc(_p(c), c.shape[1], c.numel() // dc, _p(cand), B, cand.shape[1], _p(qt),
                                          _p(w), F, H, dc, int(k), _p(out),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _inputs(seed, B, L, C, k, lens):
    case = synth.latent_hs(B=B, L=L, n_cand=C, k_top=k, seed=seed, lens=lens)
    c = case.c.to(DEV)
    qts = [api.li_absorb_query(case.q[l].to(DEV), case.w_dec[l].to(DEV)) for l in range(4)]
    lens_d = case.lens.to(DEV)
    sc = api.li_latent_score(qts[0], case.w[0].to(DEV), c, lens=lens_d)
    cand = api.li_topk(sc, C, lens=lens_d, max_len=L)
    return c, cand, torch.stack(qts[1:]).contiguous(), case.w[1:].contiguous().to(DEV)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # two calls in a row with different shapes and inputs: the second call reuses
    # the array the first one filled
    for seed, B, L, C, k, lens in [(81, 3, 4000, 1024, 256, [4000, 2500, 700]), (82, 2, 3000, 900, 300, None)]:
        c, cand, qt, w = _inputs(seed, B, L, C, k, lens)
        ref = api.li_hs_refine(c, cand, qt, w, k)
        out = torch.full((qt.shape[0], B, k), -7, dtype=torch.int32, device=DEV)
        assert _call_noalloc(c, cand, qt, w, k, out) == _lib.LI_OK
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), ref.cpu().numpy())
    assert api.li_get_last_error() == _lib.LI_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 3 followers x 16 requests x 65536 candidates = 3 Mi floats > 1 Mi capacity:
    # rejected on the host before anything touches a device
    p = ctypes.c_void_p(256)
    st = _lib.load().li_hs_refine_noalloc(p, 0, 1 << 20, p, 16, 65536, p, p, 3, 64, 256, 8, p, None)
    assert st == _lib.LI_ERR_INVALID_ARG
