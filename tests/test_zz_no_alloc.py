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


def _random_hs(F, B, L, C, seed):
    """Random latent rows, absorbed queries and weights (no anchor scan needed): every request's
    candidates are its first C positions, in ascending order."""
    g = torch.Generator(device=DEV).manual_seed(seed)
    c = torch.randn(B, L, 256, generator=g, device=DEV).to(torch.bfloat16)
    qt = torch.randn(F, B, 64, 256, generator=g, device=DEV).div_(16).to(torch.bfloat16)
    w = torch.randn(F, B, 64, generator=g, device=DEV).mul_(0.1)
    cand = torch.arange(C, dtype=torch.int32, device=DEV).repeat(B, 1).contiguous()
    return c, cand, qt, w


@pytest.mark.gpu
def test_noalloc_alternating_long_and_many_row_calls_stay_exact_and_ok():
    # A: one follower, 4 requests, the most candidates the array takes (260,096): its scores fill
    #    almost all of the array, including the end where B keeps its histograms.
    # B: four followers, 16 requests: 512 KB of histograms at the array's end.
    # Alternating them, every call must select what li_hs_refine selects with a fresh workspace,
    # and report no error.
    big = _random_hs(1, 4, 260096, 260096, 91)
    many = _random_hs(4, 16, 1024, 512, 92)
    lib = _lib.load()
    assert lib.li_hs_refine_workspace(4, 260096, 1) <= 4 * _lib.LI_HS_NOALLOC_MAX_SCRATCH_FLOATS
    for case, k in [(big, 2048), (many, 100), (big, 2048), (many, 100)]:
        c, cand, qt, w = case
        ref = api.li_hs_refine(c, cand, qt, w, k)
        out = torch.full((qt.shape[0], qt.shape[1], k), -7, dtype=torch.int32, device=DEV)
        assert _call_noalloc(c, cand, qt, w, k, out) == _lib.LI_OK
        torch.cuda.synchronize()
        assert api.li_get_last_error() == _lib.LI_OK
        assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # rejected on the host before anything touches a device: the limit is the whole workspace
    # li_hs_refine would take (candidate scores plus histograms), 4 MiB
    lib = _lib.load()
    cap = 4 * _lib.LI_HS_NOALLOC_MAX_SCRATCH_FLOATS
    p = ctypes.c_void_p(256)
    for F, B, C in [(3, 16, 65536), (1, 4, 262144), (1, 4, 260100), (3, 16, 19800)]:
        assert lib.li_hs_refine_workspace(B, C, F) > cap, (F, B, C)
        st = lib.li_hs_refine_noalloc(p, 0, 1 << 20, p, B, C, p, p, F, 64, 256, 8, p, None)
        assert st == _lib.LI_ERR_INVALID_ARG, (F, B, C)
    # the largest accepted sizes the header names
    assert lib.li_hs_refine_workspace(4, 260096, 1) <= cap
    assert lib.li_hs_refine_workspace(16, 19796, 3) <= cap
