"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/li.h declares, and rejects bad arguments before it touches
the device."""
import ctypes
import os
import re

import pytest

from sparse_attention_lightning_score_b200 import _lib

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "li.h")


def declared_symbols():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(li_[a-z0-9_]+)\s*\(", src, re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ["li_absorb_query", "li_index_score", "li_topk", "li_latent_score", "li_hs_refine",
                 "li_get_last_error", "li_quantize_query", "li_decode_select", "li_decode_select_workspace"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, name


def test_workspace_size_by_operation_matches_each_calls_own_size():
    """The one-call workspace form (op, rows, max_len, k) against the per-call sizes."""
    lib = _lib.load()
    for rows in [1, 8, 8192]:
        d = _lib.ScoreDesc(rows, 64, 128, 8192, 1, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
        assert lib.li_workspace_size(_lib.LI_OP_SCORE, rows, 8192, 2048) == lib.li_index_score_workspace(ctypes.byref(d))
        d.causal = 0
        d.max_len = 32768
        assert lib.li_workspace_size(_lib.LI_OP_DECODE_SELECT, rows, 32768, 2048) == \
            lib.li_decode_select_workspace(ctypes.byref(d))
        assert lib.li_workspace_size(_lib.LI_OP_TOPK, rows, 32768, 2048) == 0
    for B, C in [(1, 8192), (16, 8192), (3, 100)]:
        need = lib.li_workspace_size(_lib.LI_OP_HS, B, C, 2048)
        assert need == lib.li_hs_refine_workspace(B, C, 4)
        assert all(need >= lib.li_hs_refine_workspace(B, C, F) for F in (1, 2, 3))
    assert lib.li_workspace_size(99, 8, 100, 16) == 0
    assert lib.li_workspace_size(_lib.LI_OP_HS, -1, 100, 16) == 0


def test_status_strings():
    assert _lib.status_string(_lib.LI_OK) == "LI_OK"
    assert _lib.status_string(_lib.LI_ERR_TIMEOUT) == "LI_ERR_TIMEOUT"


def test_invalid_arguments_rejected_on_host():
    lib = _lib.load()
    p = ctypes.c_void_p(16)
    # k out of range, negative sizes, unaligned leading dimension, null descriptor
    assert lib.li_topk(p, 4, None, 1, 4, 0, 0, 0, p, None, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_topk(p, 4, None, 1, 4, 0, 0, _lib.LI_TOPK_MAX_LEN + 1, p, None, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_topk(p, 6, None, 1, 6, 0, 0, 2, p, None, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_topk(p, 4, None, -1, 4, 0, 0, 2, p, None, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_index_score(p, p, p, p, 0, None, p, 8, None, None, 0, None) == _lib.LI_ERR_INVALID_ARG
    d = _lib.ScoreDesc(2, 64, 128, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert lib.li_index_score(p, p, p, p, 0, None, p, 50, ctypes.byref(d), None, 0, None) == _lib.LI_ERR_INVALID_ARG
    d.causal = 1
    assert lib.li_index_score(p, p, p, p, 100, None, p, 100, ctypes.byref(d), None, 0, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_absorb_query(p, p, p, 1, 64, 128, 100, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_hs_refine(p, 0, 10, p, 1, 8, p, p, 0, 64, 256, 4, p, p, 0, None) == _lib.LI_ERR_INVALID_ARG


def test_decode_select_rejects_bad_arguments_on_host():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    d = _lib.ScoreDesc(2, 64, 128, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    ws = lib.li_decode_select_workspace(ctypes.byref(d))
    assert ws == 2 * 2048 * 4

    def call(desc, k_top=8, ld=100, wsb=ws, wsp=p, scores=p):
        return lib.li_decode_select(p, p, p, p, 0, None, scores, ld, ctypes.byref(desc), k_top, p, None, wsp, wsb,
                                    None)

    assert call(d, k_top=0) == _lib.LI_ERR_INVALID_ARG                      # k out of range
    assert call(d, k_top=_lib.LI_TOPK_MAX_LEN + 1) == _lib.LI_ERR_INVALID_ARG
    assert call(d, wsb=ws - 4) == _lib.LI_ERR_INVALID_ARG                   # workspace too small
    assert call(d, wsp=ctypes.c_void_p(272)) == _lib.LI_ERR_INVALID_ARG     # workspace not 256-byte aligned
    assert call(d, wsp=None) == _lib.LI_ERR_INVALID_ARG
    assert call(d, ld=102) == _lib.LI_ERR_INVALID_ARG                       # ld not a multiple of 4
    assert call(d, ld=96) == _lib.LI_ERR_INVALID_ARG                        # ld below max_len
    assert call(d, scores=ctypes.c_void_p(264)) == _lib.LI_ERR_INVALID_ARG  # scores not 16-byte aligned
    c = _lib.ScoreDesc(2, 64, 128, 100, 1, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert call(c) == _lib.LI_ERR_INVALID_ARG                               # causal is not a decode step
    u = _lib.ScoreDesc(2, 48, 128, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert call(u) == _lib.LI_ERR_UNSUPPORTED                               # only the tensor-core shapes: 64 or 32 heads
    u = _lib.ScoreDesc(2, 64, 64, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert call(u) == _lib.LI_ERR_UNSUPPORTED                               # dim 128 only
    f = _lib.ScoreDesc(2, 64, 128, 100, 0, 0, _lib.LI_DTYPE_F32, _lib.LI_DTYPE_F32)
    assert call(f) == _lib.LI_ERR_UNSUPPORTED
    z = _lib.ScoreDesc(0, 64, 128, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert call(z) == _lib.LI_OK                                            # no rows: nothing to do


def test_zero_sized_calls_are_no_ops():
    lib = _lib.load()
    p = ctypes.c_void_p(16)
    assert lib.li_topk(p, 4, None, 0, 4, 0, 0, 2, p, None, None) == _lib.LI_OK
    d = _lib.ScoreDesc(0, 64, 128, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert lib.li_index_score(p, p, p, p, 0, None, p, 100, ctypes.byref(d), None, 0, None) == _lib.LI_OK


def test_workspace_sizes():
    lib = _lib.load()
    d = _lib.ScoreDesc(8192, 64, 128, 8192, 1, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert lib.li_index_score_workspace(ctypes.byref(d)) >= 8192 * 64 * (128 + 8)
    d.causal = 0
    assert lib.li_index_score_workspace(ctypes.byref(d)) == 0
    assert lib.li_hs_refine_workspace(16, 8192, 3) == 3 * 16 * 8192 * 4 + 3 * 16 * 2048 * 4  # scores + histograms
    assert lib.li_hs_refine_workspace(1, 5, 2) == 2 * 8 * 4 + 2 * 2048 * 4


def test_latent_fp8_and_layers_reject_bad_arguments_on_host():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    # (q~, w, c8, cs, cache_batch_rows, len, scores, ld, batch, heads, latent_dim, max_len, hist, stream)
    assert lib.li_latent_score_fp8(p, p, p, p, 0, None, p, 100, 2, 32, 192, 100, None, None) == _lib.LI_ERR_UNSUPPORTED
    assert lib.li_latent_score_fp8(p, p, p, p, 0, None, p, 100, 2, 64, 256, 100, None, None) == _lib.LI_ERR_UNSUPPORTED
    assert lib.li_latent_score_fp8(p, p, ctypes.c_void_p(264), p, 0, None, p, 100, 2, 64, 192, 100, None,
                                   None) == _lib.LI_ERR_INVALID_ARG          # cache not 16-byte aligned
    assert lib.li_latent_score_fp8(p, p, p, None, 0, None, p, 100, 2, 64, 192, 100, None,
                                   None) == _lib.LI_ERR_INVALID_ARG          # no scales
    assert lib.li_latent_score_fp8(p, p, p, p, 0, None, p, 50, 2, 64, 192, 100, None,
                                   None) == _lib.LI_ERR_INVALID_ARG          # ld below max_len
    assert lib.li_latent_score_fp8(p, p, p, p, 0, None, p, 100, 0, 64, 192, 100, None, None) == _lib.LI_OK
    assert lib.li_latent_score_hist(p, p, p, 0, None, p, 100, 2, 64, 256, 100, None,
                                    None) == _lib.LI_ERR_INVALID_ARG         # hist required
    # (q, w_dec, q~, layers, batch, heads, dim, latent_dim, stream)
    assert lib.li_absorb_query_layers(p, p, p, -1, 1, 64, 128, 256, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_absorb_query_layers(p, p, p, 2, 1, 64, 128, 100, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_absorb_query_layers(p, p, p, 0, 1, 64, 128, 256, None) == _lib.LI_OK


def test_head_counts_checked_on_host():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    # GLM-5's 32 indexer heads are a decode shape; prefill keeps 64
    c = _lib.ScoreDesc(8, 32, 128, 100, 1, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
    assert lib.li_index_score(p, p, p, p, 0, None, p, 100, ctypes.byref(c), p, 1 << 20,
                              None) == _lib.LI_ERR_UNSUPPORTED
    # (q~, w, c, cache_batch_rows, len, scores, ld, batch, heads, latent_dim, max_len, stream)
    assert lib.li_latent_score(p, p, p, 0, None, p, 100, 2, 16, 256, 100, None) == _lib.LI_ERR_UNSUPPORTED
    assert lib.li_latent_score(p, p, p, 0, None, p, 100, 2, 32, 192, 100, None) == _lib.LI_ERR_UNSUPPORTED
    # (c, cache_batch_rows, cache_rows, cand, batch, n_cand, q~, w, followers, heads, latent_dim, k, out, ws, bytes, st)
    assert lib.li_hs_refine(p, 0, 100, p, 1, 64, p, p, 5, 32, 256, 8, p, p, 1 << 20, None) == _lib.LI_ERR_UNSUPPORTED
    assert lib.li_hs_refine(p, 0, 100, p, 1, 64, p, p, 2, 48, 256, 8, p, p, 1 << 20, None) == _lib.LI_ERR_UNSUPPORTED


def test_graph_calls_check_arguments_on_host():
    lib = _lib.load()
    out = ctypes.c_void_p()
    assert lib.li_graph_instantiate(None, 1, ctypes.byref(out)) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_graph_instantiate(ctypes.c_void_p(256), 1, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_graph_launch(None, None) == _lib.LI_ERR_INVALID_ARG
    assert lib.li_graph_destroy(None) == _lib.LI_OK


def test_decode_select_workspace_is_one_histogram_per_row():
    lib = _lib.load()
    for L in (0, 1000, 32768, 262144):
        d = _lib.ScoreDesc(8, 64, 128, L, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3)
        assert lib.li_decode_select_workspace(ctypes.byref(d)) == 8 * 2048 * 4


def test_multi_token_descriptor_checked_on_host():
    lib = _lib.load()
    p = ctypes.c_void_p(256)
    d = _lib.ScoreDesc(6, 64, 128, 100, 0, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3, 4)  # 6 rows, 4 tokens
    assert lib.li_index_score(p, p, p, p, 0, None, p, 100, ctypes.byref(d), None, 0, None) == _lib.LI_ERR_INVALID_ARG
    ws = lib.li_decode_select_workspace(ctypes.byref(d))
    assert lib.li_decode_select(p, p, p, p, 0, None, p, 100, ctypes.byref(d), 8, p, None, p, ws,
                                None) == _lib.LI_ERR_INVALID_ARG
    c = _lib.ScoreDesc(8, 64, 128, 100, 1, 0, _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3, 2)   # causal with 2 tokens
    assert lib.li_index_score(p, p, p, p, 0, None, p, 100, ctypes.byref(c), p, 1 << 20,
                              None) == _lib.LI_ERR_UNSUPPORTED
    assert lib.li_topk_hist(p, 100, None, 6, 100, 8, p, None, p, 4, None) == _lib.LI_ERR_INVALID_ARG
