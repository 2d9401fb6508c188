"""Thin PyTorch binding over the li C ABI: same names, argument marshalling only.

Every function takes CUDA tensors, allocates the outputs (and any workspace)
with torch on the tensors' device, passes raw device pointers and the current
torch stream to ``libli.so``, and raises ``LiError`` on a non-OK status.  No
step of the indexer path runs in Python or torch.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import LiError, ScoreDesc  # noqa: F401  (re-exported)


def _ptr(t: Optional[torch.Tensor]):
    """Device address of a tensor: a CUDA tensor's own, or for a page-locked host tensor the
    address the kernels use to reach it (li_host_device_pointer)."""
    if t is None:
        return None
    if t.is_cuda:
        return ctypes.c_void_p(t.data_ptr())
    if not t.is_pinned():
        raise ValueError("host tensors handed to the kernels must be page-locked (pin_memory())")
    return ctypes.c_void_p(li_host_device_pointer(t))


def li_host_device_pointer(t: torch.Tensor) -> int:
    """Device-side address of a page-locked host tensor (raises if it is not mapped)."""
    out = ctypes.c_void_p()
    st = _lib.load().li_host_device_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(out))
    _lib.check("li_host_device_pointer", st)
    return int(out.value)


def li_copy_from_host(dst: torch.Tensor, src: torch.Tensor, stream=None):
    """dst (CUDA) <- src (page-locked host, same byte size), copied by a kernel on `stream`."""
    _need(dst, "dst")
    if src.is_cuda or not src.is_pinned() or not src.is_contiguous():
        raise ValueError("src must be a contiguous page-locked host tensor")
    nbytes = dst.numel() * dst.element_size()
    if src.numel() * src.element_size() != nbytes:
        raise ValueError("dst and src differ in size")
    st = _lib.load().li_copy_from_host(_ptr(dst), _ptr(src), nbytes, _stream(stream))
    _lib.check("li_copy_from_host", st)
    return dst


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _round4(n: int) -> int:
    return (n + 3) // 4 * 4


def li_get_last_error() -> int:
    """Synchronise the device and return (and clear) the device error status."""
    return int(_lib.load().li_get_last_error())


def li_quantize_query(q: torch.Tensor, w: Optional[torch.Tensor] = None, stream=None):
    """q bf16 [R,H,d] (+ w fp32 [R,H]) -> (q8 uint8 [R,H,d], sq fp32 [R,H], w_eff fp32 [R,H] or None)."""
    _need(q, "q", torch.bfloat16)
    R, H, d = q.shape
    q8 = torch.empty((R, H, d), dtype=torch.uint8, device=q.device)
    sq = torch.empty((R, H), dtype=torch.float32, device=q.device)
    we = None
    if w is not None:
        _need(w, "w", torch.float32)
        we = torch.empty((R, H), dtype=torch.float32, device=q.device)
    st = _lib.load().li_quantize_query(_ptr(q), _ptr(w), R, H, d, _ptr(q8), _ptr(sq), _ptr(we), _stream(stream))
    _lib.check("li_quantize_query", st)
    return q8, sq, we


def score_desc(rows, heads, dim, max_len, causal=False, causal_offset=0, q_dtype=_lib.LI_DTYPE_BF16,
               k_dtype=_lib.LI_DTYPE_E4M3, tokens_per_request=1) -> ScoreDesc:
    return ScoreDesc(int(rows), int(heads), int(dim), int(max_len), int(bool(causal)), int(causal_offset),
                     int(q_dtype), int(k_dtype), int(tokens_per_request))


def li_index_score(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, k_scale: Optional[torch.Tensor] = None, *,
                   lens: Optional[torch.Tensor] = None, causal: bool = False, causal_offset: int = 0,
                   scores: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   tokens_per_request: int = 1, stream=None):
    """DSA lightning-indexer scores.

    q: [R,H,d] bf16 (FP8 tensor-core path, k uint8/float8_e4m3fn + k_scale) or fp32
    (exact path, k fp32).  k: [R,L,d] (one cache per row) or [L,d] (shared cache).
    Returns scores fp32 [R, round4(L)]; positions a row cannot see are left unwritten.
    """
    _need(q, "q", (torch.bfloat16, torch.float32))
    _need(w, "w", torch.float32)
    _need(k, "k")
    R, H, d = q.shape
    if k.dtype == torch.float8_e4m3fn:
        k = k.view(torch.uint8)
    L = k.shape[-2]
    batch_rows = k.shape[1] if k.dim() == 3 else 0
    if q.dtype == torch.float32:
        qd, kd = _lib.LI_DTYPE_F32, _lib.LI_DTYPE_F32
    else:
        qd, kd = _lib.LI_DTYPE_BF16, _lib.LI_DTYPE_E4M3
        _need(k_scale, "k_scale", torch.float32)
    if lens is not None:
        _need(lens, "lens", torch.int32)
    desc = score_desc(R, H, d, L, causal, causal_offset, qd, kd, tokens_per_request)
    lib = _lib.load()
    if scores is None:
        scores = torch.empty((R, _round4(L)), dtype=torch.float32, device=q.device)
    need = lib.li_index_score_workspace(ctypes.byref(desc))
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib.li_index_score(_ptr(q), _ptr(w), _ptr(k), _ptr(k_scale), batch_rows, _ptr(lens), _ptr(scores),
                            scores.stride(0), ctypes.byref(desc), _ptr(workspace) if need else None,
                            need, _stream(stream))
    _lib.check("li_index_score", st)
    return scores


def li_topk(scores: torch.Tensor, k: int, *, lens: Optional[torch.Tensor] = None, max_len: Optional[int] = None,
            causal: bool = False, causal_offset: int = 0, with_values: bool = False, idx=None, vals=None,
            stream=None):
    """Per-row top-k -> idx int32 [rows, k] ascending (-1 pads) [, vals fp32 [rows, k]]."""
    _need(scores, "scores", torch.float32)
    rows, ld = scores.shape
    if max_len is None:
        max_len = ld
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    if with_values and vals is None:
        vals = torch.empty((rows, k), dtype=torch.float32, device=scores.device)
    st = _lib.load().li_topk(_ptr(scores), ld, _ptr(lens), rows, int(max_len), int(bool(causal)), int(causal_offset),
                             int(k), _ptr(idx), _ptr(vals) if with_values else None, _stream(stream))
    _lib.check("li_topk", st)
    return (idx, vals) if with_values else idx


def li_decode_select_workspace(rows: int, device, max_len: int = 0) -> torch.Tensor:
    """A zeroed workspace for li_decode_select over `rows` rows: one 2048-bin histogram per row,
    which every call leaves zero again (also the histogram buffer of li_decode_score_hist /
    li_topk_hist / li_latent_score_hist).  `max_len` does not change its size."""
    desc = score_desc(rows, 64, 128, int(max_len))
    need = _lib.load().li_decode_select_workspace(ctypes.byref(desc))
    return torch.zeros(max(int(need), 256), dtype=torch.uint8, device=device)


def li_decode_select_hist_bytes(rows: int) -> int:
    """Bytes of li_decode_select's workspace that hold the histograms (zero between calls)."""
    return rows * 2048 * 4


def li_decode_select(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, k_scale: torch.Tensor, k_top: int, *,
                     lens: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, with_values: bool = False, idx=None, vals=None,
                     tokens_per_request: int = 1, stream=None):
    """Decode score + top-k in one call -> (scores, idx[, vals]).

    Same arguments as li_index_score's decode form (q bf16 [B,64,128], k e4m3 [B,L,128] or [L,128],
    k_scale) and li_topk's k / outputs.  `workspace` is a zeroed buffer from li_decode_select_workspace
    for these rows and this length (made here when omitted); its histograms are left zero again for
    the next call.
    """
    _need(q, "q", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(k, "k")
    _need(k_scale, "k_scale", torch.float32)
    if k.dtype == torch.float8_e4m3fn:
        k = k.view(torch.uint8)
    R, H, d = q.shape
    L = k.shape[-2]
    batch_rows = k.shape[1] if k.dim() == 3 else 0
    if lens is not None:
        _need(lens, "lens", torch.int32)
    desc = score_desc(R, H, d, L, tokens_per_request=tokens_per_request)
    lib = _lib.load()
    if scores is None:
        scores = torch.empty((R, _round4(L)), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = li_decode_select_workspace(R, q.device, L)
    if idx is None:  # (idx / vals may also be page-locked host tensors: the top-k writes them directly)
        idx = torch.empty((R, k_top), dtype=torch.int32, device=q.device)
    if with_values and vals is None:
        vals = torch.empty((R, k_top), dtype=torch.float32, device=q.device)
    st = lib.li_decode_select(_ptr(q), _ptr(w), _ptr(k), _ptr(k_scale), batch_rows, _ptr(lens), _ptr(scores),
                              scores.stride(0), ctypes.byref(desc), int(k_top), _ptr(idx),
                              _ptr(vals) if with_values else None, _ptr(workspace), workspace.numel(),
                              _stream(stream))
    _lib.check("li_decode_select", st)
    return (scores, idx, vals) if with_values else (scores, idx)


def li_decode_select_score(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, k_scale: torch.Tensor,
                           workspace: torch.Tensor, *, lens: Optional[torch.Tensor] = None,
                           scores: Optional[torch.Tensor] = None, tokens_per_request: int = 1, stream=None):
    """First kernel of li_decode_select: the scores, plus the counts in the workspace's histograms."""
    _need(q, "q", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(k, "k")
    _need(k_scale, "k_scale", torch.float32)
    if k.dtype == torch.float8_e4m3fn:
        k = k.view(torch.uint8)
    R, H, d = q.shape
    L = k.shape[-2]
    batch_rows = k.shape[1] if k.dim() == 3 else 0
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if scores is None:
        scores = torch.empty((R, _round4(L)), dtype=torch.float32, device=q.device)
    desc = score_desc(R, H, d, L, tokens_per_request=tokens_per_request)
    st = _lib.load().li_decode_select_score(_ptr(q), _ptr(w), _ptr(k), _ptr(k_scale), batch_rows, _ptr(lens),
                                            _ptr(scores), scores.stride(0), ctypes.byref(desc), _ptr(workspace),
                                            workspace.numel(), _stream(stream))
    _lib.check("li_decode_select_score", st)
    return scores


def li_decode_select_finish(scores: torch.Tensor, k_top: int, workspace: torch.Tensor, *, heads: int = 64,
                            max_len: Optional[int] = None, lens: Optional[torch.Tensor] = None,
                            with_values: bool = False, idx=None, vals=None, tokens_per_request: int = 1, stream=None):
    """Second kernel of li_decode_select: the top-k from the scores and the workspace's counts."""
    _need(scores, "scores", torch.float32)
    rows, ld = scores.shape
    if max_len is None:
        max_len = ld
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if idx is None:
        idx = torch.empty((rows, k_top), dtype=torch.int32, device=scores.device)
    if with_values and vals is None:
        vals = torch.empty((rows, k_top), dtype=torch.float32, device=scores.device)
    desc = score_desc(rows, heads, 128, int(max_len), tokens_per_request=tokens_per_request)
    st = _lib.load().li_decode_select_finish(_ptr(scores), ld, _ptr(lens), ctypes.byref(desc), int(k_top), _ptr(idx),
                                             _ptr(vals) if with_values else None, _ptr(workspace), workspace.numel(),
                                             _stream(stream))
    _lib.check("li_decode_select_finish", st)
    return (idx, vals) if with_values else idx


def li_decode_score_hist(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, k_scale: torch.Tensor,
                         hist: torch.Tensor, *, lens: Optional[torch.Tensor] = None,
                         scores: Optional[torch.Tensor] = None, tokens_per_request: int = 1, stream=None):
    """First half of li_decode_select: decode scores, plus counts added to `hist` (a zeroed
    li_decode_select_workspace buffer)."""
    _need(q, "q", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(k, "k")
    _need(k_scale, "k_scale", torch.float32)
    if k.dtype == torch.float8_e4m3fn:
        k = k.view(torch.uint8)
    R, H, d = q.shape
    L = k.shape[-2]
    batch_rows = k.shape[1] if k.dim() == 3 else 0
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if scores is None:
        scores = torch.empty((R, _round4(L)), dtype=torch.float32, device=q.device)
    desc = score_desc(R, H, d, L, tokens_per_request=tokens_per_request)
    st = _lib.load().li_decode_score_hist(_ptr(q), _ptr(w), _ptr(k), _ptr(k_scale), batch_rows, _ptr(lens),
                                          _ptr(scores), scores.stride(0), ctypes.byref(desc), _ptr(hist),
                                          _stream(stream))
    _lib.check("li_decode_score_hist", st)
    return scores


def li_topk_hist(scores: torch.Tensor, k: int, hist: torch.Tensor, *, lens: Optional[torch.Tensor] = None,
                 max_len: Optional[int] = None, with_values: bool = False, idx=None, vals=None,
                 tokens_per_request: int = 1, stream=None):
    """Second half of li_decode_select: li_topk using (and clearing) the scorer's histogram."""
    _need(scores, "scores", torch.float32)
    rows, ld = scores.shape
    if max_len is None:
        max_len = ld
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    if with_values and vals is None:
        vals = torch.empty((rows, k), dtype=torch.float32, device=scores.device)
    st = _lib.load().li_topk_hist(_ptr(scores), ld, _ptr(lens), rows, int(max_len), int(k), _ptr(idx),
                                  _ptr(vals) if with_values else None, _ptr(hist), int(tokens_per_request),
                                  _stream(stream))
    _lib.check("li_topk_hist", st)
    return (idx, vals) if with_values else idx


def li_merge_shards(vals: torch.Tensor, idx: torch.Tensor, shard_len: int, k_out: int, *,
                    with_values: bool = False, out_idx=None, out_vals=None, workspace=None, stream=None):
    """Global top-k from per-shard selections: vals fp32 / idx int32 [shards, rows, k] (local
    positions, each shard's list ascending then -1) -> out_idx int32 [rows, k_out] of global
    positions (shard p covers p*shard_len ..) [, out_vals]."""
    _need(vals, "vals", torch.float32)
    _need(idx, "idx", torch.int32)
    P, R, k = vals.shape
    lib = _lib.load()
    need = lib.li_merge_shards_workspace(P, R, k)
    if workspace is None or workspace.numel() < need:
        workspace = torch.zeros(max(int(need), 256), dtype=torch.uint8, device=vals.device)  # histograms start zero
    if out_idx is None:
        out_idx = torch.empty((R, k_out), dtype=torch.int32, device=vals.device)
    if with_values and out_vals is None:
        out_vals = torch.empty((R, k_out), dtype=torch.float32, device=vals.device)
    st = lib.li_merge_shards(_ptr(vals), _ptr(idx), P, R, k, int(shard_len), int(k_out), _ptr(out_idx),
                             _ptr(out_vals) if with_values else None, _ptr(workspace), workspace.numel(),
                             _stream(stream))
    _lib.check("li_merge_shards", st)
    return (out_idx, out_vals) if with_values else out_idx


def li_absorb_query(q: torch.Tensor, w_dec: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """q bf16 [B,H,d], W_dec bf16 [H,d,dc] -> q~ bf16 [B,H,dc]."""
    _need(q, "q", torch.bfloat16)
    _need(w_dec, "w_dec", torch.bfloat16)
    B, H, d = q.shape
    dc = w_dec.shape[2]
    if out is None:
        out = torch.empty((B, H, dc), dtype=torch.bfloat16, device=q.device)
    st = _lib.load().li_absorb_query(_ptr(q), _ptr(w_dec), _ptr(out), B, H, d, dc, _stream(stream))
    _lib.check("li_absorb_query", st)
    return out


def li_absorb_query_layers(q: torch.Tensor, w_dec: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """q bf16 [G,B,H,d], W_dec bf16 [G,H,d,dc] -> q~ bf16 [G,B,H,dc], all G layers in one launch."""
    _need(q, "q", torch.bfloat16)
    _need(w_dec, "w_dec", torch.bfloat16)
    G, B, H, d = q.shape
    dc = w_dec.shape[3]
    if out is None:
        out = torch.empty((G, B, H, dc), dtype=torch.bfloat16, device=q.device)
    st = _lib.load().li_absorb_query_layers(_ptr(q), _ptr(w_dec), _ptr(out), G, B, H, d, dc, _stream(stream))
    _lib.check("li_absorb_query_layers", st)
    return out


def li_latent_score_hist(q_tilde: torch.Tensor, w: torch.Tensor, c: torch.Tensor, hist: torch.Tensor, *,
                         lens: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None, stream=None):
    """li_latent_score that also adds its scores' first-digit counts to `hist` (zeroed [B, 2048] uint32
    buffer, e.g. from li_decode_select_workspace) for li_topk_hist."""
    _need(q_tilde, "q_tilde", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(c, "c", torch.bfloat16)
    B, H, dc = q_tilde.shape
    L = c.shape[-2]
    batch_rows = c.shape[1] if c.dim() == 3 else 0
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if scores is None:
        scores = torch.empty((B, _round4(L)), dtype=torch.float32, device=c.device)
    st = _lib.load().li_latent_score_hist(_ptr(q_tilde), _ptr(w), _ptr(c), batch_rows, _ptr(lens), _ptr(scores),
                                          scores.stride(0), B, H, dc, L, _ptr(hist), _stream(stream))
    _lib.check("li_latent_score_hist", st)
    return scores


def li_latent_score_fp8(q_tilde: torch.Tensor, w: torch.Tensor, c8: torch.Tensor, c_scale: torch.Tensor, *,
                        lens: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                        hist: Optional[torch.Tensor] = None, stream=None):
    """Latent scan over an FP8 latent cache: q~ bf16 [B,64,192], w fp32 [B,64], c8 e4m3/uint8
    [B,L,192] (or shared [L,192]) with fp32 per-row scales -> scores fp32 [B, round4(L)].
    With `hist` (zeroed [B, 2048] buffer) the first-digit counts for li_topk_hist are added."""
    _need(q_tilde, "q_tilde", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(c8, "c8")
    _need(c_scale, "c_scale", torch.float32)
    if c8.dtype == torch.float8_e4m3fn:
        c8 = c8.view(torch.uint8)
    B, H, dc = q_tilde.shape
    L = c8.shape[-2]
    batch_rows = c8.shape[1] if c8.dim() == 3 else 0
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if scores is None:
        scores = torch.empty((B, _round4(L)), dtype=torch.float32, device=c8.device)
    st = _lib.load().li_latent_score_fp8(_ptr(q_tilde), _ptr(w), _ptr(c8), _ptr(c_scale), batch_rows, _ptr(lens),
                                         _ptr(scores), scores.stride(0), B, H, dc, L, _ptr(hist), _stream(stream))
    _lib.check("li_latent_score_fp8", st)
    return scores


def li_latent_score(q_tilde: torch.Tensor, w: torch.Tensor, c: torch.Tensor, *, lens: Optional[torch.Tensor] = None,
                    scores: Optional[torch.Tensor] = None, stream=None):
    """q~ bf16 [B,H,dc], w fp32 [B,H], c bf16 [B,L,dc] (or shared [L,dc]) -> scores fp32 [B, round4(L)]."""
    _need(q_tilde, "q_tilde", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(c, "c", torch.bfloat16)
    B, H, dc = q_tilde.shape
    L = c.shape[-2]
    batch_rows = c.shape[1] if c.dim() == 3 else 0
    if lens is not None:
        _need(lens, "lens", torch.int32)
    if scores is None:
        scores = torch.empty((B, _round4(L)), dtype=torch.float32, device=c.device)
    st = _lib.load().li_latent_score(_ptr(q_tilde), _ptr(w), _ptr(c), batch_rows, _ptr(lens), _ptr(scores),
                                     scores.stride(0), B, H, dc, L, _stream(stream))
    _lib.check("li_latent_score", st)
    return scores


def li_hs_refine_workspace(batch: int, n_cand: int, followers: int, device) -> torch.Tensor:
    """A zeroed workspace for li_hs_refine / li_hs_refine_fp8 (its histogram part stays zero between calls)."""
    need = _lib.load().li_hs_refine_workspace(int(batch), int(n_cand), int(followers))
    return torch.zeros(max(int(need), 16), dtype=torch.uint8, device=device)


def li_hs_refine(c: torch.Tensor, cand: torch.Tensor, q_tilde: torch.Tensor, w: torch.Tensor, k: int, *,
                 out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Followers re-score the anchor's candidates and keep their own top-k.

    c bf16 [B,L,dc] (or shared [L,dc]); cand int32 [B,C] ascending, -1 padding last;
    q~ bf16 [F,B,H,dc]; w fp32 [F,B,H] -> out int32 [F,B,k] cache positions.
    """
    _need(c, "c", torch.bfloat16)
    _need(cand, "cand", torch.int32)
    _need(q_tilde, "q_tilde", torch.bfloat16)
    _need(w, "w", torch.float32)
    F, B, H, dc = q_tilde.shape
    C = cand.shape[1]
    batch_rows = c.shape[1] if c.dim() == 3 else 0
    cache_rows = c.numel() // dc
    lib = _lib.load()
    need = lib.li_hs_refine_workspace(B, C, F)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = li_hs_refine_workspace(B, C, F, c.device)
    if out is None:
        out = torch.empty((F, B, k), dtype=torch.int32, device=c.device)
    st = lib.li_hs_refine(_ptr(c), batch_rows, cache_rows, _ptr(cand), B, C, _ptr(q_tilde), _ptr(w), F, H, dc, int(k),
                          _ptr(out), _ptr(workspace), need, _stream(stream))
    _lib.check("li_hs_refine", st)
    return out


def li_sparse_attention_workspace(batch: int, heads: int, k: int, device) -> torch.Tensor:
    need = _lib.load().li_sparse_attention_workspace(int(batch), int(heads), int(k))
    return torch.empty(max(int(need), 256), dtype=torch.uint8, device=device)


def li_sparse_attention(q: torch.Tensor, kv: torch.Tensor, sel: torch.Tensor, scale: float, *,
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Attention of each query head over the selected cache rows (absorbed-MLA decode form).

    q bf16 [B,H,576] (H a multiple of 64); kv bf16 [B,L,576] (or one shared [L,576]); sel int32 [B,k]
    cache rows, -1 = none -> out fp32 [B,H,512] = softmax(scale * q . kv[sel]) @ kv[sel, :512].
    """
    _need(q, "q", torch.bfloat16)
    _need(kv, "kv", torch.bfloat16)
    _need(sel, "sel", torch.int32)
    B, H, D = q.shape
    k = sel.shape[1]
    batch_rows = kv.shape[1] if kv.dim() == 3 else 0
    cache_rows = kv.shape[-2]
    if out is None:
        out = torch.empty((B, H, 512), dtype=torch.float32, device=q.device)
    lib = _lib.load()
    need = lib.li_sparse_attention_workspace(B, H, k)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = li_sparse_attention_workspace(B, H, k, q.device)
    st = lib.li_sparse_attention(_ptr(q), _ptr(kv), batch_rows, cache_rows, _ptr(sel), B, H, k, float(scale),
                                 _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _lib.check("li_sparse_attention", st)
    return out


def li_hs_refine_fp8(c8: torch.Tensor, c_scale: torch.Tensor, cand: torch.Tensor, q_tilde: torch.Tensor,
                     w: torch.Tensor, k: int, *, out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """li_hs_refine over the FP8 d_c = 192 latent: c8 e4m3/uint8 [B,L,192] (or shared [L,192]) with
    c_scale fp32 [B,L] (or [L]); cand int32 [B,C]; q~ bf16 [F,B,64,192]; w fp32 [F,B,64]
    -> out int32 [F,B,k] cache positions."""
    if c8.dtype == torch.float8_e4m3fn:
        c8 = c8.view(torch.uint8)
    _need(c8, "c8", torch.uint8)
    _need(c_scale, "c_scale", torch.float32)
    _need(cand, "cand", torch.int32)
    _need(q_tilde, "q_tilde", torch.bfloat16)
    _need(w, "w", torch.float32)
    F, B, H, dc = q_tilde.shape
    C = cand.shape[1]
    batch_rows = c8.shape[1] if c8.dim() == 3 else 0
    cache_rows = c8.numel() // dc
    lib = _lib.load()
    need = lib.li_hs_refine_workspace(B, C, F)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = li_hs_refine_workspace(B, C, F, c8.device)
    if out is None:
        out = torch.empty((F, B, k), dtype=torch.int32, device=c8.device)
    st = lib.li_hs_refine_fp8(_ptr(c8), _ptr(c_scale), batch_rows, cache_rows, _ptr(cand), B, C, _ptr(q_tilde),
                              _ptr(w), F, H, dc, int(k), _ptr(out), _ptr(workspace), need, _stream(stream))
    _lib.check("li_hs_refine_fp8", st)
    return out


def li_selftest_wait_timeout(limit_ns: int, stream=None):
    st = _lib.load().li_selftest_wait_timeout(int(limit_ns), _stream(stream))
    _lib.check("li_selftest_wait_timeout", st)
