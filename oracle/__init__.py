"""Lightning-indexer oracle: plain fp64 CPU definitions (ctypes wrapper over ``oracle.c``).

TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the CPU
baseline leg of the benchmark may import this package; the product path (the
CUDA library and its binding) never does, and shares no code with it.

Functions marked "parity unpinned" in their docstring have no independent pin;
every other function is checked against hand-computed values, library routines,
identities or invariants in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, E4M3, F64 = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-pthread", _SRC, "-o", _LIB, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_index_score.restype = ctypes.c_int
        L.orc_topk.restype = ctypes.c_int
        L.orc_hs_refine.restype = ctypes.c_int
        _lib = L
    return _lib


class _ScoreArgs(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("L", ctypes.c_int),
                ("q_dtype", ctypes.c_int), ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("w", ctypes.c_void_p),
                ("k_dtype", ctypes.c_int), ("k", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("k_batch_rows", ctypes.c_longlong), ("len", ctypes.c_void_p),
                ("causal", ctypes.c_int), ("causal_offset", ctypes.c_int)]


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _raw(x, dtype_tag):
    """Accept numpy arrays or torch tensors; bf16 / e4m3 come as their raw bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16).numpy().view(np.uint16)
            elif x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8).numpy()
            else:
                x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    want = {F32: np.float32, BF16: np.uint16, E4M3: np.uint8, F64: np.float64}[dtype_tag]
    return np.ascontiguousarray(x, dtype=want)


def nthreads_default() -> int:
    return max(1, os.cpu_count() or 1)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------
def e4m3_decode(b: int) -> float:
    return lib().orc_e4m3_decode(int(b))


def e4m3_encode(x: float) -> int:
    return int(lib().orc_e4m3_encode(float(x)))


def bf16_to_f32(b: int) -> float:
    return float(lib().orc_bf16_to_f32(int(b)))


# ---------------------------------------------------------------------------
# query quantisation
# ---------------------------------------------------------------------------
def quantize_query(q_bf16, w):
    """q [R, H, d] bf16, w [R, H] fp32 -> (q8 uint8 [R,H,d], sq fp32 [R,H], w_eff fp32 [R,H])."""
    q = _raw(q_bf16, BF16)
    R, H, d = q.shape
    w = _c(w if not hasattr(w, "numpy") else w.detach().cpu().numpy(), np.float32)
    q8 = np.empty((R, H, d), np.uint8)
    sq = np.empty((R, H), np.float32)
    we = np.empty((R, H), np.float32)
    lib().orc_quantize_query(_p(q), _p(w), R, H, d, _p(q8), _p(sq), _p(we))
    return q8, sq, we


# ---------------------------------------------------------------------------
# indexer score
# ---------------------------------------------------------------------------
def index_score(q, q_dtype, w, k, k_dtype, *, q_scale=None, k_scale=None, k_batch_rows=0,
                lens=None, L=None, causal=False, causal_offset=0, rows=None, with_mag=False,
                nthreads=None):
    """I[r, s] = sum_j w[r,j] * ReLU(q[r,j,:] . k[s,:]) in fp64.

    q: [R, H, d] (dtype tag F32/BF16/E4M3/F64) with optional q_scale [R, H];
    k: key rows of d elements with optional per-row k_scale; request r's cache
    starts at row r * k_batch_rows (0 = one shared cache).  Positions that row r
    may not see hold -inf.  Returns out [n_rows, L] (and mag, the sum of
    |w_j| * |q_j . k_s|, when ``with_mag``).
    """
    qa = _raw(q, q_dtype)
    R, H, d = qa.shape
    ka = _raw(k, k_dtype)
    wa = _raw(w, F32).reshape(R, H)
    qs = None if q_scale is None else _raw(q_scale, F32)
    ks = None if k_scale is None else _raw(k_scale, F32)
    ln = None if lens is None else _c(np.asarray(lens), np.int32)
    if L is None:
        L = ka.reshape(-1, d).shape[0] if k_batch_rows == 0 else int(k_batch_rows)
    args = _ScoreArgs(R, H, d, int(L), q_dtype, _p(qa), _p(qs), _p(wa), k_dtype, _p(ka), _p(ks),
                      int(k_batch_rows), _p(ln), int(bool(causal)), int(causal_offset))
    rows_a = None if rows is None else _c(np.asarray(rows), np.int32)
    n_rows = R if rows_a is None else len(rows_a)
    out = np.empty((n_rows, int(L)), np.float64)
    mag = np.empty((n_rows, int(L)), np.float64) if with_mag else None
    lib().orc_index_score(ctypes.byref(args), _p(rows_a), n_rows, _p(out), _p(mag),
                          nthreads or nthreads_default())
    return (out, mag) if with_mag else out


# ---------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------
def topk(scores, k, lens=None, causal=False, causal_offset=0, max_len=None):
    """Per row: the k largest of the first len[r] scores (ties -> lower position,
    NaN lowest), reported in ascending position order and padded with -1.
    Returns (idx int32 [rows, k], vals fp64 [rows, k], pads -inf)."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    if s.ndim == 1:
        s = s[None]
    rows, ld = s.shape
    if max_len is None:
        max_len = ld
    ln = None if lens is None else _c(np.asarray(lens), np.int32)
    idx = np.empty((rows, k), np.int32)
    vals = np.empty((rows, k), np.float64)
    lib().orc_topk(_p(s), ctypes.c_longlong(ld), _p(ln), rows, int(max_len), int(bool(causal)),
                   int(causal_offset), int(k), _p(idx), _p(vals))
    return idx, vals


# ---------------------------------------------------------------------------
# LatentIndex
# ---------------------------------------------------------------------------
def absorb(q_bf16, wdec_bf16):
    """q~[b,j,:] = W_dec[j]^T q[b,j,:] in fp64.  q [B,H,d], W_dec [H,d,dc] -> [B,H,dc]."""
    q = _raw(q_bf16, BF16)
    W = _raw(wdec_bf16, BF16)
    B, H, d = q.shape
    dc = W.shape[2]
    out = np.empty((B, H, dc), np.float64)
    lib().orc_absorb(_p(q), _p(W), B, H, d, dc, _p(out))
    return out


def decode_keys(wdec_bf16, crow_bf16):
    """Per-head keys of one latent row, k[j,:] = W_dec[j] c.  -> [H, d]."""
    W = _raw(wdec_bf16, BF16)
    c = _raw(crow_bf16, BF16)
    H, d, dc = W.shape
    out = np.empty((H, d), np.float64)
    lib().orc_decode_keys(_p(W), _p(c), H, d, dc, _p(out))
    return out


def latent_score_rebuilt(q_bf16, w, wdec_bf16, c_bf16, b, positions, c_batch_rows=None):
    """Scores of request b at the given latent rows via explicitly rebuilt per-layer keys."""
    q = _raw(q_bf16, BF16)
    W = _raw(wdec_bf16, BF16)
    c = _raw(c_bf16, BF16)
    wa = _raw(w, F32)
    B, H, d = q.shape
    dc = W.shape[2]
    if c_batch_rows is None:
        c_batch_rows = c.shape[1] if c.ndim == 3 else 0
    pos = _c(np.asarray(positions), np.int32)
    out = np.empty(len(pos), np.float64)
    lib().orc_latent_score_rebuilt(_p(q), _p(wa), _p(W), _p(c), ctypes.c_longlong(c_batch_rows), int(b),
                                   H, d, dc, _p(pos), len(pos), _p(out))
    return out


def latent_score(qt, qt_dtype, w, c_bf16, *, lens=None, c_batch_rows=None, rows=None, with_mag=False,
                 nthreads=None):
    """I[b, s] = sum_j w[b,j] * ReLU(q~[b,j,:] . c[b,s,:]) in fp64 (the DSA score on latent rows)."""
    c = _raw(c_bf16, BF16)
    if c_batch_rows is None:
        c_batch_rows = c.shape[1] if c.ndim == 3 else 0
    L = c.shape[-2]
    return index_score(qt, qt_dtype, w, c, BF16, k_batch_rows=c_batch_rows, lens=lens, L=L, rows=rows,
                       with_mag=with_mag, nthreads=nthreads)


def hs_refine(qt, qt_dtype, w, c_bf16, cand, k, *, c_batch_rows=None, nthreads=None, with_scores=False):
    """Followers re-score the anchor's candidates and keep their own top-k.

    qt [F,B,H,dc], w [F,B,H], c [B,L,dc] (or a shared [L,dc]), cand int [B,C]
    (negative = padding) -> out int32 [F,B,k] cache positions, ascending, -1 pads.
    """
    q = _raw(qt, qt_dtype)
    F, B, H, dc = q.shape
    wa = _raw(w, F32)
    c = _raw(c_bf16, BF16)
    if c_batch_rows is None:
        c_batch_rows = c.shape[1] if c.ndim == 3 else 0
    cd = _c(np.asarray(cand), np.int32)
    C = cd.shape[1]
    out = np.empty((F, B, k), np.int32)
    cs = np.empty((F, B, C), np.float64) if with_scores else None
    lib().orc_hs_refine(qt_dtype, _p(q), _p(wa), _p(c), ctypes.c_longlong(c_batch_rows), _p(cd), F, B, H, dc,
                        C, int(k), _p(out), _p(cs), nthreads or nthreads_default())
    return (out, cs) if with_scores else out


# ---------------------------------------------------------------------------
# the consumer: sparse attention over a selection
# ---------------------------------------------------------------------------
def _bf16_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sparse_attention(q_bf16, kv_bf16, sel, scale, *, dv=512, with_mag=False):
    """Each query head's attention over the selected cache rows, in fp64.

    Multi-layer Indexer (long-version transcript): a DSA layer attends, for each
    new token, only the positions its indexer selected.  Reading of the shape
    (the pages give none): DeepSeek-V3.2's absorbed-MLA decode form, where one
    cache row per position is the key and its first ``dv`` elements the value.

        o[b,h,:] = sum_i p_i kv[b, s_i, :dv],
        p = softmax over i of scale * (q[b,h,:] . kv[b, s_i, :])

    over the valid selections s_i (0 <= s_i < cache rows; duplicates count
    once per listing); a request without any gets o = 0.
    q [B,H,D] bf16; kv [B,L,D] bf16 (or one shared [L,D]); sel int [B,k].
    Returns o [B,H,dv] (and mag = sum_i p_i |kv[b,s_i,:dv]|, the scale of each
    output's sum, when ``with_mag``).  Matrix products and exp are numpy's.
    """
    q = _bf16_f64(_raw(q_bf16, BF16))
    kv = _bf16_f64(_raw(kv_bf16, BF16))
    sel = np.asarray(sel)
    B, H, D = q.shape
    out = np.zeros((B, H, dv))
    mag = np.zeros((B, H, dv))
    for b in range(B):
        cache = kv[b] if kv.ndim == 3 else kv
        s = sel[b]
        s = s[(s >= 0) & (s < cache.shape[0])]
        if s.size == 0:
            continue
        keys = cache[s]                              # [n, D]
        logits = scale * (q[b] @ keys.T)             # [H, n]
        logits = logits - logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p = p / p.sum(axis=1, keepdims=True)         # softmax over the selected positions
        out[b] = p @ keys[:, :dv]
        mag[b] = p @ np.abs(keys[:, :dv])
    return (out, mag) if with_mag else out


def hs_refine_fp8(qt_bf16, w, c_e4m3, c_scale, cand, k, *, with_scores=False):
    """Followers re-score the anchor's candidates over an FP8 latent (e4m3 rows with one scale per row,
    DeepSeek-V3.2's d_c = 192 layout) and keep their own top-k: LatentIndex abstract (followers refine
    the anchor's candidate set), with each follower's absorbed query quantised per (follower, request,
    head) as quantize_query does.  A composition of quantize_query, index_score (e4m3 keys with row
    scales) and topk; ties go to the lower cache position (candidates are listed in position order).

    qt [F,B,H,dc] bf16, w [F,B,H], c_e4m3 [B,L,dc] bytes (or shared [L,dc]), c_scale [B,L] (or [L]),
    cand int [B,C] (negative = padding) -> out int32 [F,B,k] cache positions ascending, -1 pads
    (and the candidate scores [F,B,C], -inf for padding, with ``with_scores``).
    """
    F, B, H, dc = tuple(qt_bf16.shape)
    c8 = _raw(c_e4m3, E4M3)
    cs = _raw(c_scale, F32)
    cd = np.asarray(cand)
    C = cd.shape[1]
    out = np.full((F, B, k), -1, np.int32)
    scores = np.full((F, B, C), -np.inf)
    for f in range(F):
        q8, sq, _ = quantize_query(qt_bf16[f], np.asarray(w[f] if not hasattr(w, "numpy") else w[f].numpy()))
        for b in range(B):
            rows8 = c8[b] if c8.ndim == 3 else c8
            rs = cs[b] if cs.ndim == 2 else cs
            valid = np.nonzero(cd[b] >= 0)[0]
            if valid.size == 0:
                continue
            pos = cd[b, valid]
            wf = np.asarray(w[f, b] if not hasattr(w, "numpy") else w[f, b].numpy(), np.float32)[None]
            s = index_score(q8[b:b + 1], E4M3, wf, rows8[pos], E4M3, q_scale=sq[b:b + 1], k_scale=rs[pos])[0]
            scores[f, b, valid] = s
            kk = min(k, valid.size)
            sel, _ = topk(s[None], kk)
            chosen = np.sort(pos[sel[0][sel[0] >= 0]])
            out[f, b, :chosen.size] = chosen
    return (out, scores) if with_scores else out
