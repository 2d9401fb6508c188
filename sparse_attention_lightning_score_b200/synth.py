"""Seeded synthetic inputs for the lightning-indexer path.

This module is the only code that the fp64 oracle (``oracle/``) and the CUDA
path share: both consume the tensors it returns.  It draws random numbers and
lays them out in the storage formats the indexer reads.  It computes no
indexer score, no top-k selection, no query quantisation and no decoder
absorption.

Workload shapes follow the lightning-indexer settings of the pages:

* DSA decode -- one query token per request scans its whole cache and keeps
  k=2048 positions (Multi-layer Indexer abstract; IndexCache explainer,
  "Symbol Map", k = 2,048).
* DSA causal prefill -- every query token scans its prefix (IndexCache
  explainer, "Why This Exists").
* LatentIndex -- one latent cache shared by a G=4 layer group, per-layer key
  decoders, hierarchical selection (LatentIndex abstract and Figure 1).

Random draws use ``torch.Generator(device).manual_seed(seed)`` in a fixed
order that each function documents.  The FP8 key cache is produced with
torch's own ``float8_e4m3fn`` cast after a per-token absmax scale (the cache
storage format the indexer is given, not a step of the scan).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

E4M3_MAX = 448.0


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(g: torch.Generator, *shape, device: str = "cpu") -> torch.Tensor:
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)


def encode_e4m3_cache(k: torch.Tensor):
    """Store fp32 keys ``[..., d]`` as an e4m3 cache with one fp32 scale per token.

    scale = absmax(k[token, :]) / 448 (1 when the row is all zero); the bytes are
    torch's ``float8_e4m3fn`` cast of ``k / scale`` (clamped to +-448).  Returns
    ``(uint8 [..., d], fp32 [...])``.
    """
    absmax = k.abs().amax(dim=-1)
    scale = torch.where(absmax > 0, absmax / E4M3_MAX, torch.ones_like(absmax))
    y = (k / scale.unsqueeze(-1)).clamp_(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale.contiguous()


# --------------------------------------------------------------------------
# Tiny fp32 case
# --------------------------------------------------------------------------
@dataclass
class TinyFp32:
    q: torch.Tensor        # fp32 [1, H, d]
    k: torch.Tensor        # fp32 [L, d]
    w: torch.Tensor        # fp32 [1, H]
    planted: torch.Tensor  # int64 [n_plant]
    k_top: int


def tiny_fp32(H: int = 4, d: int = 32, L: int = 1024, n_plant: int = 8, k_top: int = 64,
              seed: int = 0, device: str = "cpu") -> TinyFp32:
    """One fp32 query, H heads, cache of L keys; draws q, k, w, planted positions.

    q, k ~ N(0,1); w ~ U(0,1).  ``n_plant`` distinct positions get the key
    3 * mean_j q[0, j, :] so that the top-k is not a coin toss.
    """
    g = _gen(seed, device)
    q = _randn(g, 1, H, d, device=device)
    k = _randn(g, L, d, device=device)
    w = torch.rand(1, H, generator=g, device=device, dtype=torch.float32)
    planted = torch.randperm(L, generator=g, device=device)[:n_plant]
    k[planted] = 3.0 * q[0].mean(dim=0)
    return TinyFp32(q=q, k=k, w=w, planted=planted, k_top=k_top)


# --------------------------------------------------------------------------
# DSA decode: B requests, each with its own FP8 key cache
# --------------------------------------------------------------------------
@dataclass
class DsaDecode:
    q: torch.Tensor        # bf16 [B, H, d]   indexer queries (one decode token per request)
    w: torch.Tensor        # fp32 [B, H]      per-head weights
    k8: torch.Tensor       # uint8 [B, L, d]  e4m3 key cache bytes
    ks: torch.Tensor       # fp32 [B, L]      per-token key scale
    lens: torch.Tensor     # int32 [B]        visible cache length per request
    planted: torch.Tensor  # int64 [B, n_plant]
    k_top: int


def dsa_decode(B: int = 8, L: int = 32768, H: int = 64, d: int = 128, k_top: int = 2048,
               plant_frac: float = 0.01, seed: int = 1, lens: Optional[list] = None,
               device: str = "cpu") -> DsaDecode:
    """Draw order: q, k, w, then per request the planted positions.

    q ~ N(0,1) rounded to bf16; k ~ N(0,1); w ~ N(0, 0.1^2).  In every request a
    fraction ``plant_frac`` of the positions gets the key 4*sqrt(d)*u_b, where u_b
    is the unit vector along the mean over heads of that request's query.  The
    keys are then stored as an e4m3 cache with per-token scales.
    """
    g = _gen(seed, device)
    q = _randn(g, B, H, d, device=device).to(torch.bfloat16)
    k = _randn(g, B, L, d, device=device)
    w = _randn(g, B, H, device=device) * 0.1
    n_plant = int(round(plant_frac * L))
    planted = torch.empty(B, n_plant, dtype=torch.int64, device=device)
    for b in range(B):
        planted[b] = torch.randperm(L, generator=g, device=device)[:n_plant]
        qbar = q[b].float().mean(dim=0)
        u = qbar / qbar.norm()
        k[b, planted[b]] = 4.0 * math.sqrt(d) * u
    k8, ks = encode_e4m3_cache(k)
    del k
    if lens is None:
        lens_t = torch.full((B,), L, dtype=torch.int32, device=device)
    else:
        lens_t = torch.tensor(lens, dtype=torch.int32, device=device)
    return DsaDecode(q=q, w=w, k8=k8, ks=ks, lens=lens_t, planted=planted, k_top=k_top)


# --------------------------------------------------------------------------
# DSA causal prefill: T query tokens over their own prefix of one FP8 cache
# --------------------------------------------------------------------------
@dataclass
class DsaPrefill:
    q: torch.Tensor    # bf16 [T, H, d]
    w: torch.Tensor    # fp32 [T, H]
    k8: torch.Tensor   # uint8 [L, d]
    ks: torch.Tensor   # fp32 [L]
    k_top: int


def dsa_prefill(T: int = 8192, L: int = 8192, H: int = 64, d: int = 128, k_top: int = 2048,
                drift: float = 0.02, seed: int = 2, device: str = "cpu") -> DsaPrefill:
    """Draw order: drift steps, q noise, k noise, w.

    A random walk m[0] = 0, m[s] = m[s-1] + drift * N(0, I_d) is added to both the
    query of token t (m[t]) and the key of position s (m[s]), so nearby tokens
    share a direction ("smooth random-walk drift to induce locality").  Query
    token t sits at cache position t.
    """
    assert T <= L
    g = _gen(seed, device)
    steps = _randn(g, L, d, device=device) * drift
    steps[0].zero_()
    m = torch.cumsum(steps, dim=0)
    q = (_randn(g, T, H, d, device=device) + m[:T].unsqueeze(1)).to(torch.bfloat16)
    k = _randn(g, L, d, device=device) + m
    w = _randn(g, T, H, device=device) * 0.1
    k8, ks = encode_e4m3_cache(k)
    return DsaPrefill(q=q, w=w, k8=k8, ks=ks, k_top=k_top)


# --------------------------------------------------------------------------
# LatentIndex: one latent cache per request shared by a G-layer group
# --------------------------------------------------------------------------
@dataclass
class LatentGroup:
    c: torch.Tensor        # bf16 [B, L, dc]     shared latent cache
    w_dec: torch.Tensor    # bf16 [G, H, d, dc]  per-layer key decoders
    q: torch.Tensor        # bf16 [G, B, H, d]   per-layer indexer queries
    w: torch.Tensor        # fp32 [G, B, H]      per-layer head weights
    lens: torch.Tensor     # int32 [B]
    planted: Optional[torch.Tensor] = None  # int64 [B, n_plant]
    k_top: int = 2048
    n_cand: int = 0


def latent_group(B: int = 4, L: int = 65536, H: int = 64, d: int = 128, dc: int = 256,
                 G: int = 4, k_top: int = 2048, seed: int = 3, plant_frac: float = 0.0,
                 n_cand: int = 0, lens: Optional[list] = None, device: str = "cpu") -> LatentGroup:
    """Draw order: c (request by request), W_dec, q, w, then planted rows.

    c ~ N(0,1) and q ~ N(0,1) rounded to bf16; W_dec ~ N(0, (1/sqrt(dc))^2) rounded
    to bf16 (so a decoded key has unit variance per component); w ~ N(0, 0.1^2).
    With ``plant_frac`` > 0, every request draws a unit direction u_b and that
    fraction of its rows is replaced by 4*sqrt(dc)*u_b: a group of strongly
    aligned tokens with four times the typical norm.
    """
    g = _gen(seed, device)
    c = torch.empty(B, L, dc, dtype=torch.bfloat16, device=device)
    for b in range(B):
        c[b] = _randn(g, L, dc, device=device).to(torch.bfloat16)
    w_dec = (_randn(g, G, H, d, dc, device=device) / math.sqrt(dc)).to(torch.bfloat16)
    q = _randn(g, G, B, H, d, device=device).to(torch.bfloat16)
    w = _randn(g, G, B, H, device=device) * 0.1
    planted = None
    n_plant = int(round(plant_frac * L))
    if n_plant > 0:
        planted = torch.empty(B, n_plant, dtype=torch.int64, device=device)
        for b in range(B):
            u = _randn(g, dc, device=device)
            u = u / u.norm()
            planted[b] = torch.randperm(L, generator=g, device=device)[:n_plant]
            c[b, planted[b]] = (4.0 * math.sqrt(dc) * u).to(torch.bfloat16)
    if lens is None:
        lens_t = torch.full((B,), L, dtype=torch.int32, device=device)
    else:
        lens_t = torch.tensor(lens, dtype=torch.int32, device=device)
    return LatentGroup(c=c, w_dec=w_dec, q=q, w=w, lens=lens_t, planted=planted,
                       k_top=k_top, n_cand=n_cand)


def latent_hs(B: int = 1, L: int = 131072, H: int = 64, d: int = 128, dc: int = 256,
              F: int = 3, n_cand: int = 8192, k_top: int = 2048, plant_frac: float = 0.005,
              seed: int = 4, lens: Optional[list] = None, device: str = "cpu") -> LatentGroup:
    """Hierarchical-selection workload: layer 0 is the anchor, layers 1..F follow."""
    return latent_group(B=B, L=L, H=H, d=d, dc=dc, G=1 + F, k_top=k_top, seed=seed,
                        plant_frac=plant_frac, n_cand=n_cand, lens=lens, device=device)


# --------------------------------------------------------------------------
# LatentIndex with DeepSeek-V3.2's latent layout and an FP8 latent cache
# --------------------------------------------------------------------------
@dataclass
class LatentFp8:
    c: torch.Tensor        # bf16 [B, L, 192]    latent rows before FP8 storage
    c8: torch.Tensor       # uint8 [B, L, 192]   e4m3 bytes of the cache
    cs: torch.Tensor       # fp32 [B, L]         per-row scales
    w_dec: torch.Tensor    # bf16 [G, H, 128, 192] per-layer key decoders
    q: torch.Tensor        # bf16 [G, B, H, 128] per-layer indexer queries
    w: torch.Tensor        # fp32 [G, B, H]
    lens: torch.Tensor     # int32 [B]
    k_top: int = 2048


def latent_rope_nope(B: int = 4, L: int = 65536, H: int = 64, G: int = 4, k_top: int = 2048, seed: int = 5,
                     lens: Optional[list] = None, device: str = "cpu") -> LatentFp8:
    """Shared latent of 64 RoPE + 128 NoPE dimensions for 128-wide indexer keys of
    64 RoPE + 64 NoPE dimensions (DeepSeek-V3.2's sizes, LatentIndex appendix,
    Table 5), stored as an e4m3 cache with per-row scales.

    Draw order: c (request by request), the NoPE decoders, q, w.  c ~ N(0,1) and
    q ~ N(0,1) rounded to bf16; w ~ N(0, 0.1^2).  Each layer's decoder copies
    the 64 RoPE latent dimensions to the key's 64 RoPE dimensions unchanged and
    maps the 128 NoPE latent dimensions to the key's 64 NoPE dimensions with a
    random matrix ~ N(0, (1/sqrt(128))^2) rounded to bf16.
    """
    g = _gen(seed, device)
    c = torch.empty(B, L, 192, dtype=torch.bfloat16, device=device)
    for b in range(B):
        c[b] = _randn(g, L, 192, device=device).to(torch.bfloat16)
    nope = (_randn(g, G, H, 64, 128, device=device) / math.sqrt(128)).to(torch.bfloat16)
    w_dec = torch.zeros(G, H, 128, 192, dtype=torch.bfloat16, device=device)
    w_dec[:, :, torch.arange(64), torch.arange(64)] = 1.0
    w_dec[:, :, 64:, 64:] = nope
    q = _randn(g, G, B, H, 128, device=device).to(torch.bfloat16)
    w = _randn(g, G, B, H, device=device) * 0.1
    c8, cs = encode_e4m3_cache(c.float())
    if lens is None:
        lens_t = torch.full((B,), L, dtype=torch.int32, device=device)
    else:
        lens_t = torch.tensor(lens, dtype=torch.int32, device=device)
    return LatentFp8(c=c, c8=c8, cs=cs, w_dec=w_dec, q=q, w=w, lens=lens_t, k_top=k_top)


# --------------------------------------------------------------------------
# Plain score rows for the top-k select alone
# --------------------------------------------------------------------------
def score_rows(rows: int, L: int, seed: int = 5, ties: int = 0, device: str = "cpu") -> torch.Tensor:
    """fp32 [rows, L] ~ N(0,1); with ``ties`` > 0 values are drawn from only
    ``ties`` distinct levels so that many entries tie exactly."""
    g = _gen(seed, device)
    if ties > 0:
        lv = _randn(g, ties, device=device)
        ix = torch.randint(0, ties, (rows, L), generator=g, device=device)
        return lv[ix].contiguous()
    return _randn(g, rows, L, device=device)


# --------------------------------------------------------------------------
# Named workloads (sizes as quoted for the indexer benchmarks)
# --------------------------------------------------------------------------
WORKLOADS = {
    "tiny_fp32": dict(kind="tiny"),
    "dsa_decode_b8_l32k": dict(kind="decode", B=8, L=32768),
    "dsa_prefill_t8k": dict(kind="prefill", T=8192, L=8192),
    "latent_g4_b4_l64k": dict(kind="latent", B=4, L=65536),
    "latent_hs_b1_l128k": dict(kind="hs", B=1, L=131072),
    "latent_hs_b16_l128k": dict(kind="hs", B=16, L=131072),
}
