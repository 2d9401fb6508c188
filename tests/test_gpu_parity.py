"""GPU parity: every CUDA path against the fp64 oracle on the same seeded inputs.

Integer work (quantised bytes, top-k indices on identical fp32 inputs, HS
gathers) must match bit for bit; floating-point scores must match within the
tolerance of tests/_checks.py.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_lightning_score_b200 import api, synth
from sparse_attention_lightning_score_b200._lib import LI_ERR_BOUNDS, LI_ERR_TIMEOUT, LI_OK, LiError
from tests._checks import assert_scores_close, assert_topk_equivalent

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _np(t):
    return t.detach().cpu().numpy()


# ---------------------------------------------------------------------------
# query quantisation: bit-exact bytes, scales and folded weights
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("R,H,d", [(8, 64, 128), (3, 5, 96), (1, 64, 128)])
def test_quantize_query_bit_exact(R, H, d):
    g = torch.Generator().manual_seed(R * 100 + d)
    q = (torch.randn(R, H, d, generator=g) * torch.exp(torch.randn(R, H, 1, generator=g) * 3)).to(torch.bfloat16)
    q[0, 0] = 0.0                      # all-zero head
    q[0, 1 % H, :4] = torch.tensor([1.0, -2.0, 0.5, 4.0])
    q[-1, -1] *= 1e-30                 # tiny values (bf16 keeps the exponent range)
    w = torch.randn(R, H, generator=g)
    q8_o, sq_o, we_o = oracle.quantize_query(q, w.numpy())
    q8, sq, we = api.li_quantize_query(q.to(DEV), w.to(DEV))
    assert np.array_equal(_np(q8), q8_o)
    assert np.array_equal(_np(sq).view(np.uint32), sq_o.view(np.uint32))
    assert np.array_equal(_np(we).view(np.uint32), we_o.view(np.uint32))


def _near_midpoint_heads(n_heads, seed):
    """bf16 heads [n_heads, 128] whose quotients x / (absmax / 448) land within 8 fp32 ulps of an e4m3
    rounding midpoint (exact ties included): the hard cases of the quantiser's rounding.  Found by
    brute force over bf16 pairs with numpy's IEEE fp32 division."""
    A = ((np.arange(0x3d80, 0x4180, dtype=np.uint32) << 16).view(np.float32))
    X = ((np.arange(0x3980, 0x4180, dtype=np.uint32) << 16).view(np.float32))
    pairs = {}
    for a in A:
        sq = np.float32(a) / np.float32(448.0)
        xs = X[X <= a]
        qv = xs / sq
        m = qv.view(np.uint32) & 0xFFFFF
        near = (np.abs(m.astype(np.int64) - 0x80000) <= 8) & (qv >= 2.0 ** -6) & (qv <= 448)
        if near.any():
            pairs[float(a)] = xs[near]
    rng = np.random.default_rng(seed)
    keys = sorted(pairs)
    heads = np.empty((n_heads, 128), np.float32)
    for h in range(n_heads):
        a = keys[rng.integers(len(keys))]
        xs = pairs[a]
        row = rng.choice(xs, 127) * rng.choice([-1.0, 1.0], 127).astype(np.float32)
        heads[h, 0] = a * rng.choice([-1.0, 1.0])
        heads[h, 1:] = row
        rng.shuffle(heads[h])
    return torch.from_numpy(heads).to(torch.bfloat16)


def test_quantize_query_near_rounding_midpoints():
    q = _near_midpoint_heads(4 * 64, seed=3).view(4, 64, 128)
    w = torch.randn(4, 64, generator=torch.Generator().manual_seed(3))
    q8_o, sq_o, we_o = oracle.quantize_query(q, w.numpy())
    q8, sq, we = api.li_quantize_query(q.to(DEV), w.to(DEV))
    assert np.array_equal(_np(q8), q8_o)
    assert np.array_equal(_np(sq).view(np.uint32), sq_o.view(np.uint32))
    # the decode scorer quantises in its prologue: same bytes, so the same scores as the
    # oracle's quantised query within the FP8 tolerance
    k = torch.randn(4, 300, 128, generator=torch.Generator().manual_seed(4))
    k8, ks = synth.encode_e4m3_cache(k)
    ref, mag = oracle.index_score(q8_o, oracle.E4M3, w, k8, oracle.E4M3, q_scale=sq_o, k_scale=ks,
                                  k_batch_rows=300, L=300, with_mag=True)
    sc = api.li_index_score(q.to(DEV), w.to(DEV), k8.to(DEV), ks.to(DEV))
    assert_scores_close(_np(sc)[:, :300], ref, mag, 1e-2)


def _sweep_heads(absmax_bits):
    """Heads of 128 bf16 values: per absmax A, element 0 of every head is +-A and the other 127 run
    through every bf16 value x with |x| <= A, both signs (NaN excluded)."""
    heads = []
    for ab in absmax_bits:
        a = np.array([ab << 16], np.uint32).view(np.float32)[0]
        mags = (np.arange(0, ab + 1, dtype=np.uint32) << 16).view(np.float32)
        vals = np.concatenate([mags, -mags])
        n = -(-vals.size // 127)
        vals = np.concatenate([vals, np.zeros(n * 127 - vals.size, np.float32)]).reshape(n, 127)
        first = np.where(np.arange(n) % 2 == 0, a, -a).astype(np.float32)[:, None]
        heads.append(np.concatenate([first, vals], axis=1))
    h = np.concatenate(heads)
    pad = -h.shape[0] % 64
    h = np.concatenate([h, np.zeros((pad, 128), np.float32)])
    return torch.from_numpy(h).view(-1, 64, 128).to(torch.bfloat16)


@pytest.mark.parametrize("absmax_bits", [
    [0x0b00, 0x1e40, 0x2d07, 0x3a91, 0x3f80, 0x3fe0, 0x40a5, 0x4122, 0x43e0, 0x4661],
    [0x0080, 0x0100, 0x0d80, 0x3c00, 0x4000, 0x42f3, 0x5555, 0x6a00, 0x7f00, 0x7f7f],
])
def test_quantize_query_every_bf16_below_absmax(absmax_bits):
    # the quantiser's division-free rounding decision against the oracle's IEEE division for every bf16
    # input below each absmax: subnormal scales, tiny and huge absmax, exact e4m3 rounding midpoints
    q = _sweep_heads(absmax_bits)
    w = torch.randn(q.shape[:2], generator=torch.Generator().manual_seed(7))
    q8_o, sq_o, we_o = oracle.quantize_query(q, w.numpy())
    q8, sq, we = api.li_quantize_query(q.to(DEV), w.to(DEV))
    assert np.array_equal(_np(q8), q8_o)
    assert np.array_equal(_np(sq).view(np.uint32), sq_o.view(np.uint32))
    assert np.array_equal(_np(we).view(np.uint32), we_o.view(np.uint32))


# ---------------------------------------------------------------------------
# tiny fp32 case: exact scalar path, tolerance 1e-4
# ---------------------------------------------------------------------------
def test_tiny_fp32_score_and_topk():
    case = synth.tiny_fp32()
    ref, mag = oracle.index_score(case.q, oracle.F32, case.w, case.k, oracle.F32, with_mag=True)
    sc = api.li_index_score(case.q.to(DEV), case.w.to(DEV), case.k.to(DEV))
    L = case.k.shape[0]
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-4)
    idx = api.li_topk(sc, case.k_top, max_len=L)
    ridx, _ = oracle.topk(ref, case.k_top)
    assert_topk_equivalent(_np(idx), ridx, ref, 1e-4)
    assert set(case.planted.tolist()) <= set(_np(idx)[0].tolist())


# ---------------------------------------------------------------------------
# DSA decode scorer (FP8, tcgen05)
# ---------------------------------------------------------------------------
def _oracle_decode(case, rows=None):
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    L = case.k8.shape[1]
    return oracle.index_score(q8, oracle.E4M3, case.w, case.k8, oracle.E4M3, q_scale=sq, k_scale=case.ks,
                              k_batch_rows=L, L=L, lens=case.lens.numpy(), rows=rows, with_mag=True)


@pytest.mark.parametrize("B,L,lens", [(3, 1000, [1000, 517, 129]), (2, 4096, None), (5, 300, [0, 1, 127, 128, 300])])
def test_dsa_decode_scores(B, L, lens):
    case = synth.dsa_decode(B=B, L=L, seed=21, lens=lens)
    ref, mag = _oracle_decode(case)
    sc = api.li_index_score(case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV),
                            lens=case.lens.to(DEV))
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-2)
    assert api.li_get_last_error() == LI_OK


def test_dsa_decode_shared_cache():
    case = synth.dsa_decode(B=4, L=777, seed=22)
    k8, ks = case.k8[0], case.ks[0]
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    ref, mag = oracle.index_score(q8, oracle.E4M3, case.w, k8, oracle.E4M3, q_scale=sq, k_scale=ks, with_mag=True)
    sc = api.li_index_score(case.q.to(DEV), case.w.to(DEV), k8.to(DEV), ks.to(DEV))
    assert_scores_close(_np(sc)[:, :777], ref, mag, 1e-2)


def test_dsa_decode_bench_config_full():
    """The benchmarked decode step at full size (B=8, L=32768): every score and
    every top-2048 selection against the oracle."""
    case = synth.dsa_decode()  # B=8, L=32768, k=2048
    ref, mag = _oracle_decode(case)
    q, w, k8, ks = case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV)
    sc = api.li_index_score(q, w, k8, ks)
    assert_scores_close(_np(sc)[:, :32768], ref, mag, 1e-2)
    idx = api.li_topk(sc, 2048, max_len=32768)
    ridx, _ = oracle.topk(ref, 2048)
    assert_topk_equivalent(_np(idx), ridx, ref, 1e-2)
    assert api.li_get_last_error() == LI_OK


# ---------------------------------------------------------------------------
# top-k: bit-exact against the oracle on identical fp32 rows
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("rows,L,k,ties", [(8, 32768, 2048, 0), (1, 131072, 8192, 0), (16, 131072, 2048, 0),
                                           (3, 5000, 100, 7), (200, 3000, 64, 0), (2, 262144, 2048, 3),
                                           (4, 4096, 4096, 0), (6, 100, 2048, 0), (1, 9, 3, 2)])
def test_topk_bit_exact(rows, L, k, ties):
    s = synth.score_rows(rows, L, seed=rows + L + k, ties=ties)
    ld = (L + 3) // 4 * 4
    buf = torch.full((rows, ld), float("nan"))
    buf[:, :L] = s
    idx, vals = api.li_topk(buf.to(DEV), k, max_len=L, with_values=True)
    ridx, rvals = oracle.topk(s.double().numpy(), k)
    assert np.array_equal(_np(idx), ridx)
    assert np.array_equal(_np(vals).astype(np.float64), rvals)


def test_topk_ragged_and_causal_rows():
    rows, L, k = 300, 2500, 256
    s = synth.score_rows(rows, L, seed=31)
    lens = torch.randint(0, L + 1, (rows,), generator=torch.Generator().manual_seed(3), dtype=torch.int32)
    lens[:4] = torch.tensor([0, 1, k, k + 1], dtype=torch.int32)
    sd = s.to(DEV)
    idx = api.li_topk(sd, k, lens=lens.to(DEV), max_len=L)
    ridx, _ = oracle.topk(s.double().numpy(), k, lens=lens.numpy())
    assert np.array_equal(_np(idx), ridx)
    idx = api.li_topk(sd, k, causal=True, causal_offset=5, max_len=L)
    ridx, _ = oracle.topk(s.double().numpy(), k, causal=True, causal_offset=5, max_len=L)
    assert np.array_equal(_np(idx), ridx)


def test_topk_special_values():
    row = torch.tensor([[float("nan"), -0.0, 0.0, float("-inf"), 1.0, float("nan"), 0.0, -0.0]])
    for k in (1, 2, 3, 5, 7):
        idx = api.li_topk(row.to(DEV), k)
        ridx, _ = oracle.topk(row.double().numpy(), k)
        assert np.array_equal(_np(idx), ridx), k
    eq = torch.full((2, 40000), 1.5)
    idx = api.li_topk(eq.to(DEV), 2048)
    assert np.array_equal(_np(idx), np.tile(np.arange(2048, dtype=np.int32), (2, 1)))


# ---------------------------------------------------------------------------
# LatentIndex: absorption and latent scoring
# ---------------------------------------------------------------------------
def test_absorb_matches_oracle():
    case = synth.latent_group(B=5, L=8, seed=41)
    for layer in range(2):
        qt = api.li_absorb_query(case.q[layer].to(DEV), case.w_dec[layer].to(DEV))
        ref = oracle.absorb(case.q[layer], case.w_dec[layer])
        got = qt.float().cpu().double().numpy()
        absq = np.abs(case.q[layer].double().numpy())
        absw = np.abs(case.w_dec[layer].double().numpy())
        cond = np.einsum("bjd,jdc->bjc", absq, absw)
        # one round-to-nearest into bf16 (8 significant bits: relative error <= 2^-8)
        # plus fp32 accumulation over d terms
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * cond)


@pytest.mark.parametrize("B,L,lens", [(3, 1000, [1000, 333, 1]), (2, 5000, None)])
def test_latent_scores(B, L, lens):
    case = synth.latent_group(B=B, L=L, seed=42, lens=lens, plant_frac=0.01)
    qt = api.li_absorb_query(case.q[0].to(DEV), case.w_dec[0].to(DEV))
    ref, mag = oracle.latent_score(qt.cpu(), oracle.BF16, case.w[0], case.c, lens=case.lens.numpy(), with_mag=True)
    sc = api.li_latent_score(qt, case.w[0].to(DEV), case.c.to(DEV), lens=case.lens.to(DEV))
    assert_scores_close(_np(sc)[:, :L], ref, mag, 1e-2)
    assert api.li_get_last_error() == LI_OK


def test_latent_group_step_against_fp64_definition():
    """One G=4 group step at reduced length: absorb -> score -> top-k per layer,
    against the oracle's fp64 absorption (no bf16 rounding of q~)."""
    case = synth.latent_group(B=2, L=6000, seed=43)
    c = case.c.to(DEV)
    for layer in range(4):
        qt = api.li_absorb_query(case.q[layer].to(DEV), case.w_dec[layer].to(DEV))
        sc = api.li_latent_score(qt, case.w[layer].to(DEV), c)
        idx = api.li_topk(sc, 512, max_len=6000)
        qt64 = oracle.absorb(case.q[layer], case.w_dec[layer])
        ref, mag = oracle.latent_score(qt64, oracle.F64, case.w[layer], case.c, with_mag=True)
        assert_scores_close(_np(sc)[:, :6000], ref, mag, 1e-2)
        ridx, _ = oracle.topk(ref, 512)
        assert_topk_equivalent(_np(idx), ridx, ref, 1e-2)


def test_latent_group_full_size():
    """The LatentIndex group at its own shape (LatentIndex abstract and Figure 1: a G = 4 layer group
    shares one latent cache; each layer absorbs its decoder into its query, scans the cache and keeps
    its own top-k): B = 4 requests, L = 65536, d_c = 256 bf16, k = 2048, the generator's own seed.
    Each layer's scores and selection are checked on two requests (a different pair per layer, so
    every request is checked twice) against the fp64 definition, absorption included."""
    B, L, k = 4, 65536, 2048
    case = synth.latent_group(B=B, L=L, seed=3)
    c = case.c.to(DEV)
    rep = []
    for layer in range(4):
        qt = api.li_absorb_query(case.q[layer].to(DEV), case.w_dec[layer].to(DEV))
        sc = api.li_latent_score(qt, case.w[layer].to(DEV), c)
        idx = api.li_topk(sc, k, max_len=L)
        rows = [layer, (layer + 2) % B]
        qt64 = oracle.absorb(case.q[layer], case.w_dec[layer])
        ref, mag = oracle.latent_score(qt64, oracle.F64, case.w[layer], case.c, rows=rows, with_mag=True)
        assert_scores_close(_np(sc)[rows, :L], ref, mag, 1e-2)
        ridx, _ = oracle.topk(ref, k)
        assert_topk_equivalent(_np(idx)[rows], ridx, ref, 1e-2, report=rep)
    # the bf16 rounding of q~ moves a few borderline entries; never more than a handful a row
    assert all(n <= 32 for _, n in rep), rep
    assert api.li_get_last_error() == LI_OK


# ---------------------------------------------------------------------------
# failure path: bounded waits and out-of-range lengths report, never trap
# ---------------------------------------------------------------------------
def test_bounded_wait_reports_timeout():
    assert api.li_get_last_error() == LI_OK
    api.li_selftest_wait_timeout(1_000_000)  # 1 ms
    assert api.li_get_last_error() == LI_ERR_TIMEOUT
    assert api.li_get_last_error() == LI_OK


def test_bad_length_reports_bounds():
    case = synth.dsa_decode(B=2, L=256, seed=5)
    lens = torch.tensor([256, 9999], dtype=torch.int32, device=DEV)
    api.li_index_score(case.q.to(DEV), case.w.to(DEV), case.k8.to(DEV), case.ks.to(DEV), lens=lens)
    assert api.li_get_last_error() == LI_ERR_BOUNDS
    assert api.li_get_last_error() == LI_OK


def test_unsupported_shapes_raise():
    q = torch.zeros(2, 48, 128, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(2, 48, device=DEV)
    k = torch.zeros(2, 64, 128, dtype=torch.uint8, device=DEV)
    ks = torch.ones(2, 64, device=DEV)
    with pytest.raises(LiError):
        api.li_index_score(q, w, k, ks)            # 48 heads: neither indexer shape
    with pytest.raises(LiError):                   # 32 heads are a decode shape only
        api.li_index_score(q[:, :32].contiguous(), w[:, :32].contiguous(), k[0], ks[0], causal=True)


# ---------------------------------------------------------------------------
# graph-captured decode step (public API): host inputs in, selections out
# ---------------------------------------------------------------------------
def test_decode_indexer_graph_step():
    from sparse_attention_lightning_score_b200.step import DecodeIndexer
    case = synth.dsa_decode(B=3, L=5000, k_top=300, seed=23, lens=[5000, 2100, 40])
    ix = DecodeIndexer(case.k8.to(DEV), case.ks.to(DEV), heads=64, k=300, lens=case.lens.to(DEV))
    ref, _ = _oracle_decode(case)
    ridx, _ = oracle.topk(ref, 300, lens=case.lens.numpy())
    got = ix.step(case.q, case.w).numpy().copy()
    assert_topk_equivalent(got, ridx, ref, 1e-2, n_valid=case.lens.numpy())
    # a second step with new inputs through the same graph
    case2 = synth.dsa_decode(B=3, L=5000, k_top=300, seed=24, lens=[5000, 2100, 40])
    case2.k8, case2.ks = case.k8, case.ks
    ref2, _ = _oracle_decode(case2)
    ridx2, _ = oracle.topk(ref2, 300, lens=case.lens.numpy())
    got2 = ix.step(case2.q, case2.w).numpy().copy()
    assert_topk_equivalent(got2, ridx2, ref2, 1e-2, n_valid=case.lens.numpy())
    assert ix.h2d_bytes == 3 * 64 * 128 * 2 + 3 * 64 * 4 and ix.d2h_bytes == 3 * 300 * 4
    # the same steps through DMA copies instead of the kernels' own transfers
    ix2 = DecodeIndexer(case.k8.to(DEV), case.ks.to(DEV), heads=64, k=300, lens=case.lens.to(DEV), zero_copy=False)
    assert np.array_equal(ix2.step(case2.q, case2.w).numpy(), got2)
    assert np.array_equal(ix.step(case.q, case.w).numpy(), got)
    assert api.li_get_last_error() == LI_OK


@pytest.mark.parametrize("streams", [1, 2])
def test_decode_pipeline_matches_single_steps(streams):
    """Five independent steps in one pipelined graph (transfers overlapped with the kernels, device
    slots reused two steps later; with two compute streams, neighbouring steps' kernels overlap too)
    select exactly what five separate graph steps select."""
    from sparse_attention_lightning_score_b200.step import DecodeIndexer, DecodePipeline
    cases = [synth.dsa_decode(B=3, L=6000, k_top=500, seed=70 + i) for i in range(3)]
    caches = [(c.k8.to(DEV), c.ks.to(DEV)) for c in cases]
    order = [0, 1, 2, 1, 0]
    pipe = DecodePipeline([caches[i] for i in order], heads=64, k=500, streams=streams)
    g = torch.Generator().manual_seed(77)
    qs = [torch.randn(3, 64, 128, generator=g).to(torch.bfloat16) for _ in order]
    ws = [torch.randn(3, 64, generator=g) * 0.1 for _ in order]
    for i in range(len(order)):
        pipe.q_host[i].copy_(qs[i])
        pipe.w_host[i].copy_(ws[i])
    for rep in range(2):  # the same graph twice: slots and host buffers are reused
        got = [t.clone() for t in pipe.run()]
        for i, c in enumerate(order):
            one = DecodeIndexer(caches[c][0], caches[c][1], heads=64, k=500)
            want = one.step(qs[i], ws[i]).clone()
            assert torch.equal(got[i], want), (rep, i)
    assert pipe.h2d_bytes_per_step == 3 * 64 * 128 * 2 + 3 * 64 * 4 and pipe.d2h_bytes_per_step == 3 * 500 * 4
    assert api.li_get_last_error() == LI_OK


def test_decode_pipeline_two_streams_full_size():
    """The benchmarked shape (8 requests of 32768 keys, k = 2048), six independent steps over three
    caches with ragged lengths, two compute streams: every step's selection equals that step alone."""
    from sparse_attention_lightning_score_b200.step import DecodeIndexer, DecodePipeline
    lens = torch.tensor([32768, 30000, 2048, 2049, 17, 32767, 20000, 4096], dtype=torch.int32)
    cases = [synth.dsa_decode(B=8, L=32768, seed=90 + i) for i in range(3)]
    caches = [(c.k8.to(DEV), c.ks.to(DEV)) for c in cases]
    order = [0, 1, 2, 0, 1, 2]
    pipe = DecodePipeline([caches[i] for i in order], heads=64, k=2048, lens=lens.to(DEV), streams=2)
    g = torch.Generator().manual_seed(91)
    qs = [torch.randn(8, 64, 128, generator=g).to(torch.bfloat16) for _ in order]
    ws = [torch.randn(8, 64, generator=g) * 0.1 for _ in order]
    for i in range(len(order)):
        pipe.q_host[i].copy_(qs[i])
        pipe.w_host[i].copy_(ws[i])
    got = [t.clone() for t in pipe.run()]
    got2 = [t.clone() for t in pipe.run()]
    for i, c in enumerate(order):
        one = DecodeIndexer(caches[c][0], caches[c][1], heads=64, k=2048, lens=lens.to(DEV))
        want = one.step(qs[i], ws[i]).clone()
        assert torch.equal(got[i], want), i
        assert torch.equal(got2[i], want), i
    assert api.li_get_last_error() == LI_OK


def test_copy_from_host_kernel():
    src = torch.arange(1000 * 16 + 7, dtype=torch.uint8).pin_memory()  # a tail that is not 16 bytes
    dst = torch.zeros(src.numel(), dtype=torch.uint8, device=DEV)
    api.li_copy_from_host(dst, src)
    assert torch.equal(dst.cpu(), src)
    with pytest.raises(ValueError):
        api.li_copy_from_host(dst, src.clone())  # not page-locked
    assert api.li_get_last_error() == LI_OK
