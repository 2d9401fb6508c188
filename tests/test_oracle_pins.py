"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties one oracle function to hand-computed values (tests/golden/),
a library routine on a special case, an algebraic identity, a brute-force
enumeration or an invariant, chosen so that a dropped term, a wrong sign, a
wrong index or a transposed operand fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_lightning_score_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


# ---------------------------------------------------------------------------
# e4m3 / bf16 codecs
# ---------------------------------------------------------------------------
def _torch_e4m3_decode(b):
    return torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()


def test_e4m3_decode_all_bytes_vs_torch():
    for b in range(256):
        ref = _torch_e4m3_decode(b)
        got = oracle.e4m3_decode(b)
        if (b & 0x7F) == 0x7F:
            assert math.isnan(got) and math.isnan(ref)
        else:
            assert got == ref, (b, got, ref)


def test_e4m3_decode_closed_forms():
    assert oracle.e4m3_decode(0x00) == 0.0
    assert math.copysign(1.0, oracle.e4m3_decode(0x80)) == -1.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x38) == 1.0
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0xFE) == -448.0


def test_e4m3_roundtrip_every_code():
    for b in range(256):
        if (b & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(b)) == b


def test_e4m3_ties_go_to_even_mantissa():
    pos = sorted({oracle.e4m3_decode(b) for b in range(0x7F)})
    for a, c in zip(pos[:-1], pos[1:]):
        mid = np.float32((a + c) / 2)
        assert float(mid) == (a + c) / 2  # midpoints of e4m3 neighbours are exact in fp32
        ca, cc = oracle.e4m3_encode(a), oracle.e4m3_encode(c)
        want = ca if (ca & 1) == 0 else cc
        assert oracle.e4m3_encode(float(mid)) == want
        assert oracle.e4m3_encode(float(np.nextafter(mid, np.float32(np.inf)))) == cc
        assert oracle.e4m3_encode(float(np.nextafter(mid, np.float32(-np.inf)))) == ca


def test_e4m3_encode_vs_torch_cast():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(40000, generator=g) * 100,
                   torch.randn(20000, generator=g) * 0.01,
                   torch.randn(20000, generator=g) * 1e-3,
                   (torch.rand(20000, generator=g) * 2 - 1) * 448]).clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x.numpy()], np.uint8)
    # the sign of an exact zero result may differ between conventions; compare values there
    nz = (ref & 0x7F) != 0
    assert np.array_equal(got[nz], ref[nz])
    assert np.all((got[~nz] & 0x7F) == 0)


def test_e4m3_saturates_to_448():
    for v, b in [(448.0, 0x7E), (460.0, 0x7E), (464.0, 0x7E), (465.0, 0x7E), (1e30, 0x7E),
                 (-500.0, 0xFE), (float("inf"), 0x7E), (float("-inf"), 0xFE)]:
        assert oracle.e4m3_encode(v) == b, v


def test_bf16_decode_vs_torch():
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(5000, generator=g) * 10).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_to_f32(int(b)) for b in bits], np.float32)
    assert np.array_equal(got, x.float().numpy())


# ---------------------------------------------------------------------------
# query quantisation
# ---------------------------------------------------------------------------
def test_quantize_hand_example():
    ex = GOLD["quantize_head"]
    q = torch.tensor(ex["q"], dtype=torch.bfloat16).reshape(1, 1, 4)
    q8, sq, we = oracle.quantize_query(q, np.array([[0.5]], np.float32))
    assert q8.reshape(-1).tolist() == ex["q8"]
    assert sq[0, 0] == np.float32(4.0) / np.float32(448.0)
    assert we[0, 0] == np.float32(0.5) * sq[0, 0]


def test_quantize_error_bound_and_extremes():
    g = torch.Generator().manual_seed(11)
    q = (torch.randn(3, 8, 128, generator=g) * torch.rand(3, 8, 1, generator=g) * 5).to(torch.bfloat16)
    q[1, 2] = 0  # an all-zero head
    w = torch.randn(3, 8, generator=g)
    q8, sq, we = oracle.quantize_query(q, w.numpy())
    qf = q.float().numpy().astype(np.float64)
    dec = torch.from_numpy(q8).view(torch.float8_e4m3fn).double().numpy()
    for r in range(3):
        for j in range(8):
            amax = np.abs(qf[r, j]).max()
            if amax == 0:
                assert sq[r, j] == 1.0 and np.all(q8[r, j] == 0)
                continue
            assert sq[r, j] == np.float32(amax) / np.float32(448)
            assert np.abs(dec[r, j]).max() == 448.0
            err = np.abs(dec[r, j] * sq[r, j] - qf[r, j])
            # half an e4m3 step: 2^-4 relative in the normal range, 2^-10 * sq below it
            bound = np.maximum(np.abs(qf[r, j]) * 2.0 ** -4, 2.0 ** -10 * sq[r, j]) * (1 + 1e-6)
            assert np.all(err <= bound)
    assert np.array_equal(we, w.numpy() * sq)


# ---------------------------------------------------------------------------
# indexer score
# ---------------------------------------------------------------------------
def test_score_hand_example():
    ex = GOLD["score_2x3"]
    q = np.array(ex["q"], np.float32)[None]
    w = np.array(ex["w"], np.float32)[None]
    k = np.array(ex["k"], np.float32)
    got = oracle.index_score(q, oracle.F32, w, k, oracle.F32)
    assert got[0].tolist() == ex["I"]


def _rand_case(seed, R=3, H=5, d=7, L=40):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((R, H, d)).astype(np.float32)
    w = rng.standard_normal((R, H)).astype(np.float32)
    k = rng.standard_normal((L, d)).astype(np.float32)
    return q, w, k


def test_score_relu_identities_against_matmul():
    # ReLU(x) - ReLU(-x) = x and ReLU(x) + ReLU(-x) = |x|, so
    #   I(q) - I(-q) = (sum_j w_j q_j) . k      and   I(q) + I(-q) = sum_j w_j |q_j . k|
    q, w, k = _rand_case(1)
    Ip = oracle.index_score(q, oracle.F32, w, k, oracle.F32)
    Im = oracle.index_score(-q, oracle.F32, w, k, oracle.F32)
    qd, wd, kd = q.astype(np.float64), w.astype(np.float64), k.astype(np.float64)
    lin = np.einsum("rj,rjd->rd", wd, qd) @ kd.T
    absx = np.einsum("rj,rjs->rs", wd, np.abs(np.einsum("rjd,sd->rjs", qd, kd)))
    np.testing.assert_allclose(Ip - Im, lin, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Ip + Im, absx, rtol=1e-12, atol=1e-12)


def test_score_single_head_nonneg_is_matmul():
    rng = np.random.default_rng(2)
    q = np.abs(rng.standard_normal((4, 1, 9))).astype(np.float32)
    k = np.abs(rng.standard_normal((30, 9))).astype(np.float32)
    w = np.ones((4, 1), np.float32)
    got = oracle.index_score(q, oracle.F32, w, k, oracle.F32)
    np.testing.assert_allclose(got, q[:, 0].astype(np.float64) @ k.astype(np.float64).T, rtol=1e-13)


def test_score_relu_invariants():
    q, w, k = _rand_case(3)
    got = oracle.index_score(q, oracle.F32, np.abs(w), k, oracle.F32)
    assert np.all(got >= 0)
    # keys opposite to every head's query give no positive dot product -> score 0
    qq = np.abs(q[:1])
    kk = -np.abs(k)
    assert np.all(oracle.index_score(qq, oracle.F32, w[:1], kk, oracle.F32) == 0)
    # additive in the heads: the H-head score is the sum of one-head scores
    tot = sum(oracle.index_score(q[:, j:j + 1], oracle.F32, w[:, j:j + 1], k, oracle.F32)
              for j in range(q.shape[1]))
    np.testing.assert_allclose(oracle.index_score(q, oracle.F32, w, k, oracle.F32), tot, rtol=1e-12, atol=1e-12)


def test_score_fp8_scales_match_decoded_values():
    case = synth.dsa_decode(B=2, L=300, H=4, d=32, seed=9)
    q8, sq, _ = oracle.quantize_query(case.q, case.w.numpy())
    got = oracle.index_score(q8, oracle.E4M3, case.w, case.k8, oracle.E4M3, q_scale=sq, k_scale=case.ks,
                             k_batch_rows=300, L=300)
    qd = torch.from_numpy(q8).view(torch.float8_e4m3fn).double() * torch.from_numpy(sq).double()[..., None]
    kd = case.k8.view(torch.float8_e4m3fn).double() * case.ks.double()[..., None]
    for b in range(2):
        ref = oracle.index_score(qd[b:b + 1].numpy(), oracle.F64, case.w[b:b + 1], kd[b].numpy(), oracle.F64)
        np.testing.assert_allclose(got[b], ref[0], rtol=1e-12, atol=1e-9)


def test_score_visibility_rules():
    q, w, k = _rand_case(4, R=6, L=10)
    pre = oracle.index_score(q, oracle.F32, w, k, oracle.F32, causal=True)
    dec = oracle.index_score(q, oracle.F32, w, k, oracle.F32, lens=[t + 1 for t in range(6)])
    assert np.array_equal(pre, dec)
    for t in range(6):
        assert np.all(np.isneginf(pre[t, t + 1:])) and np.all(np.isfinite(pre[t, :t + 1]))
    off = oracle.index_score(q, oracle.F32, w, k, oracle.F32, causal=True, causal_offset=2)
    assert np.all(np.isfinite(off[0, :3])) and np.isneginf(off[0, 3])


def test_score_per_request_caches():
    rng = np.random.default_rng(5)
    R, H, d, L = 3, 4, 8, 20
    q = rng.standard_normal((R, H, d)).astype(np.float32)
    w = rng.standard_normal((R, H)).astype(np.float32)
    k = rng.standard_normal((R, L, d)).astype(np.float32)
    got = oracle.index_score(q, oracle.F32, w, k, oracle.F32, k_batch_rows=L, L=L)
    for r in range(R):
        one = oracle.index_score(q[r:r + 1], oracle.F32, w[r:r + 1], k[r], oracle.F32)
        assert np.array_equal(got[r], one[0])
    sel = oracle.index_score(q, oracle.F32, w, k, oracle.F32, k_batch_rows=L, L=L, rows=[2, 0])
    assert np.array_equal(sel, got[[2, 0]])


def test_score_magnitude_bounds_score():
    q, w, k = _rand_case(6)
    I, M = oracle.index_score(q, oracle.F32, w, k, oracle.F32, with_mag=True)
    assert np.all(np.abs(I) <= M * (1 + 1e-12))


# ---------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------
def test_topk_hand_example():
    ex = GOLD["topk_ties"]
    idx, vals = oracle.topk(np.array([ex["scores"]]), ex["k"])
    assert idx[0].tolist() == ex["idx"]
    assert vals[0].tolist() == [ex["scores"][i] for i in ex["idx"]]


def _brute_topk(v, k):
    """The unique m-subset S (m = min(k, n)) such that every member outranks every
    non-member, rank = (value desc, position asc); found by enumerating subsets."""
    n = len(v)
    m = min(k, n)
    found = []
    for S in itertools.combinations(range(n), m):
        Sset = set(S)
        ok = all((v[i] > v[o]) or (v[i] == v[o] and i < o) for i in S for o in range(n) if o not in Sset)
        if ok:
            found.append(list(S))
    assert len(found) == 1
    return found[0]


def test_topk_bruteforce_enumeration():
    rng = np.random.default_rng(8)
    for trial in range(150):
        n = int(rng.integers(1, 10))
        k = int(rng.integers(1, 10))
        v = rng.integers(0, 3, n).astype(np.float64) if trial % 2 else rng.standard_normal(n)
        idx, _ = oracle.topk(v[None], k)
        want = _brute_topk(list(v), k)
        assert idx[0].tolist() == want + [-1] * (k - len(want))


def test_topk_vs_numpy_stable_argsort():
    rng = np.random.default_rng(9)
    for ties in (0, 5, 50):
        v = rng.integers(0, ties, 5000).astype(np.float64) if ties else rng.standard_normal(5000)
        for k in (1, 17, 2048, 5000):
            idx, _ = oracle.topk(v[None], k)
            ref = np.sort(np.argsort(-v, kind="stable")[:k])
            assert np.array_equal(idx[0], ref)


def test_topk_invariants_and_padding():
    rng = np.random.default_rng(10)
    s = rng.standard_normal((4, 300))
    lens = [0, 5, 200, 300]
    idx, vals = oracle.topk(s, 64, lens=lens)
    for r, n in enumerate(lens):
        m = min(64, n)
        sel = idx[r, :m]
        assert np.all(idx[r, m:] == -1) and np.all(np.isneginf(vals[r, m:]))
        assert np.all(np.diff(sel) > 0) and np.all(sel < n) and np.all(sel >= 0)
        if n:
            rest = np.setdiff1d(np.arange(n), sel)
            if len(rest):
                assert s[r, sel].min() >= s[r, rest].max()


def test_topk_special_values():
    v = np.array([[np.nan, -0.0, 0.0, -np.inf, 1.0, np.nan]])
    idx, _ = oracle.topk(v, 4)
    assert idx[0].tolist() == [1, 2, 3, 4]  # NaN lowest; -0 and +0 tie -> lower position
    idx, _ = oracle.topk(np.full((1, 10), 3.0), 4)
    assert idx[0].tolist() == [0, 1, 2, 3]


def test_topk_causal_rows():
    rng = np.random.default_rng(12)
    s = rng.standard_normal((6, 6))
    idx, _ = oracle.topk(s, 3, causal=True)
    for t in range(6):
        n = t + 1
        want = np.sort(np.argsort(-s[t, :n], kind="stable")[:3])
        assert idx[t, :min(3, n)].tolist() == want.tolist()


def test_tiny_planted_tokens_are_selected():
    case = synth.tiny_fp32()
    I = oracle.index_score(case.q, oracle.F32, case.w, case.k, oracle.F32)
    idx, _ = oracle.topk(I, case.k_top)
    assert set(case.planted.tolist()) <= set(idx[0].tolist())


# ---------------------------------------------------------------------------
# LatentIndex absorption and hierarchical selection
# ---------------------------------------------------------------------------
def _small_latent(seed=13, B=2, L=50, H=4, d=8, dc=16, G=4):
    return synth.latent_group(B=B, L=L, H=H, d=d, dc=dc, G=G, seed=seed, plant_frac=0.1)


def test_absorb_vs_einsum():
    case = _small_latent()
    got = oracle.absorb(case.q[0], case.w_dec[0])
    ref = np.einsum("bjd,jdc->bjc", case.q[0].double().numpy(), case.w_dec[0].double().numpy())
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_decode_keys_vs_einsum():
    case = _small_latent()
    got = oracle.decode_keys(case.w_dec[1], case.c[0, 3])
    ref = case.w_dec[1].double().numpy() @ case.c[0, 3].double().numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_absorbed_scores_equal_rebuilt_key_scores():
    # LatentIndex: scoring the shared cache with the absorbed query equals scoring
    # per-layer keys rebuilt by the decoder, without rebuilding them.
    case = _small_latent()
    for layer in range(2):
        qt = oracle.absorb(case.q[layer], case.w_dec[layer])
        I = oracle.latent_score(qt, oracle.F64, case.w[layer], case.c)
        for b in range(2):
            pos = list(range(0, 50, 3))
            reb = oracle.latent_score_rebuilt(case.q[layer], case.w[layer], case.w_dec[layer], case.c, b, pos)
            np.testing.assert_allclose(I[b, pos], reb, rtol=1e-12, atol=1e-12)


def test_hs_hand_example():
    ex = GOLD["hs_small"]
    c = torch.tensor(ex["latent_rows"], dtype=torch.bfloat16)[None]
    qt = np.array(ex["follower_q_tilde"], np.float64)[None, None]
    w = np.array(ex["follower_w"], np.float32)[None, None]
    out = oracle.hs_refine(qt, oracle.F64, w, c, np.array([ex["candidates"]]), ex["k"])
    assert out[0, 0].tolist() == ex["out"]


def _hs_case(seed=14, B=2, L=200, C=40, k=10, F=3):
    case = synth.latent_hs(B=B, L=L, H=4, d=8, dc=16, F=F, n_cand=C, k_top=k, seed=seed, plant_frac=0.05)
    qts = np.stack([oracle.absorb(case.q[l], case.w_dec[l]) for l in range(1 + F)])
    anchor = oracle.latent_score(qts[0], oracle.F64, case.w[0], case.c)
    cand, _ = oracle.topk(anchor, C)
    return case, qts, cand


def test_hs_followers_stay_inside_candidates():
    case, qts, cand = _hs_case()
    out = oracle.hs_refine(qts[1:], oracle.F64, case.w[1:], case.c, cand, 10)
    for f in range(3):
        for b in range(2):
            assert set(out[f, b].tolist()) <= set(cand[b].tolist())
            assert np.all(np.diff(out[f, b]) > 0)


def test_hs_all_positions_as_candidates_is_full_selection():
    case, qts, _ = _hs_case()
    L = case.c.shape[1]
    cand = np.tile(np.arange(L, dtype=np.int32), (2, 1))
    out = oracle.hs_refine(qts[1:], oracle.F64, case.w[1:], case.c, cand, 10)
    for f in range(3):
        full = oracle.latent_score(qts[1 + f], oracle.F64, case.w[1 + f], case.c)
        idx, _ = oracle.topk(full, 10)
        assert np.array_equal(out[f], idx)


def test_hs_k_equal_to_candidates_returns_them():
    case, qts, cand = _hs_case(C=10, k=10)
    out = oracle.hs_refine(qts[1:], oracle.F64, case.w[1:], case.c, cand, 10)
    for f in range(3):
        assert np.array_equal(out[f], cand)


def test_hs_padding_and_position_tie_break():
    # two identical latent rows at positions 7 and 3, listed 7 first: equal scores,
    # the lower cache position must win; -1 candidates are never selected
    c = torch.zeros(1, 10, 4, dtype=torch.bfloat16)
    c[0, 7] = torch.tensor([1.0, 2.0, 0.0, 0.0])
    c[0, 3] = torch.tensor([1.0, 2.0, 0.0, 0.0])
    c[0, 5] = torch.tensor([0.5, 0.0, 0.0, 0.0])
    qt = np.array([[[[1.0, 1.0, 0.0, 0.0]]]])
    w = np.ones((1, 1, 1), np.float32)
    out = oracle.hs_refine(qt, oracle.F64, w, c, np.array([[7, 3, -1, 5]]), 1)
    assert out[0, 0].tolist() == [3]
    out = oracle.hs_refine(qt, oracle.F64, w, c, np.array([[7, -1, -1, -1]]), 3)
    assert out[0, 0].tolist() == [7, -1, -1]


# ---------------------------------------------------------------------------
# the consumer: sparse attention over a selection
# ---------------------------------------------------------------------------
def test_sparse_attention_hand_example():
    ex = GOLD["sparse_attention_small"]
    q = torch.tensor(ex["q"], dtype=torch.bfloat16)
    kv = torch.tensor(ex["kv_rows"], dtype=torch.bfloat16)
    got = oracle.sparse_attention(q, kv, np.array(ex["sel"]), math.log(3.0), dv=ex["dv"])
    np.testing.assert_allclose(got, np.array(ex["out"]), rtol=1e-15, atol=1e-15)


def _attn_case(seed=3, B=2, H=3, L=40, D=12, dv=8, k=10):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, D, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, L, D, generator=g).to(torch.bfloat16)
    sel = np.stack([np.sort(np.random.default_rng(seed + b).choice(L, k, replace=False)) for b in range(B)])
    return q, kv, sel, dv


def test_sparse_attention_uniform_and_hard_limits():
    q, kv, sel, dv = _attn_case()
    vals = kv.double().numpy()
    # scale -> 0: every selected position gets the same weight, o = mean of the values
    o0 = oracle.sparse_attention(q, kv, sel, 1e-12, dv=dv)
    for b in range(2):
        np.testing.assert_allclose(o0[b], np.tile(vals[b, sel[b], :dv].mean(0), (3, 1)), rtol=1e-9, atol=1e-9)
    # scale -> large: the position with the largest logit takes all the weight
    oh = oracle.sparse_attention(q, kv, sel, 1e4, dv=dv)
    qd = q.double().numpy()
    for b in range(2):
        for h in range(3):
            best = sel[b][np.argmax(vals[b, sel[b]] @ qd[b, h])]
            np.testing.assert_allclose(oh[b, h], vals[b, best, :dv], rtol=1e-12, atol=1e-12)


def test_sparse_attention_two_positions_closed_form():
    # two selections with logits l0, l1: o = (e^l0 v0 + e^l1 v1) / (e^l0 + e^l1); listing a position
    # twice doubles its weight
    q, kv, sel, dv = _attn_case(B=1, H=1, k=2)
    s = 0.37
    v = kv.double().numpy()[0]
    l = [s * float(v[i] @ q.double().numpy()[0, 0]) for i in sel[0]]
    e = [math.exp(x) for x in l]
    want = (e[0] * v[sel[0][0], :dv] + e[1] * v[sel[0][1], :dv]) / (e[0] + e[1])
    np.testing.assert_allclose(oracle.sparse_attention(q, kv, sel, s, dv=dv)[0, 0], want, rtol=1e-12)
    twice = np.array([[sel[0][0], sel[0][1], sel[0][0]]])
    want2 = (2 * e[0] * v[sel[0][0], :dv] + e[1] * v[sel[0][1], :dv]) / (2 * e[0] + e[1])
    np.testing.assert_allclose(oracle.sparse_attention(q, kv, twice, s, dv=dv)[0, 0], want2, rtol=1e-12)


def test_sparse_attention_invariants():
    q, kv, sel, dv = _attn_case()
    o = oracle.sparse_attention(q, kv, sel, 0.5, dv=dv)
    # the order of the selection does not matter; pads and out-of-range rows are skipped
    perm = np.stack([s[::-1] for s in sel])
    padded = np.concatenate([perm, np.full((2, 3), -1), np.full((2, 1), 10 ** 6)], axis=1)
    np.testing.assert_allclose(oracle.sparse_attention(q, kv, padded, 0.5, dv=dv), o, rtol=1e-13, atol=1e-13)
    # each head attends on its own (the softmax runs over positions, not heads)
    for h in range(3):
        oh = oracle.sparse_attention(q[:, h:h + 1].contiguous(), kv, sel, 0.5, dv=dv)
        np.testing.assert_allclose(oh[:, 0], o[:, h], rtol=1e-13, atol=1e-13)
    # a request reads its own cache: request 1 alone against a shared copy of its rows
    o1 = oracle.sparse_attention(q[1:], kv[1], sel[1:], 0.5, dv=dv)
    np.testing.assert_allclose(o1[0], o[1], rtol=1e-13, atol=1e-13)
    # the output is a convex combination of the selected values, and mag bounds it
    o, mag = oracle.sparse_attention(q, kv, sel, 0.5, dv=dv, with_mag=True)
    assert np.all(np.abs(o) <= mag + 1e-12)
    for b in range(2):
        vals = kv.double().numpy()[b, sel[b], :dv]
        assert np.all(o[b] <= vals.max(0) + 1e-12) and np.all(o[b] >= vals.min(0) - 1e-12)
    # no valid selection: zero
    none = np.full((2, 4), -1)
    assert np.all(oracle.sparse_attention(q, kv, none, 0.5, dv=dv) == 0.0)


def _hs8_case(seed=21, B=2, L=120, F=2, H=3):
    g = torch.Generator().manual_seed(seed)
    c = torch.randn(B, L, 12, generator=g)
    from sparse_attention_lightning_score_b200 import synth as sy
    c8, cs = sy.encode_e4m3_cache(c.view(B * L, 12))
    qt = torch.randn(F, B, H, 12, generator=g).to(torch.bfloat16)
    w = torch.randn(F, B, H, generator=g)
    return qt, w, c8.view(B, L, 12), cs.view(B, L)


def test_hs_fp8_all_positions_as_candidates_is_full_selection():
    qt, w, c8, cs = _hs8_case()
    B, L = c8.shape[0], c8.shape[1]
    cand = np.tile(np.arange(L, dtype=np.int32), (B, 1))
    out = oracle.hs_refine_fp8(qt, w, c8, cs, cand, 7)
    for f in range(qt.shape[0]):
        q8, sq, _ = oracle.quantize_query(qt[f], w[f].numpy())
        full = oracle.index_score(q8, oracle.E4M3, w[f], c8, oracle.E4M3, q_scale=sq, k_scale=cs, k_batch_rows=L, L=L)
        idx, _ = oracle.topk(full, 7)
        assert np.array_equal(out[f], idx)


def test_hs_fp8_k_equal_to_candidates_and_padding():
    qt, w, c8, cs = _hs8_case()
    cand = np.array([[3, 17, 40, 99, -1, -1], [0, 5, 6, 7, 8, 119]], np.int32)
    out = oracle.hs_refine_fp8(qt, w, c8, cs, cand, 6)
    for f in range(qt.shape[0]):
        assert out[f, 0].tolist() == [3, 17, 40, 99, -1, -1]     # pads never selected
        assert out[f, 1].tolist() == [0, 5, 6, 7, 8, 119]
    out = oracle.hs_refine_fp8(qt, w, c8, cs, np.full((2, 4), -1, np.int32), 3)
    assert np.all(out == -1)
