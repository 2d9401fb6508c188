"""Multi-rank host logic on CPU: gloo, world size 2, spawned processes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_attention_lightning_score_b200.dist import max_over_ranks, shard_lens, shard_rows


def test_shard_rows_cover_exactly_once():
    for total in (0, 1, 7, 8, 1000, 8192):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = shard_rows(total, world, r)
                assert 0 <= a <= b <= total
                seen.extend(range(a, b))
            assert seen == list(range(total))
    with pytest.raises(ValueError):
        shard_rows(5, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from sparse_attention_lightning_score_b200 import dist as D
    import oracle
    from sparse_attention_lightning_score_b200 import synth
    d = D.init("gloo", timeout_s=60)
    try:
        # every rank scores its shard of one batch of decode requests on the CPU oracle
        case = synth.dsa_decode(B=5, L=200, H=4, d=32, seed=3)
        a, b = D.shard_rows(5, world, rank)
        out = oracle.index_score(case.q[a:b].float(), oracle.F32, case.w[a:b], case.k8[a:b], oracle.E4M3,
                                 k_scale=case.ks[a:b], k_batch_rows=200, L=200)
        tmax = D.max_over_ranks([float(rank + 1), -float(rank)])
        gathered = [None] * world
        d.all_gather_object(gathered, (a, b, out))
        q.put((rank, tmax, gathered))
    finally:
        d.destroy_process_group()


def test_two_rank_sharding_and_max_over_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from sparse_attention_lightning_score_b200 import synth
    case = synth.dsa_decode(B=5, L=200, H=4, d=32, seed=3)
    full = oracle.index_score(case.q.float(), oracle.F32, case.w, case.k8, oracle.E4M3, k_scale=case.ks,
                              k_batch_rows=200, L=200)
    for rank, tmax, gathered in res:
        assert tmax == [2.0, 0.0]
        rows = np.concatenate([g[2] for g in gathered])
        assert [g[:2] for g in gathered] == [(0, 3), (3, 5)]
        assert np.array_equal(rows, full)


def test_max_over_ranks_single_process_is_identity():
    assert max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_shard_lens_split_every_length():
    for L, P in ((32768, 4), (10000, 3), (7, 2)):
        sl = -(-L // P)
        for n in (0, 1, sl - 1, sl, sl + 1, L):
            parts = [shard_lens(n, p, sl) for p in range(P)]
            assert sum(parts) == n
            # full slices, then at most one partial one, then empty ones
            assert parts == sorted(parts, reverse=True)
            assert sum(1 for x in parts if 0 < x < sl) <= 1
            t = shard_lens(torch.tensor([n, L], dtype=torch.int32), 1, sl)
            assert t.tolist() == [shard_lens(n, 1, sl), shard_lens(L, 1, sl)] and t.dtype == torch.int32


def test_merge_of_shard_selections_is_the_full_selection():
    """The merge's premise, on the oracle: the top-k over the union of every shard's own top-k
    (positions made global, lists laid side by side in shard order) is the top-k of the whole row,
    ties included."""
    import oracle
    from sparse_attention_lightning_score_b200 import synth
    rows = synth.score_rows(3, 9000, seed=8, ties=40).double().numpy()  # many exact ties
    k, P = 300, 4
    sl = -(-9000 // P)
    lens = np.array([9000, 5000, 1234])
    full, _ = oracle.topk(rows, k, lens=lens)
    cand_v, cand_p = [], []
    for p in range(P):
        lo = p * sl
        part = rows[:, lo:lo + sl]
        ln = np.clip(lens - lo, 0, part.shape[1])
        idx, vals = oracle.topk(part, k, lens=ln)
        cand_v.append(np.where(idx >= 0, vals, -np.inf))
        cand_p.append(np.where(idx >= 0, idx + lo, -1))
    cv, cp = np.concatenate(cand_v, axis=1), np.concatenate(cand_p, axis=1)
    nvalid = (cp >= 0).sum(axis=1)
    sel, _ = oracle.topk(cv, k, lens=nvalid)  # slot order is global position order
    merged = np.where(sel >= 0, np.take_along_axis(cp, np.maximum(sel, 0), axis=1), -1)
    assert np.array_equal(merged, full)


def _gather_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from sparse_attention_lightning_score_b200 import dist as D
    d = D.init("gloo", timeout_s=60)
    try:
        vals = torch.full((3, 5), float(rank)) + torch.arange(5).float()
        idx = torch.full((3, 5), 10 * rank, dtype=torch.int32)
        gv, gi = D.gather_selections(vals, idx)
        q.put((rank, gv.numpy(), gi.numpy()))
    finally:
        d.destroy_process_group()


def test_two_rank_gather_of_selections_is_in_rank_order():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gv, gi in res:
        assert gv.shape == (2, 3, 5) and gi.shape == (2, 3, 5)
        for r in range(world):
            assert np.array_equal(gv[r], np.full((3, 5), float(r)) + np.arange(5)) and np.all(gi[r] == 10 * r)
