"""Multi-rank host logic on CPU: gloo, world size 2, spawned processes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_attention_lightning_score_b200.dist import max_over_ranks, shard_rows


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
