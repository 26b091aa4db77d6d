"""The request-sharded round's one exchange, on CPU ranks (gloo).

Two (and three) ranks each hold a contiguous shard of a batch's survivals;
`sharded.gather_survivals` must give every rank the whole batch in rank
order, so that the scheduler run on it (here the oracle's, since the library
needs a GPU) and `sharded.local_slice` hand each rank exactly the admitted
lengths the unsharded schedule gives its requests.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _survivals(seed, B, G):
    rng = np.random.default_rng(seed)
    c = rng.choice(np.float32([1.0, 0.9, 0.7, 0.4, 0.1]), size=(B, G))
    return np.cumprod(c, axis=1, dtype=np.float32)


def _worker(rank, world, port, B_local, G, seed, budget, q):
    sys.path.insert(0, ROOT)
    from oracle import oracle
    from speculative_decoding_draft_rank_b200 import sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        S = _survivals(seed, world * B_local, G)
        S_local = torch.from_numpy(S[rank * B_local:(rank + 1) * B_local].copy())
        S_all = sharded.gather_survivals(S_local)
        same_batch = bool(np.array_equal(S_all.numpy(), S))
        kn = np.array([0, 4, 9], np.int32)
        kt = np.array([10.0, 11.0, 15.0])
        res = oracle.schedule(S_all.numpy().astype(np.float64), kn, kt, budget, oracle.SCHED_GREEDY_EARLY_STOP)
        mine = sharded.local_slice(torch.from_numpy(res.ell), rank, B_local)
        ref = oracle.schedule(S.astype(np.float64), kn, kt, budget, oracle.SCHED_GREEDY_EARLY_STOP)
        # Every rank's slice, gathered back, is the unsharded answer.
        parts = [torch.zeros(B_local, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(parts, mine.to(torch.int32))
        q.put((rank, same_batch, bool(np.array_equal(torch.cat(parts).numpy(), ref.ell)),
               bool(np.array_equal(mine.numpy(), ref.ell[rank * B_local:(rank + 1) * B_local])), res.n_adm))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B_local,G,budget", [(2, 7, 4, -1), (2, 16, 3, 20), (3, 5, 5, -1)])
def test_sharded_schedule_matches_unsharded(world, B_local, G, budget):
    sys.path.insert(0, ROOT)
    from oracle import oracle
    oracle._load()   # build the oracle once, before the ranks start
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B_local, G, 1234 + world, budget, q))
             for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    n_adm = {r[4] for r in results}
    assert len(n_adm) == 1   # every rank took the same global decision
    for rank, same_batch, all_ok, mine_ok, _ in results:
        assert same_batch, f"rank {rank} gathered a different batch"
        assert all_ok and mine_ok, f"rank {rank} admitted lengths differ from the unsharded schedule"
