"""bench.py's multi-rank logic on CPU: two gloo ranks, each with its own batch
(seeded by rank), the step time reduced as the max over ranks and the KV
bytes summed -- the rules the N-GPU bench line follows."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_450_b200 import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, ws, lr = bench.dist_env()
        seed = bench.rank_seed(0, r)
        w = W.make_decode_workload(W.TINY, seed=seed)
        t_local = 1.0 + r              # rank 1 is the slower one
        t = bench.max_over_ranks(t_local)
        total = bench.sum_over_ranks(w.kv_bytes())
        bench.barrier()
        out[r] = (r, ws, lr, seed, t, total, w.kv_bytes(), int(w.context_lens.sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_aggregation():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    (r0, ws0, lr0, s0, t0, tot0, kv0, n0), (r1, ws1, lr1, s1, t1, tot1, kv1, n1) = res[0], res[1]
    assert ws0 == ws1 == 2 and (lr0, lr1) == (0, 1)
    assert s0 != s1                      # independent batches per rank
    assert t0 == t1 == 2.0               # max over ranks
    assert tot0 == tot1 == kv0 + kv1     # whole-job bytes
    assert n0 != n1


def test_single_process_helpers_without_a_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5 and bench.sum_over_ranks(2.0) == 2.0
    assert bench.rank_seed(7, 0) == 7 and bench.rank_seed(7, 3) == 3007
    bench.barrier()
