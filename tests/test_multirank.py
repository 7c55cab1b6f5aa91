"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

The path shards into independent (sequence, head) units, so ranks exchange
nothing on the data path; the only collectives are the MAX reduction of the
timed region and the SUM of processed tokens, checked here, plus distinct
per-rank batches."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from gated_delta_rule_64_b200.inputs import PREFILL_BF16, make_inputs
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, _ = bench.env_rank()
        ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(ms, w)
        tok = bench.sum_over_ranks(4096.0 * (rank + 1), w)
        seed = bench.rank_seed(PREFILL_BF16.seed, rank)
        x = make_inputs(PREFILL_BF16.replace(T=64, H=2, seed=seed))
        results[rank] = (r, w, mx, tok, seed, float(x.v[0, 0, 0, 0]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_shard():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True, start_method="spawn")
    r0, r1 = results[0], results[1]
    assert (r0[0], r0[1]) == (0, 2) and (r1[0], r1[1]) == (1, 2)
    assert r0[2] == r1[2] == 15.0                 # max over ranks of the timed region
    assert r0[3] == r1[3] == 4096.0 * 3           # tokens of all ranks
    assert r0[4] != r1[4] and r0[5] != r1[5]      # each rank draws its own batch
