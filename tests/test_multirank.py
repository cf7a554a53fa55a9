"""Multi-process paths of bench.py on CPU with the gloo backend (world size 2).

The block does not shard across GPUs (all slices run on one GPU), so
``bench.py --gpus N`` runs N independent replicas: the only cross-rank steps are
the barrier, the max over ranks of the measured times, and rank 0 alone
printing (and, for the reference arm, alone running the oracle).
"""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench

    bench.barrier(world)
    m = bench.allreduce_max(10.0 * (rank + 1), world)
    bench.barrier(world)
    # the reference arm: only rank 0 does work and prints; other ranks return 0 at once
    rc = bench.run_reference(bench.parse_args(["--impl", "reference"])) if rank != 0 else 0
    out.put((rank, m, rc))
    dist.destroy_process_group()


def test_two_rank_max_and_barrier():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [20.0, 20.0]
    assert res[1][2] == 0
