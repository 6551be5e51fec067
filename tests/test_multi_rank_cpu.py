"""The multi-rank path of bench.py on CPU: two gloo ranks, as torchrun would
start them.  The forward needs no collective (token-sharded replicas), so the
host logic is what is shared: each rank draws its own token rows, all ranks
hold identical weights, and the step time is the max over ranks."""
import hashlib
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    wl = synth.WORKLOADS["toy_fp32"].with_tokens(16)
    rows = bench.rank_token_rows(wl, rank)
    x = synth.make_x_rows(wl, 0, rows)
    w = synth.make_inputs(wl, 0, with_x=False)
    wsig = hashlib.sha256(b"".join(w[k].tobytes() for k in synth.WEIGHT_NAMES)).hexdigest()
    # a rank-dependent "step time": the reduction must return the largest
    t = bench.max_over_ranks(1.5 + rank)
    gathered = [None] * world
    dist.all_gather_object(gathered, (rows.tolist(), x.sum().item(), wsig))
    if rank == 0:
        out.put((t, gathered))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_rank_replicas_on_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    t, gathered = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert t == 1.5 + (world - 1)
    rows = [set(g[0]) for g in gathered]
    assert not (rows[0] & rows[1])                     # disjoint token shards
    assert gathered[0][1] != gathered[1][1]            # different inputs per rank
    assert gathered[0][2] == gathered[1][2]            # identical weight replicas


def test_single_process_max_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
