"""The N>1 path on CPU: world-size-2 gloo process groups running the
replica partitioning and the max-over-ranks timing reduction used by
bench.py.  No GPU involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from vision_transformer_encoder_layernorm_b200 import replicas

C3_GRIDS = [(26, 30), (24, 37), (30, 32), (60, 65), (76, 58)]


def test_partition_covers_and_balances():
    for world in (1, 2, 3, 4, 8):
        parts = replicas.partition_images(C3_GRIDS, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(C3_GRIDS)))
    parts = replicas.partition_images(C3_GRIDS, 2)
    # the two largest images (4408 and 3900 tokens) go to different ranks
    assert (4 in parts[0]) != (4 in parts[1])
    assert (3 in parts[0]) != (3 in parts[1])
    assert replicas.partition_images(C3_GRIDS, 8)[5:] == [[], [], []]
    with pytest.raises(ValueError):
        replicas.partition_images(C3_GRIDS, 0)


def test_partition_is_lpt_optimal_on_small_cases():
    # brute force over all assignments of 5 images to 2 ranks
    import itertools
    costs = [replicas.image_cost(h * w, 1152, 4304) for h, w in C3_GRIDS]
    best = min(max(sum(c for c, a in zip(costs, asg) if a == r) for r in (0, 1))
               for asg in itertools.product((0, 1), repeat=5))
    parts = replicas.partition_images(C3_GRIDS, 2)
    got = max(sum(costs[i] for i in p) for p in parts)
    assert got <= best * 4 / 3 + 1e-6       # Graham's LPT bound


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    parts = replicas.partition_images(C3_GRIDS, world)
    gathered = [None] * world
    dist.all_gather_object(gathered, parts)
    t = replicas.max_over_ranks(1.5 + rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, gathered, t))


def test_gloo_two_ranks_agree_and_reduce_max():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gathered, t in out:
        assert gathered[0] == gathered[1]                  # same partition on every rank
        assert t == 2.5                                    # max over ranks
    assert replicas.max_over_ranks(3.0) == 3.0             # no process group
