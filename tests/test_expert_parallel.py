"""Expert parallelism on CPU with two gloo ranks: routing is replicated, each
rank runs only the experts of its contiguous slice (the oracle's expert-range
partial, the shared expert on rank 0), and the all-reduced partials equal the
whole layer."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg():
    from synthetic import CONFIGS
    cfg = dict(CONFIGS["tiny"])
    cfg.update(T=6, E=8, k=2, seed=61, shared=("affine", 8, 64), f_shared=128)
    return cfg


def _rank(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import oracle_run
    from synthetic import make_custom

    from bit_quantized_moe_route_b200.layer import expert_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = _cfg()
        inp = make_custom(cfg)
        part = oracle_run(inp, expert_range=expert_range(rank, world, cfg["E"]), include_shared=rank == 0)
        t = torch.from_numpy(np.ascontiguousarray(part["out"]))
        dist.all_reduce(t)
        if rank == 0:
            full = oracle_run(inp)["out"]
            q.put(float(np.abs(t.numpy() - full).max() / np.abs(full).max()))
    finally:
        dist.destroy_process_group()


def test_expert_ranges_partition_the_experts():
    from bit_quantized_moe_route_b200.layer import expert_range
    for E, world in ((8, 2), (256, 3), (7, 4), (3, 8)):
        cuts = [expert_range(r, world, E) for r in range(world)]
        assert cuts[0][0] == 0 and cuts[-1][1] == E
        assert all(a[1] == b[0] for a, b in zip(cuts, cuts[1:]))
        sizes = [e - b for b, e in cuts]
        assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        expert_range(2, 2, 8)


def test_two_rank_allreduce_of_partials_is_the_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert q.get(timeout=10) < 1e-13
