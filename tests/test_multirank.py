"""The multi-GPU form of the benchmark, run as world-size-2 gloo ranks on the
CPU: each rank draws its own data-parallel shard of the workload (same
shapes, its own seed), and the step time is the maximum over ranks while the
work is summed.  There is no collective on the data path."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_455_b200 import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = W.CONFIGS["qwen"]
        layout = W.make_layout(cfg, shard=rank)
        # fake per-rank timings: rank r is slower by r ms
        ms, attn, byt, seqs = bench.combine_ranks(dist, torch.device("cpu"), 1.0 + rank,
                                                  0.1 * (rank + 1), 1000 * (rank + 1),
                                                  cfg.num_seqs)
        out[rank] = (ms, attn, byt, seqs, layout.context_lens.tolist(),
                     layout.block_tables.shape)
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_and_max_time():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    for r in (r0, r1):
        assert r[0] == 2.0                        # max of 1.0 and 2.0 ms
        assert abs(r[1] - 0.2) < 1e-12            # max attention time
        assert r[2] == 3000.0                     # bytes summed over ranks
        assert r[3] == 128.0                      # sequences summed over ranks
    assert r0[4] != r1[4], "ranks must draw different shards"
    assert len(r0[4]) == len(r1[4]) == 64


def test_single_rank_combine_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(None, None, 1.5, 0.5, 10, 64) == (1.5, 0.5, 10.0, 64.0)


def test_shard_zero_is_the_single_gpu_workload():
    from paged_kv_cache_455_b200 import workloads as W
    cfg = W.CONFIGS["mix"]
    a, b = W.make_layout(cfg), W.make_layout(cfg, shard=0)
    assert np.array_equal(a.block_tables, b.block_tables)
    c = W.make_layout(cfg, shard=3)
    assert not np.array_equal(a.context_lens, c.context_lens)
