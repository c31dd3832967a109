"""Multi-rank host logic on CPU (gloo, world size 2): batch sharding covers
every (b, h) sequence once, per-rank results assembled from the shards equal
the unsharded result, and timing reductions take the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from structured_sparse_state_b200.sharding import batch_shard


@pytest.mark.parametrize("B,world", [(8, 2), (7, 2), (1, 4), (9, 4), (3, 8)])
def test_batch_shard_partitions_rows(B, world):
    rows = []
    sizes = []
    for r in range(world):
        a, b = batch_shard(B, world, r)
        rows += list(range(a, b))
        sizes.append(b - a)
    assert rows == list(range(B))
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, outdir):
    import torch.distributed as dist

    import oracle
    import pdssm_inputs as gen
    from structured_sparse_state_b200.sharding import batch_shard, max_over_ranks

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        inp = gen.generate(gen.workload(4, B=5, H=2, L=64))
        a, b = batch_shard(5, world, rank)
        y, hl = oracle.scan_fwd(inp.pi, inp.k[a:b], inp.d[a:b], inp.b[a:b], inp.c[a:b],
                                inp.h0[a:b])
        np.save(os.path.join(outdir, f"y{rank}.npy"), y)
        t = max_over_ranks(float(rank + 1) * 1.5)
        np.save(os.path.join(outdir, f"t{rank}.npy"), np.array([t]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_shards_match_unsharded(tmp_path):
    import oracle
    import pdssm_inputs as gen
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    inp = gen.generate(gen.workload(4, B=5, H=2, L=64))
    y_full, _ = oracle.scan_fwd(inp.pi, inp.k, inp.d, inp.b, inp.c, inp.h0)
    parts = [np.load(tmp_path / f"y{r}.npy") for r in range(world)]
    assert np.array_equal(np.concatenate(parts, axis=0), y_full)
    for r in range(world):
        assert float(np.load(tmp_path / f"t{r}.npy")[0]) == 3.0
