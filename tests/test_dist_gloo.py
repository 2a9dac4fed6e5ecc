"""Multi-rank plumbing on CPU (gloo, world size 2): head sharding needs no
exchange (each rank's heads give exactly the full-problem result for those
heads), and the bench's max/sum-over-ranks timing reductions."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import qattn_oracle as O
from quantized_exact_attention_qattn_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    d = bench.init_dist(world, "gloo")
    # timing reductions
    assert bench.max_over_ranks(float(rank + 1), d) == float(world)
    assert bench.sum_over_ranks(1.0, d) == float(world)
    # head-sharded oracle attention: shard, compute, gather, compare with full
    wk = synth.custom(31, 1, 150, 5, 64, rope=False)
    h0, h1 = bench.shard_heads(wk.Hq, world, rank)
    q8, qs = O.quant_q(wk.q)
    k8, ks = O.quant_k(wk.k, O.k_mean(wk.k))
    v8t, vs = O.quant_v(wk.v)
    part, _, _ = O.attention(q8[:, h0:h1], qs[:, h0:h1], k8[:, h0:h1], ks[:, h0:h1],
                             v8t[:, h0:h1], vs[:, h0:h1], wk.Nkv)
    parts = [None] * world
    dist.all_gather_object(parts, (h0, h1, part))
    if rank == 0:
        full, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, wk.Nkv)
        got = np.concatenate([p for _, _, p in sorted(parts, key=lambda x: x[0])], axis=2)
        np.save(out_path, np.array([np.array_equal(got, full)]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_gloo_sharding_and_timing(tmp_path):
    out = str(tmp_path / "ok.npy")
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert bool(np.load(out)[0])


@pytest.mark.parametrize("H,world", [(56, 2), (56, 8), (5, 2), (3, 4), (1, 1)])
def test_shard_heads_partitions_every_head_once(H, world):
    ranges = [bench.shard_heads(H, world, r) for r in range(world)]
    covered = [h for a, b in ranges for h in range(a, b)]
    assert covered == list(range(H))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_percentile_nearest_rank():
    import bench
    vals = [5.0, 1.0, 3.0, 2.0, 4.0]
    assert bench.percentile(vals, 0.0) == 1.0
    assert bench.percentile(vals, 1.0) == 5.0
    assert bench.percentile(vals, 0.5) == 3.0
    assert bench.percentile([7.0], 0.9) == 7.0
    ten = [float(i) for i in range(10)]
    assert bench.percentile(ten, 0.1) == 1.0 and bench.percentile(ten, 0.9) == 8.0
