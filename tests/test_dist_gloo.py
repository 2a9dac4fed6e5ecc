"""Multi-rank plumbing on CPU (gloo, world size 2): head sharding needs no
exchange (each rank's heads give exactly the full-problem result for those
heads, also when each rank runs the whole path on its column slice of the raw
interleaved QKV buffer), and the bench's max/sum-over-ranks timing reductions."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import qattn_oracle as O
from quantized_exact_attention_qattn_b200 import shard, synth


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
    # one interleaved problem split by heads at the raw input, as bench.py
    # --shard-heads splits it: each rank runs the whole path (prep, K mean,
    # quantization, attention) on the column slice of the QKV buffer holding its
    # heads; gathered, every head equals the unsplit problem's
    wc = synth.make("canonical", N=300, H=6)
    (q0, q1), (k0, k1) = shard.kv_shard(wc.Hq, wc.Hkv, world, rank)
    full5 = wc.qkv.reshape(1, wc.Nq, 3, wc.Hq, wc.D)
    sl = [shard.head_slice(full5[:, :, i], a, b) for i, (a, b) in
          enumerate([(q0, q1), (k0, k1), (k0, k1)])]
    assert all(np.shares_memory(x, full5) for x in sl)      # views, no copy
    mine = O.pipeline(sl[0], sl[1], sl[2], wc.q_weight, wc.k_weight, wc.eps, wc.rotary_dim,
                      wc.theta)["out"]
    raw_parts = [None] * world
    dist.all_gather_object(raw_parts, (q0, mine))
    if rank == 0:
        full, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, wk.Nkv)
        got = np.concatenate([p for _, _, p in sorted(parts, key=lambda x: x[0])], axis=2)
        ref = O.pipeline(wc.q, wc.k, wc.v, wc.q_weight, wc.k_weight, wc.eps, wc.rotary_dim,
                         wc.theta)["out"]
        got2 = np.concatenate([p for _, p in sorted(raw_parts, key=lambda x: x[0])], axis=2)
        np.save(out_path, np.array([np.array_equal(got, full) and np.array_equal(got2, ref)]))
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


@pytest.mark.parametrize("Hq,Hkv,world", [(16, 4, 2), (16, 4, 4), (56, 56, 8), (6, 3, 2)])
def test_kv_shard_keeps_gqa_groups_whole(Hq, Hkv, world):
    got = [shard.kv_shard(Hq, Hkv, world, r) for r in range(world)]
    assert [h for (a, b), _ in got for h in range(a, b)] == list(range(Hq))
    for (q0, q1), (k0, k1) in got:
        assert all(h // (Hq // Hkv) in range(k0, k1) for h in range(q0, q1))
