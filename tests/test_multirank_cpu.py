"""The multi-GPU path on the CPU: two gloo ranks each advance their own,
independently seeded caches (the oracle stands in for the device step), with
no collective on the data path; the job's time is the max over ranks and its
work the sum.  Each rank's results must equal a single-process run of the
same seed, so sharding changes nothing but where a cache runs."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from kv_cache_sparse_b200.workloads import TINY, ChunkSource
from oracle import h2o_oracle as orc

WL = TINY.scaled(name="tiny_multirank", seq_len=TINY.chunk * 6)


def run_rank_work(rank: int):
    """What one rank does: its own caches, its own seed."""
    src = ChunkSource(WL, seed=bench.rank_seed(rank))
    cache = orc.OracleCache(WL.batch, WL.n_q_heads, WL.n_kv_heads, WL.head_dim, WL.capacity,
                            WL.window)
    outs = []
    for c in range(WL.steps):
        q, kn, vn = (t.double().numpy() for t in src.chunk(c))
        O, _ = cache.step(q, kn, vn)
        outs.append(O)
    return np.stack(outs), cache.pos.copy(), WL.steps * WL.batch * WL.chunk


def _worker(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        outs, pos, tokens = run_rank_work(rank)
        fake_time = 1.0 + rank          # rank 1 is the slow one
        t_job = bench.max_over_ranks(fake_time, world)
        tok_job = bench.sum_over_ranks(tokens, world)
        np.savez(os.path.join(result_dir, f"r{rank}.npz"), outs=outs, pos=pos,
                 t_job=t_job, tok_job=tok_job, tokens=tokens)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_shard_independent_caches(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [np.load(tmp_path / f"r{r}.npz") for r in range(world)]
    for r in range(world):
        outs, pos, tokens = run_rank_work(r)          # single-process reference
        assert np.array_equal(res[r]["outs"], outs)
        assert np.array_equal(res[r]["pos"], pos)
        assert float(res[r]["t_job"]) == 2.0           # max over ranks
        assert float(res[r]["tok_job"]) == world * tokens
    # different seeds: the ranks really run different caches
    assert not np.array_equal(res[0]["outs"], res[1]["outs"])
    # value = total work / max time
    assert float(res[0]["tok_job"]) / float(res[0]["t_job"]) == world * res[0]["tokens"] / 2.0
