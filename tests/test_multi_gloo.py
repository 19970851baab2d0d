"""Multi-process host logic of the data-parallel path, on CPU with gloo.

Decode attention over (sequence, KV head) units needs no exchange between
GPUs: N ranks run N independent shards (weak scaling) and only the timing is
reduced (max over ranks) together with the unit count (sum).  Two gloo ranks
check the shard assignment and both reductions.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from compressed_space_decode_b200 import multi, synthetic
    r, lr, w = multi.env_rank()
    assert (r, lr, w) == (rank, rank, world)
    wl = synthetic.workloads()["gqa_b16_q32_kv4_L32768_paged"]
    mine = multi.shard_workload(wl, r, w)
    # every rank keeps the shapes of one GPU's workload, with its own data
    assert (mine.batch, mine.q_heads, mine.kv_heads, mine.seq_lens) == (wl.batch, wl.q_heads, wl.kv_heads,
                                                                        wl.seq_lens)
    seeds = [None] * w
    dist.all_gather_object(seeds, mine.seed)
    ms = multi.max_over_ranks(10.0 + rank)
    units = multi.sum_over_ranks(mine.kv_token_heads)
    multi.barrier()
    out[rank] = (seeds, ms, units)
    dist.destroy_process_group()


def test_two_rank_shards_and_reductions():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    from compressed_space_decode_b200 import synthetic
    wl = synthetic.workloads()["gqa_b16_q32_kv4_L32768_paged"]
    for rank in range(world):
        seeds, ms, units = res[rank]
        assert len(set(seeds)) == world          # independent data per rank
        assert ms == 11.0                        # max over ranks
        assert units == world * wl.kv_token_heads  # whole-job unit count
