"""N>1 host path on CPU: two gloo ranks shard a decode batch and a prefill's
kv-head groups, run the oracle on their shards, and gather; the result must
equal the single-process oracle run.  Also checks the max-over-ranks timing
reduction and the whole-job throughput aggregation."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_aware_b200 import parallel as PAR


def test_shard_range_partitions():
    for n in range(0, 20):
        for w in range(1, 6):
            parts = [PAR.shard_range(n, w, r) for r in range(w)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(w - 1))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    assert PAR.kv_group_shard(32, 4, 2, 1) == (16, 32)
    assert PAR.aggregate_throughput(10.0, [1.0, 2.0]) == 10.0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from sparse_attention_aware_b200 import workloads as W
        # decode: shard the batch
        lens = [300, 1000, 57, 640, 1200]
        cache, q = W.random_decode(11, len(lens), 8, 2, 64, lens, 16)
        k = 40
        lo, hi = PAR.shard_range(len(lens), world, rank)
        sub = W.PagedCache(cache.k, cache.v, cache.page_table[lo:hi].contiguous(), cache.seq_lens[lo:hi].contiguous())
        idx, cnt = oracle.select_topk(sub, q[lo:hi], k)
        out, lse = oracle.decode_tokens(sub, q[lo:hi], idx, cnt, 0.125)
        got = PAR.gather_concat(torch.from_numpy(out.reshape(hi - lo, 8, 64)))
        # prefill: shard kv-head groups
        wl = W.random_prefill(12, 200, 8, 2, 32, 64)
        h0, h1 = PAR.kv_group_shard(8, 2, world, rank)
        nB = 4
        mask = np.ones((8, nB * (nB + 1) // 2), dtype=np.uint8)
        rows = [t * 8 + h for t in range(200) for h in range(h0, h1)]
        pout, _ = oracle.prefill(wl.cache, wl.q, 64, mask, 0.2, rows=rows)
        pgot = PAR.gather_concat(torch.from_numpy(pout.reshape(200, h1 - h0, 32)), dim=1)
        t = PAR.max_over_ranks([1.0 + rank, 5.0 - rank])
        if rank == 0:
            torch.save({"decode": got, "prefill": pgot, "max": t}, os.path.join(out_dir, "gathered.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_matches_single_process(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = torch.load(os.path.join(tmp_path, "gathered.pt"))
    import oracle
    from sparse_attention_aware_b200 import workloads as W
    lens = [300, 1000, 57, 640, 1200]
    cache, q = W.random_decode(11, len(lens), 8, 2, 64, lens, 16)
    idx, cnt = oracle.select_topk(cache, q, 40)
    out, _ = oracle.decode_tokens(cache, q, idx, cnt, 0.125)
    np.testing.assert_array_equal(res["decode"].numpy(), out.reshape(5, 8, 64))
    wl = W.random_prefill(12, 200, 8, 2, 32, 64)
    mask = np.ones((8, 10), dtype=np.uint8)
    pout, _ = oracle.prefill(wl.cache, wl.q, 64, mask, 0.2)
    np.testing.assert_array_equal(res["prefill"].numpy(), pout.reshape(200, 8, 32))
    assert res["max"] == [2.0, 5.0]
