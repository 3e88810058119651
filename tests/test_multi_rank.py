"""Multi-rank host logic on CPU (gloo, world size 2).

Requests are independent, so N GPUs shard them with no collective on the data
path: rank r decodes the global requests r*B .. r*B+B-1.  Two gloo ranks each
decode their shard with the oracle; gathered, the shards must equal one decode
of all requests.  The job's time is the slowest rank's (a max all-reduce), and
the throughput counts every rank's candidates over that time.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from trie_constrained_beam_fr_b200 import synth

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, result_dir: str):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        w = synth.scaled(synth.WORKLOADS["tiny"], B=2)
        sids = synth.workload_catalog(w)
        b0, B = bench.rank_requests(rank, WORLD, w.B)
        res = oracle.decode(oracle.Config.from_workload(w, B=B, b_offset=b0), oracle.Catalog(sids, w.codebook_sizes))
        shards = [None] * WORLD
        dist.all_gather_object(shards, (b0, res.sids.tolist(), res.scores.tolist()))
        slowest = bench.max_over_ranks(10.0 + rank, WORLD, dist)
        if rank == 0:
            np.save(os.path.join(result_dir, "shards.npy"), np.array(shards, dtype=object), allow_pickle=True)
            np.save(os.path.join(result_dir, "slowest.npy"), np.array([slowest]))
    finally:
        dist.destroy_process_group()


def test_request_sharding_over_two_gloo_ranks(tmp_path):
    mp.spawn(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    shards = np.load(tmp_path / "shards.npy", allow_pickle=True)
    slowest = float(np.load(tmp_path / "slowest.npy")[0])
    assert slowest == 11.0
    w = synth.scaled(synth.WORKLOADS["tiny"], B=2 * WORLD)
    sids = synth.workload_catalog(w)
    full = oracle.decode(oracle.Config.from_workload(w), oracle.Catalog(sids, w.codebook_sizes))
    got_sids = np.concatenate([np.array(s[1]) for s in sorted(shards, key=lambda s: s[0])])
    got_scores = np.concatenate([np.array(s[2]) for s in sorted(shards, key=lambda s: s[0])])
    np.testing.assert_array_equal(got_sids, full.sids)
    np.testing.assert_array_equal(got_scores, full.scores)


def test_rank_layout_and_job_throughput():
    assert bench.rank_requests(0, 4, 32) == (0, 32)
    assert bench.rank_requests(3, 4, 32) == (96, 32)
    with pytest.raises(ValueError):
        bench.rank_requests(4, 4, 32)
    assert bench.max_over_ranks(1.5, 1) == 1.5
    # 4 ranks x 24,576 candidates x 10 decodes in 11.3 ms
    assert bench.job_throughput(4, 24576, 10, 11.3) == pytest.approx(4 * 24576 * 10 / 0.0113)
