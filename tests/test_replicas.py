"""Data-parallel replicas on the host: two gloo ranks on CPU.

Each rank owns its own sequences (no data-path collective); the only
collective is the maximum of the ranks' times.  A rank's inputs are exactly
the inputs of the same global sequences in a single run.
"""
import datetime
import os
import socket

import numpy as np
import pytest

from rank_kv_cache_lrkv_b200 import replicas
from rank_kv_cache_lrkv_b200 import workloads as wk

BASE = wk.QWEN3_LAYER_8K.with_(T=64, n_decode=2, B=2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = replicas.shard(BASE, rank, world)
        k = np.stack([wk.stream(wl, "k", 0, b, 0, n=8) for b in range(wl.B)])
        qv = wk.queries(wl, 0, 1)
        t_max = replicas.max_over_ranks(10.0 + 3.0 * rank, world)
        owned = torch.tensor(list(replicas.owned_sequences(BASE, rank, world)))
        got = [torch.zeros_like(owned) for _ in range(world)]
        dist.all_gather(got, owned)
        q.put((rank, t_max, [g.tolist() for g in got], k, qv))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(60)
            if p.is_alive():
                p.terminate()
    assert [p.exitcode for p in procs] == [0, 0]
    # the job time is the slowest rank's, on every rank
    assert [r[1] for r in res] == [13.0, 13.0]
    # disjoint shards covering the global sequences
    assert res[0][2] == [[0, 1], [2, 3]] == res[1][2]
    # rank r's sequence b is global sequence r * B + b of one run
    glob = BASE.with_(B=4)
    qg = wk.queries(glob, 0, 1)
    for rank, _, _, k, qv in res:
        for b in range(BASE.B):
            g = rank * BASE.B + b
            np.testing.assert_array_equal(k[b], wk.stream(glob, "k", 0, g, 0, n=8))
            np.testing.assert_array_equal(qv[b], qg[g])
    # the two shards differ
    assert not np.array_equal(res[0][3], res[1][3])


def test_single_rank_and_rates():
    assert replicas.max_over_ranks(5.5, 1) == 5.5
    assert replicas.shard(BASE, 0, 1) == BASE
    assert list(replicas.owned_sequences(BASE, 1, 3)) == [2, 3]
    with pytest.raises(ValueError):
        replicas.shard(BASE, 2, 2)
    # whole-job rate: B tokens per step per rank over the slowest rank's time
    assert replicas.aggregate_tokens_per_s(4, 256, 2, 50.0) == pytest.approx(4 * 256 * 2 / 0.05)
    with pytest.raises(ValueError):
        replicas.aggregate_tokens_per_s(4, 256, 2, 0.0)
