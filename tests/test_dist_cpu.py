"""Multi-rank host logic of bench.py on CPU ranks (gloo, world size 2): the
step time is the max over ranks and the value aggregates every rank's batch."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [3.0, 5.0][rank]
    got = bench.max_over_ranks(ms, world, "cpu")
    q.put((rank, got, bench.whole_job_tokens_per_s(8, world, got)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == 5.0                          # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 8 / 5e-3)  # both ranks' sequences per slowest step


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.whole_job_tokens_per_s(8, 1, 2.0) == pytest.approx(4000.0)


def test_encoder_workload_and_bytes():
    import bench
    W = bench.workload(6)
    assert (W["ratio"], W["decoder"], W["layers"], W["B"], W["L"]) == (2, False, 18, 8, 1 << 19)
    ub = bench.unique_bytes_per_seq_flat(W["L"], W["layers"], 3, W["ratio"])
    assert ub["index"] == 3 * (1 << 19) * 128  # every Full layer streams the whole indexer K
    assert ub["kv"] == 3 * 512 * 144 and ub["swa"] == 18 * 128 * 512
    assert ub["total"] == sum(v for k, v in ub.items() if k != "total")
    dec = bench.workload(4)
    assert (dec["ratio"], dec["decoder"], dec["layers"]) == (1, True, 20)
