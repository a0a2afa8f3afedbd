"""Context-parallel decode on CPU: the exchange protocol of
fp4_kv_cache_nvfp4_b200.context_parallel on gloo ranks (world size 2 and 4,
one shard per rank) and with every shard in one process, the kernels replaced
by the oracle on each shard's entries.  The merged index sets must equal the
single-sequence oracle's exactly, the merged attention within the tolerance."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import _cp_util as U

LENS = [40000, 36500]  # > 2048 blocks each: the block level runs on the whole sequence


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _span(G):
    return (max(LENS) + G - 1) // G // 64 * 64 + 64  # a multiple of the page size


def _run(orc, G, owned, exchange):
    from fp4_kv_cache_nvfp4_b200 import context_parallel as cp
    data = U.seq_data(orc, LENS)
    q_idx, w, q, swa = U.layer_inputs(len(LENS))
    modes = orc.schedule(True)[:U.N_LAYERS]
    import torch
    swa_lens = torch.tensor([min(128, L) for L in LENS], dtype=torch.int32)
    shards = U.cpu_shards(LENS, G, _span(G), owned)
    ops = U.OracleOps(orc, data, len(LENS))
    res = cp.decode_step(modes, [None] * len(modes), shards, ops, exchange, *U.torch_inputs(q_idx, w, q, swa),
                         swa_lens)
    return res, data, (q_idx, w, q, swa), modes


@pytest.mark.parametrize("G", [2, 4])
def test_all_shards_in_one_process(orc, G):
    from fp4_kv_cache_nvfp4_b200 import context_parallel as cp
    assert all(L > (G - 1) * _span(G) for L in LENS)
    res, data, (q_idx, w, q, swa), modes = _run(orc, G, None, cp.LocalExchange())
    ref = U.reference(orc, data, LENS, modes, q_idx, w, q, swa)
    U.compare(res, ref, LENS, modes, f"G={G} local", atol=1e-5, rtol_l2=1e-5)


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        from fp4_kv_cache_nvfp4_b200 import context_parallel as cp
        oracle.build()
        res, data, (q_idx, w, q_, swa), modes = _run(oracle, world, [rank], cp.DistExchange())
        if rank == 0:
            ref = U.reference(oracle, data, LENS, modes, q_idx, w, q_, swa)
            U.compare(res, ref, LENS, modes, f"gloo world {world}", atol=1e-5, rtol_l2=1e-5)
        # every rank holds the same merged results
        first = np.concatenate([r["out"].numpy().ravel() for r in res])
        q.put((rank, float(first.sum()), [r["idx"].numpy().tolist() for r in res[:1]]))
    except Exception as e:  # report to the parent instead of hanging the others
        q.put((rank, repr(e), None))
        raise
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_one_shard_each(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=600) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, s, sets in res:
        assert sets is not None, f"rank {rank}: {s}"
    assert len({s for _, s, _ in res}) == 1           # same merged output on every rank
    assert len({str(x) for _, _, x in res}) == 1      # same merged sets on every rank
