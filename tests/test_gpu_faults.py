"""Failure detection without a GPU fault: a bounded wait that runs out.

The block-level indexer's copy ring waits on mbarriers with a poll limit.  A
test hook lowers that limit to zero, so every wait of the ring gives up at
once: the kernel must still drain its own copies, reach every barrier and
return, set CSA2_DEV_TIMEOUT in the caller's error word, and leave the context
and the workspace usable, so that the next call (default limit) is exact.
Nothing here faults, traps or hangs: a wait that gives up only skips the
synchronisation, and every copy stays inside the cache and the CTA's staging
ring.
"""
import numpy as np
import pytest
import torch

import synth
from _gpu_util import PagedSeqs, bits16, check_sets, dev

pytestmark = pytest.mark.gpu
SEED = 1002
DEV_TIMEOUT = 0x10


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def test_block_indexer_wait_runs_out_and_reports(csa2, orc):
    lens = [70000, 20001]  # > 2048 blocks each: the block-scoring ring runs
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens)
    for b, L in enumerate(lens):
        ps.append(b, 0, synth.kv_rows(SEED, b, 0, L), synth.idx_k_rows(SEED, b, 0, L))
    sl = dev(np.array(lens, np.int32))
    d = csa2.default_desc(csa2.FULL, 1)
    ws = torch.zeros(csa2.workspace_bytes(d, csa2.BLOCK, B, max_len), dtype=torch.uint8, device="cuda")
    q = bits16(np.concatenate([synth.q_idx(SEED, 0, b) for b in range(B)]))
    w = dev(np.concatenate([synth.w_idx(SEED, 0, b) for b in range(B)]))
    blocks = torch.empty((B, 2048), dtype=torch.int32, device="cuda")

    prev = csa2.test_set_wait_limit(0)
    try:
        csa2.indexer_topk(d, ps.cache, csa2.BLOCK, q, w, sl, blocks, B, max_len, ws, err=ps.err)
        torch.cuda.synchronize()  # the kernels returned: no wait hung
        flags = int(ps.err.item())
    finally:
        assert csa2.test_set_wait_limit(prev) == 0
    assert flags & DEV_TIMEOUT, f"error word {flags:#x}: the timeout was not reported"

    # the context and the workspace are intact: the next call is exact
    ps.err.zero_()
    csa2.indexer_topk(d, ps.cache, csa2.BLOCK, q, w, sl, blocks, B, max_len, ws, err=ps.err)
    assert ps.errors() == 0
    got = blocks.cpu().numpy()
    for b, L in enumerate(lens):
        idx = synth.idx_k_rows(SEED, b, 0, L)
        want = orc.select_blocks(orc.pool_blocks(idx), L, synth.q_idx(SEED, 0, b)[0], synth.w_idx(SEED, 0, b)[0])
        check_sets(got[b], want, f"block set of sequence {b} after the timeout")
