"""The allocation-free decode indexer (csa2_indexer_topk_noalloc) against the
workspace one (csa2_indexer_topk).

Some callers cannot allocate device memory where they run the indexer (while
a CUDA graph is being captured, inside a framework that owns all device
memory, in a serving loop that must not touch the allocator).  The no-alloc
entry point serves them from a static 16 MiB scratch inside the library; it
must give exactly the selections the workspace entry point gives, call after
call, even though every call reuses the same scratch.  This file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from _gpu_util import PagedSeqs, bits16, check_sets, dev

pytestmark = pytest.mark.gpu
SEED = 1001


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def _fill(ps, seq, L):
    ps.append(seq, 0, synth.kv_rows(SEED, seq, 0, L), synth.idx_k_rows(SEED, seq, 0, L))


def test_noalloc_indexer_matches_workspace_indexer(csa2):
    lens = [20001, 70000, 3000, 16384]
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens)
    for b, L in enumerate(lens):
        _fill(ps, b, L)
    sl = dev(np.array(lens, np.int32))
    d = csa2.default_desc(csa2.FULL, 1)
    ws = torch.zeros(csa2.workspace_bytes(d, csa2.BLOCK, B, max_len), dtype=torch.uint8, device="cuda")
    q0 = bits16(np.concatenate([synth.q_idx(SEED, 0, b) for b in range(B)]))
    w0 = dev(np.concatenate([synth.w_idx(SEED, 0, b) for b in range(B)]))
    q4 = bits16(np.concatenate([synth.q_idx(SEED, 4, b) for b in range(B)]))
    w4 = dev(np.concatenate([synth.w_idx(SEED, 4, b) for b in range(B)]))

    ref_blocks = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    ref_tok = torch.empty((B, 512), dtype=torch.int32, device="cuda")
    ref_rei = torch.empty((B, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.BLOCK, q0, w0, sl, ref_blocks, B, max_len, ws, err=ps.err)
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, q0, w0, sl, ref_tok, B, max_len, ws, cand_blocks=ref_blocks,
                      err=ps.err)
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, q4, w4, sl, ref_rei, B, max_len, ws, cand_blocks=ref_blocks,
                      err=ps.err)
    torch.cuda.synchronize()

    for call in range(2):  # two calls in a row share (and reuse) the static scratch
        blocks = torch.full((B, 2048), -5, dtype=torch.int32, device="cuda")
        tok = torch.full((B, 512), -5, dtype=torch.int32, device="cuda")
        rei = torch.full((B, 512), -5, dtype=torch.int32, device="cuda")
        csa2.indexer_topk_noalloc(d, ps.cache, csa2.BLOCK, q0, w0, sl, blocks, B, max_len, err=ps.err)
        csa2.indexer_topk_noalloc(d, ps.cache, csa2.TOKEN, q0, w0, sl, tok, B, max_len, cand_blocks=blocks,
                                  err=ps.err)
        csa2.indexer_topk_noalloc(d, ps.cache, csa2.TOKEN, q4, w4, sl, rei, B, max_len, cand_blocks=blocks,
                                  err=ps.err)
        torch.cuda.synchronize()
        check_sets(blocks.cpu().numpy(), ref_blocks.cpu().numpy(), f"block level, call {call}")
        check_sets(tok.cpu().numpy(), ref_tok.cpu().numpy(), f"token level, call {call}")
        check_sets(rei.cpu().numpy(), ref_rei.cpu().numpy(), f"token level (Reindex q), call {call}")
    assert ps.errors() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(csa2):
    d = csa2.default_desc(csa2.FULL, 1)
    # 64 sequences of 2^20 entries need far more than the 16 MiB scratch
    assert csa2.workspace_bytes(d, csa2.BLOCK, 64, 1 << 20) > 16 << 20
    # a cache descriptor large enough for that request; the call is rejected on
    # the host before any pointer is used
    cache = csa2._binding._Cache(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 64, 16384, 64 * 16384)
    L = csa2.lib()
    P = ctypes.c_void_p
    st = L.csa2_indexer_topk_noalloc(ctypes.byref(d), ctypes.byref(cache), csa2.BLOCK, P(0x1000), P(0x1000),
                                     P(0x1000), None, P(0x1000), 64, 1 << 20, None, None)
    assert st == 4  # CSA2_ERR_WORKSPACE


def test_noalloc_flat_indexer_matches_workspace_indexer(csa2):
    """The flat indexer (keep_blocks = 0, Top-512 over every entry) through the
    static scratch, twice, against the workspace entry point."""
    lens = [70000, 300, 40000]
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens)
    for b, L in enumerate(lens):
        _fill(ps, b, L)
    sl = dev(np.array(lens, np.int32))
    d = csa2.default_desc(csa2.FULL, 2, keep_blocks=0)
    ws = torch.zeros(csa2.workspace_bytes(d, csa2.TOKEN, B, max_len), dtype=torch.uint8, device="cuda")
    q = bits16(np.concatenate([synth.q_idx(SEED, 6, b) for b in range(B)]))
    w = dev(np.concatenate([synth.w_idx(SEED, 6, b) for b in range(B)]))
    ref = torch.empty((B, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, q, w, sl, ref, B, max_len, ws, err=ps.err)
    for call in range(2):
        got = torch.full((B, 512), -5, dtype=torch.int32, device="cuda")
        csa2.indexer_topk_noalloc(d, ps.cache, csa2.TOKEN, q, w, sl, got, B, max_len, err=ps.err)
        torch.cuda.synchronize()
        check_sets(got.cpu().numpy(), ref.cpu().numpy(), f"flat, call {call}")
    assert ps.errors() == 0
