"""The C-ABI library loads, exports every symbol include/csa2.h declares, and
rejects bad arguments on the host before touching the GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def csa2():
    from fp4_kv_cache_nvfp4_b200 import build
    build.build()
    import fp4_kv_cache_nvfp4_b200 as m
    return m


def _declared():
    with open(os.path.join(ROOT, "include", "csa2.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", src)))


def test_header_declares_the_abi():
    names = _declared()
    for n in ("csa2_kv_quant_append", "csa2_indexer_topk", "csa2_sparse_attn_decode", "csa2_sparse_attn_prefill",
              "csa2_decode_layers", "csa2_indexer_workspace_bytes"):
        assert n in names


def test_every_declared_symbol_is_exported(csa2):
    L = csa2.lib()
    for n in _declared():
        assert hasattr(L, n), n
    assert csa2.abi_version() == 1
    assert csa2.device_accessible(None) == 0  # answered before any CUDA call


def test_schedule_and_defaults(csa2):
    F, RI, R = csa2.FULL, csa2.REINDEX, csa2.REUSE
    assert csa2.schedule(True) == [F, R, R, R] + [RI, R, R, R] * 4
    assert csa2.schedule(False) == [F, R, R, R, R, R] * 3
    d = csa2.default_desc(csa2.FULL, 1)
    assert (d.topk, d.block, d.keep_blocks, d.window, d.n_heads, d.head_dim, d.idx_heads, d.idx_dim) == \
        (512, 8, 2048, 128, 16, 128, 4, 64)


def _cache_struct(csa2, **over):
    c = csa2._binding._Cache(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 64, 16, 4)
    for k, v in over.items():
        setattr(c, k, v)
    return c


def test_host_validation_without_gpu(csa2):
    L = csa2.lib()
    d = csa2.default_desc(csa2.FULL, 1)
    c = _cache_struct(csa2)
    P = ctypes.c_void_p
    ws = 0x100000
    # bad dimensions -> UNSUPPORTED; bad sizes/modes -> INVALID_ARG; small workspace -> WORKSPACE
    bad = csa2.default_desc(csa2.FULL, 1, n_heads=8)
    assert L.csa2_sparse_attn_decode(ctypes.byref(bad), ctypes.byref(c), P(0x1000), P(0x1000), P(0x1000),
                                     P(0x1000), None, P(0x1000), P(0x1000), 1, None, None) == 2
    reuse = csa2.default_desc(csa2.REUSE, 1)
    assert L.csa2_indexer_topk(ctypes.byref(reuse), ctypes.byref(c), 0, P(0x1000), P(0x1000), P(0x1000), None, None,
                               P(0x1000), None, 1, 1000, P(ws), 1 << 30, None, None) == 1
    assert L.csa2_indexer_topk(ctypes.byref(d), ctypes.byref(c), 0, P(0x1000), P(0x1000), P(0x1000), None, None,
                               P(0x1000), None, 1, 1000, P(ws), 16, None, None) == 4
    assert L.csa2_indexer_topk(ctypes.byref(d), ctypes.byref(c), 7, P(0x1000), P(0x1000), P(0x1000), None, None,
                               P(0x1000), None, 1, 1000, P(ws), 1 << 30, None, None) == 1
    big = csa2.default_desc(csa2.FULL, 1, topk=513)
    assert L.csa2_sparse_attn_decode(ctypes.byref(big), ctypes.byref(c), P(0x1000), P(0x1000), P(0x1000),
                                     P(0x1000), None, P(0x1000), P(0x1000), 1, None, None) == 1
    # misaligned pointers and bad cache geometry
    assert L.csa2_sparse_attn_decode(ctypes.byref(d), ctypes.byref(c), P(0x1000), P(0x1000), P(0x1001),
                                     P(0x1000), None, P(0x1000), P(0x1000), 1, None, None) == 1
    # the prefill indexer reads q_idx in 16-byte rows: 4-byte alignment is rejected
    assert L.csa2_indexer_topk(ctypes.byref(csa2.default_desc(csa2.FULL, 2)), ctypes.byref(c), 1, P(0x1004),
                               P(0x1000), P(0x1000), P(0x1000), None, P(0x1000), None, 1, 1000, P(ws), 1 << 30, None,
                               None) == 1
    # prefill attention loads q and writes out in 16-byte vectors: 4-byte alignment is rejected
    for qp, op in ((0x1004, 0x1000), (0x1000, 0x1004)):
        assert L.csa2_sparse_attn_prefill(ctypes.byref(d), ctypes.byref(c), P(qp), P(0x1000), P(0x1000), P(0x1000),
                                          0, 1, P(op), P(0x1000), 1, None, None) == 1
    c2 = _cache_struct(csa2, page_size=12)
    assert L.csa2_kv_quant_append(ctypes.byref(c2), P(0x1000), 0, None, 1, 1, P(0x1000), None, None) == 1
    assert L.csa2_kv_quant_append(ctypes.byref(c), P(0x1000), 0, None, 1, 3, P(0x1000), None, None) == 1
    assert L.csa2_kv_quant_append(ctypes.byref(c), None, 0, None, 0, 1, None, None, None) == 0  # empty: no-op
    assert L.csa2_sparse_attn_decode(ctypes.byref(d), ctypes.byref(c), None, None, None, None, None, None, None, 0,
                                     None, None) == 0
    # a Reindex or Reuse first layer is rejected by the schedule driver
    descs = (csa2.LayerDesc * 2)(csa2.default_desc(csa2.REUSE, 1), d)
    ptrs = (ctypes.c_void_p * 2)(0x1000, 0x1000)
    assert L.csa2_decode_layers(2, descs, ctypes.byref(c), ptrs, ptrs, ptrs, ptrs, P(0x1000), None, P(0x1000),
                                P(0x1000), ptrs, ptrs, 1, 1000, P(ws), 1 << 30, None, None) == 1
    # block-level context above the compiled limit; prefill above 16,384 entries
    assert L.csa2_indexer_topk(ctypes.byref(d), ctypes.byref(c), 0, P(0x1000), P(0x1000), P(0x1000), None, None,
                               P(0x1000), None, 1, (1 << 21) + 1, P(ws), 1 << 40, None, None) == 2
    assert L.csa2_status_string(3) == b"CUDA error"


def test_workspace_sizes(csa2):
    d = csa2.default_desc(csa2.FULL, 1)
    small = csa2.workspace_bytes(d, csa2.TOKEN, 8, 4096)
    big = csa2.workspace_bytes(d, csa2.BLOCK, 8, 1 << 20)
    assert 0 < small < big
    assert big % 256 == 0
    # block arrays: scores + bitmap + boundary list per sequence at 131,072 blocks
    assert big >= 8 * (131072 * (4 + 8) + 131072 // 8)
    assert csa2.workspace_bytes(d, csa2.TOKEN, 4096, 16384, prefill=True) >= 4096 * 16384 * 4


def test_flat_indexer_arguments(csa2):
    """keep_blocks = 0 removes the block level (the encoder's layers): the
    indexer then runs at TOKEN level over every entry, with no candidates, up
    to 2^21 entries, and its workspace holds one row per entry."""
    L = csa2.lib()
    c = _cache_struct(csa2)
    P = ctypes.c_void_p
    ws = 0x100000
    flat = csa2.default_desc(csa2.FULL, 2, keep_blocks=0)
    # no BLOCK level without blocks
    assert L.csa2_indexer_topk(ctypes.byref(flat), ctypes.byref(c), csa2.BLOCK, P(0x1000), P(0x1000), P(0x1000),
                               None, None, P(0x1000), None, 1, 1000, P(ws), 1 << 30, None, None) == 1
    # no candidate blocks for a flat layer
    assert L.csa2_indexer_topk(ctypes.byref(flat), ctypes.byref(c), csa2.TOKEN, P(0x1000), P(0x1000), P(0x1000),
                               None, P(0x1000), P(0x1000), None, 1, 1000, P(ws), 1 << 30, None, None) == 1
    # above the compiled limit of 2^21 entries
    assert L.csa2_indexer_topk(ctypes.byref(flat), ctypes.byref(c), csa2.TOKEN, P(0x1000), P(0x1000), P(0x1000),
                               None, None, P(0x1000), None, 1, (1 << 21) + 1, P(ws), 1 << 40, None, None) == 2
    # within the limits the call gets as far as the workspace check
    assert L.csa2_indexer_topk(ctypes.byref(flat), ctypes.byref(c), csa2.TOKEN, P(0x1000), P(0x1000), P(0x1000),
                               None, None, P(0x1000), None, 1, 1000, P(ws), 16, None, None) == 4
    # a negative keep_blocks is still rejected
    bad = csa2.default_desc(csa2.FULL, 2, keep_blocks=-1)
    assert L.csa2_indexer_topk(ctypes.byref(bad), ctypes.byref(c), csa2.TOKEN, P(0x1000), P(0x1000), P(0x1000),
                               None, None, P(0x1000), None, 1, 1000, P(ws), 1 << 30, None, None) == 1
    # workspace: scores, boundary list and two bitmaps per entry, not per block
    hier = csa2.workspace_bytes(csa2.default_desc(csa2.FULL, 2), csa2.BLOCK, 8, 1 << 20)
    fl = csa2.workspace_bytes(flat, csa2.TOKEN, 8, 1 << 20)
    assert fl > hier and fl % 256 == 0
    assert fl >= 8 * ((1 << 20) * (4 + 8) + 2 * (1 << 20) // 8)
    # the decode driver takes flat layers without a cand_blocks buffer (and
    # still needs its workspace)
    descs = (csa2.LayerDesc * 2)(flat, csa2.default_desc(csa2.REUSE, 2, keep_blocks=0))
    ptrs = (ctypes.c_void_p * 2)(0x1000, 0x1000)
    assert L.csa2_decode_layers(2, descs, ctypes.byref(c), ptrs, ptrs, ptrs, ptrs, P(0x1000), None, None,
                                P(0x1000), ptrs, ptrs, 1, 1000, P(ws), 16, None, None) == 4
    assert L.csa2_decode_layers(2, descs, None, ptrs, ptrs, ptrs, ptrs, P(0x1000), None, None,
                                P(0x1000), ptrs, ptrs, 1, 1000, P(ws), 1 << 30, None, None) == 1  # no cache
    hdesc = (csa2.LayerDesc * 2)(csa2.default_desc(csa2.FULL, 1), csa2.default_desc(csa2.REUSE, 1))
    assert L.csa2_decode_layers(2, hdesc, ctypes.byref(c), ptrs, ptrs, ptrs, ptrs, P(0x1000), None, None,
                                P(0x1000), ptrs, ptrs, 1, 1000, P(ws), 1 << 30, None, None) == 1


def test_noalloc_scratch_limits_per_mode(csa2):
    """The allocation-free indexer's 16 MiB scratch holds the hierarchical
    layout of 8 sequences of 2^20 entries, the flat layout of one such
    sequence, but not the flat layout of two (flat rows are entries, not
    blocks of 8)."""
    lim = 16 << 20
    hier = csa2.default_desc(csa2.FULL, 1)
    flat = csa2.default_desc(csa2.FULL, 2, keep_blocks=0)
    assert csa2.workspace_bytes(hier, csa2.BLOCK, 8, 1 << 20) <= lim
    assert csa2.workspace_bytes(flat, csa2.TOKEN, 1, 1 << 20) <= lim
    assert csa2.workspace_bytes(flat, csa2.TOKEN, 2, 1 << 20) > lim
    assert csa2.workspace_bytes(hier, csa2.BLOCK, 64, 1 << 20) > lim
