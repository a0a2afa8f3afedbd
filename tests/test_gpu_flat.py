"""The flat indexer (no block level: the encoder's CSA2 layers) and the
encoder-side decode step, CUDA path vs the CPU oracle.

A layer descriptor with keep_blocks = 0 selects the Top-512 over every entry
of the context.  Above 16,384 entries the block-level kernels run with one row
per entry; at or below it the token kernel takes all entries as one candidate
set.  Sets are bit-exact; attention within max-abs 2e-3 and rel-L2 1e-3."""
import numpy as np
import pytest
import torch

import synth
from _gpu_util import (PagedSeqs, bits16, check_sets, compare_encoder_seq, dev, encoder_layer_inputs,
                       run_encoder_step)

pytestmark = pytest.mark.gpu
SEED = 1006


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


CHUNK = 1 << 16


def _fill(ps, seq, L, ratio=2, seed=SEED, keep_kv=True, idx=None):
    """Append L entries (64K at a time); return (kv rows or None, indexer K)."""
    idx = synth.idx_k_rows(seed, seq, 0, L) if idx is None else idx
    kvs = []
    for e0 in range(0, L, CHUNK):
        m = min(CHUNK, L - e0)
        kv = synth.kv_rows(seed, seq, e0 * ratio, m * ratio)
        ps.append(seq, e0, kv, idx[e0:e0 + m], ratio=ratio)
        if keep_kv:
            kvs.append(kv)
    return (np.concatenate(kvs) if keep_kv else None), idx


def _flat_desc(csa2, mode=0):
    return csa2.default_desc(mode, 2, keep_blocks=0)


def _ws(csa2, n, max_len):
    return torch.zeros(csa2.workspace_bytes(_flat_desc(csa2), csa2.TOKEN, n, max_len), dtype=torch.uint8,
                       device="cuda")


def _q(B, layer=0, seed=SEED):
    q = np.concatenate([synth.q_idx(seed, layer, b) for b in range(B)])
    w = np.concatenate([synth.w_idx(seed, layer, b) for b in range(B)])
    return q, w


def _run_flat(csa2, ps, lens, q, w, ws=None):
    B, max_len = len(lens), max(lens)
    ws = _ws(csa2, B, max_len) if ws is None else ws
    out = torch.full((B, 512), -7, dtype=torch.int32, device="cuda")
    csa2.indexer_topk(_flat_desc(csa2), ps.cache, csa2.TOKEN, bits16(q), dev(w), dev(np.array(lens, np.int32)), out,
                      B, max_len, ws, err=ps.err)
    return out.cpu().numpy()


# 300,000 entries: more than 262,144 rows, so the selection's final pass works
# on the bitmaps in global memory; 20,001 and 70,000 keep them in shared memory.
@pytest.mark.parametrize("page_size", [64, 8, 1024])  # 64, 1024: rows as tensor boxes; 8: 16-byte copies
def test_flat_indexer_bitexact(csa2, orc, page_size):
    lens = [20001, 70000, 300000, 3000, 400, 1]
    B = len(lens)
    ps = PagedSeqs(csa2, lens, page_size=page_size)
    idxs = [_fill(ps, b, L, keep_kv=False)[1] for b, L in enumerate(lens)]
    ws = _ws(csa2, B, max(lens))
    for layer in (0, 6):  # two calls on one workspace: it is left clean
        q, w = _q(B, layer)
        got = _run_flat(csa2, ps, lens, q, w, ws)
        for b, L in enumerate(lens):
            check_sets(got[b], orc.select_tokens(idxs[b], L, None, q[b], w[b]), f"layer {layer} seq {b} (L={L})")
    assert ps.errors() == 0


def test_flat_indexer_one_candidate_set(csa2, orc):
    """At most 16,384 entries: the whole context is one candidate set."""
    lens = [16384, 513, 5]
    B = len(lens)
    ps = PagedSeqs(csa2, lens)
    idxs = [_fill(ps, b, L)[1] for b, L in enumerate(lens)]
    q, w = _q(B, 12)
    got = _run_flat(csa2, ps, lens, q, w)
    for b, L in enumerate(lens):
        check_sets(got[b], orc.select_tokens(idxs[b], L, None, q[b], w[b]), f"seq {b}")
    assert ps.errors() == 0


def test_flat_indexer_ties_and_planted(csa2, orc):
    """All scores 0: the 512 lowest positions.  Then a query that favours 300
    planted entries spread over the context: they all make the set, and the
    remaining 212 places go to the lowest-index entries of the tied rest."""
    L = 300000
    ps = PagedSeqs(csa2, [L])
    rng = np.random.default_rng(3)
    kf = np.zeros((L, 64), np.float32)
    hot = np.sort(rng.choice(L, 300, replace=False))
    kf[hot, 5] = 1.0 + rng.random(300).astype(np.float32)
    idx = synth.to_bf16_bits(kf)
    _fill(ps, 0, L, keep_kv=False, idx=idx)
    w = np.ones((1, 4), np.float32)
    zero = np.zeros((1, 4, 64), np.uint16)
    assert _run_flat(csa2, ps, [L], zero, w)[0].tolist() == list(range(512))
    qf = np.zeros((1, 4, 64), np.float32)
    qf[0, :, 5] = 1.0
    q = synth.to_bf16_bits(qf)
    got = _run_flat(csa2, ps, [L], q, w)[0]
    want = orc.select_tokens(idx, L, None, q[0], w[0])
    check_sets(got, want, "planted")
    assert set(hot.tolist()) <= set(got.tolist())
    assert ps.errors() == 0


def test_encoder_decode_layers_vs_oracle(csa2, orc):
    lens = [40000, 9000, 130]
    B = len(lens)
    ps = PagedSeqs(csa2, lens)
    data = [_fill(ps, b, L) for b, L in enumerate(lens)]
    q_idx, w, q, swa = encoder_layer_inputs(SEED, B, lens, 18)
    snap = [t.clone() for t in (ps.cache.codes, ps.cache.scales, ps.cache.idx_k)]
    r = run_encoder_step(csa2, ps, lens, q_idx, w, q, swa)
    for a, b_ in zip(snap, (ps.cache.codes, ps.cache.scales, ps.cache.idx_k)):
        assert torch.equal(a, b_)
    for b, L in enumerate(lens):
        codes, scales = orc.quant_rows(data[b][0], ratio=2)
        compare_encoder_seq(orc, r, b, L, codes, scales, data[b][1], q_idx[b], w[b], q[b], swa[b], f"seq {b}")
    assert ps.errors() == 0


def test_flat_indexer_few_ties_at_the_boundary(csa2, orc):
    """500 high rows and 30 identical rows just below them: the K-th score is
    shared by the 30, and the 12 lowest-index ones complete the set (the
    selection's list-and-sort path, which handles up to 256 ties)."""
    L = 300000
    ps = PagedSeqs(csa2, [L])
    rng = np.random.default_rng(4)
    kf = np.zeros((L, 64), np.float32)
    picks = rng.choice(L, 530, replace=False)
    hot, tied = picks[:500], np.sort(picks[500:])
    kf[hot, 5] = 2.0 + rng.random(500).astype(np.float32)
    kf[tied, 5] = 1.5
    idx = synth.to_bf16_bits(kf)
    _fill(ps, 0, L, keep_kv=False, idx=idx)
    qf = np.zeros((1, 4, 64), np.float32)
    qf[0, :, 5] = 1.0
    q, w = synth.to_bf16_bits(qf), np.ones((1, 4), np.float32)
    got = _run_flat(csa2, ps, [L], q, w)[0]
    check_sets(got, orc.select_tokens(idx, L, None, q[0], w[0]), "ties")
    assert set(tied[:12].tolist()) <= set(got.tolist()) and not set(tied[12:].tolist()) & set(got.tolist())
    assert ps.errors() == 0
