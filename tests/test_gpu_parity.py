"""CUDA path vs the CPU oracle, element by element, on seeded inputs spanning
several tiles and ragged tails.  Bit-exact for codes, scales, indexer K,
pooled K and Top-K sets; attention within max-abs 2e-3 and rel-L2 1e-3."""
import numpy as np
import pytest
import torch

import synth
from _gpu_util import PagedSeqs, bits16, check_attn, check_sets, dev

pytestmark = pytest.mark.gpu
SEED = 1001


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def _fill(ps, seq, L, ratio=1, chunk=None, bf16=False, seed=SEED):
    kv = synth.kv_rows(seed, seq, 0, L * ratio)
    idx = synth.idx_k_rows(seed, seq, 0, L)
    src = synth.to_bf16_bits(kv) if bf16 else kv
    ps.append(seq, 0, src, idx, ratio=ratio, chunk=chunk)
    return kv, idx


# ---------------------------------------------------------------------------
# quant-append
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("ratio,bf16,chunk", [(1, False, None), (1, False, 37), (1, True, 1000), (2, False, 513),
                                              (2, True, None)])
def test_quant_append_bitexact(csa2, orc, ratio, bf16, chunk):
    lens = [4096 + 37, 1000, 9]
    ps = PagedSeqs(csa2, lens)
    for b, L in enumerate(lens):
        kv, idx = _fill(ps, b, L, ratio=ratio, chunk=chunk, bf16=bf16)
        if bf16:
            kv = orc.bf16_to_f32(synth.to_bf16_bits(kv)).reshape(kv.shape)
        codes, scales = orc.quant_rows(kv, ratio=ratio)
        gc, gs, gk, gp = ps.unpage(b, L)
        np.testing.assert_array_equal(gc, codes)
        np.testing.assert_array_equal(gs, scales)
        np.testing.assert_array_equal(gk, idx)
        np.testing.assert_array_equal(gp, orc.pool_blocks(idx))
    assert ps.errors() == 0


def test_quant_append_decode_steps(csa2, orc):
    """One entry per sequence per call, the way a decode step appends."""
    lens = [70, 9]
    ps = PagedSeqs(csa2, lens)
    kvs = [synth.kv_rows(SEED, b, 0, L) for b, L in enumerate(lens)]
    idxs = [synth.idx_k_rows(SEED, b, 0, L) for b, L in enumerate(lens)]
    for p in range(max(lens)):
        seqs = [b for b, L in enumerate(lens) if p < L]
        sl = np.concatenate([ps.slots(b, [p]) for b in seqs]).astype(np.int64)
        kv = np.concatenate([kvs[b][p:p + 1] for b in seqs])
        ik = np.concatenate([idxs[b][p:p + 1] for b in seqs])
        csa2.kv_quant_append(ps.cache, dev(kv), bits16(ik), dev(sl), err=ps.err)
    for b, L in enumerate(lens):
        gc, gs, gk, gp = ps.unpage(b, L)
        codes, scales = orc.quant_rows(kvs[b])
        np.testing.assert_array_equal(gc, codes)
        np.testing.assert_array_equal(gs, scales)
        np.testing.assert_array_equal(gp, orc.pool_blocks(idxs[b]))
    assert ps.errors() == 0


def test_quant_append_special_values(csa2, orc):
    x = np.zeros((4, 256), np.float32)
    x[0, :16] = [6, -6, 0.5, -0.5, 1, 1.5, 2, 3, 4, -4, 0, -0.0, 1.25, -2.5, 5, -0.01]
    x[1, :16] = 5.0 * 2.0 ** -10        # amax / 6 below 2^-10: zero scale
    x[2] = np.linspace(-1e4, 1e4, 256)  # saturating scales
    x[3, 16:32] = -0.0
    ps = PagedSeqs(csa2, [4])
    ps.append(0, 0, x, np.zeros((4, 64), np.uint16))
    gc, gs, _, _ = ps.unpage(0, 4)
    codes, scales = orc.quant_rows(x)
    np.testing.assert_array_equal(gc, codes)
    np.testing.assert_array_equal(gs, scales)


# ---------------------------------------------------------------------------
# indexer
# ---------------------------------------------------------------------------

def _ws(csa2, n, max_len, prefill=False):
    d = csa2.default_desc(csa2.FULL, 1)
    nb = csa2.workspace_bytes(d, csa2.BLOCK, n, max_len, prefill)
    return torch.zeros(nb, dtype=torch.uint8, device="cuda")


def _indexer_inputs(B, layer=0, seed=SEED):
    q = np.concatenate([synth.q_idx(seed, layer, b) for b in range(B)])
    w = np.concatenate([synth.w_idx(seed, layer, b) for b in range(B)])
    return q, w


@pytest.mark.parametrize("page_size", [64, 16])
def test_block_topk_bitexact(csa2, orc, page_size):
    # pooled rows in 1 KiB page runs (64 entries a page) or 256-byte ones (16)
    lens = [16392, 20001, 70000, 1000, 16384]
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens, page_size=page_size)
    idxs = [_fill(ps, b, L)[1] for b, L in enumerate(lens)]
    q, w = _indexer_inputs(B)
    ws = _ws(csa2, B, max_len)
    out = torch.full((B, 2048), -7, dtype=torch.int32, device="cuda")
    sl = dev(np.array(lens, np.int32))
    d = csa2.default_desc(csa2.FULL, 1)
    for rep in range(2):  # the workspace is left clean for the next call
        csa2.indexer_topk(d, ps.cache, csa2.BLOCK, bits16(q), dev(w), sl, out, B, max_len, ws, err=ps.err)
        got = out.cpu().numpy()
        for b, L in enumerate(lens):
            want = orc.select_blocks(orc.pool_blocks(idxs[b]), L, q[b], w[b])
            check_sets(got[b], want, f"seq {b} rep {rep}")
    assert ps.errors() == 0


def test_block_topk_all_ties(csa2, orc):
    L = 8 * 5000 + 3
    ps = PagedSeqs(csa2, [L])
    _fill(ps, 0, L)
    ws = _ws(csa2, 1, L)
    out = torch.empty((1, 2048), dtype=torch.int32, device="cuda")
    q = np.zeros((1, 4, 64), np.uint16)  # every score is 0: the lowest 2048 blocks win
    w = np.ones((1, 4), np.float32)
    csa2.indexer_topk(csa2.default_desc(), ps.cache, csa2.BLOCK, bits16(q), dev(w), dev(np.array([L], np.int32)),
                      out, 1, L, ws)
    assert out.cpu().numpy()[0].tolist() == list(range(2048))


@pytest.mark.parametrize("lens", [[16392, 20001, 70000], [1, 7, 8, 9, 511, 512, 513, 4096, 16384]])
def test_token_topk_bitexact(csa2, orc, lens):
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens)
    idxs = [_fill(ps, b, L)[1] for b, L in enumerate(lens)]
    ws = _ws(csa2, B, max_len)
    sl = dev(np.array(lens, np.int32))
    d = csa2.default_desc(csa2.FULL, 1)
    blocks = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    q0, w0 = _indexer_inputs(B, 0)
    csa2.indexer_topk(d, ps.cache, csa2.BLOCK, bits16(q0), dev(w0), sl, blocks, B, max_len, ws, err=ps.err)
    for layer in (0, 4):  # the Full layer's own q, then a Reindex layer's q on the same blocks
        q, w = _indexer_inputs(B, layer)
        out = torch.empty((B, 512), dtype=torch.int32, device="cuda")
        csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q), dev(w), sl, out, B, max_len, ws, cand_blocks=blocks,
                          err=ps.err)
        got = out.cpu().numpy()
        for b, L in enumerate(lens):
            ob = orc.select_blocks(orc.pool_blocks(idxs[b]), L, q0[b], w0[b])
            want = orc.select_tokens(idxs[b], L, ob, q[b], w[b])
            check_sets(got[b], want, f"layer {layer} seq {b}")
    if max_len <= 16384:  # flat path (no candidate blocks)
        out = torch.empty((B, 512), dtype=torch.int32, device="cuda")
        csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q0), dev(w0), sl, out, B, max_len, ws, err=ps.err)
        for b, L in enumerate(lens):
            check_sets(out.cpu().numpy()[b], orc.select_tokens(idxs[b], L, None, q0[b], w0[b]), f"flat {b}")
    assert ps.errors() == 0


def test_token_select_ties_and_wide_range(csa2, orc):
    # Two cases the token select's one-warp bin resolution does not cover.
    # Sequence 0: q = 0, so every score is 0 and all 16,384 candidates tie;
    # the lowest 512 positions win.  Sequence 1: one indexer-K row is +-2^100
    # with the signs of head 0's query, so its score lies ~100 binades above
    # the others and the K-th key falls more than 8 binades below the largest;
    # that entry is selected, the rest must match the oracle.  Both take the
    # three-digit select.
    lens = [20000, 20000]
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens)
    q, w = _indexer_inputs(B)
    q[0] = 0
    idx0 = synth.idx_k_rows(SEED, 0, 0, lens[0])
    kf = orc.bf16_to_f32(synth.idx_k_rows(SEED, 1, 0, lens[1])).reshape(lens[1], 64)
    qf = orc.bf16_to_f32(q[1]).reshape(4, 64)
    kf[12345] = np.where(qf[0] >= 0, 1.0, -1.0) * 2.0 ** 100
    idx1 = synth.to_bf16_bits(kf)
    for b, (L, idx) in enumerate(zip(lens, (idx0, idx1))):
        ps.append(b, 0, synth.kv_rows(SEED, b, 0, L), idx)
    ws = _ws(csa2, B, max_len)
    sl = dev(np.array(lens, np.int32))
    d = csa2.default_desc(csa2.FULL, 1)
    blocks = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.BLOCK, bits16(q), dev(w), sl, blocks, B, max_len, ws, err=ps.err)
    out = torch.empty((B, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q), dev(w), sl, out, B, max_len, ws, cand_blocks=blocks,
                      err=ps.err)
    got = out.cpu().numpy()
    assert got[0].tolist() == list(range(512))
    for b, idx in ((0, idx0), (1, idx1)):
        ob = orc.select_blocks(orc.pool_blocks(idx), lens[b], q[b], w[b])
        want = orc.select_tokens(idx, lens[b], ob, q[b], w[b])
        check_sets(got[b], want, f"seq {b}")
    assert 12345 in got[1].tolist()
    assert ps.errors() == 0


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _swa(B, L_list, layer=0, window=128, seed=SEED):
    s = np.zeros((B, window, 256), np.uint16)
    for b, L in enumerate(L_list):
        n = min(window, L)
        s[b, :n] = synth.swa_rows(seed, layer, b, n)
    return s


@pytest.mark.parametrize("mode", [0, 2])  # Full (gathers after the wait) and Reuse (gathers before it)
def test_attn_decode_parity(csa2, orc, mode):
    lens = [5000, 300, 100, 1]
    B = len(lens)
    ps = PagedSeqs(csa2, lens)
    data = [_fill(ps, b, L) for b, L in enumerate(lens)]
    rng = np.random.default_rng(0)
    idx = np.full((B, 512), -1, np.int32)
    for b, L in enumerate(lens):
        k = min(512, L)
        idx[b, :k] = np.sort(rng.choice(L, k, replace=False))
    idx[0, 100] = -1  # a hole in the middle of a set is skipped
    q = np.concatenate([synth.q_heads(SEED, 0, b) for b in range(B)])
    swa = _swa(B, lens)
    out = torch.empty((B, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_decode(csa2.default_desc(mode), ps.cache, bits16(q), dev(idx), bits16(swa),
                            dev(np.array(lens, np.int32)), out, lse, B, err=ps.err)
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    for b, L in enumerate(lens):
        codes, scales = orc.quant_rows(data[b][0])
        ro, rl = orc.attend(q[b], idx[b], codes, scales, swa[b, :min(128, L)])
        check_attn(o[b], l[b], ro, rl, f"seq {b}")
    assert ps.errors() == 0


def test_attn_decode_swa_lens(csa2, orc):
    L = 3000
    ps = PagedSeqs(csa2, [L, L])
    kv, _ = _fill(ps, 0, L)
    _fill(ps, 1, L)
    idx = np.tile(np.arange(0, 1024, 2, dtype=np.int32), (2, 1))
    q = np.concatenate([synth.q_heads(SEED, 3, b) for b in range(2)])
    swa = _swa(2, [L, L], layer=3)
    swl = np.array([128, 5], np.int32)
    out = torch.empty((2, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((2, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_decode(csa2.default_desc(), ps.cache, bits16(q), dev(idx), bits16(swa),
                            dev(np.array([L, L], np.int32)), out, lse, 2, swa_lens=dev(swl))
    kv1 = synth.kv_rows(SEED, 1, 0, L)
    c1, s1 = orc.quant_rows(kv1)
    ro, rl = orc.attend(q[1], idx[1], c1, s1, swa[1, :5])
    check_attn(out.cpu().numpy()[1], lse.cpu().numpy()[1], ro, rl, "swa_lens 5")


# ---------------------------------------------------------------------------
# schedule
# ---------------------------------------------------------------------------

def _decode_layer_inputs(B, lens, n_layers=20, seed=SEED):
    q_idx = np.stack([np.concatenate([synth.q_idx(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    w = np.stack([np.concatenate([synth.w_idx(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    q = np.stack([np.concatenate([synth.q_heads(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    swa = np.zeros((B, n_layers, 128, 256), np.uint16)
    for b, L in enumerate(lens):
        for l in range(n_layers):
            n = min(128, L)
            swa[b, l, :n] = synth.swa_rows(seed, l, b, n)
    return q_idx, w, q, swa  # [B, layers, ...]


def run_decode_layers(csa2, ps, lens, q_idx, w, q, swa, max_len, ws=None):
    B = len(lens)
    modes = csa2.schedule(True)
    n = len(modes)
    descs = [csa2.default_desc(m, 1) for m in modes]
    qi_t = [bits16(np.ascontiguousarray(q_idx[:, l])) for l in range(n)]
    w_t = [dev(np.ascontiguousarray(w[:, l])) for l in range(n)]
    q_t = [bits16(np.ascontiguousarray(q[:, l])) for l in range(n)]
    s_t = [bits16(np.ascontiguousarray(swa[:, l])) for l in range(n)]
    out = [torch.empty((B, 16, 128), dtype=torch.float32, device="cuda") for _ in range(n)]
    lse = [torch.empty((B, 16), dtype=torch.float32, device="cuda") for _ in range(n)]
    cand = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    sets = torch.full((n, B, 512), -9, dtype=torch.int32, device="cuda")
    ws = _ws(csa2, B, max_len) if ws is None else ws
    csa2.decode_layers(descs, ps.cache, qi_t, w_t, q_t, s_t, dev(np.array(lens, np.int32)), cand, sets, out, lse, B,
                       max_len, ws, err=ps.err)
    torch.cuda.synchronize()
    return dict(blocks=cand.cpu().numpy(), sets=sets.cpu().numpy(), out=[o.cpu().numpy() for o in out],
                lse=[x.cpu().numpy() for x in lse], modes=modes)


@pytest.mark.parametrize("page_size", [64, 8, 1024])
def test_decode_layers_vs_oracle(csa2, orc, page_size):
    lens = [20000, 9000, 130]
    B, max_len = len(lens), max(lens)
    ps = PagedSeqs(csa2, lens, page_size=page_size)
    data = [_fill(ps, b, L) for b, L in enumerate(lens)]
    q_idx, w, q, swa = _decode_layer_inputs(B, lens)
    snap = [t.clone() for t in (ps.cache.codes, ps.cache.scales, ps.cache.idx_k, ps.cache.pooled)]
    r = run_decode_layers(csa2, ps, lens, q_idx, w, q, swa, max_len)
    for a, b_ in zip(snap, (ps.cache.codes, ps.cache.scales, ps.cache.idx_k, ps.cache.pooled)):
        assert torch.equal(a, b_)  # Reindex/Reuse layers never write the shared cache
    modes = orc.schedule(True)
    for b, L in enumerate(lens):
        codes, scales = orc.quant_rows(data[b][0])
        idx = data[b][1]
        ref = orc.decode_step(modes, L, codes, scales, idx, orc.pool_blocks(idx), q_idx[b], w[b], q[b], swa[b])
        check_sets(r["blocks"][b], ref["blocks"], f"blocks {b}")
        last = None
        for l, m in enumerate(modes):
            if m != 2:
                check_sets(r["sets"][l, b], ref["idx"][l], f"set layer {l} seq {b}")
                last = l
            else:
                check_sets(r["sets"][last, b], ref["idx"][l], f"reuse layer {l} seq {b}")
            check_attn(r["out"][l][b], r["lse"][l][b], ref["out"][l], ref["lse"][l], f"layer {l} seq {b}")
    assert ps.errors() == 0


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------

def test_prefill_parity(csa2, orc):
    seed = 1003
    tokens, T = 4096 + 62, 700
    ratio = 2
    n_ent = tokens // 2
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    kv = synth.kv_rows(seed, 0, 0, tokens)
    idx_k = synth.idx_k_rows(seed, 0, 0, n_ent)
    ps.append(0, 0, synth.to_bf16_bits(kv), idx_k, ratio=2, chunk=999)
    kvb = orc.bf16_to_f32(synth.to_bf16_bits(kv)).reshape(kv.shape)
    codes, scales = orc.quant_rows(kvb, ratio=2)
    q_pos = np.arange(tokens - T, tokens, dtype=np.int32)
    q_idx = synth.q_idx(seed, 0, 0, T)
    w = synth.w_idx(seed, 0, 0, T)
    d = csa2.default_desc(csa2.FULL, 2)
    ws = _ws(csa2, T, n_ent, prefill=True)
    out_idx = torch.empty((T, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q_idx), dev(w), dev(np.array([n_ent], np.int32)), out_idx, T,
                      n_ent, ws, q_pos=dev(q_pos), err=ps.err)
    got = out_idx.cpu().numpy()
    want = orc.prefill_indexer(q_pos, ratio, n_ent, idx_k, q_idx, w)
    check_sets(got, want, "prefill indexer")
    swa_start = int(q_pos[0]) - 127
    swa = synth.swa_rows(seed, 0, 0, tokens - swa_start)
    q = synth.q_heads(seed, 0, 0, T)
    out = torch.empty((T, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_prefill(d, ps.cache, bits16(q), out_idx, dev(q_pos), bits16(swa), swa_start, n_ent, out, lse,
                             T, err=ps.err)
    ro, rl = orc.prefill_attn(q_pos, q, want, codes, scales, swa, swa_start)
    check_attn(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, "prefill attention")
    assert ps.errors() == 0


@pytest.mark.parametrize("page_size", [16, 64])
def test_prefill_scattered_queries(csa2, orc, page_size):
    # queries at non-consecutive positions, in no particular order: the window
    # branch walks the union of 16 queries' windows, the indexer's query tiles
    # and the per-query kernels see unrelated neighbours.  Pages of 16 entries
    # take the scorer's cp.async producer, pages of 64 its tensor boxes.
    seed = 1003
    tokens = 4096 + 62
    n_ent = tokens // 2
    ps = PagedSeqs(csa2, [n_ent], pooled=False, page_size=page_size)
    kv = synth.kv_rows(seed, 0, 0, tokens)
    idx_k = synth.idx_k_rows(seed, 0, 0, n_ent)
    ps.append(0, 0, synth.to_bf16_bits(kv), idx_k, ratio=2, chunk=999)
    kvb = orc.bf16_to_f32(synth.to_bf16_bits(kv)).reshape(kv.shape)
    codes, scales = orc.quant_rows(kvb, ratio=2)
    rng = np.random.default_rng(5)
    q_pos = rng.choice(np.arange(700, tokens), size=96, replace=False).astype(np.int32)
    T = len(q_pos)
    q_idx = synth.q_idx(seed, 0, 0, T)
    w = synth.w_idx(seed, 0, 0, T)
    d = csa2.default_desc(csa2.FULL, 2)
    ws = _ws(csa2, T, n_ent, prefill=True)
    out_idx = torch.empty((T, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q_idx), dev(w), dev(np.array([n_ent], np.int32)), out_idx, T,
                      n_ent, ws, q_pos=dev(q_pos), err=ps.err)
    want = orc.prefill_indexer(q_pos, 2, n_ent, idx_k, q_idx, w)
    check_sets(out_idx.cpu().numpy(), want, "prefill indexer, scattered queries")
    swa_start = int(q_pos.min()) - 127
    swa = synth.swa_rows(seed, 0, 0, tokens - swa_start)
    q = synth.q_heads(seed, 0, 0, T)
    out = torch.empty((T, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_prefill(d, ps.cache, bits16(q), out_idx, dev(q_pos), bits16(swa), swa_start, n_ent, out, lse,
                             T, err=ps.err)
    ro, rl = orc.prefill_attn(q_pos, q, want, codes, scales, swa, swa_start)
    check_attn(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, "prefill attention, scattered queries")
    assert ps.errors() == 0


def test_prefill_early_queries(csa2, orc):
    # queries from the first token on: windows shorter than 128 tokens, fewer
    # than 512 visible entries (sets padded with -1), and more queries than
    # the persistent attention kernel has CTAs, so every CTA reuses both of
    # its query buffers several times
    seed = 1003
    tokens = 2400
    n_ent = tokens // 2
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    kv = synth.kv_rows(seed, 1, 0, tokens)
    idx_k = synth.idx_k_rows(seed, 1, 0, n_ent)
    ps.append(0, 0, synth.to_bf16_bits(kv), idx_k, ratio=2, chunk=777)
    kvb = orc.bf16_to_f32(synth.to_bf16_bits(kv)).reshape(kv.shape)
    codes, scales = orc.quant_rows(kvb, ratio=2)
    q_pos = np.arange(0, tokens, 2, dtype=np.int32)
    T = len(q_pos)
    q_idx = synth.q_idx(seed, 1, 0, T)
    w = synth.w_idx(seed, 1, 0, T)
    d = csa2.default_desc(csa2.FULL, 2)
    ws = _ws(csa2, T, n_ent, prefill=True)
    out_idx = torch.empty((T, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q_idx), dev(w), dev(np.array([n_ent], np.int32)), out_idx, T,
                      n_ent, ws, q_pos=dev(q_pos), err=ps.err)
    want = orc.prefill_indexer(q_pos, 2, n_ent, idx_k, q_idx, w)
    check_sets(out_idx.cpu().numpy(), want, "prefill indexer, early queries")
    assert (want[0] == -1).all() and (want[-1] >= 0).all()
    swa = synth.swa_rows(seed, 1, 0, tokens)
    q = synth.q_heads(seed, 1, 0, T)
    out = torch.empty((T, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_prefill(d, ps.cache, bits16(q), out_idx, dev(q_pos), bits16(swa), 0, n_ent, out, lse, T,
                             err=ps.err)
    ro, rl = orc.prefill_attn(q_pos, q, want, codes, scales, swa, 0)
    check_attn(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, "prefill attention, early queries")
    assert ps.errors() == 0


@pytest.mark.parametrize("T", [1, 37, 150, 300])
def test_prefill_attention_few_queries_per_cta(csa2, orc, T):
    # fewer queries than the persistent attention kernel has CTAs (T = 1, 37:
    # CTAs of one query or none), two per CTA (150, 300 over 148 CTAs): the
    # pipeline's first and last query paths and the deferred epilogue at a
    # CTA's end.  Index sets are given directly: sorted visible entries with
    # -1 padding and -1 holes.
    seed = 1005
    tokens = 2048 + 320
    n_ent = tokens // 2
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    kv = synth.kv_rows(seed, 2, 0, tokens)
    ps.append(0, 0, synth.to_bf16_bits(kv), synth.idx_k_rows(seed, 2, 0, n_ent), ratio=2, chunk=999)
    kvb = orc.bf16_to_f32(synth.to_bf16_bits(kv)).reshape(kv.shape)
    codes, scales = orc.quant_rows(kvb, ratio=2)
    q_pos = np.arange(tokens - T, tokens, dtype=np.int32)
    rng = np.random.default_rng(T)
    sets = np.full((T, 512), -1, np.int32)
    for i, p in enumerate(q_pos):
        vis = int(p) // 2 + 1
        k = int(rng.integers(300, 513))
        sel = np.sort(rng.choice(vis, min(k, vis), replace=False)).astype(np.int32)
        sel[rng.random(sel.size) < 0.05] = -1  # holes
        sets[i, :sel.size] = sel
    swa_start = int(q_pos[0]) - 127
    swa = synth.swa_rows(seed, 2, 0, tokens - swa_start)
    q = synth.q_heads(seed, 2, 0, T)
    d = csa2.default_desc(csa2.REUSE, 2)
    out = torch.empty((T, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_prefill(d, ps.cache, bits16(q), dev(sets), dev(q_pos), bits16(swa), swa_start, n_ent, out, lse,
                             T, err=ps.err)
    ro, rl = orc.prefill_attn(q_pos, q, sets, codes, scales, swa, swa_start)
    check_attn(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, f"prefill attention, T = {T}")
    assert ps.errors() == 0


@pytest.mark.parametrize("window,topk", [(64, 256), (100, 512), (128, 384)])
def test_prefill_attention_window_and_topk(csa2, orc, window, topk):
    # a window shorter than 128 tokens (rows of the 128-row window tile whose
    # token is older than the window stay masked) and index sets narrower than
    # 512 (slots past topk are absent), over 400 consecutive queries
    seed = 1006
    tokens = 3000
    n_ent = tokens // 2
    T = 400
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    kv = synth.kv_rows(seed, 3, 0, tokens)
    ps.append(0, 0, synth.to_bf16_bits(kv), synth.idx_k_rows(seed, 3, 0, n_ent), ratio=2, chunk=999)
    kvb = orc.bf16_to_f32(synth.to_bf16_bits(kv)).reshape(kv.shape)
    codes, scales = orc.quant_rows(kvb, ratio=2)
    q_pos = np.arange(tokens - T, tokens, dtype=np.int32)
    rng = np.random.default_rng(window + topk)
    sets = np.full((T, topk), -1, np.int32)
    for i, p in enumerate(q_pos):
        vis = int(p) // 2 + 1
        sel = np.sort(rng.choice(vis, min(topk, vis), replace=False)).astype(np.int32)
        sets[i, :sel.size] = sel
    swa_start = int(q_pos[0]) - window + 1
    swa = synth.swa_rows(seed, 3, 0, tokens - swa_start)
    q = synth.q_heads(seed, 3, 0, T)
    d = csa2.default_desc(csa2.REUSE, 2, window=window, topk=topk)
    out = torch.empty((T, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_prefill(d, ps.cache, bits16(q), dev(sets), dev(q_pos), bits16(swa), swa_start, n_ent, out, lse,
                             T, err=ps.err)
    ro, rl = orc.prefill_attn(q_pos, q, sets, codes, scales, swa, swa_start, window=window)
    check_attn(out.cpu().numpy(), lse.cpu().numpy(), ro, rl, f"prefill attention, window {window}, topk {topk}")
    assert ps.errors() == 0


def test_prefill_indexer_exact_fallback_on_ties(csa2, orc):
    # Entries 0..4999 share one indexer-K row, so their scores tie exactly.  A
    # query that sees more than 2048 of them has too many candidates at the
    # approximate threshold and must be recomputed by the exact fallback; the
    # queries at the end of the context mix tied and distinct rows.  Either way
    # the sets must equal the oracle's (ties to the lowest position).
    seed = 1003
    n_ent = 6000
    tokens = 2 * n_ent
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    kv = synth.kv_rows(seed, 0, 0, tokens)
    idx_k = synth.idx_k_rows(seed, 0, 0, n_ent).copy()
    idx_k[:5000] = idx_k[0]
    ps.append(0, 0, synth.to_bf16_bits(kv), idx_k, ratio=2, chunk=999)
    q_pos = np.concatenate([np.arange(6000, 6200), np.arange(tokens - 200, tokens)]).astype(np.int32)
    T = len(q_pos)
    q_idx = synth.q_idx(seed, 0, 0, T)
    w = synth.w_idx(seed, 0, 0, T)
    d = csa2.default_desc(csa2.FULL, 2)
    ws = _ws(csa2, T, n_ent, prefill=True)
    out_idx = torch.empty((T, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q_idx), dev(w), dev(np.array([n_ent], np.int32)), out_idx, T,
                      n_ent, ws, q_pos=dev(q_pos), err=ps.err)
    want = orc.prefill_indexer(q_pos, 2, n_ent, idx_k, q_idx, w)
    check_sets(out_idx.cpu().numpy(), want, "prefill indexer with tied scores")
    assert ps.errors() == 0


def test_prefill_indexer_sampled_entries_lead(csa2, orc):
    # Every eighth entry's indexer-K row is scaled by 4, so those entries hold
    # the largest scores.  A threshold estimated from one key per 8 entries then
    # sits far too high and the candidates kernel must count the remaining keys
    # too; the sets must still equal the oracle's.
    seed = 1003
    n_ent = 8000
    tokens = 2 * n_ent
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    kv = synth.kv_rows(seed, 2, 0, tokens)
    kf = orc.bf16_to_f32(synth.idx_k_rows(seed, 2, 0, n_ent)).reshape(n_ent, 64)
    kf[::8] *= 4.0
    idx_k = synth.to_bf16_bits(kf)
    ps.append(0, 0, synth.to_bf16_bits(kv), idx_k, ratio=2, chunk=999)
    q_pos = np.concatenate([np.arange(3000, 3100), np.arange(tokens - 300, tokens)]).astype(np.int32)
    T = len(q_pos)
    q_idx = synth.q_idx(seed, 2, 0, T)
    w = synth.w_idx(seed, 2, 0, T)
    d = csa2.default_desc(csa2.FULL, 2)
    ws = _ws(csa2, T, n_ent, prefill=True)
    out_idx = torch.empty((T, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d, ps.cache, csa2.TOKEN, bits16(q_idx), dev(w), dev(np.array([n_ent], np.int32)), out_idx, T,
                      n_ent, ws, q_pos=dev(q_pos), err=ps.err)
    want = orc.prefill_indexer(q_pos, 2, n_ent, idx_k, q_idx, w)
    assert (want[-1] % 8 == 0).mean() > 0.5  # the scaled entries dominate the sets
    check_sets(out_idx.cpu().numpy(), want, "prefill indexer, sampled entries lead")
    assert ps.errors() == 0


# ---------------------------------------------------------------------------
# device-side error reporting (bounds checks turn bad input into flags)
# ---------------------------------------------------------------------------

def test_device_errors_are_flagged(csa2):
    ps = PagedSeqs(csa2, [100])
    kv = synth.kv_rows(SEED, 0, 0, 2)
    n_slots = ps.cache.codes.shape[0]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa2.kv_quant_append(ps.cache, dev(kv), None, dev(np.array([0, n_slots + 5], np.int64)), err=err)
    torch.cuda.synchronize()
    assert err.item() & 0x1
    err.zero_()
    idx = np.full((1, 512), -1, np.int32)
    idx[0, :3] = [0, 5, 100]  # 100 >= L
    out = torch.empty((1, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 16), dtype=torch.float32, device="cuda")
    csa2.sparse_attn_decode(csa2.default_desc(), ps.cache, bits16(synth.q_heads(SEED, 0, 0)), dev(idx),
                            bits16(np.zeros((1, 128, 256), np.uint16)), dev(np.array([100], np.int32)), out, lse, 1,
                            err=err)
    torch.cuda.synchronize()
    assert err.item() & 0x4
    assert np.isfinite(out.cpu().numpy()).all()
