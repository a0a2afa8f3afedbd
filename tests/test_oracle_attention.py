"""Pins of the oracle's attention, window and schedule (no GPU)."""
import json
import os

import numpy as np

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    return synth.to_bf16_bits(np.asarray(x, np.float32))


def _cache(n, seed=0):
    x = synth.kv_rows(1001, seed, 0, n)
    return x


def test_zero_query_gives_multiset_mean(orc):
    n = 300
    codes, scales = orc.quant_rows(_cache(n))
    xh = orc.dequant(codes, scales)
    idx = np.full(512, -1, np.int32)
    idx[:40] = np.arange(0, 80, 2)
    idx[40:45] = [1, 3, 5, 7, 9]
    swa = synth.swa_rows(1001, 0, 0, 20)
    q = np.zeros((16, 128), np.uint16)
    out, lse = orc.attend(q, idx, codes, scales, swa)
    sel = idx[idx >= 0]
    vals = np.concatenate([xh[sel, 128:], orc.bf16_to_f32(swa).reshape(20, 256)[:, 128:].astype(np.float64)])
    want = vals.mean(axis=0)
    assert np.allclose(out, want[None, :], atol=1e-6, rtol=1e-6)
    assert np.allclose(lse, np.log(len(sel) + 20), atol=1e-6)


def test_no_dedup_between_sparse_and_window(orc):
    # the same value reached both through the FP4 cache and the SWA counts twice
    x = np.zeros((2, 256), np.float32)
    x[0, 128:] = 6.0
    x[1, 128:] = 0.0
    codes, scales = orc.quant_rows(x)
    swa = np.zeros((1, 256), np.float32)
    swa[0, 128:] = 6.0
    idx = np.array([0, 1], np.int32)
    out, _ = orc.attend(np.zeros((16, 128), np.uint16), idx, codes, scales, bf(swa))
    assert np.allclose(out, 4.0)  # (6 + 0 + 6) / 3


def test_single_key(orc):
    x = _cache(1, seed=3)
    codes, scales = orc.quant_rows(x)
    xh = orc.dequant(codes, scales)[0]
    q = synth.q_heads(1001, 0, 0)[0]
    out, lse = orc.attend(q, np.array([0], np.int32), codes, scales, np.zeros((0, 256), np.uint16))
    assert np.allclose(out, xh[None, 128:], atol=0, rtol=1e-7)
    qf = orc.bf16_to_f32(q).reshape(16, 128).astype(np.float64)
    assert np.allclose(lse, qf @ xh[:128] / np.sqrt(128.0), rtol=1e-6)


def test_lse_merge_equals_one_softmax(orc):
    n = 700
    codes, scales = orc.quant_rows(_cache(n, seed=1))
    xh = orc.dequant(codes, scales)
    rng = np.random.default_rng(0)
    idx = np.sort(rng.choice(n, 512, replace=False)).astype(np.int32)
    swa = synth.swa_rows(1001, 2, 0, 128)
    q = synth.q_heads(1001, 2, 0)[0]
    out, lse = orc.attend(q, idx, codes, scales, swa)
    qf = orc.bf16_to_f32(q).reshape(16, 128).astype(np.float64)
    sw = orc.bf16_to_f32(swa).reshape(128, 256).astype(np.float64)
    K = np.concatenate([xh[idx, :128], sw[:, :128]])
    V = np.concatenate([xh[idx, 128:], sw[:, 128:]])
    z = qf @ K.T / np.sqrt(128.0)
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    want = (p @ V) / p.sum(axis=1, keepdims=True)
    want_lse = m[:, 0] + np.log(p.sum(axis=1))
    np.testing.assert_allclose(out, want, rtol=2e-6, atol=2e-6)
    np.testing.assert_allclose(lse, want_lse, rtol=1e-6, atol=1e-6)


def _decode_inputs(L, n_layers=20, seed=1001, seq=0):
    x = synth.kv_rows(seed, seq, 0, L)
    codes, scales = __import__("oracle").quant_rows(x)
    k = synth.idx_k_rows(seed, seq, 0, L)
    pooled = __import__("oracle").pool_blocks(k)
    q_idx = np.concatenate([synth.q_idx(seed, l, seq) for l in range(n_layers)])
    w = np.concatenate([synth.w_idx(seed, l, seq) for l in range(n_layers)])
    q = np.concatenate([synth.q_heads(seed, l, seq) for l in range(n_layers)])
    nsw = min(L, 128)
    swa = np.zeros((n_layers, 128, 256), np.uint16)
    for l in range(n_layers):
        swa[l, :nsw] = synth.swa_rows(seed, l, seq, nsw)
    return codes, scales, k, pooled, q_idx, w, q, swa


def test_schedule_matches_pages(orc):
    with open(os.path.join(GOLD, "pages_facts.json")) as f:
        facts = json.load(f)
    name = {0: "F", 1: "RI", 2: "R"}
    assert [name[m] for m in orc.schedule(True)] == facts["decoder_schedule"]["value"]
    assert [name[m] for m in orc.schedule(False)] == facts["encoder_schedule"]["value"]
    assert facts["hier_blocks"]["value"] * facts["hier_block_size"]["value"] == facts["hier_positions"]["value"]


def test_decode_step_schedule_invariants(orc):
    L = 8 * 2048 + 8 * 300 + 5  # hierarchical path active, partial last block
    codes, scales, k, pooled, q_idx, w, q, swa = _decode_inputs(L)
    snap = [a.copy() for a in (codes, scales, k, pooled)]
    modes = orc.schedule(True)
    r = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa)
    for a, b in zip(snap, (codes, scales, k, pooled)):
        np.testing.assert_array_equal(a, b)     # the step never writes the cache
    idx = r["idx"]
    cand = set(t for j in r["blocks"] if j >= 0 for t in range(8 * j, min(8 * j + 8, L)))
    for l, m in enumerate(modes):
        if m == 2:
            np.testing.assert_array_equal(idx[l], idx[l - 1])   # Reuse = previous set
        else:
            assert set(idx[l].tolist()) <= cand              # Full/Reindex stay within the candidates
            assert (idx[l] >= 0).all()
    # Reindex re-scores with its own q: its sets differ from the Full layer's
    assert not np.array_equal(idx[4], idx[0])
    # a Reindex layer given the Full layer's indexer q reproduces the Full set
    q_idx2, w2 = q_idx.copy(), w.copy()
    q_idx2[4], w2[4] = q_idx[0], w[0]
    r2 = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx2, w2, q, swa)
    np.testing.assert_array_equal(r2["idx"][4], idx[0])
    # each layer reads only its own SWA: swapping layers 6 and 7's windows changes only them
    swa2 = swa.copy()
    swa2[[6, 7]] = swa[[7, 6]]
    r3 = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa2)
    changed = [l for l in range(20) if not np.array_equal(r3["out"][l], r["out"][l])]
    assert changed == [6, 7]


def test_encoder_decode_step_is_flat(orc):
    # keep = 0 (the encoder's layers): each Full layer's set is the Top-512 of
    # ALL L scores by (score desc, index asc), here ranked by numpy; a planted
    # entry whose block pools to ~0 is found by the flat selection and missed
    # by the decoder's hierarchy on the same context.
    L = 8 * 2048 + 8 * 300 + 5
    codes, scales, k, pooled, q_idx, w, q, swa = _decode_inputs(L, n_layers=18, seed=1003)
    modes = orc.schedule(False)
    u = np.random.default_rng(11).standard_normal((4, 64)).astype(np.float32)
    q_idx[0] = bf(u)
    w[0] = 1.0
    e = 8 * 1234 + 3
    v = 8.0 * u.sum(0)                    # positive dot with every head
    kf = np.tile(-v * (3.0 / 7.0), (8, 1))
    kf[3] = v                             # the block pools to -v/4: score 0
    k[8 * 1234:8 * 1235] = bf(kf)
    pooled = orc.pool_blocks(k)
    r = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa, keep=0)
    for l, m in enumerate(modes):
        if m == 2:
            np.testing.assert_array_equal(r["idx"][l], r["idx"][l - 1])
        else:
            s = orc.score_rows(q_idx[l], w[l], k).astype(np.float64)
            order = np.lexsort((np.arange(L), -s))[:512]
            assert sorted(order.tolist()) == r["idx"][l].tolist()
        o, lse = orc.attend(q[l], r["idx"][l], codes, scales, swa[l, :128])
        np.testing.assert_array_equal(o, r["out"][l])
        np.testing.assert_array_equal(lse, r["lse"][l])
    assert e in r["idx"][0].tolist()
    rh = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa, keep=2048)
    assert e not in rh["idx"][0].tolist()
    assert 1234 not in orc.select_blocks(pooled, L, q_idx[0], w[0]).tolist()  # pruned by the hierarchy


def test_decode_window_boundary(orc):
    # L < 128: only the first L SWA rows take part (a sentinel in row L must not count)
    L = 50
    codes, scales, k, pooled, q_idx, w, q, swa = _decode_inputs(L, n_layers=1)
    modes = np.array([0], np.int32)
    r1 = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa)
    swa2 = swa.copy()
    swa2[0, L:] = bf(np.full((128 - L, 256), 1e4))
    r2 = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa2)
    np.testing.assert_array_equal(r1["out"], r2["out"])
    swa3 = swa.copy()
    swa3[0, L - 1] = bf(np.full(256, 50.0))
    r3 = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx, w, q, swa3)
    assert not np.array_equal(r1["out"], r3["out"])


def test_prefill_window_and_visibility(orc):
    ratio, tokens = 2, 600
    n_ent = tokens // 2
    x = synth.kv_rows(1003, 0, 0, tokens)
    codes, scales = orc.quant_rows(x, ratio=2)
    k = synth.idx_k_rows(1003, 0, 0, n_ent)
    q_pos = np.arange(400, 600, dtype=np.int32)
    T = q_pos.size
    qi = synth.q_idx(1003, 0, 0, T)
    w = synth.w_idx(1003, 0, 0, T)
    idx = orc.prefill_indexer(q_pos, ratio, n_ent, k, qi, w, 128)
    for t, p in enumerate(q_pos):
        vis = orc.visible_entries(int(p), ratio, n_ent)
        assert vis == (int(p) + 1) // 2                    # (j+1)*2 - 1 <= p
        sel = idx[t][idx[t] >= 0]
        assert sel.size == min(128, vis) and sel.max() < vis
    # prefill window: token p-128 is outside, p-127 inside
    swa_start = 400 - 127
    swa = synth.swa_rows(1003, 0, 0, 600 - swa_start)
    q = synth.q_heads(1003, 0, 0, T)
    o1, _ = orc.prefill_attn(q_pos, q, idx, codes, scales, swa, swa_start)
    swa2 = swa.copy()
    p = 500
    swa2[p - 128 - swa_start] = bf(np.full(256, 30.0))
    o2, _ = orc.prefill_attn(q_pos, q, idx, codes, scales, swa2, swa_start)
    t = p - 400
    np.testing.assert_array_equal(o1[t], o2[t])
    assert not np.array_equal(o1[t - 1], o2[t - 1])  # query p-1 sees token p-128


def test_cache_accounting(orc):
    # Full layers carry the cache: 3 encoder Full layers at ratio 2, 1 decoder Full at ratio 1
    ratios = [2, 2, 2, 1]
    main = 256 * 0.5 + 16  # FP4 codes + one E4M3 byte per 16 channels
    ours = orc.cache_bytes_per_token(ratios, main, 64 * 2)
    # closed form with these dimensions: 3 x (144 + 128) / 2 + (144 + 128)
    assert ours == 3 * (144 + 128) / 2 + (144 + 128) == 680.0
    # one Full layer at ratio 1 alone is one entry per token
    assert orc.cache_bytes_per_token([1], main, 128) == 272.0
    # FP4 + E4M3/16 is 4.5 bits per channel: a bit over half of 8-bit storage
    assert main / 256 * 8 == 4.5
    # consistency report (not an assertion): the pages' 890 B/token over the
    # same 2.5 Full entries per token is 356 B per entry, against our 272
    with open(os.path.join(GOLD, "pages_facts.json")) as f:
        facts = json.load(f)
    pages = facts["kv_bytes_per_token"]["value"]
    print(f"cache bytes/token: ours {ours:.0f} with 256-ch FP4 main + 64-d bf16 indexer K; pages {pages} "
          f"(= {pages / 2.5:.0f} B per Full entry at 2.5 entries/token)")


def _batch_case(keep, lens, modes, seed):
    """Per-sequence caches and per-layer inputs for decode_batch / decode_step."""
    n = len(modes)
    caches, q_idx, w, q, swa = [], [], [], [], []
    for b, L in enumerate(lens):
        codes, scales, k, pooled, qi, wi, qh, sw = _decode_inputs(int(L), n_layers=n, seed=seed, seq=b)
        caches.append((codes, scales, k, pooled))
        q_idx.append(qi)
        w.append(wi)
        q.append(qh)
        swa.append(sw)
    return caches, np.stack(q_idx), np.stack(w), np.stack(q), np.stack(swa)


def test_decode_batch_equals_per_sequence_steps(orc):
    # decode_batch (the CPU baseline's entry point) runs decode_step on every
    # sequence with its own per-sequence strides: ragged lengths, a distinct
    # cache per sequence (different seq seeds), both indexer modes.  A wrong
    # offset of q, q_idx, w, swa, the outputs or the block list would mix
    # sequences and fail the bit-exact comparison.
    lens = [8 * 2048 + 8 * 37 + 3, 130, 5000, 8 * 2048 + 1]
    for keep, decoder, seed in ((2048, True, 1002), (0, False, 1006)):
        modes = orc.schedule(decoder)[:8]
        caches, q_idx, w, q, swa = _batch_case(keep, lens, modes, seed)
        r = orc.decode_batch(modes, lens, [c[0] for c in caches], [c[1] for c in caches],
                             [c[2] for c in caches], [c[3] for c in caches], q_idx, w, q, swa, keep=keep)
        for b, L in enumerate(lens):
            codes, scales, k, pooled = caches[b]
            one = orc.decode_step(modes, L, codes, scales, k, pooled, q_idx[b], w[b], q[b], swa[b], keep=keep)
            np.testing.assert_array_equal(r["idx"][b], one["idx"])
            np.testing.assert_array_equal(r["out"][b], one["out"])
            np.testing.assert_array_equal(r["lse"][b], one["lse"])
            if keep:
                np.testing.assert_array_equal(r["blocks"][b], one["blocks"])
        # the sequences really differ (distinct caches and queries)
        assert not np.array_equal(r["out"][0], r["out"][3])
        assert not np.array_equal(r["idx"][0], r["idx"][3])
