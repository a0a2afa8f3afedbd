"""Pins of the oracle's indexer: score function, Top-K, hierarchy (no GPU)."""
import itertools

import numpy as np

import synth


def bf(x):
    return synth.to_bf16_bits(np.asarray(x, np.float32))


def test_score_one_hot_closed_form(orc):
    rng = np.random.default_rng(0)
    k = synth.idx_k_rows(1001, 3, 0, 1)[0]
    kf = orc.bf16_to_f32(k)
    for _ in range(50):
        d = rng.integers(0, 64, 4)
        a = rng.choice([-2.0, -0.5, 0.5, 1.0, 3.0], 4)
        q = np.zeros((4, 64), np.float32)
        q[np.arange(4), d] = a
        w = rng.uniform(0, 1, 4).astype(np.float32)
        # products of bf16 values are exact; relu then a weighted sum of 4 terms
        want = np.float32(0)
        for h in range(4):
            want = np.float32(np.float64(w[h]) * max(np.float64(a[h]) * kf[d[h]], 0.0) + np.float64(want))
        assert orc.score(bf(q), w, k) == want


def test_score_relu_and_weights(orc):
    k = bf(np.ones(64))
    q = np.ones((4, 64), np.float32)
    q[1] *= -1  # negative dot: contributes nothing
    q[2] *= 2
    w = np.array([0.5, 0.9, 0.25, 0.0], np.float32)
    assert orc.score(bf(q), w, k) == np.float32(0.5 * 64 + 0.25 * 128)
    assert orc.score(bf(-np.ones((4, 64))), np.ones(4, np.float32), k) == 0.0


def test_score_is_sequential_fp32(orc):
    # 2^24 + 1 + 1: summed left to right in fp32 each +1 is lost (ties to even);
    # a pairwise or fp64 sum would give 2^24 + 2.
    q = np.zeros((4, 64), np.float32)
    k = np.zeros(64, np.float32)
    q[0, :3] = [4096.0, 1.0, 1.0]
    k[:3] = [4096.0, 1.0, 1.0]
    w = np.array([1, 0, 0, 0], np.float32)
    assert orc.score(bf(q), w, bf(k)) == np.float32(2.0 ** 24)
    # the same terms in the other order keep both ones
    q[0, :3] = [1.0, 1.0, 4096.0]
    k[:3] = [1.0, 1.0, 4096.0]
    assert orc.score(bf(q), w, bf(k)) == np.float32(2.0 ** 24 + 2)


def test_score_within_fp32_bound_of_fp64(orc):
    rows = synth.idx_k_rows(1001, 0, 0, 2000)
    qi = synth.q_idx(1001, 0, 0)[0]
    w = synth.w_idx(1001, 0, 0)[0]
    got = orc.score_rows(qi, w, rows).astype(np.float64)
    qf = orc.bf16_to_f32(qi).reshape(4, 64).astype(np.float64)
    kf = orc.bf16_to_f32(rows).reshape(-1, 64).astype(np.float64)
    dots = kf @ qf.T
    ref = (np.maximum(dots, 0) * w[None, :].astype(np.float64)).sum(axis=1)
    bound = (70 * 2.0 ** -24) * ((np.abs(kf) @ np.abs(qf).T) * w[None, :]).sum(axis=1) + 1e-30
    assert np.all(np.abs(got - ref) <= bound)


def _check_topk(scores, sel, k):
    n = scores.size
    m = min(n, k)
    assert (sel[m:] == -1).all() and (np.diff(sel[:m]) > 0).all()
    chosen = set(sel[:m].tolist())
    for i in chosen:            # every chosen item outranks every other item
        for j in range(n):
            if j in chosen:
                continue
            assert scores[i] > scores[j] or (scores[i] == scores[j] and i < j)


def test_topk_brute_force_tiny(orc):
    rng = np.random.default_rng(1)
    for n, k in itertools.product([1, 2, 5, 17, 64], [1, 3, 8, 64, 100]):
        s = rng.integers(-3, 4, n).astype(np.float32)  # plenty of ties
        _check_topk(s, orc.topk(s, k), k)
        s = rng.standard_normal(n).astype(np.float32)
        _check_topk(s, orc.topk(s, k), k)


def test_topk_ties_to_lower_index(orc):
    s = np.zeros(1000, np.float32)
    assert orc.topk(s, 512).tolist() == list(range(512))
    s[[999, 500]] = 1.0
    assert orc.topk(s, 3).tolist() == [0, 500, 999]
    s = np.zeros(10, np.float32)
    s[3] = -0.0  # -0 and +0 are equal scores
    assert orc.topk(s, 4).tolist() == [0, 1, 2, 3]


def test_hierarchy_equals_flat_when_small(orc):
    L = 4096  # 512 blocks <= 2048: every block is a candidate
    k = synth.idx_k_rows(1001, 0, 0, L)
    pooled = orc.pool_blocks(k)
    qi, w = synth.q_idx(1001, 0, 0)[0], synth.w_idx(1001, 0, 0)[0]
    blocks = orc.select_blocks(pooled, L, qi, w)
    assert blocks[:512].tolist() == list(range(512)) and (blocks[512:] == -1).all()
    np.testing.assert_array_equal(orc.select_tokens(k, L, blocks, qi, w), orc.select_tokens(k, L, None, qi, w))


def test_hierarchy_planted_blocks(orc):
    L = 8 * 3000 + 5  # 3001 blocks > 2048, last block partial
    rng = np.random.default_rng(2)
    kf = rng.standard_normal((L, 64)).astype(np.float32) * 0.05
    qf = np.zeros((4, 64), np.float32)
    qf[:, 0] = 1.0
    hot = rng.choice(3001, 2048, replace=False)
    for j in hot:                      # planted blocks score high, the rest ~0
        kf[8 * j:8 * j + 8, 0] += 4.0
    k = bf(kf)
    pooled = orc.pool_blocks(k)
    w = np.ones(4, np.float32)
    blocks = orc.select_blocks(pooled, L, bf(qf), w)
    assert sorted(hot.tolist()) == blocks.tolist()
    # candidates are exactly the positions of the kept blocks below L
    sel, sc, pos = orc.select_tokens(k, L, blocks, bf(qf), w, return_scores=True)
    want = [t for j in sorted(hot.tolist()) for t in range(8 * j, min(8 * j + 8, L))]
    assert pos.tolist() == want
    _check_topk(sc, np.searchsorted(pos, sel[sel >= 0]), 512)


def test_hierarchy_block_topk_by_brute_force(orc):
    rng = np.random.default_rng(5)
    for L in [8 * 2049, 8 * 2100 + 3]:
        k = bf(rng.standard_normal((L, 64)))
        pooled = orc.pool_blocks(k)
        qi, w = bf(rng.standard_normal((4, 64))), rng.uniform(0, 1, 4).astype(np.float32)
        blocks, bs = orc.select_blocks(pooled, L, qi, w, return_scores=True)
        order = sorted(range(bs.size), key=lambda j: (-bs[j], j))[:2048]
        assert sorted(order) == blocks.tolist()


def test_short_contexts(orc):
    for L in [1, 7, 8, 9, 511, 512, 513]:
        k = synth.idx_k_rows(1001, 9, 0, L)
        qi, w = synth.q_idx(1001, 1, 0)[0], synth.w_idx(1001, 1, 0)[0]
        blocks = orc.select_blocks(orc.pool_blocks(k), L, qi, w)
        sel = orc.select_tokens(k, L, blocks, qi, w)
        m = min(L, 512)
        assert (sel[:m] >= 0).all() and (sel[m:] == -1).all()
        if L <= 512:
            assert sel[:m].tolist() == list(range(L))


def test_flat_selection_is_the_prefill_selection_of_a_query_that_sees_everything(orc):
    # The flat reading (no block level) selects exactly what the prefill
    # indexer selects for a query at the last token: every entry is visible to it.
    for ratio, L in [(2, 3000), (1, 777), (2, 513)]:
        k = synth.idx_k_rows(1006, 3, 0, L)
        qi, w = synth.q_idx(1006, 0, 3)[0], synth.w_idx(1006, 0, 3)[0]
        flat = orc.select_tokens(k, L, None, qi, w)
        assert orc.visible_entries(ratio * L - 1, ratio, L) == L
        pre = orc.prefill_indexer(np.array([ratio * L - 1], np.int32), ratio, L, k, qi[None], w[None])[0]
        np.testing.assert_array_equal(flat, pre)
        # one token earlier at ratio 2 the last entry is not complete yet
        if ratio == 2:
            assert orc.visible_entries(ratio * L - 2, ratio, L) == L - 1


def test_flat_selection_brute_force_small(orc):
    # Top-512 of all L scores by (score desc, index asc), ascending: a Python sort
    # of the oracle's per-row scores, with ties planted by duplicated rows.
    rng = np.random.default_rng(9)
    L = 1500
    k = bf(rng.standard_normal((L, 64)))
    k[700:760] = k[5]  # 61 equal scores
    qi, w = bf(rng.standard_normal((4, 64))), rng.uniform(0, 1, 4).astype(np.float32)
    s = orc.score_rows(qi, w, k)
    order = sorted(range(L), key=lambda j: (-float(s[j]), j))[:512]
    assert orc.select_tokens(k, L, None, qi, w).tolist() == sorted(order)
