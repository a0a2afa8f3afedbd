"""Context-parallel decode on one GPU: G = 2 and 4 shards of two long
sequences run one after another through the library's kernels (the exchange is
a stack on the device), against the oracle's decode step of each whole
sequence: index sets exact, attention within max-abs 2e-3 / rel-L2 1e-3.  And
the three exchange kernels on their own: rescoring bit-equal to the oracle's
scores, the Top-K merge equal to a brute-force ranking (ties, empty pairs),
the log-sum-exp merge equal to one softmax."""
import numpy as np
import pytest
import torch

import _cp_util as U
import synth
from _gpu_util import PagedSeqs, bits16, dev

pytestmark = pytest.mark.gpu
LENS = [70000, 60000]


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


@pytest.fixture(scope="module")
def filled(csa2, orc):
    ps = PagedSeqs(csa2, LENS, extra_pages=4)
    for b, L in enumerate(LENS):
        ps.append(b, 0, synth.kv_rows(U.SEED, b, 0, L), synth.idx_k_rows(U.SEED, b, 0, L))
    return ps, U.seq_data(orc, LENS)


@pytest.mark.parametrize("G", [2, 4])
def test_context_parallel_step_matches_whole_sequence(csa2, orc, filled, G):
    from fp4_kv_cache_nvfp4_b200 import context_parallel as cp
    ps, data = filled
    B = len(LENS)
    span = (max(LENS) + G - 1) // G // 64 * 64 + 64
    shards = cp.make_shards(ps.cache, LENS, G, span)
    q_idx, w, q, swa = U.layer_inputs(B)
    modes = orc.schedule(True)[:U.N_LAYERS]
    descs = [csa2.default_desc(m, 1) for m in modes]
    swa_lens = dev(np.array([min(128, L) for L in LENS], np.int32))
    res = cp.decode_step(modes, descs, shards, cp.KernelOps(B, err=ps.err), cp.LocalExchange(),
                         [bits16(x) for x in q_idx], [dev(x) for x in w], [bits16(x) for x in q],
                         [bits16(x) for x in swa], swa_lens)
    torch.cuda.synchronize()
    assert ps.errors() == 0
    ref = U.reference(orc, data, LENS, modes, q_idx, w, q, swa)
    U.compare(res, ref, LENS, modes, f"G={G}")


def test_score_ids_bit_equal_to_oracle(csa2, orc, filled):
    ps, data = filled
    B = len(LENS)
    d = csa2.default_desc(csa2.FULL, 1)
    rng = np.random.default_rng(3)
    q_idx = np.concatenate([synth.q_idx(U.SEED, 0, b) for b in range(B)])
    w = np.concatenate([synth.w_idx(U.SEED, 0, b) for b in range(B)])
    sl = dev(np.array(LENS, np.int32))
    for level, rows_of in ((csa2.BLOCK, lambda b: data[b][3]), (csa2.TOKEN, lambda b: data[b][2])):
        n_ids = [(L + 7) // 8 if level == csa2.BLOCK else L for L in LENS]
        ids = np.stack([rng.integers(0, n, 700) for n in n_ids]).astype(np.int32)
        ids[:, ::7] = -1
        sc = torch.empty(ids.shape, dtype=torch.float32, device="cuda")
        gid = torch.empty(ids.shape, dtype=torch.int32, device="cuda")
        csa2.indexer_score_ids(d, ps.cache, level, bits16(q_idx), dev(w), sl, dev(ids), 1000, sc, gid, B,
                               max(LENS), err=ps.err)
        sc, gid = sc.cpu().numpy(), gid.cpu().numpy()
        for b in range(B):
            ok = ids[b] >= 0
            want = orc.score_rows(q_idx[b], w[b], rows_of(b)[ids[b, ok]])
            np.testing.assert_array_equal(sc[b, ok].view(np.uint32), want.view(np.uint32))
            assert np.isneginf(sc[b, ~ok]).all()
            np.testing.assert_array_equal(gid[b], np.where(ok, ids[b] + 1000, -1))
    assert ps.errors() == 0


@pytest.mark.parametrize("parts,plen,k", [(2, 2048, 2048), (4, 512, 512), (8, 512, 512), (3, 100, 512)])
def test_topk_merge_equals_brute_force(csa2, parts, plen, k):
    rng = np.random.default_rng(parts * 1000 + plen)
    n = 3
    ids = np.full((parts, n, plen), -1, np.int32)
    sc = np.zeros((parts, n, plen), np.float32)
    for g in range(parts):
        for b in range(n):
            m = rng.integers(plen // 2, plen + 1)
            ids[g, b, :m] = np.sort(rng.choice(10000, m, replace=False)) + g * 10000
            sc[g, b, :m] = rng.integers(0, 50, m).astype(np.float32) * 0.25  # many ties
    lo, hi = 10000, 20000
    out = torch.empty((n, k), dtype=torch.int32, device="cuda")
    loc = torch.empty((n, k), dtype=torch.int32, device="cuda")
    csa2.topk_merge(dev(sc), dev(ids), k, out, loc, lo, hi)
    out, loc = out.cpu().numpy(), loc.cpu().numpy()
    for b in range(n):
        s, i = sc[:, b].reshape(-1), ids[:, b].reshape(-1)
        ok = i >= 0
        s, i = s[ok], i[ok]
        top = np.sort(i[np.lexsort((i, -s.astype(np.float64)))[:k]])
        want = np.full(k, -1, np.int32)
        want[:top.size] = top
        np.testing.assert_array_equal(out[b], want)
        mine = top[(top >= lo) & (top < hi)] - lo
        wl = np.full(k, -1, np.int32)
        wl[:mine.size] = mine
        np.testing.assert_array_equal(loc[b], wl)


def test_lse_merge_equals_one_softmax(csa2):
    rng = np.random.default_rng(9)
    G, rows = 3, 4
    o = rng.standard_normal((G, rows, 16, 128)).astype(np.float32)
    x = (rng.standard_normal((G, rows, 16)) * 3).astype(np.float32)
    x[1, 2] = -np.inf                      # an empty partial
    x[:, 3, 5] = -np.inf                   # a head empty everywhere
    out = torch.empty((rows, 16, 128), device="cuda")
    lse = torch.empty((rows, 16), device="cuda")
    csa2.attn_lse_merge(dev(o), dev(x), out, lse)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    xd = x.astype(np.float64)
    M = np.max(xd, axis=0)
    Ms = np.where(np.isneginf(M), 0.0, M)
    f = np.where(np.isneginf(xd), 0.0, np.exp(xd - Ms[None]))
    den = f.sum(0)
    want = (f[..., None] * o).sum(0) / np.where(den > 0, den, 1.0)[..., None]
    want_lse = np.where(den > 0, Ms + np.log(np.where(den > 0, den, 1.0)), -np.inf)
    np.testing.assert_allclose(out, want, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(lse, want_lse, rtol=1e-6, atol=1e-6)
    assert (out[3, 5] == 0).all() and np.isneginf(lse[3, 5])
