"""Context-parallel test helpers: seeded sequences, the oracle's full-sequence
decode step, and CPU stand-ins for the library's kernels (the oracle on each
shard's entries, numpy for the merges) so that the exchange protocol of
fp4_kv_cache_nvfp4_b200.context_parallel can run on gloo ranks without a GPU."""
from __future__ import annotations

import numpy as np
import torch

import synth

SEED = 1004
N_LAYERS = 8  # Full, 3 Reuse, Reindex, 3 Reuse


def seq_data(orc, lens):
    """Per sequence: codes, scales, indexer K, pooled indexer K (whole sequence)."""
    out = []
    for b, L in enumerate(lens):
        codes, scales = orc.quant_rows(synth.kv_rows(SEED, b, 0, L))
        k = synth.idx_k_rows(SEED, b, 0, L)
        out.append((codes, scales, k, orc.pool_blocks(k)))
    return out


def layer_inputs(B):
    q_idx = np.stack([np.concatenate([synth.q_idx(SEED, l, b) for b in range(B)]) for l in range(N_LAYERS)])
    w = np.stack([np.concatenate([synth.w_idx(SEED, l, b) for b in range(B)]) for l in range(N_LAYERS)])
    q = np.stack([np.concatenate([synth.q_heads(SEED, l, b) for b in range(B)]) for l in range(N_LAYERS)])
    swa = np.stack([np.stack([synth.swa_rows(SEED, l, b, 128) for b in range(B)]) for l in range(N_LAYERS)])
    return q_idx, w, q, swa  # [layers, B, ...]


def reference(orc, data, lens, modes, q_idx, w, q, swa):
    """The oracle's decode step of every whole sequence."""
    return [orc.decode_step(modes, L, *data[b], q_idx[:, b], w[:, b], q[:, b], swa[:, b]) for b, L in enumerate(lens)]


class CpuShard:
    def __init__(self, g, lo, span, lens, holds_window):
        self.g, self.lo, self.span, self.holds_window = g, lo, span, holds_window
        self.lens = torch.tensor([min(span, L - lo) for L in lens], dtype=torch.int32)


def cpu_shards(lens, G, span, owned=None):
    return [CpuShard(g, g * span, span, lens, g == G - 1) for g in (range(G) if owned is None else owned)]


class OracleOps:
    """The kernels' contract restated with the oracle on each shard's slice."""

    def __init__(self, orc, data, B, keep=2048, topk=512):
        self.orc, self.data, self.B, self.keep, self.topk = orc, data, B, keep, topk

    def _slice(self, s, b):
        L = int(s.lens[b])
        codes, scales, k, _ = self.data[b]
        kl = k[s.lo:s.lo + L]
        return L, codes[s.lo:s.lo + L], scales[s.lo:s.lo + L], kl, self.orc.pool_blocks(kl)

    def block_topk(self, s, desc, q_idx, w):
        out = np.full((self.B, self.keep), -1, np.int32)
        for b in range(self.B):
            L, _, _, _, pooled = self._slice(s, b)
            out[b] = self.orc.select_blocks(pooled, L, q_idx[b], w[b], self.keep)
        return torch.from_numpy(out)

    def token_topk(self, s, desc, q_idx, w, cand_local):
        out = np.full((self.B, self.topk), -1, np.int32)
        for b in range(self.B):
            L, _, _, kl, _ = self._slice(s, b)
            out[b] = self.orc.select_tokens(kl, L, cand_local[b].numpy(), q_idx[b], w[b], self.topk)
        return torch.from_numpy(out)

    def score_ids(self, s, desc, level, q_idx, w, ids, offset):
        ids = ids.numpy()
        sc = np.full(ids.shape, -np.inf, np.float32)
        gid = np.full(ids.shape, -1, np.int32)
        for b in range(self.B):
            _, _, _, kl, pooled = self._slice(s, b)
            rows = pooled if level == 0 else kl
            ok = ids[b] >= 0
            sc[b, ok] = self.orc.score_rows(q_idx[b], w[b], rows[ids[b, ok]])
            gid[b, ok] = ids[b, ok] + offset
        return torch.from_numpy(sc), torch.from_numpy(gid)

    def merge(self, S, I, k, lo, hi):
        S, I = S.numpy(), I.numpy()  # [G, B, part]
        out = np.full((self.B, k), -1, np.int32)
        loc = np.full((self.B, k), -1, np.int32)
        for b in range(self.B):
            sc, ids = S[:, b].reshape(-1).astype(np.float64), I[:, b].reshape(-1)
            ok = ids >= 0
            sc, ids = sc[ok], ids[ok]
            top = np.sort(ids[np.lexsort((ids, -sc))[:k]])
            out[b, :top.size] = top
            mine = top[(top >= lo) & (top < hi)] - lo
            loc[b, :mine.size] = mine
        return torch.from_numpy(out), torch.from_numpy(loc)

    def attend(self, s, desc, q, local_set, swa, swa_lens):
        out = np.zeros((self.B, 16, 128), np.float32)
        lse = np.full((self.B, 16), -np.inf, np.float32)
        for b in range(self.B):
            _, codes, scales, _, _ = self._slice(s, b)
            sel = local_set[b].numpy()
            n_win = int(swa_lens[b])
            if (sel >= 0).sum() + n_win == 0:
                continue
            out[b], lse[b] = self.orc.attend(q[b], sel, codes, scales, swa[b][:n_win])
        return torch.from_numpy(out), torch.from_numpy(lse)

    def lse_merge(self, outs, lses):
        o, x = outs.numpy().astype(np.float64), lses.numpy().astype(np.float64)  # [G, B, 16, ...]
        M = x.max(axis=0)
        f = np.where(np.isneginf(x), 0.0, np.exp(x - np.where(np.isneginf(M), 0.0, M)[None]))
        den = f.sum(axis=0)
        out = (f[..., None] * o).sum(axis=0) / np.where(den > 0, den, 1.0)[..., None]
        lse = np.where(den > 0, M + np.log(np.where(den > 0, den, 1.0)), -np.inf)
        return torch.from_numpy(out.astype(np.float32)), torch.from_numpy(lse.astype(np.float32))


def torch_inputs(q_idx, w, q, swa):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    return [t(x) for x in q_idx], [t(x) for x in w], [t(x) for x in q], [t(x) for x in swa]


def compare(res, ref, lens, modes, what, atol=2e-3, rtol_l2=1e-3):
    """Sets exact; attention within the tolerance."""
    for l in range(len(modes)):
        idx = res[l]["idx"].cpu().numpy()
        out = res[l]["out"].cpu().numpy().astype(np.float64)
        lse = res[l]["lse"].cpu().numpy().astype(np.float64)
        for b in range(len(lens)):
            np.testing.assert_array_equal(idx[b], ref[b]["idx"][l], err_msg=f"{what} layer {l} seq {b} set")
            r = ref[b]["out"][l].astype(np.float64)
            assert np.abs(out[b] - r).max() <= atol, f"{what} layer {l} seq {b} max-abs"
            assert np.linalg.norm(out[b] - r) <= rtol_l2 * np.linalg.norm(r), f"{what} layer {l} seq {b} rel-L2"
            assert np.abs(lse[b] - ref[b]["lse"][l]).max() <= atol, f"{what} layer {l} seq {b} lse"
