"""Context-parallel decode of long sequences: the entries of every sequence
split into G contiguous shards, one per GPU.

Pages: native context window of one million tokens (conexaotc.com.br, opening
paragraphs); Top-512 per Full/Reindex layer and the hierarchical indexer of up
to 2048 blocks of 8 (CSA2 paragraph); Reindex re-scores the Full layer's
candidates with its own indexer Q, Reuse re-uses the latest set ("Como
funciona", e-cogni.com.br).

Shard g holds entries [g*S, g*S + S) of each sequence.  Each shard runs the
ordinary kernels on its own entries; between shards only small lists move:

  Full layer     block level: each shard's local Top-2048 blocks, rescored
                 (csa2_indexer_score_ids, bit-equal scores) and made global;
                 all-gather; csa2_topk_merge gives the global Top-2048 and each
                 shard's local candidate blocks.  Token level: the same with
                 each shard's local Top-512 positions.
  Reindex layer  token level on the Full layer's local candidates, as above.
  Reuse layer    nothing to select.
  every layer    attention of each shard over its local share of the set (the
                 window on the last shard), all-gather of the partial
                 (out, lse), csa2_attn_lse_merge.

Every member of a global Top-K is in its own shard's local Top-K, so the
merged sets are exactly the single-GPU sets (ties to the lower position), and
the merged attention is the single-GPU attention up to rounding.

This module only sequences calls: the selection, scoring and merging run in
the library's kernels (``KernelOps``), the transfers in ``torch.distributed``
collectives (``DistExchange``, NCCL over NVLink) or, for G shards held by one
process, a stack on the device (``LocalExchange``).  No tile is read from a
peer's memory: every shard gathers small lists into its own memory.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as B

FULL, REINDEX, REUSE = B.FULL, B.REINDEX, B.REUSE
BLOCK, TOKEN = B.BLOCK, B.TOKEN


@dataclass
class Shard:
    """One shard: global index g, first entry lo (a multiple of the page size),
    span S (entries per shard), the cache view of its pages, the per-sequence
    entry counts it holds (every one >= 1) and whether it holds the window."""
    g: int
    lo: int
    span: int
    cache: object
    lens: torch.Tensor
    holds_window: bool
    workspace: torch.Tensor | None = None


def make_shards(cache, lens, G: int, span: int, owned=None, device=None) -> list[Shard]:
    """Shards of a cache holding sequences of the given lengths (host list or
    array).  span must be a multiple of the page size; every shard must hold
    at least one entry of every sequence.  owned: the shard indices this
    process holds (all by default)."""
    lens = [int(x) for x in lens]
    if span % cache.page_size or span % 8:
        raise ValueError("the shard span must be a multiple of the page size and of 8")
    if any(L <= (G - 1) * span or L > G * span for L in lens):
        raise ValueError("every shard must hold at least one entry of every sequence")
    device = device or cache.idx_k.device
    out = []
    for g in (range(G) if owned is None else owned):
        lo = g * span
        loc = torch.tensor([min(span, L - lo) for L in lens], dtype=torch.int32, device=device)
        out.append(Shard(g, lo, span, cache.shard(lo // cache.page_size, span // cache.page_size), loc, g == G - 1))
    return out


class LocalExchange:
    """All G shards in this process: a gather is a stack in shard order."""

    def all_gather(self, parts: list[torch.Tensor]) -> torch.Tensor:
        return torch.stack(parts)


class DistExchange:
    """One shard per rank (rank = shard index): torch.distributed all-gather."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)

    def all_gather(self, parts: list[torch.Tensor]) -> torch.Tensor:
        (t,) = parts
        t = t.contiguous()
        bufs = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(bufs, t, group=self.group)
        return torch.stack(bufs)


class KernelOps:
    """The CUDA path: every step is a library kernel on the given stream."""

    def __init__(self, B_: int, err=None, stream=None, keep: int = 2048, topk: int = 512):
        self.B, self.err, self.stream, self.keep, self.topk = B_, err, stream, keep, topk

    def _ws(self, s: Shard, desc):
        if s.workspace is None:
            s.workspace = torch.zeros(B.workspace_bytes(desc, BLOCK, self.B, s.span), dtype=torch.uint8,
                                      device=s.lens.device)
        return s.workspace

    def block_topk(self, s: Shard, desc, q_idx, w):
        out = torch.empty((self.B, self.keep), dtype=torch.int32, device=s.lens.device)
        B.indexer_topk(desc, s.cache, BLOCK, q_idx, w, s.lens, out, self.B, s.span, self._ws(s, desc), err=self.err,
                       stream=self.stream)
        return out

    def token_topk(self, s: Shard, desc, q_idx, w, cand_local):
        out = torch.empty((self.B, self.topk), dtype=torch.int32, device=s.lens.device)
        B.indexer_topk(desc, s.cache, TOKEN, q_idx, w, s.lens, out, self.B, s.span, self._ws(s, desc),
                       cand_blocks=cand_local, err=self.err, stream=self.stream)
        return out

    def score_ids(self, s: Shard, desc, level: int, q_idx, w, ids, offset: int):
        sc = torch.empty(ids.shape, dtype=torch.float32, device=ids.device)
        gid = torch.empty(ids.shape, dtype=torch.int32, device=ids.device)
        B.indexer_score_ids(desc, s.cache, level, q_idx, w, s.lens, ids, offset, sc, gid, self.B, s.span,
                            err=self.err, stream=self.stream)
        return sc, gid

    def merge(self, scores, ids, k: int, lo: int, hi: int):
        out = torch.empty((self.B, k), dtype=torch.int32, device=scores.device)
        loc = torch.empty((self.B, k), dtype=torch.int32, device=scores.device)
        B.topk_merge(scores, ids, k, out, loc, lo, hi, stream=self.stream)
        return out, loc

    def attend(self, s: Shard, desc, q, local_set, swa, swa_lens):
        out = torch.empty((self.B, 16, 128), dtype=torch.float32, device=q.device)
        lse = torch.empty((self.B, 16), dtype=torch.float32, device=q.device)
        B.sparse_attn_decode(desc, s.cache, q, local_set, swa, s.lens, out, lse, self.B, swa_lens=swa_lens,
                             err=self.err, stream=self.stream)
        return out, lse

    def lse_merge(self, outs, lses):
        out = torch.empty(outs.shape[1:], dtype=torch.float32, device=outs.device)
        lse = torch.empty(lses.shape[1:], dtype=torch.float32, device=lses.device)
        B.attn_lse_merge(outs, lses, out, lse, stream=self.stream)
        return out, lse


def decode_step(modes, descs, shards: list[Shard], ops, exchange, q_idx, w, q, swa, swa_lens):
    """One decode step of len(modes) layers over the shards this process holds.

    Per layer l: q_idx[l] [B,4,64] bf16 bits and w[l] [B,4] (Full/Reindex), q[l]
    [B,16,128], swa[l] [B,window,256] and swa_lens [B] (the window's valid
    rows; read by the shard that holds the window).  Returns, per layer, the
    global index set [B,512] (positions of the whole sequence) and the merged
    (out [B,16,128], lse [B,16]); every process gets the same results."""
    keep, topk = ops.keep, ops.topk
    no_window = torch.zeros_like(swa_lens)
    cand_local = [None] * len(shards)
    set_local = [None] * len(shards)
    set_global = None
    res = []
    for l, m in enumerate(modes):
        if m == FULL:
            sc, gid = [], []
            for s in shards:
                blk = ops.block_topk(s, descs[l], q_idx[l], w[l])
                a, b = ops.score_ids(s, descs[l], BLOCK, q_idx[l], w[l], blk, s.lo // 8)
                sc.append(a)
                gid.append(b)
            S, I = exchange.all_gather(sc), exchange.all_gather(gid)
            for i, s in enumerate(shards):
                _, cand_local[i] = ops.merge(S, I, keep, s.lo // 8, (s.lo + s.span) // 8)
        if m in (FULL, REINDEX):
            if cand_local[0] is None:
                raise ValueError("a Reindex layer needs a preceding Full layer")
            sc, gid = [], []
            for i, s in enumerate(shards):
                tok = ops.token_topk(s, descs[l], q_idx[l], w[l], cand_local[i])
                a, b = ops.score_ids(s, descs[l], TOKEN, q_idx[l], w[l], tok, s.lo)
                sc.append(a)
                gid.append(b)
            S, I = exchange.all_gather(sc), exchange.all_gather(gid)
            for i, s in enumerate(shards):
                set_global, set_local[i] = ops.merge(S, I, topk, s.lo, s.lo + s.span)
        elif set_global is None:
            raise ValueError("a Reuse layer needs a preceding index set")
        outs, lses = [], []
        for i, s in enumerate(shards):
            o, x = ops.attend(s, descs[l], q[l], set_local[i], swa[l], swa_lens if s.holds_window else no_window)
            outs.append(o)
            lses.append(x)
        out, lse = ops.lse_merge(exchange.all_gather(outs), exchange.all_gather(lses))
        res.append(dict(idx=set_global, out=out, lse=lse))
    return res
