"""Seeded synthetic inputs shared by the tests, the oracle runs and the benchmark.

This module holds none of the method's arithmetic: it only draws random
numbers and lays out the workloads.  Every tensor role draws from its own
counter-seeded stream (numpy Philox keyed by [base seed, role, ...]), so a
slice of rows can be regenerated on its own and the oracle and the CUDA path
receive the very same values.

Workloads (sizes of the five benchmark configurations):
  c1  one Full layer, one decode step, L = 4096, B = 1
  c2  decoder stack (20 layers), L = 65,536, B = 8
  c3  encoder prefill, 32,768 tokens (16,384 ratio-2 entries), last 4096
      tokens are the queries, 6 layers (1 Full + 5 Reuse)
  c4  decoder stack, L = 1,048,576, B = 8, plus one append per sequence
  c5  64 ragged sequences, L log-uniform in [4096, 2^20], 64-entry pages in a
      random permutation, plus a 16,384-row bf16 append burst
Distributions: main-KV rows fp32 N(0,1) times a per-channel gain U(0.5, 2)
(separately for the 128 K and the 128 V channels, shared by all positions and
sequences); indexer q and k bf16 N(0,1); indexer weights U(0,1); attention q
bf16 N(0,1); SWA rows bf16 N(0,1) times the same gain.
"""
from __future__ import annotations

import math

import numpy as np

ROLES = {"gain": 1, "kv": 2, "idx_k": 3, "q": 4, "q_idx": 5, "w": 6, "swa": 7, "lens": 8, "pages": 9, "burst": 10,
         "tok": 11, "hidden": 12, "w_kv": 13}
D_MODEL = 4096  # hidden size of the synthetic SWA replay (the pages give none)
CHUNK = 4096  # rows per independently seeded chunk
CH, IDD, H, D, IH = 256, 64, 16, 128, 4

CONFIGS = {
    1: dict(name="full-layer-4k-b1", seed=1001, L=4096, B=1, ratio=1, layers=1),
    2: dict(name="decoder-20l-64k-b8", seed=1002, L=65536, B=8, ratio=1, layers=20),
    3: dict(name="encoder-prefill-32k-t4096-6l", seed=1003, tokens=32768, T=4096, ratio=2, layers=6),
    4: dict(name="decoder-20l-1m-b8", seed=1004, L=1 << 20, B=8, ratio=1, layers=20),
    5: dict(name="ragged-64seq-paged", seed=1005, B=64, lo=4096, hi=1 << 20, page=64, burst=16384, layers=20),
    # the encoder's 18 CSA2 layers per generated token: 1M tokens at ratio 2
    6: dict(name="encoder-decode-18l-1m-b8", seed=1006, L=1 << 19, B=8, ratio=2, layers=18, decoder=False),
}


def rng(seed: int, role: str, *keys: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed), ROLES[role]] + [int(k) & 0xFFFFFFFF for k in keys])
    return np.random.Generator(np.random.Philox(ss))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16) by torch's round-to-nearest-even cast."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def gain(seed: int) -> np.ndarray:
    """Per-channel gain [256] (K channels 0..127, V channels 128..255)."""
    return rng(seed, "gain").uniform(0.5, 2.0, CH).astype(np.float32)


def _chunked(seed, role, seq, start, count, width, draw):
    out = np.empty((count, width), np.float32)
    c0, c1 = start // CHUNK, (start + count - 1) // CHUNK if count else start // CHUNK - 1
    for c in range(c0, c1 + 1):
        blk = draw(rng(seed, role, seq, c), (CHUNK, width))
        lo = max(start, c * CHUNK)
        hi = min(start + count, (c + 1) * CHUNK)
        out[lo - start:hi - start] = blk[lo - c * CHUNK:hi - c * CHUNK]
    return out


def _normal(g, shape):
    return g.standard_normal(shape, dtype=np.float32)


def kv_rows(seed: int, seq: int, start: int, count: int, g: np.ndarray | None = None) -> np.ndarray:
    """Main-KV source rows [count, 256] fp32 for token positions start.. of seq."""
    g = gain(seed) if g is None else g
    return _chunked(seed, "kv", seq, start, count, CH, _normal) * g[None, :]


def kv_rows_bf16(seed: int, seq: int, start: int, count: int, g: np.ndarray | None = None) -> np.ndarray:
    return to_bf16_bits(kv_rows(seed, seq, start, count, g))


def idx_k_rows(seed: int, seq: int, start: int, count: int) -> np.ndarray:
    """Indexer-K rows [count, 64] bf16 bits."""
    return to_bf16_bits(_chunked(seed, "idx_k", seq, start, count, IDD, _normal))


def q_heads(seed: int, layer: int, seq: int, n: int = 1) -> np.ndarray:
    """Attention queries [n, 16, 128] bf16 bits."""
    return to_bf16_bits(_normal(rng(seed, "q", layer, seq), (n, H, D)))


def q_idx(seed: int, layer: int, seq: int, n: int = 1) -> np.ndarray:
    """Indexer queries [n, 4, 64] bf16 bits."""
    return to_bf16_bits(_normal(rng(seed, "q_idx", layer, seq), (n, IH, IDD)))


def w_idx(seed: int, layer: int, seq: int, n: int = 1) -> np.ndarray:
    """Indexer head weights [n, 4] fp32 U(0,1)."""
    return rng(seed, "w", layer, seq).uniform(0.0, 1.0, (n, IH)).astype(np.float32)


def swa_rows(seed: int, layer: int, seq: int, n: int, g: np.ndarray | None = None) -> np.ndarray:
    """SWA K|V rows [n, 256] bf16 bits of one layer."""
    g = gain(seed) if g is None else g
    return to_bf16_bits(_normal(rng(seed, "swa", layer, seq), (n, CH)) * g[None, :])


def hidden_rows(seed: int, layer: int, seq: int, n: int, d: int = D_MODEL) -> np.ndarray:
    """Synthetic hidden states [n, d] bf16 bits N(0,1) of a layer's window tokens
    (the input of the SWA Bounded Replay)."""
    return to_bf16_bits(_normal(rng(seed, "hidden", layer, seq), (n, d)))


def kv_projection(seed: int, layer: int, d: int = D_MODEL) -> np.ndarray:
    """Synthetic K|V projection [256, d] bf16 bits: N(0, 1/d) times the per-channel
    gain, so the replayed rows have the SWA rows' distribution."""
    g = gain(seed)
    return to_bf16_bits(_normal(rng(seed, "w_kv", layer), (CH, d)) * (g[:, None] / np.float32(math.sqrt(d))))


def ragged_lens(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    """L_i = floor(exp(U(ln lo, ln hi)))."""
    u = rng(seed, "lens").uniform(math.log(lo), math.log(hi), B)
    return np.floor(np.exp(u)).astype(np.int64).clip(lo, hi)


def page_table(seed: int, lens, page_size: int, shuffle: bool = True, max_pages: int | None = None):
    """Page table [B, max_pages] int32 covering each sequence's entries, with
    the physical pages a random permutation (or in order).  Unused slots -1.
    Returns (table, n_phys_pages)."""
    lens = np.asarray(lens, np.int64)
    need = (lens + page_size - 1) // page_size
    mp = int(need.max()) if max_pages is None else max_pages
    total = int(need.sum())
    perm = rng(seed, "pages").permutation(total).astype(np.int32) if shuffle else np.arange(total, dtype=np.int32)
    table = np.full((lens.size, mp), -1, np.int32)
    o = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[o:o + n]
        o += n
    return table, total


def slots(table: np.ndarray, seq: int, positions: np.ndarray, page_size: int) -> np.ndarray:
    """Physical entry slots of the given positions of one sequence (input layout)."""
    positions = np.asarray(positions, np.int64)
    return table[seq, positions // page_size].astype(np.int64) * page_size + positions % page_size
