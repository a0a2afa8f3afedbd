"""Helpers of the GPU parity tests: paged caches filled through the C ABI from
the seeded generators, and the comparison rules."""
from __future__ import annotations

import numpy as np
import torch

import synth

ATOL, RTOL_L2 = 2e-3, 1e-3  # attention tolerance: max-abs and relative L2 against the oracle


def dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bits16(x: np.ndarray) -> torch.Tensor:
    return dev(np.ascontiguousarray(x, np.uint16).view(np.int16))


class PagedSeqs:
    """A paged cache holding B sequences of the given entry lengths."""

    def __init__(self, csa2, lens, page_size=64, shuffle=True, seed=7, pooled=True, extra_pages=0,
                 main_kv_on_host=False):
        self.csa2 = csa2
        self.lens = np.asarray(lens, np.int64)
        self.page = page_size
        cap = self.lens + extra_pages * page_size
        self.table, n_phys = synth.page_table(seed, cap, page_size, shuffle)
        self.cache = csa2.KVCache(n_phys, page_size, torch.from_numpy(self.table), pooled=pooled,
                                  main_kv_on_host=main_kv_on_host)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def slots(self, seq, positions):
        return synth.slots(self.table, seq, positions, self.page)

    def append(self, seq, start, kv_rows, idx_rows, ratio=1, chunk=None):
        """Append entries start.. of one sequence: kv_rows fp32 [n*ratio,256]
        (or bf16 bits as uint16), idx_rows bf16 bits [n,64]."""
        n = idx_rows.shape[0]
        chunk = chunk or n
        for o in range(0, n, chunk):
            m = min(chunk, n - o)
            sl = dev(self.slots(seq, np.arange(start + o, start + o + m)).astype(np.int64))
            kv = kv_rows[o * ratio:(o + m) * ratio]
            kvt = bits16(kv).view(torch.bfloat16) if kv.dtype == np.uint16 else dev(kv.astype(np.float32))
            self.csa2.kv_quant_append(self.cache, kvt, bits16(idx_rows[o:o + m]), sl, ratio=ratio, err=self.err)

    def unpage(self, seq, L):
        s = torch.from_numpy(self.slots(seq, np.arange(L))).cuda()
        c = self.cache
        pooled = None
        if c.pooled is not None:
            ps = torch.from_numpy(self.slots(seq, np.arange(0, L, 8)) // 8).cuda()
            pooled = c.pooled[ps].cpu().numpy().view(np.uint16)
        sm = s.to(c.codes.device)  # the main KV may sit in pinned host memory
        return (c.codes[sm].cpu().numpy(), c.scales[sm].cpu().numpy(), c.idx_k[s].cpu().numpy().view(np.uint16),
                pooled)

    def errors(self):
        torch.cuda.synchronize()
        return int(self.err.item())


def check_attn(out, lse, ref_out, ref_lse, what=""):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref_out, np.float64)
    assert np.isfinite(out).all(), what
    err = np.abs(out - ref).max()
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= ATOL, f"{what} max-abs {err}"
    assert rel <= RTOL_L2, f"{what} rel-L2 {rel}"
    lerr = np.abs(np.asarray(lse, np.float64) - np.asarray(ref_lse, np.float64)).max()
    assert lerr <= ATOL, f"{what} lse max-abs {lerr}"


def check_sets(got, want, what=""):
    """Top-K sets are exact: scores are bit-identical by construction, so no
    near-tie exemption is needed (the exemption rule would apply only where the
    oracle's K-th and (K+1)-th scores differ by < 1e-6 relative)."""
    got, want = np.asarray(got), np.asarray(want)
    if not np.array_equal(got, want):
        bad = np.nonzero(got != want)
        raise AssertionError(f"{what}: {bad[0].size} index mismatches, first at {tuple(b[0] for b in bad)}")


# ---------------------------------------------------------------------------
# the encoder side of a decode step (flat indexer)
# ---------------------------------------------------------------------------

def encoder_layer_inputs(seed, B, lens, n_layers):
    q_idx = np.stack([np.concatenate([synth.q_idx(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    w = np.stack([np.concatenate([synth.w_idx(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    q = np.stack([np.concatenate([synth.q_heads(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    swa = np.zeros((B, n_layers, 128, 256), np.uint16)
    for b, L in enumerate(lens):
        for l in range(n_layers):
            swa[b, l, :min(128, L)] = synth.swa_rows(seed, l, b, min(128, L))
    return q_idx, w, q, swa


def run_encoder_step(csa2, ps, lens, q_idx, w, q, swa):
    """The encoder's 18 CSA2 layers (3 x (Full + 5 Reuse), ratio 2, flat
    indexer) through the schedule driver; no candidate-block buffer."""
    B, max_len = len(lens), int(max(lens))
    modes = csa2.schedule(False)
    n = len(modes)
    descs = [csa2.default_desc(m, 2, keep_blocks=0) for m in modes]
    t16 = lambda a: bits16(np.ascontiguousarray(a))  # noqa: E731
    out = [torch.empty((B, 16, 128), device="cuda") for _ in range(n)]
    lse = [torch.empty((B, 16), device="cuda") for _ in range(n)]
    sets = torch.full((n, B, 512), -9, dtype=torch.int32, device="cuda")
    ws = torch.zeros(csa2.workspace_bytes(descs[0], csa2.TOKEN, B, max_len), dtype=torch.uint8, device="cuda")
    csa2.decode_layers(descs, ps.cache, [t16(q_idx[:, l]) for l in range(n)],
                       [dev(np.ascontiguousarray(w[:, l])) for l in range(n)], [t16(q[:, l]) for l in range(n)],
                       [t16(swa[:, l]) for l in range(n)], dev(np.asarray(lens, np.int32)), None, sets, out, lse, B,
                       max_len, ws, err=ps.err)
    torch.cuda.synchronize()
    return dict(sets=sets.cpu().numpy(), out=[o.cpu().numpy() for o in out], lse=[x.cpu().numpy() for x in lse],
                modes=modes)


def compare_encoder_seq(orc, r, b, L, codes, scales, idx, q_idx, w, q, swa, what):
    modes = np.array(r["modes"], np.int32)
    ref = orc.decode_step(modes, int(L), codes, scales, idx, orc.pool_blocks(idx), q_idx, w, q, swa, keep=0)
    last = 0
    for l, m in enumerate(modes):
        if m != 2:
            last = l
        check_sets(r["sets"][last, b], ref["idx"][l], f"{what} layer {l} set")
        check_attn(r["out"][l][b], r["lse"][l][b], ref["out"][l], ref["lse"][l], f"{what} layer {l}")
