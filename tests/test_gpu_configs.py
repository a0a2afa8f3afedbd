"""The benchmark configurations at full size (five of the decoder and prefill,
and the encoder side of a decode step), in the launch configuration bench.py
times (decode: quant-append + the schedule driver), checked
against the oracle: every sequence where the oracle can afford it, sampled
sequences or queries otherwise (the rest of the batch is filled with seeded
device-side data of the same distribution, so the GPU still runs the full
launch).  Bit-exact sets/codes, attention within max-abs 2e-3 / rel-L2 1e-3."""
import numpy as np
import pytest
import torch

import synth
from _gpu_util import (PagedSeqs, bits16, check_attn, check_sets, compare_encoder_seq, dev, encoder_layer_inputs,
                       run_encoder_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


CHUNK = 1 << 16


def fill_synth(ps, orc, seq, L, seed, ratio=1, bf16=False):
    """Append L entries of seeded synth data; return the oracle's view of them."""
    g = synth.gain(seed)
    codes = np.empty((L, 128), np.uint8)
    scales = np.empty((L, 16), np.uint8)
    idx = np.empty((L, 64), np.uint16)
    for e0 in range(0, L, CHUNK):
        m = min(CHUNK, L - e0)
        kv = synth.kv_rows(seed, seq, e0 * ratio, m * ratio, g)
        ik = synth.idx_k_rows(seed, seq, e0, m)
        src = synth.to_bf16_bits(kv) if bf16 else kv
        ps.append(seq, e0, src, ik, ratio=ratio)
        if bf16:
            kv = orc.bf16_to_f32(src).reshape(kv.shape)
        codes[e0:e0 + m], scales[e0:e0 + m] = orc.quant_rows(kv, ratio=ratio)
        idx[e0:e0 + m] = ik
    return codes, scales, idx


def fill_device(ps, csa2, seq, L, gen):
    """Append L entries of seeded device-side data (same distributions)."""
    gain = torch.from_numpy(synth.gain(1)).cuda()
    for e0 in range(0, L, CHUNK):
        m = min(CHUNK, L - e0)
        kv = torch.randn((m, 256), generator=gen, device="cuda") * gain
        ik = torch.randn((m, 64), generator=gen, device="cuda").to(torch.bfloat16).view(torch.int16)
        sl = dev(ps.slots(seq, np.arange(e0, e0 + m)).astype(np.int64))
        csa2.kv_quant_append(ps.cache, kv, ik, sl, err=ps.err)


def layer_inputs(seed, B, lens, n_layers):
    q_idx = np.stack([np.concatenate([synth.q_idx(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    w = np.stack([np.concatenate([synth.w_idx(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    q = np.stack([np.concatenate([synth.q_heads(seed, l, b) for l in range(n_layers)]) for b in range(B)])
    swa = np.zeros((B, n_layers, 128, 256), np.uint16)
    for b, L in enumerate(lens):
        for l in range(n_layers):
            swa[b, l, :min(128, L)] = synth.swa_rows(seed, l, b, min(128, L))
    return q_idx, w, q, swa


def run_step(csa2, ps, lens, q_idx, w, q, swa, n_layers):
    B = len(lens)
    max_len = int(max(lens))
    modes = csa2.schedule(True)[:n_layers]
    descs = [csa2.default_desc(m, 1) for m in modes]
    t16 = lambda a: bits16(np.ascontiguousarray(a))  # noqa: E731
    out = [torch.empty((B, 16, 128), device="cuda") for _ in range(n_layers)]
    lse = [torch.empty((B, 16), device="cuda") for _ in range(n_layers)]
    cand = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    sets = torch.empty((n_layers, B, 512), dtype=torch.int32, device="cuda")
    ws = torch.zeros(csa2.workspace_bytes(descs[0], csa2.BLOCK, B, max_len), dtype=torch.uint8, device="cuda")
    csa2.decode_layers(descs, ps.cache, [t16(q_idx[:, l]) for l in range(n_layers)],
                       [dev(np.ascontiguousarray(w[:, l])) for l in range(n_layers)],
                       [t16(q[:, l]) for l in range(n_layers)], [t16(swa[:, l]) for l in range(n_layers)],
                       dev(np.asarray(lens, np.int32)), cand, sets, out, lse, B, max_len, ws, err=ps.err)
    torch.cuda.synchronize()
    return dict(blocks=cand.cpu().numpy(), sets=sets.cpu().numpy(), out=[o.cpu().numpy() for o in out],
                lse=[x.cpu().numpy() for x in lse], modes=modes)


def compare_seq(orc, r, b, L, codes, scales, idx, q_idx, w, q, swa, n_layers, what):
    modes = np.array(r["modes"], np.int32)
    ref = orc.decode_step(modes, int(L), codes, scales, idx, orc.pool_blocks(idx), q_idx, w, q, swa)
    check_sets(r["blocks"][b], ref["blocks"], f"{what} blocks")
    last = 0
    for l in range(n_layers):
        if modes[l] != 2:
            last = l
        check_sets(r["sets"][last, b], ref["idx"][l], f"{what} layer {l} set")
        check_attn(r["out"][l][b], r["lse"][l][b], ref["out"][l], ref["lse"][l], f"{what} layer {l}")


def test_config1_full_layer_4k(csa2, orc):
    c = synth.CONFIGS[1]
    L, seed = c["L"], c["seed"]
    ps = PagedSeqs(csa2, [L])
    codes, scales, idx = fill_synth(ps, orc, 0, L, seed)
    q_idx, w, q, swa = layer_inputs(seed, 1, [L], 1)
    r = run_step(csa2, ps, [L], q_idx, w, q, swa, 1)
    compare_seq(orc, r, 0, L, codes, scales, idx, q_idx[0], w[0], q[0], swa[0], 1, "config 1")
    assert ps.errors() == 0


def test_config2_decoder_64k_b8(csa2, orc):
    c = synth.CONFIGS[2]
    L, B, seed = c["L"], c["B"], c["seed"]
    ps = PagedSeqs(csa2, [L] * B)
    data = [fill_synth(ps, orc, b, L, seed) for b in range(B)]
    q_idx, w, q, swa = layer_inputs(seed, B, [L] * B, 20)
    r = run_step(csa2, ps, [L] * B, q_idx, w, q, swa, 20)
    for b in range(B):
        compare_seq(orc, r, b, L, *data[b], q_idx[b], w[b], q[b], swa[b], 20, f"config 2 seq {b}")
    assert ps.errors() == 0


def test_config4_decoder_1m_b8_sampled(csa2, orc):
    """B = 8 at L = 2^20 plus the step's append; sequences 0 and 5 are checked
    against the oracle."""
    c = synth.CONFIGS[4]
    L, B, seed = c["L"], c["B"], c["seed"]
    ps = PagedSeqs(csa2, [L] * B)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    sampled = {0: None, 5: None}
    for b in range(B):
        if b in sampled:
            # the last entry arrives through a one-row append, the way a decode step adds it
            sampled[b] = fill_synth(ps, orc, b, L - 1, seed)
        else:
            fill_device(ps, csa2, b, L - 1, gen)
    # the step's quant-append of token L-1 for every sequence
    kv_new = np.concatenate([synth.kv_rows(seed, b, L - 1, 1) for b in range(B)])
    ik_new = np.concatenate([synth.idx_k_rows(seed, b, L - 1, 1) for b in range(B)])
    sl = np.concatenate([ps.slots(b, [L - 1]) for b in range(B)]).astype(np.int64)
    csa2.kv_quant_append(ps.cache, dev(kv_new), bits16(ik_new), dev(sl), err=ps.err)
    q_idx, w, q, swa = layer_inputs(seed, B, [L] * B, 20)
    r = run_step(csa2, ps, [L] * B, q_idx, w, q, swa, 20)
    for b, (codes, scales, idx) in sampled.items():
        c1, s1 = orc.quant_rows(kv_new[b:b + 1])
        codes = np.concatenate([codes, c1])
        scales = np.concatenate([scales, s1])
        idx = np.concatenate([idx, ik_new[b:b + 1]])
        gc, gs, gk, gp = ps.unpage(b, L)
        np.testing.assert_array_equal(gc, codes)
        np.testing.assert_array_equal(gs, scales)
        np.testing.assert_array_equal(gp, orc.pool_blocks(idx))
        compare_seq(orc, r, b, L, codes, scales, idx, q_idx[b], w[b], q[b], swa[b], 20, f"config 4 seq {b}")
    assert ps.errors() == 0


def test_config5_ragged_paged_sampled(csa2, orc):
    """64 sequences, log-uniform lengths in [4096, 2^20], permuted 64-entry
    pages; one decode step, then a 16,384-row bf16 append burst (256 rows at
    the tail of every sequence).  The shortest, a middle and the longest
    sequence are checked against the oracle; the burst is checked bit-exact on
    the same sequences."""
    c = synth.CONFIGS[5]
    B, seed = c["B"], c["seed"]
    lens = synth.ragged_lens(seed, B, c["lo"], c["hi"])
    burst = c["burst"] // B
    ps = PagedSeqs(csa2, lens, extra_pages=(burst + 63) // 64, seed=seed)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    order = np.argsort(lens)
    sampled = {int(order[0]): None, int(order[B // 2]): None, int(order[-1]): None}
    for b in range(B):
        if b in sampled:
            sampled[b] = fill_synth(ps, orc, b, int(lens[b]), seed)
        else:
            fill_device(ps, csa2, b, int(lens[b]), gen)
    q_idx, w, q, swa = layer_inputs(seed, B, lens, 20)
    r = run_step(csa2, ps, lens, q_idx, w, q, swa, 20)
    for b, (codes, scales, idx) in sampled.items():
        compare_seq(orc, r, b, int(lens[b]), codes, scales, idx, q_idx[b], w[b], q[b], swa[b], 20,
                    f"config 5 seq {b} (L={lens[b]})")
    # the burst: 256 bf16 rows per sequence at its tail, all in one call
    rows = np.concatenate([synth.kv_rows_bf16(seed + 1, b, int(lens[b]), burst) for b in range(B)])
    irows = np.concatenate([synth.idx_k_rows(seed + 1, b, int(lens[b]), burst) for b in range(B)])
    sl = np.concatenate([ps.slots(b, np.arange(lens[b], lens[b] + burst)) for b in range(B)]).astype(np.int64)
    csa2.kv_quant_append(ps.cache, bits16(rows).view(torch.bfloat16), bits16(irows), dev(sl), err=ps.err)
    torch.cuda.synchronize()
    for b, (codes, scales, idx) in sampled.items():
        L0 = int(lens[b])
        o = list(range(B)).index(b) * burst
        bc, bs = orc.quant_rows(orc.bf16_to_f32(rows[o:o + burst]).reshape(burst, 256))
        gc, gs, gk, gp = ps.unpage(b, L0 + burst)
        np.testing.assert_array_equal(gc[L0:], bc)
        np.testing.assert_array_equal(gs[L0:], bs)
        np.testing.assert_array_equal(gk[L0:], irows[o:o + burst])
        np.testing.assert_array_equal(gp, orc.pool_blocks(np.concatenate([idx, irows[o:o + burst]])))
    assert ps.errors() == 0


def test_config3_encoder_prefill_sampled(csa2, orc):
    """32,768 tokens -> 16,384 ratio-2 entries; the last 4096 tokens are the
    queries; 1 Full + 5 Reuse layers.  The GPU runs all 4096 queries; 160
    queries (both ends of the chunk and a stride through it) are checked."""
    c = synth.CONFIGS[3]
    tokens, T, seed = c["tokens"], c["T"], c["seed"]
    n_ent = tokens // 2
    ps = PagedSeqs(csa2, [n_ent], pooled=False)
    codes, scales, idx = fill_synth(ps, orc, 0, n_ent, seed, ratio=2, bf16=True)
    q_pos = np.arange(tokens - T, tokens, dtype=np.int32)
    q_idx = synth.q_idx(seed, 0, 0, T)
    w = synth.w_idx(seed, 0, 0, T)
    d_full = csa2.default_desc(csa2.FULL, 2)
    ws = torch.zeros(csa2.workspace_bytes(d_full, csa2.TOKEN, T, n_ent, prefill=True), dtype=torch.uint8,
                     device="cuda")
    sets = torch.empty((T, 512), dtype=torch.int32, device="cuda")
    csa2.indexer_topk(d_full, ps.cache, csa2.TOKEN, bits16(q_idx), dev(w), dev(np.array([n_ent], np.int32)), sets, T,
                      n_ent, ws, q_pos=dev(q_pos), err=ps.err)
    swa_start = int(q_pos[0]) - 127
    outs = []
    for l in range(6):
        q = synth.q_heads(seed, l, 0, T)
        swa = synth.swa_rows(seed, l, 0, tokens - swa_start)
        out = torch.empty((T, 16, 128), device="cuda")
        lse = torch.empty((T, 16), device="cuda")
        d = csa2.default_desc(csa2.FULL if l == 0 else csa2.REUSE, 2)
        csa2.sparse_attn_prefill(d, ps.cache, bits16(q), sets, dev(q_pos), bits16(swa), swa_start, n_ent, out, lse,
                                 T, err=ps.err)
        outs.append((q, swa, out.cpu().numpy(), lse.cpu().numpy()))
    got = sets.cpu().numpy()
    pick = np.unique(np.concatenate([np.arange(16), np.arange(T - 16, T), np.arange(0, T, 32)]))
    want = orc.prefill_indexer(q_pos[pick], 2, n_ent, idx, q_idx[pick], w[pick])
    check_sets(got[pick], want, "config 3 indexer")
    for l, (q, swa, o, lse) in enumerate(outs):
        ro, rl = orc.prefill_attn(q_pos[pick], q[pick], want, codes, scales, swa, swa_start)
        check_attn(o[pick], lse[pick], ro, rl, f"config 3 layer {l}")
    assert ps.errors() == 0


def test_config6_encoder_decode_1m_b8_sampled(csa2, orc):
    """The encoder side of one generated token at 1M tokens: B = 8 sequences of
    524,288 entries at ratio 2 through the 18 encoder layers (3 x (Full + 5
    Reuse), flat indexer), the launch configuration bench.py --config 6 times.
    Sequences 0 and 3 are checked against the oracle; the rest of the batch
    holds seeded device-side data."""
    c = synth.CONFIGS[6]
    L, B, seed = c["L"], c["B"], c["seed"]
    ps = PagedSeqs(csa2, [L] * B)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    sampled = {0: None, 3: None}
    for b in range(B):
        if b in sampled:
            sampled[b] = fill_synth(ps, orc, b, L, seed, ratio=2)
        else:
            fill_device(ps, csa2, b, L, gen)
    q_idx, w, q, swa = encoder_layer_inputs(seed, B, [L] * B, 18)
    r = run_encoder_step(csa2, ps, [L] * B, q_idx, w, q, swa)
    for b, (codes, scales, idx) in sampled.items():
        compare_encoder_seq(orc, r, b, L, codes, scales, idx, q_idx[b], w[b], q[b], swa[b], f"config 6 seq {b}")
    assert ps.errors() == 0
