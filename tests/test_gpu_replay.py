"""SWA Bounded Replay on the GPU (tcgen05 projection) against the oracle: the
replayed window rows within the bound of their two bf16 roundings plus fp32
accumulation over d_model products of the fp64 definition (the tensor core
accumulates in fp32, in its own order; almost every row element is equal),
ring slots outside the window untouched, and the decode attention over the
replayed window within max-abs 2e-3 / rel-L2 1e-3 of the oracle's attention
over the same rows."""
import numpy as np
import pytest
import torch

import synth
from _gpu_util import PagedSeqs, bits16, check_attn, dev

pytestmark = pytest.mark.gpu
SEED = 1004


@pytest.fixture(scope="module")
def csa2():
    import fp4_kv_cache_nvfp4_b200 as m
    assert torch.cuda.is_available()
    m.lib()
    return m


def _ulps(a, b):
    """Distance in bf16 ulps of two bf16 bit arrays (order-preserving integers)."""
    def key(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(key(a) - key(b))


@pytest.mark.parametrize("d_model", [256, 4096])
def test_replay_rows_and_window_attention(csa2, orc, d_model):
    lens = [50, 128, 1000, 777]
    B, W = len(lens), 128
    layer = 3
    h = np.stack([synth.hidden_rows(SEED, layer, b, W, d_model) for b in range(B)])
    w_kv = synth.kv_projection(SEED, layer, d_model)
    sentinel = np.uint16(0x7F7F)
    swa = torch.full((B, W, 256), int(sentinel), dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sl = dev(np.array(lens, np.int32))
    for call in range(2):  # the replay is a pure function of its inputs
        csa2.swa_replay(bits16(h), bits16(w_kv), sl, swa, B, W, err=err)
        torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = swa.cpu().numpy().view(np.uint16)
    for b, L in enumerate(lens):
        n = min(W, L)
        want = orc.swa_replay(h[b, :n], w_kv)
        slots = (L - n + np.arange(n)) % W
        # bound: the two roundings to bf16 (half an ulp each; an ulp is at most
        # 2^-7 of the value, at the bottom of a binade) plus fp32 accumulation
        # over d_model products, |err| <= d 2^-24 sum|h w|
        hf = orc.bf16_to_f32(h[b, :n]).astype(np.float64)
        wf = orc.bf16_to_f32(w_kv).astype(np.float64)
        gf = orc.bf16_to_f32(got[b, slots]).astype(np.float64)
        rf = orc.bf16_to_f32(want).astype(np.float64)
        bound = 2.0 ** -7 * np.abs(rf) + 2.0 * d_model * 2.0 ** -24 * (np.abs(hf) @ np.abs(wf).T)
        excess = np.abs(gf - rf) - bound
        assert excess.max() <= 0, f"seq {b}: beyond the bound by {excess.max()}"
        u = _ulps(got[b, slots], want)
        assert (u == 0).mean() > 0.97 and (u <= 1).mean() > 0.999, f"seq {b}: {(u == 0).mean()}"
        untouched = np.setdiff1d(np.arange(W), slots)
        assert (got[b, untouched] == sentinel).all()

    # the window branch (plus a sparse set) over the replayed rows
    ps = PagedSeqs(csa2, lens)
    q = np.concatenate([synth.q_heads(SEED, layer, b) for b in range(B)])
    rng = np.random.default_rng(5)
    idx = np.full((B, 512), -1, np.int32)
    for b, L in enumerate(lens):
        ps.append(b, 0, synth.kv_rows(SEED, b, 0, L), synth.idx_k_rows(SEED, b, 0, L))
        sel = np.sort(rng.choice(L, min(512, L), replace=False))
        idx[b, :sel.size] = sel
    d = csa2.default_desc(csa2.REUSE, 1)
    out = torch.empty((B, 16, 128), device="cuda")
    lse = torch.empty((B, 16), device="cuda")
    csa2.sparse_attn_decode(d, ps.cache, bits16(q), dev(idx), swa, sl, out, lse, B, err=ps.err)
    torch.cuda.synchronize()
    assert ps.errors() == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b, L in enumerate(lens):
        # the oracle's attention over the very rows the kernel replayed (the
        # rows themselves were checked against the oracle's replay above)
        n = min(W, L)
        codes, scales = orc.quant_rows(synth.kv_rows(SEED, b, 0, L))
        ro, rl = orc.attend(q[b], idx[b], codes, scales, got[b, (L - n + np.arange(n)) % W])
        check_attn(out[b], lse[b], ro, rl, f"replayed window, seq {b}")


@pytest.mark.parametrize("d_model,W", [(64, 64), (192, 128), (320, 32)])
def test_replay_small_d_model_and_short_window(csa2, orc, d_model, W):
    """d_model split four ways leaves some CTAs of a cluster with no slice (64:
    three of four; 192: one; 320: slices of 1, 1, 1, 2) and their partial is
    zero; a window shorter than the 128-row tile reads the next sequence's rows
    past n_b and discards them.  Rows within the bound of the oracle, other ring
    slots untouched."""
    lens = [W // 2, W, 3 * W + 5, 1]
    B = len(lens)
    layer = 5
    h = np.stack([synth.hidden_rows(SEED, layer, b, W, d_model) for b in range(B)])
    w_kv = synth.kv_projection(SEED, layer, d_model)
    sentinel = np.uint16(0x7F7F)
    swa = torch.full((B, W, 256), int(sentinel), dtype=torch.int16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa2.swa_replay(bits16(h), bits16(w_kv), dev(np.array(lens, np.int32)), swa, B, W, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = swa.cpu().numpy().view(np.uint16)
    for b, L in enumerate(lens):
        n = min(W, L)
        want = orc.swa_replay(h[b, :n], w_kv)
        slots = (L - n + np.arange(n)) % W
        hf = orc.bf16_to_f32(h[b, :n]).astype(np.float64)
        wf = orc.bf16_to_f32(w_kv).astype(np.float64)
        gf = orc.bf16_to_f32(got[b, slots]).astype(np.float64)
        rf = orc.bf16_to_f32(want).astype(np.float64)
        bound = 2.0 ** -7 * np.abs(rf) + 2.0 * d_model * 2.0 ** -24 * (np.abs(hf) @ np.abs(wf).T)
        assert (np.abs(gf - rf) - bound).max() <= 0, f"seq {b}"
        assert (_ulps(got[b, slots], want) <= 1).mean() > 0.999
        untouched = np.setdiff1d(np.arange(W), slots)
        assert (got[b, untouched] == sentinel).all()
