"""Global-KV tiering: the main KV (FP4 codes and E4M3 scales) and the SWA rows
in pinned host memory that the kernels read in place, the indexer K in device
memory.  Attention then moves only its selected 144-byte entries and its window
rows over the host link.  The quant-append writes the main KV there, and the
schedule driver's results must equal those of the all-device cache bit for bit,
and the oracle's."""
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


def _fill(ps, seq, L):
    kv = synth.kv_rows(SEED, seq, 0, L)
    idx = synth.idx_k_rows(SEED, seq, 0, L)
    ps.append(seq, 0, kv, idx)
    return kv, idx


def _inputs(B, lens, n_layers=20):
    q_idx = np.stack([np.concatenate([synth.q_idx(SEED, l, b) for l in range(n_layers)]) for b in range(B)])
    w = np.stack([np.concatenate([synth.w_idx(SEED, l, b) for l in range(n_layers)]) for b in range(B)])
    q = np.stack([np.concatenate([synth.q_heads(SEED, l, b) for l in range(n_layers)]) for b in range(B)])
    swa = np.zeros((B, n_layers, 128, 256), np.uint16)
    for b, L in enumerate(lens):
        for l in range(n_layers):
            swa[b, l, :min(128, L)] = synth.swa_rows(SEED, l, b, min(128, L))
    return q_idx, w, q, swa


def _run(csa2, ps, lens, q_idx, w, q, swa, swa_on_host):
    B, max_len = len(lens), max(lens)
    modes = csa2.schedule(True)
    n = len(modes)
    descs = [csa2.default_desc(m, 1) for m in modes]
    t16 = lambda a: bits16(np.ascontiguousarray(a))  # noqa: E731
    if swa_on_host:
        s_t = [torch.from_numpy(np.ascontiguousarray(swa[:, l]).view(np.int16)).pin_memory() for l in range(n)]
        assert all(csa2.device_accessible(t) == 1 for t in s_t)
    else:
        s_t = [t16(swa[:, l]) for l in range(n)]
    out = [torch.empty((B, 16, 128), device="cuda") for _ in range(n)]
    lse = [torch.empty((B, 16), device="cuda") for _ in range(n)]
    cand = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    sets = torch.full((n, B, 512), -9, dtype=torch.int32, device="cuda")
    ws = torch.zeros(csa2.workspace_bytes(descs[0], csa2.BLOCK, B, max_len), dtype=torch.uint8, device="cuda")
    csa2.decode_layers(descs, ps.cache, [t16(q_idx[:, l]) for l in range(n)],
                       [dev(np.ascontiguousarray(w[:, l])) for l in range(n)], [t16(q[:, l]) for l in range(n)],
                       s_t, dev(np.asarray(lens, np.int32)), cand, sets, out, lse, B, max_len, ws, err=ps.err)
    torch.cuda.synchronize()
    return dict(blocks=cand.cpu().numpy(), sets=sets.cpu().numpy(), out=np.stack([o.cpu().numpy() for o in out]),
                lse=np.stack([x.cpu().numpy() for x in lse]), modes=modes)


def test_main_kv_and_window_in_host_memory(csa2, orc):
    lens = [20000, 9000, 130]
    B = len(lens)
    on_dev = PagedSeqs(csa2, lens)
    on_host = PagedSeqs(csa2, lens, main_kv_on_host=True)
    assert on_host.cache.codes.device.type == "cpu" and on_host.cache.codes.is_pinned()
    assert csa2.device_accessible(on_host.cache.codes) == 1 and csa2.device_accessible(on_host.cache.scales) == 1
    data = []
    for b, L in enumerate(lens):
        data.append(_fill(on_dev, b, L))
        _fill(on_host, b, L)
    torch.cuda.synchronize()
    # the quant-append wrote the same bytes into host memory
    for b, L in enumerate(lens):
        gc_d, gs_d, _, _ = on_dev.unpage(b, L)
        gc_h, gs_h, _, _ = on_host.unpage(b, L)
        np.testing.assert_array_equal(gc_h, gc_d)
        np.testing.assert_array_equal(gs_h, gs_d)
    q_idx, w, q, swa = _inputs(B, lens)
    r_dev = _run(csa2, on_dev, lens, q_idx, w, q, swa, swa_on_host=False)
    r_host = _run(csa2, on_host, lens, q_idx, w, q, swa, swa_on_host=True)
    np.testing.assert_array_equal(r_host["blocks"], r_dev["blocks"])
    np.testing.assert_array_equal(r_host["sets"], r_dev["sets"])
    np.testing.assert_array_equal(r_host["out"], r_dev["out"])  # same kernels, same bytes: bit-identical
    np.testing.assert_array_equal(r_host["lse"], r_dev["lse"])
    modes = orc.schedule(True)
    b, L = 1, lens[1]
    codes, scales = orc.quant_rows(data[b][0])
    idx = data[b][1]
    ref = orc.decode_step(modes, L, codes, scales, idx, orc.pool_blocks(idx), q_idx[b], w[b], q[b], swa[b])
    last = 0
    for l, m in enumerate(modes):
        if m != 2:
            last = l
        check_sets(r_host["sets"][last, b], ref["idx"][l], f"layer {l} set")
        check_attn(r_host["out"][l][b], r_host["lse"][l][b], ref["out"][l], ref["lse"][l], f"layer {l}")
    assert on_dev.errors() == 0 and on_host.errors() == 0
