"""CPU oracle for the CSA2 sparse-attention step over an NVFP4 main-KV cache.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product path never
does.  It shares no code with the CUDA library.

The arithmetic lives in ``csa2_oracle.c`` (plain C, ``-O2 -ffp-contract=off``,
no fast-math).  This module only compiles it with gcc and marshals numpy arrays.
Every function cites, in the C file, the page section it follows and the
reading taken where the pages are silent.

Parity pins: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, library casts (torch float8/bfloat16) or
invariants, except where a docstring below says "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libcsa2_oracle.so")
_lock = threading.Lock()
_lib = None

FULL, REINDEX, REUSE = 0, 1, 2
H, D, IH, ID, CH = 16, 128, 4, 64, 256
CODE_BYTES, N_SCALES = 128, 16


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (seconds)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int


def _declare(L: ctypes.CDLL) -> None:
    L.orc_e4m3_value.restype = ctypes.c_double
    L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
    L.orc_e2m1_value.restype = ctypes.c_double
    L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_e2m1_encode.restype = ctypes.c_uint8
    L.orc_e2m1_encode.argtypes = [ctypes.c_float]
    for n in ("orc_e4m3_encode_n", "orc_e2m1_encode_n", "orc_f32_to_bf16_n"):
        getattr(L, n).restype = None
        getattr(L, n).argtypes = [_P, _P, _I64]
    L.orc_quant_entry.argtypes = [_P, _P, _P]
    L.orc_dequant_entry.argtypes = [_P, _P, _P]
    L.orc_quant_rows.argtypes = [_P, _I64, _I32, _P, _P]
    L.orc_pool_blocks.argtypes = [_P, _I64, _P]
    L.orc_score.restype = ctypes.c_float
    L.orc_score.argtypes = [_P, _P, _P]
    L.orc_score_rows.argtypes = [_P, _P, _P, _I64, _P]
    L.orc_topk_labels.restype = _I64
    L.orc_topk_labels.argtypes = [_P, _P, _I64, _I64, _P, _I64]
    L.orc_select_blocks.restype = _I64
    L.orc_select_blocks.argtypes = [_P, _I64, _P, _P, _I64, _P, _P]
    L.orc_select_tokens.restype = _I64
    L.orc_select_tokens.argtypes = [_P, _I64, _P, _I64, _P, _P, _I64, _P, _P, _P, _P]
    L.orc_attend.argtypes = [_P, _P, _I64, _P, _P, _P, _I64, _P, _P]
    L.orc_schedule.restype = _I32
    L.orc_schedule.argtypes = [_I32, _P]
    L.orc_decode_step.argtypes = [_I32, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P]
    L.orc_decode_batch.argtypes = [_I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P,
                                   _P, _P]
    L.orc_visible_entries.restype = _I64
    L.orc_visible_entries.argtypes = [_I64, _I32, _I64]
    L.orc_prefill_indexer.argtypes = [_I64, _P, _I32, _I64, _P, _P, _P, _I64, _P]
    L.orc_prefill_attn.argtypes = [_I64, _P, _P, _P, _I64, _P, _P, _P, _I64, _I64, _P, _P]
    L.orc_swa_replay.argtypes = [_P, _P, _I64, _I64, _P]
    L.orc_cache_bytes_per_token.restype = ctypes.c_double
    L.orc_cache_bytes_per_token.argtypes = [_I32, _P, ctypes.c_double, ctypes.c_double]


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# formats
# --------------------------------------------------------------------------

def e4m3_value(b: int) -> float:
    return lib().orc_e4m3_value(int(b) & 0xFF)


def e2m1_value(c: int) -> float:
    return lib().orc_e2m1_value(int(c) & 0xF)


def e4m3_encode(x) -> np.ndarray:
    x = _c(np.atleast_1d(x), np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(x), _p(out), x.size)
    return out


def e2m1_encode(x) -> np.ndarray:
    x = _c(np.atleast_1d(x), np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(x), _p(out), x.size)
    return out


def f32_to_bf16(x) -> np.ndarray:
    x = _c(np.atleast_1d(x), np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_bf16_n(_p(x), _p(out), x.size)
    return out


def bf16_to_f32(h) -> np.ndarray:
    h = _c(np.atleast_1d(h), np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# quantisation
# --------------------------------------------------------------------------

def quant_rows(src: np.ndarray, ratio: int = 1):
    """fp32 rows [n*ratio, 256] -> (codes u8 [n,128], scales u8 [n,16])."""
    src = _c(src, np.float32)
    assert src.ndim == 2 and src.shape[1] == CH and src.shape[0] % ratio == 0
    n = src.shape[0] // ratio
    codes = np.empty((n, CODE_BYTES), np.uint8)
    scales = np.empty((n, N_SCALES), np.uint8)
    lib().orc_quant_rows(_p(src), n, ratio, _p(codes), _p(scales))
    return codes, scales


def dequant(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """(codes [n,128], scales [n,16]) -> float64 [n,256] (exact)."""
    codes = _c(codes, np.uint8).reshape(-1, CODE_BYTES)
    scales = _c(scales, np.uint8).reshape(-1, N_SCALES)
    out = np.empty((codes.shape[0], CH), np.float64)
    L = lib()
    for i in range(codes.shape[0]):
        L.orc_dequant_entry(_p(codes[i]), _p(scales[i]), _p(out[i]))
    return out


# --------------------------------------------------------------------------
# indexer
# --------------------------------------------------------------------------

def pool_blocks(idx_k: np.ndarray) -> np.ndarray:
    """bf16 bits [L,64] -> pooled bf16 bits [ceil(L/8),64]."""
    idx_k = _c(idx_k, np.uint16)
    L_ = idx_k.shape[0]
    out = np.empty(((L_ + 7) // 8, ID), np.uint16)
    lib().orc_pool_blocks(_p(idx_k), L_, _p(out))
    return out


def score(q_idx: np.ndarray, w: np.ndarray, k: np.ndarray) -> float:
    q_idx, w, k = _c(q_idx, np.uint16), _c(w, np.float32), _c(k, np.uint16)
    return float(lib().orc_score(_p(q_idx), _p(w), _p(k)))


def score_rows(q_idx: np.ndarray, w: np.ndarray, rows: np.ndarray) -> np.ndarray:
    q_idx, w, rows = _c(q_idx, np.uint16), _c(w, np.float32), _c(rows, np.uint16)
    out = np.empty(rows.shape[0], np.float32)
    lib().orc_score_rows(_p(q_idx), _p(w), _p(rows), rows.shape[0], _p(out))
    return out


def topk(scores: np.ndarray, k: int, labels: np.ndarray | None = None, k_out: int | None = None) -> np.ndarray:
    scores = _c(scores, np.float32)
    labels = None if labels is None else _c(labels, np.int32)
    k_out = k if k_out is None else k_out
    out = np.empty(max(k_out, 1), np.int32)
    lib().orc_topk_labels(_p(scores), _p(labels), scores.size, k, _p(out), k_out)
    return out[:k_out]


def select_blocks(pooled, L: int, q_idx, w, keep: int = 2048, return_scores: bool = False):
    pooled, q_idx, w = _c(pooled, np.uint16), _c(q_idx, np.uint16), _c(w, np.float32)
    out = np.empty(keep, np.int32)
    sc = np.empty((L + 7) // 8, np.float32) if return_scores else None
    lib().orc_select_blocks(_p(pooled), L, _p(q_idx), _p(w), keep, _p(out), _p(sc))
    return (out, sc) if return_scores else out


def select_tokens(idx_k, L: int, blocks, q_idx, w, topk_: int = 512, return_scores: bool = False):
    idx_k, q_idx, w = _c(idx_k, np.uint16), _c(q_idx, np.uint16), _c(w, np.float32)
    blocks = None if blocks is None else _c(blocks, np.int32)
    nb = 0 if blocks is None else blocks.size
    out = np.empty(topk_, np.int32)
    cap = 8 * nb if blocks is not None else L
    sc = np.empty(max(cap, 1), np.float32)
    pos = np.empty(max(cap, 1), np.int32)
    nc = ctypes.c_int64(0)
    lib().orc_select_tokens(_p(idx_k), L, _p(blocks), nb, _p(q_idx), _p(w), topk_, _p(out), _p(sc), _p(pos),
                            ctypes.byref(nc))
    if return_scores:
        return out, sc[:nc.value], pos[:nc.value]
    return out


# --------------------------------------------------------------------------
# attention and schedule
# --------------------------------------------------------------------------

def attend(q, idx, codes, scales, swa):
    """One query (16 heads): sparse branch over idx (entry positions into
    codes/scales, -1 skipped) + SWA branch over swa [n,256] bf16 bits."""
    q, idx = _c(q, np.uint16), _c(idx, np.int32)
    codes, scales, swa = _c(codes, np.uint8), _c(scales, np.uint8), _c(swa, np.uint16)
    out = np.empty((H, D), np.float32)
    lse = np.empty(H, np.float32)
    n_swa = swa.shape[0] if swa.size else 0
    lib().orc_attend(_p(q), _p(idx), idx.size, _p(codes), _p(scales), _p(swa), n_swa, _p(out), _p(lse))
    return out, lse


def schedule(decoder: bool = True) -> np.ndarray:
    modes = np.empty(20, np.int32)
    n = lib().orc_schedule(1 if decoder else 0, _p(modes))
    return modes[:n]


def decode_step(modes, L: int, codes, scales, idx_k, pooled, q_idx, w, q, swa, window=128, keep=2048, topk_=512):
    """One decode step of one sequence.  Per-layer arrays have a leading layer
    axis: q_idx [n,4,64], w [n,4], q [n,16,128], swa [n,window,256] (rows beyond
    min(window, L) ignored).  keep=0: flat indexer over all L entries (the
    encoder's layers), pooled unused."""
    modes = _c(modes, np.int32)
    n = modes.size
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    idx_k, pooled = _c(idx_k, np.uint16), _c(pooled, np.uint16)
    q_idx, w, q, swa = _c(q_idx, np.uint16), _c(w, np.float32), _c(q, np.uint16), _c(swa, np.uint16)
    assert swa.shape[1] == window
    blocks = np.full(keep, -1, np.int32)
    sets = np.empty((n, topk_), np.int32)
    out = np.empty((n, H, D), np.float32)
    lse = np.empty((n, H), np.float32)
    lib().orc_decode_step(n, _p(modes), L, _p(codes), _p(scales), _p(idx_k), _p(pooled), _p(q_idx), _p(w), _p(q),
                          _p(swa), window, keep, topk_, _p(blocks), _p(sets), _p(out), _p(lse))
    return dict(blocks=blocks, idx=sets, out=out, lse=lse)


def decode_batch(modes, Ls, codes, scales, idx_k, pooled, q_idx, w, q, swa, window=128, keep=2048, topk_=512):
    """decode_step over a list of sequences, OpenMP-parallel over sequences.
    codes/scales/idx_k/pooled are lists of per-sequence arrays; q_idx, w, q and
    swa carry a leading [n_seq, n_layers] pair of axes."""
    modes = _c(modes, np.int32)
    nl, ns = modes.size, len(Ls)
    Ls = _c(np.asarray(Ls), np.int64)
    keep_alive = [_c(a, np.uint8) for a in codes] + [_c(a, np.uint8) for a in scales] + \
                 [_c(a, np.uint16) for a in idx_k] + [_c(a, np.uint16) for a in pooled]
    ptrs = [np.array([a.ctypes.data for a in keep_alive[i * ns:(i + 1) * ns]], np.uint64) for i in range(4)]
    q_idx, w, q, swa = _c(q_idx, np.uint16), _c(w, np.float32), _c(q, np.uint16), _c(swa, np.uint16)
    blocks = np.full((ns, keep), -1, np.int32)
    sets = np.empty((ns, nl, topk_), np.int32)
    out = np.empty((ns, nl, H, D), np.float32)
    lse = np.empty((ns, nl, H), np.float32)
    lib().orc_decode_batch(ns, nl, _p(modes), _p(Ls), _p(ptrs[0]), _p(ptrs[1]), _p(ptrs[2]), _p(ptrs[3]), _p(q_idx),
                           _p(w), _p(q), _p(swa), window, keep, topk_, _p(blocks), _p(sets), _p(out), _p(lse))
    del keep_alive
    return dict(blocks=blocks, idx=sets, out=out, lse=lse)


def visible_entries(p: int, ratio: int, n_entries: int) -> int:
    return int(lib().orc_visible_entries(p, ratio, n_entries))


def prefill_indexer(q_pos, ratio: int, n_entries: int, idx_k, q_idx, w, topk_=512):
    q_pos = _c(q_pos, np.int32)
    idx_k, q_idx, w = _c(idx_k, np.uint16), _c(q_idx, np.uint16), _c(w, np.float32)
    out = np.empty((q_pos.size, topk_), np.int32)
    lib().orc_prefill_indexer(q_pos.size, _p(q_pos), ratio, n_entries, _p(idx_k), _p(q_idx), _p(w), topk_, _p(out))
    return out


def prefill_attn(q_pos, q, idx, codes, scales, swa, swa_start: int, window: int = 128):
    q_pos = _c(q_pos, np.int32)
    q, idx = _c(q, np.uint16), _c(idx, np.int32)
    codes, scales, swa = _c(codes, np.uint8), _c(scales, np.uint8), _c(swa, np.uint16)
    T = q_pos.size
    assert int(q_pos.min()) - window + 1 >= swa_start or swa_start == 0
    out = np.empty((T, H, D), np.float32)
    lse = np.empty((T, H), np.float32)
    lib().orc_prefill_attn(T, _p(q_pos), _p(q), _p(idx), idx.shape[1], _p(codes), _p(scales), _p(swa), swa_start,
                           window, _p(out), _p(lse))
    return out, lse


def swa_replay(h, w_kv) -> np.ndarray:
    """Replayed window rows: bf16 bits [n, 256] = bf16(h [n, d] . w_kv [256, d]^T)."""
    h, w_kv = _c(h, np.uint16), _c(w_kv, np.uint16)
    n, d = h.shape
    assert w_kv.shape == (CH, d)
    out = np.empty((n, CH), np.uint16)
    lib().orc_swa_replay(_p(h), _p(w_kv), n, d, _p(out))
    return out


def cache_bytes_per_token(full_ratios, main_entry_bytes: float, idx_entry_bytes: float) -> float:
    r = _c(np.asarray(full_ratios), np.int32)
    return float(lib().orc_cache_bytes_per_token(r.size, _p(r), main_entry_bytes, idx_entry_bytes))
