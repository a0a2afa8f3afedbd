"""ctypes marshalling for include/csa2.h.  No arithmetic of the method lives here."""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libcsa2.so")

FULL, REINDEX, REUSE = 0, 1, 2
BLOCK, TOKEN = 0, 1
F32, BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported dimension or size", 3: "CUDA error",
          4: "workspace missing or too small"}


class CSA2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: csa2 status {status} ({STATUS.get(status, '?')})")
        self.status = status


class LayerDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("mode", "ratio", "topk", "block", "keep_blocks", "window", "n_heads",
                                                "head_dim", "idx_heads", "idx_dim")]


class _Cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("idx_k", ctypes.c_void_p),
                ("idx_k_pooled", ctypes.c_void_p), ("page_table", ctypes.c_void_p), ("page_size", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("n_phys_pages", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded libcsa2.so.  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(lib_path):
                raise ImportError(f"libcsa2.so not built ({lib_path}); run python -m fp4_kv_cache_nvfp4_b200.build")
            L = ctypes.CDLL(lib_path)
            L.csa2_layer_desc_default.argtypes = [ctypes.POINTER(LayerDesc), _I32, _I32]
            L.csa2_layer_desc_default.restype = None
            L.csa2_schedule.argtypes = [_I32, _P]
            L.csa2_schedule.restype = _I32
            L.csa2_kv_quant_append.argtypes = [ctypes.POINTER(_Cache), _P, _I32, _P, _I64, _I32, _P, _P, _P]
            L.csa2_indexer_workspace_bytes.argtypes = [ctypes.POINTER(LayerDesc), _I32, _I32, _I64, _I32]
            L.csa2_indexer_workspace_bytes.restype = _SZ
            L.csa2_indexer_topk.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_Cache), _I32, _P, _P, _P, _P,
                                            _P, _P, _P, _I32, _I64, _P, _SZ, _P, _P]
            L.csa2_sparse_attn_decode.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_Cache), _P, _P, _P, _P,
                                                  _P, _P, _P, _I32, _P, _P]
            L.csa2_sparse_attn_prefill.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_Cache), _P, _P, _P, _P,
                                                   _I32, _I32, _P, _P, _I32, _P, _P]
            L.csa2_decode_layers.argtypes = [_I32, ctypes.POINTER(LayerDesc), ctypes.POINTER(_Cache), _P, _P, _P, _P,
                                             _P, _P, _P, _P, _P, _P, _I32, _I64, _P, _SZ, _P, _P]
            for n in ("csa2_kv_quant_append", "csa2_indexer_topk", "csa2_sparse_attn_decode",
                      "csa2_sparse_attn_prefill", "csa2_decode_layers"):
                getattr(L, n).restype = _I32
            L.csa2_indexer_topk_noalloc.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_Cache), _I32, _P, _P,
                                                    _P, _P, _P, _I32, _I64, _P, _P]
            L.csa2_indexer_topk_noalloc.restype = _I32
            L.csa2_status_string.argtypes = [_I32]
            L.csa2_status_string.restype = ctypes.c_char_p
            L.csa2_abi_version.restype = _I32
            L.csa2_device_accessible.argtypes = [_P]
            L.csa2_device_accessible.restype = _I32
            L.csa2_indexer_score_ids.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(_Cache), _I32, _P, _P,
                                                 _P, _P, _I32, _I32, _P, _P, _I32, _I64, _P, _P]
            L.csa2_topk_merge.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _I32, _P, _P, _I32, _P]
            L.csa2_attn_lse_merge.argtypes = [_I32, _P, _P, _P, _P, _I32, _P]
            for n in ("csa2_indexer_score_ids", "csa2_topk_merge", "csa2_attn_lse_merge"):
                getattr(L, n).restype = _I32
            L.csa2_swa_replay.argtypes = [_P, _P, _P, _P, _I32, _I32, _I32, _P, _P]
            L.csa2_swa_replay.restype = _I32
            L.csa2_test_empty_chain.argtypes = [_I32, _I32, _I32, _P, _P]
            L.csa2_test_empty_chain.restype = _I32
            L.csa2_test_set_wait_limit.argtypes = [ctypes.c_uint32]
            L.csa2_test_set_wait_limit.restype = ctypes.c_uint32
            _lib = L
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(status: int, what: str) -> None:
    if status != 0:
        raise CSA2Error(status, what)


def abi_version() -> int:
    return int(lib().csa2_abi_version())


def device_accessible(t) -> int:
    """1 if kernels can read the tensor (or raw address) in place, 0 if not, -1 on a CUDA error."""
    return int(lib().csa2_device_accessible(_ptr(t)))


def indexer_score_ids(desc: LayerDesc, cache: KVCache, level: int, q_idx, w, seq_lens, ids, id_offset: int,
                      scores, ids_out, n: int, max_len: int, err=None, stream=None) -> None:
    """Scores of the given ids (exact chains) and the ids plus id_offset."""
    _check(lib().csa2_indexer_score_ids(ctypes.byref(desc), ctypes.byref(cache.struct()), level, _ptr(q_idx),
                                        _ptr(w), _ptr(seq_lens), _ptr(ids), ids.shape[-1], id_offset, _ptr(scores),
                                        _ptr(ids_out), n, max_len, _ptr(err), _stream(stream)), "indexer_score_ids")


def topk_merge(scores, ids, k: int, out, out_local=None, lo: int = 0, hi: int = 0, stream=None) -> None:
    """Top-k of gathered (score, id) pairs [parts, n, part_len]; ids ascending in pair order."""
    parts, n, plen = scores.shape
    _check(lib().csa2_topk_merge(_ptr(scores), _ptr(ids), parts, plen, k, lo, hi, _ptr(out), _ptr(out_local), n,
                                 _stream(stream)), "topk_merge")


def attn_lse_merge(out_parts, lse_parts, out, lse, stream=None) -> None:
    """Log-sum-exp merge of partial attention outputs [G, rows, 16, 128] / [G, rows, 16]."""
    _check(lib().csa2_attn_lse_merge(out_parts.shape[0], _ptr(out_parts), _ptr(lse_parts), _ptr(out), _ptr(lse),
                                     out_parts.shape[1], _stream(stream)), "attn_lse_merge")


def swa_replay(h, w_kv, seq_lens, swa_kv, B: int, window: int = 128, err=None, stream=None) -> None:
    """Recompute the window K|V rows of B sequences from their hidden states
    h [B, window, d_model] and the projection w_kv [256, d_model] (bf16 bits)."""
    _check(lib().csa2_swa_replay(_ptr(h), _ptr(w_kv), _ptr(seq_lens), _ptr(swa_kv), B, h.shape[-1], window,
                                 _ptr(err), _stream(stream)), "swa_replay")


def test_set_wait_limit(polls: int) -> int:
    """Test hook: poll limit of the block-level indexer's cp.async copy-ring
    waits (returns the previous limit)."""
    return int(lib().csa2_test_set_wait_limit(polls))


def test_empty_chain(n_kernels: int, ctas: int, threads: int = 128, sink=None, stream=None) -> None:
    """Measurement helper: n_kernels empty dependent kernels (programmatic
    dependent launch) on the stream."""
    _check(lib().csa2_test_empty_chain(n_kernels, ctas, threads, _ptr(sink), _stream(stream)), "test_empty_chain")


def default_desc(mode: int = FULL, ratio: int = 1, **over) -> LayerDesc:
    d = LayerDesc()
    lib().csa2_layer_desc_default(ctypes.byref(d), mode, ratio)
    for k, v in over.items():
        setattr(d, k, v)
    return d


def schedule(decoder: bool = True) -> list[int]:
    buf = (ctypes.c_int32 * 20)()
    n = lib().csa2_schedule(1 if decoder else 0, ctypes.cast(buf, _P))
    return list(buf[:n])


class KVCache:
    """Paged FP4 main-KV cache + indexer K (+ pooled indexer K) in device memory.

    page_table: int32 [n_seqs, max_pages] (host or device tensor) mapping the
    entry pages of each sequence to physical pages (-1 = none).
    main_kv_on_host: keep codes and scales (the main KV) in pinned host memory
    that the device reads in place; the indexer K stays in device memory."""

    def __init__(self, n_phys_pages: int, page_size: int, page_table: torch.Tensor, device="cuda",
                 pooled: bool = True, main_kv_on_host: bool = False):
        n = n_phys_pages * page_size
        self.page_size, self.n_phys_pages = page_size, n_phys_pages
        if main_kv_on_host:
            self.codes = torch.zeros((n, 128), dtype=torch.uint8, pin_memory=True)
            self.scales = torch.zeros((n, 16), dtype=torch.uint8, pin_memory=True)
            for t in (self.codes, self.scales):
                if device_accessible(t) != 1:
                    raise RuntimeError("pinned host memory is not mapped into the device address space")
        else:
            self.codes = torch.zeros((n, 128), dtype=torch.uint8, device=device)
            self.scales = torch.zeros((n, 16), dtype=torch.uint8, device=device)
        self.idx_k = torch.zeros((n, 64), dtype=torch.int16, device=device)
        self.pooled = torch.zeros((n // 8, 64), dtype=torch.int16, device=device) if pooled else None
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self._s = _Cache(self.codes.data_ptr(), self.scales.data_ptr(), self.idx_k.data_ptr(),
                         self.pooled.data_ptr() if pooled else None, self.page_table.data_ptr(), page_size,
                         self.page_table.shape[1], n_phys_pages)

    def struct(self) -> _Cache:
        return self._s

    def shard(self, page_lo: int, n_pages: int) -> "KVCache":
        """A view of pages [page_lo, page_lo + n_pages) of every sequence: the
        same cache arrays with that slice of the page table, so entry e of the
        view is entry page_lo * page_size + e of the sequence (a context-parallel
        shard)."""
        v = KVCache.__new__(KVCache)
        v.page_size, v.n_phys_pages = self.page_size, self.n_phys_pages
        v.codes, v.scales, v.idx_k, v.pooled = self.codes, self.scales, self.idx_k, self.pooled
        v.page_table = self.page_table[:, page_lo:page_lo + n_pages].contiguous()
        v._s = _Cache(self._s.codes, self._s.scales, self._s.idx_k, self._s.idx_k_pooled, v.page_table.data_ptr(),
                      self.page_size, v.page_table.shape[1], self.n_phys_pages)
        return v


def kv_quant_append(cache: KVCache, kv_src: torch.Tensor, idx_k_src, slot_mapping: torch.Tensor, ratio: int = 1,
                    err=None, stream=None) -> None:
    dt = BF16 if kv_src.dtype == torch.bfloat16 else F32
    n = slot_mapping.numel()
    _check(lib().csa2_kv_quant_append(ctypes.byref(cache.struct()), _ptr(kv_src), dt, _ptr(idx_k_src), n, ratio,
                                      _ptr(slot_mapping), _ptr(err), _stream(stream)), "kv_quant_append")


def workspace_bytes(desc: LayerDesc, level: int, n: int, max_len: int, prefill: bool = False) -> int:
    return int(lib().csa2_indexer_workspace_bytes(ctypes.byref(desc), level, n, max_len, 1 if prefill else 0))


def indexer_topk(desc: LayerDesc, cache: KVCache, level: int, q_idx, w, seq_lens, out, n: int, max_len: int,
                 workspace: torch.Tensor, q_pos=None, cand_blocks=None, err=None, stream=None) -> None:
    _check(lib().csa2_indexer_topk(ctypes.byref(desc), ctypes.byref(cache.struct()), level, _ptr(q_idx), _ptr(w),
                                   _ptr(seq_lens), _ptr(q_pos), _ptr(cand_blocks), _ptr(out), None, n, max_len,
                                   _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(err),
                                   _stream(stream)), "indexer_topk")


def sparse_attn_decode(desc: LayerDesc, cache: KVCache, q, topk_idx, swa_kv, seq_lens, out, lse, B: int,
                       swa_lens=None, err=None, stream=None) -> None:
    _check(lib().csa2_sparse_attn_decode(ctypes.byref(desc), ctypes.byref(cache.struct()), _ptr(q), _ptr(topk_idx),
                                         _ptr(swa_kv), _ptr(seq_lens), _ptr(swa_lens), _ptr(out), _ptr(lse), B,
                                         _ptr(err), _stream(stream)), "sparse_attn_decode")


def sparse_attn_prefill(desc: LayerDesc, cache: KVCache, q, topk_idx, q_pos, swa_kv, swa_start: int, seq_len: int,
                        out, lse, T: int, err=None, stream=None) -> None:
    _check(lib().csa2_sparse_attn_prefill(ctypes.byref(desc), ctypes.byref(cache.struct()), _ptr(q), _ptr(topk_idx),
                                          _ptr(q_pos), _ptr(swa_kv), swa_start, seq_len, _ptr(out), _ptr(lse), T,
                                          _ptr(err), _stream(stream)), "sparse_attn_prefill")


def decode_layers(descs: list[LayerDesc], cache: KVCache, q_idx: list, w: list, q: list, swa_kv: list, seq_lens,
                  cand_blocks, idx_sets, out: list, lse: list, B: int, max_len: int, workspace: torch.Tensor,
                  swa_lens=None, err=None, stream=None) -> None:
    n = len(descs)
    D = (LayerDesc * n)(*descs)
    arr = lambda xs: (ctypes.c_void_p * n)(*[_ptr(x) for x in xs])  # noqa: E731
    keep = [arr(q_idx), arr(w), arr(q), arr(swa_kv), arr(out), arr(lse)]
    _check(lib().csa2_decode_layers(n, D, ctypes.byref(cache.struct()), ctypes.cast(keep[0], _P),
                                    ctypes.cast(keep[1], _P), ctypes.cast(keep[2], _P), ctypes.cast(keep[3], _P),
                                    _ptr(seq_lens), _ptr(swa_lens), _ptr(cand_blocks), _ptr(idx_sets),
                                    ctypes.cast(keep[4], _P), ctypes.cast(keep[5], _P), B, max_len,
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(err),
                                    _stream(stream)), "decode_layers")


def indexer_topk_noalloc(desc: LayerDesc, cache: KVCache, level: int, q_idx, w, seq_lens, out, n: int, max_len: int,
                         cand_blocks=None, err=None, stream=None) -> None:
    """Decode indexer without a caller workspace (static 16 MiB library scratch);
    for callers that cannot allocate device memory at this point."""
    _check(lib().csa2_indexer_topk_noalloc(ctypes.byref(desc), ctypes.byref(cache.struct()), level, _ptr(q_idx),
                                           _ptr(w), _ptr(seq_lens), _ptr(cand_blocks), _ptr(out), n, max_len,
                                           _ptr(err), _stream(stream)), "indexer_topk_noalloc")
