// C ABI of the CSA2 library: host-side validation, then kernel launches.
// Every check below runs before the first CUDA call, so a rejected call has no
// side effect on the device.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

using namespace csa2;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

csa2_status check_desc(const csa2_layer_desc* d) {
    if (!d) return CSA2_ERR_INVALID_ARG;
    if (d->n_heads != 16 || d->head_dim != 128 || d->idx_heads != 4 || d->idx_dim != 64 || d->block != 8)
        return CSA2_ERR_UNSUPPORTED;
    if (d->ratio != 1 && d->ratio != 2) return CSA2_ERR_INVALID_ARG;
    if (d->topk < 1 || d->topk > kMaxTopk) return CSA2_ERR_INVALID_ARG;
    if (d->keep_blocks < 0 || d->keep_blocks > kMaxKeep) return CSA2_ERR_INVALID_ARG;  // 0: flat indexer
    if (d->window < 1 || d->window > kMaxWindow) return CSA2_ERR_INVALID_ARG;
    if (d->mode < CSA2_MODE_FULL || d->mode > CSA2_MODE_REUSE) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

csa2_status check_cache(const csa2_kv_cache* c, bool need_idx, bool need_pooled) {
    if (!c || !c->codes || !c->scales || !c->page_table) return CSA2_ERR_INVALID_ARG;
    if (!aligned(c->codes, 16) || !aligned(c->scales, 16) || !aligned(c->page_table, 4)) return CSA2_ERR_INVALID_ARG;
    if (c->page_size < 8 || (c->page_size & (c->page_size - 1)) != 0 || c->page_size > (1 << 20) ||
        c->max_pages_per_seq < 1 || c->n_phys_pages < 1)
        return CSA2_ERR_INVALID_ARG;
    if ((int64_t)c->max_pages_per_seq * c->page_size > (int64_t(1) << 31)) return CSA2_ERR_INVALID_ARG;
    if (c->n_phys_pages > (int64_t(1) << 40) / c->page_size) return CSA2_ERR_INVALID_ARG;
    if (need_idx && (!c->idx_k || !aligned(c->idx_k, 16))) return CSA2_ERR_INVALID_ARG;
    if (need_pooled && (!c->idx_k_pooled || !aligned(c->idx_k_pooled, 16))) return CSA2_ERR_INVALID_ARG;
    if (c->idx_k_pooled && !aligned(c->idx_k_pooled, 16)) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

// Where p lives: 0 device (or managed) memory, 1 host memory mapped into the
// device address space at p, -1 host memory the device cannot read in place.
// The answers for the last two pointers asked are kept, so repeated calls (and
// calls under stream capture) do not query the driver again.
int memory_kind(const void* p) {
    static thread_local const void* last[2] = {nullptr, nullptr};
    static thread_local int last_kind[2] = {0, 0};
    static thread_local int next = 0;
    for (int i = 0; i < 2; ++i)
        if (p == last[i]) return last_kind[i];
    cudaPointerAttributes at{};
    int kind = 0;
    if (cudaPointerGetAttributes(&at, p) == cudaSuccess) {
        if (at.type == cudaMemoryTypeHost) kind = at.devicePointer == p ? 1 : -1;
        else if (at.type == cudaMemoryTypeUnregistered) kind = -1;
    } else {
        (void)cudaGetLastError();
    }
    last[next] = p;
    last_kind[next] = kind;
    next ^= 1;
    return kind;
}

csa2_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return CSA2_OK;
    (void)cudaGetLastError();
    return CSA2_ERR_CUDA;
}

}  // namespace

extern "C" {

void csa2_layer_desc_default(csa2_layer_desc* d, int32_t mode, int32_t ratio) {
    if (!d) return;
    d->mode = mode;
    d->ratio = ratio;
    d->topk = 512;
    d->block = 8;
    d->keep_blocks = 2048;
    d->window = 128;
    d->n_heads = 16;
    d->head_dim = 128;
    d->idx_heads = 4;
    d->idx_dim = 64;
}

int32_t csa2_schedule(int32_t decoder, int32_t* modes) {
    const int n = decoder ? 20 : 18, g = decoder ? 4 : 6;
    if (!modes) return n;
    for (int l = 0; l < n; ++l) {
        if (l % g) modes[l] = CSA2_MODE_REUSE;
        else modes[l] = (decoder && l > 0) ? CSA2_MODE_REINDEX : CSA2_MODE_FULL;
    }
    return n;
}

csa2_status csa2_kv_quant_append(const csa2_kv_cache* cache, const void* kv_src, int32_t src_dtype,
                                 const uint16_t* idx_k_src, int64_t n_entries, int32_t ratio,
                                 const int64_t* slot_mapping, int32_t* err_word, void* stream) {
    csa2_status s = check_cache(cache, idx_k_src != nullptr, false);
    if (s != CSA2_OK) return s;
    if (n_entries < 0 || (ratio != 1 && ratio != 2)) return CSA2_ERR_INVALID_ARG;
    if (src_dtype != CSA2_SRC_F32 && src_dtype != CSA2_SRC_BF16) return CSA2_ERR_INVALID_ARG;
    if (n_entries == 0) return CSA2_OK;
    if (!kv_src || !slot_mapping || !aligned(kv_src, 16) || !aligned(slot_mapping, 8)) return CSA2_ERR_INVALID_ARG;
    if (idx_k_src && !aligned(idx_k_src, 4)) return CSA2_ERR_INVALID_ARG;
    if (err_word && !aligned(err_word, 4)) return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_quant_append(*cache, kv_src, src_dtype == CSA2_SRC_BF16, idx_k_src, n_entries, ratio,
                                         slot_mapping, err_word, (cudaStream_t)stream));
}

size_t csa2_indexer_workspace_bytes(const csa2_layer_desc* desc, int32_t level, int32_t n, int64_t max_len,
                                    int32_t prefill) {
    if (!desc || n < 1 || max_len < 1) return 0;
    if (prefill) return prefill_ws_layout(n, max_len).total;
    (void)level;
    return decode_ws_layout(n, max_len, desc->keep_blocks == 0).total;
}

}  // extern "C"

// pre: the token level may read cand_blocks, the lengths and the cache before
// the preceding kernel completes (a Reindex layer inside the decode driver)
static csa2_status indexer_topk(const csa2_layer_desc* desc, const csa2_kv_cache* cache, int32_t level,
                                const uint16_t* q_idx, const float* w, const int32_t* seq_lens, const int32_t* q_pos,
                                const int32_t* cand_blocks, int32_t* idx_out, float* score_out, int32_t n,
                                int64_t max_len, void* workspace, size_t ws_bytes, int32_t* err_word, void* stream,
                                int pre) {
    csa2_status s = check_desc(desc);
    if (s != CSA2_OK) return s;
    if (desc->mode == CSA2_MODE_REUSE) return CSA2_ERR_INVALID_ARG;
    if (level != CSA2_LEVEL_BLOCK && level != CSA2_LEVEL_TOKEN) return CSA2_ERR_INVALID_ARG;
    const bool prefill = q_pos != nullptr;
    const bool flat = desc->keep_blocks == 0;  // no block level: Top-K over every entry
    if (prefill && level != CSA2_LEVEL_TOKEN) return CSA2_ERR_INVALID_ARG;
    if (flat && (level != CSA2_LEVEL_TOKEN || cand_blocks)) return CSA2_ERR_INVALID_ARG;
    s = check_cache(cache, true, level == CSA2_LEVEL_BLOCK);
    if (s != CSA2_OK) return s;
    if (score_out) return CSA2_ERR_UNSUPPORTED;
    if (n < 1 || max_len < 1 || !q_idx || !w || !seq_lens || !idx_out) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_idx, 4) || !aligned(w, 16) || !aligned(seq_lens, 4) || !aligned(idx_out, 4))
        return CSA2_ERR_INVALID_ARG;
    if (cand_blocks && (!aligned(cand_blocks, 4) || prefill || level != CSA2_LEVEL_TOKEN)) return CSA2_ERR_INVALID_ARG;
    if (level == CSA2_LEVEL_BLOCK && (max_len > kMaxBlockLevelLen || n > 1024)) return CSA2_ERR_UNSUPPORTED;
    if (level == CSA2_LEVEL_BLOCK && cache->n_phys_pages * cache->page_size / 8 > 0x7fffffff) return CSA2_ERR_UNSUPPORTED;
    const bool flat_rows = flat && !prefill && max_len > kMaxCand;  // scored by the block-level kernels, row = entry
    if (flat_rows && (max_len > kMaxBlockLevelLen || n > 1024)) return CSA2_ERR_UNSUPPORTED;
    if (flat_rows && cache->n_phys_pages * cache->page_size > 0x7fffffff) return CSA2_ERR_UNSUPPORTED;
    if (prefill && max_len > kMaxCand) return CSA2_ERR_UNSUPPORTED;
    if (prefill && !aligned(q_idx, 16)) return CSA2_ERR_INVALID_ARG;  // read in 16-byte rows by the tensor-core tiles
    if (max_len > (int64_t)cache->max_pages_per_seq * cache->page_size) return CSA2_ERR_INVALID_ARG;
    const size_t need = csa2_indexer_workspace_bytes(desc, level, n, max_len, prefill ? 1 : 0);
    if (!workspace || !aligned(workspace, 256) || ws_bytes < need) return CSA2_ERR_WORKSPACE;
    if (err_word && !aligned(err_word, 4)) return CSA2_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    if (prefill)
        return from_cuda(launch_prefill_topk(*cache, q_idx, w, seq_lens, q_pos, desc->ratio, desc->topk, idx_out, n,
                                             max_len, ws, err_word, st));
    if (level == CSA2_LEVEL_BLOCK)
        return from_cuda(launch_block_topk(*cache, q_idx, w, seq_lens, desc->keep_blocks, idx_out, n, max_len, ws,
                                           err_word, st));
    if (flat_rows)
        return from_cuda(launch_block_topk(*cache, q_idx, w, seq_lens, desc->topk, idx_out, n, max_len, ws, err_word,
                                           st, true));
    // a flat selection over at most 16,384 entries runs as one candidate set
    return from_cuda(launch_token_topk(*cache, q_idx, w, seq_lens, cand_blocks, flat ? kMaxKeep : desc->keep_blocks,
                                       desc->topk, idx_out, n, max_len, ws, err_word, st, pre));
}

extern "C" {

csa2_status csa2_indexer_topk(const csa2_layer_desc* desc, const csa2_kv_cache* cache, int32_t level,
                              const uint16_t* q_idx, const float* w, const int32_t* seq_lens, const int32_t* q_pos,
                              const int32_t* cand_blocks, int32_t* idx_out, float* score_out, int32_t n,
                              int64_t max_len, void* workspace, size_t ws_bytes, int32_t* err_word, void* stream) {
    return indexer_topk(desc, cache, level, q_idx, w, seq_lens, q_pos, cand_blocks, idx_out, score_out, n, max_len,
                        workspace, ws_bytes, err_word, stream, 0);
}

}  // extern "C"

// pre: what the kernel may read before the preceding kernel completes (kPre*)
static csa2_status attn_decode(const csa2_layer_desc* desc, const csa2_kv_cache* cache, const uint16_t* q,
                               const int32_t* topk_idx, const uint16_t* swa_kv, const int32_t* seq_lens,
                               const int32_t* swa_lens, float* out, float* lse, int32_t B, int32_t* err_word,
                               void* stream, int pre) {
    csa2_status s = check_desc(desc);
    if (s != CSA2_OK) return s;
    s = check_cache(cache, false, false);
    if (s != CSA2_OK) return s;
    if (B < 0) return CSA2_ERR_INVALID_ARG;
    if (B == 0) return CSA2_OK;
    if (!q || !topk_idx || !swa_kv || !seq_lens || !out || !lse) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q, 4) || !aligned(topk_idx, 4) || !aligned(swa_kv, 16) || !aligned(seq_lens, 4) ||
        !aligned(out, 4) || !aligned(lse, 4) || (swa_lens && !aligned(swa_lens, 4)))
        return CSA2_ERR_INVALID_ARG;
    if (err_word && !aligned(err_word, 4)) return CSA2_ERR_INVALID_ARG;
    AttnArgs a{};
    a.cache = *cache;
    a.q = q;
    a.idx = topk_idx;
    a.swa = swa_kv;
    a.seq_lens = seq_lens;
    a.swa_lens = swa_lens;
    a.q_pos = nullptr;
    a.out = out;
    a.lse = lse;
    a.err = err_word;
    a.rows = B;
    a.topk = desc->topk;
    a.window = desc->window;
    a.page_shift = page_shift_of(*cache);
    a.pre = pre;
    return from_cuda(launch_sparse_attn(a, (cudaStream_t)stream));
}

extern "C" {

csa2_status csa2_sparse_attn_decode(const csa2_layer_desc* desc, const csa2_kv_cache* cache, const uint16_t* q,
                                    const int32_t* topk_idx, const uint16_t* swa_kv, const int32_t* seq_lens,
                                    const int32_t* swa_lens, float* out, float* lse, int32_t B, int32_t* err_word,
                                    void* stream) {
    return attn_decode(desc, cache, q, topk_idx, swa_kv, seq_lens, swa_lens, out, lse, B, err_word, stream, 0);
}

csa2_status csa2_sparse_attn_prefill(const csa2_layer_desc* desc, const csa2_kv_cache* cache, const uint16_t* q,
                                     const int32_t* topk_idx, const int32_t* q_pos, const uint16_t* swa_kv,
                                     int32_t swa_start, int32_t seq_len, float* out, float* lse, int32_t T,
                                     int32_t* err_word, void* stream) {
    csa2_status s = check_desc(desc);
    if (s != CSA2_OK) return s;
    s = check_cache(cache, false, false);
    if (s != CSA2_OK) return s;
    if (T < 0 || swa_start < 0 || seq_len < 1) return CSA2_ERR_INVALID_ARG;
    if (T == 0) return CSA2_OK;
    if (!q || !topk_idx || !q_pos || !swa_kv || !out || !lse) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(topk_idx, 4) || !aligned(q_pos, 4) || !aligned(swa_kv, 16) || !aligned(out, 16) ||
        !aligned(lse, 4))
        return CSA2_ERR_INVALID_ARG;
    if (err_word && !aligned(err_word, 4)) return CSA2_ERR_INVALID_ARG;
    if ((cache->n_phys_pages << page_shift_of(*cache)) > INT32_MAX) return CSA2_ERR_UNSUPPORTED;  // int32 slots
    AttnArgs a{};
    a.cache = *cache;
    a.q = q;
    a.idx = topk_idx;
    a.swa = swa_kv;
    a.seq_lens = nullptr;
    a.swa_lens = nullptr;
    a.q_pos = q_pos;
    a.out = out;
    a.lse = lse;
    a.err = err_word;
    a.rows = T;
    a.topk = desc->topk;
    a.window = desc->window;
    a.swa_start = swa_start;
    a.seq_len_prefill = seq_len;
    a.page_shift = page_shift_of(*cache);
    a.pre = 0;
    return from_cuda(launch_sparse_attn(a, (cudaStream_t)stream));
}

csa2_status csa2_decode_layers(int32_t n_layers, const csa2_layer_desc* descs, const csa2_kv_cache* cache,
                               const uint16_t* const* q_idx, const float* const* w, const uint16_t* const* q,
                               const uint16_t* const* swa_kv, const int32_t* seq_lens, const int32_t* swa_lens,
                               int32_t* cand_blocks, int32_t* idx_sets, float* const* out, float* const* lse,
                               int32_t B, int64_t max_len, void* workspace, size_t ws_bytes, int32_t* err_word,
                               void* stream) {
    if (n_layers < 1 || !descs || !cache || !q_idx || !w || !q || !swa_kv || !out || !lse || !idx_sets)
        return CSA2_ERR_INVALID_ARG;
    if (descs[0].mode != CSA2_MODE_FULL) return CSA2_ERR_INVALID_ARG;
    const bool flat = descs[0].keep_blocks == 0;  // every indexer layer selects over all entries
    if (!flat && !cand_blocks) return CSA2_ERR_INVALID_ARG;
    // validate every layer before launching anything
    for (int l = 0; l < n_layers; ++l) {
        csa2_status s = check_desc(&descs[l]);
        if (s != CSA2_OK) return s;
        if (descs[l].topk != descs[0].topk || descs[l].keep_blocks != descs[0].keep_blocks)
            return CSA2_ERR_INVALID_ARG;
        if (!q[l] || !swa_kv[l] || !out[l] || !lse[l]) return CSA2_ERR_INVALID_ARG;
        if (descs[l].mode != CSA2_MODE_REUSE && (!q_idx[l] || !w[l])) return CSA2_ERR_INVALID_ARG;
    }
    const size_t need =
        csa2_indexer_workspace_bytes(&descs[0], flat ? CSA2_LEVEL_TOKEN : CSA2_LEVEL_BLOCK, B, max_len, 0);
    if (!workspace || ws_bytes < need) return CSA2_ERR_WORKSPACE;
    const int topk = descs[0].topk;
    const int32_t* cur = nullptr;
    // A main KV in host memory: each new index set's rows are copied once into
    // the workspace's staged cache, and every attention layer reads them there.
    const int kind = memory_kind(cache->codes);
    if (kind < 0) return CSA2_ERR_INVALID_ARG;  // host memory the kernels cannot read in place
    const bool host_kv = kind == 1;
    const DecodeWs wl = decode_ws_layout(B, max_len, flat);
    char* wsb = static_cast<char*>(workspace);
    StageArgs sa{};
    csa2_kv_cache staged{};
    if (host_kv) {
        sa.cache = *cache;
        sa.seq_lens = seq_lens;
        sa.stage_codes = reinterpret_cast<uint8_t*>(wsb + wl.stage_codes);
        sa.stage_scales = reinterpret_cast<uint8_t*>(wsb + wl.stage_scales);
        sa.stage_idx = reinterpret_cast<int32_t*>(wsb + wl.stage_idx);
        sa.stage_pt = reinterpret_cast<int32_t*>(wsb + wl.stage_pt);
        sa.err = err_word;
        sa.topk = topk;
        sa.stage_rows = wl.stage_rows;
        sa.page_shift = page_shift_of(*cache);
        staged.codes = sa.stage_codes;
        staged.scales = sa.stage_scales;
        staged.idx_k = cache->idx_k;
        staged.idx_k_pooled = nullptr;
        staged.page_table = sa.stage_pt;
        staged.page_size = wl.stage_rows;
        staged.max_pages_per_seq = 1;
        staged.n_phys_pages = B;
    }
    for (int l = 0; l < n_layers; ++l) {
        const csa2_layer_desc& d = descs[l];
        int32_t* set = idx_sets + (int64_t)l * B * topk;
        csa2_status s = CSA2_OK;
        if (flat && d.mode != CSA2_MODE_REUSE) {
            // no candidate set: Full and Reindex layers both select over every entry
            s = csa2_indexer_topk(&d, cache, CSA2_LEVEL_TOKEN, q_idx[l], w[l], seq_lens, nullptr, nullptr, set,
                                  nullptr, B, max_len, workspace, ws_bytes, err_word, stream);
            cur = set;
        } else if (d.mode == CSA2_MODE_FULL) {
            s = csa2_indexer_topk(&d, cache, CSA2_LEVEL_BLOCK, q_idx[l], w[l], seq_lens, nullptr, nullptr,
                                  cand_blocks, nullptr, B, max_len, workspace, ws_bytes, err_word, stream);
            if (s == CSA2_OK)
                s = csa2_indexer_topk(&d, cache, CSA2_LEVEL_TOKEN, q_idx[l], w[l], seq_lens, nullptr, cand_blocks,
                                      set, nullptr, B, max_len, workspace, ws_bytes, err_word, stream);
            cur = set;
        } else if (d.mode == CSA2_MODE_REINDEX) {
            // the Full layer's candidates were written launches back
            s = indexer_topk(&d, cache, CSA2_LEVEL_TOKEN, q_idx[l], w[l], seq_lens, nullptr, cand_blocks, set, nullptr,
                             B, max_len, workspace, ws_bytes, err_word, stream, 1);
            cur = set;
        }
        if (s != CSA2_OK) return s;
        if (host_kv && d.mode != CSA2_MODE_REUSE) {  // stage the new set's rows
            sa.idx = cur;
            s = from_cuda(launch_stage_rows(sa, B, (cudaStream_t)stream));
            if (s != CSA2_OK) return s;
        }
        // Not the call's first kernel: the cache, the lengths and the SWA
        // history were complete before that kernel passed its wait, and a Reuse
        // layer's index set (and its staged rows) were written two or more
        // launches back.
        s = attn_decode(&d, host_kv ? &staged : cache, q[l], host_kv ? sa.stage_idx : cur, swa_kv[l], seq_lens,
                        swa_lens, out[l], lse[l], B, err_word, stream,
                        kPreHist | (d.mode == CSA2_MODE_REUSE ? kPreIdx : 0));
        if (s != CSA2_OK) return s;
    }
    return CSA2_OK;
}

const char* csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_INVALID_ARG: return "invalid argument";
        case CSA2_ERR_UNSUPPORTED: return "unsupported dimension or size";
        case CSA2_ERR_CUDA: return "CUDA error";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

int32_t csa2_abi_version(void) { return CSA2_ABI_VERSION; }

int32_t csa2_device_accessible(const void* p) {
    if (!p) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    switch (at.type) {
        case cudaMemoryTypeDevice: return at.device == dev ? 1 : 0;
        case cudaMemoryTypeManaged: return 1;
        case cudaMemoryTypeHost: return at.devicePointer == p ? 1 : 0;
        default: return 0;
    }
}

}  // extern "C"
