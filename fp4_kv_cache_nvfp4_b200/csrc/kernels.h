// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

// log2 of a power-of-two page size (validated by the ABI layer)
inline int page_shift_of(const csa2_kv_cache& c) {
    int s = 0;
    while ((1 << s) < c.page_size) ++s;
    return s;
}

// Launch configuration with programmatic dependent launch enabled, and an
// optional thread-block cluster.
struct LaunchCfg {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    LaunchCfg(dim3 grid, dim3 block, size_t smem, cudaStream_t stream, unsigned cluster_x = 0) {
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        int n = 0;
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
        if (cluster_x > 1) {
            attr[n].id = cudaLaunchAttributeClusterDimension;
            attr[n].val.clusterDim.x = cluster_x;
            attr[n].val.clusterDim.y = 1;
            attr[n].val.clusterDim.z = 1;
            ++n;
        }
        cfg.attrs = attr;
        cfg.numAttrs = n;
    }
};

// Workspace layout of the decode indexer (byte offsets; all 256-aligned).
struct DecodeWs {
    size_t blk_scores, blk_hist, blk_thr, blk_ctr, blk_bitmap, blk_bnd, blk_bnd_cnt, blk_tie;
    size_t blk_abv, blk_abv_cnt;  // flat: rows above the K-th's bin, and their count
    // staged rows of one index set when the main KV is in host memory
    size_t stage_codes, stage_scales, stage_idx, stage_pt;
    int stage_rows;               // rows per sequence in the staged cache (a power of two >= topk)
    size_t tok_keys, tok_ctr, tok_hist;
    size_t total;
    int64_t nblk_pad;  // per-sequence stride of block arrays
};
// flat: rows are entries (the indexer without a block level), not blocks of 8
DecodeWs decode_ws_layout(int n, int64_t max_len, bool flat = false);

struct PrefillWs {
    size_t keys;   // [T][stride]: 16-bit approximate keys, later (aliased) 32-bit exact keys of the fallback
    size_t flags;  // [T] int32: 1 = the query takes the exact fallback
    size_t kmax;   // [tiles] float: max |indexer K| seen by each tensor-core scoring CTA
    size_t total;
    int64_t stride;
    int kmax_parts;
};
PrefillWs prefill_ws_layout(int T, int64_t n_entries);

cudaError_t launch_quant_append(const csa2_kv_cache& cache, const void* src, bool bf16, const uint16_t* idx_src,
                                int64_t n, int ratio, const int64_t* slot_mapping, int32_t* err,
                                cudaStream_t stream);

cudaError_t launch_block_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                              const int32_t* seq_lens, int keep, int32_t* out, int n, int64_t max_len,
                              char* ws, int32_t* err, cudaStream_t stream, bool flat = false);

cudaError_t launch_token_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                              const int32_t* seq_lens, const int32_t* cand_blocks, int keep, int topk, int32_t* out,
                              int n, int64_t max_len, char* ws, int32_t* err, cudaStream_t stream,
                              int pre = 0);

cudaError_t launch_prefill_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                                const int32_t* seq_lens, const int32_t* q_pos, int ratio, int topk, int32_t* out,
                                int T, int64_t max_len, char* ws, int32_t* err, cudaStream_t stream);

// Attention rows: decode (row = sequence) or prefill (row = query of sequence 0).
struct AttnArgs {
    csa2_kv_cache cache;
    const uint16_t* q;        // [rows][16][128] bf16
    const int32_t* idx;       // [rows][topk]
    const uint16_t* swa;      // decode: [rows][window][256]; prefill: token rows from swa_start
    const int32_t* seq_lens;  // decode: [rows]; prefill: nullptr
    const int32_t* swa_lens;  // decode: nullable
    const int32_t* q_pos;     // prefill: [rows]; decode: nullptr
    float* out;
    float* lse;
    int32_t* err;
    int rows, topk, window, swa_start, seq_len_prefill;
    int page_shift;
    // What the kernel may read before the preceding kernel in the stream has
    // completed (programmatic dependent launch).  Nothing is written before the
    // wait, and q and the newest SWA row (which a model computes from the
    // previous layer's output) are always read after it.  kPreIdx: the index
    // set and the cache; kPreHist: the lengths and the SWA rows other than the
    // newest.
    int pre;
};
constexpr int kPreIdx = 1;
constexpr int kPreHist = 2;
cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t stream);
// Prefill attention on tcgen05 (prefill_attn.cu): a persistent kernel over at most n_ctas CTAs.
cudaError_t launch_prefill_attn_tc(const AttnArgs& a, int n_ctas, cudaStream_t stream);

// Copies the FP4 rows of a decode index set into the staged cache (stage.cu).
struct StageArgs {
    csa2_kv_cache cache;   // the main KV (host memory)
    const int32_t* idx;    // [B][topk]
    const int32_t* seq_lens;
    uint8_t* stage_codes;  // [B * stage_rows][128]
    uint8_t* stage_scales; // [B * stage_rows][16]
    int32_t* stage_idx;    // [B][topk]: i for a staged row, -1 otherwise
    int32_t* stage_pt;     // [B]: page b of the staged cache is sequence b's
    int32_t* err;
    int topk, stage_rows, page_shift;
};
cudaError_t launch_stage_rows(const StageArgs& a, int B, cudaStream_t stream);

}  // namespace csa2
