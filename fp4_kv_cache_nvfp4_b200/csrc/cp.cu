// Context-parallel decode of one long sequence: the kernels of the exchange
// steps.  The sequence's entries are split into G contiguous shards (one per
// GPU); every shard runs the ordinary indexer and attention kernels on its own
// entries.  What crosses between shards is small:
//   - per indexer level, each shard's local Top-K as (score, global id) pairs
//     (csa2_indexer_score_ids rescores its selected ids with the same
//     sequential FMA chains the selection used, so the scores are bit-equal);
//     every shard merges the G lists into the global Top-K
//     (csa2_topk_merge), exactly the set a single GPU selects, because every
//     member of the global Top-K is in its own shard's local Top-K;
//   - per attention layer, each shard's partial (out, lse) over its share of
//     the selected entries, merged by log-sum-exp (csa2_attn_lse_merge).
// Pages: native context window of one million tokens (conexaotc.com.br,
// opening paragraphs); Top-512 and the hierarchical indexer of 2048 blocks of
// 8 (CSA2 paragraph).
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace csa2 {

struct ScoreIdsArgs {
    csa2_kv_cache cache;
    const uint16_t* q_idx;
    const float* w;
    const int32_t* seq_lens;
    const int32_t* ids;  // [n][k]
    float* scores;       // [n][k]
    int32_t* ids_out;    // [n][k] or null
    int32_t* err;
    int64_t max_len;
    int k, level, page_shift, id_offset;
};

constexpr int SI_THREADS = 128;

// One thread per id: its row (pooled block row or entry row) in 8 16-byte
// loads, then the exact score chain.
__global__ void __launch_bounds__(SI_THREADS) score_ids_kernel(ScoreIdsArgs a) {
    __shared__ float4 qd[kID];
    __shared__ float4 s_w;
    const int b = blockIdx.y, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    load_q_idx(a.q_idx + (int64_t)b * kIH * kID, qd);
    if (tid == 0) s_w = *reinterpret_cast<const float4*>(a.w + (int64_t)b * kIH);
    __syncthreads();
    const int i = blockIdx.x * SI_THREADS + tid;
    if (i >= a.k) return;
    const int32_t L = seq_len_checked(a.seq_lens, b, a.max_len, a.err);
    const int32_t id = a.ids[(int64_t)b * a.k + i];
    float s = -INFINITY;
    int32_t gid = -1;
    const int32_t lim = a.level == CSA2_LEVEL_BLOCK ? (L + kBlk - 1) / kBlk : L;
    if (id >= 0 && id < lim) {
        const int32_t pos = a.level == CSA2_LEVEL_BLOCK ? id * kBlk : id;
        const int64_t slot = entry_slot(a.cache, a.page_shift, b, pos, a.err);
        if (slot >= 0) {
            const uint4* row = a.level == CSA2_LEVEL_BLOCK
                                   ? reinterpret_cast<const uint4*>(a.cache.idx_k_pooled + (slot >> 3) * kID)
                                   : reinterpret_cast<const uint4*>(a.cache.idx_k + slot * kID);
            uint32_t kr[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = __ldg(row + c);
                kr[4 * c] = v.x;
                kr[4 * c + 1] = v.y;
                kr[4 * c + 2] = v.z;
                kr[4 * c + 3] = v.w;
            }
            s = idx_score1(kr, qd, s_w);
            gid = id + a.id_offset;
        }
    } else if (id >= lim) {
        dev_error(a.err, CSA2_DEV_INDEX);
    }
    a.scores[(int64_t)b * a.k + i] = s;
    if (a.ids_out) a.ids_out[(int64_t)b * a.k + i] = gid;
}

struct MergeArgs {
    const float* scores;  // [n_parts][n][part_len]
    const int32_t* ids;   // [n_parts][n][part_len]; -1 = no pair
    int32_t* out;         // [n][k]
    int32_t* out_local;   // [n][k] or null
    int n, n_parts, part_len, k, lo, hi;
};

constexpr int MG_THREADS = 512;
constexpr int MG_MAX_PAIRS = 16384;
constexpr size_t MG_OFF_HIST = (size_t)MG_MAX_PAIRS * 4;
constexpr size_t MG_OFF_L0 = MG_OFF_HIST + kHistBins * 4;
constexpr size_t MG_OFF_L1 = MG_OFF_L0 + (size_t)MG_MAX_PAIRS * 2;
constexpr size_t MG_OFF_TMP = MG_OFF_L1 + (size_t)MG_MAX_PAIRS * 2;
constexpr size_t MG_SMEM = MG_OFF_TMP + 64 * 4;

// One CTA per row: keys of the valid pairs in shared memory (pair i of row b
// is element (i / part_len, b, i % part_len) of the gathered [parts][n][len]
// arrays), the radix select of the Top-k by (score desc, id asc), emission in
// pair order (the ids are ascending in pair order), then this shard's run of
// the result.
__global__ void __launch_bounds__(MG_THREADS) topk_merge_kernel(MergeArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + MG_OFF_HIST);
    uint16_t* l0 = reinterpret_cast<uint16_t*>(smem + MG_OFF_L0);
    uint16_t* l1 = reinterpret_cast<uint16_t*>(smem + MG_OFF_L1);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(smem + MG_OFF_TMP);
    const int b = blockIdx.x, tid = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    const int n_pairs = a.n_parts * a.part_len;
    auto at = [&](int i) { return ((int64_t)(i / a.part_len) * a.n + b) * a.part_len + i % a.part_len; };
    for (int i = tid; i < kHistBins; i += MG_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n_pairs; i += MG_THREADS) {
        const int64_t e = at(i);
        const uint32_t key = a.ids[e] >= 0 ? score_key(a.scores[e]) : 0u;
        keys[i] = key;
        hist_add(hist, key >> 20, key != 0u);
    }
    __syncthreads();
    uint32_t nv = 0;
    for (int i = tid; i < kHistBins; i += MG_THREADS) nv += hist[i];
    uint32_t n_valid;
    block_excl_scan(nv, tmp, &n_valid);
    const uint32_t kk = min((uint32_t)a.k, n_valid);
    int32_t* out = a.out + (int64_t)b * a.k;
    uint32_t T = 0xffffffffu, need = 0;
    if (kk > 0) {
        int b1;
        uint32_t above;
        find_kth_bin(hist, kHistBins, kk, tmp, &b1, &above);
        refine_threshold(keys, n_pairs, (uint32_t)b1, kk - above, hist, l0, l1, tmp, &T, &need);
    }
    // T = 0xffffffff selects nothing; key 0 (no pair) is never above T
    emit_sorted(keys, n_pairs, T, need, kk, a.k, out, tmp, [&](int i) { return a.ids[at(i)]; });
    if (!a.out_local) return;
    __syncthreads();  // the global result is written
    // the ascending result's members in [lo, hi) form one run: find its ends
    __shared__ int s_run[2];
    if (tid == 0) {
        s_run[0] = (int)kk;
        s_run[1] = (int)kk;
    }
    __syncthreads();
    for (int i = tid; i < (int)kk; i += MG_THREADS) {
        const int32_t v = out[i];
        const int32_t prev = i > 0 ? out[i - 1] : INT32_MIN;
        if (v >= a.lo && prev < a.lo) s_run[0] = i;
        if (v >= a.hi && prev < a.hi) s_run[1] = i;
    }
    __syncthreads();
    int32_t* loc = a.out_local + (int64_t)b * a.k;
    const int r0 = s_run[0], n_loc = max(0, s_run[1] - r0);
    for (int i = tid; i < a.k; i += MG_THREADS) loc[i] = i < n_loc ? out[r0 + i] - a.lo : -1;
}

// out = sum_g exp(lse_g - M) out_g / sum_g exp(lse_g - M), lse = M + log(sum):
// one warp per (row, head), 4 dims per lane.
__global__ void __launch_bounds__(32) lse_merge_kernel(int n_parts, const float* __restrict__ outs,
                                                       const float* __restrict__ lses, float* out, float* lse,
                                                       int rows) {
    const int r = blockIdx.x / kH, h = blockIdx.x % kH, lane = threadIdx.x;
    pdl_wait();
    pdl_trigger();
    const int64_t stride_o = (int64_t)rows * kH * kD, stride_l = (int64_t)rows * kH;
    float M = -INFINITY;
    for (int g = 0; g < n_parts; ++g) M = fmaxf(M, lses[g * stride_l + (int64_t)r * kH + h]);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    for (int g = 0; g < n_parts; ++g) {
        const float l = lses[g * stride_l + (int64_t)r * kH + h];
        const float f = l == -INFINITY ? 0.f : expf(l - M);
        const float4 v =
            *reinterpret_cast<const float4*>(outs + g * stride_o + ((int64_t)r * kH + h) * kD + 4 * lane);
        num.x += f * v.x;
        num.y += f * v.y;
        num.z += f * v.z;
        num.w += f * v.w;
        den += f;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    *reinterpret_cast<float4*>(out + ((int64_t)r * kH + h) * kD + 4 * lane) =
        make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
    if (lane == 0) lse[(int64_t)r * kH + h] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace csa2

using namespace csa2;

namespace {
bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
csa2_status status_of(cudaError_t e) {
    if (e == cudaSuccess) return CSA2_OK;
    (void)cudaGetLastError();
    return CSA2_ERR_CUDA;
}
}  // namespace

extern "C" {

CSA2_API csa2_status csa2_indexer_score_ids(const csa2_layer_desc* desc, const csa2_kv_cache* cache, int32_t level,
                                            const uint16_t* q_idx, const float* w, const int32_t* seq_lens,
                                            const int32_t* ids, int32_t k, int32_t id_offset, float* scores,
                                            int32_t* ids_out, int32_t n, int64_t max_len, int32_t* err_word,
                                            void* stream) {
    if (!desc || !cache || !q_idx || !w || !seq_lens || !ids || !scores || n < 1 || k < 1 || max_len < 1)
        return CSA2_ERR_INVALID_ARG;
    if (desc->n_heads != 16 || desc->head_dim != 128 || desc->idx_heads != 4 || desc->idx_dim != 64 ||
        desc->block != 8)
        return CSA2_ERR_UNSUPPORTED;
    if (level != CSA2_LEVEL_BLOCK && level != CSA2_LEVEL_TOKEN) return CSA2_ERR_INVALID_ARG;
    if (!cache->page_table || cache->page_size < 8 || (cache->page_size & (cache->page_size - 1)) ||
        cache->max_pages_per_seq < 1 || cache->n_phys_pages < 1)
        return CSA2_ERR_INVALID_ARG;
    const void* rows = level == CSA2_LEVEL_BLOCK ? (const void*)cache->idx_k_pooled : (const void*)cache->idx_k;
    if (!rows || !al(rows, 16) || !al(q_idx, 4) || !al(w, 16) || !al(seq_lens, 4) || !al(ids, 4) ||
        !al(scores, 4) || (ids_out && !al(ids_out, 4)) || (err_word && !al(err_word, 4)))
        return CSA2_ERR_INVALID_ARG;
    if (max_len > (int64_t)cache->max_pages_per_seq * cache->page_size || id_offset < 0) return CSA2_ERR_INVALID_ARG;
    ScoreIdsArgs a{};
    a.cache = *cache;
    a.q_idx = q_idx;
    a.w = w;
    a.seq_lens = seq_lens;
    a.ids = ids;
    a.scores = scores;
    a.ids_out = ids_out;
    a.err = err_word;
    a.max_len = max_len;
    a.k = k;
    a.level = level;
    a.page_shift = page_shift_of(*cache);
    a.id_offset = id_offset;
    LaunchCfg c(dim3((unsigned)((k + SI_THREADS - 1) / SI_THREADS), (unsigned)n), dim3(SI_THREADS), 0,
                (cudaStream_t)stream);
    return status_of(cudaLaunchKernelEx(&c.cfg, score_ids_kernel, a));
}

CSA2_API csa2_status csa2_topk_merge(const float* scores, const int32_t* ids, int32_t n_parts, int32_t part_len,
                                     int32_t k, int32_t lo, int32_t hi, int32_t* out, int32_t* out_local, int32_t n,
                                     void* stream) {
    if (!scores || !ids || !out || n < 1 || n_parts < 1 || part_len < 1 ||
        (int64_t)n_parts * part_len > MG_MAX_PAIRS || k < 1 || k > kMaxKeep || lo < 0 || hi < lo)
        return CSA2_ERR_INVALID_ARG;
    if (!al(scores, 4) || !al(ids, 4) || !al(out, 4) || (out_local && !al(out_local, 4)))
        return CSA2_ERR_INVALID_ARG;
    static bool done[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return status_of(e);
    if (dev < 0 || dev >= 64) return CSA2_ERR_CUDA;
    if (!done[dev]) {
        e = cudaFuncSetAttribute((const void*)topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)MG_SMEM);
        if (e != cudaSuccess) return status_of(e);
        done[dev] = true;
    }
    MergeArgs a{scores, ids, out, out_local, n, n_parts, part_len, k, lo, hi};
    LaunchCfg c(dim3((unsigned)n), dim3(MG_THREADS), MG_SMEM, (cudaStream_t)stream);
    return status_of(cudaLaunchKernelEx(&c.cfg, topk_merge_kernel, a));
}

CSA2_API csa2_status csa2_attn_lse_merge(int32_t n_parts, const float* out_parts, const float* lse_parts, float* out,
                                         float* lse, int32_t rows, void* stream) {
    if (n_parts < 1 || rows < 0 || !out_parts || !lse_parts || !out || !lse) return CSA2_ERR_INVALID_ARG;
    if (!al(out_parts, 16) || !al(out, 16) || !al(lse_parts, 4) || !al(lse, 4)) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;
    LaunchCfg c(dim3((unsigned)rows * kH), dim3(32), 0, (cudaStream_t)stream);
    return status_of(cudaLaunchKernelEx(&c.cfg, lse_merge_kernel, n_parts, out_parts, lse_parts, out, lse, rows));
}

}  // extern "C"
