// Indexer kernels: score = sum_h w_h * ReLU(q_h . k) and Top-K selection.
//
// Pages: CSA2 paragraph of "DeepSeek lanca V4.1-Flash..." (conexaotc.com.br):
// Full layers select Top-512, Reindex layers re-score the Full layer's indexer
// K with their own indexer Q, and the decoder's hierarchical indexer keeps up
// to 2048 blocks of 8 positions (16,384 candidates); "Como funciona"
// (e-cogni.com.br) for the Reindex/Reuse semantics.
//
// Arithmetic contract (shared with the CPU oracle by definition, not by code):
// each head's dot product is a sequential fp32 FMA chain over d = 0..63, the
// head sum a sequential fp32 FMA chain over h = 0..3, Top-K ranks by
// (score desc, index asc).  Every score is therefore bit-identical to the
// oracle's and the selected sets are exact.
//
// Kernels
//   block_score_kernel  (K2)  stream the pooled indexer K of every block of a
//                              sequence, write fp32 scores and a 4096-bin
//                              histogram of the top 12 key bits; the last CTA
//                              of a sequence finds the bin holding the
//                              keep-th largest score.  HBM-bound: 128 B/block.
//   block_select_kernel (K3)  mark blocks above that bin in a bitmap, collect
//                              the bin's members; the last CTA refines the
//                              boundary with two 10-bit passes and emits the
//                              kept blocks in ascending order.
//   token_topk_kernel   (K4)  score the <= 16,384 candidates (1 KiB runs of 8
//                              indexer-K rows), the last CTA of a sequence
//                              selects the Top-K with a 12/10/10-bit radix
//                              select in shared memory.
//   prefill_score_kernel / prefill_select_kernel: the same per query over the
//                              entries visible to it.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

// ----------------------------------------------------------------------------
// score of one indexer-K row held as 32 bf16x2 words; qd[d] = (q_0..q_3)[d]
// ----------------------------------------------------------------------------
__device__ __forceinline__ float idx_score(const uint32_t (&k)[32], const float4* __restrict__ qd, float4 w) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float k0 = bf16_lo(k[i]), k1 = bf16_hi(k[i]);
        const float4 q0 = qd[2 * i], q1 = qd[2 * i + 1];
        a0 = __fmaf_rn(q0.x, k0, a0);
        a1 = __fmaf_rn(q0.y, k0, a1);
        a2 = __fmaf_rn(q0.z, k0, a2);
        a3 = __fmaf_rn(q0.w, k0, a3);
        a0 = __fmaf_rn(q1.x, k1, a0);
        a1 = __fmaf_rn(q1.y, k1, a1);
        a2 = __fmaf_rn(q1.z, k1, a2);
        a3 = __fmaf_rn(q1.w, k1, a3);
    }
    float s = 0.f;
    s = __fmaf_rn(w.x, a0 > 0.f ? a0 : 0.f, s);
    s = __fmaf_rn(w.y, a1 > 0.f ? a1 : 0.f, s);
    s = __fmaf_rn(w.z, a2 > 0.f ? a2 : 0.f, s);
    s = __fmaf_rn(w.w, a3 > 0.f ? a3 : 0.f, s);
    return s;
}

// Two rows at once (amortises the q reads from shared memory).
__device__ __forceinline__ void idx_score2(const uint32_t (&k)[32], const uint32_t (&m)[32],
                                           const float4* __restrict__ qd, float4 w, float& s_k, float& s_m) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float k0 = bf16_lo(k[i]), k1 = bf16_hi(k[i]);
        const float m0 = bf16_lo(m[i]), m1 = bf16_hi(m[i]);
        const float4 q0 = qd[2 * i], q1 = qd[2 * i + 1];
        a0 = __fmaf_rn(q0.x, k0, a0);
        a1 = __fmaf_rn(q0.y, k0, a1);
        a2 = __fmaf_rn(q0.z, k0, a2);
        a3 = __fmaf_rn(q0.w, k0, a3);
        b0 = __fmaf_rn(q0.x, m0, b0);
        b1 = __fmaf_rn(q0.y, m0, b1);
        b2 = __fmaf_rn(q0.z, m0, b2);
        b3 = __fmaf_rn(q0.w, m0, b3);
        a0 = __fmaf_rn(q1.x, k1, a0);
        a1 = __fmaf_rn(q1.y, k1, a1);
        a2 = __fmaf_rn(q1.z, k1, a2);
        a3 = __fmaf_rn(q1.w, k1, a3);
        b0 = __fmaf_rn(q1.x, m1, b0);
        b1 = __fmaf_rn(q1.y, m1, b1);
        b2 = __fmaf_rn(q1.z, m1, b2);
        b3 = __fmaf_rn(q1.w, m1, b3);
    }
    float s = 0.f, t = 0.f;
    s = __fmaf_rn(w.x, a0 > 0.f ? a0 : 0.f, s);
    t = __fmaf_rn(w.x, b0 > 0.f ? b0 : 0.f, t);
    s = __fmaf_rn(w.y, a1 > 0.f ? a1 : 0.f, s);
    t = __fmaf_rn(w.y, b1 > 0.f ? b1 : 0.f, t);
    s = __fmaf_rn(w.z, a2 > 0.f ? a2 : 0.f, s);
    t = __fmaf_rn(w.z, b2 > 0.f ? b2 : 0.f, t);
    s = __fmaf_rn(w.w, a3 > 0.f ? a3 : 0.f, s);
    t = __fmaf_rn(w.w, b3 > 0.f ? b3 : 0.f, t);
    s_k = s;
    s_m = t;
}

// Load q_idx [4][64] bf16 of one sequence/query into qd[64] (transposed, fp32).
__device__ __forceinline__ void load_q_idx(const uint16_t* q, float4* qd) {
    for (int d = threadIdx.x; d < kID; d += blockDim.x) {
        qd[d] = make_float4(bf16_bits_to_f32(q[d]), bf16_bits_to_f32(q[kID + d]), bf16_bits_to_f32(q[2 * kID + d]),
                            bf16_bits_to_f32(q[3 * kID + d]));
    }
}

// Row r of a staged tile: 128 B in 8 chunks of 16 B, chunk c stored at
// position c ^ (r & 7) so that 8 consecutive rows read at one logical chunk hit
// 8 distinct bank groups.
__device__ __forceinline__ void read_row(const uint8_t* tile, int r, uint32_t (&k)[32]) {
    const uint8_t* row = tile + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
        k[4 * c] = v.x;
        k[4 * c + 1] = v.y;
        k[4 * c + 2] = v.z;
        k[4 * c + 3] = v.w;
    }
}

// ----------------------------------------------------------------------------
// Top-K of the keys[0..nslots) held in shared memory (key 0 = not a candidate):
// emits pos_of(slot) of the Top-min(topk, valid) slots, ascending by slot, and
// -1 after them.  Whole block; scratch: hist[4096], list[nslots] (u16), tmp[64].
// ----------------------------------------------------------------------------
template <class PosFn>
__device__ void select_sorted(const uint32_t* keys, int nslots, int topk, int32_t* __restrict__ out, uint32_t* hist,
                              uint16_t* list, uint32_t* tmp, PosFn pos_of) {
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int i = tid; i < kHistBins; i += nt) hist[i] = 0;
    if (tid == 0) tmp[48] = 0;
    __syncthreads();
    uint32_t nv = 0;
    for (int i = tid; i < nslots; i += nt) {
        const uint32_t k = keys[i];
        if (k) {
            atomicAdd(&hist[k >> 20], 1u);
            ++nv;
        }
    }
    uint32_t n_valid;
    block_excl_scan(nv, tmp, &n_valid);  // also orders the histogram writes
    const uint32_t kk = min((uint32_t)topk, n_valid);
    if (kk == 0) {
        for (int i = tid; i < topk; i += nt) out[i] = -1;
        return;
    }
    int b1, d2, d3;
    uint32_t above;
    find_kth_bin(hist, kHistBins, kk, tmp, &b1, &above);
    uint32_t need = kk - above;
    for (int i = tid; i < nslots; i += nt) {
        const uint32_t k = keys[i];
        if (k && (int)(k >> 20) == b1) list[atomicAdd(&tmp[48], 1u)] = (uint16_t)i;
    }
    for (int i = tid; i < 1024; i += nt) hist[i] = 0;
    __syncthreads();
    const int nl = (int)tmp[48];
    for (int i = tid; i < nl; i += nt) atomicAdd(&hist[(keys[list[i]] >> 10) & 1023u], 1u);
    __syncthreads();
    find_kth_bin(hist, 1024, need, tmp, &d2, &above);
    need -= above;
    for (int i = tid; i < 1024; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < nl; i += nt) {
        const uint32_t k = keys[list[i]];
        if ((int)((k >> 10) & 1023u) == d2) atomicAdd(&hist[k & 1023u], 1u);
    }
    __syncthreads();
    find_kth_bin(hist, 1024, need, tmp, &d3, &above);
    need -= above;  // ties at the threshold key still to take, lowest slots first
    const uint32_t T = ((uint32_t)b1 << 20) | ((uint32_t)d2 << 10) | (uint32_t)d3;

    // ordered emission: warp w owns slots [w*seg, (w+1)*seg), 32 at a time
    const int lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
    const int seg = ((nslots + nw - 1) / nw + 31) & ~31;
    const int lo = wid * seg, hi = min(nslots, lo + seg);
    uint32_t n_gt = 0, n_eq = 0;
    for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const uint32_t k = i < hi ? keys[i] : 0u;
        n_gt += __popc(__ballot_sync(0xffffffffu, k > T));
        n_eq += __popc(__ballot_sync(0xffffffffu, k == T));
    }
    // per-warp totals -> exclusive prefixes of ties and of selections
    uint32_t* wt = tmp;  // [0..nw) ties, [32..32+nw) selections
    __syncthreads();
    if (lane == 0) {
        wt[wid] = n_eq;
        wt[32 + wid] = n_gt;
    }
    __syncthreads();
    uint32_t tie_base = 0, sel_base = 0;
    for (int v = 0; v < wid; ++v) tie_base += wt[v];
    for (int v = 0; v < wid; ++v) {
        const uint32_t ties_v = wt[v];
        uint32_t tb = 0;
        for (int u = 0; u < v; ++u) tb += wt[u];
        const uint32_t take = tb >= need ? 0u : min(ties_v, need - tb);
        sel_base += wt[32 + v] + take;
    }
    const unsigned lt = (1u << lane) - 1u;
    for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const uint32_t k = i < hi ? keys[i] : 0u;
        const unsigned meq = __ballot_sync(0xffffffffu, k == T);
        const uint32_t rank = tie_base + __popc(meq & lt);
        const bool sel = (k > T) || (k == T && rank < need);
        const unsigned msel = __ballot_sync(0xffffffffu, sel);
        if (sel) out[sel_base + __popc(msel & lt)] = pos_of(i);
        sel_base += __popc(msel);
        tie_base += __popc(meq);
    }
    for (int i = kk + tid; i < topk; i += nt) out[i] = -1;
}

// ============================================================================
// K2: block scores + histogram
// ============================================================================
constexpr int K2_THREADS = 256;
constexpr int K2_ROW = 2 * K2_THREADS;  // rows per round (two per thread)
constexpr int K2_ROUNDS = 4;
constexpr int K2_CHUNK = K2_ROW * K2_ROUNDS;  // 2048 blocks per CTA
constexpr size_t K2_STAGE = (size_t)K2_ROW * 128;
constexpr size_t K2_SMEM = 2 * K2_STAGE + kHistBins * 4 + kID * 16 + 64 * 4;

struct BlockArgs {
    csa2_kv_cache cache;
    const uint16_t* q_idx;
    const float* w;
    const int32_t* seq_lens;
    int32_t* out;
    float* scores;     // [n][nblk_pad]
    uint32_t* hist;    // [n][4096]
    int32_t* thr;      // [n][4]
    uint32_t* ctr;     // [n][2]
    uint32_t* bitmap;  // [n][nblk_pad/32]
    uint64_t* bnd;     // [n][nblk_pad]
    uint32_t* bnd_cnt; // [n]
    int32_t* err;
    int64_t nblk_pad;
    int64_t max_len;
    int keep;
};

__device__ __forceinline__ int64_t seq_len_checked(const int32_t* seq_lens, int b, int64_t max_len, int32_t* err) {
    int64_t L = seq_lens[b];
    if (L < 1 || L > max_len) {
        if (threadIdx.x == 0) dev_error(err, CSA2_DEV_LEN);
        return 0;
    }
    return L;
}

__device__ __forceinline__ void k2_issue(const BlockArgs& a, int b, int64_t j0, int64_t c1, uint8_t* stage) {
    // 8 x 16 B per row; copy ci = tid + 256 i covers row ci/8, chunk ci%8
#pragma unroll
    for (int i = 0; i < 8 * K2_ROW / K2_THREADS; ++i) {
        const int ci = threadIdx.x + K2_THREADS * i;
        const int r = ci >> 3, c = ci & 7;
        const int64_t j = j0 + r;
        uint8_t* dst = stage + r * 128 + ((c ^ (r & 7)) << 4);
        if (j < c1) {
            const int64_t slot = entry_slot(a.cache, b, j * kBlk, a.err);
            if (slot >= 0) {
                cp_async16(dst, a.cache.idx_k_pooled + (slot >> 3) * kID + c * 8);
                continue;
            }
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
}

__global__ void __launch_bounds__(K2_THREADS) block_score_kernel(BlockArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* stage = smem;
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + 2 * K2_STAGE);
    float4* qd = reinterpret_cast<float4*>(hist + kHistBins);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(qd + kID);
    __shared__ int s_last;

    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.y;
    const int64_t L = seq_len_checked(a.seq_lens, b, a.max_len, a.err);
    const int64_t nblk = (L + kBlk - 1) / kBlk;
    if (nblk <= a.keep) return;
    const int64_t c0 = (int64_t)blockIdx.x * K2_CHUNK;
    if (c0 >= nblk) return;
    const int64_t c1 = min(c0 + K2_CHUNK, nblk);
    const int nrounds = (int)((c1 - c0 + K2_ROW - 1) / K2_ROW);

    k2_issue(a, b, c0, c1, stage);
    cp_async_commit();
    load_q_idx(a.q_idx + (int64_t)b * kIH * kID, qd);
    const float4 w = *reinterpret_cast<const float4*>(a.w + (int64_t)b * kIH);
    for (int i = threadIdx.x; i < kHistBins; i += K2_THREADS) hist[i] = 0;
    float* scores = a.scores + (int64_t)b * a.nblk_pad;

    for (int r = 0; r < nrounds; ++r) {
        if (r + 1 < nrounds) {
            k2_issue(a, b, c0 + (int64_t)(r + 1) * K2_ROW, c1, stage + ((r + 1) & 1) * K2_STAGE);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint8_t* tile = stage + (r & 1) * K2_STAGE;
        const int r0 = threadIdx.x, r1 = threadIdx.x + K2_THREADS;
        const int64_t j0 = c0 + (int64_t)r * K2_ROW + r0, j1 = c0 + (int64_t)r * K2_ROW + r1;
        uint32_t k[32], m[32];
        read_row(tile, r0, k);
        read_row(tile, r1, m);
        float s0, s1;
        idx_score2(k, m, qd, w, s0, s1);
        if (j0 < c1) {
            scores[j0] = s0;
            atomicAdd(&hist[score_key(s0) >> 20], 1u);
        }
        if (j1 < c1) {
            scores[j1] = s1;
            atomicAdd(&hist[score_key(s1) >> 20], 1u);
        }
        __syncthreads();
    }

    uint32_t* gh = a.hist + (int64_t)b * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += K2_THREADS)
        if (hist[i]) atomicAdd(&gh[i], hist[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t nch = (uint32_t)((nblk + K2_CHUNK - 1) / K2_CHUNK);
        s_last = atomicAdd(&a.ctr[2 * b], 1u) == nch - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < kHistBins; i += K2_THREADS) {
        hist[i] = __ldcg(&gh[i]);
        gh[i] = 0;
    }
    __syncthreads();
    int bin;
    uint32_t above;
    find_kth_bin(hist, kHistBins, (uint32_t)a.keep, tmp, &bin, &above);
    if (threadIdx.x == 0) {
        a.thr[4 * b] = bin;
        a.thr[4 * b + 1] = (int32_t)above;
        a.ctr[2 * b] = 0;
    }
}

// ============================================================================
// K3: block select (filter + last-CTA finalize)
// ============================================================================
constexpr int K3_THREADS = 512;
constexpr int K3_CHUNK = 8192;
constexpr size_t K3_SMEM = (size_t)2 * (kMaxBlockLevelLen / kBlk / 32) * 4 + 1024 * 4 + 64 * 4;

__global__ void __launch_bounds__(K3_THREADS) block_select_kernel(BlockArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_last;
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.y;
    const int64_t L = seq_len_checked(a.seq_lens, b, a.max_len, a.err);
    const int64_t nblk = (L + kBlk - 1) / kBlk;
    int32_t* out = a.out + (int64_t)b * a.keep;
    if (nblk <= a.keep) {
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i < a.keep; i += K3_THREADS) out[i] = i < nblk ? i : -1;
        return;
    }
    const int64_t c0 = (int64_t)blockIdx.x * K3_CHUNK;
    if (c0 >= nblk) return;
    const int64_t c1 = min(c0 + K3_CHUNK, nblk);
    const uint32_t bstar = (uint32_t)__ldcg(&a.thr[4 * b]);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const float* scores = a.scores + (int64_t)b * a.nblk_pad;
    uint32_t* bitmap = a.bitmap + (int64_t)b * (a.nblk_pad >> 5);
    uint64_t* bnd = a.bnd + (int64_t)b * a.nblk_pad;
    for (int64_t base = c0 + wid * 32; base < c1; base += K3_THREADS) {
        const int64_t j = base + lane;
        const uint32_t key = j < c1 ? score_key(__ldcg(&scores[j])) : 0u;
        const uint32_t bin = key >> 20;
        const unsigned mgt = __ballot_sync(0xffffffffu, j < c1 && bin > bstar);
        const unsigned meq = __ballot_sync(0xffffffffu, j < c1 && bin == bstar);
        if (lane == 0) bitmap[base >> 5] = mgt;
        if (meq) {
            const int leader = __ffs(meq) - 1;
            uint32_t pos = 0;
            if (lane == leader) pos = atomicAdd(&a.bnd_cnt[b], (uint32_t)__popc(meq));
            pos = __shfl_sync(0xffffffffu, pos, leader);
            if ((meq >> lane) & 1u)
                bnd[pos + __popc(meq & ((1u << lane) - 1u))] = ((uint64_t)key << 32) | (uint64_t)j;
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t nch = (uint32_t)((nblk + K3_CHUNK - 1) / K3_CHUNK);
        s_last = atomicAdd(&a.ctr[2 * b + 1], 1u) == nch - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- finalize: exact threshold inside the boundary bin -----------------
    const int nwords = (int)((nblk + 31) >> 5);
    uint32_t* bm = reinterpret_cast<uint32_t*>(smem);
    uint32_t* tie = bm + (kMaxBlockLevelLen / kBlk / 32);
    uint32_t* hist = tie + (kMaxBlockLevelLen / kBlk / 32);
    uint32_t* tmp = hist + 1024;
    const uint32_t n_bnd = __ldcg(&a.bnd_cnt[b]);
    uint32_t need = (uint32_t)a.keep - (uint32_t)__ldcg(&a.thr[4 * b + 1]);
    int d2, d3;
    uint32_t above;
    for (int i = threadIdx.x; i < 1024; i += K3_THREADS) hist[i] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS)
        atomicAdd(&hist[(uint32_t)(__ldcg(&bnd[i]) >> 42) & 1023u], 1u);
    __syncthreads();
    find_kth_bin(hist, 1024, need, tmp, &d2, &above);
    need -= above;
    for (int i = threadIdx.x; i < 1024; i += K3_THREADS) hist[i] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS) {
        const uint32_t key = (uint32_t)(__ldcg(&bnd[i]) >> 32);
        if ((int)((key >> 10) & 1023u) == d2) atomicAdd(&hist[key & 1023u], 1u);
    }
    __syncthreads();
    find_kth_bin(hist, 1024, need, tmp, &d3, &above);
    need -= above;
    const uint32_t T = (bstar << 20) | ((uint32_t)d2 << 10) | (uint32_t)d3;

    for (int i = threadIdx.x; i < nwords; i += K3_THREADS) {
        bm[i] = __ldcg(&bitmap[i]);
        tie[i] = 0;
    }
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS) {
        const uint64_t v = __ldcg(&bnd[i]);
        const uint32_t key = (uint32_t)(v >> 32), j = (uint32_t)v;
        if (key > T) atomicOr(&bm[j >> 5], 1u << (j & 31));
        else if (key == T) atomicOr(&tie[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    // ordered scan over words: thread t owns words [t*per, (t+1)*per)
    const int per = (nwords + K3_THREADS - 1) / K3_THREADS;
    const int w0 = threadIdx.x * per, w1 = min(nwords, w0 + per);
    uint32_t my_ties = 0;
    for (int i = w0; i < w1; ++i) my_ties += __popc(tie[i]);
    uint32_t tot;
    uint32_t rank = block_excl_scan(my_ties, tmp, &tot);
    uint32_t my_sel = 0;
    for (int i = w0; i < w1; ++i) {
        uint32_t t = tie[i], kept = 0;
        while (t && rank < need) {
            const uint32_t lb = t & (0u - t);
            kept |= lb;
            t ^= lb;
            ++rank;
        }
        rank += __popc(t);
        bm[i] |= kept;
        my_sel += __popc(bm[i]);
    }
    uint32_t base = block_excl_scan(my_sel, tmp, &tot);
    for (int i = w0; i < w1; ++i) {
        uint32_t m = bm[i];
        while (m) {
            const int bit = __ffs(m) - 1;
            m &= m - 1;
            if (base < (uint32_t)a.keep) out[base] = i * 32 + bit;
            ++base;
        }
    }
    for (int i = (int)tot + threadIdx.x; i < a.keep; i += K3_THREADS) out[i] = -1;
    if (threadIdx.x == 0) {
        a.bnd_cnt[b] = 0;
        a.ctr[2 * b + 1] = 0;
    }
}

// ============================================================================
// K4: token scores over the candidates + last-CTA Top-K
// ============================================================================
constexpr int K4_THREADS = 512;
constexpr int K4_CHUNK = 1024;  // candidate slots per CTA (two rounds of 512)
constexpr size_t K4_STAGE = (size_t)K4_THREADS * 128;
constexpr size_t K4_SMEM_SCORE = 2 * K4_STAGE + kID * 16;
constexpr size_t K4_SMEM_SELECT = (size_t)kMaxCand * 4 + kHistBins * 4 + kMaxCand * 2 + 64 * 4;
constexpr size_t K4_SMEM = K4_SMEM_SCORE > K4_SMEM_SELECT ? K4_SMEM_SCORE : K4_SMEM_SELECT;

struct TokenArgs {
    csa2_kv_cache cache;
    const uint16_t* q_idx;
    const float* w;
    const int32_t* seq_lens;
    const int32_t* cand;  // [n][keep] or null (flat)
    int32_t* out;         // [n][topk]
    uint32_t* keys;       // [n][kMaxCand]
    uint32_t* ctr;        // [n]
    int32_t* err;
    int64_t max_len;
    int keep, topk;
};

// position of candidate slot i, or -1 if the slot is empty
__device__ __forceinline__ int64_t cand_pos(const TokenArgs& a, int b, int i, int64_t L) {
    int64_t blk = i >> 3;
    if (a.cand) {
        blk = __ldg(a.cand + (int64_t)b * a.keep + (i >> 3));
        if (blk < 0) return -1;
    }
    const int64_t p = blk * kBlk + (i & 7);
    return p < L ? p : -1;
}

__device__ __forceinline__ void k4_issue(const TokenArgs& a, int b, int i0, int nslots, int64_t L, uint8_t* stage) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int ci = threadIdx.x + K4_THREADS * i;
        const int r = ci >> 3, c = ci & 7;
        uint8_t* dst = stage + r * 128 + ((c ^ (r & 7)) << 4);
        const int slot_i = i0 + r;
        if (slot_i < nslots) {
            const int64_t p = cand_pos(a, b, slot_i, L);
            if (p >= 0) {
                const int64_t slot = entry_slot(a.cache, b, p, a.err);
                if (slot >= 0) {
                    cp_async16(dst, a.cache.idx_k + slot * kID + c * 8);
                    continue;
                }
            }
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
}

__global__ void __launch_bounds__(K4_THREADS) token_topk_kernel(TokenArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_last;
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.y;
    int64_t L = seq_len_checked(a.seq_lens, b, a.max_len, a.err);
    int nslots = a.cand ? a.keep * kBlk : (int)(L < (int64_t)a.keep * kBlk ? L : (int64_t)a.keep * kBlk);
    if (!a.cand && L > (int64_t)a.keep * kBlk) {
        if (threadIdx.x == 0) dev_error(a.err, CSA2_DEV_LEN);
    }
    const int nch = (nslots + K4_CHUNK - 1) / K4_CHUNK;
    if (L == 0 || nch == 0) {
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i < a.topk; i += K4_THREADS) a.out[(int64_t)b * a.topk + i] = -1;
        return;
    }
    const int i0 = blockIdx.x * K4_CHUNK;
    if (i0 >= nslots) return;

    uint8_t* stage = smem;
    float4* qd = reinterpret_cast<float4*>(smem + 2 * K4_STAGE);
    k4_issue(a, b, i0, nslots, L, stage);
    cp_async_commit();
    k4_issue(a, b, i0 + K4_THREADS, nslots, L, stage + K4_STAGE);
    cp_async_commit();
    load_q_idx(a.q_idx + (int64_t)b * kIH * kID, qd);
    const float4 w = *reinterpret_cast<const float4*>(a.w + (int64_t)b * kIH);
    uint32_t* keys = a.keys + (int64_t)b * kMaxCand;
    cp_async_wait<0>();
    __syncthreads();
    {
        uint32_t k[32], m[32];
        read_row(stage, threadIdx.x, k);
        read_row(stage + K4_STAGE, threadIdx.x, m);
        float s0, s1;
        idx_score2(k, m, qd, w, s0, s1);
        const int sa = i0 + threadIdx.x, sb = i0 + K4_THREADS + threadIdx.x;
        if (sa < nslots) keys[sa] = cand_pos(a, b, sa, L) >= 0 ? score_key(s0) : 0u;
        if (sb < nslots) keys[sb] = cand_pos(a, b, sb, L) >= 0 ? score_key(s1) : 0u;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&a.ctr[b], 1u) == (uint32_t)nch - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem);
    uint32_t* hist = skeys + kMaxCand;
    uint16_t* list = reinterpret_cast<uint16_t*>(hist + kHistBins);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(list + kMaxCand);
    for (int i = threadIdx.x; i < nslots; i += K4_THREADS) skeys[i] = __ldcg(&keys[i]);
    __syncthreads();
    select_sorted(skeys, nslots, a.topk, a.out + (int64_t)b * a.topk, hist, list, tmp,
                  [&](int i) { return (int32_t)cand_pos(a, b, i, L); });
    if (threadIdx.x == 0) a.ctr[b] = 0;
}

// ============================================================================
// Prefill (flat, causal): all scores to the workspace, then one CTA per query
// ============================================================================
constexpr int PS_THREADS = 256;
constexpr int PS_Q = 32;   // queries per CTA
constexpr int PS_E = 64;   // entries per tile
struct PrefillArgs {
    csa2_kv_cache cache;
    const uint16_t* q_idx;
    const float* w;
    const int32_t* q_pos;
    int32_t* out;
    uint32_t* keys;  // [T][stride]
    int32_t* err;
    int64_t stride;
    int T, ratio, topk, n_entries;
};

__device__ __forceinline__ int visible(int p, int ratio, int n) { return min((p + 1) / ratio, n); }

// Thread (qi, ei) of a 16 x 16 grid computes queries 2qi, 2qi+1 against entries
// 4ei .. 4ei+3 of the tile: 32 sequential fp32 FMA chains.
constexpr size_t PS_SMEM = (size_t)kID * PS_E * 4 + (size_t)kID * PS_Q * kIH * 4;

__global__ void __launch_bounds__(PS_THREADS) prefill_score_kernel(PrefillArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    float (*kt)[PS_E] = reinterpret_cast<float (*)[PS_E]>(smem);                               // [d][entry]
    float (*qs)[PS_Q][kIH] = reinterpret_cast<float (*)[PS_Q][kIH]>(smem + (size_t)kID * PS_E * 4);  // [d][q][h]
    __shared__ float ws_[PS_Q][kIH];
    __shared__ int vis[PS_Q];
    pdl_wait();
    pdl_trigger();
    const int q0 = blockIdx.x * PS_Q;
    const int tid = threadIdx.x;
    for (int i = tid; i < PS_Q * kIH * kID; i += PS_THREADS) {
        const int qq = i / (kIH * kID), h = (i / kID) % kIH, d = i % kID;
        const int t = q0 + qq;
        qs[d][qq][h] = t < a.T ? bf16_bits_to_f32(a.q_idx[(int64_t)t * kIH * kID + h * kID + d]) : 0.f;
    }
    if (tid < PS_Q * kIH) {
        const int t = q0 + tid / kIH;
        ws_[tid / kIH][tid % kIH] = t < a.T ? a.w[(int64_t)t * kIH + tid % kIH] : 0.f;
    }
    int max_vis = 0;
    if (tid < PS_Q) vis[tid] = q0 + tid < a.T ? visible(a.q_pos[q0 + tid], a.ratio, a.n_entries) : 0;
    __syncthreads();
    for (int i = 0; i < PS_Q; ++i) max_vis = max(max_vis, vis[i]);
    const int qi = tid >> 4, ei = tid & 15;
    const int n_stride_tiles = (int)(a.stride / PS_E);
    for (int tile = 0; tile < n_stride_tiles; ++tile) {
        const int e0 = tile * PS_E;
        if (e0 < max_vis) {
            __syncthreads();
            for (int i = tid; i < PS_E * 8; i += PS_THREADS) {  // 8 x 16 B per entry row
                const int r = i >> 3, c = i & 7;
                const int e = e0 + r;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (e < max_vis) {
                    const int64_t slot = entry_slot(a.cache, 0, e, a.err);
                    if (slot >= 0) v = __ldg(reinterpret_cast<const uint4*>(a.cache.idx_k + slot * kID) + c);
                }
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    kt[c * 8 + 2 * u][r] = bf16_lo(wv[u]);
                    kt[c * 8 + 2 * u + 1][r] = bf16_hi(wv[u]);
                }
            }
            __syncthreads();
            float acc[2][4][kIH];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y)
#pragma unroll
                    for (int h = 0; h < kIH; ++h) acc[x][y][h] = 0.f;
#pragma unroll 4
            for (int d = 0; d < kID; ++d) {
                const float4 kv = *reinterpret_cast<const float4*>(&kt[d][4 * ei]);
                const float4 qa = *reinterpret_cast<const float4*>(&qs[d][2 * qi][0]);
                const float4 qb = *reinterpret_cast<const float4*>(&qs[d][2 * qi + 1][0]);
                const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    acc[0][y][0] = __fmaf_rn(qa.x, kk[y], acc[0][y][0]);
                    acc[0][y][1] = __fmaf_rn(qa.y, kk[y], acc[0][y][1]);
                    acc[0][y][2] = __fmaf_rn(qa.z, kk[y], acc[0][y][2]);
                    acc[0][y][3] = __fmaf_rn(qa.w, kk[y], acc[0][y][3]);
                    acc[1][y][0] = __fmaf_rn(qb.x, kk[y], acc[1][y][0]);
                    acc[1][y][1] = __fmaf_rn(qb.y, kk[y], acc[1][y][1]);
                    acc[1][y][2] = __fmaf_rn(qb.z, kk[y], acc[1][y][2]);
                    acc[1][y][3] = __fmaf_rn(qb.w, kk[y], acc[1][y][3]);
                }
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int qq = 2 * qi + x, t = q0 + qq;
                if (t >= a.T) continue;
                uint32_t kout[4];
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    float s = 0.f;
#pragma unroll
                    for (int h = 0; h < kIH; ++h) s = __fmaf_rn(ws_[qq][h], acc[x][y][h] > 0.f ? acc[x][y][h] : 0.f, s);
                    const int e = e0 + 4 * ei + y;
                    kout[y] = e < vis[qq] ? score_key(s) : 0u;
                }
                *reinterpret_cast<uint4*>(a.keys + (int64_t)t * a.stride + e0 + 4 * ei) =
                    make_uint4(kout[0], kout[1], kout[2], kout[3]);
            }
        } else {
            for (int i = tid; i < PS_Q * PS_E / 4; i += PS_THREADS) {
                const int qq = i / (PS_E / 4), t = q0 + qq;
                if (t < a.T)
                    *reinterpret_cast<uint4*>(a.keys + (int64_t)t * a.stride + e0 + 4 * (i % (PS_E / 4))) =
                        make_uint4(0, 0, 0, 0);
            }
        }
    }
}

constexpr int PSEL_THREADS = 512;
constexpr size_t PSEL_SMEM = K4_SMEM_SELECT;

__global__ void __launch_bounds__(PSEL_THREADS) prefill_select_kernel(PrefillArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    const int n = (int)a.stride;
    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem);
    uint32_t* hist = skeys + kMaxCand;
    uint16_t* list = reinterpret_cast<uint16_t*>(hist + kHistBins);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(list + kMaxCand);
    const uint4* src = reinterpret_cast<const uint4*>(a.keys + (int64_t)t * a.stride);
    for (int i = threadIdx.x; i < n / 4; i += PSEL_THREADS) reinterpret_cast<uint4*>(skeys)[i] = __ldcs(src + i);
    __syncthreads();
    select_sorted(skeys, n, a.topk, a.out + (int64_t)t * a.topk, hist, list, tmp, [](int i) { return (int32_t)i; });
}

// ============================================================================
// host side
// ============================================================================
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// One layout for both levels: the small arrays that must start at zero come
// first, so a workspace zero-filled once stays valid for any mix of calls with
// the same (n, max_len).
DecodeWs decode_ws_layout(int n, int64_t max_len) {
    DecodeWs l{};
    size_t o = 0;
    const int64_t nblk = (max_len + kBlk - 1) / kBlk;
    l.nblk_pad = (nblk + K3_CHUNK - 1) / K3_CHUNK * K3_CHUNK;
    l.blk_hist = o; o = align256(o + (size_t)n * kHistBins * 4);
    l.blk_ctr = o; o = align256(o + (size_t)n * 8);
    l.blk_bnd_cnt = o; o = align256(o + (size_t)n * 4);
    l.tok_ctr = o; o = align256(o + (size_t)n * 4);
    l.blk_thr = o; o = align256(o + (size_t)n * 16);
    l.tok_keys = o; o = align256(o + (size_t)n * kMaxCand * 4);
    if (nblk > kMaxKeep) {
        l.blk_scores = o; o = align256(o + (size_t)n * l.nblk_pad * 4);
        l.blk_bitmap = o; o = align256(o + (size_t)n * (l.nblk_pad / 32) * 4);
        l.blk_bnd = o; o = align256(o + (size_t)n * l.nblk_pad * 8);
    }
    l.total = o;
    return l;
}

PrefillWs prefill_ws_layout(int T, int64_t n_entries) {
    PrefillWs l{};
    l.stride = (n_entries + PS_E - 1) / PS_E * PS_E;
    l.keys = 0;
    l.total = align256((size_t)T * l.stride * 4);
    return l;
}

static cudaError_t set_smem(const void* fn, size_t bytes) {
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_block_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                              const int32_t* seq_lens, int keep, int32_t* out, int n, int64_t max_len, char* ws,
                              int32_t* err, cudaStream_t stream) {
    static bool init = false;
    if (!init) {
        cudaError_t e = set_smem((const void*)block_score_kernel, K2_SMEM);
        if (e == cudaSuccess) e = set_smem((const void*)block_select_kernel, K3_SMEM);
        if (e != cudaSuccess) return e;
        init = true;
    }
    const DecodeWs l = decode_ws_layout(n, max_len);
    BlockArgs a{};
    a.cache = cache;
    a.q_idx = q_idx;
    a.w = w;
    a.seq_lens = seq_lens;
    a.out = out;
    a.scores = reinterpret_cast<float*>(ws + l.blk_scores);
    a.hist = reinterpret_cast<uint32_t*>(ws + l.blk_hist);
    a.thr = reinterpret_cast<int32_t*>(ws + l.blk_thr);
    a.ctr = reinterpret_cast<uint32_t*>(ws + l.blk_ctr);
    a.bitmap = reinterpret_cast<uint32_t*>(ws + l.blk_bitmap);
    a.bnd = reinterpret_cast<uint64_t*>(ws + l.blk_bnd);
    a.bnd_cnt = reinterpret_cast<uint32_t*>(ws + l.blk_bnd_cnt);
    a.err = err;
    a.nblk_pad = l.nblk_pad;
    a.max_len = max_len;
    a.keep = keep;
    const int64_t nblk = (max_len + kBlk - 1) / kBlk;
    LaunchCfg c2(dim3((unsigned)((nblk + K2_CHUNK - 1) / K2_CHUNK), n), dim3(K2_THREADS), K2_SMEM, stream);
    cudaError_t e = cudaLaunchKernelEx(&c2.cfg, block_score_kernel, a);
    if (e != cudaSuccess) return e;
    LaunchCfg c3(dim3((unsigned)((nblk + K3_CHUNK - 1) / K3_CHUNK), n), dim3(K3_THREADS), K3_SMEM, stream);
    return cudaLaunchKernelEx(&c3.cfg, block_select_kernel, a);
}

cudaError_t launch_token_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                              const int32_t* seq_lens, const int32_t* cand_blocks, int keep, int topk, int32_t* out,
                              int n, int64_t max_len, char* ws, int32_t* err, cudaStream_t stream) {
    static bool init = false;
    if (!init) {
        cudaError_t e = set_smem((const void*)token_topk_kernel, K4_SMEM);
        if (e != cudaSuccess) return e;
        init = true;
    }
    const DecodeWs l = decode_ws_layout(n, max_len);
    TokenArgs a{};
    a.cache = cache;
    a.q_idx = q_idx;
    a.w = w;
    a.seq_lens = seq_lens;
    a.cand = cand_blocks;
    a.out = out;
    a.keys = reinterpret_cast<uint32_t*>(ws + l.tok_keys);
    a.ctr = reinterpret_cast<uint32_t*>(ws + l.tok_ctr);
    a.err = err;
    a.max_len = max_len;
    a.keep = keep;
    a.topk = topk;
    const int nslots_max = keep * kBlk;
    LaunchCfg c(dim3((unsigned)((nslots_max + K4_CHUNK - 1) / K4_CHUNK), n), dim3(K4_THREADS), K4_SMEM, stream);
    return cudaLaunchKernelEx(&c.cfg, token_topk_kernel, a);
}

cudaError_t launch_prefill_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                                const int32_t* seq_lens, const int32_t* q_pos, int ratio, int topk, int32_t* out,
                                int T, int64_t max_len, char* ws, int32_t* err, cudaStream_t stream) {
    static bool init = false;
    if (!init) {
        cudaError_t e = set_smem((const void*)prefill_select_kernel, PSEL_SMEM);
        if (e == cudaSuccess) e = set_smem((const void*)prefill_score_kernel, PS_SMEM);
        if (e != cudaSuccess) return e;
        init = true;
    }
    (void)seq_lens;
    const PrefillWs l = prefill_ws_layout(T, max_len);
    PrefillArgs a{};
    a.cache = cache;
    a.q_idx = q_idx;
    a.w = w;
    a.q_pos = q_pos;
    a.out = out;
    a.keys = reinterpret_cast<uint32_t*>(ws + l.keys);
    a.err = err;
    a.stride = l.stride;
    a.T = T;
    a.ratio = ratio;
    a.topk = topk;
    a.n_entries = (int)max_len;
    LaunchCfg c1(dim3((unsigned)((T + PS_Q - 1) / PS_Q)), dim3(PS_THREADS), PS_SMEM, stream);
    cudaError_t e = cudaLaunchKernelEx(&c1.cfg, prefill_score_kernel, a);
    if (e != cudaSuccess) return e;
    LaunchCfg c2(dim3((unsigned)T), dim3(PSEL_THREADS), PSEL_SMEM, stream);
    return cudaLaunchKernelEx(&c2.cfg, prefill_select_kernel, a);
}

}  // namespace csa2
