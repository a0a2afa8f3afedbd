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
// Selection is a most-significant-digit radix select on order-preserving
// 32-bit keys: a 12-bit first digit (bits 31..20), then two 10-bit digits
// that only look at the slots left in the threshold bin, then an ordered
// emission (ballots in slot order) that keeps ties at the lowest index.
//
// Kernels
//   block_score_kernel  (K2)  stream the pooled indexer K of every block (or,
//                              for a flat selection, the indexer K of every
//                              entry), write fp32 scores and a per-sequence
//                              histogram of the first digit; the last CTA of a
//                              sequence finds the bin holding the keep-th
//                              score.  HBM-bound: 128 B per row.
//   block_select_kernel (K3)  mark rows above that bin in a bitmap and
//                              collect the bin's members; the last CTA refines
//                              the boundary and emits the kept rows in order
//                              (a flat selection lists and sorts them).
//   token_score_kernel  (K4a) 16 CTAs per sequence score the <= 16,384
//                              candidates (1 KiB runs of 8 indexer-K rows) into
//                              the workspace;
//   token_select_kernel (K4b) one CTA per sequence selects the Top-K of
//                              the sequence's keys.
//   prefill_tc_score_kernel / prefill_candidates_kernel: prefill, approximate
//                              scores on tcgen05, exact rescoring of the
//                              candidates and a verified exact Top-K per query;
//   prefill_score_kernel / prefill_select_kernel: the exact fallback for the
//                              queries that fail the verification.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "select.cuh"
#include "tc.cuh"

namespace csa2 {

// ----------------------------------------------------------------------------
// score of one indexer-K row held as 32 bf16x2 words; qd[d] = (q_0..q_3)[d]
// ----------------------------------------------------------------------------
// Two rows at once with packed fp32 arithmetic: fma.rn.f32x2 performs one
// fused multiply-add, rounded to nearest, in each 32-bit half.  The halves hold
// two heads of one row, so every (row, head) dot follows the scalar FMA chain
// over the dimensions bit for bit.  qh[d] = (q_0, q_1, q_2, q_3)[d]: one 16-byte
// load gives the head pairs (0, 1) and (2, 3) of dimension d for both rows.
__device__ __forceinline__ void idx_score2(const uint32_t (&k)[32], const uint32_t (&m)[32],
                                           const ulonglong2* __restrict__ qh, float4 w, float& s_k, float& s_m) {
    uint64_t k01 = 0, k23 = 0, m01 = 0, m23 = 0;  // (head h, head h + 1) dots of rows k and m; zero bits are +0
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const ulonglong2 qa = qh[2 * i], qb = qh[2 * i + 1];  // dimensions 2i and 2i + 1
        const float xk0 = bf16_lo(k[i]), xk1 = bf16_hi(k[i]), xm0 = bf16_lo(m[i]), xm1 = bf16_hi(m[i]);
        const uint64_t dk0 = pack2(xk0, xk0), dm0 = pack2(xm0, xm0), dk1 = pack2(xk1, xk1), dm1 = pack2(xm1, xm1);
        k01 = ffma2(qa.x, dk0, k01);
        k23 = ffma2(qa.y, dk0, k23);
        m01 = ffma2(qa.x, dm0, m01);
        m23 = ffma2(qa.y, dm0, m23);
        k01 = ffma2(qb.x, dk1, k01);
        k23 = ffma2(qb.y, dk1, k23);
        m01 = ffma2(qb.x, dm1, m01);
        m23 = ffma2(qb.y, dm1, m23);
    }
    float a0, a1, a2, a3, b0, b1, b2, b3;
    unpack2(k01, a0, a1);
    unpack2(k23, a2, a3);
    unpack2(m01, b0, b1);
    unpack2(m23, b2, b3);
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

// The same two rows read from a 128-byte-swizzled tile in shared memory chunk by
// chunk as the dimensions advance (rows ra and rb of the tile; chunk c of row r
// at c ^ (r & 7)), so the rows never occupy 64 registers at once.
__device__ __forceinline__ void idx_score2_tile(const uint8_t* tile, int ra, int rb, const ulonglong2* __restrict__ qh,
                                                float4 w, float& s_k, float& s_m) {
    uint64_t k01 = 0, k23 = 0, m01 = 0, m23 = 0;
    const uint8_t* pa = tile + ra * 128;
    const uint8_t* pb = tile + rb * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {  // 16-byte chunk c: dimensions 8c .. 8c + 7
        const uint4 va = *reinterpret_cast<const uint4*>(pa + ((c ^ (ra & 7)) << 4));
        const uint4 vb = *reinterpret_cast<const uint4*>(pb + ((c ^ (rb & 7)) << 4));
        const uint32_t ka[4] = {va.x, va.y, va.z, va.w}, kb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = 4 * c + u;
            const ulonglong2 qa = qh[2 * i], qb = qh[2 * i + 1];
            const float xk0 = bf16_lo(ka[u]), xk1 = bf16_hi(ka[u]), xm0 = bf16_lo(kb[u]), xm1 = bf16_hi(kb[u]);
            const uint64_t dk0 = pack2(xk0, xk0), dm0 = pack2(xm0, xm0), dk1 = pack2(xk1, xk1), dm1 = pack2(xm1, xm1);
            k01 = ffma2(qa.x, dk0, k01);
            k23 = ffma2(qa.y, dk0, k23);
            m01 = ffma2(qa.x, dm0, m01);
            m23 = ffma2(qa.y, dm0, m23);
            k01 = ffma2(qb.x, dk1, k01);
            k23 = ffma2(qb.y, dk1, k23);
            m01 = ffma2(qb.x, dm1, m01);
            m23 = ffma2(qb.y, dm1, m23);
        }
    }
    float a0, a1, a2, a3, b0, b1, b2, b3;
    unpack2(k01, a0, a1);
    unpack2(k23, a2, a3);
    unpack2(m01, b0, b1);
    unpack2(m23, b2, b3);
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

// Load q_idx [4][64] bf16 of one row into the layout idx_score2 reads:
// qh[d] = (q_0, q_1, q_2, q_3)[d].
__device__ __forceinline__ void load_q_heads(const uint16_t* q, float4* qh, int tid, int nt) {
    for (int d = tid; d < kID; d += nt)
        qh[d] = make_float4(bf16_bits_to_f32(q[d]), bf16_bits_to_f32(q[kID + d]), bf16_bits_to_f32(q[2 * kID + d]),
                            bf16_bits_to_f32(q[3 * kID + d]));
}



// Physical page of every page of entries [e0, e1) of one sequence, staged in
// shared memory once per CTA (-1 where the page table has none).
__device__ __forceinline__ void stage_pages(const csa2_kv_cache& c, int shift, int seq, int32_t e0, int32_t e1,
                                            int32_t* pg, int32_t* err) {
    const int32_t p0 = e0 >> shift, p1 = (e1 - 1) >> shift;
    for (int32_t p = p0 + threadIdx.x; p <= p1; p += blockDim.x) {
        int32_t phys = -1;
        if (p < c.max_pages_per_seq) phys = __ldg(c.page_table + (int64_t)seq * c.max_pages_per_seq + p);
        if (phys < 0 || phys >= c.n_phys_pages) {
            dev_error(err, CSA2_DEV_PAGE);
            phys = -1;
        }
        pg[p - p0] = phys;
    }
}

// ============================================================================
// K2: block scores + first-digit histogram
//
// Persistent: one CTA per SM walks a contiguous range of the flattened list of
// 512-row tiles of every sequence that needs block selection, so a ragged batch
// balances across the SMs.  Warp-specialised around a 3-stage ring of 64 KiB
// tiles: four producer warps only copy (16-byte cp.async; lane l moves chunk
// l & 7 of row 4 k + l / 8, so one instruction covers 512 contiguous bytes of a
// page; chunk c of row r lands at chunk c ^ (r & 7)) and signal a stage full
// through an mbarrier once their copies land; eight consumer warps only score
// (lane l takes rows l and l + 32 of its warp's 64: eight independent FMA
// chains) and release the stage through a second mbarrier.  Copies and FMAs
// therefore overlap instead of taking turns.  Entry rows in pages of >= 64
// entries arrive instead as 64-row tensor boxes (one 8 KiB run each).
// ============================================================================
constexpr int K2_CWARPS = 8;                    // consumer (scoring) warps
constexpr int K2_PWARPS = 4;                    // producer (copy) warps
constexpr int K2_CTHREADS = K2_CWARPS * 32;
constexpr int K2_THREADS = (K2_CWARPS + K2_PWARPS) * 32;
constexpr int K2_TILE = 512;                    // pooled rows per tile
constexpr int K2_STAGES = 3;
constexpr size_t K2_STAGE_BYTES = (size_t)K2_TILE * 128;
constexpr int K2_MAX_SEQS = 1024;
constexpr int K2_PROWS = K2_TILE / K2_PWARPS;   // 128 rows copied per producer warp
constexpr int K2_CROWS = K2_TILE / K2_CWARPS;   // 64 rows scored per consumer warp
constexpr size_t K2_OFF_HIST = K2_STAGES * K2_STAGE_BYTES;
constexpr size_t K2_OFF_QD = align16(K2_OFF_HIST + kHistBins * 4);
constexpr size_t K2_OFF_TMP = align16(K2_OFF_QD + kID * 16);  // q by dimension: 64 x 16 B
constexpr size_t K2_OFF_TS = align16(K2_OFF_TMP + 64 * 4);
constexpr size_t K2_OFF_NBLK = align16(K2_OFF_TS + (K2_MAX_SEQS + 1) * 4);
constexpr size_t K2_OFF_BAR = align16(K2_OFF_NBLK + K2_MAX_SEQS * 4);  // full[3], empty[3]
constexpr size_t K2_OFF_MISC = align16(K2_OFF_BAR + 2 * K2_STAGES * 8);  // w (float4), last, timeout
constexpr size_t K2_SMEM = align16(K2_OFF_MISC + 32);
constexpr uint32_t kWaitLimit = 1u << 22;
// Poll limit of the block-scoring copy ring's waits (cp.async rows only): the
// default above, lowered only by csa2_test_set_wait_limit.
static std::atomic<uint32_t> g_copy_wait_limit{kWaitLimit};
static_assert(K2_OFF_QD % 16 == 0 && K2_OFF_BAR % 8 == 0 && K2_OFF_MISC % 16 == 0, "K2 shared-memory layout");

struct BlockArgs {
    csa2_kv_cache cache;
    const uint16_t* q_idx;
    const float* w;
    const int32_t* seq_lens;
    int32_t* out;
    float* scores;     // [n][nblk_pad]
    uint32_t* hist;    // [n][4096]
    int32_t* thr;      // [n][4]
    uint32_t* ctr;     // [n][2]: tiles scored (K2), chunks filtered (K3)
    uint32_t* bitmap;  // [n][nblk_pad/32]
    uint64_t* bnd;     // [n][nblk_pad]
    uint32_t* bnd_cnt; // [n]
    uint32_t* tie;     // [n][nblk_pad/32] (flat only: the finalize's tie bitmap)
    int32_t* abv;      // [n][512] (flat only: rows whose first digit is above the K-th's)
    uint32_t* abv_cnt; // [n]
    const uint8_t* rows;  // scored rows: pooled indexer K (rshift 3) or indexer K (rshift 0)
    int32_t* err;
    int64_t nblk_pad;
    int64_t max_len;
    int n, keep, page_shift;
    int rshift;        // log2 entries per scored row
    int span;          // rows filtered per select CTA (a multiple of 8192)
    int tma;           // 1: rows arrive as 64-row tensor boxes (entry rows, pages of >= 64 entries)
    uint32_t wait_limit;  // polls before a wait of the copy ring gives up (cp.async rows)
};

// tile_start[b] = first tile of sequence b; returns the sequence of tile t
__device__ __forceinline__ int seq_of_tile(const int32_t* tile_start, int n, int32_t t) {
    int lo = 0, hi = n;  // tile_start[lo] <= t < tile_start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_start[mid] <= t) lo = mid;
        else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(K2_THREADS, 1) block_score_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                     BlockArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + K2_OFF_HIST);
    float4* qd = reinterpret_cast<float4*>(smem + K2_OFF_QD);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(smem + K2_OFF_TMP);
    int32_t* tile_start = reinterpret_cast<int32_t*>(smem + K2_OFF_TS);
    int32_t* s_nblk = reinterpret_cast<int32_t*>(smem + K2_OFF_NBLK);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + K2_OFF_BAR);
    uint64_t* empty = full + K2_STAGES;
    float4& s_w = *reinterpret_cast<float4*>(smem + K2_OFF_MISC);
    int& s_last = *reinterpret_cast<int*>(smem + K2_OFF_MISC + 16);
    int& s_timeout = *reinterpret_cast<int*>(smem + K2_OFF_MISC + 20);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

    pdl_wait();
    pdl_trigger();
    // 16-byte copies and vector reads need an aligned base; 128-byte-swizzled
    // tensor boxes a 1 KiB aligned one (uniform over the grid)
    if (smem_u32(smem) & (a.tma ? 1023u : 15u)) {
        if (tid == 0) dev_error(a.err, CSA2_DEV_ALIGN);
        return;
    }
    // ---- tiles of every sequence (0 for sequences that keep all blocks) ------
    {
        const int per = (a.n + K2_THREADS - 1) / K2_THREADS;
        uint32_t mine = 0;
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            if (b < a.n) {
                const int32_t L = a.seq_lens[b];
                const int32_t nblk = (L >= 1 && L <= a.max_len) ? ((L - 1) >> a.rshift) + 1 : 0;
                if (L < 1 || L > a.max_len) dev_error(a.err, CSA2_DEV_LEN);
                mine += nblk > a.keep ? (nblk + K2_TILE - 1) / K2_TILE : 0;
            }
        }
        uint32_t total;
        uint32_t base = block_excl_scan(mine, tmp, &total);
        for (int i = 0; i < per; ++i) {
            const int b = tid * per + i;
            if (b < a.n) {
                tile_start[b] = (int32_t)base;
                const int32_t L = a.seq_lens[b];
                const int32_t nblk = (L >= 1 && L <= a.max_len) ? ((L - 1) >> a.rshift) + 1 : 0;
                s_nblk[b] = nblk;
                base += nblk > a.keep ? (nblk + K2_TILE - 1) / K2_TILE : 0;
            }
        }
        if (tid == 0) {
            tile_start[a.n] = (int32_t)total;
            for (int s = 0; s < K2_STAGES; ++s) {
                // one cp.async arrival per producer thread, or one expect-tx arrival per producer warp
                mbar_init(&full[s], a.tma ? K2_PWARPS : K2_PWARPS * 32);
                mbar_init(&empty[s], K2_CWARPS);  // one arrival per consumer warp
            }
            fence_mbar_init();
            s_timeout = 0;
        }
        for (int i = tid; i < kHistBins; i += K2_THREADS) hist[i] = 0;
        __syncthreads();
    }
    const int32_t T = tile_start[a.n];
    const int32_t t0 = (int32_t)((int64_t)T * blockIdx.x / gridDim.x);
    const int32_t t1 = (int32_t)((int64_t)T * (blockIdx.x + 1) / gridDim.x);
    const int ntiles = t1 - t0;
    if (ntiles <= 0) return;

    if (wid >= K2_CWARPS && a.tma) {
        // ============ producers, tensor boxes (entry rows) ============
        // Lanes 0 and 1 of producer warp pw copy the two 64-row boxes of the
        // warp's 128 rows; a box lies in one page (pages hold >= 64 entries,
        // boxes start at multiples of 64) and lands 128-byte swizzled, chunk c
        // of row r at c ^ (r & 7), the layout the consumers read.
        const int pw = wid - K2_CWARPS;
        const int sh = a.page_shift;
        const int32_t emask = (1 << sh) - 1;
        const int32_t mpps = a.cache.max_pages_per_seq;
        auto box_slot = [&](int32_t t) -> int32_t {  // first slot of this lane's box of tile t, -1 past the end
            const int b = seq_of_tile(tile_start, a.n, t);
            const int32_t j = (t - tile_start[b]) * K2_TILE + K2_PROWS * pw + 64 * lane;
            if (lane >= 2 || j >= s_nblk[b]) return -1;
            const int32_t pg = j >> sh;
            int32_t phys = pg < mpps ? __ldg(a.cache.page_table + (int64_t)b * mpps + pg) : -1;
            if (phys < 0 || phys >= a.cache.n_phys_pages) {
                dev_error(a.err, CSA2_DEV_PAGE);
                phys = 0;  // results of this call are undefined; the copy stays in bounds
            }
            return (int32_t)(((int64_t)phys << sh) | (j & emask));
        };
        int32_t nxt = box_slot(t0);
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % K2_STAGES;
            if (i >= K2_STAGES && !mbar_wait(&empty[s], (uint32_t)((i / K2_STAGES) - 1) & 1u, kWaitLimit))
                s_timeout = 1;
            const int32_t slot = nxt;
            if (i + 1 < ntiles) nxt = box_slot(t0 + i + 1);  // the page lookup overlaps the copies
            const unsigned m = __ballot_sync(0xffffffffu, slot >= 0);
            if (lane == 0) mbar_arrive_expect_tx(&full[s], 64u * 128u * (uint32_t)__popc(m));
            __syncwarp();
            if (slot >= 0)
                tma_load_2d(smem + (size_t)s * K2_STAGE_BYTES + (size_t)(K2_PROWS * pw + 64 * lane) * 128, &tmap, 0,
                            slot, &full[s]);
        }
        // the last stages' copies have landed before this warp leaves (bounded)
        for (int i = max(0, ntiles - K2_STAGES); i < ntiles; ++i)
            if (lane == 0 && !mbar_wait(&full[i % K2_STAGES], (uint32_t)(i / K2_STAGES) & 1u, kWaitLimit))
                s_timeout = 1;
        __syncwarp();
        if (s_timeout && lane == 0) dev_error(a.err, CSA2_DEV_TIMEOUT);
        return;
    }
    if (wid >= K2_CWARPS) {
        // ================= producers =================
        const int pw = wid - K2_CWARPS;
        const int sh = a.page_shift;
        const int32_t emask = (1 << sh) - 1;
        const uint8_t* rows = a.rows;
        const int rsh = a.rshift;
        const int32_t mpps = a.cache.max_pages_per_seq;
        // rows pw*128 + 32 h + lane of tile t: row index within the sequence
        // (-1 past its end) and physical page, loaded one tile ahead
        int32_t pj[4], pp[4];
        auto fetch = [&](int32_t t) {
            const int b = seq_of_tile(tile_start, a.n, t);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int32_t j = (t - tile_start[b]) * K2_TILE + K2_PROWS * pw + 32 * h + lane;
                const int32_t pg = (j << rsh) >> sh;
                const bool in = j < s_nblk[b];
                pp[h] = (in && pg < mpps) ? __ldg(a.cache.page_table + (int64_t)b * mpps + pg) : -1;
                pj[h] = in ? j : -1;
            }
        };
        fetch(t0);
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % K2_STAGES;
            if (i >= K2_STAGES && !mbar_wait(&empty[s], (uint32_t)((i / K2_STAGES) - 1) & 1u, a.wait_limit))
                s_timeout = 1;
            int32_t prow[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                prow[h] = -1;
                if (pj[h] >= 0) {
                    int32_t phys = pp[h];
                    if (phys < 0 || phys >= a.cache.n_phys_pages) {
                        dev_error(a.err, CSA2_DEV_PAGE);
                        phys = 0;  // results of this call are undefined; the copy stays in bounds
                    }
                    prow[h] = (int32_t)((((int64_t)phys << sh) | ((pj[h] << rsh) & emask)) >> rsh);
                }
            }
            if (i + 1 < ntiles) fetch(t0 + i + 1);  // loads overlap the copies below
            uint8_t* dst0 = smem + (size_t)s * K2_STAGE_BYTES + (size_t)pw * K2_PROWS * 128;
            const int c = lane & 7;
#pragma unroll
            for (int k = 0; k < K2_PROWS / 4; ++k) {
                const int rr = 4 * k + (lane >> 3);  // register h = k / 8 of lane rr & 31 holds its page
                const int32_t v = k < 8 ? prow[0] : k < 16 ? prow[1] : k < 24 ? prow[2] : prow[3];
                const int32_t pr = __shfl_sync(0xffffffffu, v, rr & 31);
                if (pr >= 0)
                    cp_async16(dst0 + rr * 128 + ((c ^ (rr & 7)) << 4), rows + (int64_t)pr * 128 + c * 16);
            }
            cp_async_mbar_arrive(&full[s]);
        }
        cp_async_wait<0>();  // every copy has landed before this thread leaves
        if (s_timeout && lane == 0) dev_error(a.err, CSA2_DEV_TIMEOUT);
        return;
    }

    // ================= consumers =================
    const GroupBar cg{1, K2_CTHREADS};
    int cur_b = -1, nloc = 0;
    auto flush = [&](int b, int nt) {
        cg.sync();
        uint32_t* gh = a.hist + (int64_t)b * kHistBins;
        for (int i = tid; i < kHistBins; i += K2_CTHREADS) {
            const uint32_t v = hist[i];
            if (v) atomicAdd(&gh[i], v);
            hist[i] = 0;
        }
        __threadfence();
        cg.sync();
        if (tid == 0) {
            const int32_t nblk = s_nblk[b];
            const uint32_t need_t = (uint32_t)((nblk + K2_TILE - 1) / K2_TILE);
            s_last = atomicAdd(&a.ctr[2 * b], (uint32_t)nt) + (uint32_t)nt == need_t;
        }
        cg.sync();
        if (s_last) {  // the sequence's last tile is done: find the bin of the keep-th score
            __threadfence();
            for (int i = tid; i < kHistBins / 4; i += K2_CTHREADS)
                reinterpret_cast<uint4*>(hist)[i] = __ldcg(reinterpret_cast<const uint4*>(gh) + i);
            cg.sync();
            for (int i = tid; i < kHistBins / 4; i += K2_CTHREADS)
                reinterpret_cast<uint4*>(gh)[i] = make_uint4(0, 0, 0, 0);
            int bin;
            uint32_t above;
            group_find_kth_bin(hist, kHistBins, (uint32_t)a.keep, tmp, &bin, &above, cg);
            if (tid == 0) {
                a.thr[4 * b] = bin;
                a.thr[4 * b + 1] = (int32_t)above;
                a.ctr[2 * b] = 0;
            }
            for (int i = tid; i < kHistBins; i += K2_CTHREADS) hist[i] = 0;
            cg.sync();
        }
    };

    for (int i = 0; i < ntiles; ++i) {
        const int32_t t = t0 + i;
        const int s = i % K2_STAGES;
        const int b = seq_of_tile(tile_start, a.n, t);
        if (b != cur_b) {
            if (cur_b >= 0) flush(cur_b, nloc);
            load_q_heads(a.q_idx + (int64_t)b * kIH * kID, qd, tid, K2_CTHREADS);
            if (tid == 0) s_w = *reinterpret_cast<const float4*>(a.w + (int64_t)b * kIH);
            cur_b = b;
            nloc = 0;
            cg.sync();
        }
        if (!mbar_wait(&full[s], (uint32_t)(i / K2_STAGES) & 1u, a.wait_limit)) s_timeout = 1;
        const uint8_t* stage = smem + (size_t)s * K2_STAGE_BYTES;
        const int r0 = K2_CROWS * wid + lane;  // rows r0 and r0 + 32 of the tile
        float s0, s1;
        idx_score2_tile(stage, r0, r0 + 32, reinterpret_cast<const ulonglong2*>(qd), s_w, s0, s1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // the warp has read its rows of the stage
        const int32_t j = (t - tile_start[b]) * K2_TILE + r0;
        const int32_t nblk = s_nblk[b];
        float* sc = a.scores + (int64_t)b * a.nblk_pad;
        if (j < nblk) sc[j] = s0;
        if (j + 32 < nblk) sc[j + 32] = s1;
        hist_add(hist, score_key(s0) >> 20, j < nblk);
        hist_add(hist, score_key(s1) >> 20, j + 32 < nblk);
        ++nloc;
    }
    if (cur_b >= 0) flush(cur_b, nloc);
    if (s_timeout && tid == 0) dev_error(a.err, CSA2_DEV_TIMEOUT);
}

// ============================================================================
// K3: block select (filter + last-CTA finalize)
// ============================================================================
constexpr int K3_THREADS = 512;
constexpr int K3_CHUNK = 8192;
constexpr int K3_WORDS = (int)(kMaxBlockLevelLen / kBlk / 32);  // bitmap words for the largest context
constexpr int K3_BND_CAP = 12288;                               // boundary entries held in shared memory
constexpr size_t K3_OFF_LAST = (size_t)2 * K3_WORDS * 4 + 1024 * 4 + 64 * 4 + (size_t)K3_BND_CAP * 8;
constexpr size_t K3_SMEM = K3_OFF_LAST + 16;

// kFlat: rows are entries (several chunks per CTA, bitmaps possibly in global
// memory); otherwise blocks of 8 (one chunk per CTA, bitmaps in shared memory).
template <bool kFlat>
__global__ void __launch_bounds__(K3_THREADS) block_select_kernel(BlockArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int& s_last = *reinterpret_cast<int*>(smem + K3_OFF_LAST);
    pdl_wait();
    pdl_trigger();
    if (smem_u32(smem) & 15u) {  // uniform over the grid
        if (threadIdx.x == 0) dev_error(a.err, CSA2_DEV_ALIGN);
        return;
    }
    const int b = blockIdx.y;
    const int32_t L = seq_len_checked(a.seq_lens, b, a.max_len, a.err);
    const int32_t nblk = L >= 1 ? ((L - 1) >> a.rshift) + 1 : 0;
    int32_t* out = a.out + (int64_t)b * a.keep;
    if (nblk <= a.keep) {
        if (blockIdx.x == 0)
            for (int i = threadIdx.x; i < a.keep; i += K3_THREADS) out[i] = i < nblk ? i : -1;
        return;
    }
    const int32_t span = kFlat ? a.span : K3_CHUNK;
    const int32_t c0 = blockIdx.x * span;
    if (c0 >= nblk) return;
    const int32_t c1 = min(c0 + span, nblk);
    const uint32_t bstar = (uint32_t)__ldcg(&a.thr[4 * b]);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const float* scores = a.scores + (int64_t)b * a.nblk_pad;
    uint32_t* bitmap = a.bitmap + (int64_t)b * (a.nblk_pad >> 5);
    uint64_t* bnd = a.bnd + (int64_t)b * a.nblk_pad;
    constexpr int U = kFlat ? 8 : 4;  // loads in flight per thread
    // Block rows: each warp lists its boundary rows in shared memory (the
    // finalize's bitmaps, unused until then) and the CTA reserves its range of
    // the sequence's boundary list with one atomic, instead of one atomic per
    // ballot on the sequence's counter.
    constexpr int WCAP = K3_CHUNK / (K3_THREADS / 32);  // rows per warp and chunk
    uint64_t* wlist = reinterpret_cast<uint64_t*>(smem) + wid * WCAP;
    uint32_t wn = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int32_t base = c0 + wid * 32; base < c1; base += U * K3_THREADS) {
        float v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int32_t j = base + u * K3_THREADS + lane;
            v[u] = j < c1 ? __ldcg(&scores[j]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int32_t wbase = base + u * K3_THREADS;
            if (wbase >= c1) break;
            const int32_t j = wbase + lane;
            const uint32_t key = score_key(v[u]);
            const uint32_t bin = key >> 20;
            const unsigned mgt = __ballot_sync(0xffffffffu, j < c1 && bin > bstar);
            const unsigned meq = __ballot_sync(0xffffffffu, j < c1 && bin == bstar);
            if (lane == 0) bitmap[wbase >> 5] = mgt;
            if (kFlat && mgt) {  // fewer than keep rows lie above the K-th's bin: list them too
                const int leader = __ffs(mgt) - 1;
                uint32_t pos = 0;
                if (lane == leader) pos = atomicAdd(&a.abv_cnt[b], (uint32_t)__popc(mgt));
                pos = __shfl_sync(0xffffffffu, pos, leader);
                const uint32_t at = pos + __popc(mgt & ((1u << lane) - 1u));
                if (((mgt >> lane) & 1u) && at < (uint32_t)kMaxTopk) a.abv[(int64_t)b * kMaxTopk + at] = j;
            }
            if (!kFlat) {
                if ((meq >> lane) & 1u) wlist[wn + __popc(meq & lt)] = ((uint64_t)key << 32) | (uint64_t)j;
                wn += __popc(meq);
            } else if (meq) {
                const int leader = __ffs(meq) - 1;
                uint32_t pos = 0;
                if (lane == leader) pos = atomicAdd(&a.bnd_cnt[b], (uint32_t)__popc(meq));
                pos = __shfl_sync(0xffffffffu, pos, leader);
                if ((meq >> lane) & 1u) bnd[pos + __popc(meq & lt)] = ((uint64_t)key << 32) | (uint64_t)j;
            }
        }
    }
    if (!kFlat) {  // one reservation per CTA, then each warp copies its list
        uint32_t* ftmp = reinterpret_cast<uint32_t*>(smem) + 2 * K3_WORDS + 1024;
        uint32_t n_cta;
        const uint32_t woff = __shfl_sync(
            0xffffffffu, block_excl_scan(lane == 0 ? wn : 0u, ftmp, &n_cta), 0);
        if (threadIdx.x == 0) ftmp[63] = n_cta ? atomicAdd(&a.bnd_cnt[b], n_cta) : 0u;
        __syncthreads();
        const uint32_t at = ftmp[63] + woff;
        for (uint32_t i = lane; i < wn; i += 32) bnd[at + i] = wlist[i];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t nch = (uint32_t)((nblk + span - 1) / span);
        s_last = atomicAdd(&a.ctr[2 * b + 1], 1u) == nch - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- finalize: exact threshold inside the boundary bin -----------------
    // The row bitmap and the tie bitmap live in shared memory when they fit
    // (every block-level context); a flat selection over more rows works on
    // the sequence's bitmap in global memory and a tie bitmap beside it.
    const int nwords = (nblk + 31) >> 5;
    const bool gm = kFlat && nwords > K3_WORDS;
    uint32_t* sm_bm = reinterpret_cast<uint32_t*>(smem);
    uint32_t* hist = sm_bm + 2 * K3_WORDS;
    uint32_t* tmp = hist + 1024;
    uint64_t* sbnd = reinterpret_cast<uint64_t*>(tmp + 64);
    uint32_t* bm = gm ? bitmap : sm_bm;
    uint32_t* tie = gm ? a.tie + (int64_t)b * (a.nblk_pad >> 5) : sm_bm + K3_WORDS;
    const uint32_t n_bnd = __ldcg(&a.bnd_cnt[b]);
    const uint64_t* B = bnd;
    if (n_bnd <= (uint32_t)K3_BND_CAP) {  // stage the boundary list (the common case)
        load_words(reinterpret_cast<uint32_t*>(sbnd), reinterpret_cast<const uint32_t*>(bnd), 2 * (int)n_bnd);
        B = sbnd;
    }
    if (!gm) {
        load_words(bm, bitmap, nwords);
        for (int i = threadIdx.x; i < nwords; i += K3_THREADS) tie[i] = 0;
    } else {  // 16-byte groups: a sequence's bitmaps are 1 KiB aligned, padded to 256 words
        for (int i = threadIdx.x; i < (nwords + 3) / 4; i += K3_THREADS)
            reinterpret_cast<uint4*>(tie)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t need = (uint32_t)a.keep - (uint32_t)__ldcg(&a.thr[4 * b + 1]);
    int d2, d3;
    uint32_t above;
    for (int i = threadIdx.x; i < 1024; i += K3_THREADS) hist[i] = 0;
    __syncthreads();
    for (int base = wid * 32; base < (int)n_bnd; base += K3_THREADS) {
        const int i = base + lane;
        const uint32_t key = i < (int)n_bnd ? (uint32_t)(B[i] >> 32) : 0u;
        hist_add(hist, (key >> 10) & 1023u, i < (int)n_bnd);
    }
    __syncthreads();
    find_kth_bin(hist, 1024, need, tmp, &d2, &above);
    need -= above;
    const uint32_t nb2 = hist[d2];  // boundary rows in the second digit's bin
    const uint32_t hi22 = (bstar << 20) | ((uint32_t)d2 << 10);
    uint32_t T;
    if (hi22 > 0u && nb2 == need) {  // the bin is taken whole: T just below it, no ties
        T = hi22 - 1u;
        need = 0u;
    } else if (nb2 <= 32u) {  // one warp ranks the bin's keys
        uint32_t* bk = hist;  // [32] keys (the histogram is read), counter at tmp[55]
        if (threadIdx.x == 0) tmp[55] = 0u;
        __syncthreads();  // every thread has read hist[d2]
        for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS) {
            const uint32_t key = (uint32_t)(B[i] >> 32);
            if ((key >> 10) == (hi22 >> 10)) bk[atomicAdd(&tmp[55], 1u)] = key;
        }
        __syncthreads();
        if (wid == 0) {  // T = the need-th largest key of the bin
            const bool mine = (uint32_t)lane < nb2;
            const uint32_t kl = mine ? bk[lane] : 0u;
            uint32_t ge = 0;
            for (int j = 0; j < 32; ++j) {
                const uint32_t kj = __shfl_sync(0xffffffffu, kl, j);
                ge += ((uint32_t)j < nb2 && kj >= kl) ? 1u : 0u;
            }
            const uint32_t Tw = __reduce_max_sync(0xffffffffu, mine && ge >= need ? kl : 0u);
            const uint32_t gt = __popc(__ballot_sync(0xffffffffu, mine && kl > Tw));
            if (lane == 0) {
                tmp[53] = Tw;
                tmp[54] = need - gt;
            }
        }
        __syncthreads();
        T = tmp[53];
        need = tmp[54];
    } else {  // the third digit over the bin's rows
        __syncthreads();  // every thread has read hist[d2]
        for (int i = threadIdx.x; i < 1024; i += K3_THREADS) hist[i] = 0;
        __syncthreads();
        for (int base = wid * 32; base < (int)n_bnd; base += K3_THREADS) {
            const int i = base + lane;
            const uint32_t key = i < (int)n_bnd ? (uint32_t)(B[i] >> 32) : 0u;
            hist_add(hist, key & 1023u, i < (int)n_bnd && (int)((key >> 10) & 1023u) == d2);
        }
        __syncthreads();
        find_kth_bin(hist, 1024, need, tmp, &d3, &above);
        need -= above;
        T = hi22 | (uint32_t)d3;
    }
    if (kFlat) {
        // A flat selection takes keep (<= 512) of up to 2^21 rows: list them
        // (the rows above the K-th's bin, the boundary rows above T and the
        // `need` lowest-index ties) and sort the list, instead of scanning the
        // row bitmap.  More than 256 ties take the bitmap scan below.
        uint32_t my_t = 0;
        for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS) my_t += (uint32_t)(B[i] >> 32) == T ? 1u : 0u;
        uint32_t n_tie;
        (void)block_excl_scan(my_t, tmp, &n_tie);
        const uint32_t n_abv = __ldcg(&a.abv_cnt[b]);
        if (n_tie <= 256u && n_abv < (uint32_t)a.keep) {  // uniform over the CTA
            uint32_t* s_sel = sm_bm;         // [1024] selected rows, then the sort's padding
            uint32_t* s_tie = sm_bm + 1024;  // [256] rows tied at T
            uint32_t* s_cnt = sm_bm + 1280;  // boundary rows above T, ties
            if (threadIdx.x == 0) {
                s_cnt[0] = 0;
                s_cnt[1] = 0;
            }
            for (uint32_t i = threadIdx.x; i < n_abv; i += K3_THREADS)
                s_sel[i] = (uint32_t)__ldcg(a.abv + (int64_t)b * kMaxTopk + i);
            __syncthreads();
            for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS) {
                const uint64_t v = B[i];
                const uint32_t key = (uint32_t)(v >> 32), j = (uint32_t)v;
                if (key > T) {
                    const uint32_t p = atomicAdd(&s_cnt[0], 1u);
                    if (n_abv + p < 1024u) s_sel[n_abv + p] = j;
                } else if (key == T) {
                    s_tie[atomicAdd(&s_cnt[1], 1u)] = j;
                }
            }
            __syncthreads();
            const uint32_t n_gt = s_cnt[0];
            for (uint32_t t = threadIdx.x; t < n_tie; t += K3_THREADS) {  // rank of a tie among the ties
                const uint32_t j = s_tie[t];
                uint32_t r = 0;
                for (uint32_t u = 0; u < n_tie; ++u) r += s_tie[u] < j ? 1u : 0u;
                if (r < need && n_abv + n_gt + r < 1024u) s_sel[n_abv + n_gt + r] = j;
            }
            const uint32_t m = min(n_abv + n_gt + min(need, n_tie), (uint32_t)K3_THREADS);
            uint32_t P = 1;
            while (P < m) P <<= 1;
            __syncthreads();
            // Bitonic sort, ascending, one value per thread (P <= 512 threads; the
            // rest sort padding among themselves): partners closer than 32 are
            // exchanged by shuffles, farther ones through two alternating
            // shared-memory buffers, one barrier per such stage.
            const uint32_t tid_u = threadIdx.x;
            uint32_t v = tid_u < m ? s_sel[tid_u] : 0xffffffffu;
            uint32_t* xb = sm_bm + 2048;  // [2][512]
            int par = 0;
            for (uint32_t k = 2; k <= P; k <<= 1) {
                for (uint32_t jj = k >> 1; jj > 0; jj >>= 1) {
                    uint32_t o;
                    if (jj >= 32) {
                        xb[par * K3_THREADS + tid_u] = v;
                        __syncthreads();
                        o = xb[par * K3_THREADS + (tid_u ^ jj)];
                        par ^= 1;
                    } else {
                        o = __shfl_xor_sync(0xffffffffu, v, (int)jj);
                    }
                    v = (((tid_u & jj) == 0) == ((tid_u & k) == 0)) ? min(v, o) : max(v, o);
                }
            }
            s_sel[tid_u] = v;
            __syncthreads();
            for (int i = threadIdx.x; i < a.keep; i += K3_THREADS) out[i] = (uint32_t)i < m ? (int32_t)s_sel[i] : -1;
            if (threadIdx.x == 0) {
                a.bnd_cnt[b] = 0;
                a.abv_cnt[b] = 0;
                a.ctr[2 * b + 1] = 0;
            }
            return;
        }
    }
    for (uint32_t i = threadIdx.x; i < n_bnd; i += K3_THREADS) {
        const uint64_t v = B[i];
        const uint32_t key = (uint32_t)(v >> 32), j = (uint32_t)v;
        if (key > T) atomicOr(&bm[j >> 5], 1u << (j & 31));
        else if (key == T) atomicOr(&tie[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    // Ordered emission, K3_WORDS words at a time: global bitmaps are staged
    // into shared memory chunk by chunk with coalesced loads (the bitmaps that
    // live in shared memory are one chunk).  Ties are taken lowest index first
    // across chunks.
    uint32_t rank0 = 0, base0 = 0;  // ties and selected entries of the chunks before
    for (int c0w = 0; c0w < nwords; c0w += K3_WORDS) {
        const int cn = min(K3_WORDS, nwords - c0w);
        uint32_t* cbm = sm_bm;
        uint32_t* ctie = sm_bm + K3_WORDS;
        if (gm) {
            __syncthreads();  // the previous chunk is no longer read
            constexpr int V = K3_WORDS / 4 / K3_THREADS;  // 16-byte loads per thread and bitmap
            const uint4* gb = reinterpret_cast<const uint4*>(bm + c0w);
            const uint4* gt = reinterpret_cast<const uint4*>(tie + c0w);
            uint4 vb[V], vt[V];
#pragma unroll
            for (int k = 0; k < V; ++k) {  // all loads in flight at once
                const int i = threadIdx.x + k * K3_THREADS;
                vb[k] = 4 * i < cn ? __ldcg(gb + i) : make_uint4(0u, 0u, 0u, 0u);
                vt[k] = 4 * i < cn ? __ldcg(gt + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const int i = threadIdx.x + k * K3_THREADS;
                reinterpret_cast<uint4*>(cbm)[i] = vb[k];
                reinterpret_cast<uint4*>(ctie)[i] = vt[k];
            }
            __syncthreads();
        }
        uint32_t n_ties, n_sel;
        if (gm) {  // long chunks (flat selections): warp-ordered, conflict-free reads
            // warp v owns words [lo, hi) of the chunk; lane l takes words lo + 32 k + l,
            // so shared-memory reads are conflict-free and warp scans give the order
            const int pw = ((cn + K3_THREADS / 32 - 1) / (K3_THREADS / 32) + 31) & ~31;
            const int lo = wid * pw, hi = min(cn, lo + pw);
            uint32_t w_ties = 0;
            for (int i0 = lo; i0 < hi; i0 += 32) {
                const int i = i0 + lane;
                w_ties += __popc(i < hi ? ctie[i] : 0u);
            }
            for (int o = 16; o > 0; o >>= 1) w_ties += __shfl_xor_sync(0xffffffffu, w_ties, o);
            uint32_t rank = rank0 + __shfl_sync(0xffffffffu, block_excl_scan(lane == 0 ? w_ties : 0u, tmp, &n_ties), 0);
            uint32_t w_sel = 0;
            for (int i0 = lo; i0 < hi; i0 += 32) {
                const int i = i0 + lane;
                uint32_t t = i < hi ? ctie[i] : 0u;
                const uint32_t c = __popc(t);
                const uint32_t incl = warp_incl_scan(c);
                const uint32_t r = rank + incl - c;  // ties before this word, in entry order
                uint32_t take = r >= need ? 0u : min(c, need - r), kept = 0;
                while (take--) {  // the lowest-index ties of the word
                    const uint32_t lb = t & (0u - t);
                    kept |= lb;
                    t ^= lb;
                }
                if (i < hi) {
                    cbm[i] |= kept;
                    w_sel += __popc(cbm[i]);
                }
                rank += __shfl_sync(0xffffffffu, incl, 31);
            }
            for (int o = 16; o > 0; o >>= 1) w_sel += __shfl_xor_sync(0xffffffffu, w_sel, o);
            uint32_t base = base0 + __shfl_sync(0xffffffffu, block_excl_scan(lane == 0 ? w_sel : 0u, tmp, &n_sel), 0);
            for (int i0 = lo; i0 < hi; i0 += 32) {
                const int i = i0 + lane;
                uint32_t m = i < hi ? cbm[i] : 0u;
                const uint32_t c = __popc(m);
                const uint32_t incl = warp_incl_scan(c);
                uint32_t pos = base + incl - c;
                while (m) {
                    const int bit = __ffs(m) - 1;
                    m &= m - 1;
                    if (pos < (uint32_t)a.keep) out[pos] = (c0w + i) * 32 + bit;
                    ++pos;
                }
                base += __shfl_sync(0xffffffffu, incl, 31);
            }
        } else if (cn <= 8 * K3_THREADS) {  // a short chunk (contexts up to 1M): thread t owns words [8t, 8t + 8)
            const int w0 = 8 * threadIdx.x;
            uint32_t wb[8], wt[8];
            if (w0 + 8 <= cn) {  // 16-byte reads (the chunk starts 16-byte aligned)
                const uint4 b0 = reinterpret_cast<const uint4*>(cbm + w0)[0], b1 = reinterpret_cast<const uint4*>(cbm + w0)[1];
                const uint4 t0 = reinterpret_cast<const uint4*>(ctie + w0)[0], t1 = reinterpret_cast<const uint4*>(ctie + w0)[1];
                wb[0] = b0.x; wb[1] = b0.y; wb[2] = b0.z; wb[3] = b0.w; wb[4] = b1.x; wb[5] = b1.y; wb[6] = b1.z; wb[7] = b1.w;
                wt[0] = t0.x; wt[1] = t0.y; wt[2] = t0.z; wt[3] = t0.w; wt[4] = t1.x; wt[5] = t1.y; wt[6] = t1.z; wt[7] = t1.w;
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    wb[k] = w0 + k < cn ? cbm[w0 + k] : 0u;
                    wt[k] = w0 + k < cn ? ctie[w0 + k] : 0u;
                }
            }
            // one scan of (ties, rows above T): fewer than keep <= 2048 rows lie above T
            // (12 bits), at most 2^20 rows tie (20 bits); the ties taken before this
            // thread are min(its tie prefix, need), lowest index first
            uint32_t my_ties = 0, my_above = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                my_ties += __popc(wt[k]);
                my_above += __popc(wb[k]);
            }
            uint32_t tot;
            const uint32_t pre = block_excl_scan((my_ties << 12) | my_above, tmp, &tot);
            const uint32_t tie_base = rank0 + (pre >> 12);
            const uint32_t taken0 = min(rank0, need);  // ties the earlier chunks took
            const uint32_t take = tie_base >= need ? 0u : min(my_ties, need - tie_base);
            uint32_t pos = base0 + (pre & 0xfffu) + min(tie_base, need) - taken0, taken = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint32_t t = wt[k], kept = 0;
                while (t && taken < take) {  // the lowest-index ties
                    const uint32_t lb = t & (0u - t);
                    kept |= lb;
                    t ^= lb;
                    ++taken;
                }
                uint32_t m = wb[k] | kept;
                while (m) {
                    const int bit = __ffs(m) - 1;
                    m &= m - 1;
                    if (pos < (uint32_t)a.keep) out[pos] = (c0w + w0 + k) * 32 + bit;
                    ++pos;
                }
            }
            n_ties = tot >> 12;
            n_sel = (tot & 0xfffu) + min(rank0 + n_ties, need) - taken0;
        } else {  // a longer chunk: thread t owns words [t*per, (t+1)*per)
            const int per = (cn + K3_THREADS - 1) / K3_THREADS;
            const int w0 = threadIdx.x * per, w1 = min(cn, w0 + per);
            uint32_t my_ties = 0;
            for (int i = w0; i < w1; ++i) my_ties += __popc(ctie[i]);
            uint32_t rank = rank0 + block_excl_scan(my_ties, tmp, &n_ties);
            uint32_t my_sel = 0;
            for (int i = w0; i < w1; ++i) {
                uint32_t t = ctie[i], kept = 0;
                while (t && rank < need) {  // the lowest-index ties
                    const uint32_t lb = t & (0u - t);
                    kept |= lb;
                    t ^= lb;
                    ++rank;
                }
                rank += __popc(t);
                cbm[i] |= kept;
                my_sel += __popc(cbm[i]);
            }
            uint32_t base = base0 + block_excl_scan(my_sel, tmp, &n_sel);
            for (int i = w0; i < w1; ++i) {
                uint32_t m = cbm[i];
                while (m) {
                    const int bit = __ffs(m) - 1;
                    m &= m - 1;
                    if (base < (uint32_t)a.keep) out[base] = (c0w + i) * 32 + bit;
                    ++base;
                }
            }
        }
        rank0 += n_ties;
        base0 += n_sel;
    }
    const uint32_t tot = base0;
    for (int i = (int)tot + threadIdx.x; i < a.keep; i += K3_THREADS) out[i] = -1;
    if (threadIdx.x == 0) {
        a.bnd_cnt[b] = 0;
        if (kFlat) a.abv_cnt[b] = 0;
        a.ctr[2 * b + 1] = 0;
    }
}

// ============================================================================
// K4: token scores over the candidates + Top-K, in two kernels.
//
// K4a token_score_kernel: 16 CTAs per sequence; CTA p scores candidate slots
// [1024 p, 1024 p + 1024).  Warp w copies the indexer-K rows of its 8
// candidate blocks (a block's 8 rows are one 1 KiB run) into its own 8 KiB of
// shared memory, as 8-row tensor boxes (128-byte swizzled, counted on the
// warp's barrier) or with 16-byte cp.async into the same layout; lane l then
// scores the warp's rows l and l + 32 with the two-row packed chains.  The
// exact keys go to the workspace, 0 for slots without a candidate.
//
// K4b token_select_kernel: one CTA per sequence; thread t holds keys
// [16 t, 16 t + 16) in registers.  First digit: key >> 16 counted from 1022
// values below the largest key's (lower keys share bin 0), a histogram whose
// atomics spread over hundreds of bins.  The K-th key's bin, taken whole or
// holding at most 32 keys, is resolved by one warp; otherwise (or when the
// K-th key lies in the shared bin 0) a 12-bit digit and two 10-bit digits
// over the shrinking survivor lists find it.  The emission takes two block
// scans (ties at the threshold, then selected counts) and writes each
// thread's positions in slot order.
// ============================================================================
constexpr int TS_PARTS = 16;
constexpr int TS_SLOTS = kMaxCand / TS_PARTS;  // 1024 candidate slots per CTA
constexpr int TS_THREADS = 512;               // two rows per thread
constexpr int TS_BLKS = TS_SLOTS / kBlk;       // 128 candidate blocks per CTA, 8 per warp
constexpr size_t TS_OFF_QP = (size_t)TS_SLOTS * 128;                // rows | q by dimension [64] float4
constexpr size_t TS_OFF_MISC = TS_OFF_QP + kID * 16;                 // w (float4)
constexpr size_t TS_OFF_BAR = TS_OFF_MISC + 16;                      // [16] per-warp copy barriers
constexpr size_t TS_SMEM = TS_OFF_BAR + (TS_THREADS / 32) * 8;
static_assert(TS_BLKS == 8 * (TS_THREADS / 32), "K4a: 8 candidate blocks per warp");

constexpr int TK_THREADS = 1024;
constexpr int TK_PER = kMaxCand / TK_THREADS;                        // 16 keys per thread
constexpr size_t TK_OFF_KEYS = 0;                                   // [16384] u32
constexpr size_t TK_OFF_HIST = TK_OFF_KEYS + (size_t)kMaxCand * 4;   // [4096] u32
constexpr size_t TK_OFF_L0 = TK_OFF_HIST + kHistBins * 4;            // [16384] u16
constexpr size_t TK_OFF_L1 = TK_OFF_L0 + (size_t)kMaxCand * 2;       // [16384] u16
constexpr size_t TK_OFF_TMP = TK_OFF_L1 + (size_t)kMaxCand * 2;      // [64] u32
constexpr size_t TK_OFF_BK = TK_OFF_TMP + 64 * 4;                    // [32] u32 keys of the K-th bin
constexpr size_t TK_SMEM = TK_OFF_BK + 32 * 4;
static_assert(kMaxCand == kMaxKeep * kBlk && TK_PER % 4 == 0, "K4b shared-memory layout");

// The earlier (non-cluster) layout constants are still used by the prefill select.
constexpr size_t K4_OFF_HIST = (size_t)kMaxCand * 4;
constexpr size_t K4_OFF_L0 = K4_OFF_HIST + kHistBins * 4;
constexpr size_t K4_OFF_L1 = K4_OFF_L0 + (size_t)kMaxCand * 2;
constexpr size_t K4_OFF_CB = K4_OFF_L1 + (size_t)kMaxCand * 2;

struct TokenArgs {
    csa2_kv_cache cache;
    const uint16_t* q_idx;
    const float* w;
    const int32_t* seq_lens;
    const int32_t* cand;  // [n][keep] or null (flat)
    int32_t* out;         // [n][topk]
    uint32_t* keys;       // [n][16384] exact keys, K4a -> K4b
    int32_t* err;
    int64_t max_len;
    int keep, topk, page_shift;
    int pre;  // 1: the lengths, cand and the cache may be read before the preceding kernel completes
    int tma;  // 1: candidate blocks arrive as 8-row tensor boxes (else 16-byte cp.async)
};

// Candidate slot range [s0, s1) of a CTA holding `span` slots from s0, and the
// first position of candidate block k of the sequence (-1: none).
struct TokenSlots {
    int32_t L;
    int s0, s1;
    __device__ TokenSlots(const TokenArgs& a, int b, int part, int span, bool report) {
        L = seq_len_checked(a.seq_lens, b, a.max_len, report ? a.err : nullptr);
        const int32_t cap = a.keep * kBlk;
        const int nslots = a.cand ? cap : min(L, cap);
        if (!a.cand && L > cap && report && threadIdx.x == 0) dev_error(a.err, CSA2_DEV_LEN);
        s0 = part * span;
        s1 = max(s0, min(s0 + span, nslots));
    }
    __device__ int32_t block_pos(const TokenArgs& a, int b, int i) const {  // i: first slot of the block
        if (i >= s1) return -1;
        const int32_t blk = a.cand ? __ldg(a.cand + (int64_t)b * a.keep + (i >> 3)) : (i >> 3);
        return (blk >= 0 && blk * kBlk < L) ? blk * kBlk : -1;
    }
};

__global__ void __launch_bounds__(TS_THREADS, 1)
    token_score_kernel(const __grid_constant__ CUtensorMap tmap, TokenArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    float4* qp = reinterpret_cast<float4*>(smem + TS_OFF_QP);
    float4& s_w = *reinterpret_cast<float4*>(smem + TS_OFF_MISC);
    const int part = blockIdx.x % TS_PARTS;
    const int b = blockIdx.x / TS_PARTS;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

    // With a.pre (a Reindex layer inside the decode driver: its candidates come
    // from the Full layer, launches back) the candidates' slots are resolved
    // and their rows copied before waiting on the preceding kernel; q_idx and
    // w, which a model computes from the previous layer's output, are read
    // after the wait.
    const bool pre = a.pre != 0;
    if (!pre) {
        pdl_wait();
        pdl_trigger();
    }
    // 16-byte copies need a 16-byte aligned base, 128-byte-swizzled tensor
    // boxes a 1 KiB aligned one (uniform over the grid)
    if (smem_u32(smem) & (a.tma ? 1023u : 15u)) {
        if (pre) pdl_wait();
        if (tid == 0 && part == 0) dev_error(a.err, CSA2_DEV_ALIGN);
        return;
    }
    const TokenSlots ts(a, b, part, TS_SLOTS, part == 0);
    // warp w: candidate blocks 8 w + j (lane j < 8 resolves one), rows 64 w ..
    uint8_t* wrows = smem + (size_t)wid * 64 * 128;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + TS_OFF_BAR) + wid;
    int32_t mypos = -1;
    int64_t myslot = -1;
    if (lane < 8) {
        const int32_t p = ts.block_pos(a, b, ts.s0 + (8 * wid + lane) * kBlk);
        if (p >= 0) {
            myslot = entry_slot(a.cache, a.page_shift, b, p, a.err);
            mypos = myslot >= 0 ? p : -1;
        }
    }
    if (a.tma) {
        if (lane == 0) {
            mbar_init(bar, 1);  // lane 0's expect-tx arrival
            fence_mbar_init();
        }
        const unsigned m = __ballot_sync(0xffffffffu, myslot >= 0);
        if (lane == 0) mbar_arrive_expect_tx(bar, 1024u * (uint32_t)__popc(m));
        __syncwarp();
        if (myslot >= 0) tma_load_2d(wrows + lane * 1024, &tmap, 0, (int32_t)myslot, bar);
    } else {
        // lane l moves chunk l & 7 of row 4 j + l / 8 into the swizzled layout
        const uint8_t* idx_k = reinterpret_cast<const uint8_t*>(a.cache.idx_k);
        const int c = lane & 7;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int rr = 4 * j + (lane >> 3);
            const int64_t sl = __shfl_sync(0xffffffffu, myslot, rr >> 3);
            if (sl >= 0) cp_async16(wrows + rr * 128 + ((c ^ (rr & 7)) << 4), idx_k + (sl + (rr & 7)) * 128 + c * 16);
        }
        cp_async_commit();
    }
    if (pre) {
        pdl_wait();
        pdl_trigger();
    }
    load_q_heads(a.q_idx + (int64_t)b * kIH * kID, qp, tid, TS_THREADS);
    if (tid == 0) s_w = *reinterpret_cast<const float4*>(a.w + (int64_t)b * kIH);
    __syncthreads();  // q and w
    if (a.tma) {
        if (!mbar_wait(bar, 0u, kWaitLimit) && lane == 0) dev_error(a.err, CSA2_DEV_TIMEOUT);
    } else {
        cp_async_wait<0>();
    }
    __syncwarp();  // the warp's rows are visible to all its lanes
    const int32_t pA = __shfl_sync(0xffffffffu, mypos, lane >> 3);
    const int32_t pB = __shfl_sync(0xffffffffu, mypos, 4 + (lane >> 3));
    uint32_t kA[32], kB[32];
    read_row(wrows, lane, kA);
    read_row(wrows, lane + 32, kB);
    float sA, sB;
    idx_score2(kA, kB, reinterpret_cast<const ulonglong2*>(qp), s_w, sA, sB);
    uint32_t* keys = a.keys + (int64_t)b * kMaxCand + ts.s0 + 64 * wid;
    keys[lane] = (pA >= 0 && pA + (lane & 7) < ts.L) ? score_key(sA) : 0u;
    keys[lane + 32] = (pB >= 0 && pB + (lane & 7) < ts.L) ? score_key(sB) : 0u;
}

__global__ void __launch_bounds__(TK_THREADS, 1) token_select_kernel(TokenArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + TK_OFF_KEYS);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + TK_OFF_HIST);
    uint16_t* l0 = reinterpret_cast<uint16_t*>(smem + TK_OFF_L0);
    uint16_t* l1 = reinterpret_cast<uint16_t*>(smem + TK_OFF_L1);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(smem + TK_OFF_TMP);
    uint32_t* bk = reinterpret_cast<uint32_t*>(smem + TK_OFF_BK);
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int i = tid; i < 1024; i += TK_THREADS) hist[i] = 0;
    if (tid == 0) tmp[50] = 0u;  // the K-th bin's key count
    pdl_wait();
    pdl_trigger();
    if (smem_u32(smem) & 15u) {  // vector reads need an aligned base (uniform)
        if (tid == 0 && b == 0) dev_error(a.err, CSA2_DEV_ALIGN);
        return;
    }
    // every load at once: the length, the two candidate blocks of this
    // thread's 16 slots (blocks 2t, 2t + 1) and its keys (0: no candidate)
    static_assert(TK_PER == 2 * kBlk, "K4b: two candidate blocks per thread");
    const int32_t Lraw = __ldg(a.seq_lens + b);
    int32_t c0 = 2 * tid, c1 = 2 * tid + 1;
    if (a.cand) {
        c0 = c0 < a.keep ? __ldg(a.cand + (int64_t)b * a.keep + c0) : -1;
        c1 = c1 < a.keep ? __ldg(a.cand + (int64_t)b * a.keep + c1) : -1;
    }
    uint32_t kr[TK_PER];
    uint32_t mx = 0u;
    {
        const uint4* src = reinterpret_cast<const uint4*>(a.keys + (int64_t)b * kMaxCand) + tid * (TK_PER / 4);
#pragma unroll
        for (int j = 0; j < TK_PER / 4; ++j) {
            const uint4 v = __ldcg(src + j);
            kr[4 * j] = v.x;
            kr[4 * j + 1] = v.y;
            kr[4 * j + 2] = v.z;
            kr[4 * j + 3] = v.w;
            reinterpret_cast<uint4*>(keys)[tid * (TK_PER / 4) + j] = v;
        }
#pragma unroll
        for (int j = 0; j < TK_PER; ++j) mx = max(mx, kr[j]);
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) tmp[wid] = mx;
    __syncthreads();
    mx = 0u;
    for (int v = 0; v < TK_THREADS / 32; ++v) mx = max(mx, tmp[v]);
    const uint32_t top16 = mx >> 16;
    const uint32_t base = top16 > 1022u ? top16 - 1022u : 0u;
#pragma unroll
    for (int j = 0; j < TK_PER; ++j) {
        const uint32_t k = kr[j];
        hist_add(hist, (k >> 16) >= base ? (k >> 16) - base : 0u, k != 0u);
    }
    __syncthreads();  // every thread has read tmp; the histogram is complete
    int b1;
    uint32_t above, n_valid;
    group_find_kth_bin(hist, 1024, (uint32_t)a.topk, tmp, &b1, &above, GroupBar{0, TK_THREADS}, &n_valid);
    int32_t* out = a.out + (int64_t)b * a.topk;
    uint32_t kk, T = 0u, need = 0u;  // selected: keys > T and the first `need` keys == T
    if (n_valid <= (uint32_t)a.topk) {
        kk = n_valid;  // every valid candidate: the keys above 0
    } else {
        kk = (uint32_t)a.topk;
        need = kk - above;
        const uint32_t nb = hist[b1];
        const uint32_t hb = base + (uint32_t)b1;  // key >> 16 of the bin's keys (unless the shared bin 0)
        const bool shared0 = b1 == 0 && base > 0u;
        if (!shared0 && hb > 0u && nb == need) {  // the bin is taken whole: T just below it, no ties
            T = (hb << 16) - 1u;
            need = 0u;
        } else if (!shared0 && nb <= 32u) {
#pragma unroll
            for (int j = 0; j < TK_PER; ++j) {
                const uint32_t k = kr[j];
                if (k != 0u && (k >> 16) == hb) bk[atomicAdd(&tmp[50], 1u)] = k;
            }
            __syncthreads();
            if (wid == 0) {  // T = the need-th largest key of the bin
                const bool mine = (uint32_t)lane < nb;
                const uint32_t kl = mine ? bk[lane] : 0u;
                uint32_t ge = 0;
                for (int j = 0; j < 32; ++j) {
                    const uint32_t kj = __shfl_sync(0xffffffffu, kl, j);
                    ge += ((uint32_t)j < nb && kj >= kl) ? 1u : 0u;
                }
                const uint32_t Tw = __reduce_max_sync(0xffffffffu, mine && ge >= need ? kl : 0u);
                const uint32_t gt = __popc(__ballot_sync(0xffffffffu, mine && kl > Tw));
                if (lane == 0) {
                    tmp[51] = Tw;
                    tmp[52] = need - gt;
                }
            }
            __syncthreads();
            T = tmp[51];
            need = tmp[52];
        } else {  // three digits over the whole key
            __syncthreads();  // every thread has read hist[b1]
            for (int i = tid; i < kHistBins; i += TK_THREADS) hist[i] = 0;
            __syncthreads();
#pragma unroll
            for (int j = 0; j < TK_PER; ++j) hist_add(hist, kr[j] >> 20, kr[j] != 0u);
            __syncthreads();
            int g1;
            uint32_t ab;
            find_kth_bin(hist, kHistBins, kk, tmp, &g1, &ab);
            refine_threshold(keys, kMaxCand, (uint32_t)g1, kk - ab, hist, l0, l1, tmp, &T, &need);
        }
    }
    // ---- emission in slot order: one scan of (ties at T, keys above T); the
    // ties taken before this thread are min(its tie prefix, need)
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < TK_PER; ++j) {
        gt += kr[j] > T ? 1u : 0u;
        eq += (kr[j] == T && kr[j] != 0u) ? 1u : 0u;
    }
    uint32_t tot;
    __syncthreads();  // tmp is free
    const uint32_t pre = block_excl_scan((eq << 16) | gt, tmp, &tot);  // both counts < 2^15
    const uint32_t tie_base = pre >> 16;
    const uint32_t take = tie_base >= need ? 0u : min(eq, need - tie_base);
    uint32_t pos = (pre & 0xffffu) + min(tie_base, need), ties = 0;
    const int32_t L = (Lraw >= 1 && Lraw <= a.max_len) ? Lraw : 0;
    const int32_t p0 = (c0 >= 0 && c0 * kBlk < L) ? c0 * kBlk : -1;
    const int32_t p1 = (c1 >= 0 && c1 * kBlk < L) ? c1 * kBlk : -1;
#pragma unroll
    for (int j = 0; j < TK_PER; ++j) {
        const uint32_t k = kr[j];
        const bool tie = k == T && k != 0u;
        if (k > T || (tie && ties < take)) out[pos++] = (j < kBlk ? p0 : p1) + (j & 7);
        ties += tie ? 1u : 0u;
    }
    for (int i = (int)kk + tid; i < a.topk; i += TK_THREADS) out[i] = -1;
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
    uint32_t* keys;    // [T][stride] exact keys (fallback)
    uint16_t* keys16;  // [T][stride] approximate keys (aliases `keys`)
    int32_t* flags;    // [T]: null = every query takes the exact path
    float* kmax;       // [kmax_parts]
    int32_t* err;
    int64_t stride;
    int T, ratio, topk, n_entries, page_shift, kmax_parts;
    int tma_k;         // 1: K5a's entry tiles arrive as 64-row tensor boxes (pages of >= 64 entries)
};

__device__ __forceinline__ int visible(int p, int ratio, int n) { return min((p + 1) / ratio, n); }

constexpr size_t PS_OFF_W = (size_t)kID * PS_E * 4 + (size_t)kID * PS_Q * kIH * 4;
constexpr size_t PS_OFF_VIS = PS_OFF_W + PS_Q * kIH * 4;
constexpr size_t PS_SMEM = PS_OFF_VIS + PS_Q * 4;

// Thread (qi, ei) of a 16 x 16 grid computes queries 2qi, 2qi+1 against entries
// 4ei .. 4ei+3 of the tile: 32 sequential fp32 FMA chains.
__global__ void __launch_bounds__(PS_THREADS) prefill_score_kernel(PrefillArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    float (*kt)[PS_E] = reinterpret_cast<float (*)[PS_E]>(smem);                                      // [d][entry]
    float (*qs)[PS_Q][kIH] = reinterpret_cast<float (*)[PS_Q][kIH]>(smem + (size_t)kID * PS_E * 4);  // [d][q][h]
    float (*ws_)[kIH] = reinterpret_cast<float (*)[kIH]>(smem + PS_OFF_W);
    int* vis = reinterpret_cast<int*>(smem + PS_OFF_VIS);
    pdl_wait();
    pdl_trigger();
    const int q0 = blockIdx.x * PS_Q;
    const int tid = threadIdx.x;
    if (a.flags) {  // exact fallback: only tiles holding a flagged query
        const bool f = tid < PS_Q && q0 + tid < a.T && a.flags[q0 + tid] != 0;
        if (!__syncthreads_or(f)) return;
    }
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
                    const int64_t slot = entry_slot(a.cache, a.page_shift, 0, e, a.err);
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
constexpr size_t PSEL_SMEM = K4_OFF_CB + 64 * 4 + (PSEL_THREADS / 32) * 4;  // keys | hist | list0 | list1 | tmp | flag words

__device__ void prefill_select_one(const PrefillArgs& a, int t, uint8_t* smem) {
    __syncthreads();  // the previous trip's shared memory is no longer read
    const int n = (int)a.stride;
    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + K4_OFF_HIST);
    uint16_t* l0 = reinterpret_cast<uint16_t*>(smem + K4_OFF_L0);
    uint16_t* l1 = reinterpret_cast<uint16_t*>(smem + K4_OFF_L1);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(smem + K4_OFF_CB);
    for (int i = threadIdx.x; i < kHistBins; i += PSEL_THREADS) hist[i] = 0;
    load_words(skeys, a.keys + (int64_t)t * a.stride, n);
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t nv = 0;
    for (int base = wid * 32; base < n; base += PSEL_THREADS) {
        const int i = base + lane;
        const uint32_t k = i < n ? skeys[i] : 0u;
        nv += k != 0u;
        hist_add(hist, k >> 20, k != 0u);
    }
    uint32_t n_valid;
    block_excl_scan(nv, tmp, &n_valid);
    const uint32_t kk = min((uint32_t)a.topk, n_valid);
    int32_t* out = a.out + (int64_t)t * a.topk;
    if (kk == 0) {
        for (int i = threadIdx.x; i < a.topk; i += PSEL_THREADS) out[i] = -1;
        return;
    }
    int b1;
    uint32_t above, T, need;
    find_kth_bin(hist, kHistBins, kk, tmp, &b1, &above);
    refine_threshold(skeys, n, (uint32_t)b1, kk - above, hist, l0, l1, tmp, &T, &need);
    emit_sorted(skeys, n, T, need, kk, a.topk, out, tmp, [](int i) { return (int32_t)i; });
}

// One query per loop trip (grid-stride: with flags the grid is a few CTAs per
// SM and almost every trip ends at the flag).
__global__ void __launch_bounds__(PSEL_THREADS) prefill_select_kernel(PrefillArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    pdl_wait();
    pdl_trigger();
    if (!a.flags) {
        for (int t = blockIdx.x; t < a.T; t += gridDim.x) prefill_select_one(a, t, smem);
        return;
    }
    // exact fallback: this CTA's queries t = blockIdx.x + j gridDim.x, their flags
    // read side by side, chunks of PSEL_THREADS trips
    for (int j0 = 0; blockIdx.x + (int64_t)j0 * gridDim.x < a.T; j0 += PSEL_THREADS) {
        const int64_t tj = blockIdx.x + (int64_t)(j0 + threadIdx.x) * gridDim.x;
        const bool f = tj < a.T && a.flags[tj] != 0;
        const unsigned m = __ballot_sync(0xffffffffu, f);
        __syncthreads();  // the previous chunk's trips no longer read the words below
        uint32_t* words = reinterpret_cast<uint32_t*>(smem + K4_OFF_CB + 64 * 4);
        if ((threadIdx.x & 31) == 0) words[threadIdx.x >> 5] = m;
        __syncthreads();
        for (int w = 0; w < PSEL_THREADS / 32; ++w) {
            uint32_t bits = words[w];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                prefill_select_one(a, (int)(blockIdx.x + (int64_t)(j0 + 32 * w + b) * gridDim.x), smem);
            }
        }
    }
}

// ============================================================================
// Prefill indexer on tensor cores, exact by verification
//
// K5a scores every (query, visible entry) pair on the tensor cores, bf16 x bf16
// -> fp32 (exact products, fp32 sums in the tensor core's order), and writes
// the top 16 bits of each score's order-preserving key.  K5b, one CTA per
// query, takes the entries at or above a 16-bit threshold B as candidates
// (about 800: B from a sample of the keys, or the 768th largest key), rescores
// them with the exact sequential-FMA chain and selects the exact Top-K among
// them; it then checks
// that no other entry can reach that Top-K: every non-candidate's approximate
// score lies below the candidates' 16-bit threshold B, and
// |approximate - exact| <= delta = 2^-12 sum_h |w_h| ||q_h||_1 max|k|, a bound
// several times above the rounding of either sum of 64 exact products.  If
// B + delta >= the K-th exact score, the query is flagged and the exact
// CUDA-core kernels recompute it.  The output is therefore the exact Top-K.
// ============================================================================
constexpr int PT_SPLIT = 2048;    // entries per CTA (grid.y splits the entry range)
constexpr int PT_CAND = 768;      // candidates per query when the threshold comes from every key
constexpr int PT_CAND_MAX = 2048; // more candidates (ties at the 16-bit threshold) -> exact fallback

// K5a on tcgen05: a CTA scores 128 queries (MMA M, one TMEM lane each) against
// its range of entries, 64 at a time (MMA N), all four heads (4 accumulators
// of 64 columns, double-buffered: 512 TMEM columns).
//   warps 0-7  epilogue: warp w reads lane quarter w & 3 of the four
//              accumulators (one query per thread, entries 32 (w >> 2) ..
//              + 31 of the 64) with tcgen05.ld, computes sum_h w_h relu(.)
//              and writes the keys
//   warp 8     producer: each K tile as one 64-row tensor box (pages of >= 64
//              entries) or by cp.async (the canonical 128-byte swizzle either
//              way) into a 6-stage ring; the cp.async path waits for its own
//              copies two tiles behind and fences them for the tensor core
//   warp 9     MMA: one thread issues 16 tcgen05.mma per tile and commits to
//              the tile's "done" and the stage's "empty" barriers
//   warp 10    max |k| of every staged tile (the verification bound)
constexpr int TC_Q = 128;
constexpr int TC_E = 64;
constexpr int TC_STAGES = 6;
constexpr int TC_EPI_WARPS = 8;                      // 2 per TMEM lane quarter, 32 entries of a tile each
constexpr int TC_W_PROD = TC_EPI_WARPS, TC_W_MMA = TC_EPI_WARPS + 1, TC_W_KMAX = TC_EPI_WARPS + 2;
constexpr int TC_THREADS = (TC_EPI_WARPS + 3) * 32;
constexpr size_t TC_OFF_Q = 0;                                          // 4 heads x [128][128 B]
constexpr size_t TC_OFF_K = TC_OFF_Q + (size_t)kIH * TC_Q * 128;        // stages x [64][128 B]
constexpr size_t TC_OFF_BAR = TC_OFF_K + (size_t)TC_STAGES * TC_E * 128;  // full[S] empty[S] done[2] free[2]
constexpr size_t TC_OFF_MISC = TC_OFF_BAR + (2 * TC_STAGES + 4) * 8;    // tmem base, timeout
constexpr size_t TC_OFF_PG = TC_OFF_MISC + 16;                          // physical pages of the entry range
constexpr int TC_MAX_PG = PT_SPLIT / kBlk;                              // pages are >= 8 entries
constexpr size_t TC_SMEM = 120 * 1024;                                  // one CTA per SM: it owns all of TMEM
static_assert(TC_OFF_PG + TC_MAX_PG * 4 <= TC_SMEM && TC_OFF_K % 1024 == 0, "K5a (tcgen05) shared-memory layout");

__global__ void __launch_bounds__(TC_THREADS, 1)
    prefill_tc_score_kernel(const __grid_constant__ CUtensorMap tmap, PrefillArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + TC_OFF_BAR);
    uint64_t* empty = full + TC_STAGES;
    uint64_t* done = empty + TC_STAGES;
    uint64_t* tfree = done + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + TC_OFF_MISC);
    int* s_timeout = reinterpret_cast<int*>(smem + TC_OFF_MISC + 4);
    int32_t* s_pg = reinterpret_cast<int32_t*>(smem + TC_OFF_PG);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int q0 = blockIdx.x * TC_Q;
    const int part = blockIdx.x + gridDim.x * blockIdx.y;
    pdl_wait();
    pdl_trigger();
    if (smem_u32(smem) & 1023u) {  // the swizzled operand tiles need a 1 KiB-aligned base (uniform)
        if (tid == 0) dev_error(a.err, CSA2_DEV_ALIGN);
        return;
    }
    // entry range of this CTA: the split, cut at the largest visibility of its queries
    int max_vis = 0;
    for (int i = lane; i < TC_Q; i += 32)
        if (q0 + i < a.T) max_vis = max(max_vis, visible(a.q_pos[q0 + i], a.ratio, a.n_entries));
    for (int o = 16; o > 0; o >>= 1) max_vis = max(max_vis, __shfl_xor_sync(0xffffffffu, max_vis, o));
    const int e_beg = blockIdx.y * PT_SPLIT, e_end = min(e_beg + PT_SPLIT, max_vis);
    if (e_beg >= e_end) {
        if (tid == 0) a.kmax[part] = 0.f;
        return;
    }
    const int ntile = (e_end - e_beg + TC_E - 1) / TC_E;
    // physical pages of the entries [e_beg, e_end), loaded once (-1: outside the cache)
    const int sh = a.page_shift;
    const int pg0 = e_beg >> sh, npg = ((e_end - 1) >> sh) - pg0 + 1;
    for (int i = tid; i < npg; i += TC_THREADS) {
        const int pg = pg0 + i;
        int32_t phys = pg < a.cache.max_pages_per_seq ? __ldg(a.cache.page_table + pg) : -1;
        if (phys < 0 || phys >= a.cache.n_phys_pages) {
            dev_error(a.err, CSA2_DEV_PAGE);
            phys = -1;
        }
        s_pg[i] = phys;
    }
    // Q of the 128 queries, one 128-byte-swizzled tile per head
    for (int i = tid; i < TC_Q * kIH * 8; i += TC_THREADS) {
        const int q = i >> 5, h = (i >> 3) & 3, c = i & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (q0 + q < a.T) v = __ldg(reinterpret_cast<const uint4*>(a.q_idx + ((int64_t)(q0 + q) * kIH + h) * kID) + c);
        *reinterpret_cast<uint4*>(smem + TC_OFF_Q + (size_t)h * TC_Q * 128 + q * 128 + ((c ^ (q & 7)) << 4)) = v;
    }
    if (tid == 0) {
        for (int s = 0; s < TC_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);  // the MMA commit and the max-|k| warp
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&done[b], 1);
            mbar_init(&tfree[b], TC_EPI_WARPS);  // one arrival per epilogue warp
        }
        *s_timeout = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_proxy_async_smem();  // the Q tiles are read by the tensor core
    if (wid == TC_W_MMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(512)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (wid == TC_W_PROD && a.tma_k) {
        // ============ producer, tensor boxes: a tile's 64 entries lie in one page ============
        if (lane == 0) {
            const int32_t emask = (1 << sh) - 1;
            for (int i = 0; i < ntile; ++i) {
                const int s = i % TC_STAGES, e0 = e_beg + i * TC_E;
                if (i >= TC_STAGES && !mbar_wait(&empty[s], (uint32_t)((i / TC_STAGES) - 1) & 1u, kWaitLimit))
                    *s_timeout = 1;
                int32_t phys = s_pg[(e0 >> sh) - pg0];
                if (phys < 0) phys = 0;  // flagged above; the copy stays in bounds
                mbar_arrive_expect_tx(&full[s], (uint32_t)TC_E * 128u);
                tma_load_2d(smem + TC_OFF_K + (size_t)s * TC_E * 128, &tmap, 0, (phys << sh) | (e0 & emask), &full[s]);
            }
        }
        __syncwarp();
    } else if (wid == TC_W_PROD) {
        // ================= producer =================
        const int32_t emask = (1 << sh) - 1;
        auto issue = [&](int i) {
            const int s = i % TC_STAGES, e0 = e_beg + i * TC_E;
            uint8_t* st = smem + TC_OFF_K + (size_t)s * TC_E * 128;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = lane + 32 * rr, e = e0 + r;
                const int32_t phys = e < e_end ? s_pg[(e >> sh) - pg0] : -1;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint8_t* dst = st + r * 128 + ((c ^ (r & 7)) << 4);
                    if (phys >= 0) cp_async16(dst, a.cache.idx_k + (((int64_t)phys << sh) | (e & emask)) * kID + c * 8);
                    else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
        };
        auto publish = [&](int i) {  // tile i's copies have landed: make them visible to the tensor core
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[i % TC_STAGES]);
        };
        for (int i = 0; i < ntile + 2; ++i) {
            if (i < ntile) {
                if (i >= TC_STAGES &&
                    !mbar_wait(&empty[i % TC_STAGES], (uint32_t)((i / TC_STAGES) - 1) & 1u, kWaitLimit))
                    *s_timeout = 1;
                issue(i);
            }
            cp_async_commit();
            if (i >= 2) {
                cp_async_wait<2>();  // tile i - 2 is in shared memory
                publish(i - 2);
            }
        }
    } else if (wid == TC_W_MMA) {
        // ================= MMA issue =================
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TC_E >> 3) << 17) |
                                   ((uint32_t)(TC_Q >> 4) << 24);  // bf16 x bf16 -> f32, K-major, M 128, N 64
            for (int i = 0; i < ntile; ++i) {
                const int s = i % TC_STAGES, buf = i & 1;
                if (!mbar_wait(&full[s], (uint32_t)(i / TC_STAGES) & 1u, kWaitLimit)) *s_timeout = 1;
                if (i >= 2 && !mbar_wait(&tfree[buf], (uint32_t)((i >> 1) - 1) & 1u, kWaitLimit)) *s_timeout = 1;
                tc_fence_after();
                const uint64_t db = umma_desc_sw128(smem_u32(smem + TC_OFF_K + (size_t)s * TC_E * 128));
#pragma unroll
                for (int h = 0; h < kIH; ++h) {
                    const uint64_t da = umma_desc_sw128(smem_u32(smem + TC_OFF_Q + (size_t)h * TC_Q * 128));
#pragma unroll
                    for (int kk = 0; kk < kID / 16; ++kk)  // +32 B per k-step of 16
                        umma_bf16(tmem + (uint32_t)(buf * kIH * TC_E + h * TC_E), da + 2u * kk, db + 2u * kk, idesc,
                                  kk > 0 ? 1u : 0u);
                }
                umma_commit(&done[buf]);
                umma_commit(&empty[s]);
            }
        }
        __syncwarp();
    } else if (wid == TC_W_KMAX) {
        // ================= max |k| of the staged tiles =================
        uint32_t kmax_bits = 0;
        for (int i = 0; i < ntile; ++i) {
            const int s = i % TC_STAGES, e0 = e_beg + i * TC_E;
            if (!mbar_wait(&full[s], (uint32_t)(i / TC_STAGES) & 1u, kWaitLimit)) *s_timeout = 1;
            const uint8_t* st = smem + TC_OFF_K + (size_t)s * TC_E * 128;
            for (int j = lane; j < TC_E * 8; j += 32) {
                if (e0 + (j >> 3) >= e_end) continue;
                const uint4 v = *reinterpret_cast<const uint4*>(st + j * 16);
                const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) kmax_bits = max(kmax_bits, max(x[u] & 0x7fffu, (x[u] >> 16) & 0x7fffu));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        for (int o = 16; o > 0; o >>= 1) kmax_bits = max(kmax_bits, __shfl_xor_sync(0xffffffffu, kmax_bits, o));
        if (lane == 0) a.kmax[part] = __uint_as_float(kmax_bits << 16);
    } else {
        // ================= epilogue: thread = query = TMEM lane =================
        const int quarter = wid & 3, half = wid >> 2;
        const int ql = 32 * quarter + lane, t = q0 + ql;
        float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
        int vis = 0;
        if (t < a.T) {
            w = *reinterpret_cast<const float4*>(a.w + (int64_t)t * kIH);
            vis = visible(a.q_pos[t], a.ratio, a.n_entries);
        }
        const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
        // (w_h, w_h) pairs: fma.rn.f32x2 rounds each half as the scalar FMA chain over the heads does
        const uint64_t wx2 = pack2(w.x, w.x), wy2 = pack2(w.y, w.y), wz2 = pack2(w.z, w.z), ww2 = pack2(w.w, w.w);
        for (int i = 0; i < ntile; ++i) {
            const int buf = i & 1, e0 = e_beg + i * TC_E;
            if (!mbar_wait(&done[buf], (uint32_t)(i >> 1) & 1u, kWaitLimit)) *s_timeout = 1;
            tc_fence_after();
#pragma unroll 1
            for (int c = 2 * half; c < 2 * half + 2; ++c) {  // this warp's 32 of the 64 entries
                uint32_t v0[16], v1[16], v2[16], v3[16];
                const uint32_t col = lane_base + (uint32_t)(buf * kIH * TC_E + 16 * c);
                tmem_ld16(col, v0);
                tmem_ld16(col + TC_E, v1);
                tmem_ld16(col + 2 * TC_E, v2);
                tmem_ld16(col + 3 * TC_E, v3);
                tmem_wait_ld();
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 16; j += 2) {  // entries j and j + 1 in the halves of packed FMAs
                    const auto relu2 = [](uint32_t lo, uint32_t hi) {
                        return pack2(fmaxf(__uint_as_float(lo), 0.f), fmaxf(__uint_as_float(hi), 0.f));
                    };
                    uint64_t s2 = ffma2(wx2, relu2(v0[j], v0[j + 1]), 0ull);
                    s2 = ffma2(wy2, relu2(v1[j], v1[j + 1]), s2);
                    s2 = ffma2(wz2, relu2(v2[j], v2[j + 1]), s2);
                    s2 = ffma2(ww2, relu2(v3[j], v3[j + 1]), s2);
                    float sa, sb;
                    unpack2(s2, sa, sb);
                    const uint32_t ka = e0 + 16 * c + j < vis ? score_key(sa) >> 16 : 0u;
                    const uint32_t kb = e0 + 16 * c + j + 1 < vis ? score_key(sb) >> 16 : 0u;
                    pk[j >> 1] = ka | (kb << 16);
                }
                if (t < a.T) {
                    uint4* dst = reinterpret_cast<uint4*>(a.keys16 + (int64_t)t * a.stride + e0 + 16 * c);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tfree[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();  // every accumulator has been read
    if (wid == TC_W_MMA) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512) : "memory");
    }
    if (tid == 0 && *s_timeout) dev_error(a.err, CSA2_DEV_TIMEOUT);
}

constexpr int PC_THREADS = 320;                       // 3 rounds of exact rescoring cover 960 candidates
constexpr int PC_CTAS = 4;                            // resident CTAs per SM the layout is sized for
constexpr int PC_CH = (kMaxCand / 8 + PC_THREADS - 1) / PC_THREADS;  // 16-byte chunks of 8 keys per thread (at most)
constexpr int PC_SB = 512;                            // sample histogram: 1/64 binade per bin, 8 binades
constexpr int PC_SAMPLE_CAND = 800;                   // candidates the sample's threshold aims at
constexpr int PC_CAND_LO = 600;                       // fewer -> the threshold from every key instead
// Region A: the visible entries' 16-bit keys while the candidates are chosen;
// afterwards the candidates' exact keys, the select's histogram and lists.
constexpr size_t PC_OFF_K16 = 0;                                   // [16384] u16
constexpr size_t PC_OFF_CK = 0;                                    // [2048] u32
constexpr size_t PC_OFF_HIST = PC_OFF_CK + PT_CAND_MAX * 4;        // [4096] u32
constexpr size_t PC_OFF_L0 = PC_OFF_HIST + kHistBins * 4;          // [2048] u16
constexpr size_t PC_OFF_L1 = PC_OFF_L0 + PT_CAND_MAX * 2;          // [2048] u16
// Region B: the sample histogram, then the sequence's page table.
constexpr size_t PC_OFF_HS = (size_t)kMaxCand * 2;                 // [512] u32, one key per chunk
constexpr size_t PC_OFF_PTAB = PC_OFF_HS;                          // [1536] i32 physical page per page index
constexpr int PC_PTAB = 1536;
// Region C: the histogram of every key, then the candidate list.
constexpr size_t PC_OFF_HE = PC_OFF_PTAB + PC_PTAB * 4;            // [1024] u32
constexpr size_t PC_OFF_CAND = PC_OFF_HE;                          // [2048] u16 candidate entries
constexpr size_t PC_OFF_QD = PC_OFF_CAND + PT_CAND_MAX * 2;        // [64] float4
constexpr size_t PC_OFF_TMP = PC_OFF_QD + kID * 16;                // [64] u32
constexpr size_t PC_OFF_MISC = PC_OFF_TMP + 64 * 4;                // w (float4), l1[4], kmax bits, largest exact key, mbarrier
constexpr size_t PC_SMEM = PC_OFF_MISC + 48;
static_assert(PC_OFF_L1 + PT_CAND_MAX * 2 <= PC_OFF_HS, "K5b region A");
static_assert(PC_SB <= PC_PTAB && 1024 * 4 == PT_CAND_MAX * 2, "K5b regions B and C");
static_assert(54 + PC_THREADS / 32 <= 64, "K5b scratch words");
static_assert(PC_CH * 8 * PC_THREADS >= kMaxCand && PC_CH <= 8 && PC_THREADS % 32 == 0, "K5b key chunks");
static_assert(PC_OFF_QD % 16 == 0 && PC_OFF_MISC % 16 == 0 && PC_OFF_HIST % 16 == 0, "K5b shared-memory layout");
static_assert(PC_CTAS * (PC_SMEM + 1024) <= 228 * 1024, "K5b residency");

// Key j (0..7) of a chunk of eight 16-bit keys.
__device__ __forceinline__ uint32_t chunk_key(const uint4& v, int j) {
    const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
    return (j & 1) ? w >> 16 : w & 0xffffu;
}
// Largest key of a chunk whose first nv entries are visible.
__device__ __forceinline__ uint32_t chunk_max(const uint4& v, int nv) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (j < nv) m = max(m, chunk_key(v, j));
    return m;
}
// Bit j set when key j is >= thr and entry j is visible.  The high key of a
// word is >= thr exactly when the word is >= thr << 16.
__device__ __forceinline__ uint32_t chunk_sel(const uint4& v, uint32_t thr, int nv) {
    const uint32_t th = thr << 16;
    const uint32_t m = (uint32_t)((v.x << 16) >= th) | ((uint32_t)(v.x >= th) << 1) |
                       ((uint32_t)((v.y << 16) >= th) << 2) | ((uint32_t)(v.y >= th) << 3) |
                       ((uint32_t)((v.z << 16) >= th) << 4) | ((uint32_t)(v.z >= th) << 5) |
                       ((uint32_t)((v.w << 16) >= th) << 6) | ((uint32_t)(v.w >= th) << 7);
    return nv >= 8 ? m : m & ((1u << max(nv, 0)) - 1u);
}
// Histogram (top bin = mx) of the visible keys lying dlo..dhi values below mx.
__device__ __forceinline__ void chunk_hist_range(const uint4* k16v, int n_ch, int n_vis, uint32_t mx, uint32_t dlo,
                                                 uint32_t dhi, uint32_t* h) {
    for (int i = threadIdx.x; i < n_ch; i += PC_THREADS) {
        const uint4 v = k16v[i];
        const int nv = n_vis - 8 * i;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t dist = mx - chunk_key(v, j);
            hist_add(h, 1023u - dist, j < nv && dist - dlo <= dhi - dlo);
        }
    }
}

// float value of an order-preserving key (inverse of score_key)
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__global__ void __launch_bounds__(PC_THREADS, PC_CTAS) prefill_candidates_kernel(PrefillArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint4* k16v = reinterpret_cast<uint4*>(smem + PC_OFF_K16);
    uint32_t* ck = reinterpret_cast<uint32_t*>(smem + PC_OFF_CK);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + PC_OFF_HIST);
    uint16_t* l0 = reinterpret_cast<uint16_t*>(smem + PC_OFF_L0);
    uint16_t* l1 = reinterpret_cast<uint16_t*>(smem + PC_OFF_L1);
    uint32_t* hs = reinterpret_cast<uint32_t*>(smem + PC_OFF_HS);
    uint32_t* he = reinterpret_cast<uint32_t*>(smem + PC_OFF_HE);
    int32_t* ptab = reinterpret_cast<int32_t*>(smem + PC_OFF_PTAB);
    uint16_t* cand = reinterpret_cast<uint16_t*>(smem + PC_OFF_CAND);
    float4* qd = reinterpret_cast<float4*>(smem + PC_OFF_QD);
    uint32_t* tmp = reinterpret_cast<uint32_t*>(smem + PC_OFF_TMP);
    float4& s_w = *reinterpret_cast<float4*>(smem + PC_OFF_MISC);
    float* s_l1 = reinterpret_cast<float*>(smem + PC_OFF_MISC + 16);       // [4]
    uint32_t* s_u = reinterpret_cast<uint32_t*>(smem + PC_OFF_MISC + 32);  // kmax bits, largest exact key
    uint64_t* kbar = reinterpret_cast<uint64_t*>(smem + PC_OFF_MISC + 40);  // the keys' bulk copy
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int t = blockIdx.x;
    pdl_wait();
    pdl_trigger();
    const int n_vis = visible(a.q_pos[t], a.ratio, a.n_entries);
    int32_t* out = a.out + (int64_t)t * a.topk;
    if (n_vis <= 0) {
        for (int i = tid; i < a.topk; i += PC_THREADS) out[i] = -1;
        if (tid == 0) a.flags[t] = 0;
        return;
    }
    // query, weights, ||q_h||_1, max |k| over the scoring CTAs
    const uint16_t* qb = a.q_idx + (int64_t)t * kIH * kID;
    for (int d = tid; d < kID; d += PC_THREADS)
        qd[d] = make_float4(bf16_bits_to_f32(qb[d]), bf16_bits_to_f32(qb[kID + d]), bf16_bits_to_f32(qb[2 * kID + d]),
                            bf16_bits_to_f32(qb[3 * kID + d]));
    if (wid < kIH) {
        float v = fabsf(bf16_bits_to_f32(qb[wid * kID + lane])) + fabsf(bf16_bits_to_f32(qb[wid * kID + 32 + lane]));
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) s_l1[wid] = v;
    }
    if (wid == kIH) {
        uint32_t m = 0;
        for (int i = lane; i < a.kmax_parts; i += 32) m = max(m, __float_as_uint(a.kmax[i]));
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_u[0] = m;
    }
    if (tid == 0) {
        s_w = *reinterpret_cast<const float4*>(a.w + (int64_t)t * kIH);
        s_u[1] = 0u;
    }
    // the visible entries' 16-bit keys, 8 to a 16-byte chunk: one bulk copy
    // (rows are 128 B aligned)
    const int n_ch = (n_vis + 7) >> 3;
    if (tid == 0) {
        mbar_init(kbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(kbar, (uint32_t)n_ch * 16u);
        bulk_load(k16v, a.keys16 + (int64_t)t * a.stride, (uint32_t)n_ch * 16u, kbar);
    }
    const bool limited = n_vis > PT_CAND;
    __syncthreads();  // the barrier is initialised; query and weights are staged
    if (!mbar_wait(kbar, 0u, kWaitLimit)) {
        if (tid == 0) {
            dev_error(a.err, CSA2_DEV_TIMEOUT);
            a.flags[t] = 1;
        }
        mbar_wait(kbar, 0u, kWaitLimit);  // the copy may still land: bounded second wait
        return;
    }

    // ---- candidates: entries whose 16-bit key is >= thr16.  A histogram of
    // one key per chunk (entry 8i), counted from the sample's largest key,
    // puts thr16 at the lower edge of the bin that holds the sample's key of
    // the rank about PC_SAMPLE_CAND keys clear.  When the count falls outside
    // [PC_CAND_LO, PT_CAND_MAX], or the sample has too few keys within 8
    // binades of its largest, thr16 is the PT_CAND-th largest key instead, from
    // a histogram of every key within 8 binades of the row's largest (a row
    // whose PT_CAND-th key lies lower takes the exact fallback).  Any threshold
    // is sound: the candidates' Top-K is verified below against the best score
    // a non-candidate can reach.
    uint32_t thr16 = 0u;
    bool sampled = false, need_exact = false;
    if (limited) {
        for (int i = tid; i < PC_SB; i += PC_THREADS) hs[i] = 0;
        uint32_t smp[PC_CH];
        uint32_t smx = 0;
#pragma unroll
        for (int c = 0; c < PC_CH; ++c) {
            const int i = tid + c * PC_THREADS;
            smp[c] = i < n_ch ? (reinterpret_cast<const uint32_t*>(k16v)[4 * i] & 0xffffu) : 0u;  // entry 8i
            smx = max(smx, smp[c]);
        }
        smx = __reduce_max_sync(0xffffffffu, smx);
        if (lane == 0) tmp[wid] = smx;
        __syncthreads();
        smx = 0;
        for (int v = 0; v < PC_THREADS / 32; ++v) smx = max(smx, tmp[v]);
#pragma unroll
        for (int c = 0; c < PC_CH; ++c) {
            const uint32_t dist = smx - smp[c];
            hist_add(hs, (PC_SB - 1) - (dist >> 1), tid + c * PC_THREADS < n_ch && dist < 1024u);
        }
        __syncthreads();
        const uint32_t ks = (uint32_t)(((int64_t)PC_SAMPLE_CAND * n_ch + n_vis - 1) / n_vis);
        int b;
        uint32_t above, counted;
        group_find_kth_bin(hs, PC_SB, ks, tmp, &b, &above, GroupBar{0, PC_THREADS}, &counted);
        if (counted >= ks) {
            thr16 = smx - (2u * (uint32_t)(PC_SB - 1 - b) + 1u);
            sampled = true;
        } else {
            need_exact = true;
        }
    }
    // the sample histogram is read: region B takes the page table (loads in
    // flight through the compaction)
    const int n_pg = min(((n_vis - 1) >> a.page_shift) + 1, PC_PTAB);
    for (int j = tid; j < n_pg; j += PC_THREADS)
        ptab[j] = j < a.cache.max_pages_per_seq ? __ldg(a.cache.page_table + j) : -1;
    // thr16 = the PT_CAND-th largest key within 8 binades of the maximum;
    // false (and the row flagged) when fewer keys lie there
    auto exact_threshold = [&]() -> bool {
        uint32_t mx = 0;
        for (int i = tid; i < n_ch; i += PC_THREADS) mx = max(mx, chunk_max(k16v[i], n_vis - 8 * i));
        for (int i = tid; i < 1024; i += PC_THREADS) he[i] = 0;
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) tmp[54 + wid] = mx;
        __syncthreads();
        mx = 0;
        for (int v = 0; v < PC_THREADS / 32; ++v) mx = max(mx, tmp[54 + v]);
        chunk_hist_range(k16v, n_ch, n_vis, mx, 0u, 1023u, he);
        __syncthreads();
        int b;
        uint32_t above, counted;
        group_find_kth_bin(he, 1024, PT_CAND, tmp, &b, &above, GroupBar{0, PC_THREADS}, &counted);
        if (counted < (uint32_t)PT_CAND) {
            if (tid == 0) a.flags[t] = 1;
            return false;
        }
        thr16 = mx - (1023u - (uint32_t)b);
        return true;
    };
    if (need_exact && !exact_threshold()) return;

    // ---- compaction in entry order (the output must come out ascending):
    // lane l of warp v owns a contiguous run of cpl chunks (16-byte reads
    // 16 * cpl bytes apart, distinct banks within each 8-lane phase); the
    // counting pass keeps each chunk's 8-bit selection mask for the writing
    // pass, which needs one prefix over the lanes and warps
    const int cpw = ((n_ch + PC_THREADS / 32 - 1) / (PC_THREADS / 32) + 31) & ~31;
    const int cpl = cpw >> 5;
    const int c0 = wid * cpw + lane * cpl;
    uint32_t mlo = 0, mhi = 0, off = 0;
    int m = 0;
    auto count_pass = [&]() {
        uint32_t mine = 0;
        mlo = 0;
        mhi = 0;
#pragma unroll
        for (int s = 0; s < PC_CH; ++s) {
            const int i = c0 + s;
            uint32_t mk = 0;
            if (s < cpl && i < n_ch) mk = chunk_sel(k16v[i], thr16, n_vis - 8 * i);
            mine += __popc(mk);
            if (s < 4) mlo |= mk << (8 * s);
            else mhi |= mk << (8 * (s - 4));
        }
        const uint32_t inc = warp_incl_scan(mine);
        if (lane == 31) tmp[wid] = inc;
        __syncthreads();
        uint32_t tot = 0;
        off = inc - mine;
        for (int v = 0; v < PC_THREADS / 32; ++v) {
            if (v < wid) off += tmp[v];
            tot += tmp[v];
        }
        m = (int)tot;
    };
    count_pass();
    if (sampled && (m < PC_CAND_LO || m > PT_CAND_MAX)) {
        if (!exact_threshold()) return;
        count_pass();
    }
    if (m > PT_CAND_MAX) {  // too many ties at the 16-bit threshold: exact fallback
        if (tid == 0) a.flags[t] = 1;
        return;
    }
#pragma unroll
    for (int s = 0; s < PC_CH; ++s) {
        uint32_t mk = (s < 4 ? mlo >> (8 * s) : mhi >> (8 * (s - 4))) & 0xffu;
        while (mk) {
            cand[off++] = (uint16_t)(8 * (c0 + s) + __ffs(mk) - 1);
            mk &= mk - 1u;
        }
    }
    __syncthreads();

    // ---- exact scores of the candidates (the oracle's sequential FMA chains)
    // and the largest of them
    const float4 w = s_w;
    const int64_t pmask = (int64_t(1) << a.page_shift) - 1;
    uint32_t cmx = 0u;
    for (int i = tid; i < m; i += PC_THREADS) {
        const int e = cand[i];
        int64_t slot;
        if ((e >> a.page_shift) < n_pg) {
            const int32_t phys = ptab[e >> a.page_shift];
            if (phys < 0 || phys >= a.cache.n_phys_pages) {
                dev_error(a.err, CSA2_DEV_PAGE);
                slot = -1;
            } else {
                slot = ((int64_t)phys << a.page_shift) | ((int64_t)e & pmask);
            }
        } else {
            slot = entry_slot(a.cache, a.page_shift, 0, e, a.err);
        }
        uint32_t key = 0u;
        if (slot >= 0) {
            uint32_t kr[32];
            const uint4* src = reinterpret_cast<const uint4*>(a.cache.idx_k + slot * kID);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = __ldg(src + c);
                kr[4 * c] = v.x;
                kr[4 * c + 1] = v.y;
                kr[4 * c + 2] = v.z;
                kr[4 * c + 3] = v.w;
            }
            key = score_key(idx_score1(kr, qd, w));
        }
        ck[i] = key;
        cmx = max(cmx, key);
    }
    for (int i = tid; i < 1024; i += PC_THREADS) hist[i] = 0;
    cmx = __reduce_max_sync(0xffffffffu, cmx);
    if (lane == 0) atomicMax(&s_u[1], cmx);
    __syncthreads();

    // ---- exact Top-K among the candidates.  First digit: key >> 16 counted
    // from 1022 values below the largest key's (lower keys share bin 0).  The
    // K-th key's bin, taken whole or holding at most 32 keys, is resolved by
    // one warp; otherwise (or when the K-th key lies in the shared bin 0) the
    // three-digit radix select over the whole key finds it.
    const uint32_t top16 = s_u[1] >> 16;
    const uint32_t base = top16 > 1022u ? top16 - 1022u : 0u;
    for (int i = tid; i < m; i += PC_THREADS) {
        const uint32_t k = ck[i];
        hist_add(hist, (k >> 16) >= base ? (k >> 16) - base : 0u, k != 0u);
    }
    __syncthreads();
    int b1;
    uint32_t above, n_valid;
    group_find_kth_bin(hist, 1024, (uint32_t)a.topk, tmp, &b1, &above, GroupBar{0, PC_THREADS}, &n_valid);
    if (n_valid == 0u) {
        for (int i = tid; i < a.topk; i += PC_THREADS) out[i] = -1;
        if (tid == 0) a.flags[t] = 0;
        return;
    }
    uint32_t kk, T = 0u, need = 0u;
    if (n_valid <= (uint32_t)a.topk) {
        kk = n_valid;  // every valid candidate: the keys above 0
        if (limited) {  // a non-candidate may belong to the Top-K
            if (tid == 0) a.flags[t] = 1;
            return;
        }
    } else {
        kk = (uint32_t)a.topk;
        need = kk - above;
        const uint32_t nb = hist[b1];
        const uint32_t hb = base + (uint32_t)b1;  // key >> 16 of the bin's keys (unless the shared bin 0)
        const bool shared0 = b1 == 0 && base > 0u;
        if (!shared0 && hb > 0u && nb == need) {  // the bin is taken whole: T just below it, no ties
            T = (hb << 16) - 1u;
            need = 0u;
        } else if (!shared0 && nb <= 32u) {
            uint32_t* bk = reinterpret_cast<uint32_t*>(l0);  // the bin's keys
            if (tid == 0) tmp[50] = 0u;
            __syncthreads();
            for (int i0 = wid * 32; i0 < m; i0 += PC_THREADS) {
                const int i = i0 + lane;
                const uint32_t k = i < m ? ck[i] : 0u;
                const bool in = k != 0u && (k >> 16) == hb;
                const unsigned bm = __ballot_sync(0xffffffffu, in);
                if (bm) {
                    const int leader = __ffs(bm) - 1;
                    uint32_t pos = 0;
                    if (lane == leader) pos = atomicAdd(&tmp[50], (uint32_t)__popc(bm));
                    pos = __shfl_sync(0xffffffffu, pos, leader);
                    if (in) bk[pos + __popc(bm & ((1u << lane) - 1u))] = k;
                }
            }
            __syncthreads();
            if (wid == 0) {  // T = the need-th largest key of the bin
                const bool mine = (uint32_t)lane < nb;
                const uint32_t kl = mine ? bk[lane] : 0u;
                uint32_t ge = 0;
                for (int j = 0; j < 32; ++j) {
                    const uint32_t kj = __shfl_sync(0xffffffffu, kl, j);
                    ge += ((uint32_t)j < nb && kj >= kl) ? 1u : 0u;
                }
                const uint32_t Tw = __reduce_max_sync(0xffffffffu, mine && ge >= need ? kl : 0u);
                const uint32_t gt = __popc(__ballot_sync(0xffffffffu, mine && kl > Tw));
                if (lane == 0) {
                    tmp[51] = Tw;
                    tmp[52] = need - gt;
                }
            }
            __syncthreads();
            T = tmp[51];
            need = tmp[52];
        } else {
            __syncthreads();  // every thread has read hist[b1]
            for (int i = tid; i < kHistBins; i += PC_THREADS) hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < m; i += PC_THREADS) hist_add(hist, ck[i] >> 20, ck[i] != 0u);
            __syncthreads();
            int g1;
            uint32_t ab;
            find_kth_bin(hist, kHistBins, kk, tmp, &g1, &ab);
            refine_threshold(ck, m, (uint32_t)g1, kk - ab, hist, l0, l1, tmp, &T, &need);
        }
    }
    // ---- no entry outside the candidates can reach the K-th exact score
    if (limited) {
        const double bound = (double)key_value(thr16 << 16);  // non-candidates score below this (approximately)
        const double delta = 0x1p-12 * (fabs((double)w.x) * s_l1[0] + fabs((double)w.y) * s_l1[1] +
                                        fabs((double)w.z) * s_l1[2] + fabs((double)w.w) * s_l1[3]) *
                             (double)__uint_as_float(s_u[0]);
        if (kk < (uint32_t)a.topk || !(bound + delta < (double)key_value(T))) {
            if (tid == 0) a.flags[t] = 1;
            return;
        }
    }
    emit_sorted(ck, m, T, need, kk, a.topk, out, tmp, [&](int i) { return (int32_t)cand[i]; });
    if (tid == 0) a.flags[t] = 0;
}

// ============================================================================
// host side
// ============================================================================
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// One layout for both levels: the small arrays that must start at zero come
// first, so a workspace zero-filled once stays valid for any mix of calls with
// the same (n, max_len).
DecodeWs decode_ws_layout(int n, int64_t max_len, bool flat) {
    DecodeWs l{};
    size_t o = 0;
    const int64_t nrows = flat ? max_len : (max_len + kBlk - 1) / kBlk;  // rows scored per sequence
    l.nblk_pad = (nrows + K3_CHUNK - 1) / K3_CHUNK * K3_CHUNK;
    l.blk_hist = o; o = align256(o + (size_t)n * kHistBins * 4);
    l.blk_ctr = o; o = align256(o + (size_t)n * 8);
    l.blk_bnd_cnt = o; o = align256(o + (size_t)n * 4);
    l.blk_abv_cnt = o; o = align256(o + (size_t)n * 4);
    l.tok_ctr = o; o = align256(o + (size_t)n * 4);
    l.tok_hist = o; o = align256(o + (size_t)n * kHistBins * 4);
    l.blk_thr = o; o = align256(o + (size_t)n * 16);
    l.tok_keys = o; o = align256(o + (size_t)n * kMaxCand * 4);
    l.stage_rows = kMaxTopk;
    l.stage_codes = o; o = align256(o + (size_t)n * l.stage_rows * kCodeBytes);
    l.stage_scales = o; o = align256(o + (size_t)n * l.stage_rows * kScales);
    l.stage_idx = o; o = align256(o + (size_t)n * kMaxTopk * 4);
    l.stage_pt = o; o = align256(o + (size_t)n * 4);
    // the scored rows' arrays (any keep below the row count needs them)
    l.blk_scores = o; o = align256(o + (size_t)n * l.nblk_pad * 4);
    l.blk_bitmap = o; o = align256(o + (size_t)n * (l.nblk_pad / 32) * 4);
    l.blk_bnd = o; o = align256(o + (size_t)n * l.nblk_pad * 8);
    if (flat) {
        l.blk_tie = o; o = align256(o + (size_t)n * (l.nblk_pad / 32) * 4);
        l.blk_abv = o; o = align256(o + (size_t)n * kMaxTopk * 4);
    }
    l.total = o;
    return l;
}

PrefillWs prefill_ws_layout(int T, int64_t n_entries) {
    PrefillWs l{};
    l.stride = (n_entries + PS_E - 1) / PS_E * PS_E;
    l.kmax_parts = (int)(((T + TC_Q - 1) / TC_Q) * ((n_entries + PT_SPLIT - 1) / PT_SPLIT));
    size_t o = 0;
    l.keys = o; o = align256(o + (size_t)T * l.stride * 4);
    l.flags = o; o = align256(o + (size_t)T * 4);
    l.kmax = o; o = align256(o + (size_t)l.kmax_parts * 4);
    l.total = o;
    return l;
}

// Dynamic shared-memory opt-in, once per device.
static cudaError_t ensure_smem(const void* fn, size_t bytes, bool* done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev]) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

// The indexer-K rows as a 2-D tensor [n_slots][64] bf16 read in 64-row boxes,
// 128-byte swizzled.  Returns false when the map cannot be made.
static bool entry_row_map(const csa2_kv_cache& cache, CUtensorMap* map, uint32_t box_rows = 64u) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kID, (cuuint64_t)(cache.n_phys_pages * cache.page_size)};
    const cuuint64_t strides[1] = {(cuuint64_t)kID * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kID, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (void*)cache.idx_k, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count() {
    static int n[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        n[dev] = v;
    }
    return n[dev];
}

cudaError_t launch_block_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                              const int32_t* seq_lens, int keep, int32_t* out, int n, int64_t max_len, char* ws,
                              int32_t* err, cudaStream_t stream, bool flat) {
    static bool d2[64], d3[64];
    cudaError_t e = ensure_smem((const void*)block_score_kernel, K2_SMEM, d2);
    static bool d3f[64];
    if (e == cudaSuccess) e = ensure_smem((const void*)block_select_kernel<false>, K3_SMEM, d3);
    if (e == cudaSuccess) e = ensure_smem((const void*)block_select_kernel<true>, K3_SMEM, d3f);
    if (e != cudaSuccess) return e;
    if (n > K2_MAX_SEQS) return cudaErrorInvalidValue;
    const DecodeWs l = decode_ws_layout(n, max_len, flat);
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
    a.tie = flat ? reinterpret_cast<uint32_t*>(ws + l.blk_tie) : nullptr;
    a.abv = flat ? reinterpret_cast<int32_t*>(ws + l.blk_abv) : nullptr;
    a.abv_cnt = reinterpret_cast<uint32_t*>(ws + l.blk_abv_cnt);
    a.rows = reinterpret_cast<const uint8_t*>(flat ? cache.idx_k : cache.idx_k_pooled);
    a.rshift = flat ? 0 : 3;
    a.err = err;
    a.nblk_pad = l.nblk_pad;
    a.max_len = max_len;
    a.n = n;
    a.keep = keep;
    a.page_shift = page_shift_of(cache);
    const int64_t nblk = flat ? max_len : (max_len + kBlk - 1) / kBlk;
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    a.tma = flat && cache.page_size >= 64 && entry_row_map(cache, &map) ? 1 : 0;
    // A tensor-box ring keeps the fixed limit: a wait that gave up there could
    // leave bulk copies in flight into the CTA's shared memory when it exits.
    // The cp.async ring's producers drain their own copies before they leave,
    // so its limit may be lowered (csa2_test_set_wait_limit).
    a.wait_limit = a.tma ? kWaitLimit : g_copy_wait_limit.load(std::memory_order_relaxed);
    if (nblk > keep) {
        const int64_t tiles = (int64_t)n * ((nblk + K2_TILE - 1) / K2_TILE);
        const int grid = (int)std::min<int64_t>(tiles, sm_count());
        LaunchCfg c2(dim3((unsigned)grid), dim3(K2_THREADS), K2_SMEM, stream);
        e = cudaLaunchKernelEx(&c2.cfg, block_score_kernel, map, a);
        if (e != cudaSuccess) return e;
    }
    // one CTA per SM holds the select's shared memory: give each CTA several
    // 8192-row chunks when the batch has more chunks than one wave
    const int64_t chunks = (nblk + K3_CHUNK - 1) / K3_CHUNK;
    const int64_t cpb = flat ? std::max<int64_t>(1, (chunks * n + sm_count() - 1) / sm_count()) : 1;
    a.span = (int)(K3_CHUNK * cpb);
    LaunchCfg c3(dim3((unsigned)((nblk + a.span - 1) / a.span), n), dim3(K3_THREADS), K3_SMEM, stream);
    return flat ? cudaLaunchKernelEx(&c3.cfg, block_select_kernel<true>, a)
                : cudaLaunchKernelEx(&c3.cfg, block_select_kernel<false>, a);
}

cudaError_t launch_token_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                              const int32_t* seq_lens, const int32_t* cand_blocks, int keep, int topk, int32_t* out,
                              int n, int64_t max_len, char* ws, int32_t* err, cudaStream_t stream,
                              int pre) {
    static bool d4[64], d5[64];
    cudaError_t e = ensure_smem((const void*)token_score_kernel, TS_SMEM, d4);
    if (e == cudaSuccess) e = ensure_smem((const void*)token_select_kernel, TK_SMEM, d5);
    if (e != cudaSuccess) return e;
    TokenArgs a{};
    a.cache = cache;
    a.q_idx = q_idx;
    a.w = w;
    a.seq_lens = seq_lens;
    a.cand = cand_blocks;
    a.out = out;
    a.keys = reinterpret_cast<uint32_t*>(ws + decode_ws_layout(n, max_len, false).tok_keys);
    a.err = err;
    a.max_len = max_len;
    a.keep = keep;
    a.topk = topk;
    a.page_shift = page_shift_of(cache);
    a.pre = pre;
    // candidate blocks as 8-row tensor boxes when every slot is an int32
    // coordinate (a block's 8 rows lie in one page: pages hold >= 8 entries)
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    a.tma = (cache.n_phys_pages << a.page_shift) <= INT32_MAX && entry_row_map(cache, &map, kBlk) ? 1 : 0;
    LaunchCfg c1(dim3((unsigned)n * TS_PARTS), dim3(TS_THREADS), TS_SMEM, stream);
    e = cudaLaunchKernelEx(&c1.cfg, token_score_kernel, map, a);
    if (e != cudaSuccess) return e;
    LaunchCfg c2(dim3((unsigned)n), dim3(TK_THREADS), TK_SMEM, stream);
    return cudaLaunchKernelEx(&c2.cfg, token_select_kernel, a);
}

cudaError_t launch_prefill_topk(const csa2_kv_cache& cache, const uint16_t* q_idx, const float* w,
                                const int32_t* seq_lens, const int32_t* q_pos, int ratio, int topk, int32_t* out,
                                int T, int64_t max_len, char* ws, int32_t* err, cudaStream_t stream) {
    static bool d1[64], d2[64], d3[64], d4[64];
    cudaError_t e = ensure_smem((const void*)prefill_select_kernel, PSEL_SMEM, d1);
    if (e == cudaSuccess) e = ensure_smem((const void*)prefill_score_kernel, PS_SMEM, d2);
    if (e == cudaSuccess) e = ensure_smem((const void*)prefill_tc_score_kernel, TC_SMEM, d3);
    if (e == cudaSuccess) e = ensure_smem((const void*)prefill_candidates_kernel, PC_SMEM, d4);
    if (e != cudaSuccess) return e;
    (void)seq_lens;
    const PrefillWs l = prefill_ws_layout(T, max_len);
    PrefillArgs a{};
    a.cache = cache;
    a.q_idx = q_idx;
    a.w = w;
    a.q_pos = q_pos;
    a.out = out;
    a.keys = reinterpret_cast<uint32_t*>(ws + l.keys);
    a.keys16 = reinterpret_cast<uint16_t*>(ws + l.keys);
    a.flags = reinterpret_cast<int32_t*>(ws + l.flags);
    a.kmax = reinterpret_cast<float*>(ws + l.kmax);
    a.kmax_parts = l.kmax_parts;
    a.err = err;
    a.stride = l.stride;
    a.T = T;
    a.ratio = ratio;
    a.topk = topk;
    a.n_entries = (int)max_len;
    a.page_shift = page_shift_of(cache);
    // tensor-core scores -> candidates, exact rescoring and verification; then
    // the exact CUDA-core path for the queries that failed the check (it exits
    // at once for the others)
    // entry tiles as 64-row tensor boxes when a tile lies in one page and every
    // slot is an int32 coordinate
    CUtensorMap kmap;
    memset(&kmap, 0, sizeof(kmap));
    a.tma_k = cache.page_size >= TC_E && (cache.n_phys_pages << a.page_shift) <= INT32_MAX &&
                      entry_row_map(cache, &kmap)
                  ? 1
                  : 0;
    LaunchCfg c0(dim3((unsigned)((T + TC_Q - 1) / TC_Q), (unsigned)((max_len + PT_SPLIT - 1) / PT_SPLIT)),
                 dim3(TC_THREADS), TC_SMEM, stream);
    e = cudaLaunchKernelEx(&c0.cfg, prefill_tc_score_kernel, kmap, a);
    if (e != cudaSuccess) return e;
    LaunchCfg cc(dim3((unsigned)T), dim3(PC_THREADS), PC_SMEM, stream);
    e = cudaLaunchKernelEx(&cc.cfg, prefill_candidates_kernel, a);
    if (e != cudaSuccess) return e;
    LaunchCfg c1(dim3((unsigned)((T + PS_Q - 1) / PS_Q)), dim3(PS_THREADS), PS_SMEM, stream);
    e = cudaLaunchKernelEx(&c1.cfg, prefill_score_kernel, a);
    if (e != cudaSuccess) return e;
    LaunchCfg c2(dim3((unsigned)std::min(T, 2 * sm_count())), dim3(PSEL_THREADS), PSEL_SMEM, stream);
    return cudaLaunchKernelEx(&c2.cfg, prefill_select_kernel, a);
}

}  // namespace csa2

extern "C" CSA2_API uint32_t csa2_test_set_wait_limit(uint32_t polls) {
    if (polls > csa2::kWaitLimit) polls = csa2::kWaitLimit;
    return csa2::g_copy_wait_limit.exchange(polls);
}
