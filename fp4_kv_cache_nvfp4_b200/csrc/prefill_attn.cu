// K7: prefill attention on the 5th-generation tensor cores (tcgen05).
//
// Pages: "Como funciona" (e-cogni.com.br): a Reuse layer runs sparse
// attention directly on the re-used Top-K indices, every layer keeps its own
// Q and SWA KV; the 128-token window runs in every layer (conexaotc.com.br,
// Causal Encoder-Decoder paragraph).
//
// Per query (16 heads of dim 128 sharing one K and one V): its 512 selected
// FP4 entries are 4 tiles of 128 keys and its window of up to 128 bf16 tokens
// a fifth.  One softmax runs over all 640 keys (the same value as two branches
// merged by log-sum-exp), so no separate window kernel is needed:
//   S^T[128 keys x 16 heads] = K^[128 x 128] . Q^T   (5 times, kind::f16)
//   P = exp2(S * log2(e) / sqrt(128) - max), fp16
//   O^T[128 dims x 16 heads] += V^T[128 x 128 keys] . P^T   (5 times)
// The dequantised K^ / V^ tiles (E2M1 x E4M3 -> fp16 is exact: at most 6
// significant bits, magnitudes 2^-10..2688; bf16 -> fp16 is exact in range)
// are written once in one layout that both products read: two 64-dim halves,
// 16 KiB apart, each [128 keys][128 B] with 8-key groups 1024 B apart and
// chunk c of key row r at c ^ (r & 7) (the 128-byte swizzle).  That is the
// K-major operand of the first product (M = keys) and, through the MN-major
// descriptor (LBO = 16 KiB between the halves, SBO = 1024 B between 8-key
// groups), the transposed operand of the second (M = dims).
//
// Persistent: CTA c takes a contiguous range of queries.  The window tiles
// stay in shared memory across them, one row per token (row = token mod
// 128): the next query of a prefill chunk adds one token, so one row is
// converted instead of 128.  The softmax masks a window row whose token, the
// one in [p - 127, p] congruent to the row, is before the window's start.
//   warps 0-3   softmax and epilogue: thread = TMEM lane = key of a tile
//               (S) and dim (O); per-head max and sum across the 4 warps
//   warp 4      per query: the selected entries' physical slots, the window
//               range, Q converted to fp16 in its swizzled tile
//   warp 5      TMEM owner and MMA issue (one lane); order S(0), then S(j+1)
//               before O(j), so the softmax of query j overlaps the products
//               of query j+1
//   warps 6-13  operand producers: the window rows a query adds, then 8 FP4
//               tiles per query (K of its 4 selected tiles, one query ahead,
//               then V) into a 3-slot ring; each thread one half row per
//               tile, the raw bytes of the next 4 tiles in flight in registers
// Slots and windows rotate over three query buffers, Q, P and the 2 x 128
// TMEM columns over two.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

constexpr int PT_TILES = 5;                              // 4 selected tiles + the window
constexpr int PT_NSLOT = 3;                              // operand ring slots
constexpr int PT_NQB = 3;                                // slot-list / window buffers
constexpr int PT_PREF = 4;                               // FP4 tiles whose raw bytes are in flight
constexpr uint32_t PT_HALF = 128 * 128;                  // one 64-dim half of a tile: 16 KiB
constexpr uint32_t PT_TILE = 2 * PT_HALF;                // 32 KiB
constexpr uint32_t PT_PTILE = 2 * 16 * 128;              // P^T of one tile: two 64-key halves x 16 heads x 128 B
constexpr int PT_THREADS = 14 * 32;
constexpr int PT_DQ0 = 6 * 32;                           // first producer thread
constexpr size_t PT_OFF_RING = 0;
constexpr size_t PT_OFF_KW = PT_OFF_RING + (size_t)PT_NSLOT * PT_TILE;      // window K tile
constexpr size_t PT_OFF_VW = PT_OFF_KW + PT_TILE;                           // window V tile
constexpr size_t PT_OFF_P = PT_OFF_VW + PT_TILE;                            // [2][5][4 KiB]
constexpr size_t PT_OFF_Q = PT_OFF_P + 2 * (size_t)PT_TILES * PT_PTILE;     // [2][2 halves][16][128 B]
constexpr size_t PT_OFF_SLOT = PT_OFF_Q + 2 * 4096;                         // [3][512] int32
constexpr size_t PT_OFF_WIN = PT_OFF_SLOT + (size_t)PT_NQB * 512 * 4;       // [3] (window start, query position)
constexpr size_t PT_OFF_TAG = PT_OFF_WIN + 32;                              // [2][128] token of each window row
constexpr size_t PT_OFF_RED = PT_OFF_TAG + 2 * 128 * 4;                     // [2][4 warps][16] floats
constexpr size_t PT_OFF_BAR = PT_OFF_RED + 2 * 4 * 16 * 4;
constexpr int PT_NBAR = 2 * PT_NSLOT + 2 * PT_NQB + 2 * 6 + 4;
constexpr size_t PT_OFF_MISC = PT_OFF_BAR + (size_t)PT_NBAR * 8;            // tmem base, timeout flag
constexpr size_t PT_SMEM = PT_OFF_MISC + 16 + 1024;                         // + slack for the 1 KiB alignment
static_assert(PT_OFF_KW % 1024 == 0 && PT_OFF_P % 1024 == 0 && PT_OFF_Q % 1024 == 0 && PT_OFF_BAR % 8 == 0,
              "K7 layout");
static_assert(PT_SMEM <= 227 * 1024, "K7 shared memory");
constexpr uint32_t kPtWaitLimit = 1u << 22;
constexpr uint32_t PT_TMEM_COLS = 256;  // per query buffer: S of 5 tiles (80 columns) at 0, O (16) at 96

// Shared-memory descriptor of an MN-major, 128-byte-swizzled operand: rows of
// 128 B (64 M-elements of one K index), 8-row groups SBO = 1024 B apart along
// K, 64-element M groups `lbo` bytes apart.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// D[128 x 16] (+)= A . B^T with fp16 operands, fp32 accumulators; a_mn: A is MN-major
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t acc, bool a_mn) {
    const uint32_t idesc = (1u << 4) | (a_mn ? (1u << 15) : 0u) | ((uint32_t)(16 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

// Raw bytes of one producer thread's half row of one FP4 tile.
struct PtRaw {
    uint4 c0, c1;  // 32 code bytes = 64 channels
    uint32_t sc;   // their 4 scales
    uint32_t ok;   // 0: the entry is absent (a zero row)
};

__global__ void __launch_bounds__(PT_THREADS, 1) prefill_attn_tc_kernel(AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PT_OFF_BAR);
    uint64_t* full = bars;                       // [3] ring slot filled (8 producer warps)
    uint64_t* empty = full + PT_NSLOT;           // [3] ring slot read by the tensor core
    uint64_t* slot_ready = empty + PT_NSLOT;     // [3] slots and window range of a query (warp 4)
    uint64_t* slot_free = slot_ready + PT_NQB;   // [3] (8 producer warps + 4 softmax warps)
    uint64_t* q_ready = slot_free + PT_NQB;      // [2] Q tile written (warp 4)
    uint64_t* q_free = q_ready + 2;              // [2] Q tile read (MMA commit)
    uint64_t* s_full = q_free + 2;               // [2] S complete (MMA commit)
    uint64_t* p_ready = s_full + 2;              // [2] P^T written (4 softmax warps)
    uint64_t* o_full = p_ready + 2;              // [2] O complete (MMA commit)
    uint64_t* tmem_free = o_full + 2;            // [2] S and O read (4 softmax warps)
    uint64_t* kw_ready = tmem_free + 2;          // window K rows of the next query written (8 warps)
    uint64_t* kw_done = kw_ready + 1;            // window K tile read (MMA commit)
    uint64_t* vw_ready = kw_done + 1;
    uint64_t* vw_done = vw_ready + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + PT_OFF_MISC);
    int* s_timeout = reinterpret_cast<int*>(smem + PT_OFF_MISC + 4);
    int32_t* s_slot = reinterpret_cast<int32_t*>(smem + PT_OFF_SLOT);
    int2* s_win = reinterpret_cast<int2*>(smem + PT_OFF_WIN);
    int32_t* s_tag = reinterpret_cast<int32_t*>(smem + PT_OFF_TAG);  // [0..127] K rows, [128..255] V rows
    float* s_red = reinterpret_cast<float*>(smem + PT_OFF_RED);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // this CTA's contiguous range of queries
    const int per = (a.rows + (int)gridDim.x - 1) / (int)gridDim.x;
    const int q0 = blockIdx.x * per, nq = max(0, min(a.rows - q0, per));

    if (tid == 0) {
        for (int s = 0; s < PT_NSLOT; ++s) {
            mbar_init(&full[s], 8);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < PT_NQB; ++b) {
            mbar_init(&slot_ready[b], 1);
            mbar_init(&slot_free[b], 12);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_ready[b], 1);
            mbar_init(&q_free[b], 1);
            mbar_init(&s_full[b], 1);
            mbar_init(&p_ready[b], 4);
            mbar_init(&o_full[b], 1);
            mbar_init(&tmem_free[b], 4);
        }
        mbar_init(kw_ready, 8);
        mbar_init(kw_done, 1);
        mbar_init(vw_ready, 8);
        mbar_init(vw_done, 1);
        *s_timeout = 0;
        fence_mbar_init();
    }
    // window tiles start as zeros (a masked row still meets P = 0 in P V, so it
    // must hold a finite value) with no token in any row
    for (int i = tid; i < 2 * (int)PT_TILE / 16; i += PT_THREADS)
        reinterpret_cast<uint4*>(smem + PT_OFF_KW)[i] = make_uint4(0, 0, 0, 0);
    for (int i = tid; i < 256; i += PT_THREADS) s_tag[i] = INT32_MIN;
    fence_proxy_async_smem();
    if (wid == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(PT_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    pdl_wait();
    pdl_trigger();
    const int32_t L = a.seq_len_prefill;
    auto timeout = [&]() { *s_timeout = 1; };

    if (wid == 4) {
        // ============ slots, window range and Q of each query ============
        for (int j = 0; j < nq; ++j) {
            const int q = q0 + j, sb = j % PT_NQB, qb = j & 1;
            if (j >= PT_NQB && !mbar_wait(&slot_free[sb], (uint32_t)((j - PT_NQB) / PT_NQB) & 1u, kPtWaitLimit))
                timeout();
            if (j >= 2 && !mbar_wait(&q_free[qb], (uint32_t)((j - 2) >> 1) & 1u, kPtWaitLimit)) timeout();
            int32_t* sl = s_slot + sb * 512;
            for (int k = lane; k < 512; k += 32) {
                int32_t slot = -1;
                const int32_t pos = k < a.topk ? a.idx[(int64_t)q * a.topk + k] : -1;
                if (pos >= 0) {
                    if (pos < L) slot = (int32_t)entry_slot(a.cache, a.page_shift, 0, pos, a.err);
                    else dev_error(a.err, CSA2_DEV_INDEX);
                }
                sl[k] = slot;
            }
            if (lane == 0) {
                const int p = a.q_pos[q];
                int lo = max(0, p - a.window + 1);
                if (lo < a.swa_start) {  // the window's rows are not all in swa_kv: no window
                    dev_error(a.err, CSA2_DEV_INDEX);
                    lo = p + 1;
                }
                s_win[sb] = make_int2(lo, p);
            }
            // Q: 16 heads x 128 dims, fp16, half h of the dims at +2 KiB, head rows of 128 B
            uint8_t* qt = smem + PT_OFF_Q + (size_t)qb * 4096;
            for (int i = lane; i < 16 * 16; i += 32) {
                const int h = i >> 4, c8 = i & 15, half = c8 >> 3, c = c8 & 7;
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.q + ((int64_t)q * kH + h) * kD) + c8);
                *reinterpret_cast<uint4*>(qt + half * 2048 + h * 128 + ((c ^ (h & 7)) << 4)) =
                    make_uint4(bf2_to_h2(v.x), bf2_to_h2(v.y), bf2_to_h2(v.z), bf2_to_h2(v.w));
            }
            fence_proxy_async_smem();  // Q is read by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&slot_ready[sb]);
                mbar_arrive(&q_ready[qb]);
            }
        }
    } else if (wid == 5) {
        // ================= MMA issue: S(0), then S(j + 1) before O(j) =================
        if (lane == 0) {
            uint32_t pos = 0;  // ring position
            auto ring_wait = [&](int& s) {
                s = (int)(pos % PT_NSLOT);
                if (!mbar_wait(&full[s], (pos / PT_NSLOT) & 1u, kPtWaitLimit)) timeout();
                tc_fence_after();
            };
            auto mma_s = [&](int j) {  // S^T(j) = K^ Q^T over the 4 selected tiles and the window tile
                const int qb = j & 1;
                const uint32_t ph = (uint32_t)(j >> 1) & 1u;
                if (!mbar_wait(&q_ready[qb], ph, kPtWaitLimit)) timeout();
                if (j >= 2 && !mbar_wait(&tmem_free[qb], ph ^ 1u, kPtWaitLimit)) timeout();
                const uint32_t tS = tmem + (uint32_t)qb * 128u;
                const uint32_t qaddr = smem_u32(smem + PT_OFF_Q + (size_t)qb * 4096);
                for (int t = 0; t < PT_TILES; ++t) {
                    uint32_t ka;
                    int s = -1;
                    if (t < 4) {
                        ring_wait(s);
                        ka = smem_u32(smem + PT_OFF_RING + (size_t)s * PT_TILE);
                    } else {
                        if (!mbar_wait(kw_ready, (uint32_t)j & 1u, kPtWaitLimit)) timeout();
                        tc_fence_after();
                        ka = smem_u32(smem + PT_OFF_KW);
                    }
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {  // 16 dims per step; dims 64.. in the second half
                        const uint64_t da = umma_desc_sw128(ka + (uint32_t)(ks >> 2) * PT_HALF) + 2u * (ks & 3);
                        const uint64_t db = umma_desc_sw128(qaddr + (uint32_t)(ks >> 2) * 2048u) + 2u * (ks & 3);
                        umma_f16(tS + 16u * t, da, db, ks > 0 ? 1u : 0u, false);
                    }
                    if (s >= 0) {
                        umma_commit(&empty[s]);
                        ++pos;
                    }
                }
                umma_commit(&q_free[qb]);
                umma_commit(kw_done);
                umma_commit(&s_full[qb]);
            };
            auto mma_o = [&](int j) {  // O^T(j) += V^T P^T over the 4 selected tiles and the window tile
                const int qb = j & 1;
                const uint32_t ph = (uint32_t)(j >> 1) & 1u;
                if (!mbar_wait(&p_ready[qb], ph, kPtWaitLimit)) timeout();
                tc_fence_after();
                const uint32_t tO = tmem + (uint32_t)qb * 128u + 96u;
                for (int t = 0; t < PT_TILES; ++t) {
                    uint32_t va;
                    int s = -1;
                    if (t < 4) {
                        ring_wait(s);
                        va = smem_u32(smem + PT_OFF_RING + (size_t)s * PT_TILE);
                    } else {
                        if (!mbar_wait(vw_ready, (uint32_t)j & 1u, kPtWaitLimit)) timeout();
                        tc_fence_after();
                        va = smem_u32(smem + PT_OFF_VW);
                    }
                    const uint32_t pa = smem_u32(smem + PT_OFF_P + ((size_t)qb * PT_TILES + t) * PT_PTILE);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {  // 16 keys per step: two 8-key groups of 1024 B
                        const uint64_t da = umma_desc_sw128_mn(va + (uint32_t)ks * 2048u, PT_HALF);
                        const uint64_t db = umma_desc_sw128(pa + (uint32_t)(ks >> 2) * 2048u) + 2u * (ks & 3);
                        umma_f16(tO, da, db, (t > 0 || ks > 0) ? 1u : 0u, true);
                    }
                    if (s >= 0) {
                        umma_commit(&empty[s]);
                        ++pos;
                    }
                }
                umma_commit(vw_done);
                umma_commit(&o_full[qb]);
            };
            if (nq > 0) mma_s(0);
            for (int j = 0; j < nq; ++j) {
                if (j + 1 < nq) mma_s(j + 1);
                mma_o(j);
            }
        }
        __syncwarp();
    } else if (wid >= 6) {
        // ============ operand producers ============
        // Tile jobs in ring order: K of query 0, then per query j the K of
        // query j + 1 and the V of query j; job n < 4: K(0) tile n; job
        // 4 + 8 j + r: K(j + 1) tile r (r < 4, absent for the last query) or
        // V(j) tile r - 4.
        const int dt = tid - PT_DQ0, key = dt >> 1, h = dt & 1;
        const int nend = 8 * nq + 4;
        auto job_of = [&](int n, int& j, int& v, int& t) -> bool {
            if (n < 4) {
                j = 0, v = 0, t = n;
                return nq > 0;
            }
            const int m = n - 4, jj = m >> 3, r = m & 7;
            if (r < 4) {
                j = jj + 1, v = 0, t = r;
                return jj + 1 < nq;
            }
            j = jj, v = 1, t = r - 4;
            return jj < nq;
        };
        int seen = -1;  // last query whose slot list the prefetch waited for
        auto fetch = [&](int n, PtRaw& r) {  // raw bytes of job n (any n; absent jobs give a zero row)
            int j, v, t;
            r.ok = 0u;
            if (n >= nend || !job_of(n, j, v, t)) return;
            if (j > seen) {
                if (!mbar_wait(&slot_ready[j % PT_NQB], (uint32_t)(j / PT_NQB) & 1u, kPtWaitLimit)) timeout();
                seen = j;
            }
            const int32_t slot = s_slot[(j % PT_NQB) * 512 + t * 128 + key];
            if (slot < 0) return;
            const uint4* cp = reinterpret_cast<const uint4*>(a.cache.codes + (int64_t)slot * kCodeBytes + (v ? 64 : 0) +
                                                              32 * h);
            r.c0 = __ldg(cp);
            r.c1 = __ldg(cp + 1);
            r.sc = __ldg(reinterpret_cast<const uint32_t*>(a.cache.scales + (int64_t)slot * kScales + (v ? 8 : 0) +
                                                           4 * h));
            r.ok = 1u;
        };
        // the window rows query j adds to tile K (v = 0) or V (v = 1): rows of
        // tokens in [lo, p] whose tag differs; 16 threads per row, 8 dims each
        const GroupBar pb{2, 256};
        auto window_rows = [&](int j, int v) {
            const int2 win = s_win[j % PT_NQB];
            int32_t* tag = s_tag + v * 128;
            uint8_t* tile = smem + (v ? PT_OFF_VW : PT_OFF_KW);
            const int n = win.y - win.x + 1;  // tokens in the window (<= 128; 0: none)
            for (int c = dt; c < n * 16; c += 256) {
                const int tok = win.x + (c >> 4), ch = c & 15, row = tok & 127;
                if (tag[row] == tok) continue;
                const uint4 x = __ldg(reinterpret_cast<const uint4*>(a.swa + (int64_t)(tok - a.swa_start) * kCh +
                                                                      (v ? 128 : 0)) + ch);
                *reinterpret_cast<uint4*>(tile + (size_t)(ch >> 3) * PT_HALF + row * 128 + (((ch & 7) ^ (row & 7)) << 4)) =
                    make_uint4(bf2_to_h2(x.x), bf2_to_h2(x.y), bf2_to_h2(x.z), bf2_to_h2(x.w));
            }
            pb.sync();  // every thread has read the tags
            for (int c = dt; c < n; c += 256) tag[(win.x + c) & 127] = win.x + c;
            fence_proxy_async_smem();  // the rows are read by the tensor core
            pb.sync();
            if (lane == 0) mbar_arrive(v ? vw_ready : kw_ready);
        };
        PtRaw r0, r1, r2, r3;  // raw bytes of jobs n .. n + 3
        int n = 0;
        while (n < nend) {  // skip absent jobs at the front
            int j, v, t;
            if (job_of(n, j, v, t)) break;
            ++n;
        }
        fetch(n, r0);
        fetch(n + 1, r1);
        fetch(n + 2, r2);
        fetch(n + 3, r3);
        uint32_t pos = 0;  // ring position
        for (; n < nend; ++n) {
            int j, v, t;
            if (!job_of(n, j, v, t)) {  // an absent job: its prefetched bytes move down
                r0 = r1, r1 = r2, r2 = r3;
                fetch(n + 4, r3);
                continue;
            }
            if (t == 0) {  // the window rows of this query, before its first tile of the kind
                if (j >= 1 && !mbar_wait(v ? vw_done : kw_done, (uint32_t)(j - 1) & 1u, kPtWaitLimit)) timeout();
                window_rows(j, v);
            }
            const int s = (int)(pos % PT_NSLOT);
            if (pos >= PT_NSLOT && !mbar_wait(&empty[s], ((pos / PT_NSLOT) - 1) & 1u, kPtWaitLimit)) timeout();
            uint8_t* dst = smem + PT_OFF_RING + (size_t)s * PT_TILE + (size_t)h * PT_HALF + key * 128;
            const uint32_t words[8] = {r0.c0.x, r0.c0.y, r0.c0.z, r0.c0.w, r0.c1.x, r0.c1.y, r0.c1.z, r0.c1.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {  // 8 channels per chunk, scale (c / 2) of the four
                uint4 o = make_uint4(0, 0, 0, 0);
                if (r0.ok) {
                    const uint32_t sc = e4m3_to_h2((uint8_t)((r0.sc >> (8 * (c >> 1))) & 0xffu));
                    uint32_t h0, h1, h2, h3;
                    e2m1x8_to_h2x4(words[c], h0, h1, h2, h3);
                    o = make_uint4(hmul2(h0, sc), hmul2(h1, sc), hmul2(h2, sc), hmul2(h3, sc));
                }
                *reinterpret_cast<uint4*>(dst + ((c ^ (key & 7)) << 4)) = o;
            }
            fence_proxy_async_smem();  // the tile is read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
            ++pos;
            if (v == 1 && t == 3 && lane == 0) mbar_arrive(&slot_free[j % PT_NQB]);  // done with query j's slots
            r0 = r1, r1 = r2, r2 = r3;
            fetch(n + 4, r3);
        }
    } else {
        // ============ softmax and epilogue: warps 0-3, thread = TMEM lane ============
        const GroupBar sb{1, 128};
        const uint32_t lane_base = tmem + ((uint32_t)(32 * wid) << 16);
        const float kScaleLog2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
        for (int j = 0; j < nq; ++j) {
            const int q = q0 + j, qb = j & 1, wb = j % PT_NQB;
            const uint32_t ph = (uint32_t)(j >> 1) & 1u;
            // the slots and the window of this query (written by warp 4), then its scores
            if (!mbar_wait(&slot_ready[wb], (uint32_t)(j / PT_NQB) & 1u, kPtWaitLimit)) timeout();
            if (!mbar_wait(&s_full[qb], ph, kPtWaitLimit)) timeout();
            tc_fence_after();
            const int32_t* sl = s_slot + wb * 512;
            const int2 win = s_win[wb];
            // window row `tid` holds the token of [p - 127, p] congruent to it
            const int wtok = win.y - ((win.y - tid) & 127);
            const bool wok = wtok >= win.x;
            const uint32_t tS = lane_base + (uint32_t)qb * 128u;
            // pass 1: the per-head maximum over the 640 keys (log2 domain)
            float m[16];
#pragma unroll
            for (int hh = 0; hh < 16; ++hh) m[hh] = -INFINITY;
#pragma unroll 1
            for (int t = 0; t < PT_TILES; ++t) {
                const bool ok = t < 4 ? sl[t * 128 + tid] >= 0 : wok;
                uint32_t v[16];
                tmem_ld16(tS + 16u * t, v);
                tmem_wait_ld();
                if (ok)
#pragma unroll
                    for (int hh = 0; hh < 16; ++hh) m[hh] = fmaxf(m[hh], __uint_as_float(v[hh]) * kScaleLog2);
            }
#pragma unroll
            for (int hh = 0; hh < 16; ++hh)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m[hh] = fmaxf(m[hh], __shfl_xor_sync(0xffffffffu, m[hh], o));
            float* red = s_red + (j & 1) * 64;  // alternate buffers: a fast warp's next query never overwrites this one
            if (lane == 0)
#pragma unroll
                for (int hh = 0; hh < 16; ++hh) red[wid * 16 + hh] = m[hh];
            sb.sync();
#pragma unroll
            for (int hh = 0; hh < 16; ++hh)
                m[hh] = fmaxf(fmaxf(red[hh], red[16 + hh]), fmaxf(red[32 + hh], red[48 + hh]));
            // pass 2: P = exp2(S - max) as fp16 into P^T, and the per-head sums
            float l[16];
#pragma unroll
            for (int hh = 0; hh < 16; ++hh) l[hh] = 0.f;
            uint8_t* pt = smem + PT_OFF_P + (size_t)qb * PT_TILES * PT_PTILE;
            const int k = tid;  // key within the tile
            const int ke = k & ~1, odd = k & 1;
#pragma unroll 1
            for (int t = 0; t < PT_TILES; ++t) {
                const bool ok = t < 4 ? sl[t * 128 + tid] >= 0 : wok;
                uint32_t v[16];
                tmem_ld16(tS + 16u * t, v);
                tmem_wait_ld();
                float p[16];
#pragma unroll
                for (int hh = 0; hh < 16; ++hh) {
                    p[hh] = (ok && m[hh] != -INFINITY) ? exp2f(__uint_as_float(v[hh]) * kScaleLog2 - m[hh]) : 0.f;
                    l[hh] += p[hh];
                }
                // P^T tile t: [key half][16 heads][128 B], key k of head h at chunk ((k & 63) >> 3) ^ (h & 7);
                // lanes k and k ^ 1 pair up: the even lane stores heads 0..7, the odd one heads 8..15
                uint8_t* ptt = pt + (size_t)t * PT_PTILE + (size_t)(k >> 6) * 2048;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int hs = odd ? 8 + i : i;   // head this lane stores
                    const float mine = odd ? p[8 + i] : p[i], give = odd ? p[i] : p[8 + i];
                    const float got = __shfl_xor_sync(0xffffffffu, give, 1);
                    const float lo = odd ? got : mine, hi = odd ? mine : got;  // keys ke, ke + 1
                    *reinterpret_cast<uint32_t*>(ptt + hs * 128 + ((((ke & 63) >> 3) ^ (hs & 7)) << 4) + (ke & 7) * 2) =
                        f2_to_h2(lo, hi);
                }
            }
            fence_proxy_async_smem();  // P^T is read by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&p_ready[qb]);
                mbar_arrive(&slot_free[wb]);
            }
#pragma unroll
            for (int hh = 0; hh < 16; ++hh)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], o);
            sb.sync();  // every warp has read the maxima: the buffer takes the sums
            if (lane == 0)
#pragma unroll
                for (int hh = 0; hh < 16; ++hh) red[wid * 16 + hh] = l[hh];
            sb.sync();
#pragma unroll
            for (int hh = 0; hh < 16; ++hh) l[hh] = (red[hh] + red[16 + hh]) + (red[32 + hh] + red[48 + hh]);
            // ---- O^T (thread = dim) once every P V product is done ----
            if (!mbar_wait(&o_full[qb], ph, kPtWaitLimit)) timeout();
            tc_fence_after();
            uint32_t ov[16];
            tmem_ld16(lane_base + (uint32_t)qb * 128u + 96u, ov);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_free[qb]);
            float* out = a.out + (int64_t)q * kH * kD;
#pragma unroll
            for (int hh = 0; hh < 16; ++hh) {
                const float inv = l[hh] > 0.f ? 1.f / l[hh] : 0.f;
                out[hh * kD + tid] = __uint_as_float(ov[hh]) * inv;
            }
            if (tid < 16) {
                float lt = 0.f, mt = 0.f;
#pragma unroll
                for (int hh = 0; hh < 16; ++hh)
                    if (hh == tid) {
                        lt = l[hh];
                        mt = m[hh];
                    }
                a.lse[(int64_t)q * kH + tid] = lt > 0.f ? (mt + log2f(lt)) * 0.6931471805599453f : -INFINITY;
            }
        }
    }
    tc_fence_before();
    __syncthreads();  // every accumulator has been read
    if (wid == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(PT_TMEM_COLS)
                     : "memory");
    }
    if (tid == 0 && *s_timeout) dev_error(a.err, CSA2_DEV_TIMEOUT);
}

cudaError_t launch_prefill_attn_tc(const AttnArgs& a, int n_ctas, cudaStream_t stream) {
    static bool init[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!init[dev]) {
        e = cudaFuncSetAttribute((const void*)prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)PT_SMEM);
        if (e != cudaSuccess) return e;
        init[dev] = true;
    }
    if (a.rows <= 0) return cudaSuccess;
    LaunchCfg c(dim3((unsigned)std::min(a.rows, n_ctas)), dim3(PT_THREADS), PT_SMEM, stream);
    return cudaLaunchKernelEx(&c.cfg, prefill_attn_tc_kernel, a);
}

}  // namespace csa2
