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
//   warps 0-7   softmax: warp w reads TMEM lane quarter w % 4 (thread = key
//               of a tile for S, dim for O) for heads 8 (w / 4) .. + 7; per-head
//               max and sum across the 4 warps of a head group; the epilogue
//               of query j - 1 runs after P of query j is out
//   warp 8      TMEM owner and MMA issue (one lane); order S(0), then S(j+1)
//               before O(j), so the softmax of query j overlaps the products
//               of query j+1
//   warps 9-11  per query (in turn): the selected entries' physical slots
//               (the sequence's page table cached in shared memory), the
//               window range, Q and the window rows the query adds, converted
//               to fp16 in their swizzled tiles
//   warps 12-27 converters: thread = one 16-byte quarter (32 channels) of one
//               entry of a tile, read by plain loads (the four quarters of an
//               entry's 64 K or V code bytes by four neighbouring lanes) one
//               block of four tiles ahead of the block it converts; FP4 ->
//               fp16 tile into a 3-slot ring.  The 8 FP4 tiles of query j: its
//               K, one query ahead, then its V.  The proxy fence that hands a
//               tile to the tensor core does not wait for the loads in flight
//               (measured).
// TMEM holds four query buffers of 128 columns (S of 5 tiles at 0, O at 96),
// Q and P^T two buffers each.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

constexpr int PT_TILES = 5;                              // 4 selected tiles + the window
constexpr int PT_NSLOT = 3;                              // operand ring slots
constexpr int PT_NQB = 4;                                // slot-list buffers
constexpr int PT_NTB = 4;                                // TMEM query buffers
constexpr uint32_t PT_HALF = 128 * 128;                  // one 64-dim half of a tile: 16 KiB
constexpr uint32_t PT_TILE = 2 * PT_HALF;                // 32 KiB
constexpr uint32_t PT_PTILE = 2 * 16 * 128;              // P^T of one tile: two 64-key halves x 16 heads x 128 B
constexpr int PT_NSOFT = 8, PT_W_MMA = 8, PT_W_SETUP = 9, PT_NSETUP = 3, PT_W_CONV = 12, PT_NCONV = 16, PT_WARPS = 28;
constexpr int PT_PTAB = 1024;                            // page-table entries kept in shared memory
constexpr int PT_THREADS = PT_WARPS * 32;
constexpr size_t PT_OFF_RING = 0;
constexpr size_t PT_OFF_KW = PT_OFF_RING + (size_t)PT_NSLOT * PT_TILE;      // window K tile
constexpr size_t PT_OFF_VW = PT_OFF_KW + PT_TILE;                           // window V tile
constexpr size_t PT_OFF_P = PT_OFF_VW + PT_TILE;                            // [2][5][4 KiB]
constexpr size_t PT_OFF_Q = PT_OFF_P + 2 * (size_t)PT_TILES * PT_PTILE;     // [2][2 halves][16][128 B]
constexpr size_t PT_OFF_SLOT = PT_OFF_Q + 2 * 4096;                         // [3][512] int32
constexpr size_t PT_OFF_PTAB = PT_OFF_SLOT + (size_t)PT_NQB * 512 * 4;      // [1024] the sequence's first pages
constexpr size_t PT_OFF_WIN = PT_OFF_PTAB + (size_t)PT_PTAB * 4;            // [4] (window start, query position)
constexpr size_t PT_OFF_RED = PT_OFF_WIN + 32;                              // [2][2 head groups][4 quarters][8] floats
constexpr size_t PT_OFF_INV = PT_OFF_RED + 2 * 2 * 4 * 8 * 4;              // [2][16] 1 / sum per head
constexpr size_t PT_OFF_BAR = PT_OFF_INV + 2 * 16 * 4;
constexpr int PT_NBAR = 2 * PT_NSLOT + 2 * PT_NQB + 2 * 2 + 3 * PT_NTB + 2 + 2;
constexpr size_t PT_OFF_MISC = PT_OFF_BAR + (size_t)PT_NBAR * 8;            // tmem base, timeout flag
constexpr size_t PT_SMEM = PT_OFF_MISC + 16 + 1024;                         // + slack for the 1 KiB alignment
static_assert(PT_OFF_KW % 1024 == 0 && PT_OFF_P % 1024 == 0 && PT_OFF_Q % 1024 == 0 && PT_OFF_SLOT % 16 == 0 &&
                  PT_OFF_BAR % 8 == 0,
              "K7 layout");
static_assert(PT_SMEM <= 227 * 1024, "K7 shared memory");
constexpr uint32_t kPtWaitLimit = 1u << 22;
constexpr uint32_t PT_TMEM_COLS = 128 * PT_NTB;

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

// 8 consecutive TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld8(uint32_t addr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(addr));
}

// 2^x (the hardware approximation; P is rounded to fp16 afterwards)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 8 dims (one 16-byte chunk ch of the 16 of a K or V row) of a bf16 window row
// into row `row` of a window tile, as fp16
__device__ __forceinline__ void win_store(uint8_t* tile, int row, int ch, uint4 x) {
    *reinterpret_cast<uint4*>(tile + (size_t)(ch >> 3) * PT_HALF + row * 128 + (((ch & 7) ^ (row & 7)) << 4)) =
        make_uint4(bf2_to_h2(x.x), bf2_to_h2(x.y), bf2_to_h2(x.z), bf2_to_h2(x.w));
}

__global__ void __launch_bounds__(PT_THREADS, 1) prefill_attn_tc_kernel(AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PT_OFF_BAR);
    uint64_t* full = bars;                       // [3] ring slot converted (16 converter warps)
    uint64_t* empty = full + PT_NSLOT;           // [3] ring slot read by the tensor core
    uint64_t* slot_ready = empty + PT_NSLOT;     // [4] slots and window range of a query (setup warp)
    uint64_t* slot_free = slot_ready + PT_NQB;   // [4] (16 converter warps + 8 softmax warps)
    uint64_t* q_ready = slot_free + PT_NQB;      // [2] Q tile and the query's window K rows written
    uint64_t* q_free = q_ready + 2;              // [2] Q tile read (MMA commit)
    uint64_t* s_full = q_free + 2;               // [4] S complete (MMA commit)
    uint64_t* o_full = s_full + PT_NTB;          // [4] O complete (MMA commit)
    uint64_t* tmem_free = o_full + PT_NTB;       // [4] S and O read (8 softmax warps)
    uint64_t* p_ready = tmem_free + PT_NTB;      // [2] P^T written (8 softmax warps)
    uint64_t* vw_ready = p_ready + 2;            // window V rows of a query written (setup warp)
    uint64_t* mma_done = vw_ready + 1;           // every product complete
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + PT_OFF_MISC);
    volatile int* s_timeout = reinterpret_cast<volatile int*>(smem + PT_OFF_MISC + 4);
    int32_t* s_slot = reinterpret_cast<int32_t*>(smem + PT_OFF_SLOT);
    int2* s_win = reinterpret_cast<int2*>(smem + PT_OFF_WIN);
    int32_t* s_ptab = reinterpret_cast<int32_t*>(smem + PT_OFF_PTAB);
    float* s_red = reinterpret_cast<float*>(smem + PT_OFF_RED);
    float* s_inv = reinterpret_cast<float*>(smem + PT_OFF_INV);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // this CTA's contiguous range of queries
    const int per = (a.rows + (int)gridDim.x - 1) / (int)gridDim.x;
    const int q0 = blockIdx.x * per, nq = max(0, min(a.rows - q0, per));

    if (tid == 0) {
        for (int s = 0; s < PT_NSLOT; ++s) {
            mbar_init(&full[s], PT_NCONV);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < PT_NQB; ++b) {
            mbar_init(&slot_ready[b], 1);
            mbar_init(&slot_free[b], PT_NCONV + PT_NSOFT);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&q_ready[b], 1);
            mbar_init(&q_free[b], 1);
        }
        for (int b = 0; b < PT_NTB; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&o_full[b], 1);
            mbar_init(&tmem_free[b], PT_NSOFT);
        }
        mbar_init(&p_ready[0], PT_NSOFT);
        mbar_init(&p_ready[1], PT_NSOFT);
        mbar_init(vw_ready, 1);
        mbar_init(mma_done, 1);
        *s_timeout = 0;
        fence_mbar_init();
    }
    // window tiles start as zeros (a masked row still meets P = 0 in P V, so it
    // must hold a finite value)
    for (int i = tid; i < 2 * (int)PT_TILE / 16; i += PT_THREADS)
        reinterpret_cast<uint4*>(smem + PT_OFF_KW)[i] = make_uint4(0, 0, 0, 0);
    if (wid == PT_W_MMA) {
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
    // window of a query: tokens [lo, p] (lo = p + 1: none, when its rows are not all in swa_kv)
    auto window_of = [&](int q) -> int2 {
        const int p = __ldg(a.q_pos + q);
        const int lo = max(0, p - a.window + 1);
        return make_int2(lo < a.swa_start ? p + 1 : lo, p);
    };
    // the sequence's first pages (its whole table, when it fits)
    const int n_ptab = min(a.cache.max_pages_per_seq, PT_PTAB);
    for (int i = tid; i < n_ptab; i += PT_THREADS) s_ptab[i] = __ldg(a.cache.page_table + i);
    // every row of the first query's window (later queries add their new tokens)
    if (nq > 0) {
        const int2 w0 = window_of(q0);
        for (int c = tid; c < (w0.y - w0.x + 1) * 32; c += PT_THREADS) {
            const int tok = w0.x + (c >> 5), ch = c & 31;
            const uint4 x = __ldg(reinterpret_cast<const uint4*>(a.swa + (int64_t)(tok - a.swa_start) * kCh) + ch);
            win_store(smem + (ch < 16 ? PT_OFF_KW : PT_OFF_VW), tok & 127, ch & 15, x);
        }
    }
    fence_proxy_async_smem();  // the rows are read by the tensor core
    __syncthreads();
    auto wait = [&](uint64_t* bar, uint32_t parity) {  // bounded; after one timeout every wait returns at once
        if (*s_timeout) return;
        if (!mbar_wait(bar, parity, kPtWaitLimit)) *s_timeout = 1;
    };

    if (wid == PT_W_MMA) {
        // ================= MMA issue: S(0), then S(j + 1) before O(j) =================
        if (lane == 0 && nq > 0) {
            uint32_t pos = 0;  // ring position
            auto mma_s = [&](int j) {  // S^T(j) = K^ Q^T over the 4 selected tiles and the window tile
                const int qb = j & 1, tb = j & (PT_NTB - 1);
                wait(&q_ready[qb], (uint32_t)(j >> 1) & 1u);
                if (j >= PT_NTB) wait(&tmem_free[tb], (uint32_t)((j / PT_NTB) - 1) & 1u);
                tc_fence_after();
                const uint32_t tS = tmem + (uint32_t)tb * 128u;
                const uint32_t qaddr = smem_u32(smem + PT_OFF_Q + (size_t)qb * 4096);
                for (int t = 0; t < PT_TILES; ++t) {
                    uint32_t ka;
                    int s = -1;
                    if (t < 4) {
                        s = (int)(pos % PT_NSLOT);
                        wait(&full[s], (pos / PT_NSLOT) & 1u);
                        tc_fence_after();
                        ka = smem_u32(smem + PT_OFF_RING + (size_t)s * PT_TILE);
                    } else {
                        ka = smem_u32(smem + PT_OFF_KW);  // written with Q (q_ready)
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
                umma_commit(&s_full[tb]);
            };
            auto mma_o = [&](int j) {  // O^T(j) = V^T P^T over the 4 selected tiles and the window tile
                const int tb = j & (PT_NTB - 1);
                wait(&p_ready[j & 1], (uint32_t)(j >> 1) & 1u);
                wait(vw_ready, (uint32_t)j & 1u);
                tc_fence_after();
                const uint32_t tO = tmem + (uint32_t)tb * 128u + 96u;
                for (int t = 0; t < PT_TILES; ++t) {
                    uint32_t va;
                    int s = -1;
                    if (t < 4) {
                        s = (int)(pos % PT_NSLOT);
                        wait(&full[s], (pos / PT_NSLOT) & 1u);
                        tc_fence_after();
                        va = smem_u32(smem + PT_OFF_RING + (size_t)s * PT_TILE);
                    } else {
                        va = smem_u32(smem + PT_OFF_VW);
                    }
                    const uint32_t pa = smem_u32(smem + PT_OFF_P + ((size_t)(j & 1) * PT_TILES + t) * PT_PTILE);
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
                umma_commit(&o_full[tb]);
            };
            mma_s(0);
            for (int j = 0; j < nq; ++j) {
                if (j + 1 < nq) mma_s(j + 1);
                mma_o(j);
            }
            umma_commit(mma_done);
            wait(mma_done, 0u);
        }
        __syncwarp();
    } else if (wid >= PT_W_SETUP && wid < PT_W_SETUP + PT_NSETUP) {
        // ======= per query (three warps in turn): slots, window range, Q, new window rows =======
        // physical slot of an entry (pos >= 0), the page from the cached table when it is there
        auto slot_of = [&](int32_t pos) -> int32_t {
            const int32_t pg = pos >> a.page_shift;
            if (pg >= n_ptab) return (int32_t)entry_slot(a.cache, a.page_shift, 0, pos, a.err);
            const int32_t phys = s_ptab[pg];
            if (phys < 0 || phys >= a.cache.n_phys_pages) {
                dev_error(a.err, CSA2_DEV_PAGE);
                return -1;
            }
            return (phys << a.page_shift) | (pos & ((1 << a.page_shift) - 1));
        };
        for (int j = wid - PT_W_SETUP; j < nq; j += PT_NSETUP) {
            const int q = q0 + j, b = j % PT_NQB, qb = j & 1;
            const int2 win = window_of(q);
            // the tokens of this window that the previous query's window lacks:
            // [win.x, min(win.y, prev.x - 1)] and [max(win.x, prev.y + 1), win.y]
            // (an empty window is [p + 1, p]; the first query's was written whole)
            const int2 prev = j == 0 ? win : window_of(q - 1);
            const int a0 = win.x, a1 = min(win.y, prev.x - 1), b0 = max(win.x, prev.y + 1), b1 = win.y;
            const int n1 = max(0, a1 - a0 + 1), n_new = n1 + max(0, b1 - b0 + 1);
            auto new_tok = [&](int k) { return k < n1 ? a0 + k : b0 + (k - n1); };
            // every global load of the query in flight at once
            int32_t pos[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k = lane + 32 * i;
                pos[i] = k < a.topk ? __ldg(a.idx + (int64_t)q * a.topk + k) : -1;
            }
            uint4 qv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) qv[i] = __ldg(reinterpret_cast<const uint4*>(a.q + (int64_t)q * kH * kD) + lane + 32 * i);
            uint4 wx = make_uint4(0, 0, 0, 0);  // chunk `lane` of the first new token's row (K: lanes < 16)
            if (n_new > 0)
                wx = __ldg(reinterpret_cast<const uint4*>(a.swa + (int64_t)(new_tok(0) - a.swa_start) * kCh) + lane);
            if (j >= PT_NQB) wait(&slot_free[b], (uint32_t)((j / PT_NQB) - 1) & 1u);
            int32_t* sl = s_slot + b * 512;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                int32_t slot = -1;
                if (pos[i] >= 0) {
                    if (pos[i] < L) slot = slot_of(pos[i]);
                    else dev_error(a.err, CSA2_DEV_INDEX);
                }
                sl[lane + 32 * i] = slot;
            }
            if (lane == 0) {
                if (win.x > win.y) dev_error(a.err, CSA2_DEV_INDEX);  // the window's rows are not all in swa_kv
                s_win[b] = win;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&slot_ready[b]);
            // Q: 16 heads x 128 dims, fp16, half h of the dims at +2 KiB, head rows of 128 B
            if (j >= 2) wait(&q_free[qb], (uint32_t)((j >> 1) - 1) & 1u);
            uint8_t* qt = smem + PT_OFF_Q + (size_t)qb * 4096;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i, h = e >> 4, c8 = e & 15, half = c8 >> 3, c = c8 & 7;
                *reinterpret_cast<uint4*>(qt + half * 2048 + h * 128 + ((c ^ (h & 7)) << 4)) =
                    make_uint4(bf2_to_h2(qv[i].x), bf2_to_h2(qv[i].y), bf2_to_h2(qv[i].z), bf2_to_h2(qv[i].w));
            }
            // the new K rows, once the previous query's S has read the window tile.
            // The per-query barriers of the TMEM buffers say so without aliasing:
            // the two setup warps take turns, so a barrier completed once per
            // query may be two phases behind this warp's last wait on it.
            if (j >= 1) wait(&s_full[(j - 1) & (PT_NTB - 1)], (uint32_t)((j - 1) / PT_NTB) & 1u);
            for (int k = 0; k < n_new; ++k) {
                const int tok = new_tok(k);
                const uint4 x = k == 0 ? wx
                                       : __ldg(reinterpret_cast<const uint4*>(a.swa + (int64_t)(tok - a.swa_start) * kCh) +
                                               lane);
                if (lane < 16) win_store(smem + PT_OFF_KW, tok & 127, lane, x);  // V chunks: below
            }
            fence_proxy_async_smem();  // Q and the rows are read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_ready[qb]);
            // the new V rows, once the previous query's O has read the window tile
            if (j >= 1) wait(&o_full[(j - 1) & (PT_NTB - 1)], (uint32_t)((j - 1) / PT_NTB) & 1u);
            for (int k = 0; k < n_new; ++k) {
                const int tok = new_tok(k);
                const uint4 x = k == 0 ? wx
                                       : __ldg(reinterpret_cast<const uint4*>(a.swa + (int64_t)(tok - a.swa_start) * kCh) +
                                               lane);
                if (lane >= 16) win_store(smem + PT_OFF_VW, tok & 127, lane - 16, x);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(vw_ready);
        }
    } else if (wid >= PT_W_CONV) {
        // ============ converters: FP4 rows -> fp16 operand tiles ============
        // Thread ct owns quarter qt (channels 32 qt .. 32 qt + 31 of K or V) of
        // entry e0 = ct / 4 of every tile.  The tiles come in blocks of four (one
        // query's K or V): K(0), then K(j + 1), V(j) for each j.  Block b + 1's
        // rows are loaded while block b is converted.
        const int ct = tid - PT_W_CONV * 32, qt = ct & 3, hq = qt >> 1, cq = (qt & 1) * 4, e0 = ct >> 2;
        const int nb = 2 * nq;
        auto block_of = [&](int b, int& j, int& v) {
            if (b == 0) {
                j = 0, v = 0;
                return;
            }
            const int i = b - 1, p = i >> 1;
            if (p == nq - 1) j = nq - 1, v = 1;
            else if (i & 1) j = p, v = 1;
            else j = p + 1, v = 0;
        };
        struct Row {
            uint4 c;     // 16 code bytes of the entry (zeros: absent)
            uint32_t s;  // word qt of the entry's 16 scale bytes (K's 8, then V's)
        };
        // The scale words of a query's K block serve its V block too: lanes 2, 3
        // of an entry's four hold V's scales.  Kept per query parity (V(j) follows K(j + 1)).
        uint32_t sv0[4], sv1[4];
        int seen = -1;  // last query whose slot list was waited for
        auto fetch_block = [&](int b, Row (&R)[4]) {
            int j, v;
            block_of(b, j, v);
            if (j > seen) {
                wait(&slot_ready[j % PT_NQB], (uint32_t)(j / PT_NQB) & 1u);
                seen = j;
            }
            const int32_t* sl = s_slot + (j % PT_NQB) * 512 + e0;
            int32_t slot[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) slot[t] = sl[t * 128];
            if (v == 1) {  // query j's slot list is read
                __syncwarp();
                if (lane == 0) mbar_arrive(&slot_free[j % PT_NQB]);
            }
            const uint8_t* cbase = a.cache.codes + v * 64 + qt * 16;
            const uint8_t* sbase = a.cache.scales + qt * 4;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                uint4 c = make_uint4(0u, 0u, 0u, 0u);
                if (slot[t] >= 0) c = __ldg(reinterpret_cast<const uint4*>(cbase + (int64_t)slot[t] * kCodeBytes));
                R[t].c = c;
                if (v == 0) {
                    uint32_t w = 0u;
                    if (slot[t] >= 0) w = __ldg(reinterpret_cast<const uint32_t*>(sbase + (int64_t)slot[t] * kScales));
                    R[t].s = w;
                    if (j & 1) sv1[t] = w;
                    else sv0[t] = w;
                } else {
                    R[t].s = (j & 1) ? sv1[t] : sv0[t];
                }
            }
        };
        auto convert_tile = [&](int m, int v, const Row& R) {
            const int s = m % PT_NSLOT;
            if (m >= PT_NSLOT) wait(&empty[s], (uint32_t)((m / PT_NSLOT) - 1) & 1u);
            uint8_t* dst = smem + PT_OFF_RING + (size_t)s * PT_TILE + (size_t)hq * PT_HALF + e0 * 128;
            // this quarter's two scale bytes: word 2 v + qt / 2 of the entry, from its lane
            const uint32_t wsc = __shfl_sync(0xffffffffu, R.s, (lane & ~3) | (2 * v + (qt >> 1)));
            const uint32_t b2 = (wsc >> (16 * (qt & 1))) & 0xffffu;
            // both scales of the quarter in one conversion, each then in both halves
            const __half2_raw sh = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)b2, __NV_E4M3);
            const uint32_t s2 = (uint32_t)sh.x | ((uint32_t)sh.y << 16);
            const uint32_t sc_lo = __byte_perm(s2, 0u, 0x1010), sc_hi = __byte_perm(s2, 0u, 0x3232);
            const uint32_t w[4] = {R.c.x, R.c.y, R.c.z, R.c.w};
            const bool rot = qt >> 1;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // the two quarters of one half store in rotated order (word
                // i + 2), so their chunks sit in other banks
                const int wi = rot ? (i + 2) & 3 : i;
                const uint32_t sc = (rot ? ((i + 2) & 3) >> 1 : i >> 1) ? sc_hi : sc_lo;
                uint32_t h0, h1, h2, h3;
                e2m1x8_to_h2x4(rot ? w[(i + 2) & 3] : w[i], h0, h1, h2, h3);
                *reinterpret_cast<uint4*>(dst + (((cq + wi) ^ (e0 & 7)) << 4)) =
                    make_uint4(hmul2(h0, sc), hmul2(h1, sc), hmul2(h2, sc), hmul2(h3, sc));
            }
            fence_proxy_async_smem();  // the tile is read by the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
        };
        Row RA[4], RB[4];
        if (nb > 0) fetch_block(0, RA);
        for (int b = 0; b < nb; b += 2) {
            if (b + 1 < nb) fetch_block(b + 1, RB);
            int jj, va, vb;
            block_of(b, jj, va);
#pragma unroll
            for (int t = 0; t < 4; ++t) convert_tile(4 * b + t, va, RA[t]);
            if (b + 1 >= nb) break;
            if (b + 2 < nb) fetch_block(b + 2, RA);
            block_of(b + 1, jj, vb);
#pragma unroll
            for (int t = 0; t < 4; ++t) convert_tile(4 * (b + 1) + t, vb, RB[t]);
        }
    } else {
        // ============ softmax and epilogue: warps 0-7 ============
        // warp w: TMEM lane quarter w & 3 (thread = key r of a tile for S, dim r
        // for O) and heads 8 hg .. 8 hg + 7, hg = w >> 2; per-head max and sum
        // across the 4 warps of a head group
        const int wq = wid & 3, hg = wid >> 2, r = 32 * wq + lane;
        const GroupBar sb{1, 32 * PT_NSOFT};
        const uint32_t lane_base = tmem + ((uint32_t)(32 * wq) << 16) + 8u * (uint32_t)hg;
        const float kScaleLog2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
        auto epilogue = [&](int jj) {  // O(jj) (thread = dim) / sum -> out; its TMEM buffer is free after
            const uint32_t tb = (uint32_t)jj & (PT_NTB - 1);
            uint32_t ov[8];
            tmem_ld8(lane_base + tb * 128u + 96u, ov);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_free[tb]);
            float* out = a.out + ((int64_t)(q0 + jj) * kH + 8 * hg) * kD;
#pragma unroll
            for (int hh = 0; hh < 8; ++hh)
                out[hh * kD + r] = __uint_as_float(ov[hh]) * s_inv[(jj & 1) * 16 + 8 * hg + hh];
        };
        for (int j = 0; j < nq; ++j) {
            const int q = q0 + j, tb = j & (PT_NTB - 1), wb = j % PT_NQB;
            // the slots and the window of this query (setup warp), then its scores
            wait(&slot_ready[wb], (uint32_t)(j / PT_NQB) & 1u);
            wait(&s_full[tb], (uint32_t)(j / PT_NTB) & 1u);
            tc_fence_after();
            const int32_t* sl = s_slot + wb * 512;
            const int2 win = s_win[wb];
            // window row r holds the token of [p - 127, p] congruent to it
            const int wtok = win.y - ((win.y - r) & 127);
            const bool wok = wtok >= win.x;
            const uint32_t tS = lane_base + (uint32_t)tb * 128u;
            // pass 1: the per-head maximum over the 640 keys (log2 domain)
            float m[8];
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) m[hh] = -INFINITY;
#pragma unroll 1
            for (int t = 0; t < PT_TILES; ++t) {
                const bool ok = t < 4 ? sl[t * 128 + r] >= 0 : wok;
                uint32_t v[8];
                tmem_ld8(tS + 16u * t, v);
                tmem_wait_ld();
                if (ok)
#pragma unroll
                    for (int hh = 0; hh < 8; ++hh) m[hh] = fmaxf(m[hh], __uint_as_float(v[hh]) * kScaleLog2);
            }
#pragma unroll
            for (int hh = 0; hh < 8; ++hh)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m[hh] = fmaxf(m[hh], __shfl_xor_sync(0xffffffffu, m[hh], o));
            // alternate buffers: a fast warp's next query never overwrites this one
            float* red = s_red + (j & 1) * 64 + hg * 32;
            if (lane == 0)
#pragma unroll
                for (int hh = 0; hh < 8; ++hh) red[wq * 8 + hh] = m[hh];
            sb.sync();
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) m[hh] = fmaxf(fmaxf(red[hh], red[8 + hh]), fmaxf(red[16 + hh], red[24 + hh]));
            // P^T buffer j & 1 was read by O(j - 2), waited for before the epilogue of j - 2
            // pass 2: P = exp2(S - max) as fp16 into P^T, and the per-head sums
            float l[8];
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) l[hh] = 0.f;
            uint8_t* pt = smem + PT_OFF_P + (size_t)(j & 1) * PT_TILES * PT_PTILE;
            const int ke = r & ~1, odd = r & 1;
#pragma unroll 1
            for (int t = 0; t < PT_TILES; ++t) {
                const bool ok = t < 4 ? sl[t * 128 + r] >= 0 : wok;
                uint32_t v[8];
                tmem_ld8(tS + 16u * t, v);
                tmem_wait_ld();
                // P^T tile t: [key half][16 heads][128 B], key k of head h at chunk ((k & 63) >> 3) ^ (h & 7);
                // lanes r and r ^ 1 pair up: the even lane stores heads 8 hg + 0..3, the odd one 8 hg + 4..7
                uint8_t* ptt = pt + (size_t)t * PT_PTILE + (size_t)(r >> 6) * 2048;
#pragma unroll
                for (int i = 0; i < 4; ++i) {  // heads 8 hg + i and 8 hg + 4 + i
                    const float p0 = (ok && m[i] != -INFINITY) ? ex2(__uint_as_float(v[i]) * kScaleLog2 - m[i]) : 0.f;
                    const float p1 =
                        (ok && m[4 + i] != -INFINITY) ? ex2(__uint_as_float(v[4 + i]) * kScaleLog2 - m[4 + i]) : 0.f;
                    l[i] += p0;
                    l[4 + i] += p1;
                    const int hs = 8 * hg + (odd ? 4 + i : i);  // head this lane stores
                    const float mine = odd ? p1 : p0, give = odd ? p0 : p1;
                    const float got = __shfl_xor_sync(0xffffffffu, give, 1);
                    const float lo = odd ? got : mine, hi = odd ? mine : got;  // keys ke, ke + 1
                    *reinterpret_cast<uint32_t*>(ptt + hs * 128 + ((((ke & 63) >> 3) ^ (hs & 7)) << 4) + (ke & 7) * 2) =
                        f2_to_h2(lo, hi);
                }
            }
            fence_proxy_async_smem();  // P^T is read by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&p_ready[j & 1]);
                mbar_arrive(&slot_free[wb]);
            }
#pragma unroll
            for (int hh = 0; hh < 8; ++hh)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], o);
            sb.sync();  // every warp has read the maxima: the buffer takes the sums
            if (lane == 0)
#pragma unroll
                for (int hh = 0; hh < 8; ++hh) red[wq * 8 + hh] = l[hh];
            sb.sync();
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) l[hh] = (red[hh] + red[8 + hh]) + (red[16 + hh] + red[24 + hh]);
            if (wq == 0 && lane < 8) {  // lse of head 8 hg + lane
                float lt = 0.f, mt = 0.f;
#pragma unroll
                for (int hh = 0; hh < 8; ++hh)
                    if (hh == lane) {
                        lt = l[hh];
                        mt = m[hh];
                    }
                a.lse[(int64_t)q * kH + 8 * hg + lane] = lt > 0.f ? (mt + log2f(lt)) * 0.6931471805599453f : -INFINITY;
            }
            if (j >= 1) {
                wait(&o_full[(j - 1) & (PT_NTB - 1)], (uint32_t)((j - 1) / PT_NTB) & 1u);
                tc_fence_after();
                epilogue(j - 1);
            }
            if (wq == 0 && lane < 8) {  // 1 / sum of this query, read by its epilogue (after two more barriers)
                float lt = 0.f;
#pragma unroll
                for (int hh = 0; hh < 8; ++hh)
                    if (hh == lane) lt = l[hh];
                s_inv[(j & 1) * 16 + 8 * hg + lane] = lt > 0.f ? 1.f / lt : 0.f;
            }
        }
        if (nq > 0) {
            wait(&o_full[(nq - 1) & (PT_NTB - 1)], (uint32_t)((nq - 1) / PT_NTB) & 1u);
            tc_fence_after();
            epilogue(nq - 1);
        }
    }
    tc_fence_before();
    __syncthreads();  // every accumulator has been read
    if (wid == PT_W_MMA) {
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
    // slots are kept as int32
    if ((a.cache.n_phys_pages << a.page_shift) > INT32_MAX) return cudaErrorInvalidValue;
    LaunchCfg c(dim3((unsigned)std::min(a.rows, n_ctas)), dim3(PT_THREADS), PT_SMEM, stream);
    return cudaLaunchKernelEx(&c.cfg, prefill_attn_tc_kernel, a);
}

}  // namespace csa2
