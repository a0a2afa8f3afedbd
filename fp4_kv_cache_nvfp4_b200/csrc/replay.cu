// SWA Bounded Replay, attention part: recompute a layer's 128-token SWA window
// K|V rows from the tokens' hidden states instead of keeping them.
//
// Pages: "FP4 KV, repeticion limitada y otras extensiones" (7minutos.es): on a
// miss, only 128 tokens are recomputed; "Como funciona" (e-cogni.com.br): SWA
// Bounded Replay avoids persisting the SWA cache at the cost of a small
// recompute in prefill.  The projection weights are synthetic here (the pages'
// trained weights are not available); the arithmetic is the same:
//   swa[b][(p) % window][c] = bf16( sum_k h[b][t][k] * w_kv[c][k] ),
// p = L_b - n_b + t the position of row t of the last n_b = min(window, L_b)
// tokens, c = 0..255 (K channels 0..127, V channels 128..255), fp32
// accumulation, round to nearest even.
//
// A cluster of 4 CTAs per (sequence, slice of 64 of the 256 channels), the
// cluster's CTAs splitting d_model four ways, so a layer's replay of B
// sequences spreads over 16 B SMs and every CTA reads a quarter of the
// hidden states it needs: D_r[128 tokens x 64 ch] = H[128 x d_r] .
// W_slice[64 x d_r]^T over its quarter d_r, tcgen05.mma kind::f16 (bf16 x bf16
// -> fp32, M 128, N 64, K 16), the fp32 partial in 64 TMEM columns.  The four
// partials meet through distributed shared memory: CTA r owns channels
// 16 r .. 16 r + 15 of the slice and receives the other three CTAs' partials
// of them (8 KiB each, asynchronous remote stores counted in bytes on its
// mbarrier: no cluster barrier after the products), then sums the four in rank
// order (fixed, so the result does not depend on timing) and rounds once to
// bf16.
//   warp 0   producer: one lane loads 64-dim slices of H and W_slice as
//            128-byte-swizzled TMA tensor boxes (no multicast) into a 7-stage
//            ring, completion counted in bytes on the stage's mbarrier;
//   warp 1   MMA: allocates TMEM, one lane issues 4 MMAs per slice and commits
//            to the stage's "empty" barrier, and to "done" after the last;
//   warps 2-5  epilogue: warp w owns TMEM lane quarter w % 4 (one token per
//            thread): it stores the three foreign 16-channel parts of its rows
//            into their owners' shared memory, and once its own mbarrier has
//            counted the peers' 24 KiB sums the four partials of its own part
//            and stores the bf16 row part.
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

constexpr int RP_M = 128;       // tokens per CTA (the window)
constexpr int RP_N = 64;        // channels per CTA
constexpr int RP_SLICES = kCh / RP_N;  // channel slices per sequence
constexpr int RP_KSPLIT = 4;    // CTAs of a cluster, splitting d_model
constexpr int RP_OWN = RP_N / RP_KSPLIT;  // channels each CTA of the cluster sums and stores
constexpr int RP_KS = 64;       // d_model slice per stage (128 B of bf16)
constexpr int RP_STAGES = 7;
constexpr int RP_THREADS = 6 * 32;
constexpr uint32_t RP_TILE = RP_M * RP_KS * 2;           // 16 KiB: H slice [128 tokens][64 dims]
constexpr uint32_t RP_TILE_B = RP_N * RP_KS * 2;         // 8 KiB: W slice [64 channels][64 dims]
constexpr size_t RP_OFF_A = 0;                           // [stages][128][128 B]
constexpr size_t RP_OFF_B = RP_OFF_A + (size_t)RP_STAGES * RP_TILE;    // [stages][64][128 B]
constexpr size_t RP_OFF_RED = RP_OFF_B + (size_t)RP_STAGES * RP_TILE_B;  // [source rank][4][128 rows][16 B]
constexpr size_t RP_OFF_BAR = RP_OFF_RED + (size_t)RP_KSPLIT * RP_M * RP_OWN * 4;  // full[] empty[] done recv
constexpr uint32_t RP_RECV_BYTES = (uint32_t)(RP_KSPLIT - 1) * RP_M * RP_OWN * 4;   // 24 KiB from the peers
constexpr size_t RP_OFF_MISC = RP_OFF_BAR + (2 * RP_STAGES + 2) * 8;   // tmem base, timeout
constexpr size_t RP_SMEM = RP_OFF_MISC + 16 + 1024;                    // + slack to align the base to 1 KiB
constexpr uint32_t kReplayWaitLimit = 1u << 22;
static_assert(RP_OWN == 16, "one 16-column TMEM load per owner part");
static_assert(RP_SMEM <= 227 * 1024, "shared memory");

struct ReplayArgs {
    const int32_t* seq_lens;
    uint16_t* swa;  // [B][window][256]
    int32_t* err;
    int B, d_model, window;
};

__global__ void __launch_bounds__(RP_THREADS, 1) swa_replay_kernel(const __grid_constant__ CUtensorMap map_h,
                                                                    const __grid_constant__ CUtensorMap map_w,
                                                                    ReplayArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 128-byte-swizzled tiles need a 1 KiB-aligned base: round up inside the
    // slack (the same offset in every CTA, so peer addresses line up)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + RP_OFF_BAR);
    uint64_t* empty = full + RP_STAGES;
    uint64_t* done = empty + RP_STAGES;
    uint64_t* recv = done + 1;  // the peers' partials of this CTA's channels, counted in bytes
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + RP_OFF_MISC);
    int* s_timeout = reinterpret_cast<int*>(smem + RP_OFF_MISC + 4);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // blockIdx.x = (b * RP_SLICES + slice) * RP_KSPLIT + rank; clusters are RP_KSPLIT consecutive CTAs
    const int rank = (int)(blockIdx.x % RP_KSPLIT);
    const int b = (int)(blockIdx.x / (RP_KSPLIT * RP_SLICES));
    const int n0 = (int)((blockIdx.x / RP_KSPLIT) % RP_SLICES) * RP_N;
    const int nk = a.d_model / RP_KS;
    const int k_begin = rank * nk / RP_KSPLIT, my_nk = (rank + 1) * nk / RP_KSPLIT - k_begin;

    if (tid == 0) {
        for (int s = 0; s < RP_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(recv, 1);
        mbar_arrive_expect_tx(recv, RP_RECV_BYTES);
        *s_timeout = 0;
        fence_mbar_init();
    }
    if (wid == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(RP_N)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every CTA of the cluster has started before any peer stores reach it:
    // arrive now, wait just before the first remote store
    cluster_arrive();
    const uint32_t tmem = *s_tmem;
    pdl_wait();  // the hidden states come from the preceding kernel
    pdl_trigger();
    // the sequence length, read early by the epilogue warps (its latency hides behind the products)
    const int32_t L = wid >= 2 ? a.seq_lens[b] : 0;

    if (wid == 0) {
        // ================= producer: TMA boxes of H and W =================
        if (lane == 0) {
            for (int i = 0; i < my_nk; ++i) {
                const int s = i % RP_STAGES;
                if (i >= RP_STAGES &&
                    !mbar_wait(&empty[s], (uint32_t)((i / RP_STAGES) - 1) & 1u, kReplayWaitLimit))
                    *s_timeout = 1;
                mbar_arrive_expect_tx(&full[s], RP_TILE + RP_TILE_B);
                // x = 64 i dims (128 B multiples), y = first row of the box
                const int x = (k_begin + i) * RP_KS;
                tma_load_2d(smem + RP_OFF_A + (size_t)s * RP_TILE, &map_h, x, b * a.window, &full[s]);
                tma_load_2d(smem + RP_OFF_B + (size_t)s * RP_TILE_B, &map_w, x, n0, &full[s]);
            }
            // the last stages' boxes have landed before this thread leaves (bounded)
            for (int i = max(0, my_nk - RP_STAGES); i < my_nk; ++i)
                if (!mbar_wait(&full[i % RP_STAGES], (uint32_t)(i / RP_STAGES) & 1u, kReplayWaitLimit))
                    *s_timeout = 1;
        }
        __syncwarp();
    } else if (wid == 1) {
        // ================= MMA issue =================
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(RP_N >> 3) << 17) |
                                   ((uint32_t)(RP_M >> 4) << 24);  // bf16 x bf16 -> f32, K-major, M 128, N 64
            for (int i = 0; i < my_nk; ++i) {
                const int s = i % RP_STAGES;
                if (!mbar_wait(&full[s], (uint32_t)(i / RP_STAGES) & 1u, kReplayWaitLimit)) *s_timeout = 1;
                tc_fence_after();
                const uint64_t da = umma_desc_sw128(smem_u32(smem + RP_OFF_A + (size_t)s * RP_TILE));
                const uint64_t db = umma_desc_sw128(smem_u32(smem + RP_OFF_B + (size_t)s * RP_TILE_B));
#pragma unroll
                for (int kk = 0; kk < RP_KS / 16; ++kk)  // +32 B per k-step of 16
                    umma_bf16(tmem, da + 2u * kk, db + 2u * kk, idesc, (i | kk) > 0 ? 1u : 0u);
                umma_commit(&empty[s]);
            }
            if (my_nk > 0)
                umma_commit(done);
            else
                mbar_arrive(done);  // no products: the epilogue takes a zero partial
        }
        __syncwarp();
    }

    // ================= exchange: the partials of each owner's 16 channels =================
    // Receive area [source rank][chunk c of 4 floats][128 rows][16 B]: one warp's store of a
    // chunk is 512 contiguous bytes, and the owner's reads of a chunk by consecutive rows are
    // free of bank conflicts.
    const int quarter = wid & 3, t = 32 * quarter + lane;  // epilogue warps: TMEM lane quarter, token row
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
    auto red_off = [](int src, int row, int c) { return (uint32_t)(((src * 4 + c) * RP_M + row) * 16); };
    uint32_t part[RP_KSPLIT][RP_OWN];  // this thread's row of the CTA's partial, by owner
    if (wid >= 2) {
        if (!mbar_wait(done, 0u, kReplayWaitLimit)) *s_timeout = 1;
        tc_fence_after();
#pragma unroll
        for (int r = 0; r < RP_KSPLIT; ++r) tmem_ld16(lane_base + (uint32_t)(r * RP_OWN), part[r]);
        tmem_wait_ld();
        if (my_nk == 0)  // d_model split four ways left this CTA nothing: its partial is zero
#pragma unroll
            for (int r = 0; r < RP_KSPLIT; ++r)
#pragma unroll
                for (int e = 0; e < RP_OWN; ++e) part[r][e] = 0u;
    }
    __syncwarp();
    cluster_wait();  // the peers have started (their receive areas exist)
    if (wid >= 2) {
        const uint32_t red_local = smem_u32(smem + RP_OFF_RED);
        // rounds j = 1, 2, 3 to owner rank + j: the four CTAs store to different peers at a
        // time (the owner's part is picked by selects, so `part` stays in registers)
#pragma unroll
        for (int j = 1; j < RP_KSPLIT; ++j) {
            const int r = (rank + j) % RP_KSPLIT;
            float v[RP_OWN];
#pragma unroll
            for (int e = 0; e < RP_OWN; ++e) {
                uint32_t x = part[0][e];
#pragma unroll
                for (int q = 1; q < RP_KSPLIT; ++q) x = r == q ? part[q][e] : x;
                v[e] = __uint_as_float(x);
            }
            const uint32_t ra = mapa_shared(red_local, (uint32_t)r);
            const uint32_t rb = mapa_shared(smem_u32(recv), (uint32_t)r);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                st_async_f32x4(ra + red_off(rank, t, c), make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]),
                               rb);
        }
    }
    // no barrier: an owner waits only for the bytes it receives (the senders' stores complete on its
    // mbarrier; a CTA leaves only after its own partials arrived, so every store finds its target)
    if (wid >= 2 && !mbar_wait_cluster(recv, 0u, kReplayWaitLimit)) *s_timeout = 1;

    if (wid >= 2) {
        // ================= sum in rank order, round to bf16, store =================
        const int n_b = L < 1 ? 0 : min(L, a.window);
        if (L < 1 && lane == 0 && quarter == 0 && n0 == 0 && rank == 0) dev_error(a.err, CSA2_DEV_LEN);
        float acc[RP_OWN];
#pragma unroll
        for (int e = 0; e < RP_OWN; ++e) acc[e] = 0.f;
        const uint8_t* red = smem + RP_OFF_RED;
#pragma unroll
        for (int src = 0; src < RP_KSPLIT; ++src) {
            if (src == rank) {
#pragma unroll
                for (int e = 0; e < RP_OWN; ++e) acc[e] += __uint_as_float(part[src][e]);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 x = *reinterpret_cast<const float4*>(red + red_off(src, t, c));
                    acc[4 * c] += x.x;
                    acc[4 * c + 1] += x.y;
                    acc[4 * c + 2] += x.z;
                    acc[4 * c + 3] += x.w;
                }
            }
        }
        uint32_t pk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
            pk[j] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        if (t < n_b) {
            const int64_t p = (int64_t)L - n_b + t;  // position of this row's token
            uint16_t* dst = a.swa + ((int64_t)b * a.window + (p % a.window + a.window) % a.window) * kCh + n0 +
                            rank * RP_OWN;
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
    }
    tc_fence_before();
    __syncthreads();  // every accumulator has been read
    if (wid == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(RP_N) : "memory");
    }
    if (tid == 0 && *s_timeout) dev_error(a.err, CSA2_DEV_TIMEOUT);
}

// A row-major bf16 matrix [rows][cols] as a 2-D tensor read in boxes of 64
// columns x box_rows rows, 128-byte swizzled.
static bool bf16_rows_map(const uint16_t* base, int64_t rows, int64_t cols, uint32_t box_rows, CUtensorMap* map) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)RP_KS, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace csa2

extern "C" CSA2_API csa2_status csa2_swa_replay(const uint16_t* h, const uint16_t* w_kv, const int32_t* seq_lens,
                                                uint16_t* swa_kv, int32_t B, int32_t d_model, int32_t window,
                                                int32_t* err_word, void* stream) {
    using namespace csa2;
    if (B < 0 || !h || !w_kv || !seq_lens || !swa_kv) return CSA2_ERR_INVALID_ARG;
    if (window < 1 || window > kMaxWindow) return CSA2_ERR_INVALID_ARG;
    if (d_model < RP_KS || d_model % RP_KS || d_model > (1 << 16)) return CSA2_ERR_UNSUPPORTED;
    auto al = [](const void* p, uintptr_t m) { return (reinterpret_cast<uintptr_t>(p) & (m - 1)) == 0; };
    if (!al(h, 16) || !al(w_kv, 16) || !al(swa_kv, 16) || !al(seq_lens, 4) || (err_word && !al(err_word, 4)))
        return CSA2_ERR_INVALID_ARG;
    if (B == 0) return CSA2_OK;
    static bool init[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    if (!init[dev]) {
        if (cudaFuncSetAttribute((const void*)swa_replay_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)RP_SMEM) != cudaSuccess) {
            (void)cudaGetLastError();
            return CSA2_ERR_CUDA;
        }
        init[dev] = true;
    }
    CUtensorMap mh, mw;
    memset(&mh, 0, sizeof(mh));
    memset(&mw, 0, sizeof(mw));
    if (!bf16_rows_map(h, (int64_t)B * window, d_model, RP_M, &mh) ||
        !bf16_rows_map(w_kv, kCh, d_model, RP_N, &mw))
        return CSA2_ERR_CUDA;
    ReplayArgs a{seq_lens, swa_kv, err_word, B, d_model, window};
    LaunchCfg c(dim3((unsigned)B * RP_SLICES * RP_KSPLIT), dim3(RP_THREADS), RP_SMEM, (cudaStream_t)stream,
                RP_KSPLIT);
    if (cudaLaunchKernelEx(&c.cfg, swa_replay_kernel, mh, mw, a) != cudaSuccess) {
        (void)cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}
