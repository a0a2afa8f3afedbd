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
// accumulation on the tensor cores, round to nearest even.
//
// One CTA per (sequence, slice of 32 of the 256 channels), so a layer's
// replay of B sequences spreads over 8 B SMs: D[128 tokens x 32 ch] =
// H[128 x d_model] . W_slice[32 x d_model]^T as tcgen05.mma kind::f16 (bf16 x
// bf16 -> fp32, M 128, N 32, K 16), the fp32 accumulator in 32 TMEM columns.
// The slices of one sequence read the same hidden states (from L2 after the
// first).
//   warp 0   producer: one lane loads 64-dim slices of H and W_slice as
//            128-byte-swizzled TMA tensor boxes (no multicast) into a 4-stage
//            ring, completion counted in bytes on the stage's mbarrier;
//   warp 1   MMA: allocates TMEM, one lane issues 4 MMAs per slice and commits
//            to the stage's "empty" barrier, and to "done" after the last;
//   warps 2-5  epilogue: warp w reads TMEM lane quarter w % 4 (one token per
//            thread, 32 fp32 columns), rounds to bf16 and stores its part of
//            the row.
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa2 {

constexpr int RP_M = 128;       // tokens per CTA (the window)
constexpr int RP_N = 32;        // channels per CTA
constexpr int RP_SLICES = kCh / RP_N;  // CTAs per sequence
constexpr int RP_KS = 64;       // d_model slice per stage (128 B of bf16)
constexpr int RP_STAGES = 4;
constexpr int RP_THREADS = 6 * 32;
constexpr uint32_t RP_TILE = RP_M * RP_KS * 2;           // 16 KiB: H slice [128 tokens][64 dims]
constexpr uint32_t RP_TILE_B = RP_N * RP_KS * 2;         // 4 KiB: W slice [32 channels][64 dims]
constexpr size_t RP_OFF_A = 0;                           // [stages][128][128 B]
constexpr size_t RP_OFF_B = RP_OFF_A + (size_t)RP_STAGES * RP_TILE;    // [stages][32][128 B]
constexpr size_t RP_OFF_BAR = RP_OFF_B + (size_t)RP_STAGES * RP_TILE_B;  // full[4] empty[4] done
constexpr size_t RP_OFF_MISC = RP_OFF_BAR + (2 * RP_STAGES + 1) * 8;   // tmem base, timeout
constexpr size_t RP_SMEM = RP_OFF_MISC + 16 + 1024;                    // + slack to align the base to 1 KiB
constexpr uint32_t kReplayWaitLimit = 1u << 22;

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
    // 128-byte-swizzled tiles need a 1 KiB-aligned base: round up inside the slack
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + RP_OFF_BAR);
    uint64_t* empty = full + RP_STAGES;
    uint64_t* done = empty + RP_STAGES;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + RP_OFF_MISC);
    int* s_timeout = reinterpret_cast<int*>(smem + RP_OFF_MISC + 4);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int b = blockIdx.x / RP_SLICES, n0 = (blockIdx.x % RP_SLICES) * RP_N;
    const int nk = a.d_model / RP_KS;

    if (tid == 0) {
        for (int s = 0; s < RP_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
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
    const uint32_t tmem = *s_tmem;
    pdl_wait();  // the hidden states come from the preceding kernel
    pdl_trigger();

    if (wid == 0) {
        // ================= producer: TMA boxes of H and W =================
        if (lane == 0) {
            for (int i = 0; i < nk; ++i) {
                const int s = i % RP_STAGES;
                if (i >= RP_STAGES &&
                    !mbar_wait(&empty[s], (uint32_t)((i / RP_STAGES) - 1) & 1u, kReplayWaitLimit))
                    *s_timeout = 1;
                mbar_arrive_expect_tx(&full[s], RP_TILE + RP_TILE_B);
                // x = 64 i dims (128 B multiples), y = first row of the box
                tma_load_2d(smem + RP_OFF_A + (size_t)s * RP_TILE, &map_h, i * RP_KS, b * a.window, &full[s]);
                tma_load_2d(smem + RP_OFF_B + (size_t)s * RP_TILE_B, &map_w, i * RP_KS, n0, &full[s]);
            }
            // the last stages' boxes have landed before this thread leaves (bounded)
            for (int i = max(0, nk - RP_STAGES); i < nk; ++i)
                if (!mbar_wait(&full[i % RP_STAGES], (uint32_t)(i / RP_STAGES) & 1u, kReplayWaitLimit))
                    *s_timeout = 1;
        }
        __syncwarp();
    } else if (wid == 1) {
        // ================= MMA issue =================
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(RP_N >> 3) << 17) |
                                   ((uint32_t)(RP_M >> 4) << 24);  // bf16 x bf16 -> f32, K-major, M 128, N 32
            for (int i = 0; i < nk; ++i) {
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
            umma_commit(done);
        }
        __syncwarp();
    } else {
        // ================= epilogue: thread = token = TMEM lane, 32 channels =================
        const int quarter = wid & 3, t = 32 * quarter + lane;
        const int32_t L = a.seq_lens[b];
        const int n_b = L < 1 ? 0 : min(L, a.window);
        if (L < 1 && lane == 0 && quarter == 0) dev_error(a.err, CSA2_DEV_LEN);
        if (!mbar_wait(done, 0u, kReplayWaitLimit)) *s_timeout = 1;
        tc_fence_after();
        const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
        const int64_t p = (int64_t)L - n_b + t;  // position of this row's token
        uint16_t* dst = a.swa + ((int64_t)b * a.window + (p % a.window + a.window) % a.window) * kCh + n0;
#pragma unroll 1
        for (int c = 0; c < RP_N; c += 16) {
            uint32_t v[16];
            tmem_ld16(lane_base + (uint32_t)c, v);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                pk[j] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            if (t < n_b) {
                uint4* d4 = reinterpret_cast<uint4*>(dst + c);
                d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
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
    LaunchCfg c(dim3((unsigned)B * RP_SLICES), dim3(RP_THREADS), RP_SMEM, (cudaStream_t)stream);
    if (cudaLaunchKernelEx(&c.cfg, swa_replay_kernel, mh, mw, a) != cudaSuccess) {
        (void)cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}
