// K6: decode attention over gathered FP4 main-KV entries plus the layer's
// bf16 SWA window, merged by log-sum-exp (prefill attention, K7, is in
// prefill_attn.cu).
//
// Pages: "Como funciona" (e-cogni.com.br): a Reuse layer runs sparse attention
// directly on the re-used Top-K indices; every layer keeps its own global Q and
// its own SWA KV.  The 128-token SWA window runs in every layer
// (conexaotc.com.br, Causal Encoder-Decoder paragraph).  Merge of the two
// branches by log-sum-exp: workload statement.
//
// Design (one row = one decode sequence, 16 heads that share one K and one V):
//   * a cluster of 8 CTAs per row; CTA s takes selected keys [64s, 64s+64)
//     (four warps of 16) and window keys [16s, 16s+16) (a fifth warp);
//   * each warp gathers its 16 rows (144 B per FP4 entry: codes + scales, or
//     512 B per bf16 window token) with cp.async, dequantises E2M1 x E4M3 to
//     fp16 in registers (exact: <= 6 significant bits, magnitudes 2^-10..2688)
//     straight into the mma.sync B fragments of S = Q K^T (m16n8k16, the 16
//     heads are the M dimension), and writes V as an fp16 tile;
//   * one softmax over the CTA's 80 keys (per-warp maxima and fp16 P in shared
//     memory), then P V split by output dims over four warps;
//   * the CTAs' partials go to the CTA that owns each head pair by st.async,
//     counted on its mbarrier (details at decode_attn_kernel).
// The work per row is ~5 MFLOP against 136 KiB of gathered bytes, so the kernel
// is bound by gather latency and HBM/L2 bandwidth; mma.sync keeps the math off
// the critical path.

#include "common.cuh"
#include "kernels.h"

namespace csa2 {

constexpr int ATT_SPLIT = 8;   // CTAs (cluster) per row
constexpr int ATT_WARPS = 5;   // 4 selected-key warps + 1 window warp
constexpr int ATT_THREADS = ATT_WARPS * 32;
constexpr int KPW = 16;        // keys per warp
constexpr int FP4_ROW = 144;   // staged FP4 entry: 128 code bytes + 16 scale bytes
constexpr int SWA_ROW = 528;   // staged bf16 token: 512 B + 16 B pad (bank spread)
constexpr int VT_ROW = 272;    // fp16 V tile row: 256 B + 16 B pad

// Shared-memory layout of the decode kernel (byte offsets, all 16-aligned).
constexpr int DA_KEYS = 4 * KPW + KPW;   // 64 selected + 16 window keys per CTA
constexpr int DA_PROW = DA_KEYS * 2 + 16;  // fp16 P row [80 keys] + 16 B pad (ldmatrix without bank conflicts)
constexpr int DA_RROW = kD + 4;          // received partial of one head: O[128], m, l, 2 pad (floats)
constexpr uint32_t DA_RECV_BYTES = (uint32_t)ATT_SPLIT * 2 * (kD + 2) * 4;  // bytes each CTA receives
constexpr size_t DA_OFF_FP4 = 0;                                         // [4 warps][16][144] staged rows
constexpr size_t DA_OFF_SWA = DA_OFF_FP4 + 4 * KPW * FP4_ROW;            // [16][528] staged window rows
constexpr size_t DA_OFF_VT = DA_OFF_SWA + KPW * SWA_ROW;                 // [80 keys][272 B] fp16 V tile
constexpr size_t DA_OFF_P = DA_OFF_VT + (size_t)DA_KEYS * VT_ROW;        // [16 heads][DA_PROW] fp16 P
constexpr size_t DA_OFF_RECV = DA_OFF_P + (size_t)kH * DA_PROW;          // [8 src][2 heads][DA_RROW] fp32
constexpr size_t DA_OFF_WM = DA_OFF_RECV + (size_t)ATT_SPLIT * 2 * DA_RROW * 4;  // [5 warps][16] max
constexpr size_t DA_OFF_WS = DA_OFF_WM + ATT_WARPS * kH * 4;             // [5 warps][16] sums
constexpr size_t DA_OFF_VALID = DA_OFF_WS + ATT_WARPS * kH * 4;          // [80] key valid flags
constexpr size_t DA_OFF_BAR = DA_OFF_VALID + DA_KEYS * 4;                // receive mbarrier
constexpr size_t DA_SMEM = DA_OFF_BAR + 16;
static_assert(DA_OFF_SWA % 16 == 0 && DA_OFF_VT % 16 == 0 && DA_OFF_P % 16 == 0 && DA_OFF_RECV % 16 == 0 &&
                  DA_OFF_WM % 16 == 0 && DA_OFF_BAR % 16 == 0 && DA_PROW % 16 == 0,
              "decode attention shared-memory layout");

__device__ __forceinline__ uint32_t e2m1_low_byte_to_h2(uint32_t x) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
        : "=r"(out)
        : "r"(x));
    return out;
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

constexpr uint32_t kAttnWaitLimit = 1u << 22;

// Decode attention.  A cluster of 8 CTAs per sequence; CTA s takes selected
// keys [64s, 64s + 64) (warps 0-3, 16 each) and window keys [16s, 16s + 16)
// (warp 4).
//   before the wait (what exists before the previous layer ends): gather the
//     keys' rows, dequantise K into the mma B fragments and V into a shared
//     fp16 tile [80 keys][128], initialise the receive mbarrier and pass a
//     cluster barrier (every peer's mbarrier is then ready);
//   after the wait: each warp computes S = Q K^T for its 16 keys; the CTA
//     takes one softmax over its 80 keys (per-warp maxima and fp16 P in shared
//     memory, two CTA barriers); warp w (0-3) computes O = P V for dims
//     [32w, 32w + 32); every CTA then sends its (O, max, sum) of heads 2c and
//     2c + 1 to CTA c with st.async, counted in bytes on CTA c's mbarrier, and
//     CTA c merges the 8 partials of its two heads by log-sum-exp and writes
//     them.  No cluster barrier after the wait: a CTA only waits for the bytes
//     it receives.
__global__ void __launch_bounds__(ATT_THREADS) decode_attn_kernel(AttnArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x % ATT_SPLIT;  // rank in the cluster (cluster = 8 consecutive CTAs)
    const int row = blockIdx.x / ATT_SPLIT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    float* recv = reinterpret_cast<float*>(smem + DA_OFF_RECV);
    float* wmax = reinterpret_cast<float*>(smem + DA_OFF_WM);
    float* wsum = reinterpret_cast<float*>(smem + DA_OFF_WS);
    int* valid = reinterpret_cast<int*>(smem + DA_OFF_VALID);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + DA_OFF_BAR);
    uint8_t* vt = smem + DA_OFF_VT;  // key k (0..79) at row k
    uint8_t* ps = smem + DA_OFF_P;

    // Every buffer offset assumes a 16-byte-aligned dynamic shared base; the
    // check is uniform over the grid, so no CTA waits on one that left.
    if (smem_u32(smem) & 15u) {
        pdl_wait();
        if (tid == 0) dev_error(a.err, CSA2_DEV_ALIGN);
        return;
    }
    // The receive mbarrier expects one local arrival and DA_RECV_BYTES from the
    // 8 CTAs of the cluster; the cluster barrier below makes its
    // initialisation visible to them before any of them sends.  Neither reads
    // global memory, so both run before the wait on the preceding kernel.
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, DA_RECV_BYTES);
    }
    cluster_arrive();

    const bool pre_idx = (a.pre & kPreIdx) != 0, pre_hist = (a.pre & kPreHist) != 0;
    bool waited = false;
    auto wait_once = [&]() {
        if (!waited) {
            pdl_wait();
            waited = true;
        }
    };
    if (!pre_idx && !pre_hist) wait_once();

    // ---- sequence, window --------------------------------------------------
    const int32_t L = a.seq_lens[row];
    const uint16_t* swa_base = a.swa + (int64_t)row * a.window * kCh;
    int n_swa = a.swa_lens ? a.swa_lens[row] : (L < a.window ? L : a.window);
    n_swa = max(0, min(n_swa, a.window));
    const int newest = ((pre_idx || pre_hist) && L > 0) ? (L - 1) % a.window : -1;  // read after the wait

    // ---- gather this warp's 16 keys into shared memory ---------------------
    uint8_t* st_fp4 = smem + DA_OFF_FP4 + (warp < 4 ? warp : 0) * KPW * FP4_ROW;
    uint8_t* st_swa = smem + DA_OFF_SWA;
    const int k0 = warp < 4 ? split * 64 + warp * KPW : split * KPW;
    if (warp < 4) {
        if (!pre_idx) wait_once();  // the index set comes from the preceding kernel
        int64_t slot = -1;
        if (lane < KPW) {
            const int kidx = k0 + lane;
            if (kidx < a.topk) {
                const int32_t pos = a.idx[(int64_t)row * a.topk + kidx];
                if (pos >= 0) {
                    if (pos < L) slot = entry_slot(a.cache, a.page_shift, row, pos, a.err);
                    else dev_error(a.err, CSA2_DEV_INDEX);
                }
            }
            valid[warp * KPW + lane] = slot >= 0;
        }
        // 16 rows x 9 chunks of 16 B; every lane runs all 5 trips (the shuffle
        // needs the full warp), trips past the 144 chunks copy nothing
#pragma unroll
        for (int it = 0; it < (KPW * 9 + 31) / 32; ++it) {
            const int c = lane + 32 * it;
            const int r = min(c / 9, KPW - 1), ch = c % 9;
            const int64_t s = __shfl_sync(0xffffffffu, slot, r);
            if (c < KPW * 9) {
                uint8_t* dst = st_fp4 + r * FP4_ROW + ch * 16;
                if (s >= 0) {
                    if (ch < 8) cp_async16(dst, a.cache.codes + s * kCodeBytes + ch * 16);
                    else cp_async16(dst, a.cache.scales + s * kScales);
                } else {
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
        }
    } else {
        if (lane < KPW) valid[4 * KPW + lane] = (k0 + lane) < n_swa;
        for (int c = lane; c < KPW * 32; c += 32) {
            const int r = c >> 5, ch = c & 31;
            uint8_t* dst = st_swa + r * SWA_ROW + ch * 16;
            if (k0 + r < n_swa) {
                if (k0 + r != newest) cp_async16(dst, swa_base + (int64_t)(k0 + r) * kCh + ch * 8);
            } else {
                *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            }
        }
    }
    cp_async_commit();

    // K of the warp's keys as the B fragments of S = Q K^T (two n8 tiles),
    // V into rows [16 w, 16 w + 16) of the shared fp16 V tile; `only` >= 0
    // rebuilds just that row (the newest window row, staged after the wait).
    uint32_t bk[2][8][2];
    auto build_kv = [&](int only) {
        const int key = lane >> 1, half = lane & 1;
        uint32_t* dst = reinterpret_cast<uint32_t*>(vt + (warp * KPW + key) * VT_ROW + half * 128);
        if (warp < 4) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint8_t* r = st_fp4 + (8 * j + g) * FP4_ROW;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t sc = e4m3_to_h2(r[128 + c]);
                    const uint32_t wl = *reinterpret_cast<const uint32_t*>(r + 8 * c);
                    const uint32_t wh = *reinterpret_cast<const uint32_t*>(r + 8 * c + 4);
                    bk[j][c][0] = hmul2(e2m1_low_byte_to_h2(wl >> (8 * t)), sc);
                    bk[j][c][1] = hmul2(e2m1_low_byte_to_h2(wh >> (8 * t)), sc);
                }
            }
            const uint8_t* r = st_fp4 + key * FP4_ROW;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t w = *reinterpret_cast<const uint32_t*>(r + 64 + 32 * half + 4 * i);
                const uint32_t sc = e4m3_to_h2(r[128 + 8 + 4 * half + (i >> 1)]);
                uint32_t h0, h1, h2, h3;
                e2m1x8_to_h2x4(w, h0, h1, h2, h3);
                *reinterpret_cast<uint4*>(dst + 4 * i) = make_uint4(hmul2(h0, sc), hmul2(h1, sc), hmul2(h2, sc),
                                                                    hmul2(h3, sc));
            }
        } else {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (only >= 0 && 8 * j + g != only) continue;
                const uint32_t* r = reinterpret_cast<const uint32_t*>(st_swa + (8 * j + g) * SWA_ROW);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    bk[j][c][0] = bf2_to_h2(r[8 * c + t]);
                    bk[j][c][1] = bf2_to_h2(r[8 * c + 4 + t]);
                }
            }
            if (only < 0 || key == only) {
                const uint32_t* r = reinterpret_cast<const uint32_t*>(st_swa + key * SWA_ROW) + 64 + 32 * half;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<uint4*>(dst + 4 * i) = make_uint4(
                        bf2_to_h2(r[4 * i]), bf2_to_h2(r[4 * i + 1]), bf2_to_h2(r[4 * i + 2]), bf2_to_h2(r[4 * i + 3]));
            }
        }
    };
    cp_async_wait<0>();
    __syncwarp();
    build_kv(-1);
    // the newest window row (computed from the previous layer's output) is read
    // after the wait and patched into the fragments and the V tile
    const int new_r = newest - k0;
    const bool own_newest = warp == 4 && newest >= 0 && new_r >= 0 && new_r < KPW && newest < n_swa;
    wait_once();  // every thread has waited before anything is written
    pdl_trigger();
    if (own_newest) {
        cp_async16(st_swa + new_r * SWA_ROW + lane * 16, swa_base + (int64_t)newest * kCh + lane * 8);
        cp_async_commit();
    }
    // Q (A operand rows: heads g and g + 8, bf16 pairs) of this row
    uint32_t qraw[8][4];
    {
        const uint32_t* qg = reinterpret_cast<const uint32_t*>(a.q + (int64_t)row * kH * kD + g * kD);
        const uint32_t* qg8 = qg + 8 * kD / 2;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            qraw[c][0] = __ldg(qg + 8 * c + t);
            qraw[c][1] = __ldg(qg8 + 8 * c + t);
            qraw[c][2] = __ldg(qg + 8 * c + 4 + t);
            qraw[c][3] = __ldg(qg8 + 8 * c + 4 + t);
        }
    }
    if (own_newest) {
        cp_async_wait<0>();
        __syncwarp();
        build_kv(new_r);
    }

    // ---- S = Q K^T (A operand: 16 heads x 128 dims, fp16) -------------------
    float S[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t qa[4] = {bf2_to_h2(qraw[c][0]), bf2_to_h2(qraw[c][1]), bf2_to_h2(qraw[c][2]),
                                bf2_to_h2(qraw[c][3])};
        mma16816(S[0], qa, bk[0][c][0], bk[0][c][1]);
        mma16816(S[1], qa, bk[1][c][0], bk[1][c][1]);
    }

    // ---- one softmax over the CTA's 80 keys (log2 domain) ---------------------
    const float kScaleLog2 = 1.4426950408889634f * 0.08838834764831845f;  // log2(e) / sqrt(128)
    const int kb = warp * KPW;  // this warp's first key in the CTA
    float mg = -INFINITY, mg8 = -INFINITY;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const bool ok = valid[kb + 8 * j + 2 * t + e] != 0;
            S[j][e] = ok ? S[j][e] * kScaleLog2 : -INFINITY;
            S[j][2 + e] = ok ? S[j][2 + e] * kScaleLog2 : -INFINITY;
            mg = fmaxf(mg, S[j][e]);
            mg8 = fmaxf(mg8, S[j][2 + e]);
        }
    }
    mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, 1));
    mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, 2));
    mg8 = fmaxf(mg8, __shfl_xor_sync(0xffffffffu, mg8, 1));
    mg8 = fmaxf(mg8, __shfl_xor_sync(0xffffffffu, mg8, 2));
    if (t == 0) {
        wmax[warp * kH + g] = mg;
        wmax[warp * kH + g + 8] = mg8;
    }
    __syncthreads();  // every warp's maxima (and, with them, every V tile row)
    float M = -INFINITY, M8 = -INFINITY;
#pragma unroll
    for (int w = 0; w < ATT_WARPS; ++w) {
        M = fmaxf(M, wmax[w * kH + g]);
        M8 = fmaxf(M8, wmax[w * kH + g + 8]);
    }
    float lg = 0.f, lg8 = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            S[j][e] = M == -INFINITY ? 0.f : exp2f(S[j][e] - M);
            S[j][2 + e] = M8 == -INFINITY ? 0.f : exp2f(S[j][2 + e] - M8);
            lg += S[j][e];
            lg8 += S[j][2 + e];
        }
        // P (fp16) rows g and g + 8, keys kb + 8 j + 2 t, + 1
        *reinterpret_cast<uint32_t*>(ps + g * DA_PROW + (kb + 8 * j + 2 * t) * 2) = f2_to_h2(S[j][0], S[j][1]);
        *reinterpret_cast<uint32_t*>(ps + (g + 8) * DA_PROW + (kb + 8 * j + 2 * t) * 2) = f2_to_h2(S[j][2], S[j][3]);
    }
    lg += __shfl_xor_sync(0xffffffffu, lg, 1);
    lg += __shfl_xor_sync(0xffffffffu, lg, 2);
    lg8 += __shfl_xor_sync(0xffffffffu, lg8, 1);
    lg8 += __shfl_xor_sync(0xffffffffu, lg8, 2);
    if (t == 0) {
        wsum[warp * kH + g] = lg;
        wsum[warp * kH + g + 8] = lg8;
    }
    cluster_wait();   // every peer's receive mbarrier is initialised (arrived long before)
    __syncthreads();  // P and the sums are complete

    const uint32_t my_bar = smem_u32(bar);
    if (warp < 4) {
        // ---- O[16 heads][32 w .. 32 w + 31] = P[16][80] V[80][dims] ------------
        float O[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
        const uint32_t pa_base = smem_u32(ps) + (((lane >> 3) & 1) * 8 + (lane & 7)) * DA_PROW + (lane >> 4) * 16;
        const int m = lane >> 3, r = lane & 7;
        const uint32_t vb_base = smem_u32(vt) + ((m & 1) * 8 + r) * VT_ROW + (m >> 1) * 16 + warp * 64;
#pragma unroll
        for (int ks = 0; ks < DA_KEYS / 16; ++ks) {
            uint32_t pa[4];
            ldsm_x4(pa_base + ks * 32, pa[0], pa[1], pa[2], pa[3]);
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(vb_base + ks * 16 * VT_ROW + j * 16, b0, b1, b2, b3);
                mma16816(O[j], pa, b0, b1);
                mma16816(O[j + 1], pa, b2, b3);
            }
        }
        // ---- send: heads g, g + 8 to their owner CTAs, dims 32 w + 8 j + 2 t ----
        const int hs[2] = {g, g + 8};
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int h = hs[hi];
            const uint32_t owner = (uint32_t)(h >> 1);
            const uint32_t rb = mapa_shared(my_bar, owner);
            const uint32_t ro = mapa_shared(smem_u32(recv + (split * 2 + (h & 1)) * DA_RROW), owner);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                st_async_f32x2(ro + (uint32_t)(32 * warp + 8 * j + 2 * t) * 4u, O[j][2 * hi], O[j][2 * hi + 1], rb);
        }
    } else if (lane < kH) {
        // ---- send the CTA's (max, sum) of head `lane` to its owner --------------
        const int h = lane;
        float mx = -INFINITY, sum = 0.f;
#pragma unroll
        for (int w = 0; w < ATT_WARPS; ++w) mx = fmaxf(mx, wmax[w * kH + h]);
#pragma unroll
        for (int w = 0; w < ATT_WARPS; ++w) sum += wsum[w * kH + h];
        const uint32_t owner = (uint32_t)(h >> 1);
        st_async_f32x2(mapa_shared(smem_u32(recv + (split * 2 + (h & 1)) * DA_RROW + kD), owner), mx, sum,
                       mapa_shared(my_bar, owner));
    }

    // ---- receive the 8 partials of heads 2 split, 2 split + 1 and merge -------
    if (!mbar_wait_cluster(bar, 0u, kAttnWaitLimit)) {
        if (tid == 0) dev_error(a.err, CSA2_DEV_TIMEOUT);
        return;  // nothing was received in time: leave out and lse unwritten
    }
    if (tid < 2 * kD / 4) {
        const int hh = tid / (kD / 4), d4 = (tid % (kD / 4)) * 4;
        float Mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < ATT_SPLIT; ++c) Mx = fmaxf(Mx, recv[(c * 2 + hh) * DA_RROW + kD]);
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
        float den = 0.f;
#pragma unroll
        for (int c = 0; c < ATT_SPLIT; ++c) {
            const float* p = recv + (c * 2 + hh) * DA_RROW;
            const float mc = p[kD];
            const float f = mc == -INFINITY ? 0.f : exp2f(mc - Mx);
            const float4 v = *reinterpret_cast<const float4*>(p + d4);
            num.x += v.x * f;
            num.y += v.y * f;
            num.z += v.z * f;
            num.w += v.w * f;
            den += p[kD + 1] * f;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        const int h = 2 * split + hh;
        *reinterpret_cast<float4*>(a.out + ((int64_t)row * kH + h) * kD + d4) =
            make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
        if (d4 == 0) a.lse[(int64_t)row * kH + h] = den > 0.f ? (Mx + log2f(den)) * 0.6931471805599453f : -INFINITY;
    }
}

cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t stream) {
    static bool init[64];
    static int n_sm[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!init[dev]) {
        e = cudaFuncSetAttribute((const void*)decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)DA_SMEM);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        init[dev] = true;
    }
    if (a.rows <= 0) return cudaSuccess;
    if (a.q_pos) return launch_prefill_attn_tc(a, n_sm[dev], stream);  // one persistent CTA per SM
    LaunchCfg c(dim3((unsigned)a.rows * ATT_SPLIT), dim3(ATT_THREADS), DA_SMEM, stream, ATT_SPLIT);
    return cudaLaunchKernelEx(&c.cfg, decode_attn_kernel, a);
}

}  // namespace csa2
