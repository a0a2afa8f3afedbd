// K1: FP4 quant-append of main-KV entries into the paged cache.
//
// Pages: FP4 paragraph of "DeepSeek lanca V4.1-Flash..." (conexaotc.com.br) and
// the "Cache KV principal em FP4" bullet of plugged.ninja: E2M1 values with one
// E4M3 scale per 16 channels, NVFP4 without its global scale.  Ratio 2 (encoder
// CSA2 layers, same pages' CSA2 paragraph) averages adjacent token pairs first.
//
// One warp per entry: lane l owns channels [8l, 8l+8), so a 16-channel scale
// block is a lane pair and the warp stores the entry's 128 code bytes as one
// coalesced 128-byte line.  HBM-bound: 512-1024 B read and 272 B written per
// entry.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

struct AppendArgs {
    csa2_kv_cache cache;
    const void* src;
    const uint16_t* idx_src;
    const int64_t* slot_mapping;
    int64_t n;
    int64_t n_slots;
    int ratio;
    int32_t* err;
};

template <bool kBf16>
__device__ __forceinline__ void load8(const void* src, int64_t row, int lane, float* x) {
    if (kBf16) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + row * kCh) + lane);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = bf16_lo(w[i]);
            x[2 * i + 1] = bf16_hi(w[i]);
        }
    } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + row * kCh) + 2 * lane;
        const float4 a = __ldg(p), b = __ldg(p + 1);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
}

template <bool kBf16>
__global__ void __launch_bounds__(256) quant_append_kernel(AppendArgs a) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int64_t e = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= a.n) return;
    // Every load that does not need this entry's slot is issued with it: the
    // source rows, the next entry's slot, and (for the block's pooled row) the
    // slots and indexer-K source rows of the 7 entries before this one.  The
    // cache rows of a block's earlier entries follow once the slot is known:
    // two round trips in all.
    const int64_t slot = a.slot_mapping[e];
    float x[8];
    if (a.ratio == 2) {
        float y[8];
        load8<kBf16>(a.src, 2 * e, lane, x);
        load8<kBf16>(a.src, 2 * e + 1, lane, y);
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(__fadd_rn(x[i], y[i]), 0.5f);
    } else {
        load8<kBf16>(a.src, e, lane, x);
    }
    const bool has_idx = a.idx_src != nullptr, pooled = has_idx && a.cache.idx_k_pooled != nullptr;
    uint32_t ws[8];       // indexer-K source row of entry e - d, lane's word
    int64_t pm[8];        // slot of entry e - d (d >= 1)
#pragma unroll
    for (int d = 0; d < 8; ++d) {
        const int64_t ed = e - d;
        ws[d] = (has_idx && (d == 0 || pooled) && ed >= 0)
                    ? __ldg(reinterpret_cast<const uint32_t*>(a.idx_src + ed * kID) + lane)
                    : 0u;
        pm[d] = (d > 0 && pooled && ed >= 0) ? __ldg(a.slot_mapping + ed) : -1;
    }
    const int64_t next = (pooled && e + 1 < a.n) ? __ldg(a.slot_mapping + e + 1) : -1;
    if (slot < 0 || slot >= a.n_slots) {
        if (lane == 0) dev_error(a.err, CSA2_DEV_SLOT);
        return;
    }

    // block amax over the lane pair, scale = E4M3(amax / 6)
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
    const float s = e4m3_to_f32((uint8_t)sb);

    uint32_t packed = 0;
    if (s != 0.f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) packed |= e2m1_encode(__fdiv_rn(x[i], s)) << (4 * i);
    }
    reinterpret_cast<uint32_t*>(a.cache.codes + slot * kCodeBytes)[lane] = packed;
    if ((lane & 1) == 0) a.cache.scales[slot * kScales + (lane >> 1)] = (uint8_t)sb;

    if (!has_idx) return;
    reinterpret_cast<uint32_t*>(a.cache.idx_k + slot * kID)[lane] = ws[0];

    if (!pooled) return;
    // The last appended entry of a block of 8 recomputes that block's pooled row
    // over the entries present (slot % 8 + 1 of them).  Entries appended by this
    // call are read from the source rows (other warps are still storing them),
    // earlier ones from the cache.
    const bool last_in_block = (e == a.n - 1) || ((next >> 3) != (slot >> 3));
    if (!last_in_block) return;
    const int64_t s0 = slot & ~int64_t(7);
    const int cnt = int(slot - s0) + 1;
    uint32_t wr[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {  // slot s0 + r is entry e - d of this call when the slot mapping says so
        const int d = int(slot - (s0 + r));
        wr[r] = 0u;
        if (r < cnt) {
            bool src = d == 0;
#pragma unroll
            for (int dd = 1; dd < 8; ++dd)
                if (dd == d) src = pm[dd] == s0 + r;
            uint32_t v = 0u;
#pragma unroll
            for (int dd = 0; dd < 8; ++dd)
                if (dd == d) v = ws[dd];
            wr[r] = src ? v : reinterpret_cast<const uint32_t*>(a.cache.idx_k + (s0 + r) * kID)[lane];
        }
    }
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        if (r < cnt) {
            acc0 = __fadd_rn(acc0, bf16_lo(wr[r]));
            acc1 = __fadd_rn(acc1, bf16_hi(wr[r]));
        }
    }
    const float fc = (float)cnt;
    const __nv_bfloat16 m0 = __float2bfloat16_rn(__fdiv_rn(acc0, fc));
    const __nv_bfloat16 m1 = __float2bfloat16_rn(__fdiv_rn(acc1, fc));
    const uint32_t out = uint32_t(__bfloat16_as_ushort(m0)) | (uint32_t(__bfloat16_as_ushort(m1)) << 16);
    reinterpret_cast<uint32_t*>(a.cache.idx_k_pooled + (s0 >> 3) * kID)[lane] = out;
}

cudaError_t launch_quant_append(const csa2_kv_cache& cache, const void* src, bool bf16, const uint16_t* idx_src,
                                int64_t n, int ratio, const int64_t* slot_mapping, int32_t* err,
                                cudaStream_t stream) {
    AppendArgs a{cache, src, idx_src, slot_mapping, n, cache.n_phys_pages * cache.page_size, ratio, err};
    const int warps = 8;
    const int64_t grid = (n + warps - 1) / warps;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    LaunchCfg cfg(dim3((unsigned)grid), dim3(32 * warps), 0, stream);
    return bf16 ? cudaLaunchKernelEx(&cfg.cfg, quant_append_kernel<true>, a)
                : cudaLaunchKernelEx(&cfg.cfg, quant_append_kernel<false>, a);
}

}  // namespace csa2
