// Shared device helpers of the CSA2 library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int kCh = 256;        // channels per main-KV entry (K 0..127, V 128..255)
constexpr int kCodeBytes = 128; // packed E2M1 codes per entry
constexpr int kScales = 16;     // E4M3 scales per entry (one per 16 channels)
constexpr int kIH = 4;          // indexer heads
constexpr int kID = 64;         // indexer dim
constexpr int kH = 16;          // query heads
constexpr int kD = 128;         // head dim
constexpr int kBlk = 8;         // positions per indexer block
constexpr int kMaxTopk = 512;
constexpr int kMaxKeep = 2048;
constexpr int kMaxWindow = 128;
constexpr int kMaxCand = kMaxKeep * kBlk;         // 16,384 token candidates
constexpr int64_t kMaxBlockLevelLen = 1ll << 21;  // entries, block-level indexer
constexpr int kHistBits = 12;                     // first radix digit of a score key
constexpr int kHistBins = 1 << kHistBits;

// Round a shared-memory offset up to a multiple of 16 bytes (mbarriers need 8,
// vector and bulk accesses 16).
constexpr size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// --- bf16 / fp16 bit helpers -------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// --- programmatic dependent launch ---------------------------------------------
// Every kernel waits on its predecessor before touching global memory, so the
// chain of completions stays transitive.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void dev_error(int32_t* err, int32_t bit) {
    if (err) atomicOr(err, bit);
}

// Order-preserving 32-bit key of an fp32 score: larger score -> larger key,
// -0 and +0 share one key.  Key 0 is reserved for "not a candidate".
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if ((u << 1) == 0u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Physical slot of entry `pos` of sequence `seq` (page size 1 << shift), or -1
// (and an error bit) when the page table has no page there.
__device__ __forceinline__ int64_t entry_slot(const csa2_kv_cache& c, int shift, int seq, int32_t pos, int32_t* err) {
    const int32_t pg = pos >> shift;
    if (pos < 0 || pg >= c.max_pages_per_seq) {
        dev_error(err, CSA2_DEV_PAGE);
        return -1;
    }
    const int32_t phys = __ldg(c.page_table + (int64_t)seq * c.max_pages_per_seq + pg);
    if (phys < 0 || phys >= c.n_phys_pages) {
        dev_error(err, CSA2_DEV_PAGE);
        return -1;
    }
    return ((int64_t)phys << shift) | (int64_t)(pos & ((1 << shift) - 1));
}

// --- cp.async (16 B, L2-only) -------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// --- mbarriers (CTA scope) -------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// order this thread's generic shared-memory writes before later async-proxy
// reads (tensor-core operands)
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// mbarrier initialisation visible to the async proxy (TMA completions)
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// 2-D tiled bulk tensor copy, global -> this CTA's shared memory, completion
// counted in bytes on `bar` (no multicast).  The innermost coordinate x times
// the element size must be a multiple of 16 bytes; callers pass x = 0.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int32_t x, int32_t y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// 1-D bulk copy, global -> this CTA's shared memory, completion counted in
// bytes on `bar`: both addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// One arrival on `bar` once every cp.async this thread issued before has
// landed (the barrier's expected count includes it).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Wait for the phase with the given parity; gives up after `limit` polls and
// returns false (the caller records a timeout instead of hanging).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// Barrier over the first n threads of the block (named barrier `id`); id 0
// with n = blockDim.x is the whole block.
struct GroupBar {
    int id, n;
    __device__ __forceinline__ void sync() const { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
};

// --- distributed shared memory (thread-block clusters) -----------------------------
// Address of `local_addr` (a shared-memory address of this CTA) in the CTA of
// the cluster with the given rank.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void red_add_cluster(uint32_t addr, uint32_t v) {
    asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_f32x4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}
// One 8-byte asynchronous store into a peer CTA's shared memory that counts
// its bytes on that CTA's mbarrier (both addresses in the cluster window).
__device__ __forceinline__ void st_async_f32x2(uint32_t addr, float a, float b, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "f"(a), "f"(b), "r"(mbar)
                 : "memory");
}
// The same with 16 bytes.
__device__ __forceinline__ void st_async_f32x4(uint32_t addr, float4 v, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     addr),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(mbar)
                 : "memory");
}
// Wait for a phase of this CTA's mbarrier whose bytes come from peer CTAs
// (acquire at cluster scope); gives up after `limit` polls.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}
__device__ __forceinline__ void st_async_u32x2(uint32_t addr, uint32_t a, uint32_t b, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "r"(a), "r"(b), "r"(mbar)
                 : "memory");
}
// Atomic add on a peer CTA's shared memory word; returns the previous value.
__device__ __forceinline__ uint32_t atom_add_cluster(uint32_t addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}
// Split cluster barrier: arrive (release) now, wait (acquire) later.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_sync_all() {
    cluster_arrive();
    cluster_wait();
}

// --- E2M1 / E4M3 ----------------------------------------------------------------
// Nearest E2M1 code of y, ties to the even code, saturating at 6, sign copied.
// The magnitude code is the number of rounding boundaries below |y|; at a tie
// the boundary counts only when the upper neighbour has the even code.
__device__ __forceinline__ uint32_t e2m1_encode(float y) {
    float a = fabsf(y);
    uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
    return c | ((__float_as_uint(y) >> 28) & 8u);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
    return __half2float(__half(h));
}

__device__ __forceinline__ uint32_t e4m3_to_h2(uint8_t b) {  // (s, s) as f16x2
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
    return uint32_t(h.x) | (uint32_t(h.x) << 16);
}

// Four packed bytes = eight E2M1 codes -> four f16x2 (byte i -> h[i]; the low
// nibble of a byte lands in the low half), hardware conversion.
__device__ __forceinline__ void e2m1x8_to_h2x4(uint32_t w, uint32_t& h0, uint32_t& h1, uint32_t& h2, uint32_t& h3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// bf16x2 -> f16x2 (exact for normal-range values)
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t w) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(bf16_hi(w)), "f"(bf16_lo(w)));
    return d;
}

__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// --- warp / block scans ------------------------------------------------------------
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
    int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Exclusive scan of one value per thread over the group's threads (a multiple
// of 32, <= 1024; thread index = threadIdx.x).  `tmp` holds >= 33 words of
// shared memory.  Returns the exclusive prefix; *total receives the sum.
__device__ __forceinline__ uint32_t group_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total, GroupBar g) {
    int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = g.n >> 5;
    uint32_t inc = warp_incl_scan(v);
    if (lane == 31) tmp[wid] = inc;
    g.sync();
    if (wid == 0) {
        uint32_t s = lane < nw ? tmp[lane] : 0u;
        uint32_t si = warp_incl_scan(s);
        if (lane < nw) tmp[lane] = si - s;
        if (lane == 31) tmp[32] = si;
    }
    g.sync();
    uint32_t r = tmp[wid] + inc - v;
    *total = tmp[32];
    g.sync();
    return r;
}
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
    return group_excl_scan(v, tmp, total, GroupBar{0, (int)blockDim.x});
}

// Given a histogram `hist[nbins]` in shared memory (descending rank = from the
// top bin down) find the bin holding the k-th largest item (1-based k <= total):
// *bin_out = that bin, *above_out = items in higher bins.  Every thread of the
// group calls.
// *total_out (if given) receives the histogram total; the bin is defined only
// when k <= total.
__device__ __forceinline__ void group_find_kth_bin(const uint32_t* hist, int nbins, uint32_t k, uint32_t* tmp,
                                                   int* bin_out, uint32_t* above_out, GroupBar g,
                                                   uint32_t* total_out = nullptr) {
    // each thread owns a contiguous run of bins counted from the top
    int per = (nbins + g.n - 1) / g.n;
    int hi = nbins - 1 - (int)threadIdx.x * per;  // first (highest) bin of this thread
    // the run is summed from a per-thread starting point, so that the lanes of
    // a warp read distinct banks (runs of `per` words apart would collide)
    const int rot = (int)(((uint32_t)threadIdx.x * (uint32_t)per / 32u) % (uint32_t)per);
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) {
        int r = i + rot;
        if (r >= per) r -= per;
        int b = hi - r;
        if (b >= 0) mine += hist[b];
    }
    uint32_t total;
    uint32_t before = group_excl_scan(mine, tmp, &total, g);
    if (total_out) *total_out = total;
    if (before < k && before + mine >= k) {
        uint32_t acc = before;
        for (int i = 0; i < per; ++i) {
            int b = hi - i;
            if (b < 0) break;
            if (acc + hist[b] >= k) {
                tmp[40] = (uint32_t)b;
                tmp[41] = acc;
                break;
            }
            acc += hist[b];
        }
    }
    g.sync();
    *bin_out = (int)tmp[40];
    *above_out = tmp[41];
    g.sync();
}
__device__ __forceinline__ void find_kth_bin(const uint32_t* hist, int nbins, uint32_t k, uint32_t* tmp,
                                             int* bin_out, uint32_t* above_out) {
    group_find_kth_bin(hist, nbins, k, tmp, bin_out, above_out, GroupBar{0, (int)blockDim.x});
}

}  // namespace csa2
