// Device helpers shared by the indexer kernels (indexer.cu) and the
// context-parallel merge kernels (cp.cu): the exact scalar score chain, shared
// histograms and lists, and the radix-select threshold refinement and ordered
// emission over order-preserving 32-bit keys.
#pragma once

#include "common.cuh"

namespace csa2 {

// Two fp32 lanes in one 64-bit register; fma.rn.f32x2 rounds each lane as
// fma.rn.f32 does (the two-row score chains of the block-level scorer).
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Score of one indexer-K row held as 32 bf16x2 words, qd[d] = (q_0..q_3)[d] in
// fp32: each head's dot product is a sequential FMA chain over d = 0..63 and
// the head sum a sequential FMA chain over h = 0..3 of w_h * max(dot_h, 0).
__device__ __forceinline__ float idx_score1(const uint32_t (&k)[32], const float4* __restrict__ qd, float4 w) {
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
// Shared-memory counters.  hist_add: plain shared atomics (on B200 the
// hardware resolves same-bin collisions faster than a __match_any_sync
// aggregation).  list_append: warp-aggregated; every lane of the warp calls.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
    if (active) atomicAdd(&hist[bin], 1u);
}

__device__ __forceinline__ void list_append(uint16_t* list, uint32_t* cnt, uint32_t v, bool pred) {
    const unsigned m = __ballot_sync(0xffffffffu, pred);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
    uint32_t pos = 0;
    if (lane == leader) pos = atomicAdd(cnt, (uint32_t)__popc(m));
    pos = __shfl_sync(0xffffffffu, pos, leader);
    if (pred) list[pos + __popc(m & ((1u << lane) - 1u))] = (uint16_t)v;
}

// Copy n32 words global -> shared, 16 B per load (when both pointers allow),
// many loads in flight.
__device__ __forceinline__ void load_words(uint32_t* dst, const uint32_t* src, int n32) {
    const int nt = blockDim.x;
    if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) {
        for (int j = threadIdx.x; j < n32; j += nt) dst[j] = __ldcg(src + j);
        return;
    }
    const int n4 = n32 >> 2;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    int i = threadIdx.x;
    for (; i + 3 * nt < n4; i += 4 * nt) {
        const uint4 a = __ldcg(s4 + i), b = __ldcg(s4 + i + nt), c = __ldcg(s4 + i + 2 * nt),
                    d = __ldcg(s4 + i + 3 * nt);
        d4[i] = a;
        d4[i + nt] = b;
        d4[i + 2 * nt] = c;
        d4[i + 3 * nt] = d;
    }
    for (; i < n4; i += nt) d4[i] = __ldcg(s4 + i);
    for (int j = 4 * n4 + threadIdx.x; j < n32; j += nt) dst[j] = __ldcg(src + j);
}

// ----------------------------------------------------------------------------
// Threshold refinement: the first digit b1 (key bits 31..20) holds the kk-th
// largest key and `need` of its members are still to be taken.  Two 10-bit
// digits over the shrinking member list give the exact key T; *need_out is
// then the number of ties at T to take (lowest slots first).  Whole block.
// ----------------------------------------------------------------------------
static __device__ void refine_threshold(const uint32_t* keys, int nslots, uint32_t b1, uint32_t need, uint32_t* hist,
                                 uint16_t* list0, uint16_t* list1, uint32_t* tmp, uint32_t* T_out,
                                 uint32_t* need_out) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) {
        tmp[48] = 0;
        tmp[49] = 0;
    }
    for (int i = tid; i < 1024; i += nt) hist[i] = 0;
    __syncthreads();
    for (int base = wid * 32; base < nslots; base += nt) {
        const int i = base + lane;
        const uint32_t k = i < nslots ? keys[i] : 0u;
        const bool in = k != 0u && (k >> 20) == b1;
        list_append(list0, &tmp[48], (uint32_t)i, in);
        hist_add(hist, (k >> 10) & 1023u, in);
    }
    __syncthreads();
    const int n0 = (int)tmp[48];
    int d2, d3;
    uint32_t above;
    find_kth_bin(hist, 1024, need, tmp, &d2, &above);
    need -= above;
    const uint32_t base22 = (b1 << 20) | ((uint32_t)d2 << 10);
    if (base22 > 0u && hist[d2] == need) {  // the bin is taken whole: T just below it, no ties
        *T_out = base22 - 1u;
        *need_out = 0;
        return;
    }
    __syncthreads();  // every thread has read hist[d2]
    for (int i = tid; i < 1024; i += nt) hist[i] = 0;
    __syncthreads();
    for (int base = wid * 32; base < n0; base += nt) {
        const int i = base + lane;
        const int slot = i < n0 ? (int)list0[i] : 0;
        const uint32_t k = i < n0 ? keys[slot] : 0u;
        const bool in = i < n0 && (int)((k >> 10) & 1023u) == d2;
        list_append(list1, &tmp[49], (uint32_t)slot, in);
        hist_add(hist, k & 1023u, in);
    }
    __syncthreads();
    find_kth_bin(hist, 1024, need, tmp, &d3, &above);
    need -= above;
    *T_out = (b1 << 20) | ((uint32_t)d2 << 10) | (uint32_t)d3;
    *need_out = need;
}

// Ordered emission: warp w owns slots [w*seg, (w+1)*seg), 32 at a time;
// writes pos_of(slot) of every key > T and of the first `need` keys == T, in
// slot order, then -1 from kk to topk.  Whole block.
template <class PosFn>
static __device__ void emit_sorted(const uint32_t* keys, int nslots, uint32_t T, uint32_t need, uint32_t kk, int topk,
                            int32_t* __restrict__ out, uint32_t* tmp, PosFn pos_of) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const int seg = ((nslots + nw - 1) / nw + 31) & ~31;
    const int lo = wid * seg, hi = min(nslots, lo + seg);
    uint32_t n_gt = 0, n_eq = 0;
    for (int base = lo; base < hi; base += 32) {
        const int i = base + lane;
        const uint32_t k = i < hi ? keys[i] : 0u;
        n_gt += __popc(__ballot_sync(0xffffffffu, k > T));
        n_eq += __popc(__ballot_sync(0xffffffffu, k == T));
    }
    __syncthreads();
    if (lane == 0) {
        tmp[wid] = n_eq;
        tmp[32 + wid] = n_gt;
    }
    __syncthreads();
    uint32_t tie_base = 0, sel_base = 0;
    for (int v = 0; v < wid; ++v) {
        const uint32_t take = tie_base >= need ? 0u : min(tmp[v], need - tie_base);
        sel_base += tmp[32 + v] + take;
        tie_base += tmp[v];
    }
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
    for (int i = (int)kk + tid; i < topk; i += nt) out[i] = -1;
}

// Length of sequence b, 0 (and CSA2_DEV_LEN) when outside [1, max_len].
__device__ __forceinline__ int32_t seq_len_checked(const int32_t* seq_lens, int b, int64_t max_len, int32_t* err) {
    const int32_t L = seq_lens[b];
    if (L < 1 || L > max_len) {
        if (threadIdx.x == 0) dev_error(err, CSA2_DEV_LEN);
        return 0;
    }
    return L;
}

}  // namespace csa2
