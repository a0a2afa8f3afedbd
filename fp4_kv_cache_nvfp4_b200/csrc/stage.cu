// Staging of a decode index set's FP4 rows for a main KV kept in host memory.
//
// When the main KV (codes, scales) lives in pinned host memory, every
// attention layer would gather its selected rows over the host link, and the
// Reuse layers would fetch again the rows of the set their Full or Reindex
// layer already fetched.  The schedule driver instead copies each new index
// set's rows once into a small device cache: sequence b's rows occupy page b
// of that cache, in the set's order, and the set is rewritten as positions
// 0, 1, ... (-1 kept).  Attention over the staged cache reads the same rows in
// the same order, so its results are bit-identical.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

constexpr int SG_THREADS = 256;  // 8 warps; a warp moves 32 rows per round

// grid (ceil(topk / 32 / 8), B): warp w of CTA x copies rows [32 (8 x + w), +32)
__global__ void __launch_bounds__(SG_THREADS) stage_rows_kernel(StageArgs a) {
    pdl_wait();  // the index set comes from the preceding kernel
    pdl_trigger();
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int i = (blockIdx.x * (SG_THREADS / 32) + wid) * 32 + lane;
    if (blockIdx.x == 0 && threadIdx.x == 0) a.stage_pt[b] = b;
    const int32_t L = a.seq_lens[b];
    int64_t src = -1;
    int32_t pos = -1;
    if (i < a.topk) {
        pos = a.idx[(int64_t)b * a.topk + i];
        if (pos >= L) dev_error(a.err, CSA2_DEV_INDEX);
        if (pos >= 0 && pos < L) src = entry_slot(a.cache, a.page_shift, b, pos, a.err);
        a.stage_idx[(int64_t)b * a.topk + i] = src >= 0 ? i : -1;
    }
    // 32 rows x 9 chunks of 16 B per warp: lane l moves chunks l, l + 32, ...
    // of the warp's rows, so a warp keeps 9 loads of host memory in flight
    const int64_t dst_row0 = (int64_t)b * a.stage_rows + (int64_t)(i - lane);
#pragma unroll
    for (int it = 0; it < 9; ++it) {
        const int c = lane + 32 * it;
        const int r = c / 9, ch = c % 9;
        const int64_t s = __shfl_sync(0xffffffffu, src, r);
        if (s >= 0) {
            const int64_t d = dst_row0 + r;
            if (ch < 8) {
                const uint4 v = __ldcg(reinterpret_cast<const uint4*>(a.cache.codes + s * kCodeBytes) + ch);
                reinterpret_cast<uint4*>(a.stage_codes + d * kCodeBytes)[ch] = v;
            } else {
                const uint4 v = __ldcg(reinterpret_cast<const uint4*>(a.cache.scales + s * kScales));
                *reinterpret_cast<uint4*>(a.stage_scales + d * kScales) = v;
            }
        }
    }
}

cudaError_t launch_stage_rows(const StageArgs& a, int B, cudaStream_t stream) {
    const int per_cta = SG_THREADS;  // rows per CTA (one per thread)
    LaunchCfg c(dim3((unsigned)((a.topk + per_cta - 1) / per_cta), (unsigned)B), dim3(SG_THREADS), 0, stream);
    return cudaLaunchKernelEx(&c.cfg, stage_rows_kernel, a);
}

}  // namespace csa2
