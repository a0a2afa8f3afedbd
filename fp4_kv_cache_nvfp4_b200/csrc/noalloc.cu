// Allocation-free variant of the decode indexer (csa2_indexer_topk_noalloc).
//
// Some callers cannot allocate device memory at the point where they run the
// indexer: plug-ins whose host framework owns all device memory and hands them
// only the tensors they work on, and latency-critical serving loops that must
// not call cudaMalloc (it can synchronise the device and takes the driver's
// allocation locks).  For them this entry point keeps its scratch in a fixed
// array inside the library's own device memory instead of a caller workspace.
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace csa2 {

// Scratch of the allocation-free indexer: 16 MiB of static device memory that
// every GPU which loads the library holds until the process exits.  Calls
// share it and it keeps the previous call's contents.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current.
// Host threads making their first call on one device at the same time both
// look the address up and store the same value; the slots are atomic, so
// that is not a data race.
static cudaError_t noalloc_scratch(void** out) {
    static std::atomic<void*> addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    void* p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace csa2

extern "C" CSA2_API csa2_status csa2_indexer_topk_noalloc(const csa2_layer_desc* desc, const csa2_kv_cache* cache,
                                                          int32_t level, const uint16_t* q_idx, const float* w,
                                                          const int32_t* seq_lens, const int32_t* cand_blocks,
                                                          int32_t* idx_out, int32_t n, int64_t max_len,
                                                          int32_t* err_word, void* stream) {
    using namespace csa2;
    if (!desc || n < 1 || max_len < 1) return CSA2_ERR_INVALID_ARG;
    if (err_word && (reinterpret_cast<uintptr_t>(err_word) & 3u)) return CSA2_ERR_INVALID_ARG;
    // Every argument check of csa2_indexer_topk runs before its workspace
    // check, so a call without a workspace validates the rest and launches
    // nothing.
    const csa2_status pre = csa2_indexer_topk(desc, cache, level, q_idx, w, seq_lens, nullptr, cand_blocks, idx_out,
                                              nullptr, n, max_len, nullptr, 0, err_word, stream);
    if (pre != CSA2_ERR_WORKSPACE) return pre == CSA2_OK ? CSA2_ERR_INVALID_ARG : pre;
    // the scratch must hold this call's whole workspace layout
    const size_t need = csa2_indexer_workspace_bytes(desc, level, n, max_len, 0);
    if (need == 0 || need > kNoAllocScratchBytes) return CSA2_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) {
        (void)cudaGetLastError();
        return CSA2_ERR_CUDA;
    }
    // The block-level and flat-row kernels expect their counters and
    // histograms at zero.  The previous call may have used another (n, max_len)
    // and so another layout: clear the zero-state head of this call's layout
    // first (a memset, no allocation).  The token-level kernels (a hierarchical
    // Reindex/Full token call, or a flat call over at most 16,384 entries)
    // write every key they read back, so they need no clear.
    const bool flat = desc->keep_blocks == 0;
    const bool uses_scratch = level == CSA2_LEVEL_BLOCK || (flat && max_len > kMaxCand);
    if (uses_scratch) {
        const DecodeWs l = decode_ws_layout(n, max_len, flat);
        if (cudaMemsetAsync(scratch, 0, l.blk_thr, (cudaStream_t)stream) != cudaSuccess) {
            (void)cudaGetLastError();
            return CSA2_ERR_CUDA;
        }
    }
    return csa2_indexer_topk(desc, cache, level, q_idx, w, seq_lens, nullptr, cand_blocks, idx_out, nullptr, n,
                             max_len, scratch, kNoAllocScratchBytes, err_word, stream);
}
