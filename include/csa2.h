/*
 * csa2.h -- C ABI of the CSA2 sparse global-attention step over an NVFP4
 * main-KV cache, for NVIDIA B200 (sm_100a).
 *
 * What the method is (pages: "DeepSeek lanca V4.1-Flash com contexto de um
 * milhao de tokens", conexaotc.com.br, paragraphs on CSA2 and on the FP4 KV;
 * "Como funciona", e-cogni.com.br; "Atencion escasa comprimida 2 (CSA2)" and
 * "FP4 KV, repeticion limitada", 7minutos.es):
 *   - every CSA2 layer is statically Full, Reindex or Reuse.  Full computes its
 *     own main KV, projects the indexer K from it and selects new Top-512
 *     indices; Reindex re-scores the last Full layer's indexer K with its own
 *     indexer Q; Reuse re-uses the main KV and the most recent Top-K and skips
 *     the indexer.  Every layer keeps its own query and its own 128-token SWA
 *     KV;
 *   - in the decoder a hierarchical indexer lets the Full layer keep up to
 *     2048 blocks of 8 positions (16,384 candidates) that later indexers score;
 *   - the main KV is E2M1 with one E4M3 scale per 16 channels, i.e. NVFP4
 *     without its global scale.
 * Dimensions (fixed by the workload statement, compiled in): 16 query heads of
 * dim 128 sharing one 128-d K and one 128-d V; indexer 4 heads x 64 with score
 * = sum_h w_h * ReLU(q_h . k); main-KV entry = 256 channels (K = 0..127,
 * V = 128..255) stored as 128 code bytes + 16 scale bytes.
 *
 * Conventions for every call:
 *   - all array arguments are DEVICE pointers owned by the caller, except the
 *     descriptor/cache structs and the per-layer pointer tables of
 *     csa2_decode_layers, which are HOST memory read during the call;
 *   - calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and may be captured in a CUDA graph (stated for every
 *     call except csa2_indexer_topk_noalloc);
 *   - kernels are launched with programmatic dependent launch: each waits for
 *     the preceding kernel in the stream before touching memory (inside
 *     csa2_decode_layers, see there);
 *   - host-side checks return a status and launch nothing; errors found on the
 *     device (a slot, page or index out of range) never fault: the access is
 *     skipped and a CSA2_DEV_* bit is OR-ed into *err_word (if non-NULL),
 *     which the caller reads after synchronising;
 *   - no exception crosses the ABI; the library allocates no device memory.
 *   - bf16 values are passed as their uint16_t bit patterns.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA2_ABI_VERSION 1

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad mode/level, misalignment */
    CSA2_ERR_UNSUPPORTED = 2, /* a dimension other than the compiled ones */
    CSA2_ERR_CUDA = 3,        /* a CUDA API call or launch failed */
    CSA2_ERR_WORKSPACE = 4    /* workspace missing or smaller than required */
} csa2_status;

/* bits OR-ed into *err_word by kernels */
#define CSA2_DEV_SLOT 0x1   /* slot_mapping entry outside the cache */
#define CSA2_DEV_PAGE 0x2   /* page-table entry missing or outside the cache */
#define CSA2_DEV_INDEX 0x4  /* a Top-K index >= the sequence length */
#define CSA2_DEV_LEN 0x8    /* a sequence length outside [1, capacity] */
#define CSA2_DEV_TIMEOUT 0x10 /* a bounded wait for an asynchronous copy gave up */
#define CSA2_DEV_ALIGN 0x20   /* a kernel's dynamic shared memory was not aligned as its
                               * layout needs; the kernel returned without computing */

typedef enum { CSA2_MODE_FULL = 0, CSA2_MODE_REINDEX = 1, CSA2_MODE_REUSE = 2 } csa2_mode;
typedef enum { CSA2_LEVEL_BLOCK = 0, CSA2_LEVEL_TOKEN = 1 } csa2_level;
typedef enum { CSA2_SRC_F32 = 0, CSA2_SRC_BF16 = 1 } csa2_src_dtype;

/* Per-layer descriptor.  Supported values: ratio 1 or 2; 1 <= topk <= 512;
 * block 8; 0 <= keep_blocks <= 2048; 1 <= window <= 128; n_heads 16;
 * head_dim 128; idx_heads 4; idx_dim 64.
 * keep_blocks = 0 means no block level (a flat indexer over every entry).
 * The pages place the hierarchical indexer in the decoder only ("Como
 * funciona" of e-cogni.com.br, CSA2 paragraph of conexaotc.com.br), so the
 * encoder's layers (ratio 2, 3 x (Full + 5 Reuse)) select their Top-512 among
 * all entries; csa2_layer_desc_default leaves keep_blocks at 2048, and a
 * caller running the encoder side of a decode step sets it to 0. */
typedef struct {
    int32_t mode;        /* csa2_mode */
    int32_t ratio;       /* tokens per main-KV entry: 1 decoder, 2 encoder */
    int32_t topk;        /* indices kept per Full/Reindex layer (512) */
    int32_t block;       /* positions per indexer block (8) */
    int32_t keep_blocks; /* blocks kept by the Full layer (2048); 0: flat */
    int32_t window;      /* SWA window in tokens (128) */
    int32_t n_heads;     /* 16 */
    int32_t head_dim;    /* 128 */
    int32_t idx_heads;   /* 4 */
    int32_t idx_dim;     /* 64 */
} csa2_layer_desc;

/* Paged global-KV cache (caller-owned memory).  Entry e of sequence b
 * lives in slot page_table[b][e / page_size] * page_size + e % page_size.
 * Every array must be device-accessible (see csa2_device_accessible).  codes
 * and scales (the main KV) may live in pinned host memory mapped into the
 * device address space: attention then gathers only its selected 144-byte
 * entries over the host link.  This is the global-KV tiering of the
 * deployment paragraph of conexaotc.com.br, "FP4 KV, repeticion limitada..."
 * (7minutos.es).  The indexer K arrays, which the indexer streams, belong in
 * device memory.
 *   codes        [n_slots][128] u8  : channel 2j in the low nibble of byte j
 *   scales       [n_slots][16]  u8  : E4M3 bits, scale i covers channels 16i..16i+15
 *   idx_k        [n_slots][64]  bf16: indexer K of each entry
 *   idx_k_pooled [n_slots/8][64] bf16: mean of the rows present in each
 *                block of 8 (slot / 8); NULL if no hierarchical indexer is used
 * n_slots = n_phys_pages * page_size; page_size is a power of two >= 8;
 * every array base is 16-byte aligned; page_table is [n_seqs][max_pages_per_seq]
 * int32 with -1 for unused pages; max_pages_per_seq * page_size <= 2^31. */
typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    uint16_t* idx_k;
    uint16_t* idx_k_pooled;
    const int32_t* page_table;
    int32_t page_size;
    int32_t max_pages_per_seq;
    int64_t n_phys_pages;
} csa2_kv_cache;

/* Fill a descriptor with the pages' defaults (topk 512, block 8, keep 2048,
 * window 128, 16x128 heads, 4x64 indexer) for the given mode and ratio. */
CSA2_API void csa2_layer_desc_default(csa2_layer_desc* desc, int32_t mode, int32_t ratio);

/* Layer modes of the decoder (20 layers: Full + 3 Reuse, then 4 x (Reindex +
 * 3 Reuse)) or the encoder (18 CSA2 layers: 3 x (Full + 5 Reuse)), as stated
 * by the CSA2 paragraph of the conexaotc.com.br page and the "CSA2" section of
 * 7minutos.es.  modes must hold 20 entries; returns the layer count. */
CSA2_API int32_t csa2_schedule(int32_t decoder, int32_t* modes);

/* ---------------------------------------------------------------------- */
/* (1) FP4 quant-append.  Pages: FP4 KV paragraph of conexaotc.com.br, bullet
 * "Cache KV principal em FP4" of plugged.ninja: E2M1 codes with one E4M3
 * scale per 16 channels, no global scale.  Per 16-channel block:
 * s = E4M3_RNE_satfinite(amax / 6) (fp32 division); code = E2M1 nearest
 * (ties to even, saturating, sign copied) of x / s; all codes 0 when s == 0.
 * At ratio 2 entry e is the fp32 mean (x_2e + x_2e+1) * 0.5 of two source
 * rows.  Also copies the entry's indexer-K row and, if the cache has a pooled
 * array, recomputes the pooled row of every block this call touches as
 * bf16(fp32 sequential sum of the rows present / count).
 *   kv_src       [n_entries * ratio][256] fp32 or bf16 (src_dtype)
 *   idx_k_src    [n_entries][64] bf16, or NULL to leave idx_k and pooled alone
 *   slot_mapping [n_entries] int64 physical slots
 * Entries of one sequence must be contiguous and in ascending position order,
 * and the earlier positions of a touched block must already be in the cache.
 * n_entries == 0 is a no-op. */
CSA2_API csa2_status csa2_kv_quant_append(const csa2_kv_cache* cache, const void* kv_src, int32_t src_dtype,
                                 const uint16_t* idx_k_src, int64_t n_entries, int32_t ratio,
                                 const int64_t* slot_mapping, int32_t* err_word, void* stream);

/* ---------------------------------------------------------------------- */
/* (2) Indexer Top-K.  Pages: CSA2 paragraph of conexaotc.com.br (Top-512;
 * hierarchical indexer of up to 2048 blocks of 8 = 16,384 positions) and
 * "Como funciona" of e-cogni.com.br (Reindex re-scores the shared indexer K
 * with its own indexer Q).  score = sum_h w_h * max(q_h . k, 0), each dot a
 * sequential fp32 FMA chain over the 64 dims, the head sum a sequential fp32
 * FMA chain over h; Top-K by (score desc, index asc); outputs ascending and
 * padded with -1.  The mode must be Full or Reindex (Reuse: INVALID_ARG).
 *
 * Decode (q_pos == NULL): n sequences, q_idx [n][4][64] bf16, w [n][4] fp32,
 * seq_lens [n] entries (block level: n <= 1024, max_len <= 2^21 entries).
 *   level BLOCK: idx_out [n][keep_blocks] = the Top-keep blocks by the pooled
 *     indexer K score, or every block when ceil(L/8) <= keep_blocks.
 *   level TOKEN: idx_out [n][topk] = Top-min(topk, C) positions among the
 *     C candidates: the positions < L of the blocks in cand_blocks
 *     [n][keep_blocks] (ascending, -1 padded; normally the BLOCK output of
 *     the Full layer of this step), or all L positions if cand_blocks is NULL
 *     (then L <= 8 * keep_blocks).
 *   keep_blocks = 0 (flat): level TOKEN only (BLOCK: INVALID_ARG), with
 *     cand_blocks NULL (else INVALID_ARG); idx_out [n][topk] = Top-min(topk,
 *     L) of all L positions, n <= 1024 and max_len <= 2^21 (UNSUPPORTED
 *     otherwise); above 16,384 entries the cache must hold at most 2^31 - 1
 *     slots.  The pooled indexer K is not read.
 * Prefill (q_pos != NULL, level TOKEN): n queries of sequence 0 of the page
 *   table, q_idx [n][4][64] (16-byte aligned), w [n][4], q_pos [n] absolute
 *   token positions, seq_lens [1] = entries in the cache (<= 16384); entry j
 *   is visible to the query at p iff (j+1)*ratio - 1 <= p; idx_out [n][topk].
 *   The result is the same exact Top-K: approximate tensor-core scores pick
 *   candidates, which are rescored with the sequential FMA chains and checked
 *   against a bound on the approximation; a query that fails the check is
 *   recomputed exactly.
 * score_out is reserved (pass NULL).
 * workspace: device memory of csa2_indexer_workspace_bytes() bytes (for the
 * same desc: a flat desc needs one row per entry, a hierarchical one per
 * block), 256-byte aligned, zero-filled before its first use; every call
 * leaves its counters and histograms zero again.  Calls sharing one workspace
 * must not overlap on the GPU. */
CSA2_API size_t csa2_indexer_workspace_bytes(const csa2_layer_desc* desc, int32_t level, int32_t n, int64_t max_len,
                                    int32_t prefill);
CSA2_API csa2_status csa2_indexer_topk(const csa2_layer_desc* desc, const csa2_kv_cache* cache, int32_t level,
                              const uint16_t* q_idx, const float* w, const int32_t* seq_lens, const int32_t* q_pos,
                              const int32_t* cand_blocks, int32_t* idx_out, float* score_out, int32_t n,
                              int64_t max_len, void* workspace, size_t ws_bytes, int32_t* err_word, void* stream);

/* ---------------------------------------------------------------------- */
/* (3) Sparse attention, decode.  Pages: "Como funciona" of e-cogni.com.br
 * (Reuse runs sparse attention directly on the re-used indices; every layer
 * keeps its own Q and SWA KV), SWA window of 128 tokens in every layer
 * (conexaotc.com.br, Causal Encoder-Decoder paragraph).  Per head h:
 * branch 1 = softmax((q_h . k_j) / sqrt(128)) weighted V over the selected
 * entries (index -1 skipped), k_j|v_j = e2m1(code) * e4m3(scale); branch 2 =
 * the same over the layer's SWA tokens; out = LSE merge of the two, lse =
 * log(sum of exp over both).  No de-duplication between the two branches.
 *   q        [B][16][128] bf16        topk_idx [B][topk] int32
 *   swa_kv   [B][window][256] bf16 (K|V), rows 0..swa_len-1 valid (any order)
 *   seq_lens [B] entries               swa_lens [B] or NULL (= min(window, L))
 *   out      [B][16][128] fp32         lse      [B][16] fp32 (natural log) */
CSA2_API csa2_status csa2_sparse_attn_decode(const csa2_layer_desc* desc, const csa2_kv_cache* cache, const uint16_t* q,
                                    const int32_t* topk_idx, const uint16_t* swa_kv, const int32_t* seq_lens,
                                    const int32_t* swa_lens, float* out, float* lse, int32_t B, int32_t* err_word,
                                    void* stream);

/* Sparse attention, prefill: T queries of sequence 0 of the page table at
 * absolute token positions q_pos [T]; topk_idx [T][topk]; swa_kv holds the
 * bf16 K|V rows of tokens swa_start, swa_start+1, ... and the window of the
 * query at p is tokens [max(0, p - window + 1), p] (requires swa_start <= that
 * start); seq_len = entries in the cache; out [T][16][128], lse [T][16].
 * q, swa_kv and out must be 16-byte aligned (INVALID_ARG otherwise); the
 * cache must hold fewer than 2^31 slots (UNSUPPORTED otherwise). */
CSA2_API csa2_status csa2_sparse_attn_prefill(const csa2_layer_desc* desc, const csa2_kv_cache* cache, const uint16_t* q,
                                     const int32_t* topk_idx, const int32_t* q_pos, const uint16_t* swa_kv,
                                     int32_t swa_start, int32_t seq_len, float* out, float* lse, int32_t T,
                                     int32_t* err_word, void* stream);

/* ---------------------------------------------------------------------- */
/* Schedule driver: one decode step of n_layers layers in order, each layer
 * launched on its own (Full: BLOCK then TOKEN indexer then attention;
 * Reindex: TOKEN indexer on the Full layer's cand_blocks with its own q_idx/w,
 * then attention; Reuse: attention on the latest index set).  Host arrays of
 * device pointers, one per layer: q_idx[l], w[l] (read for Full/Reindex
 * layers only), q[l], swa_kv[l], out[l], lse[l].  cand_blocks
 * [B][keep_blocks] and idx_sets [n_layers][B][topk] are device outputs; a
 * Reuse layer writes no set and reads the latest one.  Layer 0 must be Full.
 * With keep_blocks = 0 in descs (the encoder's layers: every desc must carry
 * the same keep_blocks), Full and Reindex layers take the flat TOKEN indexer
 * over all entries, cand_blocks may be NULL and is not written, and the
 * workspace is sized by csa2_indexer_workspace_bytes(descs[0], TOKEN, ...).
 * With the main KV (cache->codes, scales) in host memory, each Full or
 * Reindex layer's set is followed by one kernel that copies its selected rows
 * into a staged cache in the workspace, and every attention layer reads them
 * there: the rows of a set cross the host link once, not once per layer.
 * Results are bit-identical to a device-resident cache.  A main KV in host
 * memory that the device cannot read in place (pageable, or mapped at another
 * address) is rejected with INVALID_ARG before anything is launched.
 * Every input must be complete in stream order before the call, as usual.
 * Kernels of the call after the first read the cache, the lengths, the SWA
 * rows other than the newest, a Reuse layer's index set and a Reindex layer's
 * cand_blocks before the preceding kernel of the call has finished (a layer's
 * q, q_idx, w and newest SWA row only after it, as a model computes them from
 * the previous layer's output), so no other stream may write them while the
 * call runs. */
CSA2_API csa2_status csa2_decode_layers(int32_t n_layers, const csa2_layer_desc* descs, const csa2_kv_cache* cache,
                               const uint16_t* const* q_idx, const float* const* w, const uint16_t* const* q,
                               const uint16_t* const* swa_kv, const int32_t* seq_lens, const int32_t* swa_lens,
                               int32_t* cand_blocks, int32_t* idx_sets, float* const* out, float* const* lse,
                               int32_t B, int64_t max_len, void* workspace, size_t ws_bytes, int32_t* err_word,
                               void* stream);

/* ---------------------------------------------------------------------- */
/* SWA Bounded Replay, attention part.  Pages: "FP4 KV, repeticion limitada y
 * otras extensiones" (7minutos.es) -- on a miss only 128 tokens are
 * recomputed -- and "Como funciona" (e-cogni.com.br) -- the replay avoids
 * persisting the SWA cache at the cost of a small recompute in prefill.
 * Recomputes one layer's window K|V rows from the hidden states of the window's
 * tokens:
 *   swa_kv[b][p % window][c] = bf16_RNE( sum_k h[b][t][k] * w_kv[c][k] )
 * for the last n_b = min(window, seq_lens[b]) tokens, t = 0..n_b-1 oldest
 * first, p = seq_lens[b] - n_b + t; c = 0..255 (K channels 0..127, V
 * 128..255); fp32 accumulation (tensor-core sums over four quarters of
 * d_model, added in a fixed order, so the result does not vary from run to
 * run).  Rows of swa_kv outside
 * the window and rows t >= n_b of h are not touched / not used.
 *   h      [B][window][d_model] bf16, 16-byte aligned
 *   w_kv   [256][d_model] bf16 (row c = output channel c), 16-byte aligned
 *   swa_kv [B][window][256] bf16 (the ring csa2_sparse_attn_decode reads)
 * d_model a multiple of 64 (<= 65536; UNSUPPORTED otherwise); window <= 128. */
CSA2_API csa2_status csa2_swa_replay(const uint16_t* h, const uint16_t* w_kv, const int32_t* seq_lens,
                                     uint16_t* swa_kv, int32_t B, int32_t d_model, int32_t window, int32_t* err_word,
                                     void* stream);

/* ---------------------------------------------------------------------- */
/* Context-parallel decode of one long sequence over G shards (one per GPU).
 * Pages: native context window of one million tokens (conexaotc.com.br,
 * opening paragraphs); Top-512 and the hierarchical indexer of up to 2048
 * blocks of 8 (CSA2 paragraph).  Shard g holds the entries [g*S, g*S + S) of
 * the sequence (S a multiple of the page size) in a cache whose page table is
 * that slice of the sequence's; it runs csa2_indexer_topk and
 * csa2_sparse_attn_decode on its own entries (positions local to the shard).
 * Since every member of the global Top-K lies in its own shard's local Top-K,
 * merging the shards' local lists gives exactly the single-GPU selection:
 *   1. csa2_indexer_score_ids: the scores of a shard's selected ids (block ids
 *      at level BLOCK, entry positions at level TOKEN), computed with the
 *      sequential FMA chains of the selection (bit-equal scores), and the ids
 *      made global by adding id_offset (-1 stays -1, score -inf);
 *   2. the (score, global id) lists of all shards are gathered rank by rank
 *      (an all-gather into [G][n][k]: the ids of a row are then ascending in
 *      pair order, shard by shard);
 *   3. csa2_topk_merge: the Top-k of the gathered pairs by (score desc, id asc)
 *      -- the global set, ascending, -1 padded -- and, if out_local is given,
 *      its members in [lo, hi) minus lo: the shard's local share;
 *   4. attention per shard over its local share (the window on one shard),
 *      then csa2_attn_lse_merge of the gathered partial (out, lse).
 *   ids [n][k], scores and ids_out [n][k] (ids_out nullable); id_offset >= 0.
 *   scores, ids [n_parts][n][part_len], n_parts * part_len <= 16384 (8 shards x
 *   2048), k <= 2048; out, out_local [n][k].
 *   out_parts [n_parts][rows][16][128], lse_parts [n_parts][rows][16] (natural
 *   log, -inf for an empty partial); out [rows][16][128], lse [rows][16];
 *   out = sum_g e^(lse_g - M) out_g / sum_g e^(lse_g - M), lse = M + log(sum). */
CSA2_API csa2_status csa2_indexer_score_ids(const csa2_layer_desc* desc, const csa2_kv_cache* cache, int32_t level,
                                            const uint16_t* q_idx, const float* w, const int32_t* seq_lens,
                                            const int32_t* ids, int32_t k, int32_t id_offset, float* scores,
                                            int32_t* ids_out, int32_t n, int64_t max_len, int32_t* err_word,
                                            void* stream);
CSA2_API csa2_status csa2_topk_merge(const float* scores, const int32_t* ids, int32_t n_parts, int32_t part_len,
                                     int32_t k, int32_t lo, int32_t hi, int32_t* out, int32_t* out_local, int32_t n,
                                     void* stream);
CSA2_API csa2_status csa2_attn_lse_merge(int32_t n_parts, const float* out_parts, const float* lse_parts, float* out,
                                         float* lse, int32_t rows, void* stream);

/* ---------------------------------------------------------------------- */
/* Allocation-free decode indexer.  The pages have no counterpart to this call:
 * it is an integration convenience for callers that cannot allocate device
 * memory where they run the indexer -- plug-ins whose host framework owns all
 * device memory and hands them only the tensors they work on, and serving
 * loops that must not call cudaMalloc (it may synchronise the device and takes
 * the driver's allocation locks).  It does exactly what csa2_indexer_topk does
 * for decode (q_pos = NULL, either level), but keeps its scratch in a 16 MiB
 * array of static device memory inside the library instead of a caller
 * workspace.
 *   - allocates nothing (no cudaMalloc/cudaFree); every GPU that loads the
 *     library holds the 16 MiB until the process exits;
 *   - a call whose workspace layout (csa2_indexer_workspace_bytes for the same
 *     desc, level, n and max_len) exceeds 16 MiB returns CSA2_ERR_WORKSPACE.
 *     The limit depends on the mode: the hierarchical indexer (keep_blocks >
 *     0) scores one row per block of 8, so n = 8 sequences of 2^20 entries fit
 *     (about 13.5 MiB); the flat indexer (keep_blocks = 0) above 16,384
 *     entries scores one row per entry, so n * max_len may reach only about
 *     1.3 * 2^20 entries (one sequence of 2^20 needs about 12.4 MiB, two need
 *     about 24.8 MiB);
 *   - the first call on a device looks up the array's device address, and the
 *     first call of each level and mode runs the kernels' one-time host set-up
 *     (shared-memory attributes and the tensor-map entry point);
 *   - block-level and flat-row calls clear the counters they need (a memset on
 *     `stream`); token-level calls need no clear (they write every key they
 *     read back).  Otherwise the array keeps
 *     what the previous call left; all calls share one array per device, so
 *     calls that overlap on the GPU (other streams, other threads) race and
 *     must be serialised by the caller. */
CSA2_API csa2_status csa2_indexer_topk_noalloc(const csa2_layer_desc* desc, const csa2_kv_cache* cache,
                                               int32_t level, const uint16_t* q_idx, const float* w,
                                               const int32_t* seq_lens, const int32_t* cand_blocks,
                                               int32_t* idx_out, int32_t n, int64_t max_len, int32_t* err_word,
                                               void* stream);

/* ---------------------------------------------------------------------- */
/* Test hook with no counterpart on the pages: the poll limit of the bounded
 * waits in the block-level indexer's cp.async copy ring (the hierarchical
 * indexer's pooled rows), which otherwise give up after 2^22 polls.  A wait
 * that gives up sets CSA2_DEV_TIMEOUT in err_word; the kernel still drains its
 * own copies, reaches every barrier and returns, and that call's results are
 * undefined.  Lowering the limit (0 = every wait gives up at once) lets a test
 * drive that path; polls above 2^22 are clamped.  Process-wide, read when a
 * call is launched; returns the previous limit.  Not for production use. */
CSA2_API uint32_t csa2_test_set_wait_limit(uint32_t polls);

/* Measurement helper with no counterpart on the pages: launches n_kernels
 * empty kernels of `ctas` CTAs x `threads` threads on `stream`, each waiting on
 * its predecessor with programmatic dependent launch exactly as the decode
 * step's kernels do (the first CTA of each adds 1 to *sink, if non-NULL, a
 * device int32).  Captured in a CUDA graph it gives the floor that kernel
 * boundaries alone put under a step of that many kernels. */
CSA2_API csa2_status csa2_test_empty_chain(int32_t n_kernels, int32_t ctas, int32_t threads, int32_t* sink,
                                           void* stream);

CSA2_API const char* csa2_status_string(csa2_status s);
CSA2_API int32_t csa2_abi_version(void);

/* A helper with no counterpart on the pages, for the tiered main KV.
 * 1 if kernels on the current device may dereference p at that same address:
 * device or managed memory, or host memory allocated or registered with CUDA
 * and mapped at p.  0 for pageable host memory or another device's memory, -1
 * if CUDA reports an error.  The library does not call it on its own paths. */
CSA2_API int32_t csa2_device_accessible(const void* p);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
