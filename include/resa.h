/*
 * resa.h - C ABI of libresa, the B200 (sm_100a) hot path of Rectified Sparse
 * Attention (ReSA): group block-sparse decode attention over a paged KV cache
 * plus the periodic dense rectification that refreshes it.
 *
 * Source ("ReSA summary"): the page "Rectified Sparse Attention" of the
 * paper-graph-ui summary of arXiv 2506.04108.  Each entry point names the
 * section / equation it implements.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  The caller allocates every buffer; the library allocates no device
 *   or host memory and keeps no per-call state between calls.  All device
 *   pointers must be 16-byte aligned.  Calls are asynchronous on `stream`
 *   (never synchronised), except resa_check_device_status.
 * Precision.  q, K, V and descriptors are bf16; scores, softmax statistics
 *   and accumulation are fp32; attention outputs are fp32.
 * Value range.  resa_rectify_attention accepts every finite bf16 value: it
 *   stages each 64-key V tile in fp16 scaled by a power of two chosen from
 *   the tile's largest |v|, and undoes the scaling in fp32.  The decode entry
 *   points keep V in bf16 and sum up to ~2^17 weighted values per warp in
 *   fp32 before normalising, so they need |v| <= 1e33 (far beyond any model's
 *   activations; larger values may overflow to inf).  Non-finite inputs give
 *   non-finite outputs.
 * Cache layout (one attention layer):
 *   k, v        [num_pages][Hkv][block_size][head_dim]  bf16
 *   desc        [num_pages][Hkv][2][head_dim]           bf16, row 0 = element-wise
 *                                                       min, row 1 = max (Eq. 3)
 *   page_table  [batch][max_pages] int32: physical page of logical block i
 *   seq_len     [batch] int32: tokens in the cache, INCLUDING the decode token
 *               of the current step (the token is appended before attending).
 *   Block i of a sequence holds positions i*b .. i*b+b-1.  With L = seq_len,
 *   the complete blocks are 0 .. M-1, M = (L-1)/b, and the current block
 *   c = M holds positions M*b .. L-1 (1 to b tokens).
 * Workspace.  `ws` is caller-owned device scratch of `ws_bytes` bytes, at
 *   least resa_workspace_size(...).  Zero it once with resa_workspace_init
 *   before first use; the library leaves it reusable.  Two calls that share a
 *   workspace must not run concurrently.
 * Errors.  Host-side argument checks return a status before anything is
 *   launched.  A failed launch returns RESA_ERR_CUDA.  Range errors that only
 *   the device can see (seq_len, page ids, block ids, top-k above max_topk)
 *   set bits of an error word in the workspace and the offending item is
 *   skipped or clamped (never a trap); read and clear the word with
 *   resa_check_device_status.  Device waits are bounded; a wait that gives up
 *   sets RESA_DEVERR_TIMEOUT.  The outputs of a call that timed out are
 *   undefined, and its workspace may hold words of that call: zero it again
 *   with resa_workspace_init before the next call.
 * Supported shapes.  head_dim in {64, 128}; block_size in {16, 32, 64}
 *   (the b of the memory model, ReSA summary §3.4.3, Eq. 6); group size
 *   g = Hq / Hkv in 1 .. 16; Hkv <= 8.  Other shapes return
 *   RESA_ERR_UNSUPPORTED.  The one-launch decode step is built for
 *   block_size 16; other block sizes run it as three launches
 *   (resa_decode_step_launches).
 */
#ifndef RESA_H_
#define RESA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define RESA_API __attribute__((visibility("default")))
#else
#define RESA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RESA_OK = 0,
    RESA_ERR_NULL = 1,         /* a required pointer is NULL */
    RESA_ERR_SHAPE = 2,        /* inconsistent sizes, or workspace too small */
    RESA_ERR_RANGE = 3,        /* a host-visible value is out of range */
    RESA_ERR_UNSUPPORTED = 4,  /* valid but not implemented (shape, alignment) */
    RESA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    RESA_ERR_DEVICE_CHECK = 6  /* device-side check tripped (see error word) */
} resa_status_t;

/* Bits of the device error word (resa_check_device_status). */
#define RESA_DEVERR_SEQ_LEN 0x1u   /* seq_len < 1 or > max_pages * block_size */
#define RESA_DEVERR_PAGE 0x2u      /* page_table entry outside [0, num_pages) */
#define RESA_DEVERR_BLOCK 0x4u     /* block_idx entry outside the sequence */
#define RESA_DEVERR_TOPK 0x8u      /* topk[b] > max_topk with more blocks available: clamped */
#define RESA_DEVERR_CHUNK 0x10u    /* rectification chunk f > seq_len */
#define RESA_DEVERR_TIMEOUT 0x20u  /* a bounded device wait gave up */
#define RESA_DEVERR_ROW 0x40u      /* rows[i] outside [0, table_rows): sequence skipped */

typedef struct {
    int32_t num_q_heads;   /* Hq */
    int32_t num_kv_heads;  /* Hkv; Hq % Hkv == 0, group g = Hq / Hkv */
    int32_t head_dim;      /* d */
    int32_t block_size;    /* b, tokens per block (= tokens per page) */
    float sm_scale;        /* softmax scale; 0 selects 1/sqrt(d) (Eq. 1) */
} resa_config_t;

/* Row map.  Without one (rows == NULL) the call's sequence i is row i of
 * page_table and seq_len, which then hold `batch` rows.  With one, the call
 * covers `batch` sequences drawn from a larger table: sequence i reads row
 * rows[i] (device int32 [batch]) of page_table and seq_len, which hold
 * `table_rows` rows, while every per-call array (q, k_new, v_new, topk,
 * block lists, chunks, outputs) stays indexed by i.  This is how one batch
 * mixes sequences in different phases of their ReSA cycle (the decoding ones
 * in one resa_decode_step, the rectifying ones in one resa_rectify_attention,
 * both on the same cache; ReSA summary §3.4.2-§3.4.3, per-request
 * rectification in continuous batching).  The rows of one call must be
 * distinct.  A row outside [0, table_rows) sets RESA_DEVERR_ROW (and
 * RESA_DEVERR_SEQ_LEN) and the sequence is treated as empty. */
typedef struct {
    void *k;                    /* [num_pages][Hkv][b][d] bf16, device */
    void *v;                    /* [num_pages][Hkv][b][d] bf16, device */
    void *desc;                 /* [num_pages][Hkv][2][d] bf16, device */
    const int32_t *page_table;  /* [rows][max_pages], device */
    const int32_t *seq_len;     /* [rows], device; counts the decode token */
    int32_t batch;              /* sequences this call covers */
    int32_t max_pages;          /* row length of page_table = max blocks per sequence */
    int32_t num_pages;          /* physical pages in k / v / desc */
    const int32_t *rows;        /* row map [batch], device, or NULL (see above) */
    int32_t table_rows;         /* rows of page_table / seq_len when rows != NULL */
} resa_cache_t;

/* Bytes of workspace needed for caches of `batch` sequences with up to
 * `max_pages` blocks each and rectification chunks of up to `max_chunk`
 * tokens (0 if resa_rectify_attention is not used). */
RESA_API size_t resa_workspace_size(const resa_config_t *cfg, int32_t batch, int32_t max_pages,
                           int32_t max_chunk);

/* Zero the workspace (error word and completion counters).  Asynchronous. */
RESA_API resa_status_t resa_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream);

/* Synchronise `stream`, copy the device error word to *code_out (nullable),
 * clear it, and return RESA_ERR_DEVICE_CHECK if it was non-zero. */
RESA_API resa_status_t resa_check_device_status(void *ws, size_t ws_bytes, cudaStream_t stream,
                                       uint32_t *code_out);

/* Block key cache construction (ReSA summary §3.2 "Block Key Cache", Eq. 3;
 * Algorithm 1 initialisation): for every sequence b and kv head h, write the
 * element-wise min and max of the keys of each block that holds tokens
 * (blocks first_block[b] .. ceil(L/b)-1; the last block over its valid tokens
 * only).  first_block is a device [batch] int32 array or NULL (= 0).  Reads k,
 * writes desc.  Min/max of bf16 is exact, so descriptors are bit-exact. */
RESA_API resa_status_t resa_build_descriptors(const resa_config_t *cfg, const resa_cache_t *cache,
                                     const int32_t *first_block, void *ws, size_t ws_bytes,
                                     cudaStream_t stream);

/* Incremental cache update (Algorithm 1, "Incremental cache updates"): write
 * the decode token's key and value, k_new / v_new [batch][Hkv][d] bf16, at
 * position L-1 and fold its key into the descriptor of block (L-1)/b (a new
 * block starts with min = max = key when L-1 is a multiple of b). */
RESA_API resa_status_t resa_append_token(const resa_config_t *cfg, const resa_cache_t *cache,
                                 const void *k_new, const void *v_new, void *ws, size_t ws_bytes,
                                 cudaStream_t stream);

/* Query-aware block selection (ReSA summary §3.4.1: group pooling, Eq. 4
 * scores, Eq. 5 top-n with the local window n_local = 1):
 *   - pooled query of GQA group h: mean of q[b][h*g .. h*g+g-1] in fp32;
 *   - score of complete block i < M: sum_j max(qbar_j*max_ij, qbar_j*min_ij);
 *   - the k_eff = min(topk[b], M) highest-scoring complete blocks (ties to the
 *     lower block index), listed in ascending block order, then block c.
 * q: [batch][Hq][d] bf16.  topk: device [batch] int32 (the caller evaluates
 * Eq. 5).  Outputs: block_idx [batch][Hkv][max_topk+1] int32 and block_cnt
 * [batch][Hkv] int32 = k_eff + 1; entries past block_cnt are unspecified.
 * scores_opt (nullable): [batch][Hkv][max_pages] fp32, entries >= M
 * unspecified.  topk[b] > max_topk sets RESA_DEVERR_TOPK and is clamped. */
RESA_API resa_status_t resa_select_blocks(const resa_config_t *cfg, const resa_cache_t *cache,
                                 const void *q, const int32_t *topk, int32_t max_topk,
                                 int32_t *block_idx, int32_t *block_cnt, float *scores_opt,
                                 void *ws, size_t ws_bytes, cudaStream_t stream);

/* Group block-sparse attention, GBSA (ReSA summary §3.4.1 Eq. 2; kernel
 * §3.4.4): every query head of group h attends to the token positions t < L
 * of the blocks block_idx[b][h][0 .. block_cnt[b][h]-1] with logits
 * sm_scale * q.k, split across SMs with a log-sum-exp combine.  K/V of a
 * block are fetched once per group.  q [batch][Hq][d] bf16; out
 * [batch][Hq][d] fp32; lse_opt (nullable) [batch][Hq] fp32, natural log.
 * Block ids outside the sequence set RESA_DEVERR_BLOCK and are skipped.
 * max_topk + 1 above 1024 * 512 blocks returns RESA_ERR_RANGE. */
RESA_API resa_status_t resa_sparse_decode(const resa_config_t *cfg, const resa_cache_t *cache,
                                 const void *q, const int32_t *block_idx,
                                 const int32_t *block_cnt, int32_t max_topk, float *out,
                                 float *lse_opt, void *ws, size_t ws_bytes, cudaStream_t stream);

/* Dense rectification (ReSA summary §3.4.2; Algorithm 1, rectification
 * check): with L = seq_len[b],
 *   1. overwrite K/V at positions L-f .. L-1 with k_new / v_new [batch][f][Hkv][d];
 *   2. rebuild the descriptors of blocks (L-f)/b .. (L-1)/b;
 *   3. causal dense chunk attention: query row r of q_chunk [batch][f][Hq][d]
 *      (position L-f+r) attends to positions 0 .. L-f+r.
 * out [batch][f][Hq][d] fp32, lse_opt (nullable) [batch][f][Hq] fp32.
 * f must be in 1 .. max_chunk of the workspace; f > L sets RESA_DEVERR_CHUNK
 * and the sequence is skipped.  The keys of each (sequence, kv head) are split
 * across CTAs (enough to fill the SMs, and at least one split per 16384 keys
 * of the longest sequence); the splits' partial results live in the workspace
 * and are merged in the same call.  Two launches. */
RESA_API resa_status_t resa_rectify_attention(const resa_config_t *cfg, const resa_cache_t *cache,
                                     int32_t f, const void *q_chunk, const void *k_new,
                                     const void *v_new, float *out, float *lse_opt, void *ws,
                                     size_t ws_bytes, cudaStream_t stream);

/* One sparse decode step of one layer (Algorithm 1 inner body): append the
 * decode token (as resa_append_token), select blocks (as resa_select_blocks)
 * and attend (as resa_sparse_decode).  seq_len must already count the decode
 * token.  block_idx_opt / block_cnt_opt (nullable) receive the selection in
 * the layout of resa_select_blocks; when NULL it lives in the workspace.
 * When block_size is 16, batch * Hkv <= 74, g <= 8 and max_pages <= 65536
 * (and each of the G = 148 / (batch * Hkv) CTAs per (sequence, kv head)
 * scores at most 1024 blocks) the whole step is one cooperative launch: the
 * CTAs of a (sequence, kv head) score their share of the descriptors, agree on the selection
 * through one bounded counter in the workspace, split the selected blocks
 * evenly and hand their partial results over as words tagged with the
 * call's generation; other shapes run as three launches (append fused with the
 * scores, selection, sparse decode).  resa_decode_step_launches tells which.
 * Both give the same selection; outputs agree to fp32 rounding. */
RESA_API resa_status_t resa_decode_step(const resa_config_t *cfg, const resa_cache_t *cache,
                               const void *q, const void *k_new, const void *v_new,
                               const int32_t *topk, int32_t max_topk, float *out, float *lse_opt,
                               int32_t *block_idx_opt, int32_t *block_cnt_opt, void *ws,
                               size_t ws_bytes, cudaStream_t stream);

/* Dense decode attention, the baseline the sparse step is measured against
 * (ReSA summary §5 "Experimental Analysis", dense decoding; Eq. 1): append the
 * decode token (as resa_append_token) and attend, for every query head, to
 * every position 0 .. L-1 with logits sm_scale * q.k, split across SMs with a
 * log-sum-exp combine.  No descriptor is scored and nothing is selected; the
 * append still keeps the block key cache current for later sparse steps.
 * q [batch][Hq][d] bf16, k_new / v_new [batch][Hkv][d] bf16; out
 * [batch][Hq][d] fp32, lse_opt (nullable) [batch][Hq] fp32, natural log.
 * seq_len must already count the decode token.  One launch. */
RESA_API resa_status_t resa_dense_decode(const resa_config_t *cfg, const resa_cache_t *cache,
                                         const void *q, const void *k_new, const void *v_new,
                                         float *out, float *lse_opt, void *ws, size_t ws_bytes,
                                         cudaStream_t stream);

/* The group block-sparse decode of resa_sparse_decode for callers that
 * cannot allocate device memory.  The pages describe no such variant: it
 * exists for hosts that give this library only input and output pointers,
 * e.g. a serving engine that reserves all of HBM for its own KV-cache pool
 * at start-up, or a plugin interface that forbids device allocations after
 * initialisation, and so cannot provide a workspace.
 *   - Takes the arguments of resa_sparse_decode minus the workspace; the
 *     decode scratch (split or warp partials, split tickets, grid barrier,
 *     error word) lives in a fixed 16 MiB device array inside the library,
 *     held by every GPU that loads it until the process exits.  Nothing is
 *     allocated or freed.
 *   - Limit: batch * Hkv <= 4096 and batch * Hkv * splits * 16 * (d + 2) * 4
 *     bytes of partials must fit the array (about 16 MiB); larger calls
 *     return RESA_ERR_SHAPE.  Splits are chosen as in resa_sparse_decode, and
 *     as there max_topk + 1 above 1024 * 512 blocks returns RESA_ERR_RANGE
 *     before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (a runtime query, done once per device with that device current); make
 *     that first call before any stream capture.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents; the call clears the parts that must start at zero.
 *     Calls that overlap on the GPU (different streams, or host threads
 *     without ordering) race on the array: serialise them.
 *   - dev_error (required, device uint32, 4-byte aligned, zeroed by the
 *     caller before first use) receives, OR-ed in, the device error bits
 *     that resa_check_device_status reports for the workspace path; the call
 *     never clears it.  NULL returns RESA_ERR_NULL: the scratch array is
 *     reset by every call, so it cannot hold errors until someone reads them. */
RESA_API resa_status_t resa_sparse_decode_noalloc(const resa_config_t *cfg,
                                                  const resa_cache_t *cache, const void *q,
                                                  const int32_t *block_idx,
                                                  const int32_t *block_cnt, int32_t max_topk,
                                                  float *out, float *lse_opt,
                                                  uint32_t *dev_error, cudaStream_t stream);

/* Number of kernels each entry point launches per call (for launch
 * accounting): 1 for append and build, 2 for select, 1 for sparse decode,
 * 2 for rectify, 1 for a decode step of the fused shapes (see
 * resa_decode_step_launches for the others), 1 for the no-allocation decode,
 * 1 for the dense decode.
 * Unknown names return -1. */
RESA_API int32_t resa_kernels_per_call(const char *entry_point);

/* Kernels resa_decode_step launches for caches of `batch` sequences of
 * max_pages blocks over num_pages physical pages: 1 (fused step) or 3; -1 for
 * an invalid configuration.  Reads the current device's SM count. */
RESA_API int32_t resa_decode_step_launches(const resa_config_t *cfg, int32_t batch,
                                           int32_t max_pages, int32_t num_pages);

/* Human-readable status name. */
RESA_API const char *resa_status_string(resa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* RESA_H_ */
