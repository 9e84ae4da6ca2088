// resa_sparse_decode_noalloc: the group block-sparse decode of
// resa_sparse_decode for callers that cannot allocate device memory.
//
// Some hosts hand this library nothing but input and output pointers: a
// serving engine that reserves all of HBM for its own KV-cache pool at start
// and has no allocator to lend, or a plugin interface whose contract forbids
// device allocations after initialisation.  Such callers cannot provide the
// workspace the other entry points take.  This entry point keeps the decode
// kernel's scratch (split partials, split tickets, error word) in a
// file-scope device array instead, so it needs no workspace and calls no
// allocating routine.  The array is a fixed kScratchBytes per GPU, held for
// the life of the process by every GPU that loads the library.
#include <mutex>

#include "resa_common.cuh"

namespace resa {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kScratchMaxUnits = 4096;             // batch * Hkv
constexpr size_t kScratchHeader = 256;  // grid barrier at kDecBarrierOffset

// Shared by every call on a device; it keeps the previous call's contents.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[64];  // device address of g_decode_scratch, per device

// Host code cannot use g_decode_scratch's name as a device address; ask the
// runtime for it once per device, with that device current.
resa_status_t scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RESA_ERR_CUDA;
    if (dev < 0 || dev >= 64) return RESA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) return RESA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return RESA_OK;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace resa

using namespace resa;

extern "C" resa_status_t resa_sparse_decode_noalloc(const resa_config_t *cfg,
                                                    const resa_cache_t *cache, const void *q,
                                                    const int32_t *block_idx,
                                                    const int32_t *block_cnt, int32_t max_topk,
                                                    float *out, float *lse_opt,
                                                    uint32_t *dev_error, cudaStream_t stream) {
    if (!cfg || !cache || !q || !block_idx || !block_cnt || !out || !dev_error) return RESA_ERR_NULL;
    if (!cache->k || !cache->v || !cache->page_table || !cache->seq_len) return RESA_ERR_NULL;
    if (cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 ||
        cfg->num_q_heads % cfg->num_kv_heads != 0)
        return RESA_ERR_SHAPE;
    const int hkv = cfg->num_kv_heads, g = cfg->num_q_heads / cfg->num_kv_heads;
    if (g > kMaxGroup || !(hkv == 1 || hkv == 2 || hkv == 4 || hkv == 8) ||
        !(cfg->head_dim == 64 || cfg->head_dim == 128) ||
        !(cfg->block_size == 16 || cfg->block_size == 32 || cfg->block_size == 64))
        return RESA_ERR_UNSUPPORTED;
    if (!(cfg->sm_scale >= 0.f) || isinf(cfg->sm_scale)) return RESA_ERR_RANGE;
    if (cache->batch <= 0 || cache->max_pages <= 0 || cache->num_pages <= 0) return RESA_ERR_SHAPE;
    if (cache->rows != nullptr && cache->table_rows <= 0) return RESA_ERR_SHAPE;
    const int bs = cfg->block_size;
    if ((long long)cache->max_pages * bs > 0x7fffffffLL ||
        (long long)cache->num_pages * hkv * bs > 0x7fffffffLL || max_topk < 0)
        return RESA_ERR_RANGE;
    // The split merge holds the weights of at most kMaxDecodeSplits splits:
    // the same bound resa_sparse_decode enforces (max_topk + 1 <= 1024 * 512).
    if ((long long)max_topk + 1 > (long long)kMaxDecodeSplits * kMaxBlocksPerSplit)
        return RESA_ERR_RANGE;
    if (!al16(cache->k) || !al16(cache->v) || !al16(cache->page_table) || !al16(cache->seq_len) ||
        (cache->rows != nullptr && !al16(cache->rows)) || !al16(q) || !al16(out) ||
        (reinterpret_cast<uintptr_t>(dev_error) & 3u) != 0)
        return RESA_ERR_UNSUPPORTED;

    // Size the scratch use and refuse what does not fit.
    const int units = cache->batch * hkv;
    if (units > kScratchMaxUnits) return RESA_ERR_SHAPE;
    const int d = cfg->head_dim;
    const int splits = decode_splits_for(units, max_topk + 1);
    if (splits > kMaxDecodeSplits) return RESA_ERR_RANGE;
    const size_t tickets_bytes = align_up((size_t)units * 4, 256);
    // Per-warp partials for a grid-wide merge when they fit the array, else
    // per-split partials and the last-CTA merge.
    const size_t spread_parts = (size_t)units * splits * kDecodeWarps;
    const bool spread_fits = kScratchHeader + tickets_bytes +
                                 align_up(spread_parts * kMaxGroup * 8, 256) +
                                 spread_parts * kMaxGroup * d * 4 <=
                             kScratchBytes;
    const size_t parts = spread_fits ? spread_parts : (size_t)units * splits;
    const size_t lse_bytes = align_up(parts * kMaxGroup * 8, 256);
    const size_t o_bytes = parts * kMaxGroup * d * 4;
    if (kScratchHeader + tickets_bytes + lse_bytes + o_bytes > kScratchBytes) return RESA_ERR_SHAPE;

    void *base = nullptr;
    const resa_status_t st = scratch_address(&base);
    if (st != RESA_OK) return st;
    uint8_t *scratch = static_cast<uint8_t *>(base);
    uint32_t *tickets = reinterpret_cast<uint32_t *>(scratch + kScratchHeader);
    float *part_lse = reinterpret_cast<float *>(scratch + kScratchHeader + tickets_bytes);
    float *part_o = reinterpret_cast<float *>(scratch + kScratchHeader + tickets_bytes + lse_bytes);
    // The array keeps the previous call's contents: the grid barrier word and
    // the split tickets must start at zero.  Device errors go to the caller's
    // word, never to the array, so the next call cannot wipe them unread.
    if (cudaMemsetAsync(scratch, 0, kScratchHeader + tickets_bytes, stream) != cudaSuccess)
        return RESA_ERR_CUDA;

    Shape s{};
    s.hq = cfg->num_q_heads;
    s.hkv = hkv;
    s.g = g;
    s.d = d;
    s.bs = bs;
    s.sm_scale = cfg->sm_scale > 0.f ? cfg->sm_scale : 1.0f / sqrtf((float)d);
    s.batch = cache->batch;
    s.max_pages = cache->max_pages;
    s.num_pages = cache->num_pages;
    s.rows = RowMap{cache->rows, cache->rows ? cache->table_rows : cache->batch};
    const cudaError_t e = launch_sparse_decode(
        s, cache->k, cache->v, cache->page_table, cache->seq_len, q, block_idx, block_cnt, max_topk,
        splits, part_o, part_lse, tickets,
        spread_fits ? reinterpret_cast<uint32_t *>(scratch + kDecBarrierOffset) : nullptr, out,
        lse_opt, dev_error, stream);
    return e == cudaSuccess ? RESA_OK : RESA_ERR_CUDA;
}
