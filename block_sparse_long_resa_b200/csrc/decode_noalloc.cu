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

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kScratchMaxUnits = 4096;             // batch * Hkv
constexpr size_t kScratchHeader = 256;  // error word; grid barrier at kDecBarrierOffset

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

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Same K/V tensor-map geometry as the workspace path: one (page, head) block
// of 16 x d per box, 128-byte swizzled.
bool kv_map(CUtensorMap *map, void *base, int num_pages, int hkv, int d) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    const cuuint64_t dims[3] = {64, (cuuint64_t)(d / 64), (cuuint64_t)num_pages * hkv * kBlock};
    const cuuint64_t strides[2] = {128, (cuuint64_t)d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)(d / 64), (cuuint32_t)kBlock};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
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
                                                    uint32_t *dev_error_opt, cudaStream_t stream) {
    if (!cfg || !cache || !q || !block_idx || !block_cnt || !out) return RESA_ERR_NULL;
    if (!cache->k || !cache->v || !cache->page_table || !cache->seq_len) return RESA_ERR_NULL;
    if (cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 ||
        cfg->num_q_heads % cfg->num_kv_heads != 0)
        return RESA_ERR_SHAPE;
    const int hkv = cfg->num_kv_heads, g = cfg->num_q_heads / cfg->num_kv_heads;
    if (g > kMaxGroup || !(hkv == 1 || hkv == 2 || hkv == 4 || hkv == 8) ||
        !(cfg->head_dim == 64 || cfg->head_dim == 128) || cfg->block_size != kBlock)
        return RESA_ERR_UNSUPPORTED;
    if (!(cfg->sm_scale >= 0.f) || isinf(cfg->sm_scale)) return RESA_ERR_RANGE;
    if (cache->batch <= 0 || cache->max_pages <= 0 || cache->num_pages <= 0) return RESA_ERR_SHAPE;
    if ((long long)cache->max_pages * kBlock > 0x7fffffffLL ||
        (long long)cache->num_pages * hkv * kBlock > 0x7fffffffLL || max_topk < 0)
        return RESA_ERR_RANGE;
    if (!al16(cache->k) || !al16(cache->v) || !al16(cache->page_table) || !al16(cache->seq_len) ||
        !al16(q) || !al16(out))
        return RESA_ERR_UNSUPPORTED;

    // Size the scratch use and refuse what does not fit.
    const int units = cache->batch * hkv;
    if (units > kScratchMaxUnits) return RESA_ERR_SHAPE;
    const int d = cfg->head_dim;
    const int splits = decode_splits_for(units, max_topk + 1);
    const size_t tickets_bytes = align_up((size_t)units * 4, 256);
    const size_t lse_bytes = align_up((size_t)units * splits * kMaxGroup * 4, 256);
    const size_t o_bytes = (size_t)units * splits * kMaxGroup * d * 4;
    if (kScratchHeader + tickets_bytes + lse_bytes + o_bytes > kScratchBytes) return RESA_ERR_SHAPE;

    void *base = nullptr;
    const resa_status_t st = scratch_address(&base);
    if (st != RESA_OK) return st;
    uint8_t *scratch = static_cast<uint8_t *>(base);
    uint32_t *err = reinterpret_cast<uint32_t *>(scratch);
    uint32_t *tickets = reinterpret_cast<uint32_t *>(scratch + kScratchHeader);
    float *part_lse = reinterpret_cast<float *>(scratch + kScratchHeader + tickets_bytes);
    float *part_o = reinterpret_cast<float *>(scratch + kScratchHeader + tickets_bytes + lse_bytes);
    // The array keeps the previous call's contents: the error word and the
    // split tickets must start at zero.
    if (cudaMemsetAsync(scratch, 0, kScratchHeader + tickets_bytes, stream) != cudaSuccess)
        return RESA_ERR_CUDA;

    CUtensorMap kmap, vmap;
    if (!kv_map(&kmap, cache->k, cache->num_pages, hkv, d) ||
        !kv_map(&vmap, cache->v, cache->num_pages, hkv, d))
        return RESA_ERR_CUDA;
    Shape s{};
    s.hq = cfg->num_q_heads;
    s.hkv = hkv;
    s.g = g;
    s.d = d;
    s.bs = kBlock;
    s.sm_scale = cfg->sm_scale > 0.f ? cfg->sm_scale : 1.0f / sqrtf((float)d);
    s.batch = cache->batch;
    s.max_pages = cache->max_pages;
    s.num_pages = cache->num_pages;
    const cudaError_t e = launch_sparse_decode(
        s, kmap, vmap, cache->page_table, cache->seq_len, q, block_idx, block_cnt, max_topk,
        splits, part_o, part_lse, tickets,
        reinterpret_cast<uint32_t *>(scratch + kDecBarrierOffset), out, lse_opt,
        dev_error_opt ? dev_error_opt : err, stream);
    return e == cudaSuccess ? RESA_OK : RESA_ERR_CUDA;
}
