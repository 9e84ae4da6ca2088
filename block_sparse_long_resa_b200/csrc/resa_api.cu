// Host side of libresa: argument validation, workspace layout, TMA tensor
// maps and kernel launches for the entry points declared in include/resa.h.
#include <math.h>
#include <string.h>

#include "resa_common.cuh"

namespace resa {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;  // a driver entry point: immutable once found
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// One channel half (64 columns) of a K or V cache as a 2-D tensor: rows are
// tokens of every (page, head) block (row stride d*2 bytes); one box is the
// bs rows x 64 channels of one block, 128-byte swizzled.
bool make_kv_half_map(CUtensorMap *map, void *base, int half, int num_pages, int hkv, int d,
                      int bs) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    void *b = static_cast<uint8_t *>(base) + (size_t)half * 128;
    const cuuint64_t dims[2] = {64, (cuuint64_t)num_pages * hkv * bs};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)bs};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, b, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The same channel half as a 4-D tensor (channels, tokens, heads, pages):
// one box is the bs tokens of one head on the 64 / bs consecutive pages of a
// 64-key tile, 128-byte swizzled, laid out in shared memory exactly as that
// many single-block boxes.
bool make_kv_half_run_map(CUtensorMap *map, void *base, int half, int num_pages, int hkv, int d,
                          int bs) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    void *b = static_cast<uint8_t *>(base) + (size_t)half * 128;
    const cuuint64_t dims[4] = {64, (cuuint64_t)bs, (cuuint64_t)hkv, (cuuint64_t)num_pages};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)bs * d * 2,
                                   (cuuint64_t)hkv * bs * d * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)bs, 1, (cuuint32_t)(64 / bs)};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, b, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

resa_status_t check_config(const resa_config_t *cfg, Shape *s) {
    if (!cfg) return RESA_ERR_NULL;
    if (cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 || cfg->head_dim <= 0 ||
        cfg->block_size <= 0)
        return RESA_ERR_SHAPE;
    if (cfg->num_q_heads % cfg->num_kv_heads != 0) return RESA_ERR_SHAPE;
    const int g = cfg->num_q_heads / cfg->num_kv_heads;
    if (g > kMaxGroup) return RESA_ERR_UNSUPPORTED;
    const int hkv = cfg->num_kv_heads;
    if (!(hkv == 1 || hkv == 2 || hkv == 4 || hkv == 8)) return RESA_ERR_UNSUPPORTED;
    if (!(cfg->head_dim == 64 || cfg->head_dim == 128)) return RESA_ERR_UNSUPPORTED;
    if (!(cfg->block_size == 16 || cfg->block_size == 32 || cfg->block_size == 64))
        return RESA_ERR_UNSUPPORTED;
    if (!(cfg->sm_scale >= 0.f) || isinf(cfg->sm_scale)) return RESA_ERR_RANGE;
    s->hq = cfg->num_q_heads;
    s->hkv = hkv;
    s->g = g;
    s->d = cfg->head_dim;
    s->bs = cfg->block_size;
    s->sm_scale = cfg->sm_scale > 0.f ? cfg->sm_scale : 1.0f / sqrtf((float)cfg->head_dim);
    return RESA_OK;
}

resa_status_t check_cache(const resa_cache_t *c, Shape *s, bool need_v, bool need_desc) {
    if (!c) return RESA_ERR_NULL;
    if (!c->k || !c->page_table || !c->seq_len) return RESA_ERR_NULL;
    if (need_v && !c->v) return RESA_ERR_NULL;
    if (need_desc && !c->desc) return RESA_ERR_NULL;
    if (c->batch <= 0 || c->max_pages <= 0 || c->num_pages <= 0) return RESA_ERR_SHAPE;
    if ((long long)c->max_pages * s->bs > 0x7fffffffLL) return RESA_ERR_RANGE;
    if ((long long)c->num_pages * s->hkv * s->bs > 0x7fffffffLL) return RESA_ERR_RANGE;
    if (!aligned16(c->k) || (c->v && !aligned16(c->v)) || (c->desc && !aligned16(c->desc)) ||
        !aligned16(c->page_table) || !aligned16(c->seq_len))
        return RESA_ERR_UNSUPPORTED;
    if (c->rows != nullptr && (c->table_rows <= 0 || !aligned16(c->rows)))
        return c->table_rows <= 0 ? RESA_ERR_SHAPE : RESA_ERR_UNSUPPORTED;
    s->batch = c->batch;
    s->max_pages = c->max_pages;
    s->num_pages = c->num_pages;
    s->rows = RowMap{c->rows, c->rows ? c->table_rows : c->batch};
    return RESA_OK;
}

resa_status_t check_ws(void *ws, size_t ws_bytes, const WsLayout &w) {
    if (!ws) return RESA_ERR_NULL;
    if (!aligned16(ws)) return RESA_ERR_UNSUPPORTED;
    if (ws_bytes < w.total) return RESA_ERR_SHAPE;
    return RESA_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

resa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? RESA_OK : RESA_ERR_CUDA; }

#define RESA_TRY(expr)                        \
    do {                                      \
        resa_status_t _st = (expr);           \
        if (_st != RESA_OK) return _st;       \
    } while (0)

WsLayout layout_of(const Shape &s, int chunk) {
    return ws_layout(s.hq, s.hkv, s.d, s.bs, s.batch, s.max_pages, chunk);
}


// Score (optionally appending the decode token in the same launch), then select.
resa_status_t select_impl(const Shape &s, const resa_cache_t *c, const WsLayout &w, void *ws,
                          const void *q, const int32_t *topk, int max_topk, int32_t *idx,
                          int32_t *cnt, float *scores, const void *k_new, const void *v_new,
                          cudaStream_t st) {
    uint32_t *err = at<uint32_t>(ws, w.err);
    uint32_t *hist = at<uint32_t>(ws, w.hist);
    uint32_t *range = at<uint32_t>(ws, w.hist_range);
    const bool append = k_new != nullptr;
    RESA_TRY(cuda_status(launch_score(s, c->desc, c->page_table, c->seq_len, q, scores, hist,
                                      range, append ? c->k : nullptr, append ? c->v : nullptr,
                                      k_new, v_new, err, st)));
    RESA_TRY(cuda_status(launch_select(s, scores, hist, range, c->seq_len, topk, max_topk, idx,
                                       cnt, err, st)));
    return RESA_OK;
}

int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int c = cache[dev].load();
    if (c == 0) {
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev].store(c);
    }
    return c;
}

// CTAs per (sequence, kv head) of the fused decode step for this shape, 0 when
// the step runs as three launches (score + append, select, decode).
int fused_step_ctas(const Shape &s) {
    if (s.bs != 16) return 0;                            // 16-token blocks only
    if ((long long)s.num_pages >= (1LL << 27)) return 0;  // packed (page, tokens) work items
    return step_ctas_per_unit(s.batch * s.hkv, s.g, s.d, s.max_pages, sm_count());
}

resa_status_t decode_impl(const Shape &s, const resa_cache_t *c, const WsLayout &w, void *ws,
                          const void *q, const int32_t *idx, const int32_t *cnt, int max_topk,
                          float *out, float *lse, cudaStream_t st) {
    const int splits = decode_splits_for(s.batch * s.hkv, max_topk + 1);
    if (splits > w.dec_splits) return RESA_ERR_RANGE;  // max_topk far above max_pages
    if (splits > kMaxDecodeSplits) return RESA_ERR_RANGE;
    return cuda_status(launch_sparse_decode(
        s, c->k, c->v, c->page_table, c->seq_len, q, idx, cnt, max_topk, splits,
        at<float>(ws, w.dec_o), at<float>(ws, w.dec_lse), at<uint32_t>(ws, w.dec_ticket),
        at<uint32_t>(ws, w.err + kDecBarrierOffset), out, lse, at<uint32_t>(ws, w.err), st));
}

}  // namespace
}  // namespace resa

using namespace resa;

extern "C" {

size_t resa_workspace_size(const resa_config_t *cfg, int32_t batch, int32_t max_pages,
                           int32_t max_chunk) {
    Shape s{};
    if (check_config(cfg, &s) != RESA_OK || batch <= 0 || max_pages <= 0 || max_chunk < 0)
        return 0;
    size_t best = ws_layout(s.hq, s.hkv, s.d, s.bs, batch, max_pages, 0).total;
    for (int f = 1; f <= max_chunk; ++f) {
        if (rect_row_groups(f, s.g) > kMaxRowTiles) break;
        const size_t t = ws_layout(s.hq, s.hkv, s.d, s.bs, batch, max_pages, f).total;
        best = t > best ? t : best;
    }
    return best;
}

resa_status_t resa_workspace_init(void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (!ws) return RESA_ERR_NULL;
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, stream));
}

resa_status_t resa_check_device_status(void *ws, size_t ws_bytes, cudaStream_t stream,
                                       uint32_t *code_out) {
    if (!ws) return RESA_ERR_NULL;
    if (ws_bytes < 4) return RESA_ERR_SHAPE;
    uint32_t code = 0;
    if (cudaMemcpyAsync(&code, ws, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return RESA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return RESA_ERR_CUDA;
    if (code_out) *code_out = code;
    if (code != 0) {
        if (cudaMemsetAsync(ws, 0, 4, stream) != cudaSuccess) return RESA_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return RESA_ERR_CUDA;
        return RESA_ERR_DEVICE_CHECK;
    }
    return RESA_OK;
}

resa_status_t resa_build_descriptors(const resa_config_t *cfg, const resa_cache_t *cache,
                                     const int32_t *first_block, void *ws, size_t ws_bytes,
                                     cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, false, true));
    const WsLayout w = layout_of(s, 0);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    return cuda_status(launch_build_descriptors(s, cache->k, cache->desc, cache->page_table,
                                                cache->seq_len, first_block,
                                                at<uint32_t>(ws, w.err), stream));
}

resa_status_t resa_append_token(const resa_config_t *cfg, const resa_cache_t *cache,
                                const void *k_new, const void *v_new, void *ws, size_t ws_bytes,
                                cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, true, true));
    if (!k_new || !v_new) return RESA_ERR_NULL;
    if (!aligned16(k_new) || !aligned16(v_new)) return RESA_ERR_UNSUPPORTED;
    const WsLayout w = layout_of(s, 0);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    return cuda_status(launch_append(s, cache->k, cache->v, cache->desc, cache->page_table,
                                     cache->seq_len, k_new, v_new, at<uint32_t>(ws, w.err),
                                     stream));
}

resa_status_t resa_select_blocks(const resa_config_t *cfg, const resa_cache_t *cache,
                                 const void *q, const int32_t *topk, int32_t max_topk,
                                 int32_t *block_idx, int32_t *block_cnt, float *scores_opt,
                                 void *ws, size_t ws_bytes, cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, false, true));
    if (!q || !topk || !block_idx || !block_cnt) return RESA_ERR_NULL;
    if (max_topk < 0) return RESA_ERR_RANGE;
    if (!aligned16(q) || !aligned16(topk) || !aligned16(block_idx) || !aligned16(block_cnt) ||
        (scores_opt && !aligned16(scores_opt)))
        return RESA_ERR_UNSUPPORTED;
    const WsLayout w = layout_of(s, 0);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    float *scores = scores_opt ? scores_opt : at<float>(ws, w.scores);
    return select_impl(s, cache, w, ws, q, topk, max_topk, block_idx, block_cnt, scores, nullptr,
                       nullptr, stream);
}

resa_status_t resa_sparse_decode(const resa_config_t *cfg, const resa_cache_t *cache,
                                 const void *q, const int32_t *block_idx,
                                 const int32_t *block_cnt, int32_t max_topk, float *out,
                                 float *lse_opt, void *ws, size_t ws_bytes, cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, true, false));
    if (!q || !block_idx || !block_cnt || !out) return RESA_ERR_NULL;
    if (max_topk < 0) return RESA_ERR_RANGE;
    if (!aligned16(q) || !aligned16(out)) return RESA_ERR_UNSUPPORTED;
    const WsLayout w = layout_of(s, 0);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    return decode_impl(s, cache, w, ws, q, block_idx, block_cnt, max_topk, out, lse_opt, stream);
}

resa_status_t resa_rectify_attention(const resa_config_t *cfg, const resa_cache_t *cache,
                                     int32_t f, const void *q_chunk, const void *k_new,
                                     const void *v_new, float *out, float *lse_opt, void *ws,
                                     size_t ws_bytes, cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, true, true));
    if (!q_chunk || !k_new || !v_new || !out) return RESA_ERR_NULL;
    if (f < 1) return RESA_ERR_RANGE;
    if (rect_row_groups(f, s.g) > kMaxRowTiles) return RESA_ERR_UNSUPPORTED;
    if (!aligned16(q_chunk) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out))
        return RESA_ERR_UNSUPPORTED;
    const WsLayout w = layout_of(s, f);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    uint32_t *err = at<uint32_t>(ws, w.err);
    RESA_TRY(cuda_status(launch_rectify_writeback(s, cache->k, cache->v, cache->desc,
                                                  cache->page_table, cache->seq_len, f, k_new,
                                                  v_new, err, stream)));
    // 2-D single-block maps (K half 0, 1, V half 0, 1), then the 4-page maps
    CUtensorMap maps[8];
    const int halves = s.d / 64;
    for (int hf = 0; hf < 2; ++hf) {
        const int use = hf < halves ? hf : 0;  // d = 64: one half, second map unused
        if (!make_kv_half_map(&maps[hf], cache->k, use, s.num_pages, s.hkv, s.d, s.bs) ||
            !make_kv_half_map(&maps[2 + hf], cache->v, use, s.num_pages, s.hkv, s.d, s.bs) ||
            !make_kv_half_run_map(&maps[4 + hf], cache->k, use, s.num_pages, s.hkv, s.d, s.bs) ||
            !make_kv_half_run_map(&maps[6 + hf], cache->v, use, s.num_pages, s.hkv, s.d, s.bs))
            return RESA_ERR_CUDA;
    }
    return cuda_status(launch_rectify_attention(
        s, maps, cache->page_table, cache->seq_len, f, q_chunk, w.row_tiles, w.rect_splits,
        at<float>(ws, w.rect_o), at<float>(ws, w.rect_lse), at<uint32_t>(ws, w.rect_ticket), out,
        lse_opt, err, stream));
}

resa_status_t resa_decode_step(const resa_config_t *cfg, const resa_cache_t *cache,
                               const void *q, const void *k_new, const void *v_new,
                               const int32_t *topk, int32_t max_topk, float *out, float *lse_opt,
                               int32_t *block_idx_opt, int32_t *block_cnt_opt, void *ws,
                               size_t ws_bytes, cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, true, true));
    if (!q || !k_new || !v_new || !topk || !out) return RESA_ERR_NULL;
    if (max_topk < 0) return RESA_ERR_RANGE;
    if (max_topk > cache->max_pages && (!block_idx_opt || !block_cnt_opt)) return RESA_ERR_RANGE;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(topk) ||
        !aligned16(out) || (block_idx_opt && !aligned16(block_idx_opt)) ||
        (block_cnt_opt && !aligned16(block_cnt_opt)))
        return RESA_ERR_UNSUPPORTED;
    const WsLayout w = layout_of(s, 0);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    int32_t *idx = block_idx_opt && block_cnt_opt ? block_idx_opt : at<int32_t>(ws, w.sel_idx);
    int32_t *cnt = block_idx_opt && block_cnt_opt ? block_cnt_opt : at<int32_t>(ws, w.sel_cnt);
    const int G = fused_step_ctas(s);
    if (G > 0) {
        StepBuffers buf;
        buf.block_idx = idx;
        buf.block_cnt = cnt;
        buf.hist = at<uint32_t>(ws, w.hist);
        buf.hist_range = at<uint32_t>(ws, w.hist_range);
        buf.bars = at<unsigned long long>(ws, w.step_bars);
        buf.ukeys = at<uint32_t>(ws, w.step_keys);
        buf.part = at<unsigned long long>(ws, w.step_part);
        buf.err = at<uint32_t>(ws, w.err);
        return cuda_status(launch_decode_step_fused(s, G, cache->k, cache->v, cache->desc,
                                                    cache->page_table, cache->seq_len, q, k_new,
                                                    v_new, topk, max_topk, out, lse_opt, buf,
                                                    stream));
    }
    // append + scores in one launch (the append touches only the current
    // block, which is never scored), then select, then attend
    RESA_TRY(select_impl(s, cache, w, ws, q, topk, max_topk, idx, cnt, at<float>(ws, w.scores),
                         k_new, v_new, stream));
    return decode_impl(s, cache, w, ws, q, idx, cnt, max_topk, out, lse_opt, stream);
}

resa_status_t resa_dense_decode(const resa_config_t *cfg, const resa_cache_t *cache,
                                const void *q, const void *k_new, const void *v_new, float *out,
                                float *lse_opt, void *ws, size_t ws_bytes, cudaStream_t stream) {
    Shape s{};
    RESA_TRY(check_config(cfg, &s));
    RESA_TRY(check_cache(cache, &s, true, true));
    if (!q || !k_new || !v_new || !out) return RESA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out))
        return RESA_ERR_UNSUPPORTED;
    const WsLayout w = layout_of(s, 0);
    RESA_TRY(check_ws(ws, ws_bytes, w));
    // every block of the sequence: max_topk + 1 = max_pages entries
    const int splits = decode_splits_for(s.batch * s.hkv, s.max_pages);
    if (splits > w.dec_splits || splits > kMaxDecodeSplits) return RESA_ERR_RANGE;
    DecodeAppend app;
    app.k = cache->k;
    app.v = cache->v;
    app.desc = cache->desc;
    app.k_new = static_cast<const uint4 *>(k_new);
    app.v_new = static_cast<const uint4 *>(v_new);
    return cuda_status(launch_sparse_decode(
        s, cache->k, cache->v, cache->page_table, cache->seq_len, q, nullptr, nullptr,
        s.max_pages - 1, splits, at<float>(ws, w.dec_o), at<float>(ws, w.dec_lse),
        at<uint32_t>(ws, w.dec_ticket), at<uint32_t>(ws, w.err + kDecBarrierOffset), out, lse_opt,
        at<uint32_t>(ws, w.err), stream, app));
}

int32_t resa_decode_step_launches(const resa_config_t *cfg, int32_t batch, int32_t max_pages,
                                  int32_t num_pages) {
    Shape s{};
    if (check_config(cfg, &s) != RESA_OK || batch <= 0 || max_pages <= 0 || num_pages <= 0)
        return -1;
    s.batch = batch;
    s.max_pages = max_pages;
    s.num_pages = num_pages;
    return fused_step_ctas(s) > 0 ? 1 : 3;
}

int32_t resa_kernels_per_call(const char *entry_point) {
    if (!entry_point) return -1;
    struct {
        const char *name;
        int n;
    } table[] = {{"resa_build_descriptors", 1}, {"resa_append_token", 1},
                 {"resa_select_blocks", 2},     {"resa_sparse_decode", 1},
                 {"resa_rectify_attention", 2}, {"resa_decode_step", 1},
                 {"resa_sparse_decode_noalloc", 1}, {"resa_dense_decode", 1}};
    for (auto &e : table)
        if (strcmp(e.name, entry_point) == 0) return e.n;
    return -1;
}

const char *resa_status_string(resa_status_t st) {
    switch (st) {
        case RESA_OK: return "RESA_OK";
        case RESA_ERR_NULL: return "RESA_ERR_NULL";
        case RESA_ERR_SHAPE: return "RESA_ERR_SHAPE";
        case RESA_ERR_RANGE: return "RESA_ERR_RANGE";
        case RESA_ERR_UNSUPPORTED: return "RESA_ERR_UNSUPPORTED";
        case RESA_ERR_CUDA: return "RESA_ERR_CUDA";
        case RESA_ERR_DEVICE_CHECK: return "RESA_ERR_DEVICE_CHECK";
    }
    return "RESA_ERR_UNKNOWN";
}

}  // extern "C"
