// Dense rectification chunk attention (ReSA summary §3.4.2; Algorithm 1,
// rectification check): the f chunk queries of every group head attend
// causally to the whole cache after the chunk's fresh K/V were written back.
//
// Rows of one (sequence, kv head) are rho = r * g + j (chunk position r,
// group head j; position L - f + r).  Grid (row tiles, splits, batch * Hkv):
// a CTA owns kRectRowsPerTile rows (four warps x 16) and one contiguous range
// of KV blocks; thread 0 streams the range as tiles of four blocks (64
// tokens) through a two-stage ring with 3-D TMA loads (one per (page, head)
// block for K and for V), the warps release a stage through an mbarrier.
// The row tiles of one KV range are adjacent in the grid, so they run
// together and share the range through L2.  Partial (o, lse) per split are
// merged by the CTA that draws the last ticket of its (unit, row tile).
#include "attn_common.cuh"

namespace resa {
namespace {

constexpr int kRWarps = 4;
constexpr int kRThreads = kRWarps * 32;
constexpr int kRStages = 2;
constexpr int kBlocksPerTile = 4;


template <int D>
struct RectSmem {
    static constexpr int kTileBytes = kBlock * D * 2;
    static constexpr int kStageBytes = 2 * kBlocksPerTile * kTileBytes;  // K blocks, then V blocks
    static constexpr int kBytes = kRStages * kStageBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kRThreads)
    rectify_attn_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap,
                        const int32_t *__restrict__ page_table, const int32_t *__restrict__ seq_len,
                        int f, const uint16_t *__restrict__ q_chunk, int hkv, int g, int max_pages,
                        int num_pages, float scale_log2, float *__restrict__ part_o,
                        float *__restrict__ part_lse, uint32_t *__restrict__ tickets,
                        float *__restrict__ out, float *__restrict__ lse_out, uint32_t *err) {
    using SM = RectSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    __shared__ uint64_t full[kRStages], empty[kRStages];
    __shared__ uint32_t sh_last;

    const int tile = blockIdx.x, split = blockIdx.y, unit = blockIdx.z;
    const int RT = gridDim.x, S = gridDim.y;
    const int b = unit / hkv, h = unit % hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hq = hkv * g;
    const int rows_total = f * g;

    const int L = seq_len[b];
    bool seq_ok = L >= 1 && L <= max_pages * kBlock && f <= L;
    if (!seq_ok && threadIdx.x == 0 && tile == 0 && split == 0)
        set_error(err, (L < 1 || L > max_pages * kBlock) ? RESA_DEVERR_SEQ_LEN : RESA_DEVERR_CHUNK);
    const int start = L - f;

    // Rows of this lane and their causal limits (tokens < lim are visible).
    const int rbase = tile * kRectRowsPerTile + warp * 16;
    const int rho0 = rbase + (lane >> 2), rho1 = rho0 + 8;
    const int lim0 = (seq_ok && rho0 < rows_total) ? start + rho0 / g + 1 : 0;
    const int lim1 = (seq_ok && rho1 < rows_total) ? start + rho1 / g + 1 : 0;
    // KV blocks any row of this CTA can see, split S ways.
    const int last_row = min(rows_total, (tile + 1) * kRectRowsPerTile) - 1;
    const int lim_max = seq_ok && tile * kRectRowsPerTile < rows_total ? start + last_row / g + 1 : 0;
    const int nblk = (lim_max + kBlock - 1) / kBlock;
    const int per = (nblk + S - 1) / S;
    const int blk0 = min(nblk, split * per), blk1 = min(nblk, blk0 + per);
    const int ntiles = (blk1 - blk0 + kBlocksPerTile - 1) / kBlocksPerTile;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kRWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    auto page_of = [&](int blk) -> int {
        const int p = page_table[(size_t)b * max_pages + blk];
        return (p >= 0 && p < num_pages) ? p : -1;
    };
    auto issue = [&](int i) {  // thread 0 only
        uint8_t *st = smem + (size_t)(i % kRStages) * SM::kStageBytes;
        uint32_t bytes = 0;
        int pages[kBlocksPerTile];
        for (int sub = 0; sub < kBlocksPerTile; ++sub) {
            const int blk = blk0 + i * kBlocksPerTile + sub;
            pages[sub] = blk < blk1 ? page_of(blk) : -1;
            if (blk < blk1 && pages[sub] < 0) set_error(err, RESA_DEVERR_PAGE);
            if (pages[sub] >= 0) bytes += 2 * SM::kTileBytes;
        }
        uint64_t *bar = &full[i % kRStages];
        if (bytes == 0) {
            mbar_arrive(bar);
            return;
        }
        mbar_arrive_expect_tx(bar, bytes);
        for (int sub = 0; sub < kBlocksPerTile; ++sub) {
            if (pages[sub] < 0) continue;
            const int row = (pages[sub] * hkv + h) * kBlock;
            tma_load_3d(st + sub * SM::kTileBytes, &kmap, 0, 0, row, bar);
            tma_load_3d(st + (kBlocksPerTile + sub) * SM::kTileBytes, &vmap, 0, 0, row, bar);
        }
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < ntiles && i < kRStages; ++i) issue(i);

    uint32_t qa[D / 16][4];
    {
        auto qrow = [&](int rho) -> const uint16_t * {
            if (!seq_ok || rho >= rows_total) return nullptr;
            const int r = rho / g, j = rho % g;
            return q_chunk + (((size_t)b * f + r) * hq + (size_t)h * g + j) * D;
        };
        load_q_frags<D>(qa, qrow(rho0), qrow(rho1), lane);
    }

    RowState<D> st;
    st.init();
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
        const int stage = i % kRStages;
        if (!mbar_wait_bounded(&full[stage], (i / kRStages) & 1)) {
            ok = false;
            break;
        }
        const uint32_t sbase = smem_u32(smem + (size_t)stage * SM::kStageBytes);
        for (int sub = 0; sub < kBlocksPerTile; ++sub) {
            const int blk = blk0 + i * kBlocksPerTile + sub;
            if (blk >= blk1) break;
            if (page_of(blk) < 0) continue;
            const int tok0 = blk * kBlock;
            const int n0 = max(0, min(kBlock, lim0 - tok0));
            const int n1 = max(0, min(kBlock, lim1 - tok0));
            if (!__any_sync(0xffffffffu, n0 > 0 || n1 > 0)) continue;
            attend_tile16<D>(st, qa, sbase + sub * SM::kTileBytes,
                             sbase + (kBlocksPerTile + sub) * SM::kTileBytes, n0, n1, scale_log2,
                             lane);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (threadIdx.x == 0 && i + kRStages < ntiles) {
            if (mbar_wait_bounded(&empty[stage], (i / kRStages) & 1))
                issue(i + kRStages);
            else
                ok = false;
        }
    }
    if (!ok && lane == 0) set_error(err, RESA_DEVERR_TIMEOUT);
    finish_rows<D>(st);

    const float kLn2 = 0.6931471805599453f;
    const int cb = 2 * (lane & 3);
    const size_t slot = ((size_t)unit * RT + tile) * S + split;
    // Normalised partial rows of this split (or the final rows when S == 1).
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int rho = half ? rho1 : rho0;
        if (rho >= rows_total) continue;
        const float l = st.l[half];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse2 = l > 0.f ? st.m[half] + log2f(st.lx[half]) : -INFINITY;
        const int r = rho / g, j = rho % g;
        const size_t orow = ((size_t)b * f + r) * hq + (size_t)h * g + j;
        const int rl = rho - tile * kRectRowsPerTile;
        float *dst = S == 1 ? out + orow * D : part_o + (slot * kRectRowsPerTile + rl) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            float2 v = make_float2(st.acc[n][2 * half] * inv, st.acc[n][2 * half + 1] * inv);
            *reinterpret_cast<float2 *>(dst + n * 8 + cb) = v;
        }
        if ((lane & 3) == 0) {
            if (S == 1) {
                if (lse_out) lse_out[orow] = lse2 * kLn2;
            } else {
                part_lse[slot * kRectRowsPerTile + rl] = lse2;
            }
        }
    }
    if (S == 1) return;

    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(&tickets[(size_t)unit * kMaxRowTiles + tile], 1u);
        sh_last = ticket == (uint32_t)(S - 1);
    }
    __syncthreads();
    if (!sh_last) return;
    __threadfence();
    const size_t slot0 = ((size_t)unit * RT + tile) * S;
    const int nrows = min(kRectRowsPerTile, rows_total - tile * kRectRowsPerTile);
    for (int e = threadIdx.x; e < nrows * D; e += kRThreads) {
        const int rl = e / D, c = e % D;
        float mstar = -INFINITY;
        for (int s = 0; s < S; ++s)
            mstar = fmaxf(mstar, __ldcg(&part_lse[(slot0 + s) * kRectRowsPerTile + rl]));
        float wsum = 0.f, o = 0.f;
        if (mstar != -INFINITY) {
            for (int s = 0; s < S; ++s) {
                const float w = exp2f(__ldcg(&part_lse[(slot0 + s) * kRectRowsPerTile + rl]) - mstar);
                wsum += w;
                o += w * __ldcg(&part_o[((slot0 + s) * kRectRowsPerTile + rl) * D + c]);
            }
        }
        const int rho = tile * kRectRowsPerTile + rl;
        const int r = rho / g, j = rho % g;
        const size_t orow = ((size_t)b * f + r) * hq + (size_t)h * g + j;
        out[orow * D + c] = wsum > 0.f ? o / wsum : 0.f;
        if (lse_out && c == 0)
            lse_out[orow] = wsum > 0.f ? (mstar + log2f(wsum)) * kLn2 : -INFINITY;
    }
    if (threadIdx.x == 0) tickets[(size_t)unit * kMaxRowTiles + tile] = 0;
}

template <int D>
cudaError_t launch_d(const Shape &s, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     const int32_t *page_table, const int32_t *seq_len, int f, const void *q_chunk,
                     int row_tiles, int splits, float *part_o, float *part_lse, uint32_t *tickets,
                     float *out, float *lse, uint32_t *err, cudaStream_t st) {
    constexpr int smem = RectSmem<D>::kBytes;
    static std::atomic<int> done[64];
    cudaError_t e = ensure_smem(rectify_attn_kernel<D>, smem, done);
    if (e != cudaSuccess) return e;
    const float scale_log2 = s.sm_scale * 1.4426950408889634f;
    dim3 grid(row_tiles, splits, s.batch * s.hkv);
    rectify_attn_kernel<D><<<grid, kRThreads, smem, st>>>(
        kmap, vmap, page_table, seq_len, f, (const uint16_t *)q_chunk, s.hkv, s.g, s.max_pages,
        s.num_pages, scale_log2, part_o, part_lse, tickets, out, lse, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rectify_attention(const Shape &s, const CUtensorMap &kmap,
                                     const CUtensorMap &vmap, const int32_t *page_table,
                                     const int32_t *seq_len, int f, const void *q_chunk,
                                     int row_tiles, int splits, float *part_o, float *part_lse,
                                     uint32_t *tickets, float *out, float *lse, uint32_t *err,
                                     cudaStream_t st) {
    if (row_tiles > kMaxRowTiles) return cudaErrorInvalidValue;
    if (s.d == 128)
        return launch_d<128>(s, kmap, vmap, page_table, seq_len, f, q_chunk, row_tiles, splits,
                             part_o, part_lse, tickets, out, lse, err, st);
    if (s.d == 64)
        return launch_d<64>(s, kmap, vmap, page_table, seq_len, f, q_chunk, row_tiles, splits,
                            part_o, part_lse, tickets, out, lse, err, st);
    return cudaErrorInvalidValue;
}

}  // namespace resa
