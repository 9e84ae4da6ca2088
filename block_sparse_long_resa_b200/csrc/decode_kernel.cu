// Group block-sparse split-KV decode (GBSA, ReSA summary §3.4.1 Eq. 2; kernel
// design §3.4.4 / Algorithm 2, re-done for sm_100a).
//
// Grid (splits, Hkv, batch).  CTA (split s, kv head h, sequence b) takes the
// s-th contiguous slice of the group's selected block list; each of its four
// warps takes every fourth block of the slice and keeps its own online-softmax
// state for the group's g query heads (rows of one m16 MMA tile), so the K/V
// of a block are fetched once for the whole group.  A warp streams its blocks
// through a private ring of kStages shared-memory stages: lane 0 issues two
// 3-D TMA loads per block (K and V, each one (page, head) tile of 16 x D bf16,
// 128-byte swizzled) that complete on the stage's mbarrier.
//
// The CTA merges its warps' states, then either writes the final output (one
// split) or a partial (o, lse) and takes an atomic ticket; the CTA that draws
// the last ticket of its (sequence, kv head) merges every split's partial and
// resets the ticket.  No CTA waits on another.
#include "attn_common.cuh"

namespace resa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 3;

template <int D>
struct DecodeSmem {
    static constexpr int kTileBytes = kBlock * D * 2;               // one K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kMergeBytes = kWarps * kMaxGroup * (D + 3) * 4;
    static constexpr int kBytes = (kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes) + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads)
    sparse_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap,
                         const int32_t *__restrict__ page_table,
                         const int32_t *__restrict__ seq_len, const uint16_t *__restrict__ q,
                         const int32_t *__restrict__ block_idx,
                         const int32_t *__restrict__ block_cnt, int max_topk, int hkv, int g,
                         int max_pages, int num_pages, float scale_log2, float *__restrict__ part_o,
                         float *__restrict__ part_lse, uint32_t *__restrict__ tickets,
                         float *__restrict__ out, float *__restrict__ lse_out, uint32_t *err) {
    using SM = DecodeSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    __shared__ uint64_t bars[kWarps][kStages];
    __shared__ uint32_t sh_last;

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int S = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hq = hkv * g;
    const size_t unit = (size_t)b * hkv + h;

    int L = seq_len[b];
    int cnt = block_cnt[unit];
    if (L < 1 || L > max_pages * kBlock) {
        if (threadIdx.x == 0 && split == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        cnt = 0;
    }
    cnt = max(0, min(cnt, max_topk + 1));
    const int per = (cnt + S - 1) / S;
    const int j0 = min(cnt, split * per), j1 = min(cnt, j0 + per);
    const int32_t *list = block_idx + unit * (max_topk + 1);
    const int nblk_seq = (L + kBlock - 1) / kBlock;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < kStages; ++s) mbar_init(&bars[w][s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    // This warp's blocks: j0 + warp + kWarps * t, t = 0 .. n_mine-1.
    const int first = j0 + warp;
    const int n_mine = first < j1 ? (j1 - first + kWarps - 1) / kWarps : 0;
    uint8_t *ring = smem + (size_t)warp * kStages * SM::kStageBytes;

    // Returns valid tokens of the t-th block (0 when skipped); lane 0 issues
    // its loads into stage t % kStages (or completes the phase without data).
    auto block_tokens = [&](int t, int &page_out) -> int {
        const int blk = list[first + kWarps * t];
        int page = -1;
        if (blk >= 0 && blk < nblk_seq) page = page_table[(size_t)b * max_pages + blk];
        page_out = page;
        if (page < 0 || page >= num_pages) return 0;
        return min(kBlock, L - blk * kBlock);
    };
    auto issue = [&](int t) {
        int page;
        const int nt = block_tokens(t, page);
        uint64_t *bar = &bars[warp][t % kStages];
        if (nt > 0) {
            uint8_t *st = ring + (size_t)(t % kStages) * SM::kStageBytes;
            const int row = (page * hkv + h) * kBlock;
            mbar_arrive_expect_tx(bar, SM::kStageBytes);
            tma_load_3d(st, &kmap, 0, 0, row, bar);
            tma_load_3d(st + SM::kTileBytes, &vmap, 0, 0, row, bar);
        } else {
            const int blk = list[first + kWarps * t];
            set_error(err, (blk >= 0 && blk < nblk_seq) ? RESA_DEVERR_PAGE : RESA_DEVERR_BLOCK);
            mbar_arrive(bar);
        }
    };

    if (lane == 0)
        for (int t = 0; t < n_mine && t < kStages; ++t) issue(t);

    // Query fragments: rows r < g are the group's query heads.
    uint32_t qa[D / 16][4];
    {
        const int r0 = lane >> 2, r1 = r0 + 8;
        const uint16_t *base = q + ((size_t)b * hq + (size_t)h * g) * D;
        load_q_frags<D>(qa, r0 < g ? base + (size_t)r0 * D : nullptr,
                        r1 < g ? base + (size_t)r1 * D : nullptr, lane);
    }

    RowState<D> st;
    st.init();
    bool ok = true;
    int t_done = 0;
    for (int t = 0; t < n_mine; ++t) {
        const int stage = t % kStages;
        if (!mbar_wait_bounded(&bars[warp][stage], (t / kStages) & 1)) {
            ok = false;
            break;
        }
        int page;
        const int nt = block_tokens(t, page);
        if (nt > 0) {
            const uint32_t ks = smem_u32(ring + (size_t)stage * SM::kStageBytes);
            attend_tile16<D>(st, qa, ks, ks + SM::kTileBytes, nt, nt, scale_log2, lane);
        }
        t_done = t + 1;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && t + kStages < n_mine) issue(t + kStages);
    }
    if (!ok) {
        if (lane == 0) set_error(err, RESA_DEVERR_TIMEOUT);
        // drain: give every issued load a bounded chance to land before exit
        for (int t = t_done; t < n_mine && t < t_done + kStages; ++t)
            mbar_wait_bounded(&bars[warp][t % kStages], (t / kStages) & 1);
    }
    finish_rows<D>(st);
    __syncthreads();  // every warp is done with its ring: reuse it for the merge

    // Merge the warps: per warp m[16], l[16], lx[16], acc[16][D] (unnormalised).
    float *mw = reinterpret_cast<float *>(smem);
    float *lw = mw + kWarps * kMaxGroup;
    float *lxw = lw + kWarps * kMaxGroup;
    float *ow = lxw + kWarps * kMaxGroup;
    {
        const int r0 = lane >> 2, r1 = r0 + 8, cb = 2 * (lane & 3);
        if ((lane & 3) == 0) {
            mw[warp * kMaxGroup + r0] = st.m[0];
            mw[warp * kMaxGroup + r1] = st.m[1];
            lw[warp * kMaxGroup + r0] = st.l[0];
            lw[warp * kMaxGroup + r1] = st.l[1];
            lxw[warp * kMaxGroup + r0] = st.lx[0];
            lxw[warp * kMaxGroup + r1] = st.lx[1];
        }
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            float *o0 = ow + ((size_t)warp * kMaxGroup + r0) * D + j * 8 + cb;
            float *o1 = ow + ((size_t)warp * kMaxGroup + r1) * D + j * 8 + cb;
            o0[0] = st.acc[j][0];
            o0[1] = st.acc[j][1];
            o1[0] = st.acc[j][2];
            o1[1] = st.acc[j][3];
        }
    }
    __syncthreads();
    const float kLn2 = 0.6931471805599453f;
    float *po = part_o + (unit * S + split) * kMaxGroup * D;
    float *pl = part_lse + (unit * S + split) * kMaxGroup;
    for (int e = threadIdx.x; e < g * D; e += kThreads) {
        const int r = e / D, c = e % D;
        float mstar = -INFINITY;
        for (int w = 0; w < kWarps; ++w) mstar = fmaxf(mstar, mw[w * kMaxGroup + r]);
        float lsum = 0.f, lxsum = 0.f, o = 0.f;
        if (mstar != -INFINITY) {
            for (int w = 0; w < kWarps; ++w) {
                const float sc = exp2f(mw[w * kMaxGroup + r] - mstar);
                lsum += lw[w * kMaxGroup + r] * sc;
                lxsum += lxw[w * kMaxGroup + r] * sc;
                o += ow[((size_t)w * kMaxGroup + r) * D + c] * sc;
            }
        }
        const float lse2 = lsum > 0.f ? mstar + log2f(lxsum) : -INFINITY;
        const float on = lsum > 0.f ? o / lsum : 0.f;
        if (S == 1) {
            out[((size_t)b * hq + (size_t)h * g + r) * D + c] = on;
            if (lse_out && c == 0) lse_out[(size_t)b * hq + (size_t)h * g + r] = lse2 * kLn2;
        } else {
            po[(size_t)r * D + c] = on;
            if (c == 0) pl[r] = lse2;
        }
    }
    if (S == 1) return;

    // Split combine: the CTA that draws the last ticket merges all splits.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(&tickets[unit], 1u);
        sh_last = ticket == (uint32_t)(S - 1);
    }
    __syncthreads();
    if (!sh_last) return;
    __threadfence();
    const float *uo = part_o + unit * S * kMaxGroup * D;
    const float *ul = part_lse + unit * S * kMaxGroup;
    for (int e = threadIdx.x; e < g * D; e += kThreads) {
        const int r = e / D, c = e % D;
        float mstar = -INFINITY;
        for (int s = 0; s < S; ++s) mstar = fmaxf(mstar, __ldcg(&ul[s * kMaxGroup + r]));
        float wsum = 0.f, o = 0.f;
        if (mstar != -INFINITY) {
            for (int s = 0; s < S; ++s) {
                const float w = exp2f(__ldcg(&ul[s * kMaxGroup + r]) - mstar);
                wsum += w;
                o += w * __ldcg(&uo[((size_t)s * kMaxGroup + r) * D + c]);
            }
        }
        out[((size_t)b * hq + (size_t)h * g + r) * D + c] = wsum > 0.f ? o / wsum : 0.f;
        if (lse_out && c == 0)
            lse_out[(size_t)b * hq + (size_t)h * g + r] =
                wsum > 0.f ? (mstar + log2f(wsum)) * kLn2 : -INFINITY;
    }
    if (threadIdx.x == 0) tickets[unit] = 0;
}

template <int D>
cudaError_t launch_d(const Shape &s, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     const int32_t *page_table, const int32_t *seq_len, const void *q,
                     const int32_t *block_idx, const int32_t *block_cnt, int max_topk, int splits,
                     float *part_o, float *part_lse, uint32_t *tickets, float *out, float *lse,
                     uint32_t *err, cudaStream_t st) {
    constexpr int smem = DecodeSmem<D>::kBytes;
    static std::atomic<int> done[64];
    cudaError_t e = ensure_smem(sparse_decode_kernel<D>, smem, done);
    if (e != cudaSuccess) return e;
    const float scale_log2 = s.sm_scale * 1.4426950408889634f;
    dim3 grid(splits, s.hkv, s.batch);
    sparse_decode_kernel<D><<<grid, kThreads, smem, st>>>(
        kmap, vmap, page_table, seq_len, (const uint16_t *)q, block_idx, block_cnt, max_topk,
        s.hkv, s.g, s.max_pages, s.num_pages, scale_log2, part_o, part_lse, tickets, out, lse,
        err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_decode(const Shape &s, const CUtensorMap &kmap, const CUtensorMap &vmap,
                                 const int32_t *page_table, const int32_t *seq_len, const void *q,
                                 const int32_t *block_idx, const int32_t *block_cnt, int max_topk,
                                 int splits, float *part_o, float *part_lse, uint32_t *tickets,
                                 float *out, float *lse, uint32_t *err, cudaStream_t st) {
    if (s.d == 128)
        return launch_d<128>(s, kmap, vmap, page_table, seq_len, q, block_idx, block_cnt,
                             max_topk, splits, part_o, part_lse, tickets, out, lse, err, st);
    if (s.d == 64)
        return launch_d<64>(s, kmap, vmap, page_table, seq_len, q, block_idx, block_cnt, max_topk,
                            splits, part_o, part_lse, tickets, out, lse, err, st);
    return cudaErrorInvalidValue;
}

}  // namespace resa
