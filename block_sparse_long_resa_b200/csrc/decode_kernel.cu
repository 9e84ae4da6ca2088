// Group block-sparse split-KV decode (GBSA, ReSA summary §3.4.1 Eq. 2; the
// split-execution kernel of §3.4.4, redone for sm_100a).
//
// Grid (splits, Hkv, batch), one 8-warp CTA per SM.  CTA (s, h, b) takes the
// s-th contiguous slice of the group's selected block list (or of every block
// without a list); a block of b tokens is b / 16 tiles of 16 tokens, and warp
// w takes every eighth tile of the slice and keeps its own online-softmax
// state for the group's g query heads, so the K/V of a block are fetched once
// for the whole group.  Each warp streams its tiles through a private ring of
// kStages shared-memory stages with 16-byte cp.async copies (the (page,
// head) K and V tiles of 16 x D bf16, laid out 128-byte swizzled for
// ldmatrix): copies through the load/store path keep HBM busy with 4 KB
// tiles, where one TMA request per tile is limited by the copy engine's
// per-request rate.  Block ids and pages of the slice are staged in shared
// memory once, up front.
//
// The MMAs run with the operands swapped, S^T = K Q^T and O^T = V^T P^T
// (bf16 m16n8k16, fp32 accumulate), so the g <= 8 heads of a group fill the
// N = 8 side instead of wasting 9 of 16 M rows; P^T is transposed in
// registers with movmatrix and enters the P.V MMA as bf16 hi + lo parts.
//
// The CTA merges its warps, then writes the final output (one split) or a
// partial (o, log2-sum-exp).  When the grid fits one wave it is launched
// cooperatively and, after a bounded grid barrier, every CTA merges a slice
// of the outputs.  Otherwise each CTA draws an atomic ticket and the CTA
// drawing the last ticket of its (sequence, kv head) pulls every split's
// partial into shared memory with bulk copies, merges them and resets the
// ticket.
#include "attn_common.cuh"

namespace resa {
namespace {

constexpr int kWarps = kDecodeWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 3;

template <int D>
struct DecodeSmem {
    static constexpr int kTileBytes = kTileRows * D * 2;  // one K or V tile (16 tokens)
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
    static constexpr int kMergeBytes = kWarps * kMaxGroup * (D + 3) * 4;
    static_assert(kRingBytes >= kMaxDecodeSplits * kMaxGroup * 4 + kMaxGroup * D * 4,
                  "split merge: the weights of every split and one partial tile fit the ring");
    static constexpr int kBytes = (kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes) + 1024;
};

// Block-wide reductions through shared memory (red: kWarps floats + 1).
__device__ __forceinline__ float block_max(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float x = lane < kWarps ? red[lane] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
        if (lane == 0) red[kWarps] = x;
    }
    __syncthreads();
    const float r = red[kWarps];
    __syncthreads();
    return r;
}
__device__ __forceinline__ float block_sum(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float x = lane < kWarps ? red[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) red[kWarps] = x;
    }
    __syncthreads();
    const float r = red[kWarps];
    __syncthreads();
    return r;
}

// Merge of per-warp partials spread over the whole (co-resident) grid.
// Partial p of unit u holds, per query row, the row max m (log2 domain), the
// sum l of 2^(x - m) and the unnormalised sum o of 2^(x - m) * v over the
// warp's blocks.  Work item = (unit, row, 32 output channels); CTA c takes
// items c, c + gridsize, ...  Each warp first requests its partials' o
// values (w, w + 8, ...: up to kB loads in flight per lane, independent of
// the weights), then the CTA reads every partial's (m, l), forms M = max m
// and the weights 2^(m - M), L = sum of l * 2^(m - M), and each warp adds
// its weighted o values; out = (sum of the eight warps) / L.
template <int D>
__device__ __forceinline__ void merge_warp_partials(const float *__restrict__ part_o,
                                                    const float2 *__restrict__ part_ml, int P,
                                                    int hkv, int g, float *__restrict__ out,
                                                    float *__restrict__ lse_out, float *smem_f) {
    constexpr int C32 = D / 32;
    constexpr int kB = 40;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nctas = gridDim.x * gridDim.y * gridDim.z;
    const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    const int units = gridDim.y * gridDim.z;
    const int n_items = units * g * C32;
    const float kLn2 = 0.6931471805599453f;
    float *msm = smem_f;             // [P] row max of each partial
    float *wsm = msm + P;            // [P] its weight 2^(m - M) (0 without data)
    float *lsm = wsm + P;            // [P] its l
    float *red = lsm + P;            // [kWarps * 32] warp sums, reduction scratch
    for (int item = cta; item < n_items; item += nctas) {
        const int u = item / (g * C32), rem = item % (g * C32);
        const int r = rem / C32, cc = rem % C32;
        const float2 *ml = part_ml + (size_t)u * P * kMaxGroup + r;
        const float *uo = part_o + ((size_t)u * P * kMaxGroup + r) * D + cc * 32 + lane;
        float v[kB];
        auto load_pass = [&](int base) {
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const int pp = base + kWarps * k;
                v[k] = pp < P ? __ldcg(uo + (size_t)pp * kMaxGroup * D) : 0.f;
            }
        };
        load_pass(warp);
        float tmax = -INFINITY;
        for (int pp = threadIdx.x; pp < P; pp += kThreads) {
            const float2 x = __ldcg(ml + (size_t)pp * kMaxGroup);
            msm[pp] = x.x;
            lsm[pp] = x.y;
            if (x.y > 0.f) tmax = fmaxf(tmax, x.x);
        }
        const float M = block_max(tmax, red);
        float tl = 0.f;
        for (int pp = threadIdx.x; pp < P; pp += kThreads) {
            const float w = lsm[pp] > 0.f ? exp2f(msm[pp] - M) : 0.f;
            wsm[pp] = w;
            tl += lsm[pp] * w;
        }
        const float Lsum = block_sum(tl, red);  // its barriers also publish wsm
        float acc = 0.f;
        for (int base = warp; base < P; base += kWarps * kB) {
            if (base != warp) load_pass(base);
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const int pp = base + kWarps * k;
                if (pp < P) acc += wsm[pp] * v[k];
            }
        }
        red[warp * 32 + lane] = acc;
        __syncthreads();
        if (warp == 0) {
            float o = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) o += red[w * 32 + lane];
            const size_t orow = (size_t)(u / hkv) * hkv * g + (size_t)(u % hkv) * g + r;
            out[orow * D + cc * 32 + lane] = Lsum > 0.f ? o / Lsum : 0.f;
            if (lse_out && cc == 0 && lane == 0)
                lse_out[orow] = (Lsum > 0.f ? M + log2f(Lsum) : -INFINITY) * kLn2;
        }
        __syncthreads();
    }
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_decode_kernel(const uint8_t *k_cache, const uint8_t *v_cache,
                         const int32_t *__restrict__ page_table,
                         const int32_t *__restrict__ seq_len, const uint16_t *__restrict__ q,
                         const int32_t *__restrict__ block_idx,
                         const int32_t *__restrict__ block_cnt, int max_topk, int hkv, int g,
                         int max_pages, int num_pages, float scale_log2, float *__restrict__ part_o,
                         float *__restrict__ part_lse, uint32_t *__restrict__ tickets,
                         uint32_t *__restrict__ grid_bar, float *__restrict__ out,
                         float *__restrict__ lse_out, uint32_t *err, const DecodeAppend app,
                         const RowMap rm, int bs) {
    using SM = DecodeSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the shared array itself so that
    // accesses keep the shared address space (no generic loads)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ uint64_t merge_bar;
    __shared__ int2 meta[kMaxBlocksPerSplit];  // (page, valid tokens) of the slice's blocks
    __shared__ uint32_t sh_last;
    __shared__ float sh_lse[kMaxGroup];

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int S = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int hq = hkv * g;
    const size_t unit = (size_t)b * hkv + h;

    pdl_launch_next();
    const int row = cache_row(rm, b, threadIdx.x == 0 && split == 0 ? err : nullptr);
    const int L = row_seq_len(seq_len, row);
    if (threadIdx.x == 0) {
        mbar_init(&merge_bar, 1);
        fence_mbar_init();
    }
    // Q^T B fragments: head nt*8 + lane/4 (zero beyond g), channels 2*(lane%4)+{0,1} (+8).
    // q is an input of the step, so it is read before waiting for the selection.
    uint32_t qb[D / 16][NT][2];
    {
        const uint16_t *base = q + ((size_t)b * hq + (size_t)h * g) * D;
        const int c = 2 * (lane & 3);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int head = n * 8 + (lane >> 2);
            const uint16_t *row = head < g ? base + (size_t)head * D : nullptr;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qb[ks][n][0] = row ? *reinterpret_cast<const uint32_t *>(row + ks * 16 + c) : 0u;
                qb[ks][n][1] = row ? *reinterpret_cast<const uint32_t *>(row + ks * 16 + c + 8) : 0u;
            }
        }
    }
    pdl_wait();  // block lists / counts come from the preceding selection
    const bool seq_ok = L >= 1 && L <= max_pages * bs;
    const int nblk_seq = seq_ok ? (L + bs - 1) / bs : 0;
    // a block is bs / 16 tiles of 16 tokens
    const int sub_shift = bs == 64 ? 2 : bs == 32 ? 1 : 0;
    // without a block list (dense decoding) every block of the sequence
    int cnt = block_idx ? block_cnt[unit] : nblk_seq;
    if (!seq_ok) {
        if (threadIdx.x == 0 && split == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        cnt = 0;
    }
    cnt = max(0, min(cnt, block_idx ? max_topk + 1 : max_pages));
    const int per = (cnt + S - 1) / S;
    const int j0 = min(cnt, split * per), j1 = min(cnt, j0 + per);
    const int nslice = min(j1 - j0, kMaxBlocksPerSplit);  // the host sizes S so this holds
    const int32_t *list = block_idx ? block_idx + unit * (max_topk + 1) : nullptr;

    if (app.k_new != nullptr && cnt > 0 && j0 <= cnt - 1 && cnt - 1 < j1) {
        // Dense decoding appends the decode token itself: this CTA decodes the
        // current block (the last entry), and the barrier after the staging
        // below orders the append before its copies of that block.
        constexpr int CPR = D / 8;  // 16-byte chunks per K / V row
        if (threadIdx.x < CPR) {
            const int c = threadIdx.x, M = (L - 1) / bs, slot = (L - 1) % bs;
            const int page = page_table[(size_t)row * max_pages + M];
            if (page >= 0 && page < num_pages) {
                const uint4 kx = app.k_new[unit * CPR + c], vx = app.v_new[unit * CPR + c];
                const size_t o = (((size_t)page * hkv + h) * bs + slot) * CPR + c;
                reinterpret_cast<uint4 *>(app.k)[o] = kx;
                reinterpret_cast<uint4 *>(app.v)[o] = vx;
                uint4 *dmn = reinterpret_cast<uint4 *>(app.desc) + (((size_t)page * hkv + h) * 2) * CPR + c;
                if (slot == 0) {
                    dmn[0] = kx;
                    dmn[CPR] = kx;
                } else {
                    Bf16x8 mn = unpack8(dmn[0]), mx = unpack8(dmn[CPR]);
                    fold8(mn, mx, unpack8(kx));
                    dmn[0] = pack8(mn);
                    dmn[CPR] = pack8(mx);
                }
            } else if (c == 0) {
                set_error(err, RESA_DEVERR_PAGE);
            }
        }
    }

    for (int i = threadIdx.x; i < nslice; i += kThreads) {
        const int blk = list ? list[j0 + i] : j0 + i;
        int page = -1, ntok = 0;
        if (blk >= 0 && blk < nblk_seq) {
            page = page_table[(size_t)row * max_pages + blk];
            if (page >= 0 && page < num_pages)
                ntok = min(bs, L - blk * bs);
            else
                set_error(err, RESA_DEVERR_PAGE);
        } else {
            set_error(err, RESA_DEVERR_BLOCK);
        }
        meta[i] = make_int2(page, ntok);
    }
    __syncthreads();

    // The slice's 16-token tiles (bs / 16 per block, in order): this warp
    // takes tiles warp + kWarps * t.  Tile t goes to ring slot t % kStages:
    // its K and V (16 x D bf16 each, contiguous in the cache) are copied with
    // 16-byte cp.async, lane chunk q to the 128-byte-swizzled position of
    // (row q / 8, chunk q % 8), one copy group per tile (empty groups keep
    // the count uniform).
    const int nsub = nslice << sub_shift;
    const int n_mine = warp < nsub ? (nsub - warp + kWarps - 1) / kWarps : 0;
    uint8_t *ring = smem + (size_t)warp * kStages * SM::kStageBytes;
    constexpr int kPerLane = SM::kTileBytes / 16 / 32;
    // (page, valid tokens) of tile e of the slice
    auto tile_of = [&](int e) -> int2 {
        const int2 mt = meta[e >> sub_shift];
        const int j = e & ((1 << sub_shift) - 1);
        return make_int2(mt.x * (1 << sub_shift) + j, min(kTileRows, mt.y - kTileRows * j));
    };
    auto issue = [&](int t) {
        if (t < n_mine) {
            const int2 mt = tile_of(warp + kWarps * t);
            if (mt.y > 0) {
                const size_t tile =
                    (((size_t)(mt.x >> sub_shift) * hkv + h) << sub_shift | (mt.x & ((1 << sub_shift) - 1))) *
                    SM::kTileBytes;
                uint8_t *st = ring + (size_t)(t % kStages) * SM::kStageBytes;
#pragma unroll
                for (int k = 0; k < kPerLane; ++k) {
                    const uint32_t qc = lane + 32 * k;
                    const uint32_t so = swz128(qc >> 3, qc & 7);
                    cp_async16(st + so, k_cache + tile + qc * 16);
                    cp_async16(st + SM::kTileBytes + so, v_cache + tile + qc * 16);
                }
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int t = 0; t < kStages - 1; ++t) issue(t);

    WarpState<D, NT> st;
    st.init();
    for (int t = 0; t < n_mine; ++t) {
        issue(t + kStages - 1);  // refills the slot of block t - 1
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const int ntok = tile_of(warp + kWarps * t).y;
        if (ntok > 0) {
            const uint32_t ks = smem_u32(ring + (size_t)(t % kStages) * SM::kStageBytes);
            attend_block_swapped<D, NT>(st, qb, ks, ks + SM::kTileBytes, ntok, scale_log2, lane);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    // Row sums over the eight lanes that share each head.
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            st.l[n][k] += __shfl_xor_sync(0xffffffffu, st.l[n][k], 4);
            st.l[n][k] += __shfl_xor_sync(0xffffffffu, st.l[n][k], 8);
            st.l[n][k] += __shfl_xor_sync(0xffffffffu, st.l[n][k], 16);
        }
    __syncthreads();  // every ring is drained: reuse it for the merge

    if (grid_bar != nullptr) {
        // Spread mode (the grid is one wave, S >= 2): each warp's partial goes
        // straight to global memory; after a bounded grid barrier every CTA
        // merges a share of the outputs over all S * kWarps warp partials.
        const int P = S * kWarps;
        const size_t pidx = unit * P + (size_t)split * kWarps + warp;
        float *pw = part_o + pidx * kMaxGroup * D;
        float2 *pml = reinterpret_cast<float2 *>(part_lse) + pidx * kMaxGroup;
        const int hb = 2 * (lane & 3), d0 = lane >> 2;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int h0 = n * 8 + hb;
            if (lane < 4) {
                if (h0 < g) pml[h0] = make_float2(st.m[n][0], st.l[n][0]);
                if (h0 + 1 < g) pml[h0 + 1] = make_float2(st.m[n][1], st.l[n][1]);
            }
#pragma unroll
            for (int t = 0; t < D / 16; ++t) {
                float *o0 = pw + (size_t)h0 * D + t * 16 + d0;
                if (h0 < g) {
                    o0[0] = st.o[t][n][0];
                    o0[8] = st.o[t][n][2];
                }
                if (h0 + 1 < g) {
                    o0[D] = st.o[t][n][1];
                    o0[D + 8] = st.o[t][n][3];
                }
            }
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
            sh_last = grid_barrier_bounded(reinterpret_cast<unsigned long long *>(grid_bar), gridDim.x * gridDim.y * gridDim.z) ? 1u : 0u;
        __syncthreads();
        if (!sh_last) {
            if (threadIdx.x == 0) set_error(err, RESA_DEVERR_TIMEOUT);
            return;
        }
        __threadfence();
        merge_warp_partials<D>(part_o, reinterpret_cast<const float2 *>(part_lse), P, hkv, g, out,
                               lse_out, reinterpret_cast<float *>(smem));
        return;
    }

    float *mw = reinterpret_cast<float *>(smem);  // [kWarps][16]
    float *lw = mw + kWarps * kMaxGroup;          // [kWarps][16]
    float *ow = lw + kWarps * kMaxGroup;          // [kWarps][16][D]
    {
        const int hb = 2 * (lane & 3), d0 = lane >> 2;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            if (lane < 4) {
                mw[warp * kMaxGroup + n * 8 + hb] = st.m[n][0];
                mw[warp * kMaxGroup + n * 8 + hb + 1] = st.m[n][1];
                lw[warp * kMaxGroup + n * 8 + hb] = st.l[n][0];
                lw[warp * kMaxGroup + n * 8 + hb + 1] = st.l[n][1];
            }
#pragma unroll
            for (int t = 0; t < D / 16; ++t) {
                float *o0 = ow + ((size_t)warp * kMaxGroup + n * 8 + hb) * D + t * 16 + d0;
                o0[0] = st.o[t][n][0];
                o0[D] = st.o[t][n][1];
                o0[8] = st.o[t][n][2];
                o0[D + 8] = st.o[t][n][3];
            }
        }
    }
    __syncthreads();
    const float kLn2 = 0.6931471805599453f;
    float *po = part_o + (unit * S + split) * kMaxGroup * D;
    float *pl = part_lse + (unit * S + split) * kMaxGroup;
    for (int e = threadIdx.x; e < g * D; e += kThreads) {
        const int r = e / D, c = e % D;
        float mstar = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) mstar = fmaxf(mstar, mw[w * kMaxGroup + r]);
        float lsum = 0.f, o = 0.f;
        if (mstar != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float sc = exp2f(mw[w * kMaxGroup + r] - mstar);
                lsum += lw[w * kMaxGroup + r] * sc;
                o += ow[((size_t)w * kMaxGroup + r) * D + c] * sc;
            }
        }
        const float lse2 = lsum > 0.f ? mstar + log2f(lsum) : -INFINITY;
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

    __threadfence();
    __syncthreads();
    // The CTA that draws the last ticket of the (sequence, head) merges.
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(&tickets[unit], 1u);
        sh_last = ticket == (uint32_t)(S - 1);
    }
    __syncthreads();
    if (!sh_last) return;
    __threadfence();
    // The other CTAs' partial tiles (rows 0..g-1 of each split, contiguous)
    // come in through bulk copies into the drained ring, every split's copy in
    // flight at once; splits that do not fit are taken in further chunks.
    float *wts = reinterpret_cast<float *>(smem);  // [S][16] merge weights
    const uint32_t wts_bytes = (uint32_t)((S * kMaxGroup * 4 + 127) / 128 * 128);
    uint8_t *tiles = smem + wts_bytes;
    const uint32_t tile_bytes = (uint32_t)(g * D * 4);
    const int chunk = min(S, (int)((SM::kRingBytes - wts_bytes) / tile_bytes));
    const int nchunks = (S + chunk - 1) / chunk;
    const float *ul = part_lse + unit * S * kMaxGroup;
    const float *uo = part_o + unit * S * kMaxGroup * D;
    auto issue_chunk = [&](int ci) {  // warp 0
        const int s0 = ci * chunk, s1 = min(S, s0 + chunk);
        fence_proxy_async_global();  // generic-proxy partials -> async-proxy reads
        fence_proxy_async_smem();    // earlier generic use of the ring -> async writes
        if (lane == 0) mbar_arrive_expect_tx(&merge_bar, (uint32_t)(s1 - s0) * tile_bytes);
        __syncwarp();
        for (int sp = s0 + lane; sp < s1; sp += 32)
            bulk_load(tiles + (size_t)(sp - s0) * tile_bytes, uo + (size_t)sp * kMaxGroup * D,
                      tile_bytes, &merge_bar);
    };
    if (warp == 0) issue_chunk(0);
    for (int i = threadIdx.x; i < S * g; i += kThreads) {
        const int s = i / g, r = i % g;
        wts[s * kMaxGroup + r] = __ldcg(&ul[s * kMaxGroup + r]);
    }
    __syncthreads();
    for (int r = warp; r < g; r += kWarps) {
        float mstar = -INFINITY;
        for (int s = lane; s < S; s += 32) mstar = fmaxf(mstar, wts[s * kMaxGroup + r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
        float sum = 0.f;
        if (mstar != -INFINITY)
            for (int s = lane; s < S; s += 32) sum += exp2f(wts[s * kMaxGroup + r] - mstar);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        __syncwarp();
        for (int s = lane; s < S; s += 32)
            wts[s * kMaxGroup + r] = sum > 0.f ? exp2f(wts[s * kMaxGroup + r] - mstar) / sum : 0.f;
        if (lane == 0) sh_lse[r] = sum > 0.f ? mstar + log2f(sum) : -INFINITY;
    }
    __syncthreads();
    // Thread item = (row, float4 column); two accumulators (even / odd split)
    // keep two independent FMA chains per item.
    constexpr int C4 = D / 4;
    constexpr int kItems = (kMaxGroup * C4 + kThreads - 1) / kThreads;
    const int items = g * C4;
    float4 acc[kItems][2];
#pragma unroll
    for (int k = 0; k < kItems; ++k)
        acc[k][0] = acc[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
    bool merged = true;
    for (int ci = 0; ci < nchunks; ++ci) {
        if (!mbar_wait_bounded(&merge_bar, ci & 1)) {
            merged = false;
            break;
        }
        const int s0 = ci * chunk, s1 = min(S, s0 + chunk);
        const float4 *tf = reinterpret_cast<const float4 *>(tiles);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            const int item = threadIdx.x + k * kThreads;
            if (item < items) {
                const int r = item / C4;
#pragma unroll 4
                for (int sp = s0; sp < s1; ++sp) {
                    const float w = wts[sp * kMaxGroup + r];
                    const float4 v = tf[(size_t)(sp - s0) * items + item];
                    float4 &a = acc[k][sp & 1];
                    a.x += w * v.x;
                    a.y += w * v.y;
                    a.z += w * v.z;
                    a.w += w * v.w;
                }
            }
        }
        if (ci + 1 < nchunks) {
            __syncthreads();  // every thread is done with this chunk's tiles
            if (warp == 0) issue_chunk(ci + 1);
        }
    }
    if (!merged) {
        if (threadIdx.x == 0) set_error(err, RESA_DEVERR_TIMEOUT);
        mbar_wait_bounded(&merge_bar, 0);  // let copies in flight land before exit
        mbar_wait_bounded(&merge_bar, 1);
    } else {
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            const int item = threadIdx.x + k * kThreads;
            if (item < items) {
                const int r = item / C4, c4 = item % C4;
                const float4 a0 = acc[k][0], a1 = acc[k][1];
                const size_t orow = (size_t)b * hq + (size_t)h * g + r;
                reinterpret_cast<float4 *>(out + orow * D)[c4] =
                    make_float4(a0.x + a1.x, a0.y + a1.y, a0.z + a1.z, a0.w + a1.w);
                if (lse_out && c4 == 0) lse_out[orow] = sh_lse[r] * kLn2;
            }
        }
    }
    if (threadIdx.x == 0) tickets[unit] = 0;
}

// CTAs of one wave the device holds for this kernel (cached per device).
template <int D, int NT>
int wave_capacity(int smem) {
    static std::atomic<int> cap[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int c = cap[dev].load();
    if (c == 0) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sparse_decode_kernel<D, NT>,
                                                          kThreads, smem) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        c = per_sm * sms;
        cap[dev].store(c);
    }
    return c;
}

template <int D, int NT>
cudaError_t launch_dn(const Shape &s, const void *k, const void *v,
                      const int32_t *page_table, const int32_t *seq_len, const void *q,
                      const int32_t *block_idx, const int32_t *block_cnt, int max_topk, int splits,
                      float *part_o, float *part_lse, uint32_t *tickets, uint32_t *grid_bar,
                      float *out, float *lse, uint32_t *err, const DecodeAppend &app,
                      cudaStream_t st) {
    constexpr int smem = DecodeSmem<D>::kBytes;
    static std::atomic<int> done[64];
    cudaError_t e = ensure_smem(sparse_decode_kernel<D, NT>, smem, done);
    if (e != cudaSuccess) return e;
    const float scale_log2 = s.sm_scale * 1.4426950408889634f;
    dim3 grid(splits, s.hkv, s.batch);
    const long long ctas = (long long)splits * s.hkv * s.batch;
    // Split merge across the grid when it fits one wave (cooperative launch);
    // otherwise by the last CTA of each (sequence, head).
    // (kSpreadMaxCtas bounds the warp partials the caller's scratch holds.)
    const bool spread = grid_bar != nullptr && splits > 1 && ctas <= kSpreadMaxCtas &&
                        ctas <= wave_capacity<D, NT>(smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = spread ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, sparse_decode_kernel<D, NT>, (const uint8_t *)k,
                              (const uint8_t *)v, page_table, seq_len,
                              (const uint16_t *)q, block_idx, block_cnt, max_topk, s.hkv, s.g,
                              s.max_pages, s.num_pages, scale_log2, part_o, part_lse, tickets,
                              spread ? grid_bar : (uint32_t *)nullptr, out, lse, err, app, s.rows,
                              s.bs);
}

}  // namespace

cudaError_t launch_sparse_decode(const Shape &s, const void *k, const void *v,
                                 const int32_t *page_table, const int32_t *seq_len, const void *q,
                                 const int32_t *block_idx, const int32_t *block_cnt, int max_topk,
                                 int splits, float *part_o, float *part_lse, uint32_t *tickets,
                                 uint32_t *grid_bar, float *out, float *lse, uint32_t *err,
                                 cudaStream_t st, const DecodeAppend &app) {
#define RESA_DECODE_ARGS                                                                     \
    s, k, v, page_table, seq_len, q, block_idx, block_cnt, max_topk, splits, part_o,       \
        part_lse, tickets, grid_bar, out, lse, err, app, st
    if (s.d == 128)
        return s.g <= 8 ? launch_dn<128, 1>(RESA_DECODE_ARGS) : launch_dn<128, 2>(RESA_DECODE_ARGS);
    if (s.d == 64)
        return s.g <= 8 ? launch_dn<64, 1>(RESA_DECODE_ARGS) : launch_dn<64, 2>(RESA_DECODE_ARGS);
#undef RESA_DECODE_ARGS
    return cudaErrorInvalidValue;
}

}  // namespace resa
