// Dense rectification chunk attention on the 5th-generation tensor cores
// (ReSA summary §3.4.2; Algorithm 1, rectification check): the f chunk
// queries of every group head attend causally to the whole cache, after the
// chunk's fresh K/V were written back.
//
// Rows of one (sequence, kv head) are rho = r * g + j (chunk position r, group
// head j; position L - f + r).  Grid (row groups of 256, splits, batch * Hkv):
// a CTA owns 256 rows (two M = 128 MMA tiles) and one contiguous range of KV
// blocks, streamed as tiles of 64 keys (64 / b blocks of b tokens).
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0      TMA producer: when a tile's blocks sit on consecutive pages,
//               one 4-D tensor load per channel half of K and of V (64
//               channels x b tokens x 1 head x 64 / b pages, 8 KB, 128-byte
//               swizzled); otherwise one 2-D load (b x 64) per block and
//               half.  Both write the same shared-memory image;
//   warp 1      TMEM owner and MMA issuer (one thread): S = Q K^T into a
//               double-buffered TMEM tile (kind::f16, bf16 inputs), then
//               O += P V (kind::f16, fp16 inputs), commits on mbarriers;
//   warps 2-3   convert the V tile bf16 -> fp16 in place, scaled by a
//               power of two 2^-e chosen per tile from its largest |v| so
//               that every finite bf16 value lands in fp16's normal range
//               (e = 0, no scaling, when the largest |v| is in [2^-8, 2^16));
//               zero blocks that were not loaded;
//   warps 4-11  softmax, one thread per query row (TMEM lane): tcgen05.ld of
//               the S row, causal mask (skipped for interior tiles), base-2
//               online softmax with lazy O rescaling (only when the row
//               maximum grows by more than 8), P written as fp16 pairs into
//               tensor memory over the tile's S (tcgen05.st), where the
//               P.V MMA reads its A operand.  With E the
//               largest tile exponent seen so far, a tile's P is multiplied
//               by 2^(e - E) and O is rescaled whenever E grows, so the TMEM
//               accumulator holds 2^-E times the true sum; the epilogue
//               multiplies by 2^E.
// Three K/V stages are in flight (released per stage by the P.V commit).  P
// shares the double-buffered S columns, so writing it waits for nothing; O is
// rescaled only after the previous P.V has completed.
// P is fp16 (11-bit mantissa), so the P.V product keeps the weights' precision
// without a second MMA.  With several splits the grid is launched
// cooperatively; after a bounded grid barrier every CTA merges an equal share
// of all rows' partial (o, lse).  Waits are bounded.
#include "tc_common.cuh"

namespace resa {
namespace {

constexpr int kRows = kRectRowsPerCta;  // 256
constexpr int kKeys = 64;               // keys per KV tile
constexpr int kStages = 3;
constexpr int kNumConv = 2;             // converter warps
constexpr int kWarpSm0 = 4;             // first softmax warp
constexpr int kNumSm = 8;               // softmax warps
constexpr int kThreads = 32 * (kWarpSm0 + kNumSm);
constexpr int kSmThreads = 32 * kNumSm;
constexpr int kConvThreads = 32 * kNumConv;
constexpr float kRescaleSlack = 8.0f;   // log2 units of growth tolerated before rescaling O
constexpr int kNoExp = -1000;           // no V tile exponent seen yet

// Power-of-two exponent e of a V tile whose largest magnitude has the bf16
// bit pattern `mag` (sign cleared): the tile is stored as V * 2^-e in fp16.
// 0 when the largest |v| lies in [2^-8, 2^16) (bf16 values there are exact
// fp16 values, and smaller ones of the tile lose at most 2^-17 of the largest);
// otherwise the largest |v| * 2^-e falls in [2^14, 2^15).  Zero tiles and
// non-finite values keep e = 0.
__device__ __forceinline__ int v_tile_exponent(uint32_t mag) {
    if (mag == 0u || mag >= 0x7f80u) return 0;
    const int ex = (int)(mag >> 7) - 127;  // floor(log2|v|) for normal bf16
    if (ex >= -8 && ex <= 15) return 0;
    return min(113, max(-100, ex - 14));
}
// 2^k as a float for k in [-126, 127]; 0 below.
__device__ __forceinline__ float exp2i(int k) {
    return k < -126 ? 0.f : __int_as_float((127 + k) << 23);
}

template <int D>
struct TcLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kQTile = 128 * D * 2;     // one M tile of Q, [half][128 rows][128 B]
    static constexpr int kQHalf = 128 * 128;
    static constexpr int kKV = kKeys * D * 2;      // K or V tile, [half][64 keys][128 B]
    static constexpr int kKVHalf = kKeys * 128;
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = kQOff + 2 * kQTile;
    static constexpr int kBytes = kKVOff + kStages * 2 * kKV + 1024;
    // TMEM columns: O[mt] at mt*D, S[buf][mt] at 2*D + (2*buf + mt)*64; the
    // tile's P (fp16 pairs) overwrites the first 32 columns of its S.
    static constexpr uint32_t kTmemCols = 512;
};

__device__ __forceinline__ float ex2(float x) {  // hardware base-2 exponential
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
    const __half2 h = __floats2half2_rn(bf_lo(x), bf_hi(x));
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t x, float scale) {
    const __half2 h = __floats2half2_rn(bf_lo(x) * scale, bf_hi(x) * scale);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 1)
    rectify_tc_kernel(const __grid_constant__ CUtensorMap k0map,
                      const __grid_constant__ CUtensorMap k1map,
                      const __grid_constant__ CUtensorMap v0map,
                      const __grid_constant__ CUtensorMap v1map,
                      const __grid_constant__ CUtensorMap k0run,
                      const __grid_constant__ CUtensorMap k1run,
                      const __grid_constant__ CUtensorMap v0run,
                      const __grid_constant__ CUtensorMap v1run,
                      const int32_t *__restrict__ page_table, const int32_t *__restrict__ seq_len,
                      int f, const uint16_t *__restrict__ q_chunk, int hkv, int g, int max_pages,
                      int num_pages, float scale_log2, float *__restrict__ part_o,
                      float *__restrict__ part_lse, uint32_t *__restrict__ tickets,
                      float *__restrict__ out, float *__restrict__ lse_out, const RowMap rm,
                      int coop, uint32_t *err) {
    using LY = TcLayout<D>;
    constexpr int kBPT = kKeys / BS;  // blocks per 64-key tile
    static_assert(kKeys % BS == 0 && kBPT <= 4, "a tile holds whole blocks");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    __shared__ uint64_t q_ready, kv_full[kStages], v_ready[kStages], kv_empty[kStages], s_full[2],
        p_full, pv_done, conv_seen[kStages];
    __shared__ uint32_t tmem_base_s;
    __shared__ uint32_t stage_vmask[kStages];
    __shared__ int stage_vexp[kStages];            // V tile exponent of each stage
    __shared__ uint32_t conv_max[kStages][kNumConv];  // converter warps' largest |v| bits

    const int group = blockIdx.x, split = blockIdx.y, unit = blockIdx.z;
    const int G = gridDim.x, S = gridDim.y;
    const int b = unit / hkv, h = unit % hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hq = hkv * g;
    const int R = f * g;

    const int srow = cache_row(rm, b, threadIdx.x == 0 && group == 0 && split == 0 ? err : nullptr);
    const int L = row_seq_len(seq_len, srow);
    const bool seq_ok = L >= 1 && L <= max_pages * BS && f <= L;
    if (!seq_ok && threadIdx.x == 0 && group == 0 && split == 0)
        set_error(err, (L < 1 || L > max_pages * BS) ? RESA_DEVERR_SEQ_LEN : RESA_DEVERR_CHUNK);
    const int start = L - f;
    const int row0 = group * kRows;
    const int last_row = min(R, row0 + kRows) - 1;
    const int lim_max = (seq_ok && row0 < R) ? start + last_row / g + 1 : 0;
    const int nblk = (lim_max + BS - 1) / BS;
    int per = (nblk + S - 1) / S;
    per = (per + kBPT - 1) / kBPT * kBPT;
    const int blk0 = min(nblk, split * per), blk1 = min(nblk, blk0 + per);
    const int ntiles = (blk1 - blk0 + kBPT - 1) / kBPT;

    uint8_t *q_s = smem + LY::kQOff;
    uint8_t *kv_s = smem + LY::kKVOff;

    if (threadIdx.x == 0) {
        mbar_init(&q_ready, kSmThreads);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&v_ready[s], kConvThreads);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&conv_seen[s], kNumConv);
        }
        for (int s = 0; s < 2; ++s) mbar_init(&s_full[s], 1);
        mbar_init(&p_full, kSmThreads);
        mbar_init(&pv_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(&tmem_base_s, LY::kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base_s;

    if (warp == 0) {  // ------------------------------------------------ TMA producer
        // Page ids arrive 32 blocks (8 tiles) at a time, one id a lane, with
        // the next window's load already in flight; they are checked when used.
        constexpr int kWin = 32 / kBPT;  // tiles per window
        auto load_win = [&](int w) -> int {
            const int blk = blk0 + w * 32 + lane;
            return blk < blk1 ? page_table[(size_t)srow * max_pages + blk] : -1;
        };
        int win_cur = ntiles > 0 ? load_win(0) : -1;
        int win_next = ntiles > kWin ? load_win(1) : -1;
        bool ok = true;
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i % kStages;
            if (i >= kStages) ok = mbar_wait_bounded(&kv_empty[s], ((i / kStages) - 1) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (i > 0 && i % kWin == 0) {
                win_cur = win_next;
                win_next = i + kWin < ntiles ? load_win(i / kWin + 1) : -1;
            }
            const int blk = blk0 + i * kBPT + lane;
            int page = __shfl_sync(0xffffffffu, win_cur, ((i % kWin) * kBPT + lane) & 31);
            if (lane < kBPT && blk < blk1) {
                if (page < 0 || page >= num_pages) {
                    set_error(err, RESA_DEVERR_PAGE);
                    page = -1;
                }
            } else {
                page = -1;
            }
            const uint32_t vmask = __ballot_sync(0xffffffffu, page >= 0);
            const uint32_t bytes = (uint32_t)__popc(vmask) * 2u * LY::kHalves * BS * 128u;
            // four valid blocks on consecutive pages: one 4-page box per half
            const int page0 = __shfl_sync(0xffffffffu, page, 0);
            const bool run = __all_sync(0xffffffffu, lane >= kBPT ||
                                                          (page >= 0 && page == page0 + lane));
            if (lane == 0) {
                stage_vmask[s] = vmask;
                if (bytes == 0)
                    mbar_arrive(&kv_full[s]);
                else
                    mbar_arrive_expect_tx(&kv_full[s], bytes);
            }
            __syncwarp();
            if (run) {
                if (lane == 0) {
                    uint8_t *kt = kv_s + (size_t)s * 2 * LY::kKV;
                    uint8_t *vt = kt + LY::kKV;
                    tc::tma_load_4d(kt, &k0run, 0, 0, h, page0, &kv_full[s]);
                    tc::tma_load_4d(vt, &v0run, 0, 0, h, page0, &kv_full[s]);
                    if (LY::kHalves == 2) {
                        tc::tma_load_4d(kt + LY::kKVHalf, &k1run, 0, 0, h, page0, &kv_full[s]);
                        tc::tma_load_4d(vt + LY::kKVHalf, &v1run, 0, 0, h, page0, &kv_full[s]);
                    }
                }
            } else if (page >= 0) {
                const int y = (page * hkv + h) * BS;
                uint8_t *kt = kv_s + (size_t)s * 2 * LY::kKV;
                uint8_t *vt = kt + LY::kKV;
                const int off = lane * BS * 128;  // this block's BS rows in each half
                tc::tma_load_2d(kt + off, &k0map, 0, y, &kv_full[s]);
                tc::tma_load_2d(vt + off, &v0map, 0, y, &kv_full[s]);
                if (LY::kHalves == 2) {
                    tc::tma_load_2d(kt + LY::kKVHalf + off, &k1map, 0, y, &kv_full[s]);
                    tc::tma_load_2d(vt + LY::kKVHalf + off, &v1map, 0, y, &kv_full[s]);
                }
            }
        }
        if (!ok && lane == 0) set_error(err, RESA_DEVERR_TIMEOUT);
    } else if (warp == 1) {  // ----------------------------------------- MMA issuer
        constexpr uint32_t idesc_qk = tc::idesc_f16(1, 1, 0, 0, 128, kKeys);
        constexpr uint32_t idesc_pv = tc::idesc_f16(0, 0, 0, 1, 128, D);
        bool ok = mbar_wait_bounded(&q_ready, 0);
        auto issue_qk = [&](int i) {
            const int s = i % kStages, buf = i & 1;
            const uint32_t kt = smem_u32(kv_s + (size_t)s * 2 * LY::kKV);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const uint32_t qt = smem_u32(q_s + mt * LY::kQTile);
                const uint32_t d_tmem = tmem + 2 * D + (2 * buf + mt) * kKeys;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int half = ks / 4, kin = ks % 4;
                    const uint64_t a = tc::smem_desc(qt + half * LY::kQHalf + kin * 32, 16, 1024);
                    const uint64_t bd = tc::smem_desc(kt + half * LY::kKVHalf + kin * 32, 16, 1024);
                    tc::mma_f16_ss(d_tmem, a, bd, idesc_qk, ks > 0 ? 1u : 0u);
                }
            }
            tc::commit(&s_full[buf]);
        };
        if (lane == 0 && ok && ntiles > 0) {
            ok = mbar_wait_bounded(&kv_full[0], 0);
            tc::fence_after_sync();
            if (ok) issue_qk(0);
            for (int i = 0; i < ntiles && ok; ++i) {
                const int s = i % kStages;
                if (i + 1 < ntiles) {
                    ok = mbar_wait_bounded(&kv_full[(i + 1) % kStages], ((i + 1) / kStages) & 1);
                    tc::fence_after_sync();
                    if (!ok) break;
                    issue_qk(i + 1);  // S[(i+1)&1] was released by the softmax of tile i-1
                }
                ok = mbar_wait_bounded(&p_full, i & 1) &&
                     mbar_wait_bounded(&v_ready[s], (i / kStages) & 1);
                tc::fence_after_sync();
                if (!ok) break;
                const uint32_t vt = smem_u32(kv_s + (size_t)s * 2 * LY::kKV + LY::kKV);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    // P of this tile sits in tensor memory over its S
                    const uint32_t pt = tmem + 2 * D + (2 * (i & 1) + mt) * kKeys;
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk) {
                        const uint64_t bd = tc::smem_desc(vt + kk * 16 * 128, LY::kKVHalf, 1024);
                        tc::mma_f16_ts(tmem + mt * D, pt + kk * 8, bd, idesc_pv,
                                       (i > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc::commit(&pv_done);
                tc::commit(&kv_empty[s]);
            }
            if (!ok) set_error(err, RESA_DEVERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < kWarpSm0) {  // ---------------------------------- V converters
        const int ct = threadIdx.x - 64;
        const int cw = warp - 2;
        bool ok = true;
        for (int i = 0; i < ntiles && ok; ++i) {
            const int s = i % kStages;
            ok = mbar_wait_bounded(&kv_full[s], (i / kStages) & 1);
            if (!ok) break;
            const uint32_t vmask = stage_vmask[s];
            uint4 *vt = reinterpret_cast<uint4 *>(kv_s + (size_t)s * 2 * LY::kKV + LY::kKV);
            constexpr int kChunks = LY::kKV / 16;           // 16-byte chunks of the tile
            constexpr int kChunksPerBlock = BS * 128 / 16;  // per half
            constexpr int kPer = kChunks / kConvThreads;
            static_assert(kChunks % kConvThreads == 0, "equal converter shares");
            // the thread's chunks into registers (blocks not loaded become
            // zero) and the largest magnitude among them, two halves a word
            uint4 x[kPer];
            uint32_t m2 = 0u;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int c = ct + k * kConvThreads;
                const int blk_in_tile = (c % (LY::kKVHalf / 16)) / kChunksPerBlock;
                x[k] = ((vmask >> blk_in_tile) & 1u) ? vt[c] : make_uint4(0u, 0u, 0u, 0u);
                m2 = __vmaxu2(m2, x[k].x & 0x7fff7fffu);
                m2 = __vmaxu2(m2, x[k].y & 0x7fff7fffu);
                m2 = __vmaxu2(m2, x[k].z & 0x7fff7fffu);
                m2 = __vmaxu2(m2, x[k].w & 0x7fff7fffu);
            }
            uint32_t mag = max(m2 & 0xffffu, m2 >> 16);
            mag = __reduce_max_sync(0xffffffffu, mag);
            if ((threadIdx.x & 31) == 0) {
                conv_max[s][cw] = mag;
                mbar_arrive(&conv_seen[s]);
            }
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(&conv_seen[s], (i / kStages) & 1));
            if (!ok) break;
            mag = max(conv_max[s][0], conv_max[s][1]);
            const int e = v_tile_exponent(mag);
            if (e == 0) {
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    uint4 y = x[k];
                    y.x = bf16x2_to_f16x2(y.x);
                    y.y = bf16x2_to_f16x2(y.y);
                    y.z = bf16x2_to_f16x2(y.z);
                    y.w = bf16x2_to_f16x2(y.w);
                    vt[ct + k * kConvThreads] = y;
                }
            } else {
                const float sc = exp2i(-e);
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    uint4 y = x[k];
                    y.x = bf16x2_to_f16x2_scaled(y.x, sc);
                    y.y = bf16x2_to_f16x2_scaled(y.y, sc);
                    y.z = bf16x2_to_f16x2_scaled(y.z, sc);
                    y.w = bf16x2_to_f16x2_scaled(y.w, sc);
                    vt[ct + k * kConvThreads] = y;
                }
            }
            if (ct == 0) stage_vexp[s] = e;
            fence_proxy_async_smem();
            mbar_arrive(&v_ready[s]);
        }
        if (!ok && ct == 0) set_error(err, RESA_DEVERR_TIMEOUT);
    } else {  // -------------------------------------------------------- softmax
        const int st = threadIdx.x - 32 * kWarpSm0;  // 0..255
        const int mt = st >> 7, r = st & 127;
        const int rho = row0 + mt * 128 + r;
        const bool row_ok = seq_ok && rho < R;
        const int lim = row_ok ? start + rho / g + 1 : 0;
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        // Q row into the K-major swizzled tile (zeros for padding rows).
        {
            const uint4 *src = row_ok ? reinterpret_cast<const uint4 *>(
                                            q_chunk + (((size_t)b * f + rho / g) * hq +
                                                       (size_t)h * g + rho % g) * D)
                                      : nullptr;
            uint8_t *qt = q_s + mt * LY::kQTile;
#pragma unroll
            for (int hf = 0; hf < LY::kHalves; ++hf)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = src ? src[hf * 8 + c] : make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(qt + hf * LY::kQHalf + swz128(r, c)) = v;
                }
            fence_proxy_async_smem();
            mbar_arrive(&q_ready);
        }
        float m_use = -INFINITY, l = 0.f;
        int e_run = kNoExp;  // largest V tile exponent so far (E)
        bool ok = true;
        // Keys every valid row of this CTA may see: tiles entirely below this
        // limit (and fully loaded) need no mask.
        const int lim_cta = seq_ok ? start + row0 / g + 1 : 0;
        const int tend = blk1 * BS;
        for (int i = 0; i < ntiles; ++i) {
            const int buf = i & 1;
            ok = mbar_wait_bounded(&s_full[buf], (i / 2) & 1) &&
                 mbar_wait_bounded(&v_ready[i % kStages], (i / kStages) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc::fence_after_sync();
            // the tile's V exponent (the same for every thread of the CTA)
            const int e_t = stage_vexp[i % kStages];
            const bool e_grow = e_run != kNoExp && e_t > e_run;
            const float alpha_e = e_grow ? exp2i(e_run - e_t) : 1.f;
            e_run = e_run == kNoExp ? e_t : max(e_run, e_t);
            const float pfac = exp2i(e_t - e_run);  // 1 unless this tile is smaller
            uint32_t sv[2][32];
            const uint32_t scol = tmem + lane_base + 2 * D + (2 * buf + mt) * kKeys;
            tc::tmem_ld32(scol, sv[0]);
            tc::tmem_ld32(scol + 32, sv[1]);
            tc::tmem_wait_ld();
            const int t0 = (blk0 + i * kBPT) * BS;
            const uint32_t vmask = stage_vmask[i % kStages];
            const bool full_tile = vmask == (1u << kBPT) - 1u && t0 + kKeys <= tend && t0 + kKeys <= lim_cta;
            float x[64];  // raw logits; -inf where masked
            float mraw = -INFINITY;
            if (full_tile) {
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    x[j] = __uint_as_float(sv[j >> 5][j & 31]);
                    mraw = fmaxf(mraw, x[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const int t = t0 + j;
                    const bool valid = t < lim && t < tend && ((vmask >> (j / BS)) & 1u);
                    x[j] = valid ? __uint_as_float(sv[j >> 5][j & 31]) : -INFINITY;
                    mraw = fmaxf(mraw, x[j]);
                }
            }
            const float mtile = mraw * scale_log2;  // scale > 0 keeps the maximum
            const bool need = mtile > m_use + kRescaleSlack;
            const bool rescale = __any_sync(0xffffffffu, need);
            float alpha = 1.f;
            if (rescale) {
                const float m_new = fmaxf(m_use, mtile);
                alpha = (m_use == -INFINITY) ? 0.f : ex2(m_use - m_new);
                m_use = m_new;
                l *= alpha;
            }
            // Weights in registers (fp16 pairs) before touching the shared P tile.
            uint32_t pw[32];
            float psum = 0.f;
            if (m_use == -INFINITY) {
#pragma unroll
                for (int e = 0; e < 32; ++e) pw[e] = 0u;
            } else if (pfac != 1.f) {
                const float nm = -m_use;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float p0 = ex2(fmaf(x[2 * e], scale_log2, nm));
                    const float p1 = ex2(fmaf(x[2 * e + 1], scale_log2, nm));
                    psum += p0 + p1;
                    pw[e] = f16x2(p0 * pfac, p1 * pfac);
                }
            } else {
                const float nm = -m_use;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float p0 = ex2(fmaf(x[2 * e], scale_log2, nm));
                    const float p1 = ex2(fmaf(x[2 * e + 1], scale_log2, nm));
                    psum += p0 + p1;
                    pw[e] = f16x2(p0, p1);
                }
            }
            l += psum;
            // P goes over this tile's S (already read; the P.V that last read
            // this slot, of tile i-2, came before this tile's S in the MMA
            // order), asynchronously while O waits for the P.V of tile i-1.
            const uint32_t pcol = tmem + lane_base + 2 * D + (2 * buf + mt) * kKeys;
            tc::tmem_st32(pcol, pw);
            if (i > 0) {
                ok = mbar_wait_bounded(&pv_done, (i - 1) & 1);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc::fence_after_sync();
                if (rescale || e_grow) {
                    const float alpha_o = (rescale ? alpha : 1.f) * alpha_e;
#pragma unroll
                    for (int c4 = 0; c4 < D / 32; ++c4) {
                        uint32_t ov[32];
                        const uint32_t ocol = tmem + lane_base + mt * D + c4 * 32;
                        tc::tmem_ld32(ocol, ov);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha_o);
                        tc::tmem_st32(ocol, ov);
                    }
                }
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            mbar_arrive(&p_full);
        }
        if (!ok && lane == 0) set_error(err, RESA_DEVERR_TIMEOUT);
        // Final O row (all P.V done), normalised; partial or final output.
        float lse2 = -INFINITY;
        float inv = 0.f;
        bool have = false;
        if (ok && ntiles > 0) {
            ok = mbar_wait_bounded(&pv_done, (ntiles - 1) & 1);
            ok = __all_sync(0xffffffffu, ok);
            tc::fence_after_sync();
            have = ok;
        }
        if (l > 0.f) {
            lse2 = m_use + log2f(l);
            // O holds 2^-E times the weighted sum: undo the V scaling here
            inv = (1.f / l) * exp2i(e_run == kNoExp ? 0 : e_run);
        }
        const float kLn2 = 0.6931471805599453f;
        const int r_pos = rho / g, jh = rho % g;
        const size_t orow = ((size_t)b * f + r_pos) * hq + (size_t)h * g + jh;
        const size_t slot = ((size_t)unit * G + group) * S + split;
        float *dst = S == 1 ? out + orow * D : part_o + (slot * kRows + mt * 128 + r) * D;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t ov[32];
            if (have) {
                tc::tmem_ld32(tmem + lane_base + mt * D + c4 * 32, ov);
                tc::tmem_wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) ov[j] = 0u;
            }
            if (rho < R) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 v = make_float4(__uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv,
                                           __uint_as_float(ov[j + 2]) * inv,
                                           __uint_as_float(ov[j + 3]) * inv);
                    if (!have || l <= 0.f) v = make_float4(0.f, 0.f, 0.f, 0.f);
                    *reinterpret_cast<float4 *>(dst + c4 * 32 + j) = v;
                }
            }
        }
        if (rho < R) {
            if (S == 1) {
                if (lse_out) lse_out[orow] = have ? lse2 * kLn2 : -INFINITY;
            } else {
                part_lse[slot * kRows + mt * 128 + r] = have ? lse2 : -INFINITY;
            }
        }
    }

    // Release TMEM once every TMEM access of the CTA is done.
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, LY::kTmemCols);
    if (S == 1) return;

    // Every split's partials are written.  Within one wave (cooperative
    // launch) a bounded grid barrier lets every CTA merge an equal share of
    // all rows; tickets[0..1] hold the barrier's 64-bit (generation,
    // arrivals) word.  Beyond one wave the last split of each (unit, row
    // group) to arrive merges that group, counted by a ticket it resets.
    __threadfence();
    __syncthreads();
    __shared__ uint32_t sh_ok;
    int i0, i1, cap_rows;
    if (coop) {
        const uint32_t nctas = gridDim.x * gridDim.y * gridDim.z;
        if (threadIdx.x == 0) sh_ok = grid_barrier_bounded(reinterpret_cast<unsigned long long *>(tickets), nctas) ? 1u : 0u;
        __syncthreads();
        if (!sh_ok) {
            if (threadIdx.x == 0) set_error(err, RESA_DEVERR_TIMEOUT);
            return;
        }
        __threadfence();
        const int total = (int)gridDim.z * R;
        const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
        cap_rows = (total + (int)nctas - 1) / (int)nctas;
        i0 = cta * cap_rows;
        i1 = min(total, i0 + cap_rows);
    } else {
        uint32_t *ticket = tickets + kRectTicketBase + (size_t)unit * kMaxRowTiles + group;
        if (threadIdx.x == 0) sh_ok = atomicAdd(ticket, 1u) == (uint32_t)(S - 1) ? 1u : 0u;
        __syncthreads();
        if (!sh_ok) return;
        __threadfence();
        if (threadIdx.x == 0) *ticket = 0u;  // every split of the group has arrived
        cap_rows = kRows;
        i0 = unit * R + min(R, row0);
        i1 = unit * R + min(R, row0 + kRows);
    }
    float *wts = reinterpret_cast<float *>(smem);  // [cap_rows][S] merge weights
    float *lse_s = wts + cap_rows * S;             // [cap_rows]
    auto slot_row = [&](int item, int sp) -> size_t {
        const int u = item / R, rho = item % R;
        return (((size_t)u * G + rho / kRows) * S + sp) * kRows + rho % kRows;
    };
    for (int e = threadIdx.x; e < (i1 - i0) * S; e += kThreads) {
        const int it = e / S, sp = e % S;
        wts[it * S + sp] = __ldcg(&part_lse[slot_row(i0 + it, sp)]);
    }
    __syncthreads();
    for (int it = warp; it < i1 - i0; it += kThreads / 32) {
        float mstar = -INFINITY;
        for (int sp = lane; sp < S; sp += 32) mstar = fmaxf(mstar, wts[it * S + sp]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
        float sum = 0.f;
        if (mstar != -INFINITY)
            for (int sp = lane; sp < S; sp += 32) sum += exp2f(wts[it * S + sp] - mstar);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        __syncwarp();
        for (int sp = lane; sp < S; sp += 32)
            wts[it * S + sp] = sum > 0.f ? exp2f(wts[it * S + sp] - mstar) / sum : 0.f;
        if (lane == 0) lse_s[it] = sum > 0.f ? mstar + log2f(sum) : -INFINITY;
    }
    __syncthreads();
    constexpr int C4 = D / 4;
    for (int e = threadIdx.x; e < (i1 - i0) * C4; e += kThreads) {
        const int it = e / C4, c4 = e % C4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < S; ++sp) {
            const float w = wts[it * S + sp];
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                                        part_o + slot_row(i0 + it, sp) * D) + c4);
            acc.x += w * v.x;
            acc.y += w * v.y;
            acc.z += w * v.z;
            acc.w += w * v.w;
        }
        const int item = i0 + it;
        const int u = item / R, rho = item % R;
        const int ub = u / hkv, uh = u % hkv;
        const size_t orow = ((size_t)ub * f + rho / g) * hq + (size_t)uh * g + rho % g;
        reinterpret_cast<float4 *>(out + orow * D)[c4] = acc;
        if (lse_out && c4 == 0) lse_out[orow] = lse_s[it] * 0.6931471805599453f;
    }
}

template <int D, int BS>
cudaError_t launch_tc(const Shape &s, const CUtensorMap *maps, const int32_t *page_table,
                      const int32_t *seq_len, int f, const void *q_chunk, int groups, int splits,
                      float *part_o, float *part_lse, uint32_t *tickets, float *out, float *lse,
                      uint32_t *err, cudaStream_t st) {
    constexpr int smem = TcLayout<D>::kBytes;
    static std::atomic<int> done[64];
    cudaError_t e = ensure_smem(rectify_tc_kernel<D, BS>, smem, done);
    if (e != cudaSuccess) return e;
    const float scale_log2 = s.sm_scale * 1.4426950408889634f;
    dim3 grid(groups, splits, s.batch * s.hkv);
    // With several splits in one wave the CTAs meet at a grid barrier before
    // merging, so they must be co-resident: cooperative launch (one CTA per
    // SM).  A larger grid merges by per-group tickets instead.
    const int coop = splits > 1 && (long long)groups * splits * s.batch * s.hkv <= kNumSms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = coop ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, rectify_tc_kernel<D, BS>, maps[0], maps[1], maps[2], maps[3],
                              maps[4], maps[5], maps[6], maps[7],
                              page_table, seq_len, f, (const uint16_t *)q_chunk, s.hkv, s.g,
                              s.max_pages, s.num_pages, scale_log2, part_o, part_lse, tickets, out,
                              lse, s.rows, coop, err);
}

}  // namespace

cudaError_t launch_rectify_attention(const Shape &s, const CUtensorMap *maps,
                                     const int32_t *page_table, const int32_t *seq_len, int f,
                                     const void *q_chunk, int groups, int splits, float *part_o,
                                     float *part_lse, uint32_t *tickets, float *out, float *lse,
                                     uint32_t *err, cudaStream_t st) {
    if (groups > kMaxRowTiles) return cudaErrorInvalidValue;
#define RESA_RECT_CASE(D, BS)                                                                 \
    if (s.d == D && s.bs == BS)                                                               \
        return launch_tc<D, BS>(s, maps, page_table, seq_len, f, q_chunk, groups, splits, part_o, \
                                part_lse, tickets, out, lse, err, st);
    RESA_RECT_CASE(128, 16)
    RESA_RECT_CASE(128, 32)
    RESA_RECT_CASE(128, 64)
    RESA_RECT_CASE(64, 16)
    RESA_RECT_CASE(64, 32)
    RESA_RECT_CASE(64, 64)
#undef RESA_RECT_CASE
    return cudaErrorInvalidValue;
}

}  // namespace resa
