// Query-aware block selection (ReSA summary §3.4.1): group query pooling, the
// Quest upper-bound score of Eq. 4 for every complete block, and top-n
// selection (Eq. 5 count from the caller, ties to the lower block index) with
// the local block always appended.
//
// score_kernel streams the block key cache.  Grid (X, batch); CTA x owns a
// contiguous range of complete blocks of one sequence.  Its producer warp
// reads the page ids and issues cp.async.bulk copies of whole descriptor
// pages (all kv heads, 2*d bf16 each) into a kScoreStages-deep shared-memory
// ring, one copy per run of physically consecutive pages; four consumer warps
// score two pages per stage each (lane = d/32 channels, one butterfly per
// (page, head)).  Every score also bumps a 65536-bin histogram of the top 16
// bits of its order-preserving key, per (sequence, kv head), and the range of
// touched bins, so the selection never scans the full key range for its first
// digit.  In decode steps an extra warp of the first CTA of each sequence
// appends the decode token (K/V write, descriptor fold) in the same launch.
//
// select_kernel is one 1024-thread CTA per (sequence, kv head): it finds the
// histogram bin holding the k-th largest key (scanning only the touched bins,
// clearing them for the next call), gathers that bin's keys, radix-selects
// their low 16 bits, and compacts the blocks with key > T plus the
// lowest-index blocks with key == T in ascending order (warp ballots).
#include "resa_common.cuh"

namespace resa {
namespace {

constexpr int kScoreConsumers = 4;
constexpr int kScoreGroup = 2 * kScoreConsumers;  // pages per stage: two per consumer warp
constexpr int kScoreStages = 4;
constexpr int kScoreThreads = 32 * (1 + kScoreConsumers + 1);  // producer, consumers, append
constexpr int kHistBins = 65536;

__device__ __forceinline__ uint32_t order_key(float s) {
    s += 0.0f;  // -0 -> +0: equal scores get equal keys
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Bf16x8 {
    uint16_t v[8];
};
__device__ __forceinline__ Bf16x8 unpack8(uint4 x) {
    Bf16x8 r;
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        r.v[2 * i] = (uint16_t)(w[i] & 0xffffu);
        r.v[2 * i + 1] = (uint16_t)(w[i] >> 16);
    }
    return r;
}
__device__ __forceinline__ uint4 pack8(const Bf16x8 &r) {
    uint4 x;
    x.x = (uint32_t)r.v[0] | ((uint32_t)r.v[1] << 16);
    x.y = (uint32_t)r.v[2] | ((uint32_t)r.v[3] << 16);
    x.z = (uint32_t)r.v[4] | ((uint32_t)r.v[5] << 16);
    x.w = (uint32_t)r.v[6] | ((uint32_t)r.v[7] << 16);
    return x;
}

// grid (X, batch), block kScoreThreads, dynamic smem kScoreStages * kScoreGroup * page bytes.
template <int D, int HKV>
__global__ void __launch_bounds__(kScoreThreads)
    score_kernel(uint16_t *__restrict__ desc, const int32_t *__restrict__ page_table,
                 const int32_t *__restrict__ seq_len, const uint16_t *__restrict__ q,
                 float *__restrict__ scores, uint32_t *__restrict__ hist,
                 uint32_t *__restrict__ hist_range, int g, int max_pages, int num_pages,
                 uint4 *__restrict__ K, uint4 *__restrict__ V, const uint4 *__restrict__ k_new,
                 const uint4 *__restrict__ v_new, uint32_t *err) {
    constexpr int PAGE_ELEMS = HKV * 2 * D;  // bf16 per descriptor page
    constexpr int PAGE_BYTES = PAGE_ELEMS * 2;
    constexpr int N = D / 32;                // channels per lane
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ float qbar_s[HKV][D];
    __shared__ uint64_t full[kScoreStages], empty[kScoreStages];
    __shared__ uint32_t stage_mask[kScoreStages];
    __shared__ int stage_np[kScoreStages];

    pdl_launch_next();
    const int b = blockIdx.y, x = blockIdx.x, X = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hq = HKV * g;
    const int L = seq_len[b];
    const bool seq_ok = L >= 1 && L <= max_pages * kBlock;
    const int M = seq_ok ? (L - 1) / kBlock : 0;
    const int per = ((M + X - 1) / X + kScoreGroup - 1) / kScoreGroup * kScoreGroup;
    const int p_begin = min(M, x * per), p_end = min(M, p_begin + per);
    const int n_groups = (p_end - p_begin + kScoreGroup - 1) / kScoreGroup;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kScoreStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kScoreConsumers);
        }
        fence_mbar_init();
    }
    if (warp >= 1 && warp <= kScoreConsumers) {
        // Group pooling: mean of the g query heads, fp32, head order, then / g.
        for (int e = threadIdx.x - 32; e < HKV * D; e += 32 * kScoreConsumers) {
            const int h = e / D, j = e % D;
            const uint16_t *col = q + ((size_t)b * hq + (size_t)h * g) * D + j;
            uint16_t v[kMaxGroup];
#pragma unroll
            for (int r = 0; r < kMaxGroup; ++r) v[r] = r < g ? col[(size_t)r * D] : (uint16_t)0;
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < kMaxGroup; ++r)
                if (r < g) s += bf16_bits_to_f32(v[r]);
            qbar_s[h][j] = s / (float)g;
        }
    }
    __syncthreads();

    if (warp == 0) {  // ------------------------------------------------ producer
        pdl_wait();
        if (!seq_ok && x == 0 && lane == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        for (int i = 0; i < n_groups; ++i) {
            const int s = i % kScoreStages;
            if (i >= kScoreStages && !mbar_wait_bounded(&empty[s], ((i / kScoreStages) - 1) & 1)) {
                if (lane == 0) set_error(err, RESA_DEVERR_TIMEOUT);
                break;
            }
            const int p0 = p_begin + i * kScoreGroup;
            const int npg = min(kScoreGroup, p_end - p0);
            int pg = -1;
            if (lane < npg) {
                pg = page_table[(size_t)b * max_pages + p0 + lane];
                if (pg < 0 || pg >= num_pages) {
                    set_error(err, RESA_DEVERR_PAGE);
                    pg = -1;
                }
            }
            const uint32_t all = (1u << npg) - 1u;  // npg <= kScoreGroup < 32
            const uint32_t vmask = __ballot_sync(0xffffffffu, lane < npg && pg >= 0);
            const int first = __shfl_sync(0xffffffffu, pg, 0);
            const bool contiguous =
                vmask == all && __ballot_sync(0xffffffffu, lane < npg && pg == first + lane) == all;
            const uint32_t bytes = (uint32_t)__popc(vmask) * PAGE_BYTES;
            uint8_t *dst = ring + (size_t)s * kScoreGroup * PAGE_BYTES;
            if (lane == 0) {
                stage_mask[s] = vmask;
                stage_np[s] = npg;
                if (bytes == 0)
                    mbar_arrive(&full[s]);
                else
                    mbar_arrive_expect_tx(&full[s], bytes);
            }
            __syncwarp();
            if (bytes > 0) {
                if (contiguous) {
                    if (lane == 0) bulk_load(dst, desc + (size_t)first * PAGE_ELEMS, bytes, &full[s]);
                } else if (lane < npg && pg >= 0) {
                    bulk_load(dst + (size_t)lane * PAGE_BYTES, desc + (size_t)pg * PAGE_ELEMS,
                              PAGE_BYTES, &full[s]);
                }
            }
        }
    } else if (warp <= kScoreConsumers) {  // ------------------------- consumers
        pdl_wait();
        const int c = warp - 1;
        float qv[HKV][N];
#pragma unroll
        for (int h = 0; h < HKV; ++h)
#pragma unroll
            for (int n = 0; n < N; ++n) qv[h][n] = qbar_s[h][lane * N + n];
        // lane t < 2*HKV owns output (page c*2 + t / HKV, head t % HKV)
        const int my_pp = lane / HKV, my_h = lane % HKV;
        const bool owner = lane < 2 * HKV;
        uint32_t dmin = 0xffffffffu, dmax = 0;
        for (int i = 0; i < n_groups; ++i) {
            const int s = i % kScoreStages;
            if (!mbar_wait_bounded(&full[s], (i / kScoreStages) & 1)) {
                if (lane == 0) set_error(err, RESA_DEVERR_TIMEOUT);
                break;
            }
            const uint32_t vmask = stage_mask[s];
            const int npg = stage_np[s];
            const uint8_t *st = ring + (size_t)s * kScoreGroup * PAGE_BYTES;
            float mine = 0.f;
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
                const int j = c * 2 + pp;
                const bool present = j < npg && ((vmask >> j) & 1u);
#pragma unroll
                for (int h = 0; h < HKV; ++h) {
                    float sum = 0.f;
                    if (present) {
                        const uint16_t *row = reinterpret_cast<const uint16_t *>(
                            st + (size_t)j * PAGE_BYTES + (size_t)h * 2 * D * 2);
                        float mn[N], mx[N];
                        if constexpr (N == 4) {
                            const uint2 a = *reinterpret_cast<const uint2 *>(row + lane * 4);
                            const uint2 z = *reinterpret_cast<const uint2 *>(row + D + lane * 4);
                            mn[0] = bf_lo(a.x);
                            mn[1] = bf_hi(a.x);
                            mn[2] = bf_lo(a.y);
                            mn[3] = bf_hi(a.y);
                            mx[0] = bf_lo(z.x);
                            mx[1] = bf_hi(z.x);
                            mx[2] = bf_lo(z.y);
                            mx[3] = bf_hi(z.y);
                        } else {
                            const uint32_t a = *reinterpret_cast<const uint32_t *>(row + lane * 2);
                            const uint32_t z = *reinterpret_cast<const uint32_t *>(row + D + lane * 2);
                            mn[0] = bf_lo(a);
                            mn[1] = bf_hi(a);
                            mx[0] = bf_lo(z);
                            mx[1] = bf_hi(z);
                        }
#pragma unroll
                        for (int n = 0; n < N; ++n) sum += fmaxf(qv[h][n] * mx[n], qv[h][n] * mn[n]);
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                    if (pp == my_pp && h == my_h) mine = sum;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            const int j = c * 2 + my_pp;
            if (owner && j < npg && ((vmask >> j) & 1u)) {
                const size_t unit = (size_t)b * HKV + my_h;
                scores[unit * max_pages + p_begin + i * kScoreGroup + j] = mine;
                const uint32_t digit = order_key(mine) >> 16;
                atomicAdd(&hist[unit * kHistBins + digit], 1u);
                dmin = min(dmin, digit);
                dmax = max(dmax, digit);
            }
        }
        // touched-bin range per (sequence, head): lanes h and h + HKV share head h
        const uint32_t omin = __shfl_down_sync(0xffffffffu, dmin, HKV);
        const uint32_t omax = __shfl_down_sync(0xffffffffu, dmax, HKV);
        if (lane < HKV) {
            dmin = min(dmin, omin);
            dmax = max(dmax, omax);
            if (dmin <= dmax) {
                const size_t unit = (size_t)b * HKV + lane;
                atomicMax(&hist_range[2 * unit], (uint32_t)kHistBins - dmin);  // 0 = untouched
                atomicMax(&hist_range[2 * unit + 1], dmax + 1u);
            }
        }
    } else if (K != nullptr && x == 0) {  // ------------------------ decode-token append
        pdl_wait();
        if (!seq_ok) return;
        const int pos = L - 1;
        const int page = page_table[(size_t)b * max_pages + pos / kBlock];
        if (page < 0 || page >= num_pages) {
            if (lane == 0) set_error(err, RESA_DEVERR_PAGE);
            return;
        }
        const int slot = pos % kBlock;
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        uint4 *dsc = reinterpret_cast<uint4 *>(desc);
        for (int e = lane; e < HKV * CPR; e += 32) {
            const int h = e / CPR, cc = e % CPR;
            const uint4 kx = k_new[((size_t)b * HKV + h) * CPR + cc];
            const uint4 vx = v_new[((size_t)b * HKV + h) * CPR + cc];
            const size_t o = (((size_t)page * HKV + h) * kBlock + slot) * CPR + cc;
            K[o] = kx;
            V[o] = vx;
            uint4 *pmn = &dsc[(((size_t)page * HKV + h) * 2) * CPR + cc];
            uint4 *pmx = pmn + CPR;
            if (slot == 0) {
                *pmn = kx;
                *pmx = kx;
            } else {
                Bf16x8 mn = unpack8(*pmn), mx = unpack8(*pmx);
                const Bf16x8 xv = unpack8(kx);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    mn.v[t] = bf_min(mn.v[t], xv.v[t]);
                    mx.v[t] = bf_max(mx.v[t], xv.v[t]);
                }
                *pmn = pack8(mn);
                *pmx = pack8(mx);
            }
        }
    }
}

constexpr int kSelectThreads = 1024;
constexpr int kSelectWarps = kSelectThreads / 32;
constexpr int kKeysInSmem = 32 * 1024;  // 128 KB of keys
constexpr int kCandCap = 8 * 1024;      // keys of the boundary bin

// Exclusive scan of one value per thread over the CTA, in thread order.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_tot,
                                                         uint32_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    const uint32_t wsum = warp_tot[lane];  // kSelectWarps == 32
    uint32_t wincl = wsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, wincl, o);
        if (lane >= o) wincl += t;
    }
    const uint32_t before_warp = __shfl_sync(0xffffffffu, wincl - wsum, warp);
    total = __shfl_sync(0xffffffffu, wincl, 31);
    __syncthreads();
    return before_warp + incl - v;
}

// Radix select, most significant digit first, over n keys read through
// key(i): narrows (prefix, pmask) to the value T of the remaining-th largest
// key among those whose bits under pmask equal prefix; `remaining` ends as the
// number of keys equal to T to take.
template <typename KeyFn>
__device__ __forceinline__ void radix_select(KeyFn key, int n, int bits_left, uint32_t &prefix,
                                             uint32_t &pmask, uint32_t &remaining, uint32_t *hist,
                                             uint32_t *sh) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    while (bits_left > 0) {
        const int width = bits_left < 8 ? bits_left : 8;
        const int shift = bits_left - width;
        const uint32_t nbm = (1u << width) - 1u;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kSelectThreads) {
            const uint32_t x = key(i);
            if ((x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & nbm], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t local[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                local[j] = hist[lane * 8 + j];
                sum += local[j];
            }
            uint32_t incl = sum;  // keys in bins >= lane*8
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += t;
            }
            const uint32_t above = incl - sum;
            if (above < remaining && remaining <= incl) {
                uint32_t cum = above, dg = lane * 8, ab = above;
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    if (cum < remaining && cum + local[j] >= remaining) {
                        dg = lane * 8 + j;
                        ab = cum;
                    }
                    cum += local[j];
                }
                sh[0] = dg;
                sh[1] = ab;
            }
        }
        __syncthreads();
        remaining -= sh[1];
        prefix |= sh[0] << shift;
        pmask |= nbm << shift;
        bits_left = shift;
        __syncthreads();
    }
}

// grid (hkv, batch), block kSelectThreads,
// dynamic smem = (key_cap + kCandCap) * 4 bytes, key_cap = min(max_pages, kKeysInSmem).
__global__ void __launch_bounds__(kSelectThreads)
    select_kernel(const float *__restrict__ scores, uint32_t *__restrict__ hist,
                  uint32_t *__restrict__ hist_range, const int32_t *__restrict__ seq_len,
                  const int32_t *__restrict__ topk, int max_topk, int32_t *__restrict__ block_idx,
                  int32_t *__restrict__ block_cnt, int hkv, int max_pages, int key_cap,
                  uint32_t *err) {
    extern __shared__ uint32_t dsm[];
    uint32_t *keys_s = dsm;          // [key_cap]
    uint32_t *cand = dsm + key_cap;  // [kCandCap] low 16 bits of boundary-bin keys
    __shared__ uint32_t hist_s[256];
    __shared__ uint32_t warp_tot[kSelectWarps], warp_gt[kSelectWarps], warp_eq[kSelectWarps];
    __shared__ uint32_t sh[4];
    __shared__ uint32_t cand_n;

    pdl_launch_next();
    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t unit = (size_t)b * hkv + h;
    int32_t *out = block_idx + unit * (max_topk + 1);
    int32_t *cnt = block_cnt + unit;
    const int L = seq_len[b];
    const bool seq_ok = L >= 1 && L <= max_pages * kBlock;
    const int M = seq_ok ? (L - 1) / kBlock : 0;
    int k = topk[b];
    k = k < 0 ? 0 : k;
    bool topk_err = false;
    if (k > max_topk && M > max_topk) {
        topk_err = true;
        k = max_topk;
    }
    k = min(k, M);
    pdl_wait();

    // Touched histogram bins [dmin, dmax]; reset the range for the next call.
    const uint32_t emin = hist_range[2 * unit], emax = hist_range[2 * unit + 1];
    const int dmin = (int)(kHistBins - emin), dmax = (int)emax - 1;
    const int nbins = dmax >= dmin ? dmax - dmin + 1 : 0;
    uint32_t *hb = hist + unit * kHistBins;
    if (tid == 0) {
        cand_n = 0;
        sh[0] = sh[1] = sh[2] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        hist_range[2 * unit] = 0;
        hist_range[2 * unit + 1] = 0;
    }
    // Bins in descending order, a contiguous chunk per thread.
    const int chunk = (nbins + kSelectThreads - 1) / kSelectThreads;
    const int top = dmax - tid * chunk;
    const int lo = max(dmin, top - chunk + 1);
    uint32_t local = 0;
    for (int d = top; d >= lo; --d) local += __ldcg(&hb[d]);
    uint32_t total;
    const uint32_t above_me = block_exclusive_scan(local, warp_tot, total);
    const bool trivial = !seq_ok || k == M || k == 0;
    if (!trivial && above_me < (uint32_t)k && (uint32_t)k <= above_me + local) {
        uint32_t cum = above_me;
        for (int d = top; d >= lo; --d) {
            const uint32_t c = __ldcg(&hb[d]);
            if (cum + c >= (uint32_t)k) {
                sh[0] = (uint32_t)d;  // boundary digit
                sh[1] = cum;          // keys above it
                break;
            }
            cum += c;
        }
    }
    __syncthreads();
    for (int d = top; d >= lo; --d) hb[d] = 0;  // leave the histogram clear

    if (tid == 0) {
        if (!seq_ok) set_error(err, RESA_DEVERR_SEQ_LEN);
        if (topk_err) set_error(err, RESA_DEVERR_TOPK);
    }
    if (!seq_ok) {
        if (tid == 0) *cnt = 0;
        return;
    }
    if (k == M) {  // every complete block (also k = M = 0)
        for (int i = tid; i < M; i += kSelectThreads) out[i] = i;
        if (tid == 0) {
            out[M] = M;
            *cnt = M + 1;
        }
        return;
    }
    if (k == 0) {
        if (tid == 0) {
            out[0] = M;
            *cnt = 1;
        }
        return;
    }
    const bool hist_ok = total == (uint32_t)M;  // every complete block was scored
    if (!hist_ok && tid == 0) set_error(err, RESA_DEVERR_PAGE);
    const uint32_t d1 = sh[0];
    uint32_t remaining = (uint32_t)k - sh[1];

    // Keys into shared memory; gather the boundary bin's low halves.
    const float *src = scores + unit * max_pages;
    const bool in_smem = M <= key_cap;
    constexpr int U = 8;
    for (int i0 = warp * 32 * U; i0 < M; i0 += kSelectThreads * U) {
        uint32_t kv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 32 + lane;
            kv[u] = i < M ? order_key(src[i]) : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 32 + lane;
            const bool valid = i < M;
            if (valid && in_smem) keys_s[i] = kv[u];
            const bool is_c = valid && (kv[u] >> 16) == d1;
            const uint32_t ball = __ballot_sync(0xffffffffu, is_c);
            if (ball) {
                uint32_t base = 0;
                if (lane == 0) base = atomicAdd(&cand_n, (uint32_t)__popc(ball));
                base = __shfl_sync(0xffffffffu, base, 0);
                const uint32_t r = base + __popc(ball & ((1u << lane) - 1u));
                if (is_c && r < (uint32_t)kCandCap) cand[r] = kv[u] & 0xffffu;
            }
        }
    }
    __syncthreads();
    auto key_at = [&](int i) -> uint32_t { return in_smem ? keys_s[i] : order_key(src[i]); };
    uint32_t prefix, pmask;
    const int nc = (int)cand_n;
    if (hist_ok && nc <= kCandCap) {
        uint32_t cp = 0, cm = 0;
        radix_select([&](int i) { return cand[i]; }, nc, 16, cp, cm, remaining, hist_s, sh);
        prefix = (d1 << 16) | cp;
    } else if (hist_ok) {
        prefix = d1 << 16;
        pmask = 0xffff0000u;
        radix_select(key_at, M, 16, prefix, pmask, remaining, hist_s, sh);
    } else {  // no usable histogram: full radix select over the keys
        prefix = 0;
        pmask = 0;
        remaining = (uint32_t)k;
        radix_select(key_at, M, 32, prefix, pmask, remaining, hist_s, sh);
    }
    const uint32_t T = prefix;
    const uint32_t need_eq = remaining;

    // Ballot compaction in ascending block order: warp w owns [w*R, (w+1)*R).
    const int R = (M + kSelectWarps - 1) / kSelectWarps;
    const int w0 = warp * R, w1 = min(M, w0 + R);
    uint32_t gt = 0, eq = 0;
    for (int i = w0 + lane; i < w1; i += 32) {
        const uint32_t x = key_at(i);
        gt += x > T;
        eq += x == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
        warp_gt[warp] = gt;
        warp_eq[warp] = eq;
    }
    __syncthreads();
    uint32_t gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) {
        gt_before += warp_gt[w];
        eq_before += warp_eq[w];
    }
    uint32_t pos = gt_before + min(eq_before, need_eq);
    uint32_t eq_seen = eq_before;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = w0; base < w1; base += 32) {
        const int i = base + lane;
        const uint32_t xk = i < w1 ? key_at(i) : 0u;
        const bool is_gt = i < w1 && xk > T;
        const bool is_eq = i < w1 && xk == T;
        const uint32_t eq_ball = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t eq_rank = eq_seen + __popc(eq_ball & lt_mask);
        const bool take = is_gt || (is_eq && eq_rank < need_eq);
        const uint32_t take_ball = __ballot_sync(0xffffffffu, take);
        if (take) out[pos + __popc(take_ball & lt_mask)] = i;
        pos += __popc(take_ball);
        eq_seen += __popc(eq_ball);
    }
    if (tid == 0) {
        out[k] = M;
        *cnt = k + 1;
    }
}

template <int D>
cudaError_t launch_score_d(const Shape &s, void *desc, const int32_t *page_table,
                           const int32_t *seq_len, const void *q, float *scores, uint32_t *hist,
                           uint32_t *hist_range, void *K, void *V, const void *k_new,
                           const void *v_new, uint32_t *err, cudaStream_t st) {
    // ~2 CTAs per SM over all sequences, at least 4 stages of pages each
    const int by_work = (s.max_pages + 4 * kScoreGroup - 1) / (4 * kScoreGroup);
    const int by_sm = (2 * kNumSms + s.batch - 1) / s.batch;
    const int X = max(1, min(by_work, by_sm));
    dim3 grid(X, s.batch);
#define RESA_SCORE_CASE(H)                                                                    \
    case H: {                                                                                 \
        constexpr int smem = kScoreStages * kScoreGroup * H * 2 * D * 2;                      \
        static std::atomic<int> done[64];                                                     \
        cudaError_t e = ensure_smem(score_kernel<D, H>, smem, done);                          \
        if (e != cudaSuccess) return e;                                                       \
        return launch_pdl(score_kernel<D, H>, grid, dim3(kScoreThreads), smem, st,            \
                          (uint16_t *)desc, page_table, seq_len, (const uint16_t *)q, scores, \
                          hist, hist_range, s.g, s.max_pages, s.num_pages, (uint4 *)K,        \
                          (uint4 *)V, (const uint4 *)k_new, (const uint4 *)v_new, err);       \
    }
    switch (s.hkv) {
        RESA_SCORE_CASE(1)
        RESA_SCORE_CASE(2)
        RESA_SCORE_CASE(4)
        RESA_SCORE_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef RESA_SCORE_CASE
}

}  // namespace

cudaError_t launch_score(const Shape &s, void *desc, const int32_t *page_table,
                         const int32_t *seq_len, const void *q, float *scores, uint32_t *hist,
                         uint32_t *hist_range, void *K, void *V, const void *k_new,
                         const void *v_new, uint32_t *err, cudaStream_t st) {
    if (s.d == 128)
        return launch_score_d<128>(s, desc, page_table, seq_len, q, scores, hist, hist_range, K, V,
                                   k_new, v_new, err, st);
    if (s.d == 64)
        return launch_score_d<64>(s, desc, page_table, seq_len, q, scores, hist, hist_range, K, V,
                                  k_new, v_new, err, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_select(const Shape &s, const float *scores, uint32_t *hist,
                          uint32_t *hist_range, const int32_t *seq_len, const int32_t *topk,
                          int max_topk, int32_t *block_idx, int32_t *block_cnt, uint32_t *err,
                          cudaStream_t st) {
    const int cap = s.max_pages < kKeysInSmem ? s.max_pages : kKeysInSmem;
    const size_t smem = (size_t)(cap + kCandCap) * 4;
    static std::atomic<int> done[64];
    cudaError_t e = ensure_smem(select_kernel, (kKeysInSmem + kCandCap) * 4, done);
    if (e != cudaSuccess) return e;
    dim3 grid(s.hkv, s.batch);
    return launch_pdl(select_kernel, grid, dim3(kSelectThreads), smem, st, scores, hist,
                      hist_range, seq_len, topk, max_topk, block_idx, block_cnt, s.hkv,
                      s.max_pages, cap, err);
}

}  // namespace resa
