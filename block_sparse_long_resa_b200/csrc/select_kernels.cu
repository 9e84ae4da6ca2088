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
// select_kernel runs one thread-block cluster of eight CTAs per (sequence, kv
// head), each CTA owning one eighth of the keys.  Every CTA finds the
// histogram bin holding the k-th largest key (only the touched bins are
// read; the first CTA clears them for the next call); one pass over its slice
// counts the keys above that bin and gathers the bin's keys; the cluster's
// candidates are exchanged through distributed shared memory and a radix
// select of their low 16 bits gives the threshold T; per-CTA counts of keys
// above / equal to T give each CTA its output offset, and a ballot pass
// writes the blocks with key > T plus the lowest-index blocks with key == T
// in ascending order.
#include <cooperative_groups.h>

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
    __syncthreads();

    if (warp == 0) {  // ------------------------------------------------ producer
        static_assert(kScoreStages * kScoreGroup == 32, "one lane per page of the first stages");
        // Page ids of the first kScoreStages groups (the page table is an
        // input of the call): lane = group * kScoreGroup + slot.
        int pg_first = -1;
        {
            const int p = p_begin + lane;
            if (p < p_end) pg_first = page_table[(size_t)b * max_pages + p];
        }
        pdl_wait();  // descriptors and workspace may be written by the preceding kernels
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
            if (i < kScoreStages) {
                pg = __shfl_sync(0xffffffffu, pg_first, (i * kScoreGroup + lane) & 31);
                if (lane >= npg) pg = -1;
            } else if (lane < npg) {
                pg = page_table[(size_t)b * max_pages + p0 + lane];
            }
            if (lane < npg && (pg < 0 || pg >= num_pages)) {
                set_error(err, RESA_DEVERR_PAGE);
                pg = -1;
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
        // Group pooling: mean of the g query heads, fp32, head order, then / g
        // (q is an input of the call, read while the first copies are in flight).
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
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kScoreConsumers) : "memory");
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

constexpr int kSelCluster = 8;    // CTAs per (sequence, kv head): one thread-block cluster
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelKeys = 4096;     // keys of its slice a CTA keeps in shared memory
constexpr int kSelCandCap = 4096;  // boundary-bin keys gathered from the whole cluster
constexpr int kSelLocalCand = 1024;

// Exclusive scan of one value per thread over the CTA, in thread order.
__device__ __forceinline__ uint32_t cta_exclusive_scan(uint32_t v, uint32_t *warp_tot,
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
    const uint32_t wsum = lane < kSelWarps ? warp_tot[lane] : 0u;
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
        for (int i = tid; i < n; i += kSelThreads) {
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

// Grid (kSelCluster, hkv, batch), clusters of kSelCluster CTAs along x: one
// cluster per (sequence, kv head); CTA rank r owns keys [r*C, (r+1)*C).
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const float *__restrict__ scores, uint32_t *__restrict__ hist,
                  uint32_t *__restrict__ hist_range, const int32_t *__restrict__ seq_len,
                  const int32_t *__restrict__ topk, int max_topk, int32_t *__restrict__ block_idx,
                  int32_t *__restrict__ block_cnt, int hkv, int max_pages, uint32_t *err) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ uint32_t keys_s[kSelKeys];
    __shared__ uint32_t lc_key[kSelLocalCand];  // this CTA's boundary-bin keys (low 16 bits)
    __shared__ int32_t lc_idx[kSelLocalCand];   // and their block ids
    __shared__ uint32_t all_c[kSelCandCap];     // the cluster's boundary-bin keys
    __shared__ uint32_t hist_s[256];
    __shared__ uint32_t warp_tot[kSelWarps], warp_gt[kSelWarps], warp_eq[kSelWarps];
    __shared__ uint32_t sh[4];
    __shared__ uint32_t lc_n;                   // candidates of this CTA
    __shared__ uint32_t cta_gt, cta_eq;         // keys > T / == T in this CTA's slice

    pdl_launch_next();
    const int rank = (int)cluster.block_rank();
    const int h = blockIdx.y, b = blockIdx.z;
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
    const int C = (M + kSelCluster - 1) / kSelCluster;
    const int c0 = min(M, rank * C), c1 = min(M, c0 + C);
    pdl_wait();

    // Boundary bin of the k-th largest key from the scorer's histogram
    // (every CTA of the cluster computes the same; rank 0 clears it later).
    const uint32_t emin = hist_range[2 * unit], emax = hist_range[2 * unit + 1];
    const int dmin = (int)(kHistBins - emin), dmax = (int)emax - 1;
    const int nbins = dmax >= dmin ? dmax - dmin + 1 : 0;
    uint32_t *hb = hist + unit * kHistBins;
    if (tid == 0) {
        lc_n = 0;
        sh[0] = sh[1] = 0;
    }
    const int chunk = (nbins + kSelThreads - 1) / kSelThreads;
    const int top = dmax - tid * chunk;
    const int lo = max(dmin, top - chunk + 1);
    uint32_t local = 0;
    for (int d = top; d >= lo; --d) local += __ldcg(&hb[d]);
    uint32_t total;
    const uint32_t above_me = cta_exclusive_scan(local, warp_tot, total);
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
    const bool hist_ok = total == (uint32_t)M;
    const uint32_t d1 = sh[0];
    uint32_t remaining = (uint32_t)k - sh[1];

    // One pass over this CTA's slice: keys into shared memory, per-warp count
    // of keys above the boundary bin, the bin's keys as candidates.
    const float *src = scores + unit * max_pages;
    const int n_mine = c1 - c0;
    const bool in_smem = n_mine <= kSelKeys;
    const int R = (n_mine + kSelWarps - 1) / kSelWarps;
    const int w0 = c0 + warp * R, w1 = min(c1, w0 + R);
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t above_w = 0;
    if (!trivial) {
        constexpr int U = 4;
        for (int base = w0; base < w1; base += 32 * U) {
            uint32_t kv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * 32 + lane;
                kv[u] = i < w1 ? order_key(src[i]) : 0u;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * 32 + lane;
                const bool valid = i < w1;
                if (valid && in_smem) keys_s[i - c0] = kv[u];
                const uint32_t dg = kv[u] >> 16;
                above_w += __popc(__ballot_sync(0xffffffffu, valid && dg > d1));
                const bool is_c = valid && dg == d1;
                const uint32_t ball = __ballot_sync(0xffffffffu, is_c);
                if (ball) {
                    uint32_t cb = 0;
                    if (lane == 0) cb = atomicAdd(&lc_n, (uint32_t)__popc(ball));
                    cb = __shfl_sync(0xffffffffu, cb, 0);
                    const uint32_t r = cb + __popc(ball & lt_mask);
                    if (is_c && r < (uint32_t)kSelLocalCand) {
                        lc_key[r] = kv[u] & 0xffffu;
                        lc_idx[r] = i;
                    }
                }
            }
        }
    }
    if (lane == 0) {
        warp_gt[warp] = above_w;
        warp_eq[warp] = 0;
    }
    cluster.sync();  // #1: every CTA's candidates are ready; the histogram is read

    if (rank == 0) {  // leave the histogram clear for the next call
        for (int d = dmin + tid; d <= dmax; d += kSelThreads) hb[d] = 0;
        if (tid == 0) {
            hist_range[2 * unit] = 0;
            hist_range[2 * unit + 1] = 0;
            if (!seq_ok) set_error(err, RESA_DEVERR_SEQ_LEN);
            if (topk_err) set_error(err, RESA_DEVERR_TOPK);
        }
    }
    uint32_t T = 0, need_eq = 0;
    bool fallback = trivial ? false : !hist_ok;
    if (!trivial) {
        // Gather the cluster's candidates (distributed shared memory).
        uint32_t offs[kSelCluster], ntot = 0;
#pragma unroll
        for (int r = 0; r < kSelCluster; ++r) {
            const uint32_t n = *cluster.map_shared_rank(&lc_n, r);
            offs[r] = ntot;
            ntot += n;
            if (n > (uint32_t)kSelLocalCand) fallback = true;
        }
        if (ntot > (uint32_t)kSelCandCap) fallback = true;
        if (!fallback) {
#pragma unroll
            for (int r = 0; r < kSelCluster; ++r) {
                const uint32_t *peer = cluster.map_shared_rank(lc_key, r);
                const uint32_t n = (r + 1 < kSelCluster ? offs[r + 1] : ntot) - offs[r];
                for (uint32_t i = tid; i < n; i += kSelThreads) all_c[offs[r] + i] = peer[i];
            }
            __syncthreads();
            uint32_t cp = 0, cm = 0;
            radix_select([&](int i) { return all_c[i]; }, (int)ntot, 16, cp, cm, remaining, hist_s,
                         sh);
            T = (d1 << 16) | cp;
            need_eq = remaining;
            // this CTA's candidates above / at T, per owning warp range
            const uint32_t myn = lc_n;
            for (uint32_t c = tid; c < myn; c += kSelThreads) {
                const uint32_t key = (d1 << 16) | lc_key[c];
                const int w = (lc_idx[c] - c0) / R;
                if (key > T) atomicAdd(&warp_gt[w], 1u);
                else if (key == T) atomicAdd(&warp_eq[w], 1u);
            }
        } else {
            // Degenerate score distribution: radix over every key of the sequence.
            uint32_t prefix = 0, pmask = 0;
            remaining = (uint32_t)k;
            radix_select([&](int i) { return order_key(src[i]); }, M, 32, prefix, pmask,
                         remaining, hist_s, sh);
            T = prefix;
            need_eq = remaining;
            uint32_t gt = 0, eq = 0;
            for (int i = w0 + lane; i < w1; i += 32) {
                const uint32_t x = order_key(src[i]);
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
        }
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t g2 = 0, e2 = 0;
        for (int w = 0; w < kSelWarps; ++w) {
            g2 += warp_gt[w];
            e2 += warp_eq[w];
        }
        cta_gt = g2;
        cta_eq = e2;
    }
    cluster.sync();  // #2: per-CTA counts visible to the cluster

    if (trivial) {
        if (seq_ok) {
            if (k == M)
                for (int i = c0 + tid; i < c1; i += kSelThreads) out[i] = i;
            if (rank == 0 && tid == 0) {
                out[k] = M;
                *cnt = k + 1;
            }
        } else if (rank == 0 && tid == 0) {
            *cnt = 0;
        }
    } else {
        uint32_t gt_before = 0, eq_before = 0;
        for (int r = 0; r < rank; ++r) {
            gt_before += *cluster.map_shared_rank(&cta_gt, r);
            eq_before += *cluster.map_shared_rank(&cta_eq, r);
        }
        for (int w = 0; w < warp; ++w) {
            gt_before += warp_gt[w];
            eq_before += warp_eq[w];
        }
        auto key_at = [&](int i) -> uint32_t {
            return (in_smem && !fallback) ? keys_s[i - c0] : order_key(src[i]);
        };
        uint32_t pos = gt_before + min(eq_before, need_eq);
        uint32_t eq_seen = eq_before;
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
        if (rank == 0 && tid == 0) {
            out[k] = M;
            *cnt = k + 1;
        }
    }
    cluster.sync();  // #3: no CTA leaves while a peer may still read its shared memory
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kSelCluster, s.hkv, s.batch);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSelCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, select_kernel, scores, hist, hist_range, seq_len, topk,
                              max_topk, block_idx, block_cnt, s.hkv, s.max_pages, err);
}

}  // namespace resa
