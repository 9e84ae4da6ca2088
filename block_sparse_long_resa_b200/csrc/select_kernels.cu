// Query-aware block selection (ReSA summary §3.4.1): group query pooling, the
// Quest upper-bound score of Eq. 4 for every complete block, and top-n
// selection (Eq. 5 count from the caller, ties to the lower block index) with
// the local block always appended.
//
// score_kernel streams the block key cache.  Grid (X, batch), one CTA per
// SM; CTA x owns a contiguous range of complete blocks of one sequence, and
// its 16 scoring warps take every 16th page of it.  Each warp streams its
// descriptor pages (all kv heads, 2*d bf16 each) through a private ring in
// shared memory with 16-byte cp.async copies, several pages in flight: these
// go through the load/store path, which keeps HBM busy at any page size and
// page order, where one bulk (TMA) copy per 2 KB page would be limited by
// the copy engine's per-request rate.  Since q-bar is fixed for the call,
// max(q*max, q*min) is q times the max where q >= 0 and the min elsewhere: a
// byte permute picks that half, then one multiply and one add per channel
// (lane = d/32 channels); one transposing shuffle reduction finishes the Hkv
// sums of a page.  Every score also bumps a 65536-bin histogram of the top 16
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
// above / equal to T, pushed into every CTA of the cluster, give each CTA its
// output offset, and a ballot pass writes the blocks with key > T plus the
// lowest-index blocks with key == T in ascending order.
#include <cooperative_groups.h>

#include "resa_common.cuh"

namespace resa {
namespace {

constexpr int kScoreWarps = 16;                   // scoring warps per CTA (one CTA per SM)
constexpr int kScoreChunk = 512;                  // pages a scoring CTA takes at most, batches
constexpr int kScoreRingBytes = 192 * 1024;       // shared-memory ring budget per CTA
constexpr int kScoreThreads = 32 * (kScoreWarps + 1);  // + the decode-token append warp
constexpr int kHashSlots = 2048;  // per-CTA histogram aggregation table
constexpr uint32_t kHashEmpty = 0xffffffffu;

template <int D, int HKV>
struct ScoreCfg {
    static constexpr int kPageBytes = HKV * 2 * D * 2;  // one descriptor page, all kv heads
    // pages in flight per warp (cp.async groups outstanding)
    static constexpr int kFit = kScoreRingBytes / kScoreWarps / kPageBytes;
    static constexpr int kRing = kFit < 8 ? kFit : 8;
    static constexpr int kRingBytes = kScoreWarps * kRing * kPageBytes;
    static_assert(kRing >= 2, "at least two pages in flight per warp");
};

// grid (X, batch), block kScoreThreads, dynamic smem ScoreCfg::kRingBytes.
template <int D, int HKV>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(uint16_t *__restrict__ desc, const int32_t *__restrict__ page_table,
                 const int32_t *__restrict__ seq_len, const uint16_t *__restrict__ q,
                 float *__restrict__ scores, uint32_t *__restrict__ hist,
                 uint32_t *__restrict__ hist_range, int g, int max_pages, int num_pages,
                 uint4 *__restrict__ K, uint4 *__restrict__ V, const uint4 *__restrict__ k_new,
                 const uint4 *__restrict__ v_new, int bs, const RowMap rm, uint32_t *err) {
    using CF = ScoreCfg<D, HKV>;
    constexpr int PAGE_ELEMS = HKV * 2 * D;  // bf16 per descriptor page
    constexpr int PAGE_CHUNKS = CF::kPageBytes / 16;
    constexpr int N = D / 32;                // channels per lane
    constexpr int RING = CF::kRing;
    extern __shared__ __align__(128) uint8_t ring_all[];
    __shared__ float qbar_s[HKV][D];
    // Per-CTA aggregation of the key histogram: (head, top-16-bit digit) ->
    // count in an open-addressing table, flushed with one global atomic per
    // distinct entry; and the touched-digit range per head.
    __shared__ uint32_t hkey[kHashSlots], hcnt[kHashSlots];
    __shared__ uint32_t rng_min[HKV], rng_max[HKV];

    pdl_launch_next();
    const int b = blockIdx.y, x = blockIdx.x, X = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hq = HKV * g;
    const int row = cache_row(rm, b, x == 0 && threadIdx.x == 0 ? err : nullptr);
    const int L = row_seq_len(seq_len, row);
    const bool seq_ok = L >= 1 && L <= max_pages * bs;
    const int M = seq_ok ? (L - 1) / bs : 0;
    const int per = (M + X - 1) / X;
    const int p_begin = min(M, x * per), p_end = min(M, p_begin + per);

    if (warp < kScoreWarps) {
        for (int i = threadIdx.x; i < kHashSlots; i += 32 * kScoreWarps) {
            hkey[i] = kHashEmpty;
            hcnt[i] = 0;
        }
        if (threadIdx.x < HKV) {
            rng_min[threadIdx.x] = 0xffffffffu;
            rng_max[threadIdx.x] = 0;
        }
        // This warp's pages: p_begin + warp + kScoreWarps * t.  Lane t holds
        // the id of the warp's page t of the current batch of 32 (the page
        // table is an input of the call: read before waiting).
        const int n_mine = p_end - p_begin > warp ? (p_end - p_begin - warp + kScoreWarps - 1) / kScoreWarps : 0;
        auto batch_ids = [&](int t0) {
            const int t = t0 + lane;
            return t < n_mine ? page_table[(size_t)row * max_pages + p_begin + warp + kScoreWarps * t] : -1;
        };
        int ids = batch_ids(0);
        pdl_wait();  // descriptors may be written by the preceding kernels
        if (!seq_ok && x == 0 && warp == 0 && lane == 0) set_error(err, RESA_DEVERR_SEQ_LEN);

        uint8_t *ring = ring_all + (size_t)warp * RING * CF::kPageBytes;
        uint32_t valid_b = 0;
        auto check_batch = [&](int t0) {
            const bool v = ids >= 0 && ids < num_pages;
            if (t0 + lane < n_mine && !v) set_error(err, RESA_DEVERR_PAGE);
            valid_b = __ballot_sync(0xffffffffu, t0 + lane < n_mine && v);
        };
        check_batch(0);
        // Copy of page t into ring slot t % RING, one cp.async group per page
        // (empty groups past the end keep the group count uniform).  Pages are
        // issued in order; the ids of batch t >> 5 are in `ids`.
        uint32_t slot_valid = 0;  // bit t % RING: page t's id was valid (uniform over the warp)
        auto issue_page = [&](int t) {
            if (t < n_mine) {
                if ((t & 31) == 0 && t > 0) {
                    ids = batch_ids(t);
                    check_batch(t);
                }
                const int pg = __shfl_sync(0xffffffffu, ids, t & 31);
                const uint32_t ok = (valid_b >> (t & 31)) & 1u;
                const int slot = t % RING;
                slot_valid = (slot_valid & ~(1u << slot)) | (ok << slot);
                if (ok) {
                    const uint8_t *src = reinterpret_cast<const uint8_t *>(desc + (size_t)pg * PAGE_ELEMS);
                    uint8_t *dst = ring + (size_t)(t % RING) * CF::kPageBytes;
#pragma unroll
                    for (int c = lane; c < PAGE_CHUNKS; c += 32) cp_async16(dst + c * 16, src + c * 16);
                }
            }
            cp_async_commit();
        };
#pragma unroll
        for (int t = 0; t < RING - 1; ++t) issue_page(t);

        // Group pooling while the first pages are in flight: mean of the g
        // query heads, fp32, head order, then / g.
        for (int e = threadIdx.x; e < HKV * D; e += 32 * kScoreWarps) {
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
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kScoreWarps) : "memory");
        float qv[HKV][N];
        uint32_t sel[HKV][N / 2];
#pragma unroll
        for (int h = 0; h < HKV; ++h) {
#pragma unroll
            for (int n = 0; n < N; ++n) qv[h][n] = qbar_s[h][lane * N + n];
#pragma unroll
            for (int n = 0; n < N / 2; ++n) sel[h][n] = upper_bound_selector(qv[h][2 * n], qv[h][2 * n + 1]);
        }

        // Head h of a page is value h; after the transposing reduction lane
        // l holds the full sum of head l >> (5 - kLogP) and lane h << (5 - kLogP)
        // owns head h's output.
        constexpr int kLogP = HKV == 1 ? 0 : HKV == 2 ? 1 : HKV == 4 ? 2 : 3;
        static_assert((1 << kLogP) == HKV, "power-of-two kv heads");
        const int my_h = lane >> (5 - kLogP);
        const bool owner = (lane & ((1 << (5 - kLogP)) - 1)) == 0;
        const size_t unit = (size_t)b * HKV + my_h;
        uint32_t dmin = 0xffffffffu, dmax = 0;
        for (int t = 0; t < n_mine; ++t) {
            issue_page(t + RING - 1);  // refills the slot of page t - 1
            cp_async_wait<RING - 1>();
            __syncwarp();
            const uint8_t *pgp = ring + (size_t)(t % RING) * CF::kPageBytes;
            // Partial sums of this lane's channels: sum over n of q_n * (max_n
            // if q_n >= 0 else min_n), products rounded, added in channel order.
            float v[HKV];
#pragma unroll
            for (int h = 0; h < HKV; ++h) {
                const uint16_t *row = reinterpret_cast<const uint16_t *>(pgp + (size_t)h * 2 * D * 2);
                uint32_t mnw[N / 2], mxw[N / 2];
                if constexpr (N == 4) {
                    const uint2 a = *reinterpret_cast<const uint2 *>(row + lane * 4);
                    const uint2 z = *reinterpret_cast<const uint2 *>(row + D + lane * 4);
                    mnw[0] = a.x;
                    mnw[1] = a.y;
                    mxw[0] = z.x;
                    mxw[1] = z.y;
                } else {
                    mnw[0] = *reinterpret_cast<const uint32_t *>(row + lane * 2);
                    mxw[0] = *reinterpret_cast<const uint32_t *>(row + D + lane * 2);
                }
                float sum = 0.f;
#pragma unroll
                for (int n = 0; n < N / 2; ++n) {
                    const uint32_t w = __byte_perm(mnw[n], mxw[n], sel[h][n]);
                    sum = __fadd_rn(sum, __fmul_rn(qv[h][2 * n], __uint_as_float(w << 16)));
                    sum = __fadd_rn(sum, __fmul_rn(qv[h][2 * n + 1], __uint_as_float(w & 0xffff0000u)));
                }
                v[h] = sum;
            }
            __syncwarp();  // the slot is refilled by the next issue
            // Transposing reduction: each step halves the values a lane keeps
            // (upper half where the step's lane bit is set) and adds the
            // partner's copy of the same heads.
#pragma unroll
            for (int k = 0; k < kLogP; ++k) {
                const int mask = 16 >> k;
                const int half = HKV >> (k + 1);
                const bool upper = (lane & mask) != 0;
#pragma unroll
                for (int j = 0; j < half; ++j) {
                    const float send = upper ? v[j] : v[j + half];
                    const float keep = upper ? v[j + half] : v[j];
                    v[j] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                }
            }
#pragma unroll
            for (int mask = 16 >> kLogP; mask > 0; mask >>= 1)
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
            const int page_idx = p_begin + warp + kScoreWarps * t;
            const bool page_ok = ((slot_valid >> (t % RING)) & 1u) != 0;
            if (owner && page_ok) {
                const float mine = v[0];
                scores[unit * max_pages + page_idx] = mine;
                const uint32_t digit = order_key(mine) >> 16;
                const uint32_t key = ((uint32_t)my_h << 16) | digit;
                uint32_t slot = (digit * 0x9E3779B1u + (uint32_t)my_h * 0x85EBCA77u) >> 21;  // 11 bits
                bool placed = false;
                for (int probe = 0; probe < 64; ++probe) {
                    const uint32_t old = atomicCAS(&hkey[slot], kHashEmpty, key);
                    if (old == kHashEmpty || old == key) {
                        atomicAdd(&hcnt[slot], 1u);
                        placed = true;
                        break;
                    }
                    slot = (slot + 1) & (kHashSlots - 1);
                }
                if (!placed) atomicAdd(&hist[unit * kHistBins + digit], 1u);  // crowded table
                dmin = min(dmin, digit);
                dmax = max(dmax, digit);
            }
        }
        cp_async_wait<0>();
        if (owner && dmin <= dmax) {
            atomicMin(&rng_min[my_h], dmin);
            atomicMax(&rng_max[my_h], dmax);
        }
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kScoreWarps) : "memory");
        // Flush: one global atomic per distinct (head, digit) of the CTA, and
        // the touched-bin range once per head.
        for (int i = threadIdx.x; i < kHashSlots; i += 32 * kScoreWarps) {
            const uint32_t key = hkey[i];
            if (key != kHashEmpty)
                atomicAdd(&hist[((size_t)b * HKV + (key >> 16)) * kHistBins + (key & 0xffffu)], hcnt[i]);
        }
        if (threadIdx.x < HKV && rng_min[threadIdx.x] <= rng_max[threadIdx.x]) {
            const size_t u = (size_t)b * HKV + threadIdx.x;
            atomicMax(&hist_range[2 * u], (uint32_t)kHistBins - rng_min[threadIdx.x]);  // 0 = untouched
            atomicMax(&hist_range[2 * u + 1], rng_max[threadIdx.x] + 1u);
        }
    } else if (K != nullptr && x == 0) {  // ------------------------ decode-token append
        pdl_wait();
        if (!seq_ok) return;
        const int pos = L - 1;
        const int page = page_table[(size_t)row * max_pages + pos / bs];
        if (page < 0 || page >= num_pages) {
            if (lane == 0) set_error(err, RESA_DEVERR_PAGE);
            return;
        }
        const int slot = pos % bs;
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        uint4 *dsc = reinterpret_cast<uint4 *>(desc);
        for (int e = lane; e < HKV * CPR; e += 32) {
            const int h = e / CPR, cc = e % CPR;
            const uint4 kx = k_new[((size_t)b * HKV + h) * CPR + cc];
            const uint4 vx = v_new[((size_t)b * HKV + h) * CPR + cc];
            const size_t o = (((size_t)page * HKV + h) * bs + slot) * CPR + cc;
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
constexpr int kSelWideUnits = 64;  // from this many (sequence, kv head) units on, 2 or 4 CTAs
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

// Grid (CL, hkv, batch), clusters of CL CTAs along x: one cluster per
// (sequence, kv head); CTA rank r owns keys [r*C, (r+1)*C).
template <int CL>
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const float *__restrict__ scores, uint32_t *__restrict__ hist,
                  uint32_t *__restrict__ hist_range, const int32_t *__restrict__ seq_len,
                  const int32_t *__restrict__ topk, int max_topk, int32_t *__restrict__ block_idx,
                  int32_t *__restrict__ block_cnt, int hkv, int max_pages, int bs,
                  const RowMap rm, uint32_t *err) {
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
    __shared__ uint32_t cta_gt[CL];    // keys > T / == T in each CTA's slice
    __shared__ uint32_t cta_eq[CL];

    pdl_launch_next();
    const int rank = (int)cluster.block_rank();
    const int h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t unit = (size_t)b * hkv + h;
    int32_t *out = block_idx + unit * (max_topk + 1);
    int32_t *cnt = block_cnt + unit;
    const int L = row_seq_len(seq_len, cache_row(rm, b, nullptr));
    const bool seq_ok = L >= 1 && L <= max_pages * bs;
    const int M = seq_ok ? (L - 1) / bs : 0;
    int k = topk[b];
    k = k < 0 ? 0 : k;
    bool topk_err = false;
    if (k > max_topk && M > max_topk) {
        topk_err = true;
        k = max_topk;
    }
    k = min(k, M);
    const int C = (M + CL - 1) / CL;
    const int c0 = min(M, rank * C), c1 = min(M, c0 + C);
    pdl_wait();

    // This CTA's first slice keys are requested before the histogram is read.
    const float *src = scores + unit * max_pages;
    const int n_mine = c1 - c0;
    const bool in_smem = n_mine <= kSelKeys;
    const int R = (n_mine + kSelWarps - 1) / kSelWarps;
    const int w0 = c0 + warp * R, w1 = min(c1, w0 + R);
    constexpr int U = 4;
    float first[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int i = w0 + u * 32 + lane;
        first[u] = i < w1 ? src[i] : 0.f;
    }

    // Boundary bin of the k-th largest key from the scorer's histogram
    // (every CTA of the cluster computes the same; rank 0 clears it later).
    // Thread t sums bins dmax - t*chunk down to dmax - (t+1)*chunk + 1.
    const uint32_t emin = hist_range[2 * unit], emax = hist_range[2 * unit + 1];
    const int dmin = (int)(kHistBins - emin), dmax = (int)emax - 1;
    const int nbins = dmax >= dmin ? dmax - dmin + 1 : 0;
    uint32_t *hb = hist + unit * kHistBins;
    if (tid == 0) {
        lc_n = 0;
        sh[0] = sh[1] = 0;
    }
    constexpr int kBinRegs = 8;
    const int chunk = (nbins + kSelThreads - 1) / kSelThreads;
    const int top = dmax - tid * chunk;
    const int lo = max(dmin, top - chunk + 1);
    uint32_t binc[kBinRegs];
    uint32_t local = 0;
    if (chunk <= kBinRegs) {
#pragma unroll
        for (int j = 0; j < kBinRegs; ++j) binc[j] = (j < chunk && top - j >= lo) ? __ldcg(&hb[top - j]) : 0u;
#pragma unroll
        for (int j = 0; j < kBinRegs; ++j) local += binc[j];
    } else {
        for (int d = top; d >= lo; --d) local += __ldcg(&hb[d]);
    }
    uint32_t total;
    const uint32_t above_me = cta_exclusive_scan(local, warp_tot, total);
    const bool trivial = !seq_ok || k == M || k == 0;
    if (!trivial && above_me < (uint32_t)k && (uint32_t)k <= above_me + local) {
        uint32_t cum = above_me;
        if (chunk <= kBinRegs) {
#pragma unroll
            for (int j = 0; j < kBinRegs; ++j) {
                if (j < chunk && top - j >= lo && cum < (uint32_t)k && cum + binc[j] >= (uint32_t)k) {
                    sh[0] = (uint32_t)(top - j);  // boundary digit
                    sh[1] = cum;                  // keys above it
                }
                cum += binc[j];
            }
        } else {
            for (int d = top; d >= lo; --d) {
                const uint32_t c = __ldcg(&hb[d]);
                if (cum + c >= (uint32_t)k) {
                    sh[0] = (uint32_t)d;
                    sh[1] = cum;
                    break;
                }
                cum += c;
            }
        }
    }
    __syncthreads();
    const bool hist_ok = total == (uint32_t)M;
    const uint32_t d1 = sh[0];
    uint32_t remaining = (uint32_t)k - sh[1];

    // One pass over this CTA's slice: keys into shared memory, per-warp count
    // of keys above the boundary bin, the bin's keys as candidates.
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t above_w = 0;
    if (!trivial) {
        for (int base = w0; base < w1; base += 32 * U) {
            uint32_t kv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = base + u * 32 + lane;
                kv[u] = i < w1 ? order_key(base == w0 ? first[u] : src[i]) : 0u;
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
        uint32_t nr[CL], offs[CL + 1];
#pragma unroll
        for (int r = 0; r < CL; ++r) nr[r] = *cluster.map_shared_rank(&lc_n, r);
        offs[0] = 0;
#pragma unroll
        for (int r = 0; r < CL; ++r) {
            offs[r + 1] = offs[r] + nr[r];
            if (nr[r] > (uint32_t)kSelLocalCand) fallback = true;
        }
        const uint32_t ntot = offs[CL];
        if (ntot > (uint32_t)kSelCandCap) fallback = true;
        if (!fallback) {
            // one flattened loop over the cluster's candidates: the remote
            // loads of all ranks are in flight together
            for (uint32_t j = tid; j < ntot; j += kSelThreads) {
                int r = 0;
                uint32_t base = 0;
#pragma unroll
                for (int q = 1; q < CL; ++q)
                    if (j >= offs[q]) {
                        r = q;
                        base = offs[q];
                    }
                all_c[j] = cluster.map_shared_rank(lc_key, r)[j - base];
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
    // This CTA's counts go into every CTA's table (remote stores), so that
    // after the next cluster barrier no CTA reads a peer's shared memory and
    // each may leave when done.
    if (tid < CL) {
        uint32_t g2 = 0, e2 = 0;
        for (int w = 0; w < kSelWarps; ++w) {
            g2 += warp_gt[w];
            e2 += warp_eq[w];
        }
        cluster.map_shared_rank(cta_gt, tid)[rank] = g2;
        cluster.map_shared_rank(cta_eq, tid)[rank] = e2;
    }
    cluster.sync();  // #2: every CTA has read its peers' candidates; count tables complete

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
            gt_before += cta_gt[r];
            eq_before += cta_eq[r];
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
}

template <int D>
cudaError_t launch_score_d(const Shape &s, void *desc, const int32_t *page_table,
                           const int32_t *seq_len, const void *q, float *scores, uint32_t *hist,
                           uint32_t *hist_range, void *K, void *V, const void *k_new,
                           const void *v_new, uint32_t *err, cudaStream_t st) {
    // At least two pages per scoring warp; at least one CTA per SM over all
    // sequences, and at least one CTA per kScoreChunk pages of the longest, so
    // that a long sequence in a large batch is scored by proportionally more
    // CTAs (the shorter ones' CTAs finish early and free their SMs).
    const int by_work = (s.max_pages + 2 * kScoreWarps - 1) / (2 * kScoreWarps);
    const int by_sm = s.batch < kNumSms ? kNumSms / s.batch : 1;
    const int by_len = (s.max_pages + kScoreChunk - 1) / kScoreChunk;
    const int X = max(1, min(by_work, max(by_sm, by_len)));
    dim3 grid(X, s.batch);
#define RESA_SCORE_CASE(H)                                                                    \
    case H: {                                                                                 \
        constexpr int smem = ScoreCfg<D, H>::kRingBytes;                                      \
        static std::atomic<int> done[64];                                                     \
        cudaError_t e = ensure_smem(score_kernel<D, H>, smem, done);                          \
        if (e != cudaSuccess) return e;                                                       \
        return launch_pdl(score_kernel<D, H>, grid, dim3(kScoreThreads), smem, st,            \
                          (uint16_t *)desc, page_table, seq_len, (const uint16_t *)q, scores, \
                          hist, hist_range, s.g, s.max_pages, s.num_pages, (uint4 *)K,        \
                          (uint4 *)V, (const uint4 *)k_new, (const uint4 *)v_new, s.bs, s.rows, \
                          err);                                                               \
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
    // Large batches: fewer CTAs per (sequence, kv head), so that the grid
    // stays near one wave, as long as a CTA's keys still fit its shared
    // memory (kSelKeys).
    int cl = kSelCluster;
    if (s.batch * s.hkv >= kSelWideUnits) {
        if ((s.max_pages + 1) / 2 <= kSelKeys) cl = 2;
        else if ((s.max_pages + 3) / 4 <= kSelKeys) cl = 4;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, s.hkv, s.batch);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
#define RESA_SELECT_LAUNCH(CL)                                                                \
    cudaLaunchKernelEx(&cfg, select_kernel<CL>, scores, hist, hist_range, seq_len, topk, max_topk, \
                       block_idx, block_cnt, s.hkv, s.max_pages, s.bs, s.rows, err)
    if (cl == 2) return RESA_SELECT_LAUNCH(2);
    if (cl == 4) return RESA_SELECT_LAUNCH(4);
    return RESA_SELECT_LAUNCH(kSelCluster);
#undef RESA_SELECT_LAUNCH
}

}  // namespace resa
