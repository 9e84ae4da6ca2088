// Query-aware block selection (ReSA summary §3.4.1): group query pooling, the
// Quest upper-bound score of Eq. 4 for every complete block, and top-n
// selection (Eq. 5 count from the caller, ties to the lower block index) with
// the local block always appended.
//
// score_kernel is an HBM stream over the descriptors (2*d bf16 per block and
// kv head): each warp takes groups of kPagesPerWarp pages, every lane loads
// its channels of min and max rows (256-byte coalesced warp loads) for every
// kv head before any arithmetic, then one warp butterfly per (page, head).
//
// select_kernel is one 1024-thread CTA per (sequence, kv head): a radix
// select on order-preserving integer keys (most significant digit first,
// starting at the highest bit where the smallest and largest key differ)
// finds the k-th largest key T, then a ballot compaction writes the blocks
// with key > T plus the lowest-index blocks with key == T in ascending order.
#include "resa_common.cuh"

namespace resa {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kPagesPerWarp = 4;

template <int D>
struct LaneDesc;  // channels held by one lane: D / 32 bf16 of min and of max
template <>
struct LaneDesc<128> {
    using T = uint2;  // 4 bf16
    static constexpr int N = 4;
    __device__ static void unpack(const T &x, float (&f)[4]) {
        f[0] = bf_lo(x.x);
        f[1] = bf_hi(x.x);
        f[2] = bf_lo(x.y);
        f[3] = bf_hi(x.y);
    }
};
template <>
struct LaneDesc<64> {
    using T = uint32_t;  // 2 bf16
    static constexpr int N = 2;
    __device__ static void unpack(const T &x, float (&f)[2]) {
        f[0] = bf_lo(x);
        f[1] = bf_hi(x);
    }
};

// grid (X, batch), block kScoreThreads.
template <int D, int HKV>
__global__ void __launch_bounds__(kScoreThreads)
    score_kernel(const uint16_t *__restrict__ desc, const int32_t *__restrict__ page_table,
                 const int32_t *__restrict__ seq_len, const uint16_t *__restrict__ q,
                 float *__restrict__ scores, int g, int max_pages, int num_pages, uint32_t *err) {
    using LD = LaneDesc<D>;
    constexpr int N = LD::N;
    __shared__ float qbar_s[HKV][D];
    const int b = blockIdx.y;
    const int hq = HKV * g;
    // Group pooling: mean of the g query heads, fp32, head order, then / g.
    for (int e = threadIdx.x; e < HKV * D; e += kScoreThreads) {
        const int h = e / D, j = e % D;
        const uint16_t *col = q + ((size_t)b * hq + h * g) * D + j;
        uint16_t v[kMaxGroup];
#pragma unroll
        for (int r = 0; r < kMaxGroup; ++r) v[r] = r < g ? col[(size_t)r * D] : (uint16_t)0;
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxGroup; ++r)
            if (r < g) s += bf16_bits_to_f32(v[r]);
        qbar_s[h][j] = s / (float)g;
    }
    __syncthreads();
    const int L = seq_len[b];
    if (L < 1 || L > max_pages * kBlock) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        return;
    }
    const int M = (L - 1) / kBlock;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float qv[HKV][N];
#pragma unroll
    for (int h = 0; h < HKV; ++h)
#pragma unroll
        for (int n = 0; n < N; ++n) qv[h][n] = qbar_s[h][lane * N + n];

    const int stride = gridDim.x * kScoreWarps * kPagesPerWarp;
    const typename LD::T *dsc = reinterpret_cast<const typename LD::T *>(desc);
    for (int i0 = (blockIdx.x * kScoreWarps + warp) * kPagesPerWarp; i0 < M; i0 += stride) {
        typename LD::T mn[kPagesPerWarp][HKV], mx[kPagesPerWarp][HKV];
        int pages[kPagesPerWarp];
#pragma unroll
        for (int p = 0; p < kPagesPerWarp; ++p) {
            const int i = i0 + p;
            int page = i < M ? page_table[(size_t)b * max_pages + i] : -1;
            if (i < M && (page < 0 || page >= num_pages)) {
                if (lane == 0) set_error(err, RESA_DEVERR_PAGE);
                page = -1;
            }
            pages[p] = page;
#pragma unroll
            for (int h = 0; h < HKV; ++h) {
                if (page >= 0) {
                    const size_t row = ((size_t)page * HKV + h) * 2;  // min row, then max row
                    mn[p][h] = dsc[(row * D) / N + lane];
                    mx[p][h] = dsc[((row + 1) * D) / N + lane];
                }
            }
        }
#pragma unroll
        for (int p = 0; p < kPagesPerWarp; ++p) {
#pragma unroll
            for (int h = 0; h < HKV; ++h) {
                float s = 0.f;
                if (pages[p] >= 0) {
                    float a[N], c[N];
                    LD::unpack(mn[p][h], a);
                    LD::unpack(mx[p][h], c);
#pragma unroll
                    for (int n = 0; n < N; ++n) s += fmaxf(qv[h][n] * c[n], qv[h][n] * a[n]);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == ((p * HKV + h) & 31) && pages[p] >= 0)
                    scores[((size_t)b * HKV + h) * max_pages + i0 + p] = s;
            }
        }
    }
}

constexpr int kSelectThreads = 1024;
constexpr int kSelectWarps = kSelectThreads / 32;

__device__ __forceinline__ uint32_t order_key(float s) {
    s += 0.0f;  // -0 -> +0: equal scores get equal keys
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// grid (hkv, batch), block kSelectThreads, dynamic smem = key_cap * 4 bytes.
__global__ void __launch_bounds__(kSelectThreads)
    select_kernel(const float *__restrict__ scores, const int32_t *__restrict__ seq_len,
                  const int32_t *__restrict__ topk, int max_topk, int32_t *__restrict__ block_idx,
                  int32_t *__restrict__ block_cnt, int hkv, int max_pages, int key_cap,
                  uint32_t *err) {
    extern __shared__ uint32_t keys_s[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t red_min[kSelectWarps], red_max[kSelectWarps];
    __shared__ uint32_t warp_gt[kSelectWarps], warp_eq[kSelectWarps];
    __shared__ uint32_t sh_digit, sh_above;

    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t *out = block_idx + ((size_t)b * hkv + h) * (max_topk + 1);
    int32_t *cnt = block_cnt + (size_t)b * hkv + h;
    const int L = seq_len[b];
    if (L < 1 || L > max_pages * kBlock) {
        if (tid == 0) {
            set_error(err, RESA_DEVERR_SEQ_LEN);
            *cnt = 0;
        }
        return;
    }
    const int M = (L - 1) / kBlock;
    int k = topk[b];
    k = k < 0 ? 0 : k;
    if (k > max_topk && M > max_topk) {
        if (tid == 0) set_error(err, RESA_DEVERR_TOPK);
        k = max_topk;
    }
    k = min(k, M);
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
    const float *src = scores + ((size_t)b * hkv + h) * max_pages;
    const bool in_smem = M <= key_cap;
    if (in_smem) {
        constexpr int U = 8;  // loads in flight per thread
        for (int i0 = tid; i0 < M; i0 += U * kSelectThreads) {
            float v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * kSelectThreads;
                v[u] = i < M ? src[i] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * kSelectThreads;
                if (i < M) keys_s[i] = order_key(v[u]);
            }
        }
    }
    __syncthreads();
    auto key_at = [&](int i) -> uint32_t { return in_smem ? keys_s[i] : order_key(src[i]); };

    // Smallest and largest key: their common leading bits are every key's.
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int i = tid; i < M; i += kSelectThreads) {
        const uint32_t x = key_at(i);
        kmin = min(kmin, x);
        kmax = max(kmax, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        red_min[warp] = kmin;
        red_max[warp] = kmax;
    }
    __syncthreads();
    kmin = red_min[lane];
    kmax = red_max[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }

    uint32_t prefix, pmask;
    uint32_t remaining = (uint32_t)k;  // keys still to take at or below the current prefix
    int bits_left;
    const uint32_t diff = kmin ^ kmax;
    if (diff == 0) {
        prefix = kmin;
        pmask = 0xffffffffu;
        bits_left = 0;
    } else {
        const int hb = 31 - __clz(diff);
        pmask = hb == 31 ? 0u : ~((1u << (hb + 1)) - 1u);
        prefix = kmin & pmask;
        bits_left = hb + 1;
    }
    while (bits_left > 0) {
        const int width = bits_left < 8 ? bits_left : 8;
        const int shift = bits_left - width;
        const uint32_t nbm = (1u << width) - 1u;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int i = tid; i < M; i += kSelectThreads) {
            const uint32_t x = key_at(i);
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
            const uint32_t above = incl - sum;  // keys in bins above this lane's
            if (above < remaining && remaining <= incl) {
                uint32_t cum = above;
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    if (cum + local[j] >= remaining) {
                        sh_digit = (uint32_t)(lane * 8 + j);
                        sh_above = cum;
                        break;
                    }
                    cum += local[j];
                }
            }
        }
        __syncthreads();
        remaining -= sh_above;
        prefix |= sh_digit << shift;
        pmask |= nbm << shift;
        bits_left = shift;
        __syncthreads();  // sh_digit / hist reused by the next pass
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
        const uint32_t x = i < w1 ? key_at(i) : 0u;
        const bool is_gt = i < w1 && x > T;
        const bool is_eq = i < w1 && x == T;
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
cudaError_t launch_score_d(const Shape &s, const void *desc, const int32_t *page_table,
                           const int32_t *seq_len, const void *q, float *scores, uint32_t *err,
                           cudaStream_t st) {
    const int per_cta = kScoreWarps * kPagesPerWarp;
    dim3 grid((s.max_pages + per_cta - 1) / per_cta, s.batch);
    const uint16_t *dd = (const uint16_t *)desc;
    const uint16_t *qq = (const uint16_t *)q;
#define RESA_SCORE_CASE(H)                                                                       \
    case H:                                                                                      \
        score_kernel<D, H><<<grid, kScoreThreads, 0, st>>>(dd, page_table, seq_len, qq, scores, \
                                                           s.g, s.max_pages, s.num_pages, err); \
        break;
    switch (s.hkv) {
        RESA_SCORE_CASE(1)
        RESA_SCORE_CASE(2)
        RESA_SCORE_CASE(4)
        RESA_SCORE_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef RESA_SCORE_CASE
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score(const Shape &s, const void *desc, const int32_t *page_table,
                         const int32_t *seq_len, const void *q, float *scores, uint32_t *err,
                         cudaStream_t st) {
    if (s.d == 128) return launch_score_d<128>(s, desc, page_table, seq_len, q, scores, err, st);
    if (s.d == 64) return launch_score_d<64>(s, desc, page_table, seq_len, q, scores, err, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_select(const Shape &s, const float *scores, const int32_t *seq_len,
                          const int32_t *topk, int max_topk, int32_t *block_idx,
                          int32_t *block_cnt, uint32_t *err, cudaStream_t st) {
    constexpr int kMaxKeysInSmem = 48 * 1024;  // 192 KB of keys
    const int cap = s.max_pages < kMaxKeysInSmem ? s.max_pages : kMaxKeysInSmem;
    const size_t smem = (size_t)cap * 4;
    static std::atomic<int> done[64];
    cudaError_t e = ensure_smem(select_kernel, kMaxKeysInSmem * 4, done);
    if (e != cudaSuccess) return e;
    dim3 grid(s.hkv, s.batch);
    select_kernel<<<grid, kSelectThreads, smem, st>>>(scores, seq_len, topk, max_topk, block_idx,
                                                      block_cnt, s.hkv, s.max_pages, cap, err);
    return cudaGetLastError();
}

}  // namespace resa
