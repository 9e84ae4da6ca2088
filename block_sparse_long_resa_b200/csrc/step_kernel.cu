// Fused ReSA decode step of one layer in one persistent launch (ReSA summary
// §3.4.1 and §3.4.4; Algorithm 1 inner body): decode-token append, group
// query pooling, block scores (Eq. 4), top-k selection with the local block
// (Eq. 5 guards, ties to the lower block index) and group block-sparse
// split-KV attention (Eq. 2) with its log-sum-exp combine.
//
// Grid (G, units): G CTAs per (sequence, kv head) unit u, one CTA per SM,
// launched cooperatively so the G CTAs of a unit are co-resident.  CTA x owns
// the x-th contiguous range of the unit's complete blocks.
//
//  1. Scoring.  All 12 warps stream the range's descriptors (this head's min
//     and max rows, 4d bytes per block) through per-warp cp.async rings; the
//     order-preserving keys of the fp32 scores stay in shared memory and their
//     top 16 bits feed the unit's histogram in the workspace (aggregated per
//     CTA in a shared-memory hash table first).
//  2. Unit barrier.  Every CTA reads the touched bins and finds the boundary
//     bin d1 that holds the k-th largest key.  Blocks above it are selected
//     for certain ("definite"); blocks in it are candidates, published with a
//     composite key (low 16 key bits, then the complement of the block id, so
//     larger means higher score or, on equal scores, lower block id).  Each
//     CTA also publishes its definite count and the definite blocks beyond its
//     fair share F = ceil((k + 1) / G), then arrives at a second barrier.
//  3. The eight decode warps start at once on the CTA's own definite blocks
//     (at most F), each with a 3-stage K/V ring of 16-byte cp.async copies and
//     swapped m16n8k16 MMAs (attn_common.cuh).
//  4. Meanwhile the four control warps wait for the second barrier, find the
//     exact threshold among the unit's candidates by radix select, and build
//     the residual pool: definite blocks over the fair shares, qualifying
//     candidates, the current block.  Every CTA computes the same pool and
//     takes the slice that fills its share, so all CTAs end with F blocks at
//     most.  They also write the block list (ascending) and its count.
//  5. The decode warps finish with the residual slice; the CTA merges its
//     warps and writes a partial (o / l, log2-sum-exp); the last CTA of the
//     unit to arrive merges the G partials into the output.
//
// The append (K/V of the decode token at position L-1 and the fold of its key
// into the current block's descriptor) is done by a control warp of CTA 0 of
// each unit before it arrives at the second barrier: only the current block
// reads it, and that block is decoded after the barrier.
#include "attn_common.cuh"

namespace resa {
namespace {

constexpr int kDW = kDecodeWarps;         // decode warps
constexpr int kCW = 4;                    // control warps
constexpr int kWarpsAll = kDW + kCW;
constexpr int kThreadsAll = 32 * kWarpsAll;
constexpr int kCtlThreads = 32 * kCW;
constexpr int kKvStages = 3;
constexpr int kDescSlots = 16;            // 512-byte descriptor slots per warp in flight
constexpr int kHash = 1024;               // per-CTA digit histogram slots
constexpr uint32_t kHashEmpty = 0xffffffffu;
constexpr uint32_t kSkip = 0xffffffffu;   // work item without data (bad page id)
constexpr int kModeAll = 0, kModeNone = 1, kModeMid = 2;

template <int D>
struct StepSmem {
    static constexpr int kTileBytes = kBlock * D * 2;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = kDW * kKvStages * kStageBytes;
    static constexpr int kDescBytes = 4 * D;  // min and max rows of one (block, head)
    static_assert(kWarpsAll * kDescSlots * 512 <= kRingBytes, "descriptor rings fit the K/V rings");
    static_assert(kDW * kMaxGroup * (D + 2) * 4 <= kRingBytes, "warp states fit the rings");
    static constexpr int kKeysOff = kRingBytes;
    static constexpr int kPagesOff = kKeysOff + kStepMaxBlocks * 4;
    static constexpr int kDefOff = kPagesOff + kStepMaxBlocks * 4;
    static constexpr int kResCap = kStepMaxBlocks + 64;
    static constexpr int kResOff = kDefOff + kStepMaxBlocks * 2;
    static constexpr int kCandOff = kResOff + kResCap * 4;
    static constexpr int kCandBytes = kStepCandCap * 4 > 2 * kHash * 4 ? kStepCandCap * 4 : 2 * kHash * 4;
    static constexpr int kBytes = kCandOff + kCandBytes + 1024;  // + base alignment
};

struct StepArgs {
    uint8_t *k_cache, *v_cache;
    uint16_t *desc;
    const int32_t *page_table, *seq_len, *topk;
    const uint16_t *q;
    const uint4 *k_new, *v_new;
    int32_t *block_idx, *block_cnt;
    float *out, *lse;
    uint32_t *hist, *hist_range;
    unsigned long long *bars;
    uint32_t *tickets;
    int2 *counts;
    int32_t *ovf;
    uint32_t *cand;
    float *part_o, *part_lse;
    uint32_t *err;
    int hkv, g, max_pages, num_pages, max_topk;
    float scale_log2;
};

// ---------------------------------------------------------------------------
// Unit barrier: one 64-bit word per barrier holds (generation << 32) |
// arrivals; the last arriver's single add returns the count to zero and bumps
// the generation.  Arrive and wait are split so that a CTA can work between
// them.  The caller fences its writes before arriving.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t unit_bar_arrive(unsigned long long *bar, uint32_t n) {
    const unsigned long long old = atomicAdd(bar, 1ull);
    if ((uint32_t)old == n - 1) atomicAdd(bar, (1ull << 32) - n);
    return (uint32_t)(old >> 32);
}
__device__ __forceinline__ bool unit_bar_wait(const unsigned long long *bar, uint32_t gen) {
    for (uint32_t polls = 0;; ++polls) {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(bar) : "memory");
        if ((uint32_t)(v >> 32) != gen) return true;
        if (polls > (1u << 22)) return false;  // each poll is an L2 round trip
    }
}

__device__ __forceinline__ void ctl_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(kCtlThreads) : "memory");
}

// Exclusive scan of one value per thread over the whole CTA, in thread order.
__device__ __forceinline__ uint32_t cta_scan(uint32_t v, uint32_t *tmp, uint32_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarpsAll; ++w) {
        const uint32_t t = tmp[w];
        before += w < warp ? t : 0u;
        tot += t;
    }
    total = tot;
    __syncthreads();
    return before + incl - v;
}

// The same over the control warps (ct = thread index within them).
__device__ __forceinline__ uint32_t ctl_scan(uint32_t v, int ct, uint32_t *tmp, uint32_t &total) {
    const int lane = ct & 31, w = ct >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) tmp[w] = incl;
    ctl_sync();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kCW; ++i) {
        const uint32_t t = tmp[i];
        before += i < w ? t : 0u;
        tot += t;
    }
    total = tot;
    ctl_sync();
    return before + incl - v;
}

// The kth largest (1-based) of n distinct 32-bit keys key(0 .. n-1), by radix
// select over four 8-bit digits, most significant first, on the control warps.
template <typename KeyFn>
__device__ uint32_t ctl_select_kth(KeyFn key, int n, uint32_t kth, int ct, uint32_t *rh,
                                   uint32_t *rsh) {
    uint32_t prefix = 0, pmask = 0, remaining = kth;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = ct; i < 256; i += kCtlThreads) rh[i] = 0;
        ctl_sync();
        for (int i = ct; i < n; i += kCtlThreads) {
            const uint32_t x = key(i);
            if ((x & pmask) == prefix) atomicAdd(&rh[(x >> shift) & 255u], 1u);
        }
        ctl_sync();
        if (ct < 32) {
            // lane l holds digits 255 - 8l - j, j = 0..7 (descending)
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = rh[255 - 8 * ct - j];
                sum += c[j];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
                if (ct >= o) incl += t;
            }
            uint32_t cum = incl - sum;  // keys in higher digits than this lane's
            if (cum < remaining && remaining <= incl) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (cum < remaining && remaining <= cum + c[j]) {
                        rsh[0] = 255u - 8u * ct - j;
                        rsh[1] = cum;
                    }
                    cum += c[j];
                }
            }
        }
        ctl_sync();
        remaining -= rsh[1];
        prefix |= rsh[0] << shift;
        pmask |= 255u << shift;
    }
    return prefix;
}

// Largest i in [0, n) with a[i] <= v (a ascending, a[0] <= v).
__device__ __forceinline__ int upper_index(const int *a, int n, int v) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= v) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ uint32_t pack_item(int page, int ntok) {
    return ((uint32_t)page << 4) | (uint32_t)(ntok - 1);
}

// Indices of the small shared values.
enum {
    kVD1 = 0, kVAbove, kVDlo, kVDhi, kVHistOk, kVNd, kVNc, kVNres, kVOk, kVOk2, kVLast,
    kVOV, kVNC, kVAB, kVSpareBefore, kVDefBefore, kVQBefore, kVLo, kVHi, kVCount
};

template <int D>
__global__ void __launch_bounds__(kThreadsAll, 1) decode_step_kernel(const StepArgs a) {
    using SM = StepSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *ring = smem;
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + SM::kKeysOff);
    int32_t *pages = reinterpret_cast<int32_t *>(smem + SM::kPagesOff);
    uint16_t *own_def = reinterpret_cast<uint16_t *>(smem + SM::kDefOff);
    uint32_t *res_item = reinterpret_cast<uint32_t *>(smem + SM::kResOff);
    uint32_t *cand_s = reinterpret_cast<uint32_t *>(smem + SM::kCandOff);
    uint32_t *hkey = cand_s, *hcnt = cand_s + kHash;  // scoring phase only

    __shared__ float qbar_s[D];
    __shared__ __align__(8) uint64_t res_bar;
    __shared__ int s_coff[kNumSms + 1], s_ovoff[kNumSms + 1];
    __shared__ uint32_t s_rh[256];
    __shared__ uint32_t s_scan[kWarpsAll];
    __shared__ uint32_t s_rsh[2];
    __shared__ int s_v[kVCount];
    __shared__ float s_lse[kMaxGroup];

    pdl_launch_next();
    const int x = blockIdx.x, G = gridDim.x, u = blockIdx.y;
    const int hkv = a.hkv, g = a.g;
    const int b = u / hkv, h = u % hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cta = u * G + x;
    const int L = a.seq_len[b];
    const bool seq_ok = L >= 1 && L <= a.max_pages * kBlock;
    const int M = seq_ok ? (L - 1) / kBlock : 0;
    int kq = a.topk[b];
    kq = kq < 0 ? 0 : kq;
    bool topk_err = false;
    if (kq > a.max_topk && M > a.max_topk) {
        topk_err = true;
        kq = a.max_topk;
    }
    int keff = min(kq, M);
    int mode = keff == M ? kModeAll : keff == 0 ? kModeNone : kModeMid;
    const int per = (M + G - 1) / G;
    const int p0 = min(M, x * per);
    const int nmine = min(min(M, p0 + per) - p0, kStepMaxBlocks);  // the host keeps per <= cap
    const size_t prow = (size_t)b * a.max_pages;
    const size_t cap_base = (size_t)cta * kStepMaxBlocks;

    // ---- prologue: inputs of the call only (before the dependency wait) ----
    for (int i = tid; i < nmine; i += kThreadsAll) pages[i] = a.page_table[prow + p0 + i];
    {
        const uint16_t *qh = a.q + ((size_t)b * hkv * g + (size_t)h * g) * D;
        for (int j = tid; j < D; j += kThreadsAll) {
            float s = 0.f;
            for (int r = 0; r < g; ++r) s += bf16_bits_to_f32(qh[(size_t)r * D + j]);
            qbar_s[j] = s / (float)g;
        }
    }
    for (int i = tid; i < kHash; i += kThreadsAll) {
        hkey[i] = kHashEmpty;
        hcnt[i] = 0;
    }
    if (tid == 0) {
        mbar_init(&res_bar, 1);
        fence_mbar_init();
        s_v[kVOk] = 1;
        s_v[kVOk2] = 1;
        s_v[kVLo] = 0x7fffffff;
        s_v[kVHi] = -1;
        s_v[kVD1] = 0;
        s_v[kVAbove] = 0;
        s_v[kVHistOk] = 1;
    }
    // Q^T fragments for the decode warps: head lane/4 (zero beyond g),
    // channels 2*(lane%4)+{0,1} (+8) of each 16-channel slice.
    uint32_t qb[D / 16][1][2];
    {
        const uint16_t *base = a.q + ((size_t)b * hkv * g + (size_t)h * g) * D;
        const int head = lane >> 2, c = 2 * (lane & 3);
        const uint16_t *row = head < g ? base + (size_t)head * D : nullptr;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qb[ks][0][0] = row ? *reinterpret_cast<const uint32_t *>(row + ks * 16 + c) : 0u;
            qb[ks][0][1] = row ? *reinterpret_cast<const uint32_t *>(row + ks * 16 + c + 8) : 0u;
        }
    }
    const bool appender = x == 0 && warp == kWarpsAll - 1 && seq_ok;
    const int app_page = appender ? a.page_table[prow + (L - 1) / kBlock] : -1;
    __syncthreads();
    pdl_wait();  // descriptors and K/V may be written by the preceding kernels

    // ---- 1. scoring ----
    const bool need_hist = mode == kModeMid;
    {
        constexpr int LPP = D / 4;     // lanes per block, 4 channels each
        constexpr int PPI = 32 / LPP;  // blocks per warp iteration
        const int sub = lane / LPP, c4 = lane % LPP;
        const int ngroups = (nmine + PPI - 1) / PPI;
        const int nmy = warp < ngroups ? (ngroups - warp + kWarpsAll - 1) / kWarpsAll : 0;
        uint8_t *wring = ring + (size_t)warp * kDescSlots * 512;
        auto blk_of = [&](int it) { return (warp + kWarpsAll * it) * PPI + sub; };
        auto issue = [&](int it) {
            if (it < nmy) {
                const int pi = blk_of(it);
                if (pi < nmine) {
                    const int pg = pages[pi];
                    if (pg >= 0 && pg < a.num_pages) {
                        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.desc) +
                                             ((size_t)pg * hkv + h) * SM::kDescBytes;
                        cp_async16(wring + (size_t)(it % kDescSlots) * 512 + lane * 16, src + c4 * 16);
                    }
                }
            }
            cp_async_commit();
        };
#pragma unroll
        for (int it = 0; it < kDescSlots - 1; ++it) issue(it);
        float qv[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) qv[n] = qbar_s[4 * c4 + n];
        const uint32_t sel0 = upper_bound_selector(qv[0], qv[1]);
        const uint32_t sel1 = upper_bound_selector(qv[2], qv[3]);
        int lo = 0x7fffffff, hi = -1;  // digits that bypassed the hash table
        for (int it = 0; it < nmy; ++it) {
            issue(it + kDescSlots - 1);
            cp_async_wait<kDescSlots - 1>();
            __syncwarp();
            const uint8_t *pg = wring + (size_t)(it % kDescSlots) * 512 + sub * SM::kDescBytes;
            const uint2 mn = *reinterpret_cast<const uint2 *>(pg + 8 * c4);
            const uint2 mx = *reinterpret_cast<const uint2 *>(pg + 2 * D + 8 * c4);
            __syncwarp();  // the slot is refilled by the next issue
            const uint32_t w0 = __byte_perm(mn.x, mx.x, sel0);
            const uint32_t w1 = __byte_perm(mn.y, mx.y, sel1);
            float sum = __fmul_rn(qv[0], __uint_as_float(w0 << 16));
            sum = __fadd_rn(sum, __fmul_rn(qv[1], __uint_as_float(w0 & 0xffff0000u)));
            sum = __fadd_rn(sum, __fmul_rn(qv[2], __uint_as_float(w1 << 16)));
            sum = __fadd_rn(sum, __fmul_rn(qv[3], __uint_as_float(w1 & 0xffff0000u)));
#pragma unroll
            for (int o = LPP / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const int pi = blk_of(it);
            if (c4 == 0 && pi < nmine) {
                const int pgid = pages[pi];
                const bool ok = pgid >= 0 && pgid < a.num_pages;
                if (!ok) set_error(a.err, RESA_DEVERR_PAGE);
                const uint32_t key = ok ? order_key(sum) : 0u;
                keys[pi] = key;
                if (need_hist) {
                    const uint32_t digit = key >> 16;
                    uint32_t slot = (digit * 0x9E3779B1u) >> 22;  // 10 bits
                    bool placed = false;
                    for (int probe = 0; probe < 64; ++probe) {
                        const uint32_t old = atomicCAS(&hkey[slot], kHashEmpty, digit);
                        if (old == kHashEmpty || old == digit) {
                            atomicAdd(&hcnt[slot], 1u);
                            placed = true;
                            break;
                        }
                        slot = (slot + 1) & (kHash - 1);
                    }
                    if (!placed) {
                        atomicAdd(&a.hist[(size_t)u * kHistBins + digit], 1u);
                        lo = min(lo, (int)digit);
                        hi = max(hi, (int)digit);
                    }
                }
            }
        }
        cp_async_wait<0>();
        __syncthreads();
        if (need_hist) {
            for (int i = tid; i < kHash; i += kThreadsAll) {
                const uint32_t k = hkey[i];
                if (k != kHashEmpty) {
                    atomicAdd(&a.hist[(size_t)u * kHistBins + k], hcnt[i]);
                    lo = min(lo, (int)k);
                    hi = max(hi, (int)k);
                }
            }
            if (hi >= 0) {
                atomicMin(&s_v[kVLo], lo);
                atomicMax(&s_v[kVHi], hi);
            }
            __syncthreads();
            if (tid == 0 && s_v[kVHi] >= 0) {
                atomicMax(&a.hist_range[2 * u], (uint32_t)(kHistBins - s_v[kVLo]));  // 0 = untouched
                atomicMax(&a.hist_range[2 * u + 1], (uint32_t)(s_v[kVHi] + 1));
            }
        }
    }
    __threadfence();
    __syncthreads();

    // ---- 2. boundary bin, own lists, second barrier ----
    if (G > 1 && need_hist) {
        if (tid == 0) {
            const uint32_t gen = unit_bar_arrive(&a.bars[2 * u], G);
            s_v[kVOk] = unit_bar_wait(&a.bars[2 * u], gen) ? 1 : 0;
        }
        __syncthreads();
        if (!s_v[kVOk]) {
            if (tid == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
            return;
        }
        __threadfence();
    }
    if (need_hist) {
        const uint32_t emin = __ldcg(&a.hist_range[2 * u]), emax = __ldcg(&a.hist_range[2 * u + 1]);
        const int dlo = kHistBins - (int)emin, dhi = (int)emax - 1;
        const int nb = dhi >= dlo ? dhi - dlo + 1 : 0;
        const uint32_t *hb = a.hist + (size_t)u * kHistBins;
        const int chunk = (nb + kThreadsAll - 1) / kThreadsAll;
        const int top = dhi - tid * chunk, bot = max(dlo, top - chunk + 1);
        constexpr int kBinRegs = 8;
        uint32_t binc[kBinRegs];
        uint32_t loc = 0;
        if (chunk <= kBinRegs) {
#pragma unroll
            for (int j = 0; j < kBinRegs; ++j) {
                binc[j] = (j < chunk && top - j >= bot) ? __ldcg(&hb[top - j]) : 0u;
                loc += binc[j];
            }
        } else {
            for (int d = top; d >= bot; --d) loc += __ldcg(&hb[d]);
        }
        uint32_t total;
        const uint32_t above_me = cta_scan(loc, s_scan, total);
        if (above_me < (uint32_t)keff && (uint32_t)keff <= above_me + loc) {
            uint32_t cum = above_me;
            if (chunk <= kBinRegs) {
#pragma unroll
                for (int j = 0; j < kBinRegs; ++j) {
                    if (j < chunk && top - j >= bot && cum < (uint32_t)keff && cum + binc[j] >= (uint32_t)keff) {
                        s_v[kVD1] = top - j;
                        s_v[kVAbove] = (int)cum;
                    }
                    cum += binc[j];
                }
            } else {
                for (int d = top; d >= bot; --d) {
                    const uint32_t c = __ldcg(&hb[d]);
                    if (cum + c >= (uint32_t)keff) {
                        s_v[kVD1] = d;
                        s_v[kVAbove] = (int)cum;
                        break;
                    }
                    cum += c;
                }
            }
        }
        if (tid == 0) {
            s_v[kVDlo] = dlo;
            s_v[kVDhi] = dhi;
            s_v[kVHistOk] = total == (uint32_t)M ? 1 : 0;
        }
        __syncthreads();
        if (!s_v[kVHistOk]) {
            // The histogram was not clean at entry (an earlier call gave up
            // mid-way): every CTA of the unit sees the same sums and selects
            // no complete block.
            if (tid == 0 && x == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
            mode = kModeNone;
            keff = 0;
        }
    }
    const int W = seq_ok ? keff + 1 : 0;
    const int F = (W + G - 1) / G;
    const uint32_t d1 = (uint32_t)s_v[kVD1];
    {
        // Classify the CTA's blocks: definite (ascending local ids into
        // own_def) and candidates (composite keys into the workspace).
        constexpr int R = (kStepMaxBlocks + kThreadsAll - 1) / kThreadsAll;
        const int i0 = tid * R;
        uint32_t nd_t = 0, nc_t = 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int i = i0 + r;
            if (i < nmine) {
                const uint32_t dg = keys[i] >> 16;
                nd_t += mode == kModeAll || (mode == kModeMid && dg > d1);
                nc_t += mode == kModeMid && dg == d1;
            }
        }
        uint32_t tot;
        const uint32_t ex = cta_scan(nd_t | (nc_t << 16), s_scan, tot);
        uint32_t od = ex & 0xffffu, oc = ex >> 16;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int i = i0 + r;
            if (i < nmine) {
                const uint32_t key = keys[i];
                const uint32_t dg = key >> 16;
                if (mode == kModeAll || (mode == kModeMid && dg > d1)) {
                    own_def[od++] = (uint16_t)i;
                } else if (mode == kModeMid && dg == d1) {
                    a.cand[cap_base + oc++] = ((key & 0xffffu) << 16) | (0xffffu - (uint32_t)(p0 + i));
                }
            }
        }
        if (tid == 0) {
            s_v[kVNd] = (int)(tot & 0xffffu);
            s_v[kVNc] = (int)(tot >> 16);
        }
        __syncthreads();
        const int nd = s_v[kVNd], kept = min(nd, F);
        for (int j = kept + tid; j < nd; j += kThreadsAll) a.ovf[cap_base + (j - kept)] = p0 + own_def[j];
        if (tid == 0) a.counts[cta] = make_int2(nd, s_v[kVNc]);
    }
    __threadfence();
    __syncthreads();
    const int nd = s_v[kVNd];
    const int kept = min(nd, F);

    if (warp < kDW) {
        // ---- 3 / 5. decode warps ----
        WarpState<D, 1> st;
        st.init();
        bool ready = false;
        int nres = 0;
        auto get_item = [&](int j, uint32_t &item) -> bool {
            if (j < kept) {
                const int pg = pages[own_def[j]];
                item = (pg >= 0 && pg < a.num_pages) ? pack_item(pg, kBlock) : kSkip;
                return true;
            }
            if (!ready) {
                ready = true;
                if (mbar_wait_bounded(&res_bar, 0)) {
                    nres = s_v[kVNres];
                } else {
                    if (lane == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
                    nres = 0;
                }
            }
            if (j - kept < nres) {
                item = res_item[j - kept];
                return true;
            }
            return false;
        };
        uint8_t *wr = ring + (size_t)warp * kKvStages * SM::kStageBytes;
        constexpr int kPerLane = SM::kTileBytes / 16 / 32;
        auto issue = [&](int t) {
            uint32_t item;
            if (get_item(warp + kDW * t, item) && item != kSkip) {
                const size_t tile = ((size_t)(item >> 4) * hkv + h) * SM::kTileBytes;
                uint8_t *stg = wr + (size_t)(t % kKvStages) * SM::kStageBytes;
#pragma unroll
                for (int k = 0; k < kPerLane; ++k) {
                    const uint32_t qc = lane + 32 * k;
                    const uint32_t so = swz128(qc >> 3, qc & 7);
                    cp_async16(stg + so, a.k_cache + tile + qc * 16);
                    cp_async16(stg + SM::kTileBytes + so, a.v_cache + tile + qc * 16);
                }
            }
            cp_async_commit();
        };
#pragma unroll
        for (int t = 0; t < kKvStages - 1; ++t) issue(t);
        for (int t = 0;; ++t) {
            uint32_t item;
            if (!get_item(warp + kDW * t, item)) break;
            issue(t + kKvStages - 1);
            cp_async_wait<kKvStages - 1>();
            __syncwarp();
            if (item != kSkip) {
                const uint32_t ks = smem_u32(wr + (size_t)(t % kKvStages) * SM::kStageBytes);
                attend_block_swapped<D, 1>(st, qb, ks, ks + SM::kTileBytes, (int)(item & 15u) + 1,
                                           a.scale_log2, lane);
            }
            __syncwarp();
        }
        cp_async_wait<0>();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            st.l[0][k] += __shfl_xor_sync(0xffffffffu, st.l[0][k], 4);
            st.l[0][k] += __shfl_xor_sync(0xffffffffu, st.l[0][k], 8);
            st.l[0][k] += __shfl_xor_sync(0xffffffffu, st.l[0][k], 16);
        }
        // every decode warp's ring is drained before the states overwrite them
        asm volatile("bar.sync 2, %0;" ::"r"(kDW * 32) : "memory");
        float *mw = reinterpret_cast<float *>(ring);   // [kDW][16] row max
        float *lw = mw + kDW * kMaxGroup;              // [kDW][16] row sum
        float *ow = lw + kDW * kMaxGroup;              // [kDW][16][D]
        const int hb = 2 * (lane & 3), d0 = lane >> 2;
        if (lane < 4) {
            mw[warp * kMaxGroup + hb] = st.m[0][0];
            mw[warp * kMaxGroup + hb + 1] = st.m[0][1];
            lw[warp * kMaxGroup + hb] = st.l[0][0];
            lw[warp * kMaxGroup + hb + 1] = st.l[0][1];
        }
#pragma unroll
        for (int t = 0; t < D / 16; ++t) {
            float *o0 = ow + ((size_t)warp * kMaxGroup + hb) * D + t * 16 + d0;
            o0[0] = st.o[t][0][0];
            o0[D] = st.o[t][0][1];
            o0[8] = st.o[t][0][2];
            o0[D + 8] = st.o[t][0][3];
        }
    } else {
        // ---- 4. control warps ----
        const int ct = tid - kDW * 32;
        if (appender) {
            // decode-token append: K/V at position L-1, key folded into the
            // current block's descriptor (a new block starts from the key)
            const int slot = (L - 1) % kBlock;
            if (app_page < 0 || app_page >= a.num_pages) {
                if (lane == 0) set_error(a.err, RESA_DEVERR_PAGE);
            } else {
                constexpr int CPR = D / 8;
                uint4 *K4 = reinterpret_cast<uint4 *>(a.k_cache);
                uint4 *V4 = reinterpret_cast<uint4 *>(a.v_cache);
                uint4 *D4 = reinterpret_cast<uint4 *>(a.desc);
                for (int e = lane; e < CPR; e += 32) {
                    const uint4 kx = a.k_new[((size_t)b * hkv + h) * CPR + e];
                    const uint4 vx = a.v_new[((size_t)b * hkv + h) * CPR + e];
                    const size_t o = (((size_t)app_page * hkv + h) * kBlock + slot) * CPR + e;
                    K4[o] = kx;
                    V4[o] = vx;
                    uint4 *pmn = &D4[(((size_t)app_page * hkv + h) * 2) * CPR + e];
                    uint4 *pmx = pmn + CPR;
                    if (slot == 0) {
                        *pmn = kx;
                        *pmx = kx;
                    } else {
                        Bf16x8 mn = unpack8(*pmn), mx = unpack8(*pmx);
                        fold8(mn, mx, unpack8(kx));
                        *pmn = pack8(mn);
                        *pmx = pack8(mx);
                    }
                }
                __threadfence();
            }
        }
        ctl_sync();
        if (G > 1) {
            if (ct == 0) {
                __threadfence();
                const uint32_t gen = unit_bar_arrive(&a.bars[2 * u + 1], G);
                s_v[kVOk2] = unit_bar_wait(&a.bars[2 * u + 1], gen) ? 1 : 0;
            }
            ctl_sync();
            __threadfence();
        }
        const bool ok2 = s_v[kVOk2] != 0;
        if (!ok2 && ct == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
        // Per-CTA counts of the unit -> prefix sums (one warp, <= 5 CTAs per lane).
        if (ct < 32) {
            const int PL = (G + 31) / 32;
            const int i0 = ct * PL, i1 = min(G, i0 + PL);
            int ndv[5], ncv[5];
            int s_ov = 0, s_sp = 0, s_nc = 0, s_nd = 0;
#pragma unroll
            for (int r = 0; r < 5; ++r) {
                const int i = i0 + r;
                int2 c = make_int2(0, 0);
                if (ok2 && r < PL && i < i1) c = __ldcg(&a.counts[u * G + i]);
                ndv[r] = c.x;
                ncv[r] = c.y;
                if (r < PL && i < i1) {
                    const int kp = min(c.x, F);
                    s_ov += c.x - kp;
                    s_sp += F - kp;
                    s_nc += c.y;
                    s_nd += c.x;
                }
            }
            int e_ov = s_ov, e_sp = s_sp, e_nc = s_nc, e_nd = s_nd;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int a1 = __shfl_up_sync(0xffffffffu, e_ov, o);
                const int a2 = __shfl_up_sync(0xffffffffu, e_sp, o);
                const int a3 = __shfl_up_sync(0xffffffffu, e_nc, o);
                const int a4 = __shfl_up_sync(0xffffffffu, e_nd, o);
                if (ct >= o) {
                    e_ov += a1;
                    e_sp += a2;
                    e_nc += a3;
                    e_nd += a4;
                }
            }
            int b_ov = e_ov - s_ov, b_sp = e_sp - s_sp, b_nc = e_nc - s_nc, b_nd = e_nd - s_nd;
#pragma unroll
            for (int r = 0; r < 5; ++r) {
                const int i = i0 + r;
                if (r < PL && i < i1) {
                    if (i == x) {
                        s_v[kVSpareBefore] = b_sp;
                        s_v[kVDefBefore] = b_nd;
                    }
                    s_ovoff[i] = b_ov;
                    s_coff[i] = b_nc;
                    const int kp = min(ndv[r], F);
                    b_ov += ndv[r] - kp;
                    b_sp += F - kp;
                    b_nc += ncv[r];
                    b_nd += ndv[r];
                }
            }
            if (ct == 31) {
                s_ovoff[G] = e_ov;
                s_coff[G] = e_nc;
                s_v[kVOV] = e_ov;
                s_v[kVNC] = e_nc;
                s_v[kVAB] = e_nd;
            }
        }
        ctl_sync();
        const int OV = s_v[kVOV], NC = s_v[kVNC], AB = s_v[kVAB];
        int rem = mode == kModeMid ? keff - AB : 0;
        if (rem < 0 || rem > NC) {  // cannot happen with consistent counts
            if (ct == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
            rem = max(0, min(rem, NC));
        }
        const uint32_t *gcand = a.cand + (size_t)u * G * kStepMaxBlocks;
        auto gkey = [&](int i) -> uint32_t {
            const int src = upper_index(s_coff, G, i);
            return __ldcg(&gcand[(size_t)src * kStepMaxBlocks + (i - s_coff[src])]);
        };
        const bool in_smem = NC <= kStepCandCap;
        uint32_t tau = 0xffffffffu;
        if (rem > 0) {
            if (in_smem) {
                for (int i0 = ct; i0 < NC; i0 += 4 * kCtlThreads) {
                    uint32_t v[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int i = i0 + r * kCtlThreads;
                        v[r] = i < NC ? gkey(i) : 0u;
                    }
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int i = i0 + r * kCtlThreads;
                        if (i < NC) cand_s[i] = v[r];
                    }
                }
                ctl_sync();
                tau = ctl_select_kth([&](int i) { return cand_s[i]; }, NC, (uint32_t)rem, ct, s_rh, s_rsh);
            } else {
                tau = ctl_select_kth(gkey, NC, (uint32_t)rem, ct, s_rh, s_rsh);
            }
        }
        auto ckey = [&](int i) -> uint32_t { return in_smem ? cand_s[i] : gkey(i); };
        // Residual pool: [overflow definite blocks, CTA order][qualifying
        // candidates, candidate order][current block]; this CTA's slice.
        const int Q = rem;
        const int Rpool = seq_ok ? OV + Q + 1 : 0;
        const int S0 = s_v[kVSpareBefore];
        const int myspare = F - kept;
        const int S1 = min(Rpool, S0 + myspare);
        const int nres = max(0, S1 - S0);
        auto page_item = [&](int blk, int ntok) -> uint32_t {
            const int pg = a.page_table[prow + blk];
            if (pg < 0 || pg >= a.num_pages) {
                set_error(a.err, RESA_DEVERR_PAGE);
                return kSkip;
            }
            return pack_item(pg, ntok);
        };
        for (int pos = S0 + ct; pos < min(S1, OV); pos += kCtlThreads) {
            const int src = upper_index(s_ovoff, G, pos);
            const int blk = __ldcg(&a.ovf[((size_t)u * G + src) * kStepMaxBlocks + (pos - s_ovoff[src])]);
            res_item[pos - S0] = page_item(blk, kBlock);
        }
        if (seq_ok && ct == 0 && Rpool - 1 >= S0 && Rpool - 1 < S1)
            res_item[Rpool - 1 - S0] = page_item(M, L - M * kBlock);
        uint32_t qbefore_add = 0;
        if (Q > 0) {
            // qualifying candidates in array order: chunked scan of the flags
            const int CH = (NC + kCtlThreads - 1) / kCtlThreads;
            const int c0 = ct * CH, c1 = min(NC, c0 + CH);
            uint32_t nq = 0;
            for (int i = c0; i < c1; ++i) nq += ckey(i) >= tau;
            uint32_t qtot;
            uint32_t qp = ctl_scan(nq, ct, s_scan, qtot);
            const int myc = s_coff[x];
            for (int i = c0; i < c1; ++i) {
                const uint32_t kk = ckey(i);
                if (kk >= tau) {
                    if (i < myc) ++qbefore_add;
                    const int pos = OV + (int)qp;
                    if (pos >= S0 && pos < S1) res_item[pos - S0] = page_item(0xffff - (int)(kk & 0xffffu), kBlock);
                    ++qp;
                }
            }
        }
        if (ct == 0) s_v[kVQBefore] = 0;
        ctl_sync();
        if (qbefore_add) atomicAdd(&s_v[kVQBefore], (int)qbefore_add);
        if (ct == 0) s_v[kVNres] = ok2 ? nres : 0;
        ctl_sync();
        if (ct == 0) mbar_arrive(&res_bar);  // the decode warps may take the residual slice

        // Block list (ascending) and count.
        const int off = s_v[kVDefBefore] + s_v[kVQBefore];
        int32_t *list = a.block_idx + (size_t)u * (a.max_topk + 1);
        {
            constexpr int R2 = (kStepMaxBlocks + kCtlThreads - 1) / kCtlThreads;
            const int i0 = ct * R2;
            auto sel = [&](int i) -> bool {
                if (mode == kModeAll) return true;
                if (mode != kModeMid) return false;
                const uint32_t key = keys[i];
                const uint32_t dg = key >> 16;
                if (dg != d1) return dg > d1;
                return Q > 0 && (((key & 0xffffu) << 16) | (0xffffu - (uint32_t)(p0 + i))) >= tau;
            };
            uint32_t ns = 0;
            for (int r = 0; r < R2; ++r) {
                const int i = i0 + r;
                if (i < nmine && sel(i)) ++ns;
            }
            uint32_t tot;
            uint32_t pos = ctl_scan(ns, ct, s_scan, tot) + (uint32_t)off;
            if (ok2)
                for (int r = 0; r < R2; ++r) {
                    const int i = i0 + r;
                    if (i < nmine && sel(i) && pos < (uint32_t)keff) list[pos++] = p0 + i;
                }
        }
        if (x == 0 && ct == 0) {
            if (seq_ok) {
                list[keff] = M;
                a.block_cnt[u] = keff + 1;
            } else {
                a.block_cnt[u] = 0;
                set_error(a.err, RESA_DEVERR_SEQ_LEN);
            }
            if (topk_err) set_error(a.err, RESA_DEVERR_TOPK);
        }
        if (x == 0 && need_hist) {
            // every CTA of the unit read the histogram before the second
            // barrier: leave it clear for the next call
            uint32_t *hb = a.hist + (size_t)u * kHistBins;
            for (int d = s_v[kVDlo] + ct; d <= s_v[kVDhi]; d += kCtlThreads) hb[d] = 0;
            if (ct == 0) {
                a.hist_range[2 * u] = 0;
                a.hist_range[2 * u + 1] = 0;
            }
        }
    }
    __syncthreads();  // warp states are in shared memory

    // ---- 5. merge the warps, then the unit's CTAs ----
    const float kLn2 = 0.6931471805599453f;
    {
        const float *mw = reinterpret_cast<const float *>(ring);
        const float *lw = mw + kDW * kMaxGroup;
        const float *ow = lw + kDW * kMaxGroup;
        float *po = a.part_o + (size_t)cta * kStepMaxGroup * D;
        float *pl = a.part_lse + (size_t)cta * kMaxGroup;
        const int hq = hkv * g;
        for (int e = tid; e < g * D; e += kThreadsAll) {
            const int r = e / D, c = e % D;
            float mstar = -INFINITY;
#pragma unroll
            for (int w = 0; w < kDW; ++w) mstar = fmaxf(mstar, mw[w * kMaxGroup + r]);
            float lsum = 0.f, o = 0.f;
            if (mstar != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kDW; ++w) {
                    const float sc = exp2f(mw[w * kMaxGroup + r] - mstar);
                    lsum += lw[w * kMaxGroup + r] * sc;
                    o += ow[((size_t)w * kMaxGroup + r) * D + c] * sc;
                }
            }
            const float lse2 = lsum > 0.f ? mstar + log2f(lsum) : -INFINITY;
            const float on = lsum > 0.f ? o / lsum : 0.f;
            if (G == 1) {
                const size_t orow = (size_t)b * hq + (size_t)h * g + r;
                a.out[orow * D + c] = on;
                if (a.lse && c == 0) a.lse[orow] = lse2 * kLn2;
            } else {
                po[(size_t)r * D + c] = on;
                if (c == 0) pl[r] = lse2;
            }
        }
    }
    if (G == 1) return;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t t = atomicAdd(&a.tickets[u], 1u);
        s_v[kVLast] = t == (uint32_t)(G - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!s_v[kVLast]) return;
    __threadfence();
    // The last CTA of the unit: weights from the G partial log-sum-exps, then
    // the weighted sum of the partial outputs, pulled into shared memory with
    // cp.async in chunks of as many partials as the rings hold.
    float *wts = reinterpret_cast<float *>(ring);  // [G][kStepMaxGroup]
    const size_t wbytes = ((size_t)G * kStepMaxGroup * 4 + 127) / 128 * 128;
    const float *ul = a.part_lse + (size_t)u * G * kMaxGroup;
    for (int i = tid; i < G * g; i += kThreadsAll) {
        const int s = i / g, r = i % g;
        wts[s * kStepMaxGroup + r] = __ldcg(&ul[s * kMaxGroup + r]);
    }
    __syncthreads();
    for (int r = warp; r < g; r += kWarpsAll) {
        float mstar = -INFINITY;
        for (int s = lane; s < G; s += 32) mstar = fmaxf(mstar, wts[s * kStepMaxGroup + r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
        float sum = 0.f;
        if (mstar != -INFINITY)
            for (int s = lane; s < G; s += 32) sum += exp2f(wts[s * kStepMaxGroup + r] - mstar);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        __syncwarp();
        for (int s = lane; s < G; s += 32)
            wts[s * kStepMaxGroup + r] = sum > 0.f ? exp2f(wts[s * kStepMaxGroup + r] - mstar) / sum : 0.f;
        if (lane == 0) s_lse[r] = sum > 0.f ? mstar + log2f(sum) : -INFINITY;
    }
    __syncthreads();
    uint8_t *tiles = ring + wbytes;
    const int tile_bytes = g * D * 4;
    const int chunk = max(1, (int)((SM::kRingBytes - wbytes) / tile_bytes));
    const float *uo = a.part_o + (size_t)u * G * kStepMaxGroup * D;
    constexpr int C4 = D / 4;
    const int items = g * C4;  // float4 columns of the g rows
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int item = tid;      // g * D / 4 <= 8 * 32 < kThreadsAll
    for (int s0 = 0; s0 < G; s0 += chunk) {
        const int s1 = min(G, s0 + chunk);
        const int n16 = (s1 - s0) * items;  // 16-byte pieces
        for (int i = tid; i < n16; i += kThreadsAll) {
            const int s = s0 + i / items, k = i % items;
            cp_async16(tiles + (size_t)i * 16, uo + (size_t)s * kStepMaxGroup * D + (size_t)k * 4);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        if (item < items) {
            const int r = item / C4;
            const float4 *tf = reinterpret_cast<const float4 *>(tiles);
            for (int s = s0; s < s1; ++s) {
                const float w = wts[s * kStepMaxGroup + r];
                const float4 v = tf[(size_t)(s - s0) * items + item];
                acc.x += w * v.x;
                acc.y += w * v.y;
                acc.z += w * v.z;
                acc.w += w * v.w;
            }
        }
        __syncthreads();
    }
    if (item < items) {
        const int r = item / C4, c4 = item % C4;
        const size_t orow = (size_t)b * hkv * g + (size_t)h * g + r;
        reinterpret_cast<float4 *>(a.out + orow * D)[c4] = acc;
        if (a.lse && c4 == 0) a.lse[orow] = s_lse[r] * kLn2;
    }
    if (tid == 0) a.tickets[u] = 0;
}

}  // namespace

cudaError_t launch_decode_step_fused(const Shape &s, int G, void *k, void *v, void *desc,
                                     const int32_t *page_table, const int32_t *seq_len,
                                     const void *q, const void *k_new, const void *v_new,
                                     const int32_t *topk, int max_topk, float *out, float *lse,
                                     const StepBuffers &buf, cudaStream_t st) {
    StepArgs a;
    a.k_cache = static_cast<uint8_t *>(k);
    a.v_cache = static_cast<uint8_t *>(v);
    a.desc = static_cast<uint16_t *>(desc);
    a.page_table = page_table;
    a.seq_len = seq_len;
    a.topk = topk;
    a.q = static_cast<const uint16_t *>(q);
    a.k_new = static_cast<const uint4 *>(k_new);
    a.v_new = static_cast<const uint4 *>(v_new);
    a.block_idx = buf.block_idx;
    a.block_cnt = buf.block_cnt;
    a.out = out;
    a.lse = lse;
    a.hist = buf.hist;
    a.hist_range = buf.hist_range;
    a.bars = buf.bars;
    a.tickets = buf.tickets;
    a.counts = buf.counts;
    a.ovf = buf.ovf;
    a.cand = buf.cand;
    a.part_o = buf.part_o;
    a.part_lse = buf.part_lse;
    a.err = buf.err;
    a.hkv = s.hkv;
    a.g = s.g;
    a.max_pages = s.max_pages;
    a.num_pages = s.num_pages;
    a.max_topk = max_topk;
    a.scale_log2 = s.sm_scale * 1.4426950408889634f;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G, s.batch * s.hkv);
    cfg.blockDim = dim3(kThreadsAll);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
#define RESA_STEP_CASE(DD)                                                          \
    {                                                                               \
        constexpr int smem = StepSmem<DD>::kBytes;                                  \
        static std::atomic<int> done[64];                                           \
        cudaError_t e = ensure_smem(decode_step_kernel<DD>, smem, done);            \
        if (e != cudaSuccess) return e;                                             \
        cfg.dynamicSmemBytes = smem;                                                \
        return cudaLaunchKernelEx(&cfg, decode_step_kernel<DD>, a);                 \
    }
    if (s.d == 128) RESA_STEP_CASE(128)
    if (s.d == 64) RESA_STEP_CASE(64)
#undef RESA_STEP_CASE
    return cudaErrorInvalidValue;
}

}  // namespace resa
