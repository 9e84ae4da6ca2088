// Fused ReSA decode step of one layer in one persistent launch (ReSA summary
// §3.4.1 and §3.4.4; Algorithm 1 inner body): decode-token append, group
// query pooling, block scores (Eq. 4), top-k selection with the local block
// (Eq. 5 guards, ties to the lower block index) and group block-sparse
// split-KV attention (Eq. 2) with its log-sum-exp combine.
//
// Grid (G, units): G CTAs per (sequence, kv head) unit u, one CTA per SM,
// launched cooperatively so the G CTAs of a unit are co-resident.  CTA x owns
// the x-th contiguous range of `per` complete blocks of its unit.
//
//  1. Scoring.  All 12 warps stream the range's descriptors (this head's min
//     and max rows, 4d bytes per block) through per-warp cp.async rings, eight
//     blocks per warp step, four lanes per block.  The order-preserving keys of
//     the fp32 scores go to shared memory and to the unit's key row in the
//     workspace; their top 16 bits feed the unit's histogram (aggregated per
//     CTA in a shared-memory hash table, then one atomic per distinct digit).
//  2. Unit counter (one add, then a bounded poll).  In one round trip every
//     CTA reads the histogram bins around its own top digit and the unit's
//     whole key row (into the idle K/V ring).  The boundary digit d1 holding
//     the k-th largest key splits the blocks into definite (above d1) and
//     candidates (at d1); one pass over the keys counts the definite blocks of
//     each 32-block group and collects the candidates, and a radix select over
//     the candidates' composite keys (low 16 key bits, then the complement of
//     the block id: larger = higher score or, on equal scores, lower block id)
//     gives the exact threshold.  Every CTA holds every key, so every CTA
//     computes the same ordered work list without another exchange: the
//     selected blocks in ascending order, then the current block; CTA x takes
//     the contiguous slice [x W / G, (x + 1) W / G) of its W items.
//  3. The eight decode warps attend to the slice with per-warp 3-stage K/V
//     rings of 16-byte cp.async copies and swapped m16n8k16 MMAs
//     (attn_common.cuh); the other four warps write the slice's part of the
//     block list (ascending) and the count.
//  4. The CTA merges its warps into a partial (o / l, log2-sum-exp) written as
//     generation-tagged 64-bit words; each of the first g * d/32 CTAs polls
//     the words of one (query row, 32 channels) slice of the unit's G partials
//     until every tag is current and merges them; the others leave.
//
// The append (K/V of the decode token at position L-1 and the fold of its key
// into the current block's descriptor) is done by one warp of CTA G-1 of each
// unit during the scoring phase: only the current block reads it, that block
// is never scored, and it is the last work item, which CTA G-1 itself
// decodes, so the CTA's own barriers order the append before the read.
#include "attn_common.cuh"

namespace resa {
namespace {

constexpr int kDW = kDecodeWarps;         // decode warps
constexpr int kCW = 4;                    // the other warps
constexpr int kWarpsAll = kDW + kCW;
constexpr int kThreadsAll = 32 * kWarpsAll;
constexpr int kCtlThreads = 32 * kCW;
constexpr int kKvStages = 3;
constexpr int kScoreSlots = 4;            // descriptor ring slots per warp (8 blocks each)
constexpr int kScoreBlocks = 8;           // blocks per warp step of the scoring loop
constexpr int kHash = 1024;               // per-CTA digit histogram slots
constexpr int kMaxGroups = kHash;         // 32-block groups of a unit (group counts in the hash area)
constexpr int kCandPerWarp = 512;         // candidate segment of a warp
constexpr uint32_t kHashEmpty = 0xffffffffu;
constexpr uint32_t kSkip = 0xffffffffu;   // work item without data (bad page id)
constexpr int kModeAll = 0, kModeNone = 1, kModeMid = 2;

template <int D>
struct StepSmem {
    static constexpr int kTileBytes = kBlock * D * 2;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRingBytes = kDW * kKvStages * kStageBytes;
    static constexpr int kDescBytes = 4 * D;  // min and max rows of one (block, head)
    static constexpr int kSlotBytes = kScoreBlocks * kDescBytes;
    static_assert(kWarpsAll * kScoreSlots * kSlotBytes <= kRingBytes, "score rings fit the K/V rings");
    static_assert(kDW * kMaxGroup * (D + 2) * 4 <= kRingBytes, "warp states fit the rings");
    static_assert((step_unit_keys(D) * 2 + 8 + kWarpsAll * kCandPerWarp + 2048) * 4 <= kRingBytes,
                  "the unit's keys, page ids, candidates and radix bins fit the rings");
    static_assert(step_unit_keys(D) <= kMaxGroups * 32, "group counts fit the hash area");
    static constexpr int kKeysOff = kRingBytes;                      // u32 [kStepMaxBlocks] own keys
    static constexpr int kPagesOff = kKeysOff + kStepMaxBlocks * 4;  // i32 [kStepMaxBlocks] own pages
    static constexpr int kResCap = kStepMaxBlocks + 8;               // this CTA's items: at most F
    static constexpr int kItemOff = kPagesOff + kStepMaxBlocks * 4;  // u32 [kResCap] their block ids
    static constexpr int kResOff = kItemOff + kResCap * 4;           // u32 [kResCap] (page, tokens) items
    static constexpr int kHashOff = kResOff + kResCap * 4;           // u32 [2][kHash]
    static constexpr int kBytes = kHashOff + 2 * kHash * 4 + 128;    // + base alignment
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
    unsigned long long *bars;  // [units][kStepBarWords]: scored count, -, -, generation, padding
    uint32_t *ukeys;           // [units][key_stride] every block's key
    unsigned long long *part;  // [units * G][kStepMaxGroup][D + 1] tagged partial (o, then lse)
    uint32_t *err;
    RowMap rows;
    int hkv, g, max_pages, num_pages, max_topk, key_stride;
    float scale_log2;
};

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// Partials are written as 64-bit words (tag << 32 | value) tagged with the
// call's generation, so readers poll the words themselves (no fence, no
// barrier): a word with another tag is from an earlier call.
__device__ __forceinline__ unsigned long long tagged(uint32_t tag, uint32_t v) {
    return ((unsigned long long)tag << 32) | v;
}
__device__ __forceinline__ uint32_t tag_of(unsigned long long w) { return (uint32_t)(w >> 32); }

// Unit counter: each CTA adds one (no return value needed); waiters poll
// until all G arrived.  CTA 0 sets it back to zero once every CTA's partial
// is visible, i.e. after every CTA has passed it.  The caller fences its
// writes before arriving.
__device__ __forceinline__ bool unit_wait_count(const unsigned long long *ctr, uint32_t n) {
    for (uint32_t polls = 0;; ++polls) {
        unsigned long long v;
        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
        if (v >= (unsigned long long)n) return true;
        if (polls > (1u << 22)) return false;  // each poll is an L2 round trip
    }
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

__device__ __forceinline__ uint32_t item_of_page(int page, int num_pages, int ntok) {
    return (page >= 0 && page < num_pages) ? (((uint32_t)page << 4) | (uint32_t)(ntok - 1)) : kSkip;
}

// Composite selection key of block i whose score key is k (its top 16 bits
// are the boundary digit): larger = higher score, then lower block id.
__device__ __forceinline__ uint32_t composite(uint32_t k, int i) {
    return ((k & 0xffffu) << 16) | (0xffffu - (uint32_t)i);
}

// Indices of the small shared values.
enum {
    kVD1 = 0, kVDlo, kVDhi, kVHistOk, kVOk, kVLo, kVHi, kVAB, kVGen, kVCTop, kVCBot, kVG0, kVCount
};

template <int D>
__global__ void __launch_bounds__(kThreadsAll, 1) decode_step_kernel(const StepArgs a) {
    using SM = StepSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    // 128-byte aligned base, derived from the shared array itself so that
    // accesses keep the shared address space (no generic loads)
    uint8_t *smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    uint8_t *ring = smem;
    uint32_t *ukeys_s = reinterpret_cast<uint32_t *>(ring);  // the unit's keys (after scoring)
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + SM::kKeysOff);
    int32_t *pages = reinterpret_cast<int32_t *>(smem + SM::kPagesOff);
    uint32_t *own_item = reinterpret_cast<uint32_t *>(smem + SM::kItemOff);
    uint32_t *res_item = reinterpret_cast<uint32_t *>(smem + SM::kResOff);
    uint32_t *hkey = reinterpret_cast<uint32_t *>(smem + SM::kHashOff), *hcnt = hkey + kHash;

    __shared__ float qbar_s[D];
    __shared__ uint32_t s_scan[kWarpsAll];
    __shared__ uint32_t s_rsh[3];
    __shared__ int s_v[kVCount];
    __shared__ int s_seg[kWarpsAll];
    __shared__ float s_sc[kDW][kStepMaxGroup], s_rinv[kStepMaxGroup], s_rlse[kStepMaxGroup];

    pdl_launch_next();
    const int x = blockIdx.x, G = gridDim.x, u = blockIdx.y;
    const int hkv = a.hkv, g = a.g;
    const int b = u / hkv, h = u % hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cta = u * G + x;
    const int row = cache_row(a.rows, b, x == 0 && tid == 0 ? a.err : nullptr);
    const int L = row_seq_len(a.seq_len, row);
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
    const size_t prow = (size_t)max(row, 0) * a.max_pages;  // an invalid row reads as empty
    uint32_t *ukeys_g = a.ukeys + (size_t)u * a.key_stride;

    // ---- prologue: inputs of the call only (before the dependency wait) ----
    #pragma unroll 1
    for (int i = tid; i < nmine; i += kThreadsAll) pages[i] = a.page_table[prow + p0 + i];
    {
        const uint16_t *qh = a.q + ((size_t)b * hkv * g + (size_t)h * g) * D;
        #pragma unroll 1
        for (int j = tid; j < D; j += kThreadsAll) {
            float s = 0.f;
            #pragma unroll 1
            for (int r = 0; r < g; ++r) s += bf16_bits_to_f32(qh[(size_t)r * D + j]);
            qbar_s[j] = s / (float)g;
        }
    }
    #pragma unroll 1
    for (int i = tid; i < kHash; i += kThreadsAll) {
        hkey[i] = kHashEmpty;
        hcnt[i] = 0;
    }
    if (tid == 0) {
        s_v[kVOk] = 1;
        s_v[kVLo] = 0x7fffffff;
        s_v[kVHi] = -1;
        s_v[kVD1] = 0;
        s_v[kVHistOk] = 1;
        s_v[kVG0] = (M + 31) >> 5;  // no group (the selection loop then reads nothing)
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
    // The current block's page (its tokens are decoded by whichever CTA draws
    // it) and, for the appending warp, the decode token's K / V chunks.
    const int cur_page = seq_ok ? a.page_table[prow + M] : -1;
    constexpr int CPR = D / 8;  // 16-byte chunks per K / V row
    const bool appender = x == G - 1 && warp == kWarpsAll - 1 && seq_ok;
    uint4 app_k = make_uint4(0, 0, 0, 0), app_v = app_k;
    if (appender && lane < CPR) {
        app_k = a.k_new[((size_t)b * hkv + h) * CPR + lane];
        app_v = a.v_new[((size_t)b * hkv + h) * CPR + lane];
    }
    __syncthreads();
    pdl_wait();  // descriptors and K/V may be written by the preceding kernels
    unsigned long long *ubar = a.bars + kStepBarWords * (size_t)u;
    const uint32_t gen = tid == 0 ? (uint32_t)ld_relaxed_u64(&ubar[3]) : 0u;  // used after scoring

    // ---- 1. scoring (+ the append, whose descriptor loads are issued first) ----
    uint4 app_mn = make_uint4(0, 0, 0, 0), app_mx = app_mn;
    const int app_slot = (L - 1) % kBlock;
    const bool app_ok = appender && cur_page >= 0 && cur_page < a.num_pages;
    uint4 *app_dmn = nullptr;
    if (app_ok && lane < CPR) {
        app_dmn = reinterpret_cast<uint4 *>(a.desc) + (((size_t)cur_page * hkv + h) * 2) * CPR + lane;
        if (app_slot != 0) {
            app_mn = app_dmn[0];
            app_mx = app_dmn[CPR];
        }
    }
    {
        constexpr int CPB = SM::kDescBytes / 16;     // 16-byte chunks per block descriptor
        constexpr int RC = D / 32;                   // chunks of a row one lane reads
        constexpr int COPIES = kScoreBlocks * CPB / 32;
        const int nsteps = (nmine + kScoreBlocks - 1) / kScoreBlocks;
        const int nmy = warp < nsteps ? (nsteps - warp + kWarpsAll - 1) / kWarpsAll : 0;
        uint8_t *wring = ring + (size_t)warp * kScoreSlots * SM::kSlotBytes;
        // Block j of a slot sits at j * 4d bytes; its 16-byte chunk c at
        // (c ^ 4 (j odd)), so the two blocks a quarter-warp reads fall in
        // different banks.
        auto issue = [&](int it) {
            if (it < nmy) {
                const int blk0 = (warp + kWarpsAll * it) * kScoreBlocks;
                uint8_t *slot = wring + (size_t)(it % kScoreSlots) * SM::kSlotBytes;
#pragma unroll
                for (int i = 0; i < COPIES; ++i) {
                    const int f = i * 32 + lane;
                    const int j = f / CPB, c = f % CPB;
                    const int pi = blk0 + j;
                    if (pi < nmine) {
                        const int pg = pages[pi];
                        if (pg >= 0 && pg < a.num_pages)
                            cp_async16(slot + j * SM::kDescBytes + ((c ^ ((j & 1) << 2)) << 4),
                                       reinterpret_cast<const uint8_t *>(a.desc) +
                                           ((size_t)pg * hkv + h) * SM::kDescBytes + c * 16);
                    }
                }
            }
            cp_async_commit();
        };
#pragma unroll 1
        for (int it = 0; it < kScoreSlots - 1; ++it) issue(it);
        const int j = lane >> 2, s = lane & 3, sw = (j & 1) << 2;
        float qv[RC][8];
        uint32_t sel[RC][4];
#pragma unroll
        for (int k = 0; k < RC; ++k) {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[k][e] = qbar_s[(4 * k + s) * 8 + e];
#pragma unroll
            for (int w = 0; w < 4; ++w) sel[k][w] = upper_bound_selector(qv[k][2 * w], qv[k][2 * w + 1]);
        }
        for (int it = 0; it < nmy; ++it) {
            issue(it + kScoreSlots - 1);
            cp_async_wait<kScoreSlots - 1>();
            __syncwarp();
            const uint8_t *bp = wring + (size_t)(it % kScoreSlots) * SM::kSlotBytes + j * SM::kDescBytes;
            float part[RC];
#pragma unroll
            for (int k = 0; k < RC; ++k) {
                const int c = 4 * k + s;
                const uint4 mn = *reinterpret_cast<const uint4 *>(bp + ((c ^ sw) << 4));
                const uint4 mx = *reinterpret_cast<const uint4 *>(bp + (((c + D / 8) ^ sw) << 4));
                const uint32_t mnw[4] = {mn.x, mn.y, mn.z, mn.w};
                const uint32_t mxw[4] = {mx.x, mx.y, mx.z, mx.w};
                float acc = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t pw = __byte_perm(mnw[w], mxw[w], sel[k][w]);
                    acc = __fadd_rn(acc, __fmul_rn(qv[k][2 * w], __uint_as_float(pw << 16)));
                    acc = __fadd_rn(acc, __fmul_rn(qv[k][2 * w + 1], __uint_as_float(pw & 0xffff0000u)));
                }
                part[k] = acc;
            }
            __syncwarp();  // the slot is refilled by the next issue
            float sum = part[0];
#pragma unroll
            for (int k = 1; k < RC; ++k) sum = __fadd_rn(sum, part[k]);
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            const int pi = (warp + kWarpsAll * it) * kScoreBlocks + j;
            if (s == 0 && pi < nmine) {
                const int pg = pages[pi];
                const bool ok = pg >= 0 && pg < a.num_pages;
                if (!ok) set_error(a.err, RESA_DEVERR_PAGE);
                const uint32_t key = ok ? order_key(sum) : 0u;
                keys[pi] = key;
                ukeys_g[p0 + pi] = key;
            }
        }
        cp_async_wait<0>();
    }
    if (appender) {
        // decode-token append: K/V at position L-1, key folded into the
        // current block's descriptor (a new block starts from the key)
        if (!app_ok) {
            if (lane == 0) set_error(a.err, RESA_DEVERR_PAGE);
        } else if (lane < CPR) {
            const size_t o = (((size_t)cur_page * hkv + h) * kBlock + app_slot) * CPR + lane;
            reinterpret_cast<uint4 *>(a.k_cache)[o] = app_k;
            reinterpret_cast<uint4 *>(a.v_cache)[o] = app_v;
            if (app_slot == 0) {
                app_dmn[0] = app_k;
                app_dmn[CPR] = app_k;
            } else {
                Bf16x8 mn = unpack8(app_mn), mx = unpack8(app_mx);
                fold8(mn, mx, unpack8(app_k));
                app_dmn[0] = pack8(mn);
                app_dmn[CPR] = pack8(mx);
            }
        }
    }
    if (tid == 0) s_v[kVGen] = (int)gen;
    __syncthreads();
    const bool need_hist = mode == kModeMid;
    // The rings after scoring: the unit's keys, its page ids (block i at
    // upages_s[i + pshift]), the warps' candidate segments, the radix bins.
    uint32_t *upages_s = ukeys_s + ((M + 3) & ~3);
    const int pshift = (int)(prow & 3);
    const int cap = kCandPerWarp;
    uint32_t *cand_s = upages_s + ((M + pshift + 3) & ~3);       // [kWarpsAll][cap]
    uint32_t *rh = cand_s + kWarpsAll * cap;                     // [2048]
    if (need_hist) {
        // the first radix digit's bins are counted during the pass
        #pragma unroll 1
        for (int i = tid; i < 2048; i += kThreadsAll) rh[i] = 0;
        // per-CTA histogram of the keys' top 16 bits, then one global atomic
        // per distinct digit
        int lo = 0x7fffffff, hi = -1;
        #pragma unroll 1
        for (int i = tid; i < nmine; i += kThreadsAll) {
            const uint32_t digit = keys[i] >> 16;
            uint32_t slot = (digit * 0x9E3779B1u) >> 22;  // 10 bits
            bool placed = false;
            #pragma unroll 1
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
        __syncthreads();
        #pragma unroll 1
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
    __syncthreads();

    // ---- 2. unit barrier (the unit's page ids, an input, are copied while
    // the unit's CTAs meet), then the unit's keys and histogram ----
    // The arrival's fence comes before the page-id copies are issued, so it
    // does not wait for them.
    if (G > 1 && need_hist && tid == 0) {
        // release: the CTA's key row and histogram atomics, ordered by the
        // barrier above, are visible before the count
        asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(&ubar[0]) : "memory");
    }
    // the page-id row is copied from the 16-byte boundary at or below its
    // start, the tail (inside the row) with 4-byte copies
    if (mode == kModeAll || mode == kModeMid) {
        const int32_t *prow_al = a.page_table + (prow - pshift);
        const int nfull = (M + pshift) / 4;
        #pragma unroll 1
        for (int c = tid; c < nfull; c += kThreadsAll) cp_async16(upages_s + 4 * c, prow_al + 4 * c);
        #pragma unroll 1
        for (int e = 4 * nfull + tid; e < M + pshift; e += kThreadsAll) cp_async4(upages_s + e, prow_al + e);
    }
    cp_async_commit();
    if (G > 1 && need_hist) {
        if (tid == 0) s_v[kVOk] = unit_wait_count(&ubar[0], G) ? 1 : 0;
        __syncthreads();
        if (!s_v[kVOk]) {
            if (tid == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
            return;
        }
    }
    // in one round trip: the unit's keys (into the idle K/V rings) and the
    // histogram around this CTA's own top digit
    if (mode == kModeMid) {
        #pragma unroll 1
        for (int c = tid; c < (M + 3) / 4; c += kThreadsAll) cp_async16(ukeys_s + 4 * c, ukeys_g + 4 * c);
        cp_async_commit();
    }
    auto page_of = [&](int blk) -> int { return (int)upages_s[blk + pshift]; };
    uint32_t d1 = 0;
    int above = 0;
    if (need_hist) {
        // The boundary digit: the first read whose bins reach the unit's top
        // digit and hold at least keff keys decides it, each read one round
        // trip: (1) the kThreadsAll bins below this CTA's top digit + 128, read
        // together with the touched range; (2) the kThreadsAll bins below the
        // unit's top digit; (3) the whole touched range in contiguous chunks
        // (a thread's loads all in flight), then the chunk that holds the
        // boundary, one bin a thread.
        const uint32_t *hb = a.hist + (size_t)u * kHistBins;
        const int wtop1 = min(kHistBins - 1, s_v[kVHi] + 128);
        const uint32_t emin = __ldcg(&a.hist_range[2 * u]), emax = __ldcg(&a.hist_range[2 * u + 1]);
        const int wd1 = wtop1 - tid;
        const uint32_t wc1 = wd1 >= 0 ? __ldcg(&hb[wd1]) : 0u;
        const int dlo = kHistBins - (int)emin, dhi = (int)emax - 1;
        if (tid == 0) {
            s_v[kVDlo] = dlo;
            s_v[kVDhi] = dhi;
            s_v[kVCTop] = dhi;
            s_v[kVCBot] = dhi + 1;
        }
        // a descending scan over kThreadsAll bins (thread t: bin wtop - t)
        auto window = [&](int wtop, uint32_t c) -> bool {
            uint32_t tot;
            const uint32_t before = cta_scan(c, s_scan, tot);
            if (c > 0 && before < (uint32_t)keff && (uint32_t)keff <= before + c) {
                s_v[kVD1] = wtop - tid;
                s_v[kVAB] = (int)before;  // keys above the boundary digit
            }
            if (tid == 0 && tot > (uint32_t)M) s_v[kVHistOk] = 0;
            return tot >= (uint32_t)keff;
        };
        bool found = dhi <= wtop1 && window(wtop1, wc1);  // uniform over the CTA
        if (!found) {
            const int wd2 = dhi - tid;
            found = window(dhi, wd2 >= 0 ? __ldcg(&hb[wd2]) : 0u);
        }
        if (!found) {
            const int nb = dhi >= dlo ? dhi - dlo + 1 : 0;
            const int chunk = (nb + kThreadsAll - 1) / kThreadsAll;  // <= kThreadsAll bins
            const int top = dhi - tid * chunk, bot = max(dlo, top - chunk + 1);
            uint32_t loc = 0;
#pragma unroll 1
            for (int d0 = top; d0 >= bot; d0 -= 16) {
                uint32_t c16[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) c16[e] = d0 - e >= bot ? __ldcg(&hb[d0 - e]) : 0u;
#pragma unroll
                for (int e = 0; e < 16; ++e) loc += c16[e];
            }
            uint32_t total;
            const uint32_t before = cta_scan(loc, s_scan, total);
            if (loc > 0 && before < (uint32_t)keff && (uint32_t)keff <= before + loc) {
                s_v[kVCTop] = top;
                s_v[kVCBot] = bot;
                s_v[kVAB] = (int)before;
            }
            if (tid == 0) s_v[kVHistOk] = total == (uint32_t)M ? 1 : 0;
            __syncthreads();
            const int ctop = s_v[kVCTop], cbot = s_v[kVCBot];
            const uint32_t cbefore = (uint32_t)s_v[kVAB];
            const int d = ctop - tid;
            const uint32_t c = d >= cbot ? __ldcg(&hb[d]) : 0u;
            uint32_t tot2;
            const uint32_t b2 = cta_scan(c, s_scan, tot2);
            if (c > 0 && cbefore + b2 < (uint32_t)keff && (uint32_t)keff <= cbefore + b2 + c) {
                s_v[kVD1] = d;
                s_v[kVAB] = (int)(cbefore + b2);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    if (need_hist) {
        if (!s_v[kVHistOk]) {
            // The histogram was not clean at entry (an earlier call gave up
            // mid-way): every CTA of the unit sees the same sums and selects
            // no complete block.
            if (tid == 0 && x == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
            mode = kModeNone;
            keff = 0;
        }
        d1 = (uint32_t)s_v[kVD1];
        above = s_v[kVAB];
    }
    // Work split: the unit's ordered work list is the selected blocks in
    // ascending order, then the current block (W = keff + 1 items); CTA x
    // takes items [x*W/G, (x+1)*W/G).
    const int W = seq_ok ? keff + 1 : 0;
    const int s0 = (int)((long long)W * x / G), s1 = (int)((long long)W * (x + 1) / G);
    const int n_items = s1 - s0;  // floor(W / G) or one more
    int *gcnt = reinterpret_cast<int *>(hkey), *gpre = reinterpret_cast<int *>(hcnt);  // [ngroups]
    const int ngroups = (M + 31) >> 5;
    uint32_t tau = 0xffffffffu;
    int rem = 0;
    if (mode == kModeMid) {
        // One pass over the unit's keys, half a 32-block group per lane: the
        // half's definite count (two lanes' counts make the group's) and a
        // mask of its candidates from the lane's 16 keys (four 16-byte loads,
        // their order rotated by lane pair so that each quarter-warp's loads
        // cover all banks once), then the candidates' composite keys appended
        // to the warp's segment (offsets by a warp scan) and counted in the
        // bins of the first radix digit.
        // Per key only full-rate integer operations: a key's digit is above
        // d1 iff the key is above hi1, equal to d1 iff key - lo1 < 2^16.
        // (A ballot-per-key pass was bound by the quarter-rate vote and
        // population-count units.)
        // The last warp meanwhile pulls into L2 the K/V of the blocks above
        // the boundary digit in the CTA's own scored range: they are selected
        // whatever the candidates settle, so HBM streams the selection from
        // here on.  (Bulk prefetches queue on the copy unit; issued by every
        // warp they would hold up the whole pass.)
        const uint32_t lo1 = d1 << 16, hi1 = lo1 | 0xffffu;
        uint32_t *seg = cand_s + warp * cap;
        int nseg = 0;
        if (warp == kWarpsAll - 1) {
            #pragma unroll 1
            for (int i = lane; i < nmine; i += 32) {
                const int pg = pages[i];
                if (keys[i] > hi1 && pg >= 0 && pg < a.num_pages) {
                    const size_t t = ((size_t)pg * hkv + h) * SM::kTileBytes;
                    prefetch_l2(a.k_cache + t, SM::kTileBytes);
                    prefetch_l2(a.v_cache + t, SM::kTileBytes);
                }
            }
        }
        constexpr int kPassThreads = (kWarpsAll - 1) * 32;
        #pragma unroll 1
        for (int h0 = warp * 32; warp < kWarpsAll - 1 && h0 < 2 * ngroups; h0 += kPassThreads) {
            const int hg = h0 + lane;          // half-group: keys [16 hg, 16 hg + 16)
            const int q = hg >> 1;
            const int lim = M - hg * 16;       // keys of the half: min(16, lim)
            const uint32_t *gk = ukeys_s + (size_t)hg * 16;
            const int rot = lane >> 1;
            int nd = 0;
            uint32_t cm = 0;  // bit 4j + e: key 4 ((j + rot) & 3) + e of the half
            if (lim >= 16) {
                int nde[4] = {0, 0, 0, 0};
                uint32_t cme[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 k4 = *reinterpret_cast<const uint4 *>(gk + 4 * ((j + rot) & 3));
                    const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        nde[e] += kk[e] > hi1 ? 1 : 0;
                        cme[e] |= kk[e] - lo1 < 0x10000u ? (1u << (4 * j + e)) : 0u;
                    }
                }
                nd = (nde[0] + nde[1]) + (nde[2] + nde[3]);
                cm = (cme[0] | cme[1]) | (cme[2] | cme[3]);
            } else if (lim > 0) {
                #pragma unroll 1
                for (int t = 0; t < lim; ++t) {
                    const uint32_t k = gk[t];
                    nd += k > hi1 ? 1 : 0;
                    const int j = ((t >> 2) - rot) & 3;
                    cm |= k - lo1 < 0x10000u ? (1u << (4 * j + (t & 3))) : 0u;
                }
            }
            const int ng = nd + __shfl_xor_sync(0xffffffffu, nd, 1);
            if ((lane & 1) == 0 && q < ngroups) gcnt[q] = ng;
            const int nc = __popc(cm);
            int incl = nc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            int r = nseg + incl - nc;
            nseg += __shfl_sync(0xffffffffu, incl, 31);
            #pragma unroll 1
            while (cm != 0u) {
                const int bit = __ffs(cm) - 1;
                cm &= cm - 1u;
                const int i = hg * 16 + 4 * (((bit >> 2) + rot) & 3) + (bit & 3);
                const uint32_t cmp = composite(ukeys_s[i], i);
                atomicAdd(&rh[cmp >> 21], 1u);
                if (r < cap) seg[r] = cmp;
                ++r;
            }
        }
        if (lane == 0) s_seg[warp] = nseg;
        __syncthreads();
        // exact threshold: the rem-th largest candidate composite by radix
        // select, stopping at the first digit whose bin is taken whole
        int seg_end[kWarpsAll];
        bool fits = true;
        {
            int acc = 0;
#pragma unroll
            for (int w = 0; w < kWarpsAll; ++w) {
                fits = fits && s_seg[w] <= cap;
                acc += s_seg[w];
                seg_end[w] = acc;
            }
        }
        const int NC = seg_end[kWarpsAll - 1];
        // candidate f of the list (segments in warp order); when a segment
        // overflowed, candidates are found by scanning the keys instead
        auto for_each_cand = [&](auto fn) {
            if (fits) {
                #pragma unroll 1
                for (int f = tid; f < NC; f += kThreadsAll) {
                    int w = 0, st0 = 0;
#pragma unroll
                    for (int k2 = 0; k2 < kWarpsAll - 1; ++k2)
                        if (f >= seg_end[k2]) {
                            w = k2 + 1;
                            st0 = seg_end[k2];
                        }
                    fn(cand_s[w * cap + (f - st0)]);
                }
            } else {
                #pragma unroll 1
                for (int i = tid; i < M; i += kThreadsAll) {
                    const uint32_t k = ukeys_s[i];
                    if ((k >> 16) == d1) fn(composite(k, i));
                }
            }
        };
        rem = keff - above;
        if (rem < 1 || rem > NC) {  // cannot happen with consistent counts
            if (tid == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
            rem = max(0, min(rem, NC));
        }
        if (rem > 0) {
            // digits of 11, 8, 8 and 5 bits, most significant first (the
            // first one's bins were filled by the pass); the digit holding the
            // remaining-th largest candidate is found by one CTA-wide scan in
            // descending order
            uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)rem;
            int shift = 32;
            #pragma unroll 1
            for (int pass = 0; pass < 4; ++pass) {
                const int width = pass == 0 ? 11 : pass == 3 ? 5 : 8;
                shift -= width;
                const int nb = 1 << width;
                if (pass > 0) {
                    #pragma unroll 1
                    for (int i = tid; i < nb; i += kThreadsAll) rh[i] = 0;
                    __syncthreads();
                    for_each_cand([&](uint32_t c) {
                        if ((c & pmask) == prefix) atomicAdd(&rh[(c >> shift) & (uint32_t)(nb - 1)], 1u);
                    });
                    __syncthreads();
                }
                constexpr int kPer = (2048 + kThreadsAll - 1) / kThreadsAll;
                uint32_t cnt[kPer], sum = 0;
#pragma unroll
                for (int jj = 0; jj < kPer; ++jj) {
                    const int dgt = nb - 1 - (tid * kPer + jj);  // descending digits
                    cnt[jj] = dgt >= 0 ? rh[dgt] : 0u;
                    sum += cnt[jj];
                }
                uint32_t tot;
                uint32_t cum = cta_scan(sum, s_scan, tot);  // candidates in higher digits
                if (cum < remaining && remaining <= cum + sum) {
#pragma unroll
                    for (int jj = 0; jj < kPer; ++jj) {
                        if (cum < remaining && remaining <= cum + cnt[jj]) {
                            s_rsh[0] = (uint32_t)(nb - 1 - (tid * kPer + jj));
                            s_rsh[1] = cum;
                            s_rsh[2] = cnt[jj];
                        }
                        cum += cnt[jj];
                    }
                }
                __syncthreads();
                remaining -= s_rsh[1];
                prefix |= s_rsh[0] << shift;
                pmask |= (uint32_t)(nb - 1) << shift;
                if (remaining == s_rsh[2]) break;  // every key with this prefix is taken
            }
            tau = prefix;
            // the qualifying candidates join their groups' counts
            for_each_cand([&](uint32_t c) {
                if (c >= tau) atomicAdd(&gcnt[(int)(0xffffu - (c & 0xffffu)) >> 5], 1);
            });
        }
        __syncthreads();
        // exclusive prefix of the selected count over the groups; the group
        // that holds item s0 (selected, so of nonzero count) is noted
        {
            constexpr int RG = (kMaxGroups + kThreadsAll - 1) / kThreadsAll;
            const int q0 = tid * RG;
            int v[RG];
            uint32_t sum = 0;
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                v[r] = q0 + r < ngroups ? gcnt[q0 + r] : 0;
                sum += v[r];
            }
            uint32_t tot;
            uint32_t run = cta_scan(sum, s_scan, tot);
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                if (q0 + r < ngroups) {
                    gpre[q0 + r] = (int)run;
                    if (run <= (uint32_t)s0 && (uint32_t)s0 < run + (uint32_t)v[r]) s_v[kVG0] = q0 + r;
                }
                run += v[r];
            }
        }
        __syncthreads();
        // this CTA's items among the selected blocks: groups q with
        // gpre[q] < e and gpre[q] + gcnt[q] > s0, one warp per group
        const int e_sel = min(s1, keff);
        if (s0 < e_sel) {
            const uint32_t lt_mask = (1u << lane) - 1u;
            const int lo = s_v[kVG0];  // s0 < keff: exactly one group holds item s0
            #pragma unroll 1
            for (int q = lo + warp; q < ngroups && gpre[q] < e_sel; q += kWarpsAll) {
                const int i = q * 32 + lane;
                const uint32_t k = i < M ? ukeys_s[i] : 0u;
                const uint32_t dg = k >> 16;
                const bool sel = i < M && (dg > d1 || (dg == d1 && rem > 0 && composite(k, i) >= tau));
                const uint32_t bs = __ballot_sync(0xffffffffu, sel);
                const int rank = gpre[q] + __popc(bs & lt_mask);
                if (sel && rank >= s0 && rank < e_sel) {
                    res_item[rank - s0] = item_of_page(page_of(i), a.num_pages, kBlock);
                    own_item[rank - s0] = (uint32_t)i;
                }
            }
        }
    } else if (mode == kModeAll) {
        // every complete block is selected: items are block ids themselves
        #pragma unroll 1
        for (int j = tid; j < min(s1, M) - s0; j += kThreadsAll) {
            res_item[j] = item_of_page(page_of(s0 + j), a.num_pages, kBlock);
            own_item[j] = (uint32_t)(s0 + j);
        }
    }
    if (tid == 0 && seq_ok && keff >= s0 && keff < s1) {
        res_item[keff - s0] = item_of_page(cur_page, a.num_pages, L - M * kBlock);
        own_item[keff - s0] = (uint32_t)M;
    }
    __syncthreads();

    if (warp < kDW) {
        // ---- 3. decode warps: this CTA's items ----
        WarpState<D, 1> st;
        st.init();
        uint8_t *wr = ring + (size_t)warp * kKvStages * SM::kStageBytes;
        constexpr int kPerLane = SM::kTileBytes / 16 / 32;
        auto issue = [&](int t) {
            const int j = warp + kDW * t;
            if (j < n_items) {
                const uint32_t item = res_item[j];
                if (item != kSkip) {
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
            }
            cp_async_commit();
        };
#pragma unroll 1
        for (int t = 0; t < kKvStages - 1; ++t) issue(t);
        for (int t = 0; warp + kDW * t < n_items; ++t) {
            issue(t + kKvStages - 1);
            cp_async_wait<kKvStages - 1>();
            __syncwarp();
            const uint32_t item = res_item[warp + kDW * t];
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
        // ---- 3'. the other warps: this CTA's part of the block list, the
        // count, errors, and (a single CTA per unit) the histogram cleanup ----
        const int ct = tid - kDW * 32;
        int32_t *list = a.block_idx + (size_t)u * (a.max_topk + 1);
        #pragma unroll 1
        for (int j = ct; j < n_items; j += kCtlThreads) list[s0 + j] = (int32_t)own_item[j];
        if (x == 0 && ct == 0) {
            a.block_cnt[u] = seq_ok ? keff + 1 : 0;
            if (!seq_ok) set_error(a.err, RESA_DEVERR_SEQ_LEN);
            if (topk_err) set_error(a.err, RESA_DEVERR_TOPK);
        }
        if (G == 1 && need_hist) {
            uint32_t *hb = a.hist + (size_t)u * kHistBins;
            #pragma unroll 1
            for (int d = s_v[kVDlo] + ct; d <= s_v[kVDhi]; d += kCtlThreads) hb[d] = 0;
            if (ct == 0) {
                a.hist_range[2 * u] = 0;
                a.hist_range[2 * u + 1] = 0;
            }
        }
    }
    __syncthreads();  // warp states are in shared memory

    // ---- 4. merge the warps into this CTA's partial (tagged words) ----
    const float kLn2 = 0.6931471805599453f;
    const uint32_t tag = (uint32_t)s_v[kVGen] + 1u;
    constexpr int PS = D + 1;  // partial row: D outputs, then the log2-sum-exp
    {
        const float *mw = reinterpret_cast<const float *>(ring);
        const float *lw = mw + kDW * kMaxGroup;
        const float *ow = lw + kDW * kMaxGroup;
        unsigned long long *pp = a.part + (size_t)cta * kStepMaxGroup * PS;
        const int hq = hkv * g;
        // per row: the warps' scale factors exp2(m_w - m*), 1 / l and the
        // log2-sum-exp, once, by one warp: lane (w4, r) takes decode warps
        // w4 and w4 + 4 of row r
        static_assert(kDW == 8 && kStepMaxGroup == 8, "one warp covers 8 rows x 8 decode warps");
        if (warp == 0) {
            const int r = lane & 7, w4 = lane >> 3;
            float mstar = -INFINITY;
#pragma unroll
            for (int w = 0; w < kDW; ++w) mstar = fmaxf(mstar, mw[w * kMaxGroup + r]);
            float lsum = 0.f;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int w = w4 + 4 * k;
                const float sc = mstar != -INFINITY ? exp2f(mw[w * kMaxGroup + r] - mstar) : 0.f;
                s_sc[w][r] = sc;
                lsum += lw[w * kMaxGroup + r] * sc;
            }
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
            if (w4 == 0) {
                s_rinv[r] = lsum > 0.f ? 1.f / lsum : 0.f;
                s_rlse[r] = lsum > 0.f ? mstar + log2f(lsum) : -INFINITY;
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int e = tid; e < g * D; e += kThreadsAll) {
            const int r = e / D, c = e % D;
            float o = 0.f;
#pragma unroll
            for (int w = 0; w < kDW; ++w) o += ow[((size_t)w * kMaxGroup + r) * D + c] * s_sc[w][r];
            const float on = o * s_rinv[r];
            if (G == 1) {
                const size_t orow = (size_t)b * hq + (size_t)h * g + r;
                a.out[orow * D + c] = on;
                if (a.lse && c == 0) a.lse[orow] = s_rlse[r] * kLn2;
            } else {
                pp[(size_t)r * PS + c] = tagged(tag, __float_as_uint(on));
                if (c == 0) pp[(size_t)r * PS + D] = tagged(tag, __float_as_uint(s_rlse[r]));
            }
        }
    }
    if (G == 1) return;
    // Each (query row, 32 channels) slice of the output goes to CTA
    // slice % G, which polls the G partials' words until they carry this
    // call's tag.  CTAs without a slice leave.
    constexpr int C32 = D / 32;
    const int n_slices = g * C32;
    if (x >= n_slices) return;
    __syncthreads();  // the ring's warp states are read; it holds the reduction below
    const unsigned long long *up = a.part + (size_t)u * G * kStepMaxGroup * PS;
    constexpr int kPW = (kNumSms + kWarpsAll - 1) / kWarpsAll;  // partials per warp
    float *red = reinterpret_cast<float *>(ring);                // [kWarpsAll][33]
    float *lse_s = red + kWarpsAll * 33;                         // [G] partials' log2-sum-exp
    bool all_ok = true;
#pragma unroll 1
    for (int item = x; item < n_slices; item += G) {
        const int r = item / C32, cc = item % C32;
        // this warp's partials (warp, warp + 12, ...) at lane's channel; one
        // thread per partial for its log2-sum-exp
        unsigned long long wv[kPW];
        bool ok = false;
#pragma unroll 1
        for (uint32_t polls = 0; polls < (1u << 20) && !ok; ++polls) {
            bool good = true;
#pragma unroll
            for (int k = 0; k < kPW; ++k) {
                const int sp = warp + kWarpsAll * k;
                wv[k] = sp < G ? ld_relaxed_u64(up + ((size_t)sp * kStepMaxGroup + r) * PS + cc * 32 + lane)
                               : tagged(tag, 0u);
                good = good && tag_of(wv[k]) == tag;
            }
            if (tid < G) {
                const unsigned long long wl = ld_relaxed_u64(up + ((size_t)tid * kStepMaxGroup + r) * PS + D);
                good = good && tag_of(wl) == tag;
                lse_s[tid] = __uint_as_float((uint32_t)wl);
            }
            ok = __all_sync(0xffffffffu, good);  // each warp polls its own words
        }
        ok = __syncthreads_and(ok) != 0;  // lse_s is complete
        all_ok = all_ok && ok;
        float mstar = -INFINITY;
#pragma unroll 1
        for (int sp = lane; sp < G; sp += 32) mstar = fmaxf(mstar, lse_s[sp]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
        float lsum = 0.f, acc = 0.f;
        if (mstar != -INFINITY) {
#pragma unroll
            for (int k = 0; k < kPW; ++k) {
                const int sp = warp + kWarpsAll * k;
                if (sp < G) {
                    const float wk = exp2f(lse_s[sp] - mstar);
                    lsum += wk;
                    acc += wk * __uint_as_float((uint32_t)wv[k]);
                }
            }
        }
        red[warp * 33 + lane] = acc;
        if (lane == 0) red[warp * 33 + 32] = lsum;
        __syncthreads();
        if (warp == 0) {
            float o = 0.f, lt = 0.f;
#pragma unroll
            for (int w = 0; w < kWarpsAll; ++w) {
                o += red[w * 33 + lane];
                lt += red[w * 33 + 32];
            }
            const size_t orow = (size_t)b * hkv * g + (size_t)h * g + r;
            a.out[orow * D + cc * 32 + lane] = lt > 0.f ? o / lt : 0.f;
            if (a.lse && cc == 0 && lane == 0)
                a.lse[orow] = (lt > 0.f ? mstar + log2f(lt) : -INFINITY) * kLn2;
        }
        __syncthreads();
    }
    if (!all_ok) {
        if (tid == 0) set_error(a.err, RESA_DEVERR_TIMEOUT);
        return;
    }
    if (x == 0) {
        // Every CTA's partial is visible, so every CTA has passed the counter
        // and read the histogram: reset them for the next call and advance
        // the generation.
        if (tid == 0) {
            ubar[0] = 0;
            ubar[3] = (unsigned long long)tag;
        }
        if (need_hist) {
            uint32_t *hb = a.hist + (size_t)u * kHistBins;
#pragma unroll 1
            for (int d = s_v[kVDlo] + tid; d <= s_v[kVDhi]; d += kThreadsAll) hb[d] = 0;
            if (tid == 0) {
                a.hist_range[2 * u] = 0;
                a.hist_range[2 * u + 1] = 0;
            }
        }
    }
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
    a.ukeys = buf.ukeys;
    a.part = buf.part;
    a.err = buf.err;
    a.rows = s.rows;
    a.hkv = s.hkv;
    a.g = s.g;
    a.max_pages = s.max_pages;
    a.num_pages = s.num_pages;
    a.max_topk = max_topk;
    a.key_stride = step_key_stride(s.max_pages);
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
