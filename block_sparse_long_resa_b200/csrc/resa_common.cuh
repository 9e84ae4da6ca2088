// Internal definitions shared by the libresa translation units (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "../../include/resa.h"

namespace resa {

// ---------------------------------------------------------------------------
// Fixed shape limits
// ---------------------------------------------------------------------------
constexpr int kBlock = 16;          // tokens per block / page of the fused decode step
constexpr int kTileRows = 16;       // tokens per K / V tile (a block holds bs / 16 of them)
constexpr int kMaxGroup = 16;       // query heads per kv head (one m16 MMA tile)
constexpr int kMaxKvHeads = 8;
constexpr int kNumSms = 148;
constexpr int kMaxBlocksPerSplit = 512;  // blocks one decode CTA stages in shared memory
constexpr int kMinBlocksPerSplit = 16;   // two per warp at least

// Decode splits per (sequence, kv head): about one CTA per SM over all units,
// at least kMinBlocksPerSplit blocks each, at most kMaxBlocksPerSplit.
// Splits of one (sequence, kv head) the decode merge takes (its weights sit in
// shared memory next to the partial tiles): max_topk + 1 <= 1024 * 512 blocks.
constexpr int kMaxDecodeSplits = 1024;
inline int decode_splits_for(int units, int max_blocks) {
    const int need = (max_blocks + kMaxBlocksPerSplit - 1) / kMaxBlocksPerSplit;
    // as many splits as keep the grid within one wave of CTAs (one per SM)
    const int want = units < kNumSms ? kNumSms / units : 1;
    const int work = (max_blocks + kMinBlocksPerSplit - 1) / kMinBlocksPerSplit;
    int s = want < work ? want : work;
    s = s > need ? s : need;
    return s < 1 ? 1 : s;
}
// Decode grids of at most this many CTAs may merge their splits across the
// grid from per-warp partials (8 warps per CTA): the scratch for partials
// holds max(units * splits, kSpreadMaxCtas * 8) of them.
constexpr int kSpreadMaxCtas = kNumSms;
constexpr int kDecodeWarps = 8;
inline size_t decode_partials(int units, int splits) {
    const size_t a = (size_t)units * splits, b = (size_t)kSpreadMaxCtas * kDecodeWarps;
    return a > b ? a : b;
}
// Partial-result capacity of the workspace: enough for any top-k up to max_pages.
inline int decode_max_splits(int batch, int hkv, int max_pages) {
    const int units = batch * hkv;
    const int need = (max_pages + 1 + kMaxBlocksPerSplit - 1) / kMaxBlocksPerSplit;
    const int want = (kNumSms + units - 1) / units;
    return want > need ? want : need;
}
// Fused decode step (one persistent launch per step): G CTAs per (sequence,
// kv head) unit, G * units <= kNumSms; a CTA scores at most kStepMaxBlocks
// complete blocks; block ids must fit 16 bits (composite selection keys), so
// max_pages <= 65536.
constexpr int kStepMaxBlocks = 1024;
constexpr int kStepMaxPages = 65536;
// After scoring, every CTA of the fused step holds its unit's keys, page ids,
// boundary candidates (12 warps x 512 at most) and a 2048-bin radix
// histogram in its K/V rings (8 warps x 3 stages x a 16-token K and V tile):
// at most this many complete blocks.
constexpr int step_unit_keys(int d) {
    return (kDecodeWarps * 3 * 2 * kBlock * d * 2 / 4 - 12 * 512 - 2048 - 16) / 2 < 32768
               ? (kDecodeWarps * 3 * 2 * kBlock * d * 2 / 4 - 12 * 512 - 2048 - 16) / 2
               : 32768;
}
// Row stride (in keys) of a unit's key row in the workspace: 16-byte rows.
inline int step_key_stride(int max_pages) { return (max_pages + 3) & ~3; }
constexpr int kStepMaxGroup = 8;  // one n8 MMA tile of query heads (register budget)
// Words per unit of the fused step's counter block: one 128-byte line each, so
// the units' counters, polled by all their CTAs, do not share a line.
constexpr int kStepBarWords = 16;
// CTAs per unit of the fused step, or 0 when the shape needs the unfused path.
inline int step_ctas_per_unit(int units, int g, int d, int max_pages, int sms) {
    if (g > kStepMaxGroup || max_pages > kStepMaxPages || units <= 0) return 0;
    if (max_pages > step_unit_keys(d)) return 0;
    const int cap = sms < kNumSms ? sms : kNumSms;
    const int by_sm = cap / units;
    const int by_work = (max_pages + 63) / 64;  // about 64 blocks per CTA at least
    int G = by_sm < by_work ? by_sm : by_work;
    if (G < 2) G = by_sm >= 2 ? 2 : G;
    if (G < 2) return 0;
    if ((max_pages + G - 1) / G > kStepMaxBlocks) return 0;
    return G;
}

constexpr int kRectRowsPerCta = 256;  // query rows (chunk position x group head) per CTA
inline int rect_row_groups(int chunk, int group) {
    const int rows = chunk * group;
    return (rows + kRectRowsPerCta - 1) / kRectRowsPerCta;
}
// Key splits of a rectification: one CTA per SM over all (unit, row group)
// pairs, and at least one split per kRectKeysPerSplit keys of the longest
// sequence.  A grid within one wave merges its splits after a grid barrier
// (cooperative launch); a larger one (long sequences in a large batch) lets
// the last split of each (unit, row group) merge it.
constexpr int kRectKeysPerSplit = 16384;
inline int rect_splits_for(int batch, int hkv, int groups, long long max_keys) {
    const int units = batch * hkv * (groups > 0 ? groups : 1);
    int s = kNumSms / units;
    const long long by_len = (max_keys + kRectKeysPerSplit - 1) / kRectKeysPerSplit;
    if (by_len > s) s = (int)(by_len < 64 ? by_len : 64);
    return s < 1 ? 1 : (s > 64 ? 64 : s);
}

// ---------------------------------------------------------------------------
// Workspace layout (byte offsets).  Every region except the rectification
// partials depends only on (heads, d, batch, max_pages), so decode and
// rectification calls of different chunk sizes find the same regions; the
// rectification partials come last.
// ---------------------------------------------------------------------------
constexpr int kMaxRowTiles = 64;  // rectification row groups per (sequence, kv head)
constexpr int kRectTicketBase = 16;  // u32 words before the split tickets (grid barrier word)

// Byte offset, inside the 256-byte error header of the workspace, of the
// decode kernel's grid barrier word (64-bit: generation, arrivals).
constexpr size_t kDecBarrierOffset = 32;

struct WsLayout {
    size_t err;          // uint32 error word
    size_t dec_ticket;   // uint32 [B][Hkv]
    size_t rect_ticket;  // grid barrier word, then uint32 [B][Hkv][kMaxRowTiles] split tickets
    size_t hist;         // uint32 [B][Hkv][65536] score-key histogram (kept zero between calls)
    size_t hist_range;   // uint32 [B][Hkv][2] touched-bin range (kept zero between calls)
    size_t scores;       // f32 [B][Hkv][max_pages]
    size_t sel_idx;      // i32 [B][Hkv][max_pages + 1]
    size_t sel_cnt;      // i32 [B][Hkv]
    size_t dec_o;        // f32 [partials][kMaxGroup][d]: per split, or per warp when spread
    size_t dec_lse;      // f32 [partials][kMaxGroup] lse, or float2 (row max, row sum) when spread
    size_t step_bars;    // u64 [B][Hkv][kStepBarWords] unit counter (zero between calls) and generation of the fused step
    size_t step_keys;    // u32 [B][Hkv][step_key_stride(max_pages)] block score keys of the fused step
    size_t step_part;    // u64 [kNumSms][kStepMaxGroup][d + 1] tagged per-CTA partials of the fused step
    size_t rect_o;       // f32 [B][Hkv][row_groups][rect_splits][kRectRowsPerCta][d]
    size_t rect_lse;     // f32 [B][Hkv][row_groups][rect_splits][kRectRowsPerCta]
    size_t total;
    int dec_splits;
    int row_tiles;   // rectification row groups of kRectRowsPerCta
    int rect_splits;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Layout for a call that rectifies chunks of `chunk` tokens (0: no rectification).
inline WsLayout ws_layout(int hq, int hkv, int d, int bs, int batch, int max_pages, int chunk) {
    WsLayout w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    int g = hkv > 0 ? hq / hkv : 1;
    w.dec_splits = decode_max_splits(batch, hkv, max_pages);
    w.row_tiles = chunk > 0 ? rect_row_groups(chunk, g) : 0;
    w.rect_splits = chunk > 0 ? rect_splits_for(batch, hkv, w.row_tiles, (long long)max_pages * bs) : 0;
    size_t units = (size_t)batch * hkv;
    w.err = take(256);  // error word at 0, decode grid barrier at kDecBarrierOffset
    w.dec_ticket = take(units * 4);
    w.rect_ticket = take(kRectTicketBase * 4 + units * kMaxRowTiles * 4);
    w.hist = take(units * 65536 * 4);
    w.hist_range = take(units * 2 * 4);
    w.scores = take(units * max_pages * 4);
    w.sel_idx = take(units * (max_pages + 1) * 4);
    w.sel_cnt = take(units * 4);
    const size_t parts = decode_partials((int)units, w.dec_splits);
    w.dec_o = take(parts * kMaxGroup * d * 4);
    w.dec_lse = take(parts * kMaxGroup * 2 * 4);  // (lse) or (row max, row sum) pairs
    w.step_bars = take(units * kStepBarWords * 8);
    w.step_keys = take(units * (size_t)step_key_stride(max_pages) * 4);
    w.step_part = take((size_t)kNumSms * kStepMaxGroup * (d + 1) * 8);
    size_t rect_rows = units * w.row_tiles * w.rect_splits * kRectRowsPerCta;
    w.rect_o = take(rect_rows * d * 4);
    w.rect_lse = take(rect_rows * 4);
    w.total = off;
    return w;
}

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bit) {
    if (err) atomicOr(err, bit);
}

// Warm L2 with [p, p + bytes): a bulk prefetch, no completion to wait for
// and no shared memory (16-byte aligned address, bytes a multiple of 16).
// It is only a cache fill, so it is coherent with any concurrent write.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Row map of a call (resa_cache_t.rows / table_rows): the call's i-th
// sequence reads row rows[i] of page_table and seq_len, or row i without a map.
struct RowMap {
    const int32_t *rows;
    int table_rows;
};

// The cache row of the call's sequence i; -1 (and RESA_DEVERR_ROW) for a
// mapped row outside [0, table_rows).
__device__ __forceinline__ int cache_row(const RowMap &m, int i, uint32_t *err) {
    if (m.rows == nullptr) return i;
    const int r = m.rows[i];
    if (r < 0 || r >= m.table_rows) {
        set_error(err, RESA_DEVERR_ROW);
        return -1;
    }
    return r;
}

// seq_len of a cache row; an invalid row reads as an empty sequence.
__device__ __forceinline__ int row_seq_len(const int32_t *seq_len, int row) {
    return row >= 0 ? seq_len[row] : 0;
}

// Bounded grid barrier of a cooperatively launched (co-resident) grid; thread
// 0 of every CTA calls it after a __threadfence and a __syncthreads.  One
// 64-bit word holds (generation << 32) | arrivals: each CTA adds 1; the last
// arriver's single add of 2^32 - nctas returns the count to zero and bumps
// the generation, which the others poll for.  The count is zero between
// barriers, so grids of different sizes may share the word.  False when the
// wait gave up (the word is then left mid-barrier: the workspace must be
// re-initialised).
__device__ __forceinline__ bool grid_barrier_bounded(unsigned long long *bar, uint32_t nctas) {
    const unsigned long long old = atomicAdd(bar, 1ull);
    const uint32_t gen = (uint32_t)(old >> 32);
    if ((uint32_t)old == nctas - 1) {
        atomicAdd(bar, (1ull << 32) - nctas);
        return true;
    }
    volatile unsigned long long *vp = bar;
    for (uint32_t polls = 0; (uint32_t)(*vp >> 32) == gen;) {
        if (++polls > (1u << 22)) return false;  // each poll is an L2 round trip
    }
    return true;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t x) {
    return __uint_as_float(((uint32_t)x) << 16);
}
__device__ __forceinline__ float bf_lo(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf_hi(uint32_t pair) { return __uint_as_float(pair & 0xffff0000u); }

// Keep the earlier bit pattern on equality (matches a sequential scan).
__device__ __forceinline__ uint16_t bf_min(uint16_t cur, uint16_t x) {
    return bf16_bits_to_f32(x) < bf16_bits_to_f32(cur) ? x : cur;
}
__device__ __forceinline__ uint16_t bf_max(uint16_t cur, uint16_t x) {
    return bf16_bits_to_f32(x) > bf16_bits_to_f32(cur) ? x : cur;
}

// Eight bf16 channels (one 16-byte vector) as raw bit patterns.
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
// Fold x into a running element-wise (min, max) pair (Eq. 3).
__device__ __forceinline__ void fold8(Bf16x8 &mn, Bf16x8 &mx, const Bf16x8 &x) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        mn.v[i] = bf_min(mn.v[i], x.v[i]);
        mx.v[i] = bf_max(mx.v[i], x.v[i]);
    }
}

// Block scores as unsigned keys with the same order as the fp32 values
// (-0 and +0 map to one key, so equal scores get equal keys).
constexpr int kHistBins = 65536;  // histogram of the top 16 key bits
__device__ __forceinline__ uint32_t order_key(float s) {
    s += 0.0f;
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Byte-permute selector taking, for the two bf16 channels of a 32-bit word,
// the max half (from the second operand) where q >= 0 and the min half
// (first operand) otherwise: q * that value is max(q * max, q * min), the
// per-channel term of Eq. 4.
__device__ __forceinline__ uint32_t upper_bound_selector(float q0, float q1) {
    const uint32_t b0 = q0 >= 0.f ? 4u : 0u, b1 = q1 >= 0.f ? 4u : 0u;
    return (b0 + 0u) | ((b0 + 1u) << 4) | ((b1 + 2u) << 8) | ((b1 + 3u) << 12);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// mbarrier ------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: each try_wait suspends for a hardware-chosen interval; after
// kMaxPolls unsuccessful polls the wait gives up and reports false.
constexpr uint32_t kMaxPolls = 1u << 22;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kMaxPolls; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 16-byte asynchronous copy global -> shared through the load/store path
// (cp.async), grouped per thread with commit_group / wait_group.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// 4-byte asynchronous copy (through L1) for unaligned tails.
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// TMA: 3-D tiled bulk tensor load into shared memory, completion on an mbarrier.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// TMA: contiguous bulk copy global -> shared (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's completion and
// memory; allow the next grid to be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_next() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Warp-level tensor-core helpers (bf16 in, fp32 accumulate) ------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
// Split two fp32 weights into bf16 hi + lo parts (hi + lo carries ~16
// significant bits), packed as bf16x2 pairs for the MMA operand.
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(a, b);
    lo = pack_bf16(a - bf_lo(hi), b - bf_hi(hi));
}
// Transpose an 8x8 b16 matrix held one row-pair per lane (row lane/4,
// columns 2*(lane%4)+{0,1}) across the warp.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Byte offset of (row, 16-byte chunk) inside a tile written by TMA with
// CU_TENSOR_MAP_SWIZZLE_128B: rows are 128 bytes, chunk index XOR (row % 8).
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Raise a kernel's dynamic shared-memory limit once per device and process
// (an idempotent attribute; later calls, e.g. during CUDA-graph capture, only
// read a flag).
template <typename Kernel>
inline cudaError_t ensure_smem(Kernel kernel, int bytes, std::atomic<int> (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(1, std::memory_order_release);
    return e;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel in the stream drains; it must execute pdl_wait() before
// touching anything an earlier kernel writes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// Host-side launchers (defined in the kernel translation units)
// ---------------------------------------------------------------------------
struct Shape {
    int hq, hkv, g, d, bs;
    float sm_scale;
    int batch, max_pages, num_pages;
    RowMap rows;  // the cache's row map (rows == nullptr: identity)
};

cudaError_t launch_append(const Shape &s, void *k, void *v, void *desc, const int32_t *page_table,
                          const int32_t *seq_len, const void *k_new, const void *v_new,
                          uint32_t *err, cudaStream_t st);
cudaError_t launch_build_descriptors(const Shape &s, const void *k, void *desc,
                                     const int32_t *page_table, const int32_t *seq_len,
                                     const int32_t *first_block, uint32_t *err, cudaStream_t st);
cudaError_t launch_rectify_writeback(const Shape &s, void *k, void *v, void *desc,
                                     const int32_t *page_table, const int32_t *seq_len, int f,
                                     const void *k_new, const void *v_new, uint32_t *err,
                                     cudaStream_t st);
// Scores every complete block; with K != nullptr it also appends the decode
// token (k_new / v_new) in the same launch.
cudaError_t launch_score(const Shape &s, void *desc, const int32_t *page_table,
                         const int32_t *seq_len, const void *q, float *scores, uint32_t *hist,
                         uint32_t *hist_range, void *K, void *V, const void *k_new,
                         const void *v_new, uint32_t *err, cudaStream_t st);
cudaError_t launch_select(const Shape &s, const float *scores, uint32_t *hist,
                          uint32_t *hist_range, const int32_t *seq_len, const int32_t *topk,
                          int max_topk, int32_t *block_idx, int32_t *block_cnt, uint32_t *err,
                          cudaStream_t st);
// The decode-token append a dense decode does in the same launch (all null:
// none).  k / v / desc are the caches, k_new / v_new [batch][Hkv][d] bf16.
struct DecodeAppend {
    void *k = nullptr, *v = nullptr, *desc = nullptr;
    const uint4 *k_new = nullptr, *v_new = nullptr;
};
// block_idx == nullptr: dense decoding over every block of each sequence
// (block_cnt unused, max_topk + 1 taken as max_pages).
cudaError_t launch_sparse_decode(const Shape &s, const void *k, const void *v,
                                 const int32_t *page_table, const int32_t *seq_len, const void *q,
                                 const int32_t *block_idx, const int32_t *block_cnt, int max_topk,
                                 int splits, float *part_o, float *part_lse, uint32_t *tickets,
                                 uint32_t *grid_bar, float *out, float *lse, uint32_t *err,
                                 cudaStream_t st, const DecodeAppend &app = DecodeAppend());
// Fused decode step: append + scores + selection + sparse attention in one
// cooperative launch of G CTAs per (sequence, kv head) (step_ctas_per_unit).
struct StepBuffers {
    int32_t *block_idx, *block_cnt;  // selection output [B][Hkv][max_topk+1], [B][Hkv]
    uint32_t *hist, *hist_range;
    unsigned long long *bars;   // [B][Hkv][kStepBarWords]
    uint32_t *ukeys;
    unsigned long long *part;   // [kNumSms][kStepMaxGroup][d + 1]
    uint32_t *err;
};
cudaError_t launch_decode_step_fused(const Shape &s, int G, void *k, void *v, void *desc,
                                     const int32_t *page_table, const int32_t *seq_len,
                                     const void *q, const void *k_new, const void *v_new,
                                     const int32_t *topk, int max_topk, float *out, float *lse,
                                     const StepBuffers &buf, cudaStream_t st);
// maps: K half 0, K half 1, V half 0, V half 1 (2-D, 16 x 64 boxes, 128-byte swizzle),
// then the same four as 4-D maps whose box is one head on four consecutive pages.
cudaError_t launch_rectify_attention(const Shape &s, const CUtensorMap *maps,
                                     const int32_t *page_table, const int32_t *seq_len, int f,
                                     const void *q_chunk, int groups, int splits, float *part_o,
                                     float *part_lse, uint32_t *tickets, float *out, float *lse,
                                     uint32_t *err, cudaStream_t st);

}  // namespace resa
