// Block key cache kernels: descriptor build / refresh, decode-token append and
// rectification write-back (ReSA summary §3.2 "Block Key Cache", Eq. 3;
// Algorithm 1 incremental update; §3.4.2 descriptor recomputation).
//
// One thread owns 8 consecutive channels (one 16-byte vector) of one
// (page, kv head) row and scans the block's tokens in position order, so the
// min / max keep the same bit pattern a sequential scan keeps.  A warp reads
// whole 256-byte key rows: every load is a coalesced 16-byte vector.
#include "resa_common.cuh"

namespace resa {
namespace {

__device__ __forceinline__ size_t kv_off(int page, int h, int slot, int c, int hkv, int d,
                                         int bs) {
    return ((((size_t)page * hkv + h) * bs + slot) * d) / 8 + c;  // in uint4 units
}
__device__ __forceinline__ size_t desc_off(int page, int h, int which, int c, int hkv, int d) {
    return ((((size_t)page * hkv + h) * 2 + which) * d) / 8 + c;  // in uint4 units
}

// grid (batch), block (hkv * d/8)
__global__ void append_kernel(uint4 *__restrict__ K, uint4 *__restrict__ V,
                              uint4 *__restrict__ desc, const int32_t *__restrict__ page_table,
                              const int32_t *__restrict__ seq_len, const uint4 *__restrict__ k_new,
                              const uint4 *__restrict__ v_new, int hkv, int d, int max_pages,
                              int num_pages, int bs, const RowMap rm, uint32_t *err) {
    const int b = blockIdx.x;
    const int cpr = d / 8;  // 16-byte chunks per row
    const int h = threadIdx.x / cpr, c = threadIdx.x % cpr;
    if (h >= hkv) return;
    const int row = cache_row(rm, b, threadIdx.x == 0 ? err : nullptr);
    const int L = row_seq_len(seq_len, row);
    if (L < 1 || L > max_pages * bs) {
        if (threadIdx.x == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        return;
    }
    const int pos = L - 1;
    const int page = page_table[(size_t)row * max_pages + pos / bs];
    if (page < 0 || page >= num_pages) {
        if (threadIdx.x == 0) set_error(err, RESA_DEVERR_PAGE);
        return;
    }
    const int slot = pos % bs;
    const size_t src = (((size_t)b * hkv + h) * d) / 8 + c;
    const uint4 kx = k_new[src];
    const uint4 vx = v_new[src];
    K[kv_off(page, h, slot, c, hkv, d, bs)] = kx;
    V[kv_off(page, h, slot, c, hkv, d, bs)] = vx;
    uint4 *pmn = &desc[desc_off(page, h, 0, c, hkv, d)];
    uint4 *pmx = &desc[desc_off(page, h, 1, c, hkv, d)];
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

constexpr int kBuildThreads = 256;
constexpr int kBuildPagesPerCta = 16;

// grid (ceil(max_pages / kBuildPagesPerCta), batch), block kBuildThreads.
// Rebuilds blocks [first, ceil(L / b)) of each sequence.
__global__ void __launch_bounds__(kBuildThreads, 2)  // two CTAs an SM: twice the loads in flight
    build_desc_kernel(const uint4 *__restrict__ K, uint4 *__restrict__ desc,
                      const int32_t *__restrict__ page_table, const int32_t *__restrict__ seq_len,
                      const int32_t *__restrict__ first_block, int hkv, int d, int max_pages,
                      int num_pages, int bs, const RowMap rm, uint32_t *err) {
    const int b = blockIdx.y;
    const int cpr = d / 8;
    const int tpp = hkv * cpr;                 // threads per page
    const int ppp = kBuildThreads / tpp;       // pages per pass
    const int sub = threadIdx.x / tpp;
    const int h = (threadIdx.x % tpp) / cpr, c = threadIdx.x % cpr;
    if (sub >= ppp) return;
    const int row = cache_row(rm, b, threadIdx.x == 0 && blockIdx.x == 0 ? err : nullptr);
    const int L = row_seq_len(seq_len, row);
    if (L < 0 || L > max_pages * bs) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        return;
    }
    const int nblk = (L + bs - 1) / bs;
    const int first = first_block ? max(0, first_block[b]) : 0;
    const int blk0 = blockIdx.x * kBuildPagesPerCta;
    for (int blk = blk0 + sub; blk < blk0 + kBuildPagesPerCta; blk += ppp) {
        if (blk < first || blk >= nblk) continue;
        const int page = page_table[(size_t)row * max_pages + blk];
        if (page < 0 || page >= num_pages) {
            if (h == 0 && c == 0) set_error(err, RESA_DEVERR_PAGE);
            continue;
        }
        const int nt = min(bs, L - blk * bs);
        // 16 tokens at a time: their loads in flight together, then the
        // position-order fold
        Bf16x8 mn, mx;
        for (int t0 = 0; t0 < nt; t0 += kTileRows) {
            uint4 x[kTileRows];
#pragma unroll
            for (int t = 0; t < kTileRows; ++t)
                if (t0 + t < nt) x[t] = K[kv_off(page, h, t0 + t, c, hkv, d, bs)];
            if (t0 == 0) {
                mn = unpack8(x[0]);
                mx = mn;
            }
#pragma unroll
            for (int t = 0; t < kTileRows; ++t)
                if (t0 + t < nt && t0 + t > 0) fold8(mn, mx, unpack8(x[t]));
        }
        desc[desc_off(page, h, 0, c, hkv, d)] = pack8(mn);
        desc[desc_off(page, h, 1, c, hkv, d)] = pack8(mx);
    }
}

// grid (f / b + 2, batch), block (hkv * d/8).  Block (L-f)/b + blockIdx.x:
// writes the chunk's fresh K/V into its positions >= L-f and rebuilds its
// descriptor from the updated keys in the same pass.
__global__ void rectify_writeback_kernel(uint4 *__restrict__ K, uint4 *__restrict__ V,
                                         uint4 *__restrict__ desc,
                                         const int32_t *__restrict__ page_table,
                                         const int32_t *__restrict__ seq_len, int f,
                                         const uint4 *__restrict__ k_new,
                                         const uint4 *__restrict__ v_new, int hkv, int d,
                                         int max_pages, int num_pages, int bs,
                                         const RowMap rm, uint32_t *err) {
    const int b = blockIdx.y;
    const int cpr = d / 8;
    const int h = threadIdx.x / cpr, c = threadIdx.x % cpr;
    if (h >= hkv) return;
    const int row = cache_row(rm, b, threadIdx.x == 0 && blockIdx.x == 0 ? err : nullptr);
    const int L = row_seq_len(seq_len, row);
    if (L < 1 || L > max_pages * bs) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_error(err, RESA_DEVERR_SEQ_LEN);
        return;
    }
    if (f > L) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_error(err, RESA_DEVERR_CHUNK);
        return;
    }
    const int start = L - f;
    const int blk = start / bs + blockIdx.x;
    if (blk > (L - 1) / bs) return;
    const int page = page_table[(size_t)row * max_pages + blk];
    if (page < 0 || page >= num_pages) {
        if (threadIdx.x == 0) set_error(err, RESA_DEVERR_PAGE);
        return;
    }
    const int nt = min(bs, L - blk * bs);
    // 16 tokens at a time: all their loads first (fresh chunk values or the
    // cached keys), then the writes and the position-order min/max fold.
    Bf16x8 mn, mx;
    for (int t0 = 0; t0 < nt; t0 += kTileRows) {
        uint4 kx[kTileRows], vx[kTileRows];
#pragma unroll
        for (int t = 0; t < kTileRows; ++t) {
            const int pos = blk * bs + t0 + t;
            if (t0 + t < nt) {
                if (pos >= start) {
                    const size_t src = ((((size_t)b * f + (pos - start)) * hkv + h) * d) / 8 + c;
                    kx[t] = k_new[src];
                    vx[t] = v_new[src];
                } else {
                    kx[t] = K[kv_off(page, h, t0 + t, c, hkv, d, bs)];
                }
            }
        }
        if (t0 == 0) {
            mn = unpack8(kx[0]);
            mx = mn;
        }
#pragma unroll
        for (int t = 0; t < kTileRows; ++t) {
            const int pos = blk * bs + t0 + t;
            if (t0 + t < nt && pos >= start) {
                const size_t o = kv_off(page, h, t0 + t, c, hkv, d, bs);
                K[o] = kx[t];
                V[o] = vx[t];
            }
            if (t0 + t > 0 && t0 + t < nt) fold8(mn, mx, unpack8(kx[t]));
        }
    }
    desc[desc_off(page, h, 0, c, hkv, d)] = pack8(mn);
    desc[desc_off(page, h, 1, c, hkv, d)] = pack8(mx);
}

}  // namespace

cudaError_t launch_append(const Shape &s, void *k, void *v, void *desc, const int32_t *page_table,
                          const int32_t *seq_len, const void *k_new, const void *v_new,
                          uint32_t *err, cudaStream_t st) {
    append_kernel<<<s.batch, s.hkv * (s.d / 8), 0, st>>>(
        (uint4 *)k, (uint4 *)v, (uint4 *)desc, page_table, seq_len, (const uint4 *)k_new,
        (const uint4 *)v_new, s.hkv, s.d, s.max_pages, s.num_pages, s.bs, s.rows, err);
    return cudaGetLastError();
}

cudaError_t launch_build_descriptors(const Shape &s, const void *k, void *desc,
                                     const int32_t *page_table, const int32_t *seq_len,
                                     const int32_t *first_block, uint32_t *err, cudaStream_t st) {
    dim3 grid((s.max_pages + kBuildPagesPerCta - 1) / kBuildPagesPerCta, s.batch);
    build_desc_kernel<<<grid, kBuildThreads, 0, st>>>((const uint4 *)k, (uint4 *)desc, page_table,
                                                      seq_len, first_block, s.hkv, s.d,
                                                      s.max_pages, s.num_pages, s.bs, s.rows,
                                                      err);
    return cudaGetLastError();
}

cudaError_t launch_rectify_writeback(const Shape &s, void *k, void *v, void *desc,
                                     const int32_t *page_table, const int32_t *seq_len, int f,
                                     const void *k_new, const void *v_new, uint32_t *err,
                                     cudaStream_t st) {
    dim3 grid(f / s.bs + 2, s.batch);
    rectify_writeback_kernel<<<grid, s.hkv * (s.d / 8), 0, st>>>(
        (uint4 *)k, (uint4 *)v, (uint4 *)desc, page_table, seq_len, f, (const uint4 *)k_new,
        (const uint4 *)v_new, s.hkv, s.d, s.max_pages, s.num_pages, s.bs, s.rows, err);
    return cudaGetLastError();
}

}  // namespace resa
