// Warp-level attention over one 16-token K/V tile held in shared memory in the
// layout a 128-byte-swizzled TMA load writes: token t, channel half c occupies
// 128-byte row t * (D / 64) + c.  One warp owns 16 query rows; logits and
// P.V use bf16 m16n8k16 tensor-core MMAs with fp32 accumulators, softmax runs
// online in base 2 (FlashAttention's running max / sum, as the kernel section
// of the ReSA summary, §3.4.4, describes for each split).
#pragma once

#include "resa_common.cuh"

namespace resa {

// Online-softmax state of the two rows a lane holds (rows lane/4 and lane/4 + 8).
template <int D>
struct RowState {
    float m[2];          // running max of the base-2 logits
    float l[2];          // this lane's share of the running sum of the weights
    float lx[2];         // copy of l kept for the log-sum-exp
    float acc[D / 8][4]; // O accumulators: n-tile j covers channels 8j .. 8j+7
    __device__ __forceinline__ void init() {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
        lx[0] = lx[1] = 0.f;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    }
};

// Load the A fragments of 16 query rows (row r taken from row_ptr[r], NULL =
// zero row) for all D/16 k-slices.  row_ptr points at bf16 [D].
template <int D>
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[D / 16][4], const uint16_t *row0,
                                             const uint16_t *row1, int lane) {
    const int c = 2 * (lane & 3);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const int k0 = ks * 16 + c;
        qa[ks][0] = row0 ? *reinterpret_cast<const uint32_t *>(row0 + k0) : 0u;
        qa[ks][1] = row1 ? *reinterpret_cast<const uint32_t *>(row1 + k0) : 0u;
        qa[ks][2] = row0 ? *reinterpret_cast<const uint32_t *>(row0 + k0 + 8) : 0u;
        qa[ks][3] = row1 ? *reinterpret_cast<const uint32_t *>(row1 + k0 + 8) : 0u;
    }
}

// One 16-token tile: k_tile / v_tile are shared-memory addresses (1024-byte
// aligned) of the swizzled [16][D] bf16 tiles.  nvalid0 / nvalid1: tokens
// 0 .. nvalid-1 of the tile are visible to row0 / row1 (others get weight 0).
template <int D>
__device__ __forceinline__ void attend_tile16(RowState<D> &st, const uint32_t (&qa)[D / 16][4],
                                              uint32_t k_tile, uint32_t v_tile, int nvalid0,
                                              int nvalid1, float scale_log2, int lane) {
    constexpr int HALVES = D / 64;
    float s[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
    // S = Q K^T : ldmatrix rows = tokens (B operand, column-major K x N).
    {
        const int tok = (lane & 7) + ((lane >> 4) << 3);
        const int dsub = ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int dim = ks * 16 + dsub;
            const uint32_t row = tok * HALVES + dim / 64;
            uint32_t r[4];
            ldmatrix_x4(r, k_tile + swz128(row, (dim % 64) / 8));
            mma_bf16_16816(s[0], qa[ks], r[0], r[1]);
            mma_bf16_16816(s[1], qa[ks], r[2], r[3]);
        }
    }
    // Online softmax (base 2).  Column of s[n][e]: n*8 + 2*(lane%4) + (e & 1);
    // row: e < 2 -> row0, else row1.
    const int cb = 2 * (lane & 3);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = n * 8 + cb + (e & 1);
            const int nv = e < 2 ? nvalid0 : nvalid1;
            const float x = col < nv ? s[n][e] * scale_log2 : -INFINITY;
            s[n][e] = x;
            mx[e >> 1] = fmaxf(mx[e >> 1], x);
        }
    float alpha[2], base[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float mnew = fmaxf(st.m[r], mx[r]);
        base[r] = mnew == -INFINITY ? 0.f : mnew;
        alpha[r] = exp2f(st.m[r] - base[r]);
        st.m[r] = mnew;
    }
    // P enters the P.V MMA as bf16 hi + lo parts (two MMAs), so the weights
    // keep ~16 significant bits: rows that see only a few tokens stay within
    // the fp32-accumulation error budget.
    uint32_t pa[4], pl[4];
    float psum[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < 2; ++n) {
        const float p0 = exp2f(s[n][0] - base[0]), p1 = exp2f(s[n][1] - base[0]);
        const float p2 = exp2f(s[n][2] - base[1]), p3 = exp2f(s[n][3] - base[1]);
        split_bf16(p0, p1, pa[2 * n], pl[2 * n]);
        split_bf16(p2, p3, pa[2 * n + 1], pl[2 * n + 1]);
        psum[0] += p0 + p1;
        psum[1] += p2 + p3;
    }
    st.l[0] = st.l[0] * alpha[0] + psum[0];
    st.l[1] = st.l[1] * alpha[1] + psum[1];
    st.lx[0] = st.l[0];
    st.lx[1] = st.l[1];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        st.acc[j][0] *= alpha[0];
        st.acc[j][1] *= alpha[0];
        st.acc[j][2] *= alpha[1];
        st.acc[j][3] *= alpha[1];
    }
    // O += P V : ldmatrix.trans rows = tokens (B operand, row-major K x N).
    {
        const int tok = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dsub = (lane >> 4) * 8;
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
            const int dim = np * 16 + dsub;
            const uint32_t row = tok * HALVES + dim / 64;
            uint32_t r[4];
            ldmatrix_x4_trans(r, v_tile + swz128(row, (dim % 64) / 8));
            mma_bf16_16816(st.acc[2 * np], pa, r[0], r[1]);
            mma_bf16_16816(st.acc[2 * np + 1], pa, r[2], r[3]);
            mma_bf16_16816(st.acc[2 * np], pl, r[0], r[1]);
            mma_bf16_16816(st.acc[2 * np + 1], pl, r[2], r[3]);
        }
    }
}

// Sum each row's l over the four lanes that share it.
template <int D>
__device__ __forceinline__ void finish_rows(RowState<D> &st) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        st.l[r] += __shfl_xor_sync(0xffffffffu, st.l[r], 1);
        st.l[r] += __shfl_xor_sync(0xffffffffu, st.l[r], 2);
        st.lx[r] += __shfl_xor_sync(0xffffffffu, st.lx[r], 1);
        st.lx[r] += __shfl_xor_sync(0xffffffffu, st.lx[r], 2);
    }
}

}  // namespace resa
