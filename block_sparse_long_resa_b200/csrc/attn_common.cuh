// Warp-level group attention over one 16-token K/V block held in shared
// memory (GBSA, ReSA summary §3.4.1 Eq. 2): the g <= 16 query heads of a GQA
// group share the block's K and V.  The tiles are laid out as a 128-byte
// swizzled TMA load writes them: token t, channel half c occupies 128-byte row
// t * (D / 64) + c.  The MMAs run with the operands swapped, S^T = K Q^T and
// O^T = V^T P^T (bf16 m16n8k16, fp32 accumulate), so the heads fill the N = 8
// side; softmax runs online in base 2 (FlashAttention's running max / sum per
// split, as the kernel section §3.4.4 describes); P^T is transposed in
// registers with movmatrix and enters the P.V MMA as bf16 hi + lo parts so the
// weights keep ~16 significant bits.
#pragma once

#include "resa_common.cuh"

namespace resa {

// Per-warp attention state in the swapped layout: lane holds heads
// nt*8 + 2*(lane%4) + {0,1} and, of O^T, channels mt*16 + lane/4 (+8).
template <int D, int NT>
struct WarpState {
    float m[NT][2];
    float l[NT][2];
    float o[D / 16][NT][4];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            m[n][0] = m[n][1] = -INFINITY;
            l[n][0] = l[n][1] = 0.f;
#pragma unroll
            for (int t = 0; t < D / 16; ++t) o[t][n][0] = o[t][n][1] = o[t][n][2] = o[t][n][3] = 0.f;
        }
    }
};

// One 16-token block: K / V tiles at shared addresses k_tile / v_tile;
// tokens >= ntok are masked.  qb: B fragments of Q^T (channels x heads).
template <int D, int NT>
__device__ __forceinline__ void attend_block_swapped(WarpState<D, NT> &st,
                                                     const uint32_t (&qb)[D / 16][NT][2],
                                                     uint32_t k_tile, uint32_t v_tile, int ntok,
                                                     float scale_log2, int lane) {
    constexpr int HALVES = D / 64;
    float s[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
    {  // S^T = K Q^T: A = K tile (tokens x channels), ldmatrix rows = tokens
        const int tok = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dsub = (lane >> 4) * 8;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int dim = ks * 16 + dsub;
            uint32_t a[4];
            ldmatrix_x4(a, k_tile + swz128(tok * HALVES + dim / 64, (dim % 64) / 8));
#pragma unroll
            for (int n = 0; n < NT; ++n) mma_bf16_16816(s[n], a, qb[ks][n][0], qb[ks][n][1]);
        }
    }
    // Column (= head) softmax.  s[n][e]: token lane/4 + 8*(e>=2), head 2*(lane%4) + (e&1).
    const int t0 = lane >> 2;
    uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int tok = t0 + ((e >> 1) << 3);
            x[e] = tok < ntok ? s[n][e] * scale_log2 : -INFINITY;
        }
        float cm[2] = {fmaxf(x[0], x[2]), fmaxf(x[1], x[3])};
        float alpha[2], base[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            cm[k] = fmaxf(cm[k], __shfl_xor_sync(0xffffffffu, cm[k], 4));
            cm[k] = fmaxf(cm[k], __shfl_xor_sync(0xffffffffu, cm[k], 8));
            cm[k] = fmaxf(cm[k], __shfl_xor_sync(0xffffffffu, cm[k], 16));
            const float mnew = fmaxf(st.m[n][k], cm[k]);
            base[k] = mnew == -INFINITY ? 0.f : mnew;
            alpha[k] = exp2f(st.m[n][k] - base[k]);
            st.m[n][k] = mnew;
        }
        const float p0 = exp2f(x[0] - base[0]), p1 = exp2f(x[1] - base[1]);
        const float p2 = exp2f(x[2] - base[0]), p3 = exp2f(x[3] - base[1]);
        st.l[n][0] = st.l[n][0] * alpha[0] + p0 + p2;
        st.l[n][1] = st.l[n][1] * alpha[1] + p1 + p3;
#pragma unroll
        for (int t = 0; t < D / 16; ++t) {
            st.o[t][n][0] *= alpha[0];
            st.o[t][n][1] *= alpha[1];
            st.o[t][n][2] *= alpha[0];
            st.o[t][n][3] *= alpha[1];
        }
        // P^T (tokens x heads) as bf16 hi + lo, transposed into B fragments.
        uint32_t h01, l01, h23, l23;
        split_bf16(p0, p1, h01, l01);  // tokens 0..7 rows
        split_bf16(p2, p3, h23, l23);  // tokens 8..15 rows
        bh[n][0] = movmatrix_trans(h01);
        bh[n][1] = movmatrix_trans(h23);
        bl[n][0] = movmatrix_trans(l01);
        bl[n][1] = movmatrix_trans(l23);
    }
    {  // O^T += V^T P^T: A = V^T (channels x tokens) via ldmatrix.trans of V rows
        const int tok = (lane & 7) + (lane >> 4) * 8;
        const int dsub = ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            const int dim = mt * 16 + dsub;
            uint32_t a[4];
            ldmatrix_x4_trans(a, v_tile + swz128(tok * HALVES + dim / 64, (dim % 64) / 8));
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                mma_bf16_16816(st.o[mt][n], a, bh[n][0], bh[n][1]);
                mma_bf16_16816(st.o[mt][n], a, bl[n][0], bl[n][1]);
            }
        }
    }
}

}  // namespace resa
