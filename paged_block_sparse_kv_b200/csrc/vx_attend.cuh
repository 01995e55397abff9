// vx_attend.cuh -- one 16-token GQA attention tile on one warp, shared by the decode kernels.
//
// The tile's K and V rows (16 tokens x D bf16 each) sit in shared memory as written by TMA:
// D/64 boxes of 16 rows x 128 bytes with 128-byte swizzling.  S^T = K.Q^T with mma.m16n8k16
// (tokens x heads, heads padded to 8 per n-tile), online softmax in base 2 with tokens past
// nvalid masked, P^T moved into the B-operand layout with movmatrix, O^T += V^T.P^T with
// ldmatrix.trans for V.  Value rows past nvalid are zeroed in registers, so NaN in unused
// slots cannot leak.
#pragma once

#include "vx_internal.h"

namespace vx {

// qf: the group's query heads as mma B fragments; acc / m_run / l_run: the running output,
// maximum (log2 units) and sum of this warp's row.
template <int D, int NT>
__device__ __forceinline__ void attend_tile(uint32_t sK, uint32_t sV, int nvalid, float scale_log2,
                                            const uint32_t (&qf)[NT][D / 16][2], float (&acc)[NT][D / 16][4],
                                            float (&m_run)[NT][2], float (&l_run)[NT][2], int lane) {
    constexpr int MT = D / 16;
    constexpr int BOX_BYTES = DEC_TILE * 128;
    const int g4 = lane >> 2, q4 = lane & 3;
    // S^T[token][head] = K . Q^T
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
    {
        const int mi = lane >> 3, rr = lane & 7;
        const int tok = rr + 8 * (mi & 1);
#pragma unroll
        for (int kk = 0; kk < MT; ++kk) {
            const int chunk = (kk & 3) * 2 + (mi >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(sK + (kk >> 2) * BOX_BYTES + swz128(tok, chunk), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
        }
    }
    // online softmax (base 2), tokens >= nvalid masked
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int tok = g4 + 8 * (e >> 1);
            x[e] = tok < nvalid ? s[nt][e] * scale_log2 : -INFINITY;
        }
        float alpha[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = fmaxf(x[i], x[i + 2]);
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
            const float m_new = fmaxf(m_run[nt][i], mx);
            alpha[i] = exp2f(m_run[nt][i] - m_new);
            m_run[nt][i] = m_new;
        }
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = exp2f(x[e] - m_run[nt][e & 1]);
#pragma unroll
        for (int i = 0; i < 2; ++i) l_run[nt][i] = l_run[nt][i] * alpha[i] + p[i] + p[i + 2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][mt][e] *= alpha[e & 1];
        pb[nt][0] = movmatrix_t(pack_bf16x2(p[0], p[1]));
        pb[nt][1] = movmatrix_t(pack_bf16x2(p[2], p[3]));
    }
    // O^T[dim][head] += V^T . P^T
    {
        const int mi = lane >> 3, rr = lane & 7;
        const int tok = rr + 8 * (mi >> 1);
        const bool tail = nvalid < DEC_TILE;
        const int t_lo = 2 * q4, t_hi = 8 + 2 * q4;  // tokens of this lane's A halves
        const uint32_t mlo = (t_lo < nvalid ? 0x0000ffffu : 0u) | (t_lo + 1 < nvalid ? 0xffff0000u : 0u);
        const uint32_t mhi = (t_hi < nvalid ? 0x0000ffffu : 0u) | (t_hi + 1 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int chunk = (mt & 3) * 2 + (mi & 1);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(sV + (mt >> 2) * BOX_BYTES + swz128(tok, chunk), v0, v1, v2, v3);
            if (tail) {
                v0 &= mlo;
                v1 &= mlo;
                v2 &= mhi;
                v3 &= mhi;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt][mt], v0, v1, v2, v3, pb[nt][0], pb[nt][1]);
        }
    }
}

}  // namespace vx
