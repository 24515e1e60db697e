// tc5_solve.cuh -- the UT transform of one chunk, T = (I + A)^{-1} for the
// strictly lower 64x64 A of the chunkwise WY form ("Gated Delta Networks:
// Improving Mamba2 with Delta Rule" (paper review), section "Method").
//
// The 16x16 diagonal blocks of T are exact in fp32 registers (forward
// substitution, one warp per block, lane c owning column c); the off-diagonal
// blocks follow one block diagonal at a time with warp-level MMAs:
//   T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ.
// These 16x16 products are far below the size of one tcgen05 instruction, so
// they stay on mma.sync.
#pragma once
#include "common.cuh"
#include "mma.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace tc {

// Ad: fp32 diagonal blocks of A; Abf: bf16 A (Swz<64>); T: the result
// (Swz<64>); Xs: four 16x16 bf16 scratch tiles.  Warps 0..3 compute; every
// thread of the CTA calls (the block diagonals are separated by CTA barriers).
GDN_DEV void ut_solve(const float (*Ad)[16][17], const __nv_bfloat16* Abf, __nv_bfloat16* T,
                      __nv_bfloat16 (*Xs)[16 * 16]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int m0 = 16 * warp;
    if (warp < 4) {
        const int c = lane & 15;
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float v = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) v -= Ad[warp][i][j] * t[j];
            t[i] = (i < c) ? 0.f : v;
        }
        if (lane < 16) {
#pragma unroll
            for (int i = 0; i < 16; ++i) T[swz<C>(m0 + i, m0 + c)] = __float2bfloat16_rn(t[i]);
        }
        // zero this warp's row block right of the diagonal block
        for (int e = lane; e < 16 * C; e += 32) {
            const int r = e >> 6, cc = e & 63;
            if (cc >= m0 + 16) T[swz<C>(m0 + r, cc)] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();
    for (int dgl = 1; dgl < 4; ++dgl) {
        const int J = warp, I = warp + dgl;
        if (warp < 4 && I < 4) {
            float x[2][4] = {};
            for (int Kb = J; Kb < I; ++Kb) {
                uint32_t a[4], bt[4];
                lda<Swz<64>>(a, Abf, 16 * I, 16 * Kb);
                ldb_kn<Swz<64>>(bt, T, 16 * Kb, 16 * J);
                mma16816(x[0], a, bt[0], bt[1]);
                mma16816(x[1], a, bt[2], bt[3]);
            }
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                const int r = lane >> 2, cc = 8 * jn + 2 * (lane & 3);
                *reinterpret_cast<uint32_t*>(&Xs[warp][r * 16 + cc]) = pack_bf16(x[jn][0], x[jn][1]);
                *reinterpret_cast<uint32_t*>(&Xs[warp][(r + 8) * 16 + cc]) = pack_bf16(x[jn][2], x[jn][3]);
            }
            __syncwarp();
            uint32_t a[4], bx[4];
            lda<Swz<64>>(a, T, 16 * I, 16 * I);
            {
                const int idx = lane >> 3;
                const int row = (lane & 7) + (idx & 1) * 8, col = (idx >> 1) * 8;
                ldsm_x4_t(bx, smem_u32(&Xs[warp][row * 16 + col]));
            }
            float y[2][4] = {};
            mma16816(y[0], a, bx[0], bx[1]);
            mma16816(y[1], a, bx[2], bx[3]);
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                float z[4] = {-y[jn][0], -y[jn][1], -y[jn][2], -y[jn][3]};
                st_c<Swz<64>>(T, 16 * I, 16 * J + 8 * jn, z);
            }
        }
        __syncthreads();
    }
}

}  // namespace tc
}  // namespace gdn
