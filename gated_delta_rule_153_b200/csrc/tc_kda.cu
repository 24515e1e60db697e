// tc_kda.cu -- chunk preparation for the channel-wise gate (Kimi Delta Attention).
//
// Same recurrence with Diag(a_t) on the key index in place of the scalar a_t
// (the channel-gate reading of "Gated Delta Networks: Improving Mamba2 with
// Delta Rule", section "Method"; the variant is named in the review's linked
// reviews and in "Linear Attention Architectures: Mechanisms, Trade-offs, and
// Cross-Layer Routing").  With G the per-channel within-chunk cumsum of g,
//   A_ij = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}          (j < i)
//   P_ij = scale sum_c q_ic k_jc e^{G_ic - G_jc}           (j <= i)
//   W = T diag(beta) (K .* e^G),  U~ = T diag(beta) V,  T = (I + A)^{-1}
// and the walk needs Qg = scale Q .* e^G, Kt = K .* e^{G_last - G} and the
// per-key chunk decay e^{G_last}.
//
// The decay sits inside the contraction, so the products are factorised
// with reference rows chosen to keep every factor at most 1 (no overflow;
// a factor that underflows means the true term is smaller still).  For a
// block pair (I, J), J < I, of 16-token blocks, with f = first row of I and
// l = last row of J:
//   e^{G_ic - G_jc} = e^{G_ic - G_fc} * e^{G_fc - G_lc} * e^{G_lc - G_jc}
//                   = EL_ic * F_IJc * ER_jc,      all three <= 1,
// so A_IJ = diag(beta_I) ((K_I .* EL_I) diag(F_IJ)) (K_J .* ER_J)^T on the
// tensor cores, the per-channel F_IJ scaling the A fragments in registers.
// Inside a diagonal block the second factor would be e^{G_fc - G_jc} >= 1;
// the MMA form is used when max_c (G_fc - G_{f+15,c}) <= 80 (the factor stays
// below e^80, far inside fp32/bf16 range) and an exact elementwise sum
// otherwise.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace tc {
namespace {

using S128 = Swz<128>;
using S64 = Swz<64>;

struct KdaPrepSmem {
    __nv_bfloat16 K[C * DK];    // Tma128 (TMA)
    __nv_bfloat16 Q[C * DK];    // Tma128 (TMA); later Qg image
    __nv_bfloat16 V[C * DV];    // Tma128 (TMA)
    __nv_bfloat16 Kl[C * DK];   // K .* EL; later K .* e^G (W operand), then W image
    __nv_bfloat16 Ql[C * DK];   // Q .* EL; later Kt image
    __nv_bfloat16 Kr[C * DK];   // K .* ER; later U~ staging
    __nv_bfloat16 Kd[C * DK];   // K .* e^{G_f - G} (diagonal blocks whose span passed)
    float G[C][DK];             // per-channel cumsum
    __nv_bfloat16 P[C * C];     // Swz<64> image
    __nv_bfloat16 Ab[C * C];
    __nv_bfloat16 Tb[C * C];
    __nv_bfloat16 X[4][16 * 16];
    float Ad[4][16][17];
    float F[6][DK];             // F_IJ per channel for the six block pairs J < I
    float gl[DK];               // e^{G_last,c}
    float beta[C];
    int diag_ok[4];
    uint64_t bar;
};

__device__ __forceinline__ int pair_index(int I, int J) { return I * (I - 1) / 2 + J; }

GDN_DEV void scale_a_cols_f(uint32_t (&a)[4], const float* f, int k0) {
    const int l = threadIdx.x & 31;
    const int k = k0 + 2 * (l & 3);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int kk = k + (r >> 1) * 8;
        float2 v = unpack_bf16(a[r]);
        a[r] = pack_bf16(v.x * f[kk], v.y * f[kk + 1]);
    }
}

__global__ void __launch_bounds__(128) tc_prep_kda_kernel(const __grid_constant__ ChunkPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    KdaPrepSmem& s = *reinterpret_cast<KdaPrepSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, b = bh / p.H, h = bh % p.H;
    const int t0 = n * C;
    const int L = min(C, p.T - t0);
    const size_t row0 = ((size_t)b * p.T + t0) * p.H + h;
    const size_t rs = (size_t)p.H;

    if (tid == 0) {
        mbar_init(&s.bar, 1);
        fence_mbar_init();
        mbar_arrive_expect(&s.bar, 3 * C * DK * 2);
        const int tok = b * p.T + t0;
        tma_load_tile(s.K, &p.kmap, h, tok, &s.bar);
        tma_load_tile(s.Q, &p.qmap, h, tok, &s.bar);
        tma_load_tile(s.V, &p.vmap, h, tok, &s.bar);
    }
    // log-gates (rows past the sequence end add 0) and beta
    for (int e = tid; e < C * (DK / 4); e += 128) {
        const int r = e / (DK / 4), c4 = e % (DK / 4);
        const bool ok = r < L;
        cp_async16_zfill(&s.G[r][4 * c4], p.g + (row0 + (size_t)(ok ? r : 0) * rs) * DK + 4 * c4, ok);
    }
    cp_async_commit();
    if (tid < C) s.beta[tid] = tid < L ? p.beta[row0 + tid * rs] : 0.f;
    cp_async_wait<0>();
    __syncthreads();
    {   // per-channel cumsum: thread c owns channel c
        const int c = tid;
        float run = 0.f;
        for (int i = 0; i < C; ++i) {
            run += s.G[i][c];
            s.G[i][c] = run;
        }
        s.gl[c] = __expf(run);
    }
    __syncthreads();
    if (__syncthreads_or(!mbar_wait(&s.bar, 0, p.status))) return;

    // block spans and the six pair factors F_IJ
    if (warp < 4) {
        float sp = 0.f;
        for (int c = lane; c < DK; c += 32) sp = fmaxf(sp, s.G[16 * warp][c] - s.G[16 * warp + 15][c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sp = fmaxf(sp, __shfl_xor_sync(0xffffffffu, sp, o));
        if (lane == 0) s.diag_ok[warp] = sp <= 80.f;
    }
    for (int e = tid; e < 6 * DK; e += 128) {
        const int pi = e / DK, c = e % DK;
        const int I = pi < 1 ? 1 : (pi < 3 ? 2 : 3);
        const int J = pi - I * (I - 1) / 2;
        s.F[pi][c] = __expf(s.G[16 * I][c] - s.G[16 * J + 15][c]);
    }
    // scaled operands
    for (int e = tid; e < C * DK; e += 128) {
        const int i = e / DK, c = e % DK;
        const int f = i & ~15, l = f + 15;
        const float g = s.G[i][c];
        const uint32_t o = Tma128::off(i, c);
        const float kv = __bfloat162float(s.K[o]), qv = __bfloat162float(s.Q[o]);
        const float el = __expf(g - s.G[f][c]);
        s.Kl[o] = __float2bfloat16_rn(kv * el);
        s.Ql[o] = __float2bfloat16_rn(qv * el);
        s.Kr[o] = __float2bfloat16_rn(kv * __expf(s.G[l][c] - g));
        const float sp = s.G[f][c] - g;  // >= 0
        s.Kd[o] = __float2bfloat16_rn(sp <= 80.f ? kv * __expf(sp) : 0.f);
    }
    __syncthreads();

    const int m0 = 16 * warp, I = warp;
    // ---- A and P, row block I -------------------------------------------
    {
        float acck[4][2][4], accq[4][2][4];  // [J][n-tile][e]
#pragma unroll
        for (int J = 0; J < 4; ++J)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) acck[J][t][e] = accq[J][t][e] = 0.f;
        const bool dok = s.diag_ok[I];
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t ak0[4], aq0[4];
            lda<Tma128>(ak0, s.Kl, m0, 16 * kk);
            lda<Tma128>(aq0, s.Ql, m0, 16 * kk);
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                if (J > I) break;
                uint32_t ak[4], aq[4], bf[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) { ak[r] = ak0[r]; aq[r] = aq0[r]; }
                if (J < I) {
                    scale_a_cols_f(ak, s.F[pair_index(I, J)], 16 * kk);
                    scale_a_cols_f(aq, s.F[pair_index(I, J)], 16 * kk);
                    ldb_nk<Tma128>(bf, s.Kr, 16 * J, 16 * kk);
                } else {
                    if (!dok) break;
                    ldb_nk<Tma128>(bf, s.Kd, 16 * J, 16 * kk);
                }
                mma16816(acck[J][0], ak, bf[0], bf[1]);
                mma16816(acck[J][1], ak, bf[2], bf[3]);
                mma16816(accq[J][0], aq, bf[0], bf[1]);
                mma16816(accq[J][1], aq, bf[2], bf[3]);
            }
        }
        const int ra = m0 + (lane >> 2), rb = ra + 8;
#pragma unroll
        for (int J = 0; J < 4; ++J) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int c0 = 16 * J + 8 * t + 2 * (lane & 3);
                float a[4], pv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = (e < 2) ? ra : rb, c = c0 + (e & 1);
                    const bool live = J < I || (J == I && dok);
                    a[e] = (live && c < r) ? s.beta[r] * acck[J][t][e] : 0.f;
                    pv[e] = (live && c <= r && r < L) ? p.scale * accq[J][t][e] : 0.f;
                    if (J == I) s.Ad[I][r - m0][c - m0] = a[e];
                }
                st_c<S64>(s.Ab, m0, 16 * J + 8 * t, a);
                st_c<S64>(s.P, m0, 16 * J + 8 * t, pv);
            }
        }
        if (!dok) {
            // exact diagonal block: pairs (i, j), j <= i, summed over channels
            __syncwarp();
            for (int e = lane; e < 16 * 16; e += 32) {
                const int r = e >> 4, c = e & 15;
                if (c > r) continue;
                const int i = m0 + r, j = m0 + c;
                float sa = 0.f, sq = 0.f;
                for (int ch = 0; ch < DK; ++ch) {
                    const float d = __expf(s.G[i][ch] - s.G[j][ch]);
                    const float kj = __bfloat162float(s.K[Tma128::off(j, ch)]);
                    sa += __bfloat162float(s.K[Tma128::off(i, ch)]) * kj * d;
                    sq += __bfloat162float(s.Q[Tma128::off(i, ch)]) * kj * d;
                }
                const float a = (c < r) ? s.beta[i] * sa : 0.f;
                s.Ad[I][r][c] = a;
                s.Ab[swz<C>(i, j)] = __float2bfloat16_rn(a);
                s.P[swz<C>(i, j)] = __float2bfloat16_rn(i < L ? p.scale * sq : 0.f);
            }
        }
    }
    __syncwarp();

    // ---- UT transform (identical to the scalar-gate prep) -----------------
    {
        const int c = lane & 15;
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float v = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) v -= s.Ad[warp][i][j] * t[j];
            t[i] = (i < c) ? 0.f : v;
        }
        if (lane < 16) {
#pragma unroll
            for (int i = 0; i < 16; ++i) s.Tb[swz<C>(m0 + i, m0 + c)] = __float2bfloat16_rn(t[i]);
        }
        for (int e = lane; e < 16 * C; e += 32) {
            const int r = e >> 6, cc = e & 63;
            if (cc >= m0 + 16) s.Tb[swz<C>(m0 + r, cc)] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();
    for (int dgl = 1; dgl < 4; ++dgl) {
        const int J = warp, I2 = warp + dgl;
        if (I2 < 4) {
            float x[2][4] = {};
            for (int Kb = J; Kb < I2; ++Kb) {
                uint32_t a[4], bt[4];
                lda<S64>(a, s.Ab, 16 * I2, 16 * Kb);
                ldb_kn<S64>(bt, s.Tb, 16 * Kb, 16 * J);
                mma16816(x[0], a, bt[0], bt[1]);
                mma16816(x[1], a, bt[2], bt[3]);
            }
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                const int r = lane >> 2, cc = 8 * jn + 2 * (lane & 3);
                *reinterpret_cast<uint32_t*>(&s.X[warp][r * 16 + cc]) = pack_bf16(x[jn][0], x[jn][1]);
                *reinterpret_cast<uint32_t*>(&s.X[warp][(r + 8) * 16 + cc]) = pack_bf16(x[jn][2], x[jn][3]);
            }
            __syncwarp();
            uint32_t a[4], bx[4];
            lda<S64>(a, s.Tb, 16 * I2, 16 * I2);
            {
                const int idx = lane >> 3;
                const int row = (lane & 7) + (idx & 1) * 8, col = (idx >> 1) * 8;
                ldsm_x4_t(bx, smem_u32(&s.X[warp][row * 16 + col]));
            }
            float y[2][4] = {};
            mma16816(y[0], a, bx[0], bx[1]);
            mma16816(y[1], a, bx[2], bx[3]);
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                float z[4] = {-y[jn][0], -y[jn][1], -y[jn][2], -y[jn][3]};
                st_c<S64>(s.Tb, 16 * I2, 16 * J + 8 * jn, z);
            }
        }
        __syncthreads();
    }

    // ---- K .* e^G (W operand), Qg = scale Q .* e^G, Kt = K .* e^{G_last - G}
    for (int e = tid; e < C * DK; e += 128) {
        const int i = e / DK, c = e % DK;
        const uint32_t o = Tma128::off(i, c);
        const float g = s.G[i][c];
        const float eg = __expf(g);
        const float kv = __bfloat162float(s.K[o]);
        s.Kl[o] = __float2bfloat16_rn(kv * eg);
        s.Ql[o] = __float2bfloat16_rn(kv * __expf(s.G[C - 1][c] - g));  // Kt image
        s.Q[o] = __float2bfloat16_rn(p.scale * __bfloat162float(s.Q[o]) * eg);  // Qg image
    }
    __syncthreads();
    float aw[16][4], au[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) aw[j][e] = au[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        if (kk > warp) break;
        uint32_t a1[4];
        lda<S64>(a1, s.Tb, m0, 16 * kk);
        scale_a_cols_f(a1, s.beta, 16 * kk);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
            uint32_t bk[4], bv[4];
            ldb_kn<Tma128>(bk, s.Kl, 16 * kk, 16 * np);
            ldb_kn<Tma128>(bv, s.V, 16 * kk, 16 * np);
            mma16816(aw[2 * np], a1, bk[0], bk[1]);
            mma16816(aw[2 * np + 1], a1, bk[2], bk[3]);
            mma16816(au[2 * np], a1, bv[0], bv[1]);
            mma16816(au[2 * np + 1], a1, bv[2], bv[3]);
        }
    }
    __syncthreads();  // done reading Kl and V
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        st_c<S128>(s.Kl, m0, 8 * j, aw[j]);  // W image
        const int r = m0 + (lane >> 2), cc = 8 * (j & 1) + 2 * (lane & 3);
        __nv_bfloat16* Ust = s.Kr + (j >> 1) * (C * 16);
        *reinterpret_cast<uint32_t*>(Ust + r * 16 + cc) = pack_bf16(au[j][0], au[j][1]);
        *reinterpret_cast<uint32_t*>(Ust + (r + 8) * 16 + cc) = pack_bf16(au[j][2], au[j][3]);
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_s2g(p.W + (size_t)cid * C * DK, s.Kl, C * DK * 2);
        bulk_s2g(p.Ut + (size_t)cid * C * DV, s.Kr, C * DV * 2);
        bulk_s2g(p.P + (size_t)cid * C * C, s.P, C * C * 2);
        bulk_s2g(p.G + (size_t)cid * DK, s.gl, DK * 4);
        bulk_s2g(p.Qg + (size_t)cid * C * DK, s.Q, C * DK * 2);
        bulk_s2g(p.Kt + (size_t)cid * C * DK, s.Ql, C * DK * 2);
        if (p.Tb) bulk_s2g(p.Tb + (size_t)cid * C * C, s.Tb, C * C * 2);
        bulk_commit();
        bulk_wait_read<0>();
    }
}

}  // namespace

void launch_prep_kda(const ChunkPtrs& p, size_t nchunks, cudaStream_t st) {
    const int smem = sizeof(KdaPrepSmem) + 1024;
    cudaFuncSetAttribute(tc_prep_kda_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc_prep_kda", st, tc_prep_kda_kernel<<<(unsigned)nchunks, 128, smem, st>>>(p));
}

}  // namespace tc
}  // namespace gdn
