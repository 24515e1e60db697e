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
#include "tc5.cuh"
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
    __nv_bfloat16 Kr[C * DK];   // K .* ER; later U~^T staging
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

// Sixteen warps: warp w works on row block w % 4; in the A/P products it takes
// column block J = w / 4, in the W / U~ products the column quarter w / 4;
// the block solve runs on warps 0..3.
constexpr int KP_THREADS = 512;

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

__global__ void __launch_bounds__(KP_THREADS) tc_prep_kda_kernel(const __grid_constant__ ChunkPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    KdaPrepSmem& s = *reinterpret_cast<KdaPrepSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, h = bh % p.H;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, n);
    if (!cl.valid) return;  // past the last chunk of a packed batch
    const int L = cl.L;
    const size_t row0 = (size_t)cl.tok * p.H + h;
    const size_t rs = (size_t)p.H;

    if (tid == 0) {
        mbar_init(&s.bar, 1);
        fence_mbar_init();
        mbar_arrive_expect(&s.bar, 3 * C * DK * 2);
        const int tok = cl.tok;
        tma_load_tile(s.K, &p.kmap, h, tok, &s.bar);
        tma_load_tile(s.Q, &p.qmap, h, tok, &s.bar);
        tma_load_tile(s.V, &p.vmap, h, tok, &s.bar);
    }
    // log-gates (rows past the sequence end add 0) and beta
    for (int e = tid; e < C * (DK / 4); e += KP_THREADS) {
        const int r = e / (DK / 4), c4 = e % (DK / 4);
        const bool ok = r < L;
        cp_async16_zfill(&s.G[r][4 * c4], p.g + (row0 + (size_t)(ok ? r : 0) * rs) * DK + 4 * c4, ok);
    }
    cp_async_commit();
    if (tid < C) s.beta[tid] = tid < L ? p.beta[row0 + tid * rs] : 0.f;
    cp_async_wait<0>();
    __syncthreads();
    if (tid < DK) {   // per-channel cumsum: thread c owns channel c
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
    for (int e = tid; e < 6 * DK; e += KP_THREADS) {
        const int pi = e / DK, c = e % DK;
        const int I = pi < 1 ? 1 : (pi < 3 ? 2 : 3);
        const int J = pi - I * (I - 1) / 2;
        s.F[pi][c] = __expf(s.G[16 * I][c] - s.G[16 * J + 15][c]);
    }
    // scaled operands
    for (int e = tid; e < C * DK; e += KP_THREADS) {
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

    const int I = warp & 3, m0 = 16 * I, grp = warp >> 2;
    // ---- A and P, row block I, column block J = grp ----------------------
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
                if (J != grp) continue;
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
            if (J != grp) continue;
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
        if (!dok && I == grp) {
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
    __syncthreads();  // A's diagonal blocks complete (either warp of a pair wrote them)

    // ---- UT transform (identical to the scalar-gate prep), warps 0..3 ------
    if (warp < 4) {
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
        if (warp < 4 && I2 < 4) {
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
    for (int e = tid; e < C * DK; e += KP_THREADS) {
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
    // W, U~ for row block I, columns 32*grp .. +31
    float aw[4][4], au[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) aw[j][e] = au[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        if (kk > I) break;
        uint32_t a1[4];
        lda<S64>(a1, s.Tb, m0, 16 * kk);
        scale_a_cols_f(a1, s.beta, 16 * kk);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            uint32_t bk[4], bv[4];
            ldb_kn<Tma128>(bk, s.Kl, 16 * kk, 32 * grp + 16 * np);
            ldb_kn<Tma128>(bv, s.V, 16 * kk, 32 * grp + 16 * np);
            mma16816(aw[2 * np], a1, bk[0], bk[1]);
            mma16816(aw[2 * np + 1], a1, bk[2], bk[3]);
            mma16816(au[2 * np], a1, bv[0], bv[1]);
            mma16816(au[2 * np + 1], a1, bv[2], bv[3]);
        }
    }
    __syncthreads();  // done reading Kl and V
    stage_w_ut_cols(s.Kl, s.Kr, aw, au, m0, 32 * grp);  // W image in Kl's slot, U~^T in Kr's
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

void launch_prep5_kda(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
void launch_prep_kda(const ChunkPtrs& p, size_t nchunks, cudaStream_t st) {
    return launch_prep5_kda(p, nchunks, st);
    const int smem = sizeof(KdaPrepSmem) + 1024;
    cudaFuncSetAttribute(tc_prep_kda_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc_prep_kda", st, tc_prep_kda_kernel<<<(unsigned)nchunks, KP_THREADS, smem, st>>>(p));
}

}  // namespace tc
}  // namespace gdn

// ===========================================================================
// Channel-gate backward, local gradients (one CTA of 16 warps per chunk).
//
// The products over the value dimension (dQg = dO S0, dKt = U dS, dW = -dU S0,
// dP = lower(dO U^T)), the UT-transform chain (dT, X = dT T^T, dKg = T^T dW,
// dVb = T^T dU, dA = -T^T X) and the state terms are those of the scalar gate.
// Per-channel decays enter elementwise (e^{G_ic}, e^{G_last,c - G_ic}) and in
// the four pair products, written with D_ijc = e^{G_ic - G_jc}:
//   X1 = (dMM .* D) K,  X2 = (dMM .* D)^T K,  X3 = (dP .* D)^T Q,  X4 = (dP .* D) K
// (dMM = dA .* beta_i), which give dK += X1 + X2 + scale X3, dQ' += X4 and
// dG += K .* (X1 - X2 - scale X3) + scale Q .* X4.  They use the same block
// factorisation as the forward: for j in block J < I,
//   D_ijc = EL_ic F_IJc ER_jc,  F_IJc = e^{G_{16I,c} - G_{16J+15,c}},
// so X1 over J < I is EL .* sum_J F_IJ .* (dMM_IJ (K .* ER)_J), and inside a
// diagonal block D_ijc = EL_ic e^{G_{16I,c} - G_jc} (MMA form when the block's
// span is at most 80, exact elementwise sums otherwise).  dg is the reverse
// within-chunk cumsum of dG, per channel.
// ===========================================================================
namespace gdn {
namespace tc {
namespace {

constexpr int KL_WARPS = 16, KL_THREADS = 32 * KL_WARPS;

struct KdaLocSmem {
    __nv_bfloat16 Q[C * DK];    // Tma128 (TMA)
    __nv_bfloat16 K[C * DK];    // Tma128 (TMA)
    __nv_bfloat16 dU[C * DV];   // Swz<128> image
    __nv_bfloat16 dW[C * DK];   // Swz<128>
    __nv_bfloat16 Tb[C * C];    // Swz<64> image
    __nv_bfloat16 dP[C * C];    // Swz<64>: lower(dO U^T)
    __nv_bfloat16 dT[C * C];    // Swz<64>: dT, then X = dT T^T, then dMM
    union Scratch {
        struct {
            __nv_bfloat16 S[DV * DK];   // Swz<128>: S0, then dS
            __nv_bfloat16 dO[C * DV];   // Tma128 (TMA)
            __nv_bfloat16 U[C * DV];    // Swz<128> image
        } p1;
        struct {
            __nv_bfloat16 Kl[C * DK], Kr[C * DK], Kd[C * DK], Ql[C * DK], Kg[C * DK];
            __nv_bfloat16 V[C * DV];    // Tma128 (TMA), loaded at the start
        } p2;
        float dG[C][DK + 4];
    } u;
    // Rows padded by 4 floats: a warp reading its MMA fragment's (row, column)
    // positions (8 rows x 4 columns) then hits 2 lanes per bank instead of 8.
    float G[C][DK + 4];
    float red_b[KL_WARPS][C];
    float glp[2][4][DK];        // G_last column partials: [term][row block][channel]
    float beta[C];
    int diag_ok[4];
    uint64_t bar[3];
};

struct KdaLocPtrs {
    CUtensorMap qmap, kmap, vmap, dOmap;
    const float *g, *beta;
    const __nv_bfloat16 *S0, *U, *dS, *dU, *Tb;
    __nv_bfloat16 *dq, *dk, *dv;
    float *dg, *dbeta;
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    SeqMap seq;
};

using S128 = Swz<128>;
using S64 = Swz<64>;

__device__ __forceinline__ float bf(const __nv_bfloat16* t, uint32_t off) {
    return __bfloat162float(t[off]);
}

// Sum over the 8 row groups of a warp (lanes with equal lane % 4).
__device__ __forceinline__ float col_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    return v;
}

__global__ void __launch_bounds__(KL_THREADS) tc_bwd_local_kda_kernel(const __grid_constant__ KdaLocPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    KdaLocSmem& s = *reinterpret_cast<KdaLocSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int I = w >> 2, cq = w & 3, m0 = 16 * I;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, h = bh % p.H;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, n);
    if (!cl.valid) return;  // past the last chunk of a packed batch
    const int L = cl.L;
    const size_t row0 = (size_t)cl.tok * p.H + h;
    const size_t rs = (size_t)p.H;
    const int rl = m0 + (lane >> 2), rh = rl + 8;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&s.bar[i], 1);
        fence_mbar_init();
        const int tok = cl.tok;
        // Q, K, dO, U, dU (five 64x128 tiles), S0 (128x128), T (64x64)
        mbar_arrive_expect(&s.bar[0], (5 * C * DK + DV * DK + C * C) * 2);
        tma_load_tile(s.Q, &p.qmap, h, tok, &s.bar[0]);
        tma_load_tile(s.K, &p.kmap, h, tok, &s.bar[0]);
        tma_load_tile(s.u.p1.dO, &p.dOmap, h, tok, &s.bar[0]);
        bulk_g2s(s.u.p1.U, p.U + (size_t)cid * C * DV, C * DV * 2, &s.bar[0]);
        bulk_g2s(s.dU, p.dU + (size_t)cid * C * DV, C * DV * 2, &s.bar[0]);
        bulk_g2s(s.u.p1.S, p.S0 + (size_t)cid * DV * DK, DV * DK * 2, &s.bar[0]);
        bulk_g2s(s.Tb, p.Tb + (size_t)cid * C * C, C * C * 2, &s.bar[0]);
        mbar_arrive_expect(&s.bar[1], C * DV * 2);
        tma_load_tile(s.u.p2.V, &p.vmap, h, tok, &s.bar[1]);
    }
    for (int e = tid; e < C * (DK / 4); e += KL_THREADS) {
        const int r = e / (DK / 4), c4 = e % (DK / 4);
        const bool ok = r < L;
        cp_async16_zfill(&s.G[r][4 * c4], p.g + (row0 + (size_t)(ok ? r : 0) * rs) * DK + 4 * c4, ok);
    }
    cp_async_commit();
    if (tid < C) s.beta[tid] = tid < L ? p.beta[row0 + tid * rs] : 0.f;
    for (int e = tid; e < KL_WARPS * C; e += KL_THREADS) (&s.red_b[0][0])[e] = 0.f;
    for (int e = tid; e < 2 * 4 * DK; e += KL_THREADS) (&s.glp[0][0][0])[e] = 0.f;
    cp_async_wait<0>();
    __syncthreads();
    if (tid < DK) {  // per-channel within-chunk cumsum
        float run = 0.f;
        for (int i = 0; i < C; ++i) { run += s.G[i][tid]; s.G[i][tid] = run; }
    }
    __syncthreads();
    if (w < 4) {
        float sp = 0.f;
        for (int c = lane; c < DK; c += 32) sp = fmaxf(sp, s.G[16 * w][c] - s.G[16 * w + 15][c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sp = fmaxf(sp, __shfl_xor_sync(0xffffffffu, sp, o));
        if (lane == 0) s.diag_ok[w] = sp <= 80.f;
    }
    if (__syncthreads_or(!mbar_wait(&s.bar[0], 0, p.status))) return;
    if (L < C) {  // dO rows past the sequence end belong to the next sequence
        for (int e = tid; e < (C - L) * DV; e += KL_THREADS)
            s.u.p1.dO[Tma128::off(L + e / DV, e % DV)] = __float2bfloat16_rn(0.f);
    }
    __syncthreads();

    const float Gl_scale = 0.f;
    (void)Gl_scale;
    // this thread's 16 outputs of a 64x128 result: rows rl/rh, channels 32cq + 8j + 2(lane%4) + {0,1}
    auto col = [&](int j, int e) { return 32 * cq + 8 * j + 2 * (lane & 3) + (e & 1); };
    auto row = [&](int e) { return e < 2 ? rl : rh; };
    float dQ[4][4], dK[4][4], dG[4][4];
    float bsum_lo = 0.f, bsum_hi = 0.f;  // partial dbeta for rows rl, rh

    // ---- phase 1a: dQg = dO S0, dW = -dU S0, dP = lower(dO U^T) ---------------
    {
        float aq[4][4] = {}, aw[4][4] = {};
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t ad[4], au[4];
            lda<Tma128>(ad, s.u.p1.dO, m0, 16 * kk);
            lda<Tma128>(au, s.dU, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bs[4];
                ldb_kn<Kp<DV>>(bs, s.u.p1.S, 16 * kk, 32 * cq + 16 * np);
                mma16816(aq[2 * np], ad, bs[0], bs[1]);
                mma16816(aq[2 * np + 1], ad, bs[2], bs[3]);
                mma16816(aw[2 * np], au, bs[0], bs[1]);
                mma16816(aw[2 * np + 1], au, bs[2], bs[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = row(e), c = col(j, e);
                const float eg = __expf(s.G[r][c]);
                dQ[j][e] = eg * aq[j][e];
                dG[j][e] = p.scale * eg * aq[j][e] * bf(s.Q, Tma128::off(r, c));
            }
            float x[4] = {-aw[j][0], -aw[j][1], -aw[j][2], -aw[j][3]};
            st_c<S128>(s.dW, m0, 32 * cq + 8 * j, x);
        }
        float dp[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t ad[4], bu[4];
            lda<Tma128>(ad, s.u.p1.dO, m0, 16 * kk);
            ldb_nk<Tma128>(bu, s.u.p1.U, 16 * cq, 16 * kk);
            mma16816(dp[0], ad, bu[0], bu[1]);
            mma16816(dp[1], ad, bu[2], bu[3]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float g[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = row(e), c = 16 * cq + 8 * j + 2 * (lane & 3) + (e & 1);
                g[e] = c <= r ? dp[j][e] : 0.f;
            }
            st_c<S64>(s.dP, m0, 16 * cq + 8 * j, g);
        }
    }
    // S0 elements this thread pairs with dS below (column c = tid % 128)
    float s0r[32];
    {
        const int c = tid & (DK - 1), a0 = tid >> 7;
#pragma unroll
        for (int k = 0; k < 32; ++k) s0r[k] = bf(s.u.p1.S, Kp<DV>::off(a0 + 4 * k, c));
    }
    __syncthreads();  // everyone done with S0
    if (tid == 0) {
        mbar_arrive_expect(&s.bar[2], DV * DK * 2);
        bulk_g2s(s.u.p1.S, p.dS + (size_t)cid * DV * DK, DV * DK * 2, &s.bar[2]);
    }
    if (__syncthreads_or(!mbar_wait(&s.bar[2], 0, p.status))) return;

    // ---- phase 1b: dKt = U dS, <dS, S0> per channel -----------------------------
    {
        float ak[4][4] = {};
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t au[4];
            lda<Tma128>(au, s.u.p1.U, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bs[4];
                ldb_kn<Kp<DV>>(bs, s.u.p1.S, 16 * kk, 32 * cq + 16 * np);
                mma16816(ak[2 * np], au, bs[0], bs[1]);
                mma16816(ak[2 * np + 1], au, bs[2], bs[3]);
            }
        }
        float colp[4][2] = {};
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = row(e), c = col(j, e);
                const float et = __expf(s.G[C - 1][c] - s.G[r][c]);
                dK[j][e] = et * ak[j][e];
                const float hkt = et * ak[j][e] * bf(s.K, Tma128::off(r, c));
                dG[j][e] -= hkt;
                colp[j][e & 1] += hkt;
            }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float v = col_sum(colp[j][e]);
                if (lane < 4) s.glp[0][I][32 * cq + 8 * j + 2 * lane + e] = v;
            }
        const int c = tid & (DK - 1), a0 = tid >> 7;
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) ss += s0r[k] * bf(s.u.p1.S, Kp<DV>::off(a0 + 4 * k, c));
        s.glp[1][a0][c] = ss;
    }
    __syncthreads();  // phase-1 scratch is dead from here on

    // ---- phase 2 prologue: scaled K / Q operands ----------------------------------
    for (int e = tid; e < C * DK; e += KL_THREADS) {
        const int i = e / DK, c = e % DK;
        const int f = i & ~15, l = f + 15;
        const float g = s.G[i][c];
        const uint32_t o = Tma128::off(i, c);
        const float kv = bf(s.K, o), qv = bf(s.Q, o);
        const float el = __expf(g - s.G[f][c]);
        s.u.p2.Kl[o] = __float2bfloat16_rn(kv * el);
        s.u.p2.Ql[o] = __float2bfloat16_rn(qv * el);
        s.u.p2.Kr[o] = __float2bfloat16_rn(kv * __expf(s.G[l][c] - g));
        const float sp = s.G[f][c] - g;
        s.u.p2.Kd[o] = __float2bfloat16_rn(sp <= 80.f ? kv * __expf(sp) : 0.f);
        s.u.p2.Kg[o] = __float2bfloat16_rn(kv * __expf(g));
    }
    if (__syncthreads_or(!mbar_wait(&s.bar[1], 0, p.status))) return;
    const bool dok = s.diag_ok[I];

    // ---- phase 2: M (decayed K K^T, block J = cq) and dT -------------------------
    float M[2][4];
    {
        const int J = cq;
        float mk[2][4] = {}, tw[2][4] = {}, tu[2][4] = {};
        const bool mma_m = J < I || (J == I && dok);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            if (mma_m) {
                uint32_t ak[4], bk[4];
                lda<Tma128>(ak, s.u.p2.Kl, m0, 16 * kk);
                if (J < I) {
                    // scale the A fragment's channels by F_IJ
                    const int k = 16 * kk + 2 * (lane & 3);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int kc = k + (r >> 1) * 8;
                        const float f0 = __expf(s.G[16 * I][kc] - s.G[16 * J + 15][kc]);
                        const float f1 = __expf(s.G[16 * I][kc + 1] - s.G[16 * J + 15][kc + 1]);
                        float2 v = unpack_bf16(ak[r]);
                        ak[r] = pack_bf16(v.x * f0, v.y * f1);
                    }
                    ldb_nk<Tma128>(bk, s.u.p2.Kr, 16 * J, 16 * kk);
                } else {
                    ldb_nk<Tma128>(bk, s.u.p2.Kd, 16 * J, 16 * kk);
                }
                mma16816(mk[0], ak, bk[0], bk[1]);
                mma16816(mk[1], ak, bk[2], bk[3]);
            }
            uint32_t aw[4], au[4], bg[4], bv[4];
            lda<S128>(aw, s.dW, m0, 16 * kk);
            lda<Tma128>(au, s.dU, m0, 16 * kk);
            ldb_nk<Tma128>(bg, s.u.p2.Kg, 16 * cq, 16 * kk);
            ldb_nk<Tma128>(bv, s.u.p2.V, 16 * cq, 16 * kk);
            mma16816(tw[0], aw, bg[0], bg[1]);
            mma16816(tw[1], aw, bg[2], bg[3]);
            mma16816(tu[0], au, bv[0], bv[1]);
            mma16816(tu[1], au, bv[2], bv[3]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float dt[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = row(e), c = 16 * cq + 8 * j + 2 * (lane & 3) + (e & 1);
                dt[e] = s.beta[c] * (tw[j][e] + tu[j][e]);
                float m = 0.f;
                if (c < r) {
                    if (mma_m) {
                        m = mk[j][e];
                    } else if (J == I) {  // exact: sum_ch k_r k_c e^{G_r - G_c}
                        for (int ch = 0; ch < DK; ++ch)
                            m += bf(s.K, Tma128::off(r, ch)) * bf(s.K, Tma128::off(c, ch)) *
                                 __expf(s.G[r][ch] - s.G[c][ch]);
                    }
                }
                M[j][e] = m;
            }
            st_c<S64>(s.dT, m0, 16 * cq + 8 * j, dt);
        }
    }
    __syncthreads();

    // ---- phase 3: X = dT T^T ; dKg = T^T dW ; dVb = T^T dU ---------------------
    {
        float x[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4], bt[4];
            lda<S64>(a, s.dT, m0, 16 * kk);
            ldb_nk<S64>(bt, s.Tb, 16 * cq, 16 * kk);
            mma16816(x[0], a, bt[0], bt[1]);
            mma16816(x[1], a, bt[2], bt[3]);
        }
        float akg[4][4] = {}, avb[4][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk < I) continue;  // T[j][i] = 0 for j < i
            uint32_t a[4];
            lda_t<S64>(a, s.Tb, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bw[4], bu[4];
                ldb_kn<S128>(bw, s.dW, 16 * kk, 32 * cq + 16 * np);
                ldb_kn<Tma128>(bu, s.dU, 16 * kk, 32 * cq + 16 * np);
                mma16816(akg[2 * np], a, bw[0], bw[1]);
                mma16816(akg[2 * np + 1], a, bw[2], bw[3]);
                mma16816(avb[2 * np], a, bu[0], bu[1]);
                mma16816(avb[2 * np + 1], a, bu[2], bu[3]);
            }
        }
        const float bl = s.beta[rl], bh2 = s.beta[rh];
        __nv_bfloat16* dvp = p.dv + row0 * DV;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float dvv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = row(e), c = col(j, e);
                const float br = e < 2 ? bl : bh2;
                const float kgv = bf(s.u.p2.Kg, Tma128::off(r, c));  // k e^G
                dK[j][e] += br * __expf(s.G[r][c]) * akg[j][e];
                dG[j][e] += br * akg[j][e] * kgv;
                const float hb = akg[j][e] * kgv + avb[j][e] * bf(s.u.p2.V, Tma128::off(r, c));
                if (e < 2) bsum_lo += hb; else bsum_hi += hb;
                dvv[e] = br * avb[j][e];
            }
            const int c = col(j, 0);
            if (rl < L)
                *reinterpret_cast<uint32_t*>(dvp + (size_t)rl * rs * DV + c) = pack_bf16(dvv[0], dvv[1]);
            if (rh < L)
                *reinterpret_cast<uint32_t*>(dvp + (size_t)rh * rs * DV + c) = pack_bf16(dvv[2], dvv[3]);
        }
        __syncthreads();  // everyone done reading dT
#pragma unroll
        for (int j = 0; j < 2; ++j) st_c<S64>(s.dT, m0, 16 * cq + 8 * j, x[j]);  // X
    }
    __syncthreads();

    // ---- phase 4: dA = -T^T X (strictly lower), dbeta from M, dMM = dA beta_i ----
    {
        float da[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk < I) continue;
            uint32_t a[4], bx[4];
            lda_t<S64>(a, s.Tb, m0, 16 * kk);
            ldb_kn<S64>(bx, s.dT, 16 * kk, 16 * cq);
            mma16816(da[0], a, bx[0], bx[1]);
            mma16816(da[1], a, bx[2], bx[3]);
        }
        float mm[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = row(e), c = 16 * cq + 8 * j + 2 * (lane & 3) + (e & 1);
                const float dA = (c < r) ? -da[j][e] : 0.f;
                if (e < 2) bsum_lo += dA * M[j][e]; else bsum_hi += dA * M[j][e];
                mm[j][e] = dA * s.beta[r];
            }
        __syncthreads();  // everyone done reading X
#pragma unroll
        for (int j = 0; j < 2; ++j) st_c<S64>(s.dT, m0, 16 * cq + 8 * j, mm[j]);  // dMM
    }
    __syncthreads();

    // ---- phase 5: the four decayed pair products ---------------------------------
    // Each column block's contribution goes straight into dQ, dK and dG, so no
    // per-side accumulators stay live across the blocks.  The pair (r, r) has
    // decay 1 and adds nothing to dG (its row- and column-side terms cancel): its
    // rounded form is left out of the dG sums on both sides, so that no bf16
    // residual of it swamps the small dg of a strongly decayed chunk.
    {
        // row side: X1 = dMM (K .* decay), X4 = dP (K .* decay); blocks J < I
        // through Kr, the diagonal block through Kd, then each by its factor
        // e^{G_r - G_l} (J < I, l = last row of J) or e^{G_r - G_f} (J = I)
        for (int J = 0; J <= I; ++J) {
            if (J == I && !dok) break;
            float t1[4][4] = {}, t4[4][4] = {};
            uint32_t am[4], ap[4];
            lda<S64>(am, s.dT, m0, 16 * J);
            lda<S64>(ap, s.dP, m0, 16 * J);
            const __nv_bfloat16* B = J < I ? s.u.p2.Kr : s.u.p2.Kd;
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bk[4];
                ldb_kn<Tma128>(bk, B, 16 * J, 32 * cq + 16 * np);
                mma16816(t1[2 * np], am, bk[0], bk[1]);
                mma16816(t1[2 * np + 1], am, bk[2], bk[3]);
                mma16816(t4[2 * np], ap, bk[0], bk[1]);
                mma16816(t4[2 * np + 1], ap, bk[2], bk[3]);
            }
            const int ref = J < I ? 16 * J + 15 : m0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = row(e), c = col(j, e);
                    const uint32_t o = Tma128::off(r, c);
                    const float f = __expf(s.G[r][c] - s.G[ref][c]);
                    const float x1 = f * t1[j][e], x4 = f * t4[j][e];
                    const float self4 = J == I ? bf(s.dP, swz<C>(r, r)) * bf(s.u.p2.Kd, o) * f : 0.f;
                    dK[j][e] += x1;
                    dQ[j][e] += x4;
                    dG[j][e] += bf(s.K, o) * x1 + p.scale * bf(s.Q, o) * (x4 - self4);
                }
        }
        if (!dok) {  // exact diagonal-block sums, j <= i inside block I
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = row(e), c = col(j, e);
                    const float gr = s.G[r][c];
                    float x1 = 0.f, x4 = 0.f;
                    for (int jj = m0; jj < r; ++jj) {
                        const float d = __expf(gr - s.G[jj][c]);
                        const float kj = bf(s.K, Tma128::off(jj, c));
                        x1 += bf(s.dT, swz<C>(r, jj)) * d * kj;
                        x4 += bf(s.dP, swz<C>(r, jj)) * d * kj;
                    }
                    const float kv = bf(s.K, Tma128::off(r, c)), qv = bf(s.Q, Tma128::off(r, c));
                    dK[j][e] += x1;
                    dQ[j][e] += x4 + bf(s.dP, swz<C>(r, r)) * kv;
                    dG[j][e] += kv * x1 + p.scale * qv * x4;
                }
        }
    }
    {
        // column side: X2 = dMM^T (K .* decay), X3 = dP^T (Q .* decay); blocks J > I
        // by e^{G_f(J) - G_r}, the diagonal block by e^{G_f - G_r} (its B operands
        // carry EL_j)
        for (int J = I; J < 4; ++J) {
            if (J == I && !dok) continue;
            float t2[4][4] = {}, t3[4][4] = {};
            uint32_t am[4], ap[4];
            lda_t<S64>(am, s.dT, m0, 16 * J);
            lda_t<S64>(ap, s.dP, m0, 16 * J);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bk[4], bq[4];
                ldb_kn<Tma128>(bk, s.u.p2.Kl, 16 * J, 32 * cq + 16 * np);
                ldb_kn<Tma128>(bq, s.u.p2.Ql, 16 * J, 32 * cq + 16 * np);
                mma16816(t2[2 * np], am, bk[0], bk[1]);
                mma16816(t2[2 * np + 1], am, bk[2], bk[3]);
                mma16816(t3[2 * np], ap, bq[0], bq[1]);
                mma16816(t3[2 * np + 1], ap, bq[2], bq[3]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = row(e), c = col(j, e);
                    const uint32_t o = Tma128::off(r, c);
                    const float f = __expf(s.G[16 * J][c] - s.G[r][c]);
                    const float x2 = f * t2[j][e], x3 = f * t3[j][e];
                    const float self3 = J == I ? bf(s.dP, swz<C>(r, r)) * bf(s.u.p2.Ql, o) * f : 0.f;
                    dK[j][e] += x2 + p.scale * x3;
                    dG[j][e] -= bf(s.K, o) * (x2 + p.scale * (x3 - self3));
                }
        }
        if (!dok) {  // exact diagonal-block sums, j > i inside block I
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = row(e), c = col(j, e);
                    const float gr = s.G[r][c];
                    float x2 = 0.f, x3 = 0.f;
                    for (int jj = r + 1; jj < m0 + 16; ++jj) {
                        const float d = __expf(s.G[jj][c] - gr);
                        x2 += bf(s.dT, swz<C>(jj, r)) * d * bf(s.K, Tma128::off(jj, c));
                        x3 += bf(s.dP, swz<C>(jj, r)) * d * bf(s.Q, Tma128::off(jj, c));
                    }
                    const float kv = bf(s.K, Tma128::off(r, c));
                    dK[j][e] += x2 + p.scale * (x3 + bf(s.dP, swz<C>(r, r)) * bf(s.Q, Tma128::off(r, c)));
                    dG[j][e] -= kv * (x2 + p.scale * x3);
                }
        }
    }
    {
        const bool okl = rl < L, okh = rh < L;
        __nv_bfloat16* dqp = p.dq + row0 * DK;
        __nv_bfloat16* dkp = p.dk + row0 * DK;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = col(j, 0);
            if (okl) {
                *reinterpret_cast<uint32_t*>(dqp + (size_t)rl * rs * DK + c) =
                    pack_bf16(p.scale * dQ[j][0], p.scale * dQ[j][1]);
                *reinterpret_cast<uint32_t*>(dkp + (size_t)rl * rs * DK + c) = pack_bf16(dK[j][0], dK[j][1]);
            }
            if (okh) {
                *reinterpret_cast<uint32_t*>(dqp + (size_t)rh * rs * DK + c) =
                    pack_bf16(p.scale * dQ[j][2], p.scale * dQ[j][3]);
                *reinterpret_cast<uint32_t*>(dkp + (size_t)rh * rs * DK + c) = pack_bf16(dK[j][2], dK[j][3]);
            }
        }
    }
    // ---- dbeta (row sums) and dg (per-channel reverse cumsum of dG) ---------------
    {
        float lo = bsum_lo, hi = bsum_hi;
        lo += __shfl_xor_sync(0xffffffffu, lo, 1);
        lo += __shfl_xor_sync(0xffffffffu, lo, 2);
        hi += __shfl_xor_sync(0xffffffffu, hi, 1);
        hi += __shfl_xor_sync(0xffffffffu, hi, 2);
        if ((lane & 3) == 0) {
            s.red_b[w][rl] = lo;
            s.red_b[w][rh] = hi;
        }
    }
    __syncthreads();  // phase-2 scratch is dead; dG goes there
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) s.u.dG[row(e)][col(j, e)] = dG[j][e];
    __syncthreads();
    if (tid < DK) {
        const int c = tid;
        float run = 0.f;
        for (int rb = 0; rb < 4; ++rb)
            run += s.glp[0][rb][c] + __expf(s.G[C - 1][c]) * s.glp[1][rb][c];
        for (int i = C - 1; i >= 0; --i) {
            run += s.u.dG[i][c];
            if (i < L) p.dg[(row0 + (size_t)i * rs) * DK + c] = run;
        }
    } else if (tid < DK + C) {
        const int i = tid - DK;
        float sb = 0.f;
        for (int ww = 0; ww < KL_WARPS; ++ww) sb += (ww >> 2) == (i >> 4) ? s.red_b[ww][i] : 0.f;
        if (i < L) p.dbeta[row0 + (size_t)i * rs] = sb;
    }
}

}  // namespace

bool launch_bwd_local_kda(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp,
                          const void* dO, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                          void* ws, cudaStream_t st) {
    char* base = (char*)ws;
    KdaLocPtrs lp{};
    lp.qmap = cp.qmap; lp.kmap = cp.kmap; lp.vmap = cp.vmap;
    if (!encode_token_map(&lp.dOmap, dO, d.B, d.T, d.H)) return false;
    lp.g = cp.g; lp.beta = cp.beta;
    lp.S0 = (const __nv_bfloat16*)(base + L.S0);
    lp.U = (const __nv_bfloat16*)(base + L.U);
    lp.dS = (const __nv_bfloat16*)(base + L.dS);
    lp.dU = (const __nv_bfloat16*)(base + L.dU);
    lp.Tb = cp.Tb;
    lp.dq = (__nv_bfloat16*)dq; lp.dk = (__nv_bfloat16*)dk; lp.dv = (__nv_bfloat16*)dv;
    lp.dg = dg; lp.dbeta = dbeta; lp.status = cp.status;
    lp.B = d.B; lp.T = d.T; lp.H = d.H; lp.NT = L.NT; lp.scale = d.scale;
    lp.seq = cp.seq;
    const int smem = sizeof(KdaLocSmem) + 1024;
    cudaFuncSetAttribute(tc_bwd_local_kda_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc_bwd_local_kda", st,
               tc_bwd_local_kda_kernel<<<(unsigned)L.nchunks, KL_THREADS, smem, st>>>(lp));
    return true;
}

}  // namespace tc
}  // namespace gdn
