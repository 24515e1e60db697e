// tc_chunk.cu -- tensor-core chunkwise gated delta rule, bf16 in, fp32 state.
//
// Shapes: dk = dv = 128, chunk C = 64, scalar gate.  The chunkwise algebra is
// the WY / UT-transform form of "Gated Delta Networks: Improving Mamba2 with
// Delta Rule" (paper review), sections "Goal" and "Method"; per chunk, with
// S0 the state entering it and G the within-chunk cumsum of the log-gate g:
//   A  = strict_lower(diag(beta) (K K^T .* D)),   D_ij = exp(G_i - G_j)
//   T  = (I + A)^{-1}                              (UT transform)
//   W  = T diag(beta e^G) K,   U~ = T diag(beta) V  (WY factors)
//   P  = lower(Q K^T .* D)
//   U  = U~ - W S0^T
//   O  = diag(e^G) Q S0^T + P U
//   S1 = e^{G_last} S0 + U^T diag(e^{G_last - G}) K
//
// Kernels (one pass each over the chunks):
//   prep   -- grid over all (b, h, chunk): G, A, T, W, U~, P  ->  workspace
//   walk   -- grid over (b, h, 16-row tile of S): the sequential chain
//             U -> S1 -> ... in fp32, plus O (forward) or the chunk-start
//             states and U (backward recompute).
// Rows of S never mix (row a of S pairs only with column a of V, U, O), so the
// walk splits the state by value rows and every CTA carries its own chain.
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace {
using namespace tc;

// ---------------------------------------------------------------------------
// prep: one CTA (4 warps) per chunk.
// ---------------------------------------------------------------------------
struct PrepSmem {
    __nv_bfloat16 K[C * DK];
    __nv_bfloat16 Q[C * DK];
    __nv_bfloat16 V[C * DV];
    __nv_bfloat16 T1[C * C];  // bf16(T diag(beta e^G))
    __nv_bfloat16 T2[C * C];  // bf16(T diag(beta))
    float A[C][C + 1];
    float Tf[C][C + 1];
    float G[C];
    float beta[C];
};

__global__ void __launch_bounds__(128) tc_prep_kernel(ChunkPtrs p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    PrepSmem& s = *reinterpret_cast<PrepSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, b = bh / p.H, h = bh % p.H;
    const int t0 = n * C;
    const int L = min(C, p.T - t0);
    const size_t row0 = ((size_t)b * p.T + t0) * p.H + h;  // token-head index of row 0
    const size_t rs = (size_t)p.H;                        // token-head stride between rows

    load_tile_async<DK>(s.K, p.k + row0 * DK, rs * DK, C, L, tid, 128);
    load_tile_async<DK>(s.Q, p.q + row0 * DK, rs * DK, C, L, tid, 128);
    load_tile_async<DV>(s.V, p.v + row0 * DV, rs * DV, C, L, tid, 128);
    cp_async_commit();
    for (int e = tid; e < C * (C + 1); e += 128) (&s.Tf[0][0])[e] = 0.f;
    if (warp == 0) {
        // inclusive cumsum of the log-gate over the chunk (rows past L add 0)
        float g0 = lane < L ? p.g[row0 + lane * rs] : 0.f;
        float g1 = lane + 32 < L ? p.g[row0 + (lane + 32) * rs] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float x0 = __shfl_up_sync(0xffffffffu, g0, o);
            float x1 = __shfl_up_sync(0xffffffffu, g1, o);
            if (lane >= o) { g0 += x0; g1 += x1; }
        }
        g1 += __shfl_sync(0xffffffffu, g0, 31);
        s.G[lane] = g0;
        s.G[lane + 32] = g1;
        s.beta[lane] = lane < L ? p.beta[row0 + lane * rs] : 0.f;
        s.beta[lane + 32] = lane + 32 < L ? p.beta[row0 + (lane + 32) * rs] : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- decayed K K^T (-> A) and Q K^T (-> P), rows 16w..16w+15 ----------
    {
        const int m0 = 16 * warp;
        float acck[8][4], accq[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acck[j][e] = accq[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t ak[4], aq[4];
            lda<DK>(ak, s.K, m0, 16 * kk);
            lda<DK>(aq, s.Q, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                if (np > warp) break;  // columns beyond the diagonal block are masked
                uint32_t bf[4];
                ldb_nk<DK>(bf, s.K, 16 * np, 16 * kk);
                mma16816(acck[2 * np], ak, bf[0], bf[1]);
                mma16816(acck[2 * np + 1], ak, bf[2], bf[3]);
                mma16816(accq[2 * np], aq, bf[0], bf[1]);
                mma16816(accq[2 * np + 1], aq, bf[2], bf[3]);
            }
        }
        __nv_bfloat16* Pg = p.P + (size_t)cid * C * C;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = m0 + (lane >> 2) + 8 * hh;
                const int c0 = 8 * j + 2 * (lane & 3);
                float pv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int c = c0 + e;
                    const bool live = (j >> 1) <= warp;
                    const float dec = (c <= r) ? __expf(s.G[r] - s.G[c]) : 0.f;
                    s.A[r][c] = (live && c < r) ? s.beta[r] * acck[j][2 * hh + e] * dec : 0.f;
                    pv[e] = live ? accq[j][2 * hh + e] * dec * p.scale : 0.f;
                }
                *reinterpret_cast<uint32_t*>(Pg + (size_t)r * C + c0) = pack_bf16(pv[0], pv[1]);
            }
        }
    }
    __syncthreads();

    // ---- UT transform: T = (I + A)^{-1}, 16x16 blocks ----------------------
    if (lane < 16) {  // diagonal block `warp`, one column per lane
        const int o = 16 * warp, c = lane;
        for (int i = 0; i < 16; ++i) {
            float v;
            if (i < c) v = 0.f;
            else if (i == c) v = 1.f;
            else {
                v = 0.f;
                for (int j = c; j < i; ++j) v -= s.A[o + i][o + j] * s.Tf[o + j][o + c];
            }
            s.Tf[o + i][o + c] = v;
        }
    }
    __syncthreads();
    for (int dgl = 1; dgl < 4; ++dgl) {
        const int J = warp, I = warp + dgl;
        if (I < 4) {
            // X = sum_{K=J}^{I-1} A_IK T_KJ ; T_IJ = -T_II X
            float x[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int e = lane + 32 * t, r = e >> 4, c = e & 15;
                float acc = 0.f;
                for (int kx = 16 * J; kx < 16 * I; ++kx) acc += s.A[16 * I + r][kx] * s.Tf[kx][16 * J + c];
                x[t] = acc;
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int e = lane + 32 * t;
                s.Tf[16 * I + (e >> 4)][16 * J + (e & 15)] = x[t];
            }
            __syncwarp();
            float y[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int e = lane + 32 * t, r = e >> 4, c = e & 15;
                float acc = 0.f;
                for (int m = 0; m <= r; ++m) acc += s.Tf[16 * I + r][16 * I + m] * s.Tf[16 * I + m][16 * J + c];
                y[t] = -acc;
            }
            __syncwarp();
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int e = lane + 32 * t;
                s.Tf[16 * I + (e >> 4)][16 * J + (e & 15)] = y[t];
            }
        }
        __syncthreads();
    }
    for (int e = tid; e < C * C; e += 128) {
        const int i = e >> 6, j = e & 63;
        const float t = s.Tf[i][j] * s.beta[j];
        s.T1[swz<C>(i, j)] = __float2bfloat16_rn(t * __expf(s.G[j]));
        s.T2[swz<C>(i, j)] = __float2bfloat16_rn(t);
        if (p.Tb) p.Tb[(size_t)cid * C * C + e] = __float2bfloat16_rn(s.Tf[i][j]);
    }
    __syncthreads();

    // ---- W = T1 K, U~ = T2 V (rows 16w..16w+15, T lower triangular) --------
    {
        const int m0 = 16 * warp;
        float aw[16][4], au[16][4];
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) aw[j][e] = au[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk > warp) break;
            uint32_t a1[4], a2[4];
            lda<C>(a1, s.T1, m0, 16 * kk);
            lda<C>(a2, s.T2, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bk[4], bv[4];
                ldb_kn<DK>(bk, s.K, 16 * kk, 16 * np);
                ldb_kn<DV>(bv, s.V, 16 * kk, 16 * np);
                mma16816(aw[2 * np], a1, bk[0], bk[1]);
                mma16816(aw[2 * np + 1], a1, bk[2], bk[3]);
                mma16816(au[2 * np], a2, bv[0], bv[1]);
                mma16816(au[2 * np + 1], a2, bv[2], bv[3]);
            }
        }
        __nv_bfloat16* Wg = p.W + (size_t)cid * C * DK;
        __nv_bfloat16* Ug = p.Ut + (size_t)cid * C * DV;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int r = m0 + (lane >> 2), c = 8 * j + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(Wg + (size_t)r * DK + c) = pack_bf16(aw[j][0], aw[j][1]);
            *reinterpret_cast<uint32_t*>(Wg + (size_t)(r + 8) * DK + c) = pack_bf16(aw[j][2], aw[j][3]);
            *reinterpret_cast<uint32_t*>(Ug + (size_t)r * DV + c) = pack_bf16(au[j][0], au[j][1]);
            *reinterpret_cast<uint32_t*>(Ug + (size_t)(r + 8) * DV + c) = pack_bf16(au[j][2], au[j][3]);
        }
    }
    if (tid < C) p.G[(size_t)cid * C + tid] = s.G[tid];
}

// ---------------------------------------------------------------------------
// walk: the sequential chain over chunks for 16*MT rows of S.
// MODE 0: forward (O, hT).  MODE 1: backward recompute (store S0 and U).
// ---------------------------------------------------------------------------
template <int MT>
struct WalkStage {
    __nv_bfloat16 W[C * DK];
    __nv_bfloat16 Q[C * DK];
    __nv_bfloat16 K[C * DK];
    __nv_bfloat16 P[C * C];
    __nv_bfloat16 Ut[C][16 * MT];
    float G[C];
};

template <int MT>
struct WalkSmem {
    WalkStage<MT> st[2];
    __nv_bfloat16 S0[16 * MT * DK];   // bf16 copy of the state entering the chunk
    __nv_bfloat16 Uu[16 * MT * C];    // U^T (rows of S x tokens)
    __nv_bfloat16 Us[16 * MT * C];    // U^T scaled by e^{G_last - G_i}
    __nv_bfloat16 O[C][16 * MT];      // output staging (tokens x rows)
};

struct WalkPtrs {
    const __nv_bfloat16 *q, *k;
    const float* h0;
    const __nv_bfloat16 *W, *Ut, *P;
    const float* G;
    __nv_bfloat16* o;
    float* hT;
    __nv_bfloat16 *S0out, *Uout;
    int B, T, H, NT;
    float scale;
};

template <int MT>
__device__ void walk_issue_loads(WalkStage<MT>& st, const WalkPtrs& p, int b, int h, int bh,
                                 int n, int a0, int tid, int nth) {
    const int t0 = n * C;
    const int L = min(C, p.T - t0);
    const size_t row0 = ((size_t)b * p.T + t0) * p.H + h;
    const size_t cid = (size_t)bh * p.NT + n;
    load_tile_async<DK>(st.K, p.k + row0 * DK, (size_t)p.H * DK, C, L, tid, nth);
    load_tile_async<DK>(st.Q, p.q + row0 * DK, (size_t)p.H * DK, C, L, tid, nth);
    load_tile_async<DK>(st.W, p.W + cid * C * DK, DK, C, C, tid, nth);
    load_tile_async<C>(st.P, p.P + cid * C * C, C, C, C, tid, nth);
    constexpr int UCH = 2 * MT;  // 16-byte chunks per Ut row
    for (int e = tid; e < C * UCH; e += nth) {
        const int r = e / UCH, c = e % UCH;
        cp_async16(&st.Ut[r][8 * c], p.Ut + (cid * C + r) * DV + a0 + 8 * c);
    }
    for (int e = tid; e < C / 4; e += nth) cp_async16(&st.G[4 * e], p.G + cid * C + 4 * e);
    cp_async_commit();
}

template <int MT, int MODE>
__global__ void __launch_bounds__(128 * MT) tc_walk_kernel(WalkPtrs p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    WalkSmem<MT>& s = *reinterpret_cast<WalkSmem<MT>*>(smem_raw);
    constexpr int NTH = 128 * MT, RT = 16 * MT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int mt = warp >> 2, q4 = warp & 3;
    const int tiles = DV / RT;
    const int bh = blockIdx.x / tiles, a0 = (blockIdx.x % tiles) * RT;
    const int b = bh / p.H, h = bh % p.H;
    const int r_lo = 16 * mt + (lane >> 2);  // this thread's first state row (tile-local)

    // fp32 state, rows r_lo and r_lo+8, columns 32*q4 + 8j + 2(lane%4) + {0,1}
    float S[4][4];
    {
        const float* h0 = p.h0 ? p.h0 + ((size_t)bh * DV + a0) * DK : nullptr;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 32 * q4 + 8 * j + 2 * (lane & 3);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = r_lo + 8 * (e >> 1);
                S[j][e] = h0 ? h0[(size_t)r * DK + c + (e & 1)] : 0.f;
            }
        }
    }
    walk_issue_loads<MT>(s.st[0], p, b, h, bh, 0, a0, tid, NTH);
#pragma unroll
    for (int j = 0; j < 4; ++j) st_c<DK>(s.S0, 16 * mt, 32 * q4 + 8 * j, S[j]);

    for (int n = 0; n < p.NT; ++n) {
        WalkStage<MT>& st = s.st[n & 1];
        cp_async_wait<0>();
        __syncthreads();  // stage n landed; S0 written; previous stage free
        if (n + 1 < p.NT) walk_issue_loads<MT>(s.st[(n + 1) & 1], p, b, h, bh, n + 1, a0, tid, NTH);
        const int t0 = n * C;
        const int L = min(C, p.T - t0);
        const size_t cid = (size_t)bh * p.NT + n;

        if (MODE == 1) {  // chunk-start state, bf16, rows a0.. of [dv][dk]
            __nv_bfloat16* dst = p.S0out + (cid * DV + a0) * DK;
            for (int e = tid; e < RT * DK / 8; e += NTH) {
                const int r = e / (DK / 8), c8 = e % (DK / 8);
                *reinterpret_cast<uint4*>(dst + (size_t)r * DK + 8 * c8) =
                    *reinterpret_cast<const uint4*>(s.S0 + swz<DK>(r, 8 * c8));
            }
        }

        // X = S0 W^T and Y = S0 Q^T for tokens 16*q4 .. +15
        float X[2][4] = {}, Y[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t a[4], bw[4];
            lda<DK>(a, s.S0, 16 * mt, 16 * kk);
            ldb_nk<DK>(bw, st.W, 16 * q4, 16 * kk);
            mma16816(X[0], a, bw[0], bw[1]);
            mma16816(X[1], a, bw[2], bw[3]);
            if (MODE == 0) {
                uint32_t bq[4];
                ldb_nk<DK>(bq, st.Q, 16 * q4, 16 * kk);
                mma16816(Y[0], a, bq[0], bq[1]);
                mma16816(Y[1], a, bq[2], bq[3]);
            }
        }
        const float Gl = st.G[C - 1];
        // U^T = U~^T - X ; stage both U^T and U^T * e^{G_last - G_i}
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i0 = 16 * q4 + 8 * j + 2 * (lane & 3);
            float u[4], us[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = r_lo + 8 * (e >> 1), i = i0 + (e & 1);
                u[e] = __bfloat162float(st.Ut[i][r]) - X[j][e];
                us[e] = u[e] * __expf(Gl - st.G[i]);
            }
            st_c<C>(s.Uu, 16 * mt, 16 * q4 + 8 * j, u);
            st_c<C>(s.Us, 16 * mt, 16 * q4 + 8 * j, us);
        }
        __syncthreads();

        if (MODE == 1) {  // U (tokens x value rows a0..), bf16
            __nv_bfloat16* dst = p.Uout + cid * C * DV + a0;
            for (int e = tid; e < C * RT; e += NTH) {
                const int i = e / RT, r = e % RT;
                dst[(size_t)i * DV + r] = s.Uu[swz<C>(r, i)];
            }
        }

        // S1 = e^{G_last} S0 + (U^T .* e^{G_last-G}) K, columns 32*q4 ..
        const float gam = __expf(Gl);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) S[j][e] *= gam;
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
            uint32_t a[4];
            lda<C>(a, s.Us, 16 * mt, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bk[4];
                ldb_kn<DK>(bk, st.K, 16 * kk, 32 * q4 + 16 * np);
                mma16816(S[2 * np], a, bk[0], bk[1]);
                mma16816(S[2 * np + 1], a, bk[2], bk[3]);
            }
        }

        if (MODE == 0) {
            // O^T (rows x tokens 16*q4..) = diag-scaled Y + U^T P^T
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int i0 = 16 * q4 + 8 * j + 2 * (lane & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e) Y[j][e] *= p.scale * __expf(st.G[i0 + (e & 1)]);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                if (kk > q4) break;  // P[r][i] = 0 for i > r
                uint32_t a[4], bp[4];
                lda<C>(a, s.Uu, 16 * mt, 16 * kk);
                ldb_nk<C>(bp, st.P, 16 * q4, 16 * kk);
                mma16816(Y[0], a, bp[0], bp[1]);
                mma16816(Y[1], a, bp[2], bp[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int i0 = 16 * q4 + 8 * j + 2 * (lane & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s.O[i0 + (e & 1)][r_lo + 8 * (e >> 1)] = __float2bfloat16_rn(Y[j][e]);
            }
        }
        __syncthreads();  // everyone done with S0, Uu, Us (and O staged)
#pragma unroll
        for (int j = 0; j < 4; ++j) st_c<DK>(s.S0, 16 * mt, 32 * q4 + 8 * j, S[j]);
        if (MODE == 0) {
            const size_t row0 = ((size_t)b * p.T + t0) * p.H + h;
            constexpr int OCH = RT / 8;  // 16-byte chunks per token row
            for (int e = tid; e < L * OCH; e += NTH) {
                const int i = e / OCH, c = e % OCH;
                *reinterpret_cast<uint4*>(p.o + (row0 + (size_t)i * p.H) * DV + a0 + 8 * c) =
                    *reinterpret_cast<const uint4*>(&s.O[i][8 * c]);
            }
        }
    }
    if (MODE == 0 && p.hT) {
        float* hT = p.hT + ((size_t)bh * DV + a0) * DK;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 32 * q4 + 8 * j + 2 * (lane & 3);
#pragma unroll
            for (int e = 0; e < 4; ++e) hT[(size_t)(r_lo + 8 * (e >> 1)) * DK + c + (e & 1)] = S[j][e];
        }
    }
}

ChunkPtrs make_chunk_ptrs(const gdn_dims& d, const TcLayout& L, const void* q, const void* k,
                          const void* v, const float* g, const float* beta, void* ws) {
    ChunkPtrs p{};
    p.q = (const __nv_bfloat16*)q; p.k = (const __nv_bfloat16*)k; p.v = (const __nv_bfloat16*)v;
    p.g = g; p.beta = beta; p.B = d.B; p.T = d.T; p.H = d.H; p.NT = L.NT; p.scale = d.scale;
    char* base = (char*)ws;
    p.W = (__nv_bfloat16*)(base + L.W);
    p.Ut = (__nv_bfloat16*)(base + L.Ut);
    p.P = (__nv_bfloat16*)(base + L.P);
    p.G = (float*)(base + L.G);
    return p;
}

template <int MT, int MODE>
void launch_walk(const WalkPtrs& p, cudaStream_t st) {
    const int smem = sizeof(WalkSmem<MT>);
    cudaFuncSetAttribute(tc_walk_kernel<MT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const int grid = p.B * p.H * (DV / (16 * MT));
    GDN_LAUNCH(MODE == 0 ? "tc_walk_fwd" : "tc_walk_states", st,
               tc_walk_kernel<MT, MODE><<<grid, 128 * MT, smem, st>>>(p));
}

WalkPtrs make_walk_ptrs(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0) {
    WalkPtrs w{};
    w.q = c.q; w.k = c.k; w.h0 = h0; w.W = c.W; w.Ut = c.Ut; w.P = c.P; w.G = c.G;
    w.B = d.B; w.T = d.T; w.H = d.H; w.NT = L.NT; w.scale = d.scale;
    return w;
}

}  // namespace

namespace tc {
void launch_prep(const ChunkPtrs& p, size_t nchunks, cudaStream_t st) {
    const int smem = sizeof(PrepSmem);
    cudaFuncSetAttribute(tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc_prep", st, tc_prep_kernel<<<(unsigned)nchunks, 128, smem, st>>>(p));
}

void launch_walk_states(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp,
                        const float* h0, void* ws, cudaStream_t st) {
    WalkPtrs w = make_walk_ptrs(d, L, cp, h0);
    w.S0out = (__nv_bfloat16*)((char*)ws + L.S0);
    w.Uout = (__nv_bfloat16*)((char*)ws + L.U);
    launch_walk<1, 1>(w, st);
}
}  // namespace tc

bool tc_supported(const gdn_dims& d) {
    return d.dtype == GDN_BF16 && d.dk == DK && d.dv == DV && d.chunk == C &&
           d.gate == GDN_GATE_SCALAR;
}

size_t tc_fwd_workspace(const gdn_dims& d) { return tc_layout(d, false).end; }
size_t tc_bwd_workspace(const gdn_dims& d) { return tc_layout(d, true).end; }

void launch_tc_fwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                   const float* g, const float* beta, const float* h0, void* o, float* hT,
                   void* ws, cudaStream_t st) {
    const TcLayout L = tc_layout(d, false);
    ChunkPtrs cp = make_chunk_ptrs(d, L, q, k, v, g, beta, ws);
    launch_prep(cp, L.nchunks, st);
    WalkPtrs w = make_walk_ptrs(d, L, cp, h0);
    w.o = (__nv_bfloat16*)o;
    w.hT = hT;
    launch_walk<1, 0>(w, st);
}

}  // namespace gdn
