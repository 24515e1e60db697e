// tc_bwd.cu -- tensor-core chunkwise backward of the gated delta rule
// (bf16 q/k/v/dO, fp32 state gradients; dk = dv = 128, chunk 64, scalar gate).
//
// Reverse-mode through the chunk equations of the forward (see tc_chunk.cu):
// with dS the gradient w.r.t. the state leaving a chunk and dO the output
// gradient of its tokens,
//   dU  = P^T dO + diag(e^{G_last-G}) K dS^T
//   dS0 = e^{G_last} dS + (scale dO)^T diag(e^G) Q - dU^T W       (next chunk back)
//   dQ' = diag(e^G) dO S0 + (dP .* D) K,          dP = lower(dO U^T)
//   dK  = diag(e^{G_last-G}) U dS + diag(beta e^G) T^T dW + (dM + dM^T) K
//         + (dP .* D)^T Q',                        dW = -dU S0
//   dV  = diag(beta) T^T dU
//   dA  = strict_lower(-T^T dT T^T),  dT = dW (diag(beta e^G) K)^T + dU (diag(beta) V)^T
//   dM  = dA .* beta_i .* D
// plus the gate and beta gradients from the matching row sums, and
// dg = reverse within-chunk cumsum of dG.  (Q' = scale Q; dq = scale dQ'.)
//
// Kernels: tc_walk_bwd walks the chunks backwards for 16 rows of dS (the rows
// of dS, like those of S, never mix) and stores dS and dU per chunk;
// tc_bwd_local then computes every chunk's gradients in parallel from the
// stored S0, U (forward recompute), dS and dU.
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace tc {
void launch_prep(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
bool chunk_ptrs(ChunkPtrs& p, const gdn_dims& d, const TcLayout& L, const void* q,
                const void* k, const void* v, const float* g, const float* beta, void* ws);
void launch_walk_states(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp,
                        const float* h0, void* ws, cudaStream_t st);
void launch_prep_kda(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
bool launch_bwd_local_kda(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp,
                          const void* dO, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                          void* ws, cudaStream_t st);
bool whole_head_walk(const gdn_dims& d, const SeqMap& seq);
bool launch_walk5_bwd(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const void* dO,
                      const float* dhT, float* dh0, void* ws, cudaStream_t st);
bool launch_bwd_local5(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp, const void* dO,
                       void* dq, void* dk, void* dv, float* dg, float* dbeta, void* ws, cudaStream_t st);
bool launch_bwd_local5_kda(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp, const void* dO,
                           void* dq, void* dk, void* dv, float* dg, float* dbeta, void* ws, cudaStream_t st);
}  // namespace tc

namespace {
using namespace tc;

// ---------------------------------------------------------------------------
// reverse walk: dS for 16 value-rows, chunks NT-1 .. 0, 8 warps.
// Warp w: tokens 8w..8w+7 of dU^T, key columns 16w..16w+15 of dS.
// Chunk tiles arrive on a three-stage mbarrier ring (Q, K, dO by TMA tensor
// maps; W, P, G by bulk copies of the workspace images).
// ---------------------------------------------------------------------------
constexpr int BW_THREADS = 256;
constexpr int BW_STAGES = 3;

// One CTA walks 16*MT value rows of dS (MT m-tiles per warp).
template <int MT>
struct alignas(1024) BwStage {
    __nv_bfloat16 Q[C * DK];       // Tma128
    __nv_bfloat16 K[C * DK];       // Tma128
    __nv_bfloat16 W[C * DK];       // Tma128
    __nv_bfloat16 P[C * C];        // Swz<64>
    __nv_bfloat16 dO[C * 16 * MT]; // [token][16*MT value columns]
    float G[DK];                   // G (scalar gate) or e^{G_last,c} (channel gate)
};

template <int MT>
struct BwSmem {
    BwStage<MT> st[BW_STAGES];
    __nv_bfloat16 dS[16 * MT * DK];  // Swz<128>: bf16 copy of dS (rows x key columns)
    __nv_bfloat16 dOt[16 * MT * C];  // Swz<64>: dO^T tile
    __nv_bfloat16 dOg[16 * MT * C];  // Swz<64>: dO^T * scale * e^{G_i}
    __nv_bfloat16 dU[16 * MT * C];   // Swz<64>: dU^T
    __nv_bfloat16 dUst[C * 16 * MT]; // [token][row] staging for the dU store
    uint64_t full[BW_STAGES];
};

struct BwPtrs {
    CUtensorMap qmap, kmap, dOmap;
    const float* dhT;
    const __nv_bfloat16 *W, *P;
    const __nv_bfloat16 *Qg, *Kt;  // channel gate: prepared Q and K images
    const float* G;
    __nv_bfloat16 *dSout, *dUout;
    float* dh0;
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    SeqMap seq;
};

// KDA: Q and K arrive pre-scaled (scale Q .* e^G, K .* e^{G_last-G}) as
// workspace images, with the per-key chunk decay e^{G_last,c}.
template <int MT, bool KDA>
__device__ void bw_issue(BwStage<MT>& st, uint64_t* bar, const BwPtrs& p, const Chain& ch, int h,
                         int j, int a0) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + j;  // chunk j of the chain
    constexpr int GW = KDA ? DK : C;
    mbar_arrive_expect(bar, (3 * C * DK + C * C + C * 16 * MT) * 2 + GW * 4);
    const int tok = ch.tok0 + j * C;
    if (KDA) {
        bulk_g2s(st.Q, p.Qg + cid * C * DK, C * DK * 2, bar);
        bulk_g2s(st.K, p.Kt + cid * C * DK, C * DK * 2, bar);
    } else {
        tma_load_tile(st.Q, &p.qmap, h, tok, bar);
        tma_load_tile(st.K, &p.kmap, h, tok, bar);
    }
    tma_load_3d(st.dO, &p.dOmap, a0, h, tok, bar);
    bulk_g2s(st.W, p.W + cid * C * DK, C * DK * 2, bar);
    bulk_g2s(st.P, p.P + cid * C * C, C * C * 2, bar);
    bulk_g2s(st.G, p.G + cid * GW, GW * 4, bar);
}

template <int MT, bool KDA>
__global__ void __launch_bounds__(BW_THREADS) tc_walk_bwd_kernel(const __grid_constant__ BwPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BwSmem<MT>& s = *reinterpret_cast<BwSmem<MT>*>(align1k(smem_raw));
    constexpr int RT = 16 * MT;
    constexpr int TILES = DV / RT;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int bh = blockIdx.x / TILES, a0 = (blockIdx.x % TILES) * RT;
    const int h = bh % p.H;  // bh: state row (sequence * H + head)
    const Chain ch = chain_of(p.seq, p.T, p.H, p.NT, bh / p.H, h);
    const int nsteps = ch.n1 - ch.n0;
    const int r_lo = lane >> 2;
    const int i0 = 8 * w + 2 * (lane & 3);  // this thread's token pair in dU^T

    if (tid == 0) {
        for (int i = 0; i < BW_STAGES; ++i) mbar_init(&s.full[i], 1);
        fence_mbar_init();
    }
    // dS: m-tile mt, rows 16mt + r_lo (+8); columns 16w + 8j + 2(lane%4) + {0,1}
    float dS[MT][2][4];
    {
        const float* src = p.dhT ? p.dhT + ((size_t)bh * DV + a0) * DK : nullptr;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = 16 * w + 8 * j + 2 * (lane & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dS[mt][j][e] =
                        src ? src[(size_t)(16 * mt + r_lo + 8 * (e >> 1)) * DK + c + (e & 1)] : 0.f;
            }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int j = 0; j < 2; ++j) st_c<Swz<128>>(s.dS, 16 * mt, 16 * w + 8 * j, dS[mt][j]);
    fence_async_smem();
    __syncthreads();
    if (tid == 0)
        for (int k = 0; k < BW_STAGES - 1 && k < nsteps; ++k)
            bw_issue<MT, KDA>(s.st[k], &s.full[k], p, ch, h, nsteps - 1 - k, a0);

    for (int k = 0; k < nsteps; ++k) {  // step k handles chunk j = nsteps-1-k of the chain
        const int j = nsteps - 1 - k;
        const int sk = k % BW_STAGES;
        BwStage<MT>& st = s.st[sk];
        if (__syncthreads_or(!mbar_wait(&s.full[sk], (k / BW_STAGES) & 1, p.status))) return;  // all threads agree; stage landed; dS written; stage of step k-1 is free
        if (tid == 0 && k + BW_STAGES - 1 < nsteps) {
            const int kk = k + BW_STAGES - 1;
            bw_issue<MT, KDA>(s.st[kk % BW_STAGES], &s.full[kk % BW_STAGES], p, ch, h,
                              nsteps - 1 - kk, a0);
        }
        const size_t cid = (size_t)ch.img * p.NT + ch.n0 + j;
        const int L = min(C, ch.end - (ch.tok0 + j * C));
        // dS leaving chunk n: rows a0.. into the Kp<128> image (a0 is a multiple
        // of 16, so a 16-byte piece keeps its swizzled position)
        for (int e = tid; e < RT * 16; e += BW_THREADS) {
            const int r = e >> 4, pos = e & 15;
            *reinterpret_cast<uint4*>(p.dSout + cid * DV * DK + (pos >> 3) * (DV * 64) + (a0 + r) * 64 +
                                      (pos & 7) * 8) = *reinterpret_cast<const uint4*>(s.dS + r * DK + pos * 8);
        }
        // dO^T tiles (rows past the sequence end are zeroed: they are not ours)
        for (int e = tid; e < C * RT; e += BW_THREADS) {
            const int i = e / RT, a = e % RT;
            const float x = i < L ? __bfloat162float(st.dO[i * RT + a]) : 0.f;
            s.dOt[swz<C>(a, i)] = __float2bfloat16_rn(x);
            s.dOg[swz<C>(a, i)] = __float2bfloat16_rn(KDA ? x : x * p.scale * __expf(st.G[i]));
        }
        __syncthreads();
        const float Gl = KDA ? 0.f : st.G[C - 1];
        const float et0 = KDA ? 1.f : __expf(Gl - st.G[i0]);
        const float et1 = KDA ? 1.f : __expf(Gl - st.G[i0 + 1]);
        // dU^T (rows x tokens 8w..8w+7) = dO^T P + (dS K^T) .* e^{G_last - G_r}
        {
            float a1[MT][4] = {}, a2[MT][2][4] = {};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                if (16 * kk + 15 < 8 * w) continue;  // P[i][r] = 0 for i < r
                uint32_t bp[2];
                ldb_kn1<Swz<64>>(bp, st.P, 16 * kk, 8 * w);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t a[4];
                    lda<Swz<64>>(a, s.dOt, 16 * mt, 16 * kk);
                    mma16816(a1[mt], a, bp[0], bp[1]);
                }
            }
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t bk[2];
                ldb_nk1<Tma128>(bk, st.K, 8 * w, 16 * kk);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t a[4];
                    lda<Swz<128>>(a, s.dS, 16 * mt, 16 * kk);
                    mma16816(a2[mt][kk & 1], a, bk[0], bk[1]);
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                float u[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)  // padding tokens (past the sequence end) stay zero
                    u[e] = (i0 + (e & 1) < L)
                               ? a1[mt][e] + (a2[mt][0][e] + a2[mt][1][e]) * ((e & 1) ? et1 : et0)
                               : 0.f;
                st_c<Swz<64>>(s.dU, 16 * mt, 8 * w, u);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s.dUst[(i0 + (e & 1)) * RT + 16 * mt + r_lo + 8 * (e >> 1)] = __float2bfloat16_rn(u[e]);
            }
        }
        __syncthreads();
        // dS0 = e^{G_last} dS + dOg^T Q - dU^T W   (columns 16w..16w+15)
        {
            const float gam = KDA ? 1.f : __expf(Gl);
            float y[MT][2][4] = {}, z[MT][2][4] = {};
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk) {
                uint32_t bq[4], bw[4];
                ldb_kn<Tma128>(bq, st.Q, 16 * kk, 16 * w);
                ldb_kn<Tma128>(bw, st.W, 16 * kk, 16 * w);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t ag[4], au[4];
                    lda<Swz<64>>(ag, s.dOg, 16 * mt, 16 * kk);
                    lda<Swz<64>>(au, s.dU, 16 * mt, 16 * kk);
                    mma16816(y[mt][0], ag, bq[0], bq[1]);
                    mma16816(y[mt][1], ag, bq[2], bq[3]);
                    mma16816(z[mt][0], au, bw[0], bw[1]);
                    mma16816(z[mt][1], au, bw[2], bw[3]);
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dS[mt][j][e] =
                            (KDA ? st.G[16 * w + 8 * j + 2 * (lane & 3) + (e & 1)] : gam) *
                                dS[mt][j][e] +
                            y[mt][j][e] - z[mt][j][e];
        }
        __syncthreads();  // everyone done with dS, dOt, dOg, dU; dU staged
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j) st_c<Swz<128>>(s.dS, 16 * mt, 16 * w + 8 * j, dS[mt][j]);
        fence_async_smem();
        constexpr int PIECES = RT / 8;
        for (int e = tid; e < PIECES * C; e += BW_THREADS) {  // dU rows, 16-byte pieces
            const int i = e / PIECES, pc = e % PIECES;
            *reinterpret_cast<uint4*>(p.dUout + cid * C * DV + Tma128::off(i, a0 + 8 * pc)) =
                *reinterpret_cast<const uint4*>(&s.dUst[i * RT + 8 * pc]);
        }
    }
    if (p.dh0) {
        float* dst = p.dh0 + ((size_t)bh * DV + a0) * DK;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = 16 * w + 8 * j + 2 * (lane & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[(size_t)(16 * mt + r_lo + 8 * (e >> 1)) * DK + c + (e & 1)] = dS[mt][j][e];
            }
    }
}

// ---------------------------------------------------------------------------
// local gradients: one CTA (16 warps) per chunk.  Warp w owns rows
// 16*(w/4) .. +15 and column quarter (w%4) of every 64x128 and every 64x64
// result.
// ---------------------------------------------------------------------------
constexpr int LOC_WARPS = 16, LOC_THREADS = 32 * LOC_WARPS;

struct LocSmem {
    // Q, K, V, dO: Tma128 tiles (TMA); U, dU: Tma128 images (bulk)
    __nv_bfloat16 Q[C * DK], K[C * DK], V[C * DV], dO[C * DV], U[C * DV], dU[C * DV];
    __nv_bfloat16 S0[DV * DK];  // Kp<128>: rows a (value), cols c (key)
    __nv_bfloat16 dS[DV * DK];
    __nv_bfloat16 dW[C * DK];
    __nv_bfloat16 Tb[C * C];
    __nv_bfloat16 dPG[C * C];   // lower(dO U^T) .* D
    __nv_bfloat16 dT[C * C];
    __nv_bfloat16 X[C * C];     // dT T^T
    __nv_bfloat16 dMM[C * C];   // dA .* beta_i .* D
    float G[C], beta[C];
    float red_b[16][C];  // partial dbeta (by row), per warp
    float red_g[16][C];  // partial dG (by token), per warp
    float red_s[16][2];  // partial scalars for G_last, per warp
    uint64_t bar[2];     // [0]: inputs of the value-dimension contractions, [1]: the rest
};

struct LocPtrs {
    CUtensorMap qmap, kmap, vmap, dOmap;
    const __nv_bfloat16 *q, *k, *v, *dO;
    const float *g, *beta;
    const __nv_bfloat16 *S0, *U, *dS, *dU, *Tb;
    const float* G;
    __nv_bfloat16 *dq, *dk, *dv;
    float *dg, *dbeta;
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    int pf_stride;  // chunks a wave ahead; 0: no prefetch
    SeqMap seq;
};

// Row sums over the 4 lanes of a quad: lo -> row r_lo, hi -> row r_lo + 8.
__device__ __forceinline__ void quad_rows(float& lo, float& hi) {
    lo += __shfl_xor_sync(0xffffffffu, lo, 1);
    lo += __shfl_xor_sync(0xffffffffu, lo, 2);
    hi += __shfl_xor_sync(0xffffffffu, hi, 1);
    hi += __shfl_xor_sync(0xffffffffu, hi, 2);
}
// Column sums over the 8 row-groups of a warp (lanes with equal lane%4).
__device__ __forceinline__ float col_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    return v;
}

__global__ void __launch_bounds__(LOC_THREADS) tc_bwd_local_kernel(const __grid_constant__ LocPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    LocSmem& s = *reinterpret_cast<LocSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int rb = w >> 2, cq = w & 3;
    const int m0 = 16 * rb;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, h = bh % p.H;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, n);
    if (!cl.valid) return;  // past the last chunk of a packed batch
    const int L = cl.L;
    const size_t row0 = (size_t)cl.tok * p.H + h;
    const size_t rs = (size_t)p.H;
    const int rl = m0 + (lane >> 2), rh = rl + 8;  // this thread's two rows

    if (tid == 0) {
        mbar_init(&s.bar[0], 1);
        mbar_init(&s.bar[1], 1);
        fence_mbar_init();
        const int tok = cl.tok;
        // phase 1 (contractions over the value dimension) needs dO, Q, K, U, dU,
        // S0, dS, G; V and T are first used after it
        mbar_arrive_expect(&s.bar[0], (5 * C * DK + 2 * DV * DK) * 2 + C * 4);
        tma_load_tile(s.dO, &p.dOmap, h, tok, &s.bar[0]);
        tma_load_tile(s.Q, &p.qmap, h, tok, &s.bar[0]);
        tma_load_tile(s.K, &p.kmap, h, tok, &s.bar[0]);
        bulk_g2s(s.U, p.U + (size_t)cid * C * DV, C * DV * 2, &s.bar[0]);
        bulk_g2s(s.dU, p.dU + (size_t)cid * C * DV, C * DV * 2, &s.bar[0]);
        bulk_g2s(s.S0, p.S0 + (size_t)cid * DV * DK, DV * DK * 2, &s.bar[0]);
        bulk_g2s(s.dS, p.dS + (size_t)cid * DV * DK, DV * DK * 2, &s.bar[0]);
        bulk_g2s(s.G, p.G + (size_t)cid * C, C * 4, &s.bar[0]);
        mbar_arrive_expect(&s.bar[1], (C * DK + C * C) * 2);
        tma_load_tile(s.V, &p.vmap, h, tok, &s.bar[1]);
        bulk_g2s(s.Tb, p.Tb + (size_t)cid * C * C, C * C * 2, &s.bar[1]);
        // the chunk a wave ahead: its tiles and images wait in L2 when its CTA starts
        const int pc = cid + p.pf_stride;
        if (p.pf_stride > 0 && pc < (int)gridDim.x) {
            const int pbh = pc / p.NT, pn = pc % p.NT, ph = pbh % p.H;
            const ChunkLoc pl = chunk_loc(p.seq, p.T, p.H, pbh, pn);
            const int ptok = pl.valid ? pl.tok : 0;
            tma_prefetch_tile(&p.dOmap, ph, ptok);
            tma_prefetch_tile(&p.qmap, ph, ptok);
            tma_prefetch_tile(&p.kmap, ph, ptok);
            tma_prefetch_tile(&p.vmap, ph, ptok);
            bulk_prefetch_l2(p.U + (size_t)pc * C * DV, C * DV * 2);
            bulk_prefetch_l2(p.dU + (size_t)pc * C * DV, C * DV * 2);
            bulk_prefetch_l2(p.S0 + (size_t)pc * DV * DK, DV * DK * 2);
            bulk_prefetch_l2(p.dS + (size_t)pc * DV * DK, DV * DK * 2);
            bulk_prefetch_l2(p.Tb + (size_t)pc * C * C, C * C * 2);
        }
    }
    for (int e = tid; e < C; e += LOC_THREADS) s.beta[e] = e < L ? p.beta[row0 + e * rs] : 0.f;
    for (int e = tid; e < LOC_WARPS * C; e += LOC_THREADS) {
        (&s.red_b[0][0])[e] = 0.f;
        (&s.red_g[0][0])[e] = 0.f;
    }
    if (tid < 2 * LOC_WARPS) (&s.red_s[0][0])[tid] = 0.f;
    __syncthreads();
    if (__syncthreads_or(!mbar_wait(&s.bar[0], 0, p.status))) return;
    if (L < C) {  // dO rows past the sequence end belong to the next sequence: zero them
        for (int e = tid; e < (C - L) * DV; e += LOC_THREADS) {
            const int r = L + e / DV, c = e % DV;
            s.dO[Tma128::off(r, c)] = __float2bfloat16_rn(0.f);
        }
    }
    __syncthreads();

    const float Gl = s.G[C - 1];
    const float egl = __expf(s.G[rl]), egh = __expf(s.G[rh]);
    const float etl = __expf(Gl - s.G[rl]), eth = __expf(Gl - s.G[rh]);
    const float bl = s.beta[rl], bhh = s.beta[rh];
    float row_b_lo = 0.f, row_b_hi = 0.f;  // partial dbeta for rows rl, rh
    float row_g_lo = 0.f, row_g_hi = 0.f;  // partial dG for rows rl, rh
    float last_acc = 0.f;                  // partial dG_last (sum over rows of hkt)

    // dQ' and dK accumulators: rows rl/rh, columns 32*cq + 8j + 2(lane%4) + {0,1}
    float dQ[4][4], dK[4][4];

    // ---- phase 1: contractions over the value dimension --------------------
    {
        float acc[4][4];
        // dQg = dO S0  ->  dQ' = e^G dQg ;  dG += scale e^G sum_c dQg Q
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t a[4];
            lda<Tma128>(a, s.dO, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bf[4];
                ldb_kn<Kp<DV>>(bf, s.S0, 16 * kk, 32 * cq + 16 * np);
                mma16816(acc[2 * np], a, bf[0], bf[1]);
                mma16816(acc[2 * np + 1], a, bf[2], bf[3]);
            }
        }
        float hq_lo = 0.f, hq_hi = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 32 * cq + 8 * j + 2 * (lane & 3);
            const float2 ql = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.Q + Tma128::off(rl, c)));
            const float2 qh = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.Q + Tma128::off(rh, c)));
            hq_lo += acc[j][0] * ql.x + acc[j][1] * ql.y;
            hq_hi += acc[j][2] * qh.x + acc[j][3] * qh.y;
            dQ[j][0] = egl * acc[j][0]; dQ[j][1] = egl * acc[j][1];
            dQ[j][2] = egh * acc[j][2]; dQ[j][3] = egh * acc[j][3];
        }
        row_g_lo += p.scale * egl * hq_lo;
        row_g_hi += p.scale * egh * hq_hi;

        // dKt = U dS  ->  dK = e^{Gl-G} dKt ;  hkt = e^{Gl-G} sum_c dKt K
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t a[4];
            lda<Tma128>(a, s.U, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bf[4];
                ldb_kn<Kp<DV>>(bf, s.dS, 16 * kk, 32 * cq + 16 * np);
                mma16816(acc[2 * np], a, bf[0], bf[1]);
                mma16816(acc[2 * np + 1], a, bf[2], bf[3]);
            }
        }
        float hk_lo = 0.f, hk_hi = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 32 * cq + 8 * j + 2 * (lane & 3);
            const float2 kl = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.K + Tma128::off(rl, c)));
            const float2 kh = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.K + Tma128::off(rh, c)));
            hk_lo += acc[j][0] * kl.x + acc[j][1] * kl.y;
            hk_hi += acc[j][2] * kh.x + acc[j][3] * kh.y;
            dK[j][0] = etl * acc[j][0]; dK[j][1] = etl * acc[j][1];
            dK[j][2] = eth * acc[j][2]; dK[j][3] = eth * acc[j][3];
        }
        row_g_lo -= etl * hk_lo;
        row_g_hi -= eth * hk_hi;
        last_acc += etl * hk_lo + eth * hk_hi;

        // dW = -dU S0  -> bf16 tile
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t a[4];
            lda<Tma128>(a, s.dU, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bf[4];
                ldb_kn<Kp<DV>>(bf, s.S0, 16 * kk, 32 * cq + 16 * np);
                mma16816(acc[2 * np], a, bf[0], bf[1]);
                mma16816(acc[2 * np + 1], a, bf[2], bf[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float x[4] = {-acc[j][0], -acc[j][1], -acc[j][2], -acc[j][3]};
            st_c<DK>(s.dW, m0, 32 * cq + 8 * j, x);
        }

        // dP = lower(dO U^T), QK = Q K^T on tokens 16*cq .. +15
        float dp[2][4] = {}, qk[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t ad[4], aq[4];
            lda<Tma128>(ad, s.dO, m0, 16 * kk);
            lda<Tma128>(aq, s.Q, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 1; ++np) {
                uint32_t bu[4], bk[4];
                ldb_nk<Tma128>(bu, s.U, 16 * cq + 16 * np, 16 * kk);
                ldb_nk<Tma128>(bk, s.K, 16 * cq + 16 * np, 16 * kk);
                mma16816(dp[2 * np], ad, bu[0], bu[1]);
                mma16816(dp[2 * np + 1], ad, bu[2], bu[3]);
                mma16816(qk[2 * np], aq, bk[0], bk[1]);
                mma16816(qk[2 * np + 1], aq, bk[2], bk[3]);
            }
        }
        // hP = dP .* (scale Q K^T .* D) ;  dPG = dP .* D
        float colp[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c0 = 16 * cq + 8 * j + 2 * (lane & 3);
            float g[4];
            colp[j][0] = colp[j][1] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = (e < 2) ? rl : rh, c = c0 + (e & 1);
                const float d = (c <= r) ? __expf(s.G[r] - s.G[c]) : 0.f;
                g[e] = dp[j][e] * d;
                const float hp = g[e] * p.scale * qk[j][e];
                if (e < 2) row_g_lo += hp; else row_g_hi += hp;
                colp[j][e & 1] -= hp;
            }
            st_c<C>(s.dPG, m0, 16 * cq + 8 * j, g);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float v = col_sum(colp[j][e]);
                if (lane < 4) s.red_g[w][16 * cq + 8 * j + 2 * lane + e] += v;
            }
        // e^{G_last} <dS, S0> (each warp a slice of the 128x128 elements)
        float ss = 0.f;
        for (int e = lane + 32 * w; e < DV * DK / 8; e += LOC_THREADS) {
            const int r = e / (DK / 8), c8 = e % (DK / 8);
            const uint4 x = *reinterpret_cast<const uint4*>(s.dS + swz<DK>(r, 8 * c8));
            const uint4 y = *reinterpret_cast<const uint4*>(s.S0 + swz<DK>(r, 8 * c8));
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 a = unpack_bf16(xs[t]), bb = unpack_bf16(ys[t]);
                ss += a.x * bb.x + a.y * bb.y;
            }
        }
        ss = warp_sum(ss);
        last_acc = warp_sum(last_acc);  // over rows of this warp (both halves)
        if (lane == 0) {
            s.red_s[w][0] = ss;
            s.red_s[w][1] = last_acc;
        }
    }

    // ---- phase 2: K K^T (-> M), dT ---------------------------------------
    float M[2][4];
    {
        float kkt[2][4] = {}, tw[2][4] = {}, tu[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t ak[4];
            lda<Tma128>(ak, s.K, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 1; ++np) {
                uint32_t bk[4];
                ldb_nk<Tma128>(bk, s.K, 16 * cq + 16 * np, 16 * kk);
                mma16816(kkt[2 * np], ak, bk[0], bk[1]);
                mma16816(kkt[2 * np + 1], ak, bk[2], bk[3]);
            }
        }
        if (__syncthreads_or(!mbar_wait(&s.bar[1], 0, p.status))) return;  // all threads agree; dW tile complete; V and T landed
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t aw[4], au[4];
            lda<DK>(aw, s.dW, m0, 16 * kk);
            lda<Tma128>(au, s.dU, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 1; ++np) {
                uint32_t bk[4], bv[4];
                ldb_nk<Tma128>(bk, s.K, 16 * cq + 16 * np, 16 * kk);
                ldb_nk<Tma128>(bv, s.V, 16 * cq + 16 * np, 16 * kk);
                mma16816(tw[2 * np], aw, bk[0], bk[1]);
                mma16816(tw[2 * np + 1], aw, bk[2], bk[3]);
                mma16816(tu[2 * np], au, bv[0], bv[1]);
                mma16816(tu[2 * np + 1], au, bv[2], bv[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c0 = 16 * cq + 8 * j + 2 * (lane & 3);
            float dt[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = (e < 2) ? rl : rh, c = c0 + (e & 1);
                const float bj = s.beta[c];
                dt[e] = tw[j][e] * bj * __expf(s.G[c]) + tu[j][e] * bj;
                M[j][e] = (c < r) ? kkt[j][e] * __expf(s.G[r] - s.G[c]) : 0.f;
            }
            st_c<C>(s.dT, m0, 16 * cq + 8 * j, dt);
        }
    }
    __syncthreads();

    // ---- phase 3: X = dT T^T ; dKg = T^T dW ; dVb = T^T dU ------------------
    {
        float x[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4];
            lda<C>(a, s.dT, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 1; ++np) {
                uint32_t bt[4];
                ldb_nk<C>(bt, s.Tb, 16 * cq + 16 * np, 16 * kk);
                mma16816(x[2 * np], a, bt[0], bt[1]);
                mma16816(x[2 * np + 1], a, bt[2], bt[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) st_c<C>(s.X, m0, 16 * cq + 8 * j, x[j]);

        float akg[4][4] = {}, avb[4][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk < rb) continue;  // T[j][i] = 0 for j < i
            uint32_t a[4];
            lda_t<C>(a, s.Tb, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bw[4], bu[4];
                ldb_kn<DK>(bw, s.dW, 16 * kk, 32 * cq + 16 * np);
                ldb_kn<Tma128>(bu, s.dU, 16 * kk, 32 * cq + 16 * np);
                mma16816(akg[2 * np], a, bw[0], bw[1]);
                mma16816(akg[2 * np + 1], a, bw[2], bw[3]);
                mma16816(avb[2 * np], a, bu[0], bu[1]);
                mma16816(avb[2 * np + 1], a, bu[2], bu[3]);
            }
        }
        float hk_lo = 0.f, hk_hi = 0.f, hv_lo = 0.f, hv_hi = 0.f;
        const bool okl = rl < L, okh = rh < L;
        __nv_bfloat16* dvp = p.dv + row0 * DV;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 32 * cq + 8 * j + 2 * (lane & 3);
            const float2 kl = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.K + Tma128::off(rl, c)));
            const float2 kh = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.K + Tma128::off(rh, c)));
            const float2 vl = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.V + Tma128::off(rl, c)));
            const float2 vh = unpack_bf16(*reinterpret_cast<const uint32_t*>(s.V + Tma128::off(rh, c)));
            hk_lo += akg[j][0] * kl.x + akg[j][1] * kl.y;
            hk_hi += akg[j][2] * kh.x + akg[j][3] * kh.y;
            hv_lo += avb[j][0] * vl.x + avb[j][1] * vl.y;
            hv_hi += avb[j][2] * vh.x + avb[j][3] * vh.y;
            dK[j][0] += bl * egl * akg[j][0]; dK[j][1] += bl * egl * akg[j][1];
            dK[j][2] += bhh * egh * akg[j][2]; dK[j][3] += bhh * egh * akg[j][3];
            if (okl)
                *reinterpret_cast<uint32_t*>(dvp + (size_t)rl * rs * DV + c) =
                    pack_bf16(bl * avb[j][0], bl * avb[j][1]);
            if (okh)
                *reinterpret_cast<uint32_t*>(dvp + (size_t)rh * rs * DV + c) =
                    pack_bf16(bhh * avb[j][2], bhh * avb[j][3]);
        }
        row_b_lo += egl * hk_lo + hv_lo;
        row_b_hi += egh * hk_hi + hv_hi;
        row_g_lo += bl * egl * hk_lo;
        row_g_hi += bhh * egh * hk_hi;
    }
    __syncthreads();

    // ---- phase 4: dA = -T^T X (strictly lower) ------------------------------
    {
        float da[2][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk < rb) continue;
            uint32_t a[4];
            lda_t<C>(a, s.Tb, m0, 16 * kk);
#pragma unroll
            for (int np = 0; np < 1; ++np) {
                uint32_t bx[4];
                ldb_kn<C>(bx, s.X, 16 * kk, 16 * cq + 16 * np);
                mma16816(da[2 * np], a, bx[0], bx[1]);
                mma16816(da[2 * np + 1], a, bx[2], bx[3]);
            }
        }
        float colp[2][2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c0 = 16 * cq + 8 * j + 2 * (lane & 3);
            float mm[4];
            colp[j][0] = colp[j][1] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = (e < 2) ? rl : rh, c = c0 + (e & 1);
                const float dA = (c < r) ? -da[j][e] : 0.f;
                const float br = (e < 2) ? bl : bhh;
                // M already carries the decay D
                const float hA = dA * br * M[j][e];
                if (e < 2) { row_b_lo += dA * M[j][e]; row_g_lo += hA; }
                else { row_b_hi += dA * M[j][e]; row_g_hi += hA; }
                colp[j][e & 1] -= hA;
                mm[e] = (c < r) ? dA * br * __expf(s.G[r] - s.G[c]) : 0.f;
            }
            st_c<C>(s.dMM, m0, 16 * cq + 8 * j, mm);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float v = col_sum(colp[j][e]);
                if (lane < 4) s.red_g[w][16 * cq + 8 * j + 2 * lane + e] += v;
            }
    }
    __syncthreads();

    // ---- phase 5: dK += dMM K + dMM^T K + scale dPG^T Q ; dQ' += dPG K -------
    {
        float tq[4][4] = {};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t am[4], amt[4], ap[4], apt[4];
            const bool lo = kk <= rb, hi = kk >= rb;
            if (lo) { lda<C>(am, s.dMM, m0, 16 * kk); lda<C>(ap, s.dPG, m0, 16 * kk); }
            if (hi) { lda_t<C>(amt, s.dMM, m0, 16 * kk); lda_t<C>(apt, s.dPG, m0, 16 * kk); }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bk[4], bq[4];
                ldb_kn<Tma128>(bk, s.K, 16 * kk, 32 * cq + 16 * np);
                if (lo) {
                    mma16816(dK[2 * np], am, bk[0], bk[1]);
                    mma16816(dK[2 * np + 1], am, bk[2], bk[3]);
                    mma16816(dQ[2 * np], ap, bk[0], bk[1]);
                    mma16816(dQ[2 * np + 1], ap, bk[2], bk[3]);
                }
                if (hi) {
                    ldb_kn<Tma128>(bq, s.Q, 16 * kk, 32 * cq + 16 * np);
                    mma16816(dK[2 * np], amt, bk[0], bk[1]);
                    mma16816(dK[2 * np + 1], amt, bk[2], bk[3]);
                    mma16816(tq[2 * np], apt, bq[0], bq[1]);
                    mma16816(tq[2 * np + 1], apt, bq[2], bq[3]);
                }
            }
        }
        const bool okl = rl < L, okh = rh < L;
        __nv_bfloat16* dqp = p.dq + row0 * DK;
        __nv_bfloat16* dkp = p.dk + row0 * DK;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = 32 * cq + 8 * j + 2 * (lane & 3);
            if (okl) {
                *reinterpret_cast<uint32_t*>(dqp + (size_t)rl * rs * DK + c) =
                    pack_bf16(p.scale * dQ[j][0], p.scale * dQ[j][1]);
                *reinterpret_cast<uint32_t*>(dkp + (size_t)rl * rs * DK + c) =
                    pack_bf16(dK[j][0] + p.scale * tq[j][0], dK[j][1] + p.scale * tq[j][1]);
            }
            if (okh) {
                *reinterpret_cast<uint32_t*>(dqp + (size_t)rh * rs * DK + c) =
                    pack_bf16(p.scale * dQ[j][2], p.scale * dQ[j][3]);
                *reinterpret_cast<uint32_t*>(dkp + (size_t)rh * rs * DK + c) =
                    pack_bf16(dK[j][2] + p.scale * tq[j][2], dK[j][3] + p.scale * tq[j][3]);
            }
        }
    }

    // ---- per-token reductions: dbeta, dG -> dg --------------------------------
    quad_rows(row_b_lo, row_b_hi);
    quad_rows(row_g_lo, row_g_hi);
    if ((lane & 3) == 0) {
        s.red_b[w][rl] += row_b_lo;
        s.red_b[w][rh] += row_b_hi;
        s.red_g[w][rl] += row_g_lo;
        s.red_g[w][rh] += row_g_hi;
    }
    __syncthreads();
    if (w == 0) {
        // red_s[w][0]: warp w's slice of <dS, S0>; red_s[w][1]: its rows' sum of
        // e^{G_last-G_i} <dKt_i, k_i> over its column half.
        float ssum = 0.f, lsum = 0.f;
        for (int ww = 0; ww < LOC_WARPS; ++ww) {
            ssum += s.red_s[ww][0];
            lsum += s.red_s[ww][1];
        }
        float dG0 = 0.f, dG1 = 0.f, db0 = 0.f, db1 = 0.f;
        for (int ww = 0; ww < LOC_WARPS; ++ww) {
            dG0 += s.red_g[ww][lane];
            dG1 += s.red_g[ww][lane + 32];
            db0 += s.red_b[ww][lane];
            db1 += s.red_b[ww][lane + 32];
        }
        if (lane == 31) dG1 += __expf(Gl) * ssum + lsum;
        // reverse cumsum over the 64 tokens: dg_i = sum_{j >= i} dG_j
        float x1 = dG1, x0 = dG0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y1 = __shfl_down_sync(0xffffffffu, x1, o);
            const float y0 = __shfl_down_sync(0xffffffffu, x0, o);
            if (lane + o < 32) { x1 += y1; x0 += y0; }
        }
        x0 += __shfl_sync(0xffffffffu, x1, 0);
        if (lane < L) {
            p.dg[row0 + lane * rs] = x0;
            p.dbeta[row0 + lane * rs] = db0;
        }
        if (lane + 32 < L) {
            p.dg[row0 + (lane + 32) * rs] = x1;
            p.dbeta[row0 + (lane + 32) * rs] = db1;
        }
    }
}

template <int MT, bool KDA>
void launch_walk_bwd(const BwPtrs& bp, cudaStream_t st) {
    const int smem = sizeof(BwSmem<MT>) + 1024;
    cudaFuncSetAttribute(tc_walk_bwd_kernel<MT, KDA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         smem);
    GDN_LAUNCH("tc_walk_bwd", st,
               (tc_walk_bwd_kernel<MT, KDA><<<bp.B * bp.H * (DV / (16 * MT)), BW_THREADS, smem,
                                              st>>>(bp)));
}

// The 16-row reverse walk (few heads): bp carries the dS / dU outputs.
bool launch_walk_bwd16(const gdn_dims& d, const ChunkPtrs& cp, const void* dO, const float* dhT,
                       float* dh0, BwPtrs& bp, cudaStream_t st) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool two = (long long)chain_batches(d.B, cp.seq) * d.H * (DV / 32) >= sms;  // two m-tiles per warp
    bp.qmap = cp.qmap; bp.kmap = cp.kmap;
    if (!encode_token_map(&bp.dOmap, dO, d.B, d.T, d.H, two ? 32 : 16)) return false;
    bp.dhT = dhT; bp.W = cp.W; bp.P = cp.P; bp.G = cp.G;
    bp.dh0 = dh0; bp.status = cp.status;
    bp.B = chain_batches(d.B, cp.seq); bp.T = d.T; bp.H = d.H; bp.NT = cp.NT; bp.scale = d.scale;
    bp.seq = cp.seq;
    bp.Qg = cp.Qg; bp.Kt = cp.Kt;
    const bool kda = d.gate == GDN_GATE_CHANNEL;
    if (two) {
        if (kda) launch_walk_bwd<2, true>(bp, st);
        else launch_walk_bwd<2, false>(bp, st);
    } else {
        if (kda) launch_walk_bwd<1, true>(bp, st);
        else launch_walk_bwd<1, false>(bp, st);
    }
    return true;
}

}  // namespace

bool tc_bwd_supported(const gdn_dims& d) { return tc_supported(d); }

bool launch_tc_bwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                   const float* g, const float* beta, const float* h0, const void* dO,
                   const float* dhT, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                   float* dh0, void* ws, cudaStream_t st, const int* cu, int nseq) {
    const TcLayout L = tc_layout(d, true, nseq);
    char* base = (char*)ws;
    ChunkPtrs cp;
    if (!chunk_ptrs(cp, d, L, q, k, v, g, beta, ws)) return false;
    cp.Tb = (__nv_bfloat16*)(base + L.Tb);
    if (nseq) {
        int* cstart = (int*)(base + L.cstart);
        launch_varlen_setup(cu, nseq, d.T, cstart, cp.status, st);
        cp.seq = SeqMap{cu, cstart, nseq};
    }
    const bool kda_gate = d.gate == GDN_GATE_CHANNEL;
    if (kda_gate) launch_prep_kda(cp, L.nchunks, st);
    else launch_prep(cp, L.nchunks, st);
    launch_walk_states(d, L, cp, h0, ws, st);

    BwPtrs bp{};
    bp.dSout = (__nv_bfloat16*)(base + L.dS);
    bp.dUout = (__nv_bfloat16*)(base + L.dU);
    if (whole_head_walk(d, cp.seq) || L.nseg > 1) {
        if (!launch_walk5_bwd(d, L, cp, dO, dhT, dh0, ws, st)) return false;
    } else if (!launch_walk_bwd16(d, cp, dO, dhT, dh0, bp, st)) {
        return false;
    }
    if (kda_gate)
        return launch_bwd_local5_kda(d, L, cp, dO, dq, dk, dv, dg, dbeta, ws, st);
    return launch_bwd_local5(d, L, cp, dO, dq, dk, dv, dg, dbeta, ws, st);
    LocPtrs lp{};
    lp.qmap = cp.qmap; lp.kmap = cp.kmap; lp.vmap = cp.vmap;
    if (!encode_token_map(&lp.dOmap, dO, d.B, d.T, d.H)) return false;
    lp.q = cp.q; lp.k = cp.k; lp.v = cp.v; lp.dO = (const __nv_bfloat16*)dO; lp.g = g;
    lp.beta = beta; lp.status = cp.status;
    lp.S0 = (const __nv_bfloat16*)(base + L.S0);
    lp.U = (const __nv_bfloat16*)(base + L.U);
    lp.dS = bp.dSout; lp.dU = bp.dUout; lp.Tb = cp.Tb; lp.G = cp.G;
    lp.dq = (__nv_bfloat16*)dq; lp.dk = (__nv_bfloat16*)dk; lp.dv = (__nv_bfloat16*)dv;
    lp.dg = dg; lp.dbeta = dbeta;
    lp.B = d.B; lp.T = d.T; lp.H = d.H; lp.NT = L.NT; lp.scale = d.scale;
    lp.seq = cp.seq;
    {
        const int smem = sizeof(LocSmem) + 1024;
        cudaFuncSetAttribute(tc_bwd_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        lp.pf_stride = sms;  // one CTA per SM
        GDN_LAUNCH("tc_bwd_local", st,
                   tc_bwd_local_kernel<<<(unsigned)L.nchunks, LOC_THREADS, smem, st>>>(lp));
    }
    return true;
}

}  // namespace gdn
