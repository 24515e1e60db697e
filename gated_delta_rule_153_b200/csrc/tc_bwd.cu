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
// This file holds the 16-row reverse walk (tc_walk_bwd: the chunks backwards
// for 16 rows of dS, whose rows, like those of S, never mix, storing dS and dU
// per chunk) and the backward driver.  The whole-head reverse walk is
// tc5_walk_bwd.cu; the local gradients, computed for every chunk in parallel
// from the stored S0, U (forward recompute), dS and dU, are tc5_bwd_local.cu
// and tc5_bwd_local_kda.cu.
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
void launch_prep5_kda(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
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
                   float* dh0, void* ws, cudaStream_t st, const int* cu, int nseq, bool saved) {
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
    if (!saved) {  // else launch_tc_fwd_save left these in ws
        if (kda_gate) launch_prep5_kda(cp, L.nchunks, st);
        else launch_prep(cp, L.nchunks, st);
        launch_walk_states(d, L, cp, h0, ws, st);
    }

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
}

}  // namespace gdn
