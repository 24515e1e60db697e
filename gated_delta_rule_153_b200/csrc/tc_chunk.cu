// tc_chunk.cu -- tensor-core chunkwise gated delta rule, bf16 in, fp32 state.
//
// Shapes: dk = dv = 128, chunk C = 64, scalar gate.  The chunkwise algebra is
// the WY / UT-transform form of "Gated Delta Networks: Improving Mamba2 with
// Delta Rule" (paper review), sections "Goal" and "Method"; per chunk, with
// S0 the state entering it and G the within-chunk cumsum of the log-gate g:
//   A  = strict_lower(diag(beta) (K K^T .* D)),   D_ij = exp(G_i - G_j)
//   T  = (I + A)^{-1}                              (UT transform)
//   W  = T diag(beta e^G) K,   U~ = T diag(beta) V  (WY factors)
//   P  = scale lower(Q K^T .* D)
//   U  = U~ - W S0^T
//   O  = scale diag(e^G) Q S0^T + P U
//   S1 = e^{G_last} S0 + U^T diag(e^{G_last - G}) K
//
// This file holds the 16-row walk and the forward driver (the preparation is
// tc5_prep.cu / tc5_prep_kda.cu, the whole-head walks tc5_walk.cu):
//   walk   -- grid over (b, h, 16-row tile of S): the sequential chain
//             U -> S1 -> ... in fp32, plus O (forward) or the chunk-start
//             states and U (backward recompute).
// Rows of S never mix (row a of S pairs only with column a of V, U, O), so the
// walk splits the state by value rows and every CTA carries its own chain.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc_common.cuh"

#include <mutex>

namespace gdn {
namespace tc {
void launch_prep5_kda(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
void launch_prep5(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
void launch_prep5_conv(const ChunkPtrs& p, size_t nchunks, cudaStream_t st);
void launch_walk5_fwd(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0,
                      void* o, float* hT, void* ws, cudaStream_t st, bool save = false);
void launch_walk5_states(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0,
                         void* ws, cudaStream_t st);
}
namespace {
using namespace tc;
using S128 = Swz<128>;
using S64 = Swz<64>;
using P128 = Pad<128>;

// ---------------------------------------------------------------------------
// walk: the sequential chain over chunks for 16 rows of S, 8 warps.
// Warp w: tokens 8w..8w+7 of the U / O products, key columns 16w..16w+15 of S.
// MODE 0: forward (O, hT).  MODE 1: backward recompute (store S0 and U).
// Chunk tiles arrive on a three-stage mbarrier ring: Q and K as TMA tensor
// tiles, the workspace products (W, P, U~ tile, G) as bulk copies.
// ---------------------------------------------------------------------------
constexpr int WALK_THREADS = 256;
constexpr int WALK_STAGES = 3;

// One CTA walks 16*MT value rows of one head's state (MT m-tiles per warp).
template <int MT>
struct alignas(1024) WalkStage {
    __nv_bfloat16 Q[C * DK];                 // Tma128
    __nv_bfloat16 K[C * DK];                 // Tma128
    __nv_bfloat16 W[C * DK];                 // Tma128
    __nv_bfloat16 P[C * C];                  // Swz<64>
    __nv_bfloat16 Ut[16 * MT * C];           // rows a0.. of the U~^T image (Swz<64>)
    float G[DK];                             // G (scalar gate) or e^{G_last,c} (channel gate)
};

template <int MT>
struct WalkSmem {
    WalkStage<MT> st[WALK_STAGES];
    __nv_bfloat16 S0[16 * MT * DK];   // Swz<128>: bf16 copy of the state entering the chunk
    __nv_bfloat16 Uu[16 * MT * C];    // Swz<64>: U^T (rows of S x tokens)
    __nv_bfloat16 Us[16 * MT * C];    // Swz<64>: U^T scaled by e^{G_last - G_i}
    __nv_bfloat16 O[C * 16 * MT];     // [token][row] staging (O, or U in MODE 1)
    uint64_t full[WALK_STAGES];
};

struct WalkPtrs {
    CUtensorMap qmap, kmap;
    const float* h0;
    const __nv_bfloat16 *W, *Ut, *P;
    const float* G;
    const __nv_bfloat16 *Qg, *Kt;  // channel gate: prepared Q and K images
    __nv_bfloat16* o;
    float* hT;
    __nv_bfloat16 *S0out, *Uout;
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    SeqMap seq;
};

// KDA: the chunk's Q and K arrive pre-scaled (scale Q .* e^G, K .* e^{G_last-G})
// as workspace images, with the per-key chunk decay e^{G_last,c}.
// MODE 1 (state recompute) has no output, so it fetches neither Q nor P.
template <int MT, int MODE, bool KDA>
__device__ void walk_issue(WalkStage<MT>& st, uint64_t* bar, const WalkPtrs& p, const Chain& ch,
                           int h, int k, int tile0) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + k;  // step k of the chain
    constexpr int GW = KDA ? DK : C;
    constexpr int QP = MODE == 0 ? C * DK + C * C : 0;
    mbar_arrive_expect(bar, (2 * C * DK + QP + MT * C * 16) * 2 + GW * 4);
    const int tok = ch.tok0 + k * C;
    if (KDA) {
        if (MODE == 0) bulk_g2s(st.Q, p.Qg + cid * C * DK, C * DK * 2, bar);
        bulk_g2s(st.K, p.Kt + cid * C * DK, C * DK * 2, bar);
    } else {
        if (MODE == 0) tma_load_tile(st.Q, &p.qmap, h, tok, bar);
        tma_load_tile(st.K, &p.kmap, h, tok, bar);
    }
    bulk_g2s(st.W, p.W + cid * C * DK, C * DK * 2, bar);
    if (MODE == 0) bulk_g2s(st.P, p.P + cid * C * C, C * C * 2, bar);
    bulk_g2s(st.Ut, p.Ut + cid * C * DV + tile0 * 16 * C, MT * C * 16 * 2, bar);
    bulk_g2s(st.G, p.G + cid * GW, GW * 4, bar);
}

template <int MT, int MODE, bool KDA>
__global__ void __launch_bounds__(WALK_THREADS) tc_walk_kernel(const __grid_constant__ WalkPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    WalkSmem<MT>& s = *reinterpret_cast<WalkSmem<MT>*>(align1k(smem_raw));
    constexpr int RT = 16 * MT;           // value rows of this CTA
    constexpr int TILES = DV / RT;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int bh = blockIdx.x / TILES, tile0 = (blockIdx.x % TILES) * MT, a0 = tile0 * 16;
    const int h = bh % p.H;
    const Chain ch = chain_of(p.seq, p.T, p.H, p.NT, bh / p.H, h);
    const int nsteps = ch.n1 - ch.n0;
    const int r_lo = lane >> 2;
    const int i0 = 8 * w + 2 * (lane & 3);  // this thread's token pair in the U/O tiles

    if (tid == 0) {
        for (int i = 0; i < WALK_STAGES; ++i) mbar_init(&s.full[i], 1);
        fence_mbar_init();
    }
    // fp32 state: m-tile mt, rows 16mt + r_lo (+8); columns 16w + 8j + 2(lane%4) + {0,1}
    float S[MT][2][4];
    {
        const float* h0 = p.h0 ? p.h0 + ((size_t)bh * DV + a0) * DK : nullptr;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = 16 * w + 8 * j + 2 * (lane & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    S[mt][j][e] = h0 ? h0[(size_t)(16 * mt + r_lo + 8 * (e >> 1)) * DK + c + (e & 1)] : 0.f;
            }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int j = 0; j < 2; ++j) st_c<S128>(s.S0, 16 * mt, 16 * w + 8 * j, S[mt][j]);
    if (MODE == 1) fence_async_smem();
    __syncthreads();
    if (tid == 0)
        for (int k = 0; k < WALK_STAGES - 1 && k < nsteps; ++k)
            walk_issue<MT, MODE, KDA>(s.st[k], &s.full[k], p, ch, h, k, tile0);

    for (int k = 0; k < nsteps; ++k) {  // step k: chunk ch.n0 + k
        const int sn = k % WALK_STAGES;
        WalkStage<MT>& st = s.st[sn];
        if (__syncthreads_or(!mbar_wait(&s.full[sn], (k / WALK_STAGES) & 1, p.status))) return;  // all threads agree; stage k landed; S0 written; stage of step k-1 is free
        if (tid == 0 && k + WALK_STAGES - 1 < nsteps) {
            const int kk = k + WALK_STAGES - 1;
            walk_issue<MT, MODE, KDA>(s.st[kk % WALK_STAGES], &s.full[kk % WALK_STAGES], p, ch, h, kk,
                                tile0);
        }
        const int tok = ch.tok0 + k * C;
        const int L = min(C, ch.end - tok);
        const size_t cid = (size_t)ch.img * p.NT + ch.n0 + k;
        if (MODE == 1) {  // chunk-start state rows a0.. into the Kp<128> image
            // (a0 is a multiple of 16, so a 16-byte piece keeps its swizzled
            // position: the first half of a Swz<128> row is panel 0, the second panel 1)
            for (int e = tid; e < RT * 16; e += WALK_THREADS) {
                const int r = e >> 4, pos = e & 15;
                *reinterpret_cast<uint4*>(p.S0out + cid * DV * DK + (pos >> 3) * (DV * 64) +
                                          (a0 + r) * 64 + (pos & 7) * 8) =
                    *reinterpret_cast<const uint4*>(s.S0 + r * DK + pos * 8);
            }
        }
        const float Gl = KDA ? 0.f : st.G[C - 1];
        const float et0 = KDA ? 1.f : __expf(Gl - st.G[i0]);
        const float et1 = KDA ? 1.f : __expf(Gl - st.G[i0 + 1]);

        // X = S0 W^T, Y = S0 Q^T for tokens 8w..8w+7 (two accumulators each)
        float X[MT][2][4] = {}, Y[MT][2][4] = {};
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t bw[2], bq[2];
            ldb_nk1<Tma128>(bw, st.W, 8 * w, 16 * kk);
            if (MODE == 0) ldb_nk1<Tma128>(bq, st.Q, 8 * w, 16 * kk);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                lda<S128>(a, s.S0, 16 * mt, 16 * kk);
                mma16816(X[mt][kk & 1], a, bw[0], bw[1]);
                if (MODE == 0) mma16816(Y[mt][kk & 1], a, bq[0], bq[1]);
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float u[4], us[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = r_lo + 8 * (e >> 1), i = i0 + (e & 1);
                u[e] = __bfloat162float(st.Ut[swz<C>(16 * mt + r, i)]) - (X[mt][0][e] + X[mt][1][e]);
                us[e] = u[e] * ((e & 1) ? et1 : et0);
            }
            st_c<S64>(s.Uu, 16 * mt, 8 * w, u);
            st_c<S64>(s.Us, 16 * mt, 8 * w, us);
            if (MODE == 1) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s.O[(i0 + (e & 1)) * RT + 16 * mt + r_lo + 8 * (e >> 1)] = __float2bfloat16_rn(u[e]);
            }
        }
        __syncthreads();

        // S1 = e^{G_last} S0 + (U^T .* e^{G_last - G}) K, columns 16w..16w+15
        const float gam = KDA ? 1.f : __expf(Gl);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    S[mt][j][e] *= KDA ? st.G[16 * w + 8 * j + 2 * (lane & 3) + (e & 1)] : gam;
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk) {
            uint32_t bk[4];
            ldb_kn<Tma128>(bk, st.K, 16 * kk, 16 * w);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                lda<S64>(a, s.Us, 16 * mt, 16 * kk);
                mma16816(S[mt][0], a, bk[0], bk[1]);
                mma16816(S[mt][1], a, bk[2], bk[3]);
            }
        }
        if (MODE == 0) {
            // O^T (rows x tokens 8w..) = scale e^{G_i} Y + U^T P^T
            const float eg0 = KDA ? 1.f : p.scale * __expf(st.G[i0]);
            const float eg1 = KDA ? 1.f : p.scale * __expf(st.G[i0 + 1]);
            float o[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o[mt][e] = (Y[mt][0][e] + Y[mt][1][e]) * ((e & 1) ? eg1 : eg0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                if (16 * kk > 8 * w + 7) break;  // P[r][i] = 0 for i > r
                uint32_t bp[2];
                ldb_nk1<S64>(bp, st.P, 8 * w, 16 * kk);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t a[4];
                    lda<S64>(a, s.Uu, 16 * mt, 16 * kk);
                    mma16816(o[mt], a, bp[0], bp[1]);
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s.O[(i0 + (e & 1)) * RT + 16 * mt + r_lo + 8 * (e >> 1)] = __float2bfloat16_rn(o[mt][e]);
        }
        __syncthreads();  // done with S0, Uu, Us; O / U staged
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j) st_c<S128>(s.S0, 16 * mt, 16 * w + 8 * j, S[mt][j]);
        if (MODE == 1) fence_async_smem();
        constexpr int PIECES = RT / 8;  // 16-byte pieces per token row
        // O: rows of the sequence only.  U image: all C rows, so the rows past a
        // ragged end hold their exact value (zero) rather than stale workspace.
        const int rows_out = MODE == 0 ? L : C;
        for (int e = tid; e < PIECES * rows_out; e += WALK_THREADS) {
            const int i = e / PIECES, pc = e % PIECES;
            const uint4 v = *reinterpret_cast<const uint4*>(&s.O[i * RT + 8 * pc]);
            if (MODE == 0) {
                const size_t row = ((size_t)tok + i) * p.H + h;
                *reinterpret_cast<uint4*>(p.o + row * DV + a0 + 8 * pc) = v;
            } else {  // U image, Tma128: 16-byte piece at its swizzled position
                *reinterpret_cast<uint4*>(p.Uout + cid * C * DV + Tma128::off(i, a0 + 8 * pc)) = v;
            }
        }
    }
    if (MODE == 0 && p.hT) {
        float* hT = p.hT + ((size_t)bh * DV + a0) * DK;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = 16 * w + 8 * j + 2 * (lane & 3);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    hT[(size_t)(16 * mt + r_lo + 8 * (e >> 1)) * DK + c + (e & 1)] = S[mt][j][e];
            }
    }
}

bool make_chunk_ptrs(ChunkPtrs& p, const gdn_dims& d, const TcLayout& L, const void* q,
                     const void* k, const void* v, const float* g, const float* beta, void* ws) {
    p = ChunkPtrs{};
    if (!encode_token_map(&p.qmap, q, d.B, d.T, d.H) || !encode_token_map(&p.kmap, k, d.B, d.T, d.H) ||
        !encode_token_map(&p.vmap, v, d.B, d.T, d.H))
        return false;
    p.q = (const __nv_bfloat16*)q; p.k = (const __nv_bfloat16*)k; p.v = (const __nv_bfloat16*)v;
    p.g = g; p.beta = beta; p.B = d.B; p.T = d.T; p.H = d.H; p.NT = L.NT; p.scale = d.scale;
    char* base = (char*)ws;
    p.W = (__nv_bfloat16*)(base + L.W);
    p.Ut = (__nv_bfloat16*)(base + L.Ut);
    p.P = (__nv_bfloat16*)(base + L.P);
    p.G = (float*)(base + L.G);
    p.Kt = (__nv_bfloat16*)(base + L.Kt);
    if (d.gate == GDN_GATE_CHANNEL) p.Qg = (__nv_bfloat16*)(base + L.Qg);
    p.status = (unsigned int*)ws;
    return true;
}

template <int MT, int MODE, bool KDA>
void launch_walk_mt(const WalkPtrs& p, cudaStream_t st) {
    const int smem = sizeof(WalkSmem<MT>) + 1024;
    cudaFuncSetAttribute(tc_walk_kernel<MT, MODE, KDA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         smem);
    const int grid = p.B * p.H * (DV / (16 * MT));
    GDN_LAUNCH(MODE == 0 ? "tc_walk_fwd" : "tc_walk_states", st,
               (tc_walk_kernel<MT, MODE, KDA><<<grid, WALK_THREADS, smem, st>>>(p)));
}

// Two m-tiles per warp halve the CTA count; use them only while the grid still
// covers every SM at least once.
template <int MODE, bool KDA>
void launch_walk(const WalkPtrs& p, cudaStream_t st) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if ((long long)p.B * p.H * (DV / 32) >= sms) launch_walk_mt<2, MODE, KDA>(p, st);
    else launch_walk_mt<1, MODE, KDA>(p, st);
}

WalkPtrs make_walk_ptrs(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0) {
    WalkPtrs w{};
    w.qmap = c.qmap; w.kmap = c.kmap;
    w.h0 = h0; w.W = c.W; w.Ut = c.Ut; w.P = c.P; w.G = c.G; w.Qg = c.Qg; w.Kt = c.Kt;
    w.status = c.status;
    w.B = chain_batches(d.B, c.seq); w.T = d.T; w.H = d.H; w.NT = L.NT; w.scale = d.scale;
    w.seq = c.seq;
    return w;
}

}  // namespace

namespace tc {
// The tcgen05 walks carry a whole head per CTA; with few heads the 16-row
// walks, which spread each head over eight CTAs, fill more SMs.
bool whole_head_walk(const gdn_dims& d, const SeqMap& seq) {
    return (long long)chain_batches(d.B, seq) * d.H * 4 >= sm_count();
}

// The forward chain (and the backward's state recompute) also takes the
// tcgen05 walk when its chains are cut into runs.
bool whole_head_fwd(const gdn_dims& d, const TcLayout& L, const SeqMap& seq) {
    return whole_head_walk(d, seq) || L.nseg > 1;
}

void launch_prep(const ChunkPtrs& p, size_t nchunks, cudaStream_t st) { launch_prep5(p, nchunks, st); }

bool chunk_ptrs(ChunkPtrs& p, const gdn_dims& d, const TcLayout& L, const void* q,
                const void* k, const void* v, const float* g, const float* beta, void* ws) {
    return make_chunk_ptrs(p, d, L, q, k, v, g, beta, ws);
}

void launch_walk_states(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp,
                        const float* h0, void* ws, cudaStream_t st) {
    if (whole_head_fwd(d, L, cp.seq)) {
        launch_walk5_states(d, L, cp, h0, ws, st);
        return;
    }
    WalkPtrs w = make_walk_ptrs(d, L, cp, h0);
    w.S0out = (__nv_bfloat16*)((char*)ws + L.S0);
    w.Uout = (__nv_bfloat16*)((char*)ws + L.U);
    if (d.gate == GDN_GATE_CHANNEL) launch_walk<1, true>(w, st);
    else launch_walk<1, false>(w, st);
}
}  // namespace tc

bool tc_supported(const gdn_dims& d) {
    return d.dtype == GDN_BF16 && d.dk == DK && d.dv == DV && d.chunk == C;
}

size_t tc_fwd_workspace(const gdn_dims& d, int nseq) { return tc_layout(d, false, nseq).end; }
size_t tc_bwd_workspace(const gdn_dims& d, int nseq) { return tc_layout(d, true, nseq).end; }

namespace {
// One CTA: per-sequence chunk counts over each thread's run of sequences, a
// block scan of the run totals, then the offsets.
constexpr int kSetupThreads = 256;
__global__ void __launch_bounds__(kSetupThreads) varlen_setup_kernel(const int* cu, int nseq, int T,
                                                                     int* cstart, unsigned int* status) {
    __shared__ int part[kSetupThreads];
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) bad = (cu[0] != 0 || cu[nseq] != T) ? 1 : 0;
    __syncthreads();
    const int per = (nseq + kSetupThreads - 1) / kSetupThreads;
    const int s0 = min(nseq, tid * per), s1 = min(nseq, s0 + per);
    int sum = 0;
    for (int s = s0; s < s1; ++s) {
        const int len = cu[s + 1] - cu[s];
        if (len < 0) bad = 1;
        sum += (max(len, 0) + C - 1) / C;
    }
    part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < kSetupThreads; o <<= 1) {  // inclusive scan
        const int x = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += x;
        __syncthreads();
    }
    const bool ok = bad == 0;
    int run = ok ? part[tid] - sum : 0;
    for (int s = s0; s < s1; ++s) {
        cstart[s] = run;
        if (ok) run += (cu[s + 1] - cu[s] + C - 1) / C;
    }
    if (tid == kSetupThreads - 1) cstart[nseq] = ok ? part[tid] : 0;
    if (tid == 0 && !ok && status) atomicOr(status, 2u);
}
}  // namespace

void launch_varlen_setup(const int* cu, int nseq, int T, int* cstart, unsigned int* status,
                         cudaStream_t st) {
    GDN_LAUNCH("varlen_setup", st,
               varlen_setup_kernel<<<1, kSetupThreads, 0, st>>>(cu, nseq, T, cstart, status));
}

bool tc_fwd_whole_head(const gdn_dims& d) {
    return tc::whole_head_fwd(d, tc_layout(d, false), SeqMap{});
}

bool launch_tc_fwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                   const float* g, const float* beta, const float* h0, void* o, float* hT,
                   void* ws, cudaStream_t st, const int* cu, int nseq,
                   unsigned long long wait_ns, int stall_at) {
    const TcLayout L = tc_layout(d, false, nseq);
    ChunkPtrs cp;
    if (!make_chunk_ptrs(cp, d, L, q, k, v, g, beta, ws)) return false;
    cp.wait_ns = wait_ns;
    cp.stall_at = stall_at;
    if (nseq) {  // chains then run one per (packed sequence, head)
        int* cstart = (int*)((char*)ws + L.cstart);
        launch_varlen_setup(cu, nseq, d.T, cstart, cp.status, st);
        cp.seq = SeqMap{cu, cstart, nseq};
    }
    const bool kda = d.gate == GDN_GATE_CHANNEL;
    if (kda) launch_prep5_kda(cp, L.nchunks, st);
    else launch_prep(cp, L.nchunks, st);
    if (tc::whole_head_fwd(d, L, cp.seq)) {
        launch_walk5_fwd(d, L, cp, h0, o, hT, ws, st);
    } else {
        WalkPtrs w = make_walk_ptrs(d, L, cp, h0);
        w.o = (__nv_bfloat16*)o;
        w.hT = hT;
        if (kda) launch_walk<0, true>(w, st);
        else launch_walk<0, false>(w, st);
    }
    return true;
}

// The forward of a training step: as launch_tc_fwd, in a backward-layout
// workspace, keeping what the backward would recompute (T, the chunk-start
// states and U) next to the prepared images.
bool launch_tc_fwd_save(const gdn_dims& d, const void* q, const void* k, const void* v,
                        const float* g, const float* beta, const float* h0, void* o, float* hT,
                        void* ws, cudaStream_t st) {
    const TcLayout L = tc_layout(d, true);
    ChunkPtrs cp;
    if (!make_chunk_ptrs(cp, d, L, q, k, v, g, beta, ws)) return false;
    cp.Tb = (__nv_bfloat16*)((char*)ws + L.Tb);
    const bool kda = d.gate == GDN_GATE_CHANNEL;
    if (kda) launch_prep5_kda(cp, L.nchunks, st);
    else launch_prep(cp, L.nchunks, st);
    if (tc::whole_head_fwd(d, L, cp.seq)) {
        launch_walk5_fwd(d, L, cp, h0, o, hT, ws, st, true);
    } else {  // the 16-row walk: outputs, then the states pass the backward would run
        WalkPtrs w = make_walk_ptrs(d, L, cp, h0);
        w.o = (__nv_bfloat16*)o;
        w.hT = hT;
        if (kda) launch_walk<0, true>(w, st);
        else launch_walk<0, false>(w, st);
        launch_walk_states(d, L, cp, h0, ws, st);
    }
    return true;
}

// The training-step forward with the q/k/v prologue fused into the
// preparation's load stage: the preparation reads the raw projections,
// filters its tiles in shared memory and writes the filtered q, k, v to the
// workspace, where the walk (and later the backward) read them.
bool launch_tc_fwd_save_conv(const gdn_dims& d, int K, const void* xq, const void* xk, const void* xv,
                             const float* wq, const float* wk, const float* wv, const float* g,
                             const float* beta, const float* h0, void* o, float* hT, void* ws,
                             cudaStream_t st) {
    const TcLayout L = tc_layout(d, true);
    const ConvLayout CL = conv_layout(d, K, L.end);
    char* base = (char*)ws;
    __nv_bfloat16 *qf = (__nv_bfloat16*)(base + CL.qf), *kf = (__nv_bfloat16*)(base + CL.kf),
                  *vf = (__nv_bfloat16*)(base + CL.vf);
    ChunkPtrs cp;  // token maps over the raw projections
    if (!make_chunk_ptrs(cp, d, L, xq, xk, xv, g, beta, ws)) return false;
    cp.Tb = (__nv_bfloat16*)(base + L.Tb);
    cp.conv = ChunkPtrs::Conv{(const __nv_bfloat16*)xq, (const __nv_bfloat16*)xk, (const __nv_bfloat16*)xv,
                              wq, wk, wv, qf, kf, vf, K};
    launch_prep5_conv(cp, L.nchunks, st);
    ChunkPtrs cw;  // token maps over the filtered tensors
    if (!make_chunk_ptrs(cw, d, L, qf, kf, vf, g, beta, ws)) return false;
    cw.Tb = cp.Tb;
    if (tc::whole_head_fwd(d, L, cw.seq)) {
        launch_walk5_fwd(d, L, cw, h0, o, hT, ws, st, true);
    } else {
        WalkPtrs w = make_walk_ptrs(d, L, cw, h0);
        w.o = (__nv_bfloat16*)o;
        w.hT = hT;
        launch_walk<0, false>(w, st);
        launch_walk_states(d, L, cw, h0, ws, st);
    }
    return true;
}

// ---------------------------------------------------------------------------
// Allocation-free forward.  Some callers cannot call cudaMalloc at all: code
// running under a fixed memory budget that the allocator must not touch, a
// runtime that hands out no device memory of its own, or a host thread that
// must not allocate between steps.  gdn_chunk_fwd_noalloc runs the same
// tensor-core forward as gdn_chunk_fwd but takes its workspace from the
// file-scope device array below, so the caller passes only inputs and
// outputs.  Every GPU that loads this library holds the array until exit.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)64 << 20;  // 64 MiB per device
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per
// device; the host-side name of the array is not a device address).
void* noalloc_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace

}  // namespace gdn

extern "C" gdn_status gdn_chunk_fwd_noalloc(const gdn_dims* d, const void* q, const void* k,
                                            const void* v, const float* g, const float* beta,
                                            const float* h0, void* o, float* hT,
                                            gdn_stream_t stream) {
    const gdn_status s = gdn::validate_fwd_args(d, q, k, v, g, beta, h0, o, hT);
    if (s != GDN_OK) return s;
    if (!gdn::tc_supported(*d) || d->gate != GDN_GATE_SCALAR) return GDN_ERR_UNSUPPORTED;
    if (gdn::tc_fwd_workspace(*d) > gdn::kNoAllocScratchBytes) return GDN_ERR_WORKSPACE;
    void* ws = gdn::noalloc_scratch();
    if (!ws) return GDN_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    // the status word must start at zero; every other byte the kernels read
    // is written earlier in the same call
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned int), st) != cudaSuccess) return GDN_ERR_CUDA;
    if (!gdn::launch_tc_fwd(*d, q, k, v, g, beta, h0, o, hT, ws, st)) return GDN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

extern "C" gdn_status gdn_noalloc_device_status(gdn_stream_t stream) {
    void* ws = gdn::noalloc_scratch();
    if (!ws) return GDN_ERR_CUDA;
    return gdn_query_device_status(ws, stream);
}
