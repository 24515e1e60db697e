// tc5_walk.cu -- the forward's chunk chain on the fifth-generation tensor cores.
//
// One CTA carries one head's whole 128x128 state through its chunks (the
// chain of "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper
// review), section "Method": U = U~ - W S0^T, O = scale diag(e^G) Q S0^T + P U,
// S1 = e^{G_last} S0 + U^T diag(e^{G_last - G}) K), with every product on
// tcgen05 MMAs whose accumulators sit in tensor memory:
//   [X | Y] = S0 [W ; Q]^T   (128 x 128: X = S0 W^T, Y = S0 Q^T; one N = 128 MMA
//                             per K step)
//   D = Us^T K  (128 x 128)   Z = U^T P^T (128 x 64)
// The A operands (the bf16 state and the U images) are written by the
// epilogue straight into tensor memory, so shared memory carries only the
// chunk tiles (B operands) and the MMAs read nothing from it twice.  The fp32
// state lives in the epilogue threads' registers (thread = state row, 32 key
// columns each); every step they add D to it and store its bf16 copy as the
// next step's A operand, so the state itself never leaves fp32.
//
// Warp roles: warps 0..15 are the epilogue (TMEM lane quarter = warp % 4,
// column group = warp / 4); warp 16 allocates TMEM and its lane 0 issues
// every MMA; lane 0 of warp 17 issues the chunk loads into a three-stage
// ring as stages are released.  Per step the chain is
//   [X|Y] -> U, Us -> D -> S update + state image -> next [X|Y],
// with Z and the output store off the chain.  The epilogue reads X and Y
// together, so each accumulator needs only one buffer.  U~^T, an
// epilogue-only operand, is read from global memory into registers one chunk
// ahead.
//
// MODE 1 (state recompute for the backward) has no output: it fetches
// neither Q nor P, runs X = S0 W^T alone in place of [X|Y], skips Z, and
// stores each chunk's entering state (bf16, Swz<128> image) and U (Swz<128>,
// token rows) for the backward kernels.
//
// Channel gate: Q and K arrive as prepared images (scale Q .* e^G and
// K .* e^{G_last - G}), G holds e^{G_last,c}, Us = U, and the decay of the
// state is per key column.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace {
using namespace tc;

constexpr int W5_EPI_WARPS = 16;
constexpr int W5_THREADS = 32 * (W5_EPI_WARPS + 2);
constexpr int W5_CTRL = W5_EPI_WARPS;      // MMA warp
constexpr int W5_PROD = W5_EPI_WARPS + 1;  // load warp
constexpr int W5_STAGES = 3;
// tensor-memory columns: accumulators [X|Y], D, Z; A operands S (bf16 pairs,
// 64 columns), U and Us (32 columns each)
constexpr int TXY = 0, TD = 128, TZ = 256, TAS = 320, TAU = 384, TAUS = 416, TCOLS = 512;
constexpr uint32_t ID_XY = tc5::idesc_bf16(128, 128, false, false);
constexpr uint32_t ID_X = tc5::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_D = tc5::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_Z = tc5::idesc_bf16(128, 64, false, false);

struct alignas(1024) W5Stage {
    // K-major B of [X|Y], 128 rows (64 W tokens, then 64 Q tokens) per
    // 64-key panel: [W p0 | Q p0 | W p1 | Q p1], 8 KB each
    __nv_bfloat16 WQ[2 * C * DK];
    __nv_bfloat16 K[C * DK];  // Tma128: MN-major B of D
    __nv_bfloat16 P[C * C];   // Swz<64>: K-major B of Z
    float G[DK];              // G (scalar gate, C used) or e^{G_last,c}
};

struct W5Smem {
    W5Stage st[W5_STAGES];
    uint64_t full[W5_STAGES], empty[W5_STAGES];
    uint64_t s_ready, u_ready, x_done, d_done, o_done, fin;
    uint32_t tmem;
};

struct W5Ptrs {
    CUtensorMap qmap, kmap;
    const float* h0;
    const __nv_bfloat16 *W, *Ut, *P, *Qg, *Kt;
    const float* G;
    __nv_bfloat16* o;
    float* hT;
    __nv_bfloat16 *S0out, *Uout;  // MODE 1
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    SeqMap seq;
};

template <bool KDA, int MODE>
__device__ void w5_issue(W5Stage& st, uint64_t* bar, const W5Ptrs& p, const Chain& ch, int h, int n) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + n;  // step n of the chain
    constexpr int GW = KDA ? DK : C;
    constexpr int PANEL = C * 64;  // elements of one 64x64 panel
    mbar_arrive_expect(bar, (MODE == 0 ? 3 * C * DK + C * C : 2 * C * DK) * 2 + GW * 4);
    const __nv_bfloat16* W = p.W + cid * C * DK;
    bulk_g2s(st.WQ, W, PANEL * 2, bar);
    bulk_g2s(st.WQ + 2 * PANEL, W + PANEL, PANEL * 2, bar);
    const int tok = ch.tok0 + n * C;
    if (MODE == 0) {
        if (KDA) {
            const __nv_bfloat16* Qg = p.Qg + cid * C * DK;
            bulk_g2s(st.WQ + PANEL, Qg, PANEL * 2, bar);
            bulk_g2s(st.WQ + 3 * PANEL, Qg + PANEL, PANEL * 2, bar);
        } else {
            tma_load_3d(st.WQ + PANEL, &p.qmap, 0, h, tok, bar);
            tma_load_3d(st.WQ + 3 * PANEL, &p.qmap, 64, h, tok, bar);
        }
        bulk_g2s(st.P, p.P + cid * C * C, C * C * 2, bar);
    }
    if (KDA) bulk_g2s(st.K, p.Kt + cid * C * DK, C * DK * 2, bar);
    else tma_load_tile(st.K, &p.kmap, h, tok, bar);
    bulk_g2s(st.G, p.G + cid * GW, GW * 4, bar);
}

// Warp-uniform bounded wait: every lane agrees on the outcome.
GDN_DEV bool wait_all(uint64_t* bar, uint32_t parity, unsigned int* status) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, status));
}

// One arrival per warp, after all of its lanes' prior writes.
GDN_DEV void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}


template <bool KDA, int MODE>
__global__ void __launch_bounds__(W5_THREADS) tc5_walk_kernel(const __grid_constant__ W5Ptrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    W5Smem& s = *reinterpret_cast<W5Smem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x, h = bh % p.H;  // bh: state row (sequence * H + head)
    const Chain ch = chain_of(p.seq, p.T, p.H, p.NT, bh / p.H, h);
    const int nsteps = ch.n1 - ch.n0;

    if (tid == 0) {
        for (int i = 0; i < W5_STAGES; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + W5_EPI_WARPS);
        }
        mbar_init(&s.s_ready, W5_EPI_WARPS);
        mbar_init(&s.u_ready, W5_EPI_WARPS);
        mbar_init(&s.x_done, 1);
        mbar_init(&s.d_done, 1);
        mbar_init(&s.o_done, 1);
        mbar_init(&s.fin, 1);
        fence_mbar_init();
    }
    if (warp == W5_CTRL) tc5::alloc(&s.tmem, TCOLS);
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;

    if (warp == W5_PROD) {
        if (lane == 0) {
            int issued = 0;
            for (int n = 0; n < nsteps; ++n) {
                const int sn = n % W5_STAGES;
                if (n >= W5_STAGES && !mbar_wait(&s.empty[sn], ((n / W5_STAGES) - 1) & 1, p.status)) break;
                w5_issue<KDA, MODE>(s.st[sn], &s.full[sn], p, ch, h, n);
                issued = n + 1;
            }
            // Leave no load in flight (returns at once for stages already consumed).
            for (int n = max(0, issued - W5_STAGES); n < issued; ++n)
                mbar_wait(&s.full[n % W5_STAGES], (n / W5_STAGES) & 1, p.status);
        }
        __syncwarp();
    } else if (warp == W5_CTRL) {
        if (lane == 0) {
            const uint32_t aUs = tm + (KDA ? TAU : TAUS);
            for (int n = 0; n < nsteps; ++n) {
                const int sn = n % W5_STAGES;
                W5Stage& st = s.st[sn];
                if (!mbar_wait(&s.full[sn], (n / W5_STAGES) & 1, p.status)) break;
                if (!mbar_wait(&s.s_ready, n & 1, p.status)) break;
                tc5::fence_after();
                const uint32_t sWQ = smem_u32(st.WQ), sK = smem_u32(st.K), sP = smem_u32(st.P);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    tc5::mma_ts(tm + TXY, tm + TAS + 8 * kk, tc5::kmajor<2 * C>(sWQ, kk),
                                MODE == 0 ? ID_XY : ID_X, kk > 0);
                tc5::commit(&s.x_done);
                if (!mbar_wait(&s.u_ready, n & 1, p.status)) break;
                tc5::fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    tc5::mma_ts(tm + TD, aUs + 8 * kk, tc5::mnmajor(sK, kk, C * 128), ID_D, kk > 0);
                tc5::commit(&s.d_done);
                if (MODE == 0) {
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        tc5::mma_ts(tm + TZ, tm + TAU + 8 * kk, tc5::kmajor<C>(sP, kk), ID_Z, kk > 0);
                    tc5::commit(&s.o_done);
                }
                tc5::commit(&s.empty[sn]);
            }
            // Leave nothing in flight: every MMA retired.
            tc5::commit(&s.fin);
            mbar_wait(&s.fin, 0, p.status);
        }
        __syncwarp();
    } else {
        // ---- epilogue: thread = state row a; key columns 32*cg .. +31 of the
        // state, tokens 16*cg .. +15 of U and O ---------------------------------
        const int q = warp & 3, cg = warp >> 2, a = 32 * q + lane;
        const uint32_t trow = tm + ((uint32_t)(32 * q) << 16);
        const int t0 = 16 * cg;  // first token of this thread's U / O columns
        float S[32];
        {
            const float* h0 = p.h0 ? p.h0 + ((size_t)bh * DV + a) * DK + 32 * cg : nullptr;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v = h0 ? *reinterpret_cast<const float4*>(h0 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
            }
        }
        auto store_state = [&]() {  // bf16 pairs of this thread's 32 key columns
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = pack_bf16(S[2 * j], S[2 * j + 1]);
            tc5::st16(trow + TAS + 16 * cg, r);
            tc5::wait_st();
        };
        // MODE 1: bf16 state entering chunk n, Swz<128> image (64 contiguous bytes)
        auto store_s0 = [&](int n) {
            __nv_bfloat16* dst = p.S0out + ((size_t)ch.img * p.NT + ch.n0 + n) * DV * DK;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = 32 * cg + 8 * j;
                *reinterpret_cast<uint4*>(dst + swz<DK>(a, c)) =
                    make_uint4(pack_bf16(S[c - 32 * cg], S[c - 32 * cg + 1]), pack_bf16(S[c - 32 * cg + 2], S[c - 32 * cg + 3]),
                               pack_bf16(S[c - 32 * cg + 4], S[c - 32 * cg + 5]), pack_bf16(S[c - 32 * cg + 6], S[c - 32 * cg + 7]));
            }
        };
        store_state();
        if (MODE == 1 && nsteps > 0) store_s0(0);
        tc5::fence_before();
        warp_arrive(&s.s_ready);

        // U~^T of row a, tokens t0..t0+15: two 16-byte pieces of its Swz<64> row
        const uint32_t uo0 = swz<C>(a, t0), uo1 = swz<C>(a, t0 + 8);
        const __nv_bfloat16* Ut = p.Ut + ((size_t)ch.img * p.NT + ch.n0) * C * DV;
        uint4 ut0 = make_uint4(0, 0, 0, 0), ut1 = ut0;
        if (nsteps > 0) {
            ut0 = *reinterpret_cast<const uint4*>(Ut + uo0);
            ut1 = *reinterpret_cast<const uint4*>(Ut + uo1);
        }

        for (int n = 0; n < nsteps; ++n) {
            const int sn = n % W5_STAGES;
            const W5Stage& st = s.st[sn];
            const int L = min(C, ch.end - (ch.tok0 + n * C));
            if (!wait_all(&s.full[sn], (n / W5_STAGES) & 1, p.status)) break;
            // per-token factors, lane j (mod 16) <-> token t0 + j
            float dec = 1.f, sce = 1.f, gam = 1.f;
            if (!KDA) {
                const float gi = st.G[t0 + (lane & 15)], gl = st.G[C - 1];
                dec = __expf(gl - gi);
                sce = p.scale * __expf(gi);
                gam = __expf(gl);
            }
            // ---- U = U~ - X; Y kept for the output ------------------------------
            if (!wait_all(&s.x_done, n & 1, p.status)) break;
            tc5::fence_after();
            float y[16];
            {
                float x[16];
                tc5::ld16(x, trow + TXY + t0);
                if (MODE == 0) tc5::ld16(y, trow + TXY + C + t0);
                tc5::wait_ld();
                const __nv_bfloat16* ua = reinterpret_cast<const __nv_bfloat16*>(&ut0);
                const __nv_bfloat16* ub = reinterpret_cast<const __nv_bfloat16*>(&ut1);
                uint32_t ru[8], rs[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float u0 = __bfloat162float(j < 4 ? ua[2 * j] : ub[2 * j - 8]) - x[2 * j];
                    const float u1 = __bfloat162float(j < 4 ? ua[2 * j + 1] : ub[2 * j - 7]) - x[2 * j + 1];
                    ru[j] = pack_bf16(u0, u1);
                    if (!KDA)
                        rs[j] = pack_bf16(u0 * __shfl_sync(0xffffffffu, dec, 2 * j),
                                          u1 * __shfl_sync(0xffffffffu, dec, 2 * j + 1));
                }
                tc5::st8(trow + TAU + 8 * cg, ru);
                if (!KDA) tc5::st8(trow + TAUS + 8 * cg, rs);
                tc5::wait_st();
                tc5::fence_before();
                warp_arrive(&s.u_ready);
                if (MODE == 1) {  // U image, token rows (64 contiguous bytes per warp store)
                    __nv_bfloat16* dst = p.Uout + ((size_t)ch.img * p.NT + ch.n0 + n) * C * DV;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&ru[j]);
                        dst[swz<DV>(t0 + 2 * j, a)] = v.x;
                        dst[swz<DV>(t0 + 2 * j + 1, a)] = v.y;
                    }
                }
            }
            if (n + 1 < nsteps) {  // next chunk's U~^T, consumed one step later
                const __nv_bfloat16* Un = Ut + (size_t)(n + 1) * C * DV;
                ut0 = *reinterpret_cast<const uint4*>(Un + uo0);
                ut1 = *reinterpret_cast<const uint4*>(Un + uo1);
            }
            // ---- S1 = gamma S0 + D, and the bf16 state image -------------------
            if (!wait_all(&s.d_done, n & 1, p.status)) break;
            tc5::fence_after();
            {
                float d[32];
                tc5::ld32(d, trow + TD + 32 * cg);
                tc5::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float gj = KDA ? st.G[32 * cg + j] : gam;
                    S[j] = fmaf(gj, S[j], d[j]);
                }
            }
            store_state();
            tc5::fence_before();
            warp_arrive(&s.s_ready);
            if (MODE == 1) {
                warp_arrive(&s.empty[sn]);
                if (n + 1 < nsteps) store_s0(n + 1);
                continue;
            }
            // ---- O^T = scale e^{G_i} Y + Z, tokens t0 .. t0+15 of row a ---------
            if (!wait_all(&s.o_done, n & 1, p.status)) break;
            tc5::fence_after();
            {
                float z[16];
                tc5::ld16(z, trow + TZ + t0);
                tc5::wait_ld();
                __nv_bfloat16* o = p.o + (((size_t)ch.tok0 + n * C + t0) * p.H + h) * DV + a;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float f = KDA ? 1.f : __shfl_sync(0xffffffffu, sce, j);
                    if (t0 + j < L) o[(size_t)j * p.H * DV] = __float2bfloat16_rn(fmaf(f, y[j], z[j]));
                }
            }
            tc5::fence_before();
            warp_arrive(&s.empty[sn]);
        }
        if (MODE == 0 && p.hT) {
            float* hT = p.hT + ((size_t)bh * DV + a) * DK + 32 * cg;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(hT + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc5::fence_before();
    __syncthreads();
    if (warp == W5_CTRL) {
        tc5::fence_after();
        tc5::dealloc(tm, TCOLS);
    }
}

template <bool KDA, int MODE>
void launch_w5(const W5Ptrs& p, cudaStream_t st) {
    const int smem = sizeof(W5Smem) + 1024;
    cudaFuncSetAttribute(tc5_walk_kernel<KDA, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH(MODE == 0 ? "tc5_walk_fwd" : "tc5_walk_states", st,
               (tc5_walk_kernel<KDA, MODE><<<p.B * p.H, W5_THREADS, smem, st>>>(p)));
}

}  // namespace

namespace tc {
void launch_walk5_fwd(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0,
                      void* o, float* hT, cudaStream_t st) {
    W5Ptrs w{};
    w.qmap = c.qmap; w.kmap = c.kmap;
    w.h0 = h0; w.W = c.W; w.Ut = c.Ut; w.P = c.P; w.G = c.G; w.Qg = c.Qg; w.Kt = c.Kt;
    w.o = (__nv_bfloat16*)o; w.hT = hT; w.status = c.status;
    w.B = chain_batches(d.B, c.seq); w.T = d.T; w.H = d.H; w.NT = L.NT; w.scale = d.scale;
    w.seq = c.seq;
    if (d.gate == GDN_GATE_CHANNEL) launch_w5<true, 0>(w, st);
    else launch_w5<false, 0>(w, st);
}

void launch_walk5_states(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0,
                         void* ws, cudaStream_t st) {
    W5Ptrs w{};
    w.qmap = c.qmap; w.kmap = c.kmap;
    w.h0 = h0; w.W = c.W; w.Ut = c.Ut; w.P = c.P; w.G = c.G; w.Qg = c.Qg; w.Kt = c.Kt;
    w.S0out = (__nv_bfloat16*)((char*)ws + L.S0);
    w.Uout = (__nv_bfloat16*)((char*)ws + L.U);
    w.status = c.status;
    w.B = chain_batches(d.B, c.seq); w.T = d.T; w.H = d.H; w.NT = L.NT; w.scale = d.scale;
    w.seq = c.seq;
    if (d.gate == GDN_GATE_CHANNEL) launch_w5<true, 1>(w, st);
    else launch_w5<false, 1>(w, st);
}
}  // namespace tc
}  // namespace gdn
