// tc5_walk_bwd.cu -- the backward's reverse chunk chain on the fifth-generation
// tensor cores.
//
// Reverse mode through the chunk chain of the forward (tc5_walk.cu): with dS
// the gradient of the state leaving chunk n and dO the output gradient of
// its tokens,
//   dU^T = dO^T P + dS K~^T,  K~ = diag(e^{G_last - G}) K  (value rows x tokens)
//   dS0  = e^{G_last} dS + dO^T (scale e^G .* Q) - dU^T W  (the state entering n)
// One CTA walks one head's 128 value rows of dS backwards through the chunks:
//   F = dO^T P  (128 x 64)     E = dS K~^T  (128 x 64)        [A: dO tile, dS]
//   T = dO^T Q^ - dU^T W (128 x 128, one accumulator; the second product
//       enters with its A operand negated)                    [A: dO tile, dU]
// dS stays fp32 in the epilogue threads' registers; its bf16 copy and dU are
// written straight into tensor memory as A operands.  The dO tile is read
// as an MN-major A operand from shared memory; Q is scaled in place to
// Q^ = scale e^{G_i} Q (rows past the sequence end zeroed) before T.
// Each chunk's dS (bf16, Kp<128>) and dU (Tma128, token rows) are stored
// for the local-gradient kernel; dh0 is the dS left after chunk 0.  From the
// second step on, the epilogue writes these two images into the stage of the
// step before (dead once that step's T product and epilogue are done: dS over
// its Q and K~ tiles, dU over its W tile) and the load thread sends them out
// with bulk stores before it refills the stage.  The threads themselves then
// issue no global stores on the chain: per-thread 16-byte stores of dS rows
// fill each 32-byte sector in two halves and stalled the epilogue behind the
// store path.
//
// Warp roles as in tc5_walk.cu: 16 epilogue warps (TMEM lane quarter =
// warp % 4, column group = warp / 4), one MMA warp, one load warp with a
// three-stage ring.  Chain per step: E -> dU -> T -> dS update -> next E;
// F and the first half of T depend only on the chunk's tiles.
//
// K~ is the prepared image K .* e^{G_last - G} (per token for the scalar
// gate, per key channel for the channel gate).  Channel gate: Q arrives as
// the prepared image scale Q .* e^G, G holds e^{G_last,c}, no per-token
// factors apply, and the decay of dS is per key column.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace {
using namespace tc;

constexpr int RB_EPI_WARPS = 16;
constexpr int RB_THREADS = 32 * (RB_EPI_WARPS + 2);
constexpr int RB_CTRL = RB_EPI_WARPS;
constexpr int RB_PROD = RB_EPI_WARPS + 1;
constexpr int RB_STAGES = 3;
// tensor-memory columns: accumulators E, F, T; A operands dS (bf16 pairs), dU
constexpr int TE = 0, TF = 64, TT = 128, TADS = 256, TADU = 320, RCOLS = 512;
constexpr uint32_t ID_E = tc5::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_F = tc5::idesc_bf16(128, 64, true, true);
constexpr uint32_t ID_Y = tc5::idesc_bf16(128, 128, true, true);
constexpr uint32_t ID_Z = tc5::idesc_bf16(128, 128, false, true) | (1u << 13);  // A negated

struct alignas(1024) RbStage {
    __nv_bfloat16 Q[C * DK];   // Tma128 [token][key]; scaled in place (B of T, MN-major)
    __nv_bfloat16 K[C * DK];   // Tma128 image of K .* e^{G_last - G}: K-major B of E
    __nv_bfloat16 W[C * DK];   // Tma128 [token][key]: MN-major B of T
    __nv_bfloat16 dO[C * DV];  // Tma128 [token][value]: MN-major A of F and T
    __nv_bfloat16 P[C * C];    // Swz<64> [j][i]: MN-major B of F
    float G[DK];               // G (scalar gate, C used) or e^{G_last,c}
};

struct RbSmem {
    RbStage st[RB_STAGES];
    uint64_t full[RB_STAGES], empty[RB_STAGES];
    // q_ready[k & 1]: Q^ of step k in place (two barriers: the epilogue may
    // signal step k+1 before the MMA thread has waited for step k).
    // staged[k & 1]: the dS and dU images of step k >= 1 are in stage k-1.
    uint64_t ds_ready, q_ready[2], du_ready, e_done, t_done, fin, staged[2];
    uint32_t tmem;
};

struct RbPtrs {
    CUtensorMap qmap, kmap, dOmap;
    const float* dhT;
    const __nv_bfloat16 *W, *P, *Qg, *Kt;
    const float* G;
    __nv_bfloat16 *dSout, *dUout;
    float* dh0;
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    SeqMap seq;
    // Runs (see tc5_walk.cu), counted from the end of the chain: run i holds
    // chunks of forward run nseg-1-i.  E[(bh*nseg + i)] is the fp32 gradient
    // entering run i (i >= 1); MODE 2 writes E[..+1] from run 0 (entered with
    // dhT) and the reverse maps dS -> dS R + Q' of runs 1 .. nseg-2 (R: from I
    // without the dO terms; Q': from 0 with them).
    int nseg, seglen;
    float *E, *Mmap, *Nmap;
};

template <bool KDA>
__device__ void rb_issue(RbStage& st, uint64_t* bar, const RbPtrs& p, const Chain& ch, int h, int j,
                         bool use_do) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + j;  // chunk j of the chain
    constexpr int GW = KDA ? DK : C;
    mbar_arrive_expect(bar, ((use_do ? 4 : 2) * C * DK + (use_do ? C * C : 0)) * 2 + GW * 4);
    const int tok = ch.tok0 + j * C;
    if (use_do) {  // the dO terms: Q (scaled in place), dO, P
        if (KDA) bulk_g2s(st.Q, p.Qg + cid * C * DK, C * DK * 2, bar);
        else tma_load_tile(st.Q, &p.qmap, h, tok, bar);
        tma_load_tile(st.dO, &p.dOmap, h, tok, bar);
        bulk_g2s(st.P, p.P + cid * C * C, C * C * 2, bar);
    }
    bulk_g2s(st.K, p.Kt + cid * C * DK, C * DK * 2, bar);
    bulk_g2s(st.W, p.W + cid * C * DK, C * DK * 2, bar);
    bulk_g2s(st.G, p.G + cid * GW, GW * 4, bar);
}

// The same tiles of chunk j, pulled into L2 a step before the ring reaches them.
template <bool KDA>
__device__ void rb_prefetch(const RbPtrs& p, const Chain& ch, int h, int j, bool use_do) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + j;
    constexpr int GW = KDA ? DK : C;
    const int tok = ch.tok0 + j * C;
    if (use_do) {
        if (KDA) bulk_prefetch_l2(p.Qg + cid * C * DK, C * DK * 2);
        else tma_prefetch_tile(&p.qmap, h, tok);
        tma_prefetch_tile(&p.dOmap, h, tok);
        bulk_prefetch_l2(p.P + cid * C * C, C * C * 2);
    }
    bulk_prefetch_l2(p.Kt + cid * C * DK, C * DK * 2);
    bulk_prefetch_l2(p.W + cid * C * DK, C * DK * 2);
    bulk_prefetch_l2(p.G + cid * GW, GW * 4);
}

GDN_DEV bool rb_wait_all(uint64_t* bar, uint32_t parity, unsigned int* status) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, status));
}

GDN_DEV void rb_warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

enum { kRbStartDhT, kRbStartE, kRbStartI, kRbStartZero };

// MODE 0: the reverse walk proper (dS, dU images per chunk; dh0).  MODE 2:
// a run's reverse map (final gradient only).
template <bool KDA, int MODE>
__global__ void __launch_bounds__(RB_THREADS) tc5_walk_bwd_kernel(const __grid_constant__ RbPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    RbSmem& s = *reinterpret_cast<RbSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // ---- which run of which chain, from where, to where ----------------------
    int bh, run, start;
    bool use_do;
    float* out;
    if (MODE == 2) {
        const int per = 2 * p.nseg - 3, job = blockIdx.x % per;
        bh = blockIdx.x / per;
        run = job == 0 ? 0 : 1 + (job - 1) / 2;
        const size_t slot = ((size_t)bh * p.nseg + run) * DV * DK;
        if (job == 0) { start = kRbStartDhT; use_do = true; out = p.E + slot + (size_t)DV * DK; }
        else if ((job - 1) % 2 == 0) { start = kRbStartI; use_do = false; out = p.Mmap + slot; }
        else { start = kRbStartZero; use_do = true; out = p.Nmap + slot; }
    } else {
        bh = blockIdx.x / p.nseg;
        run = blockIdx.x % p.nseg;
        start = run == 0 ? kRbStartDhT : kRbStartE;
        use_do = true;
        // the run holding chunk 0 of the chain ends in dh0
        out = (run == p.nseg - 1 && p.dh0) ? p.dh0 + (size_t)bh * DV * DK : nullptr;
    }
    const int h = bh % p.H;  // bh: state row (sequence * H + head)
    const Chain ch = chain_of(p.seq, p.T, p.H, p.NT, bh / p.H, h);
    const int nch = ch.n1 - ch.n0;
    // forward run nseg-1-run covers chain chunks [c_lo, c_hi); walked downwards
    const int fr = p.nseg - 1 - run;
    const int c_lo = min(fr * p.seglen, nch), c_hi = min((fr + 1) * p.seglen, nch);
    const int nsteps = c_hi - c_lo;

    if (tid == 0) {
        for (int i = 0; i < RB_STAGES; ++i) {
            mbar_init(&s.full[i], 1);
            // MODE 0: the MMA commit; the epilogue's part is known from staged
            mbar_init(&s.empty[i], MODE == 0 ? 1 : 1 + RB_EPI_WARPS);
        }
        mbar_init(&s.ds_ready, RB_EPI_WARPS);
        mbar_init(&s.q_ready[0], RB_EPI_WARPS);
        mbar_init(&s.q_ready[1], RB_EPI_WARPS);
        mbar_init(&s.du_ready, RB_EPI_WARPS);
        mbar_init(&s.e_done, 1);
        mbar_init(&s.t_done, 1);
        mbar_init(&s.fin, 1);
        mbar_init(&s.staged[0], RB_EPI_WARPS);
        mbar_init(&s.staged[1], RB_EPI_WARPS);
        fence_mbar_init();
    }
    if (warp == RB_CTRL) tc5::alloc(&s.tmem, RCOLS);
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;

    if (warp == RB_PROD) {
        if (lane == 0) {
            // MODE 0: bulk stores of the dS and dU images of step m >= 1, staged
            // in stage m-1; the stage is free again once they have been read
            auto flush = [&](int m) -> bool {
                if (!mbar_wait(&s.staged[m & 1], ((m - 1) >> 1) & 1, p.status)) return false;
                const RbStage& sg = s.st[(m - 1) % RB_STAGES];
                const size_t cid = (size_t)ch.img * p.NT + ch.n0 + (c_hi - 1 - m);
                bulk_s2g(p.dSout + cid * DV * DK, sg.Q, DV * DK * 2);  // Q and K~ tiles: 32 KiB
                bulk_s2g(p.dUout + cid * C * DV, sg.W, C * DV * 2);
                bulk_commit();
                bulk_wait_read<0>();
                return true;
            };
            int issued = 0;
            bool ok = true;
            for (int k = 0; k < nsteps; ++k) {  // step k carries chunk c_hi-1-k of the chain
                const int sk = k % RB_STAGES;
                if (k >= RB_STAGES) {
                    if (MODE == 0 && !(ok = flush(k - 2))) break;
                    if (!(ok = mbar_wait(&s.empty[sk], ((k / RB_STAGES) - 1) & 1, p.status))) break;
                }
                rb_issue<KDA>(s.st[sk], &s.full[sk], p, ch, h, c_hi - 1 - k, use_do);
                if (k + RB_STAGES < nsteps)  // the step after the ring (the backward: 260 -> 256 us)
                    rb_prefetch<KDA>(p, ch, h, c_hi - 1 - (k + RB_STAGES), use_do);
                issued = k + 1;
            }
            if (MODE == 0 && ok)
                for (int m = max(1, issued - 2); m < issued && flush(m); ++m) {}
            for (int k = max(0, issued - RB_STAGES); k < issued; ++k)
                mbar_wait(&s.full[k % RB_STAGES], (k / RB_STAGES) & 1, p.status);
            bulk_wait<0>();
        }
        __syncwarp();
    } else if (warp == RB_CTRL) {
        if (lane == 0) {
            for (int k = 0; k < nsteps; ++k) {
                const int sk = k % RB_STAGES;
                RbStage& st = s.st[sk];
                if (!mbar_wait(&s.full[sk], (k / RB_STAGES) & 1, p.status)) break;
                const uint32_t sQ = smem_u32(st.Q), sK = smem_u32(st.K), sW = smem_u32(st.W),
                               sdO = smem_u32(st.dO), sP = smem_u32(st.P);
                if (use_do) {
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)  // F = dO^T P
                        tc5::mma(tm + TF, tc5::mnmajor(sdO, kk, C * 128), tc5::mnmajor(sP, kk, C * 128), ID_F,
                                 kk > 0);
                }
                if (!mbar_wait(&s.ds_ready, k & 1, p.status)) break;
                tc5::fence_after();
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)  // E = dS K~^T
                    tc5::mma_ts(tm + TE, tm + TADS + 8 * kk, tc5::kmajor<C>(sK, kk), ID_E, kk > 0);
                tc5::commit(&s.e_done);
                if (use_do) {
                    if (!mbar_wait(&s.q_ready[k & 1], (k >> 1) & 1, p.status)) break;
                    tc5::fence_after();
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)  // T = dO^T Q^
                        tc5::mma(tm + TT, tc5::mnmajor(sdO, kk, C * 128), tc5::mnmajor(sQ, kk, C * 128), ID_Y,
                                 kk > 0);
                }
                if (!mbar_wait(&s.du_ready, k & 1, p.status)) break;
                tc5::fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // T -= dU^T W
                    tc5::mma_ts(tm + TT, tm + TADU + 8 * kk, tc5::mnmajor(sW, kk, C * 128), ID_Z,
                                use_do || kk > 0);
                tc5::commit(&s.t_done);
                tc5::commit(&s.empty[sk]);
            }
            tc5::commit(&s.fin);
            mbar_wait(&s.fin, 0, p.status);
        }
        __syncwarp();
    } else {
        // ---- epilogue: thread = value row a; key columns 32*cg .. +31 of dS,
        // tokens 16*cg .. +15 of dU -------------------------------------------
        const int q = warp & 3, cg = warp >> 2, a = 32 * q + lane;
        const uint32_t trow = tm + ((uint32_t)(32 * q) << 16);
        const int t0 = 16 * cg;
        float dS[32];
        {
            const float* src = nullptr;
            if (start == kRbStartDhT && p.dhT) src = p.dhT + (size_t)bh * DV * DK;
            if (start == kRbStartE) src = p.E + ((size_t)bh * p.nseg + run) * DV * DK;
            if (src) src += (size_t)a * DK + 32 * cg;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                dS[j] = v.x; dS[j + 1] = v.y; dS[j + 2] = v.z; dS[j + 3] = v.w;
            }
            if (start == kRbStartI) {
#pragma unroll
                for (int j = 0; j < 32; ++j) dS[j] = (32 * cg + j == a) ? 1.f : 0.f;
            }
        }
        auto store_ds_tmem = [&]() {
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = pack_bf16(dS[2 * j], dS[2 * j + 1]);
            tc5::st16(trow + TADS + 16 * cg, r);
            tc5::wait_st();
        };
        store_ds_tmem();
        tc5::fence_before();
        rb_warp_arrive(&s.ds_ready);

        for (int k = 0; k < nsteps; ++k) {
            const int j = c_hi - 1 - k, sk = k % RB_STAGES;  // chunk j of the chain
            RbStage& st = s.st[sk];
            const int L = min(C, ch.end - (ch.tok0 + j * C));
            const size_t cid = (size_t)ch.img * p.NT + ch.n0 + j;
            if (!rb_wait_all(&s.full[sk], (k / RB_STAGES) & 1, p.status)) break;
            // Q^ = scale e^{G_i} Q in place, rows past the sequence end zeroed
            if (use_do && (!KDA || L < C)) {
#pragma unroll
                for (int rep = 0; rep < 2; ++rep) {
                    const int ci = tid + 32 * RB_EPI_WARPS * rep;  // 16-byte piece of the tile
                    const int i = (ci & 511) >> 3;
                    const float f = i < L ? (KDA ? 1.f : p.scale * __expf(st.G[i])) : 0.f;
                    uint4* ptr = reinterpret_cast<uint4*>(st.Q) + ci;
                    uint4 v = *ptr;
                    __nv_bfloat162* e2 = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const float2 x = __bfloat1622float2(e2[jj]);
                        e2[jj] = __floats2bfloat162_rn(x.x * f, x.y * f);
                    }
                    *ptr = v;
                }
            }
            tc5::fence_proxy_async();
            rb_warp_arrive(&s.q_ready[k & 1]);
            // the dS image of chunk j (the gradient leaving it), bf16 Kp<128>:
            // into stage k-1 for the load thread's bulk store, or to global
            // memory at the first step
            if (MODE == 0) {
                __nv_bfloat16* dst = k > 0 ? s.st[(k + RB_STAGES - 1) % RB_STAGES].Q : p.dSout + cid * DV * DK;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    *reinterpret_cast<uint4*>(dst + Kp<DV>::off(a, 32 * cg + 8 * jj)) =
                        make_uint4(pack_bf16(dS[8 * jj], dS[8 * jj + 1]), pack_bf16(dS[8 * jj + 2], dS[8 * jj + 3]),
                                   pack_bf16(dS[8 * jj + 4], dS[8 * jj + 5]), pack_bf16(dS[8 * jj + 6], dS[8 * jj + 7]));
            }
            // ---- dU = F + E, zero past the sequence end (E = dS K~^T carries
            // the factors e^{G_last - G_i}) ---------------------------------------
            const float gam = KDA ? 1.f : __expf(st.G[C - 1]);
            if (!rb_wait_all(&s.e_done, k & 1, p.status)) break;
            tc5::fence_after();
            {
                float e[16], f[16];
                tc5::ld16(e, trow + TE + t0);
                if (use_do) tc5::ld16(f, trow + TF + t0);
                tc5::wait_ld();
                uint32_t ru[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const float u0 = t0 + 2 * jj < L ? e[2 * jj] + (use_do ? f[2 * jj] : 0.f) : 0.f;
                    const float u1 = t0 + 2 * jj + 1 < L ? e[2 * jj + 1] + (use_do ? f[2 * jj + 1] : 0.f) : 0.f;
                    ru[jj] = pack_bf16(u0, u1);
                }
                tc5::st8(trow + TADU + 8 * cg, ru);
                tc5::wait_st();
                tc5::fence_before();
                rb_warp_arrive(&s.du_ready);
                if (MODE == 0) {  // dU image, Tma128 token rows: over stage k-1's W, or global
                    __nv_bfloat16* dst = k > 0 ? s.st[(k + RB_STAGES - 1) % RB_STAGES].W : p.dUout + cid * C * DV;
                    uint32_t w[8];
                    pair_columns(ru, w);
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        *reinterpret_cast<uint32_t*>(dst + Tma128::off(t0 + 2 * jj + (lane & 1), a & ~1)) = w[jj];
                    if (k > 0) {
                        tc5::fence_proxy_async();
                        rb_warp_arrive(&s.staged[k & 1]);
                    }
                }
            }
            // ---- dS0 = gamma dS + T ---------------------------------------------
            if (!rb_wait_all(&s.t_done, k & 1, p.status)) break;
            tc5::fence_after();
            {
                float t[32];
                tc5::ld32(t, trow + TT + 32 * cg);
                tc5::wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const float gj = KDA ? st.G[32 * cg + jj] : gam;
                    dS[jj] = fmaf(gj, dS[jj], t[jj]);
                }
            }
            store_ds_tmem();
            tc5::fence_before();
            rb_warp_arrive(&s.ds_ready);
            if (MODE != 0) rb_warp_arrive(&s.empty[sk]);
        }
        if (out) {
            float* dst = out + (size_t)a * DK + 32 * cg;
#pragma unroll
            for (int jj = 0; jj < 32; jj += 4)
                *reinterpret_cast<float4*>(dst + jj) = make_float4(dS[jj], dS[jj + 1], dS[jj + 2], dS[jj + 3]);
        }
    }
    tc5::fence_before();
    __syncthreads();
    if (warp == RB_CTRL) {
        tc5::fence_after();
        tc5::dealloc(tm, RCOLS);
    }
}

template <bool KDA, int MODE>
void launch_rb(const RbPtrs& p, int grid, cudaStream_t st) {
    const int smem = sizeof(RbSmem) + 1024;
    cudaFuncSetAttribute(tc5_walk_bwd_kernel<KDA, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH(MODE == 0 ? "tc5_walk_bwd" : "tc5_seg_map_bwd", st,
               (tc5_walk_bwd_kernel<KDA, MODE><<<grid, RB_THREADS, smem, st>>>(p)));
}

}  // namespace

namespace tc {
void launch_seg_scan(float* E, const float* Mmap, const float* Nmap, int nseg, int chains,
                     unsigned int* status, cudaStream_t st);

bool launch_walk5_bwd(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const void* dO,
                      const float* dhT, float* dh0, void* ws, cudaStream_t st) {
    RbPtrs p{};
    p.qmap = c.qmap; p.kmap = c.kmap;
    if (!encode_token_map(&p.dOmap, dO, d.B, d.T, d.H)) return false;
    p.dhT = dhT; p.W = c.W; p.P = c.P; p.Qg = c.Qg; p.Kt = c.Kt; p.G = c.G;
    p.dSout = (__nv_bfloat16*)((char*)ws + L.dS);
    p.dUout = (__nv_bfloat16*)((char*)ws + L.dU);
    p.dh0 = dh0; p.status = c.status;
    p.B = chain_batches(d.B, c.seq); p.T = d.T; p.H = d.H; p.NT = L.NT; p.scale = d.scale;
    p.seq = c.seq;
    p.nseg = L.nseg; p.seglen = L.seglen;
    const bool kda = d.gate == GDN_GATE_CHANNEL;
    const int chains = p.B * p.H;
    if (p.nseg > 1) {
        p.E = (float*)((char*)ws + L.segE);
        p.Mmap = (float*)((char*)ws + L.segM);
        p.Nmap = (float*)((char*)ws + L.segN);
        if (kda) launch_rb<true, 2>(p, chains * (2 * p.nseg - 3), st);
        else launch_rb<false, 2>(p, chains * (2 * p.nseg - 3), st);
        if (p.nseg > 2) launch_seg_scan(p.E, p.Mmap, p.Nmap, p.nseg, chains, p.status, st);
    }
    if (kda) launch_rb<true, 0>(p, chains * p.nseg, st);
    else launch_rb<false, 0>(p, chains * p.nseg, st);
    return true;
}
}  // namespace tc
}  // namespace gdn
