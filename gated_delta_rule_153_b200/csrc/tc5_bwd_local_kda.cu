// tc5_bwd_local_kda.cu -- the chunkwise backward's local gradients for the
// channel-wise gate (Kimi Delta Attention) on the fifth-generation tensor
// cores (bf16, dk = dv = 128, chunk 64).
//
// Reverse mode through the chunk equations of "Gated Delta Networks:
// Improving Mamba2 with Delta Rule" (paper review), section "Method", with
// Diag(a_t) on the key index (the channel-gate reading; the variant is named
// in "Linear Attention Architectures: Mechanisms, Trade-offs, and Cross-Layer
// Routing").  With G the per-key within-chunk cumsum of the log-gate,
// D_ijc = e^{G_ic - G_jc}, eG = e^G, etl = e^{G_last - G}, Kg = K .* eG:
//   dW  = -dU S0,   dT = (dW Kg^T + dU V^T) diag(beta)
//   dA  = strict_lower(-T^T dT T^T),  dMM = diag(beta) dA
//   X1' = (dA .* D) K,  X2 = (dMM .* D)^T K,  X3 = (dP .* D)^T Q,  X4 = (dP .* D) K
//   (dP = strict_lower(dO U^T); its diagonal enters dq and dk directly)
//   dq  = scale (eG .* (dO S0) + X4 + diag(dP) K)
//   dk  = etl .* (U dS) + diag(beta) eG .* (T^T dW) + diag(beta) X1' + X2
//         + scale (X3 + diag(dP) Q)
//   dv  = diag(beta) T^T dU
//   dbeta_i = sum_c [eG (T^T dW) .* K + (T^T dU) .* V + K .* X1']_ic
// dG collects the same terms times k or q (the diagonal pairs cancel and are
// left out), plus at the last token etl .* (U dS) .* K and e^{G_last} <dS, S0>,
// and dg is its reverse within-chunk cumsum per key.
//
// The products whose rows are keys run transposed: TMEM lane = key c (or
// value v), columns = tokens, so every per-key factor of the gate is a
// per-thread scalar and dg's cumsum over tokens stays inside a thread:
//   (dU S0)^T, (dO S0)^T = S0^T [dU ; dO]^T      M = 128 keys, N = 128 tokens
//   (U dS)^T = dS^T U^T,  (T^T dW)^T = dW^T T,  (T^T dU)^T = dU^T T
// The token x token products run as in the scalar-gate kernel (lane = token):
//   [dU ; dO] U^T -> dO U^T,  [dU ; dO] V^T -> dU V^T,  [dW ; .] Kg^T,
//   [dT ; .] T^T -> X,  T^T X -> dA.
// The four decayed pair products split each 16-token block pair (I, J) about
// the blocks' first and last rows: e^{G_i - G_j} = EL_i F_IJ ER_j with
// EL_i = e^{G_i - G_f(I)}, F_IJ = e^{G_f(I) - G_l(J)}, ER_j = e^{G_l(J) - G_j};
// EL and ER are at most 1 and go into the bf16 operands (K .* EL, Q .* EL,
// K .* ER), F is a per-key scalar applied to each pair's accumulator:
//   X1'^T (block I) = EL .* sum_{J <= I} F_IJ (K .* ER)_J^T dA_IJ^T
//   X2^T  (block J) = ER .* sum_{I >= J} F_IJ (K .* EL)_I^T dMM_IJ
// one M = 128 (keys), N = 16, K = 16 product per block pair and term.  F_II is
// e^{span} >= 1; a key whose block span exceeds 80 takes that block's
// diagonal pair from an exact elementwise sum instead.
//
// One CTA of sixteen warps per chunk: warp w works on TMEM lane quarter w % 4
// and token block w / 4.  Thread 0 issues the loads and the MMAs.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace {
using namespace tc;

constexpr int KB_THREADS = 512;
constexpr int PAIR = 128 * 64;       // elements of one 128-row, 64-column panel
constexpr uint32_t PB = PAIR * 2;    // its bytes: the panel stride of pair regions
// tensor-memory columns
constexpr uint32_t T_QW = 0,   // lane = key: 0..63 (dU S0)^T = -dW^T, 64..127 (dO S0)^T
    T_KT = 128,                // lane = key: (U dS)^T
    T_DP = 192,                // lane = token (rows 64..127): dO U^T
    T_DUV = 256,               // lane = token (rows 0..63): dU V^T
    T_TW = 320,                // lane = token (rows 0..63): dW Kg^T
    T_WT = 384,                // lane = key: (T^T dW)^T
    T_UT = 128,                // lane = value: (T^T dU)^T
    T_X = 192,                 // lane = token: dT T^T
    T_TX = 0,                  // lane = token: T^T X
    T_PR = 128,                // pair products: 2 x 10 x 16 columns (one round)
    T_DK = 448,                // lane = key: the dk accumulator, 16 columns per token block
    KB_TCOLS = 512;
constexpr uint32_t ID_QW = tc5::idesc_bf16(128, 128, true, false);
constexpr uint32_t ID_MN64 = tc5::idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_KK64 = tc5::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_MM64 = tc5::idesc_bf16(128, 64, true, true);
constexpr uint32_t ID_PAIR = tc5::idesc_bf16(128, 16, true, false);

struct alignas(1024) KbSmem {
    __nv_bfloat16 R1[2 * PAIR];  // [dU | dO] panels; the dO rows later hold dW
    __nv_bfloat16 R2[2 * PAIR];  // [K | Q]
    __nv_bfloat16 R3[2 * PAIR];  // [U | V]; the U rows later hold Kg
    __nv_bfloat16 R4[DV * DK];   // S0 (Kp<128>); later K .* EL | Q .* EL (Tma128)
    __nv_bfloat16 R5[DV * DK];   // dS (Kp<128>); later K .* ER (Tma128) | dT, then dMM^T | X, then dA
    // Swz<64> T, then 8 KB that the MN-major T^T view reads as its unused rows
    __nv_bfloat16 T[2 * C * C];
    __nv_bfloat16 dP[C * C];     // strict_lower(dO U^T) (Swz<64>)
    __nv_bfloat16 dPt[C * C];    // its transpose
    float Gf[4][DK], Gl[4][DK];  // G at the first / last token of each block, per key
    float btot[4][DK];           // per-block sums of g
    float dgt[4][DK];            // per-block sums of dG
    float ssp[4][DK], glp[4][DK];  // <dS, S0> and etl <dKt, k> partials per key
    float dbp[2][4][C];          // dbeta partials: [term][lane quarter][token]
    float beta[C], dPd[C];
    uint64_t bar_ld, bar_mma;
    uint32_t tmem;
};

struct KbPtrs {
    CUtensorMap qmap, kmap, vmap, dOmap;
    const float *g, *beta;
    const __nv_bfloat16 *S0, *U, *dS, *dU, *Tb;
    __nv_bfloat16 *dq, *dk, *dv;
    float *dg, *dbeta;
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    int pf_stride;  // chunks a wave ahead to pull into L2; 0: no prefetch
    SeqMap seq;
};

// Butterfly reduction of 16 per-lane values over the warp's 32 lanes in 16
// shuffles: returns, in every lane, the total of value (lane >> 1) & 15.
GDN_DEV float reduce16(float (&v)[16], int lane) {
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1) {  // lane bit 2s selects the half kept
        const bool hi = lane & (2 * s);
#pragma unroll
        for (int k = 0; k < s; ++k) {
            const float send = hi ? v[k] : v[k + s];
            const float keep = hi ? v[k + s] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * s);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

GDN_DEV float bf(const __nv_bfloat16* t, uint32_t off) { return __bfloat162float(t[off]); }

__global__ void __launch_bounds__(KB_THREADS, 1) tc5_bwd_local_kda_kernel(const __grid_constant__ KbPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    KbSmem& s = *reinterpret_cast<KbSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, h = bh % p.H;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, n);
    if (!cl.valid) return;  // past the last chunk of a packed batch
    const int L = cl.L;
    const size_t row0 = (size_t)cl.tok * p.H + h;
    const size_t rs = (size_t)p.H;

    if (tid == 0) {
        mbar_init(&s.bar_ld, 1);
        mbar_init(&s.bar_mma, 1);
        fence_mbar_init();
        const int tok = cl.tok;
        mbar_arrive_expect(&s.bar_ld, (6 * C * DK + 2 * DV * DK + C * C) * 2);
        bulk_g2s(s.R1, p.dU + (size_t)cid * C * DV, C * 64 * 2, &s.bar_ld);
        bulk_g2s(s.R1 + PAIR, p.dU + (size_t)cid * C * DV + C * 64, C * 64 * 2, &s.bar_ld);
        tma_load_3d(s.R1 + C * 64, &p.dOmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.R1 + PAIR + C * 64, &p.dOmap, 64, h, tok, &s.bar_ld);
        tma_load_3d(s.R2, &p.kmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.R2 + PAIR, &p.kmap, 64, h, tok, &s.bar_ld);
        tma_load_3d(s.R2 + C * 64, &p.qmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.R2 + PAIR + C * 64, &p.qmap, 64, h, tok, &s.bar_ld);
        bulk_g2s(s.R3, p.U + (size_t)cid * C * DV, C * 64 * 2, &s.bar_ld);
        bulk_g2s(s.R3 + PAIR, p.U + (size_t)cid * C * DV + C * 64, C * 64 * 2, &s.bar_ld);
        tma_load_3d(s.R3 + C * 64, &p.vmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.R3 + PAIR + C * 64, &p.vmap, 64, h, tok, &s.bar_ld);
        bulk_g2s(s.R4, p.S0 + (size_t)cid * DV * DK, DV * DK * 2, &s.bar_ld);
        bulk_g2s(s.R5, p.dS + (size_t)cid * DV * DK, DV * DK * 2, &s.bar_ld);
        bulk_g2s(s.T, p.Tb + (size_t)cid * C * C, C * C * 2, &s.bar_ld);
        // (no L2 prefetch of the next wave's tiles and images: measured slower,
        // the prefetches share the TMA engine with the loads themselves)
    }
    if (warp == 0) tc5::alloc(&s.tmem, KB_TCOLS);
    if (tid < C) s.beta[tid] = tid < L ? p.beta[row0 + tid * rs] : 0.f;
    // the per-key gate rows of the chunk a wave ahead (512 bytes each) into L2
    if (tid >= 64 && tid < 64 + C && p.pf_stride > 0 && cid + p.pf_stride < (int)gridDim.x) {
        const int pc = cid + p.pf_stride, pbh = pc / p.NT;
        const ChunkLoc pl = chunk_loc(p.seq, p.T, p.H, pbh, pc % p.NT);
        const int r = tid - 64;
        if (pl.valid && r < pl.L)
            bulk_prefetch_l2(p.g + (((size_t)pl.tok + r) * p.H + pbh % p.H) * DK, DK * 4);
    }

    // Thread (c, tg): key / value / TMEM lane c = 32 (warp % 4) + lane, token
    // block tg = warp / 4 (tokens 16 tg .. +15).  Lane-token epilogues: token
    // row 32 (q % 2) + lane of the lane quarter q.
    const int q = warp & 3, tg = warp >> 2, c = 32 * q + lane, i0 = 16 * tg;
    const uint32_t trow = (uint32_t)(32 * q) << 16;  // lane field of this warp's TMEM quarter
    // ---- per-key cumsum of the log-gate (rows past L add 0) ------------------
    float Gr[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int i = i0 + r;
        Gr[r] = i < L ? p.g[(row0 + (size_t)i * rs) * DK + c] : 0.f;
    }
#pragma unroll
    for (int r = 1; r < 16; ++r) Gr[r] += Gr[r - 1];
    s.btot[tg][c] = Gr[15];
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;
    {
        float pre = 0.f;
        for (int t = 0; t < tg; ++t) pre += s.btot[t][c];
#pragma unroll
        for (int r = 0; r < 16; ++r) Gr[r] += pre;
    }
    s.Gf[tg][c] = Gr[0];
    s.Gl[tg][c] = Gr[15];
    const uint32_t sR1 = smem_u32(s.R1), sR2 = smem_u32(s.R2), sR3 = smem_u32(s.R3),
                   sR4 = smem_u32(s.R4), sR5 = smem_u32(s.R5), sT = smem_u32(s.T);
    // later tiles in the S0 / dS space
    __nv_bfloat16* KEL = s.R4;                  // Tma128
    __nv_bfloat16* QEL = s.R4 + C * DK;         // Tma128
    __nv_bfloat16* KER = s.R5;                  // Tma128
    __nv_bfloat16* dTt = s.R5 + C * DK;         // Swz<64>; later dMM^T
    __nv_bfloat16* Xt = s.R5 + C * DK + C * C;  // Swz<64>; later dA
    const uint32_t sKEL = smem_u32(KEL), sQEL = smem_u32(QEL), sKER = smem_u32(KER);
    const uint32_t sdA = smem_u32(Xt), sdMMt = smem_u32(dTt), sdP = smem_u32(s.dP), sdPt = smem_u32(s.dPt);
    uint32_t mph = 0;
    float dG[16];  // this thread's dG terms (dk accumulates in TMEM)
    const uint32_t tstride = (uint32_t)(rs * DK);  // elements between tokens of a [token][key] tensor
    // raw log-gate of token t of this thread's block, key c (0 past the sequence end)
    auto graw = [&](int t) { return i0 + t < L ? p.g[(row0 + (size_t)(i0 + t) * rs) * DK + c] : 0.f; };
    bool ok = mbar_wait(&s.bar_ld, 0, p.status);
    if (__syncthreads_or(!ok)) goto done;
    // dO rows past the sequence end belong to the next sequence: zero them
    if (L < C) {
        for (int e = tid; e < (C - L) * 16; e += KB_THREADS) {
            const int r = L + (e >> 4), pc = e & 15;
            *reinterpret_cast<uint4*>(s.R1 + (pc >> 3) * PAIR + (C + r) * 64 + (pc & 7) * 8) =
                make_uint4(0, 0, 0, 0);
        }
        fence_async_smem();
    }
    tc5::fence_before();
    __syncthreads();

    // ---- phase 1: S0^T [dU ; dO]^T, dS^T U^T, [dU ; dO] U^T, [dU ; dO] V^T --------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
            tc5::mma(tm + T_QW, tc5::mnmajor(sR4, kk, 128 * 128), tc5::kmajor<128>(sR1, kk), ID_QW, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
            tc5::mma(tm + T_KT, tc5::mnmajor(sR5, kk, 128 * 128), tc5::kmajor<128>(sR3, kk), ID_MN64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
            tc5::mma(tm + T_DP, tc5::kmajor<128>(sR1, kk), tc5::kmajor<128>(sR3, kk), ID_KK64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
            tc5::mma(tm + T_DUV, tc5::kmajor<128>(sR1, kk), tc5::kmajor<128>(sR3 + C * 128, kk), ID_KK64, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();

    // ---- epilogue 1 ----------------------------------------------------------------
    if (q >= 2) {  // dP row i (lanes 64..127), columns of block tg: strict lower; the diagonal apart
        const int i = 32 * (q - 2) + lane;
        float pd[16];
        tc5::ld16(pd, tm + trow + T_DP + i0);
        tc5::wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int j = i0 + e;
            if (j == i) s.dPd[i] = pd[e];
            pd[e] = j < i ? pd[e] : 0.f;
            s.dPt[swz<64>(j, i)] = __float2bfloat16_rn(pd[e]);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
            *reinterpret_cast<uint4*>(s.dP + swz<64>(i, i0 + 8 * hh)) =
                make_uint4(pack_bf16(pd[8 * hh], pd[8 * hh + 1]), pack_bf16(pd[8 * hh + 2], pd[8 * hh + 3]),
                           pack_bf16(pd[8 * hh + 4], pd[8 * hh + 5]), pack_bf16(pd[8 * hh + 6], pd[8 * hh + 7]));
    }
    {
        const float Glast = s.Gl[3][c];
        float x[16], z[16];
        tc5::ld16(x, tm + trow + T_QW + i0);   // -dW^T
        tc5::ld16(z, tm + trow + T_KT + i0);   // (U dS)^T
        tc5::wait_ld();
        float gl = 0.f;
        uint32_t dku[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = i0 + r;
            const uint32_t kq = (c >> 6) * PAIR + swz<64>(i, c & 63);
            const float kv = bf(s.R2, kq);
            s.R1[kq + C * 64] = __float2bfloat16_rn(-x[r]);               // dW, in the dO rows
            s.R3[kq] = __float2bfloat16_rn(kv * __expf(Gr[r]));            // Kg, in the U rows
            const float dkr = __expf(Glast - Gr[r]) * z[r];               // etl .* (U dS)
            dku[r] = __float_as_uint(dkr);
            dG[r] = -dkr * kv;
            gl += dkr * kv;
        }
        tc5::st16(tm + trow + T_DK + i0, dku);
        tc5::wait_st();
        s.glp[tg][c] = gl;
        float ss = 0.f;  // <dS, S0> over value rows 32 tg .. +31 of key c
#pragma unroll 8
        for (int v = 32 * tg; v < 32 * tg + 32; ++v) {
            const uint32_t o = Kp<128>::off(v, c);
            ss += bf(s.R5, o) * bf(s.R4, o);
        }
        s.ssp[tg][c] = ss;
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();

    // ---- phase 2: [dW ; .] Kg^T, dW^T T, dU^T T ------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm + T_TW, tc5::kmajor<128>(sR1 + C * 128, kk), tc5::kmajor<128>(sR3, kk), ID_KK64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + T_WT, tc5::mnmajor(sR1 + C * 128, kk, PB), tc5::mnmajor(sT, kk, C * 128), ID_MM64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + T_UT, tc5::mnmajor(sR1, kk, PB), tc5::mnmajor(sT, kk, C * 128), ID_MM64, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();

    // ---- epilogue 2 ----------------------------------------------------------------
    {
        if (q < 2) {  // dT row i, columns of block tg (lanes 0..63)
            float tw[16], du[16];
            tc5::ld16(tw, tm + trow + T_TW + i0);   // dW Kg^T
            tc5::ld16(du, tm + trow + T_DUV + i0);  // dU V^T
            tc5::wait_ld();
            const int i = 32 * q + lane;
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                pk[e] = pack_bf16(s.beta[i0 + 2 * e] * (tw[2 * e] + du[2 * e]),
                                  s.beta[i0 + 2 * e + 1] * (tw[2 * e + 1] + du[2 * e + 1]));
            *reinterpret_cast<uint4*>(dTt + swz<64>(i, i0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(dTt + swz<64>(i, i0 + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        float wt[16], ut[16];
        tc5::ld16(wt, tm + trow + T_WT + i0);   // (T^T dW)^T
        tc5::ld16(ut, tm + trow + T_UT + i0);   // (T^T dU)^T, lane = value c
        tc5::wait_ld();
        const float Gf0 = Gr[0], Gl0 = Gr[15];
        __nv_bfloat16* dvp = p.dv + row0 * DV + c;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = i0 + r;
            const float bi = s.beta[i], eg = __expf(Gr[r]);
            const uint32_t kq = (c >> 6) * PAIR + swz<64>(i, c & 63);
            const float kv = bf(s.R2, kq), qv = bf(s.R2, kq + C * 64), vv = bf(s.R3, kq + C * 64);
            const float w = eg * wt[r];
            dG[r] += bi * w * kv;
            if (i < L) dvp[(uint32_t)i * tstride] = __float2bfloat16_rn(bi * ut[r]);
            ut[r] = w * kv + ut[r] * vv;  // dbeta term, summed over keys below
            wt[r] = bi * w;               // dk term
            const float el = __expf(Gr[r] - Gf0), er = __expf(Gl0 - Gr[r]);
            const uint32_t o = Tma128::off(i, c);
            KEL[o] = __float2bfloat16_rn(kv * el);
            QEL[o] = __float2bfloat16_rn(qv * el);
            KER[o] = __float2bfloat16_rn(kv * er);
        }
        const float b = reduce16(ut, lane);
        if (!(lane & 1)) s.dbp[0][q][i0 + (lane >> 1)] = b;
        tc5::ld16(ut, tm + trow + T_DK + i0);
        tc5::wait_ld();
        uint32_t dku[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) dku[r] = __float_as_uint(ut[r] + wt[r]);
        tc5::st16(tm + trow + T_DK + i0, dku);
        tc5::wait_st();
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();

    // ---- phase 3: X = [dT ; .] T^T ---------------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + T_X, tc5::kmajor<128>(smem_u32(dTt), kk), tc5::kmajor<C>(sT, kk), ID_KK64, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    if (q < 2) {
        const int i = 32 * q + lane;
        float x[16];
        tc5::ld16(x, tm + trow + T_X + i0);
        tc5::wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        *reinterpret_cast<uint4*>(Xt + swz<64>(i, i0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(Xt + swz<64>(i, i0 + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    // ---- phase 4: T^T X ----------------------------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + T_TX, tc5::mnmajor(sT, kk, C * 128), tc5::mnmajor(smem_u32(Xt), kk, C * 128), ID_MM64,
                     kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    // dA = strict_lower(-T^T X) (into X's slot), dMM^T (into dT's slot)
    if (q < 2) {
        const int i = 32 * q + lane;
        const float bi = s.beta[i];
        float x[16];
        tc5::ld16(x, tm + trow + T_TX + i0);
        tc5::wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int j = i0 + e;
            x[e] = j < i ? -x[e] : 0.f;
            dTt[swz<64>(j, i)] = __float2bfloat16_rn(bi * x[e]);
        }
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        *reinterpret_cast<uint4*>(Xt + swz<64>(i, i0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(Xt + swz<64>(i, i0 + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();

    // ---- phase 5a: row-side pair products (X1'^T, X4^T), block pairs J <= I ------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int I = 0; I < 4; ++I)
#pragma unroll
            for (int J = 0; J <= I; ++J) {
                const int pi = I * (I + 1) / 2 + J;
                const uint64_t a = tc5::mnmajor(sKER + 16 * J * 128, 0, C * 128);
                tc5::mma(tm + T_PR + 16 * pi, a, tc5::kmajor<C>(sdA + 16 * I * 128, J), ID_PAIR, false);
                tc5::mma(tm + T_PR + 160 + 16 * pi, a, tc5::kmajor<C>(sdP + 16 * I * 128, J), ID_PAIR, false);
            }
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    {
        // thread (c, tg): rows of block I = tg
        const int I = tg;
        const float GfI = Gr[0];
        const bool exact = GfI - Gr[15] > 80.f;  // this key's diagonal pair by elementwise sums
        float acc[16], a[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.f;
        for (int J = 0; J <= I; ++J) {
            tc5::ld16(a, tm + trow + T_PR + 16 * (I * (I + 1) / 2 + J));
            tc5::wait_ld();
            const float F = (J == I && exact) ? 0.f : __expf(GfI - s.Gl[J][c]);
#pragma unroll
            for (int r = 0; r < 16; ++r) acc[r] = fmaf(F, a[r], acc[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] *= __expf(Gr[r] - GfI);
        if (exact) {  // e^{G_r - G_jj} from the in-block partial sums of g
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                float sg = 0.f;
#pragma unroll 1
                for (int jj = r - 1; jj >= 0; --jj) {
                    sg += graw(jj + 1);
                    acc[r] += bf(Xt, swz<64>(i0 + r, i0 + jj)) * __expf(sg) *
                              bf(s.R2, (c >> 6) * PAIR + swz<64>(i0 + jj, c & 63));
                }
            }
        }
        // X1' -> dk, dG, dbeta
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = i0 + r;
            const float bi = s.beta[i], kv = bf(s.R2, (c >> 6) * PAIR + swz<64>(i, c & 63));
            dG[r] = fmaf(bi * kv, acc[r], dG[r]);
            a[r] = bi * acc[r];  // dk term
            acc[r] *= kv;
        }
        const float b = reduce16(acc, lane);
        if (!(lane & 1)) s.dbp[1][q][i0 + (lane >> 1)] = b;
        {
            tc5::ld16(acc, tm + trow + T_DK + i0);
            tc5::wait_ld();
            uint32_t dku[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) dku[r] = __float_as_uint(acc[r] + a[r]);
            tc5::st16(tm + trow + T_DK + i0, dku);
            tc5::wait_st();
        }
        // X4 -> dq (with scale e^G (dO S0) and the diagonal of dP), dG
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = 0.f;
        for (int J = 0; J <= I; ++J) {
            tc5::ld16(a, tm + trow + T_PR + 160 + 16 * (I * (I + 1) / 2 + J));
            tc5::wait_ld();
            const float F = (J == I && exact) ? 0.f : __expf(GfI - s.Gl[J][c]);
#pragma unroll
            for (int r = 0; r < 16; ++r) acc[r] = fmaf(F, a[r], acc[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] *= __expf(Gr[r] - GfI);
        if (exact) {
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                float sg = 0.f;
#pragma unroll 1
                for (int jj = r - 1; jj >= 0; --jj) {
                    sg += graw(jj + 1);
                    acc[r] += bf(s.dP, swz<64>(i0 + r, i0 + jj)) * __expf(sg) *
                              bf(s.R2, (c >> 6) * PAIR + swz<64>(i0 + jj, c & 63));
                }
            }
        }
        tc5::ld16(a, tm + trow + T_QW + 64 + i0);  // (dO S0)^T
        tc5::wait_ld();
        __nv_bfloat16* dqp = p.dq + row0 * DK + c;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = i0 + r;
            const uint32_t kq = (c >> 6) * PAIR + swz<64>(i, c & 63);
            const float kv = bf(s.R2, kq), qv = bf(s.R2, kq + C * 64);
            const float d = fmaf(__expf(Gr[r]), a[r], acc[r]);  // e^G (dO S0) + X4
            dG[r] = fmaf(p.scale * qv, d, dG[r]);
            if (i < L) dqp[(uint32_t)i * tstride] = __float2bfloat16_rn(p.scale * fmaf(s.dPd[i], kv, d));
        }
    }
    tc5::fence_before();
    __syncthreads();

    // ---- phase 5b: column-side pair products (X2^T, X3^T), block pairs I >= J ----------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int I = 0; I < 4; ++I)
#pragma unroll
            for (int J = 0; J <= I; ++J) {
                const int pi = I * (I + 1) / 2 + J;
                tc5::mma(tm + T_PR + 16 * pi, tc5::mnmajor(sKEL + 16 * I * 128, 0, C * 128),
                         tc5::kmajor<C>(sdMMt + 16 * J * 128, I), ID_PAIR, false);
                tc5::mma(tm + T_PR + 160 + 16 * pi, tc5::mnmajor(sQEL + 16 * I * 128, 0, C * 128),
                         tc5::kmajor<C>(sdPt + 16 * J * 128, I), ID_PAIR, false);
            }
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    {
        // thread (c, tg): output tokens of block J = tg
        const int J = tg;
        const float GlJ = Gr[15];
        const bool exact = Gr[0] - GlJ > 80.f;
        // X2 + scale X3 share their factors: one accumulator
        float a2[16], a3[16], side[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) side[r] = 0.f;
        for (int I = J; I < 4; ++I) {
            const int pi = I * (I + 1) / 2 + J;
            tc5::ld16(a2, tm + trow + T_PR + 16 * pi);
            tc5::ld16(a3, tm + trow + T_PR + 160 + 16 * pi);
            tc5::wait_ld();
            const float F = (I == J && exact) ? 0.f : __expf(s.Gf[I][c] - GlJ);
#pragma unroll
            for (int r = 0; r < 16; ++r) side[r] = fmaf(F, fmaf(p.scale, a3[r], a2[r]), side[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) side[r] *= __expf(GlJ - Gr[r]);
        if (exact) {  // e^{G_ii - G_r} from the in-block partial sums of g
#pragma unroll
            for (int r = 0; r < 15; ++r) {
                float sg = 0.f;
#pragma unroll 1
                for (int ii = r + 1; ii < 16; ++ii) {
                    sg += graw(ii);
                    const float d = __expf(sg);
                    const uint32_t kq = (c >> 6) * PAIR + swz<64>(i0 + ii, c & 63);
                    side[r] += d * fmaf(p.scale * bf(s.dPt, swz<64>(i0 + r, i0 + ii)), bf(s.R2, kq + C * 64),
                                        bf(dTt, swz<64>(i0 + r, i0 + ii)) * bf(s.R2, kq));
                }
            }
        }
        __nv_bfloat16* dkp = p.dk + row0 * DK + c;
        tc5::ld16(a2, tm + trow + T_DK + i0);
        tc5::wait_ld();
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int j = i0 + r;
            const uint32_t kq = (c >> 6) * PAIR + swz<64>(j, c & 63);
            const float kv = bf(s.R2, kq), qv = bf(s.R2, kq + C * 64);
            dG[r] = fmaf(-kv, side[r], dG[r]);
            const float dkj = a2[r] + side[r] + p.scale * s.dPd[j] * qv;
            if (j < L) dkp[(uint32_t)j * tstride] = __float2bfloat16_rn(dkj);
        }
    }

    // ---- dg: reverse cumsum of dG per key (plus the G_last terms); dbeta ---------------
    {
        if (tg == 3) {
            float gl = 0.f, ss = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) { gl += s.glp[t][c]; ss += s.ssp[t][c]; }
            dG[15] += gl + __expf(Gr[15]) * ss;
        }
#pragma unroll
        for (int r = 14; r >= 0; --r) dG[r] += dG[r + 1];
        s.dgt[tg][c] = dG[0];
    }
    __syncthreads();
    {
        float suf = 0.f;
        for (int t = 3; t > tg; --t) suf += s.dgt[t][c];
        float* dgp = p.dg + row0 * DK + c;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = i0 + r;
            if (i < L) dgp[(uint32_t)i * tstride] = dG[r] + suf;
        }
        if (tid < C && tid < L) {
            float b = 0.f;
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) b += s.dbp[t][qq][tid];
            p.dbeta[row0 + (size_t)tid * rs] = b;
        }
    }
done:
    tc5::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc5::fence_after();
        tc5::dealloc(tm, KB_TCOLS);
    }
}

}  // namespace

namespace tc {
bool launch_bwd_local5_kda(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp, const void* dO,
                           void* dq, void* dk, void* dv, float* dg, float* dbeta, void* ws, cudaStream_t st) {
    KbPtrs lp{};
    lp.qmap = cp.qmap; lp.kmap = cp.kmap; lp.vmap = cp.vmap;
    if (!encode_token_map(&lp.dOmap, dO, d.B, d.T, d.H)) return false;
    char* base = (char*)ws;
    lp.g = cp.g; lp.beta = cp.beta; lp.status = cp.status;
    lp.S0 = (const __nv_bfloat16*)(base + L.S0);
    lp.U = (const __nv_bfloat16*)(base + L.U);
    lp.dS = (const __nv_bfloat16*)(base + L.dS);
    lp.dU = (const __nv_bfloat16*)(base + L.dU);
    lp.Tb = cp.Tb;
    lp.dq = (__nv_bfloat16*)dq; lp.dk = (__nv_bfloat16*)dk; lp.dv = (__nv_bfloat16*)dv;
    lp.dg = dg; lp.dbeta = dbeta;
    lp.B = d.B; lp.T = d.T; lp.H = d.H; lp.NT = L.NT; lp.scale = d.scale;
    lp.seq = cp.seq;
    lp.pf_stride = sm_count();  // one CTA per SM
    const int smem = sizeof(KbSmem) + 1024;
    cudaFuncSetAttribute(tc5_bwd_local_kda_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_bwd_local_kda", st,
               tc5_bwd_local_kda_kernel<<<(unsigned)L.nchunks, KB_THREADS, smem, st>>>(lp));
    return true;
}
}  // namespace tc
}  // namespace gdn
