// tc5_bwd_local.cu -- the chunkwise backward's local gradients on the
// fifth-generation tensor cores (scalar gate, bf16, dk = dv = 128, chunk 64).
//
// Reverse mode through the chunk equations of "Gated Delta Networks:
// Improving Mamba2 with Delta Rule" (paper review), section "Method" (the WY /
// UT-transform form; see tc_chunk.cu).  Given a chunk's entering state S0 and
// U (from the forward recompute) and its dS (gradient of the state leaving it)
// and dU (from the reverse walk), with Gamma_ij = e^{G_i - G_j}, etl_i =
// e^{G_last - G_i} and gamma = e^{G_last}:
//   dq  = scale e^G .* (dO S0) + sdPG K,        sdPG = scale lower(dO U^T) .* Gamma
//   dW  = -dU S0,   dT = dW (beta e^G .* K)^T + dU (beta .* V)^T
//   dA  = strict_lower(-T^T dT T^T),   dMM = dA .* beta_i .* Gamma
//   dk  = etl .* (U dS) + beta e^G .* (T^T dW) + dMM K + dMM^T K + sdPG^T Q
//   dv  = beta .* (T^T dU)
// and the gate and beta gradients from the matching row and column sums, with
// dg the reverse within-chunk cumsum of dG.
//
// Every product is one tcgen05 MMA group with M = 128 and an fp32 accumulator
// in tensor memory.  The 64-token tiles sit in pairs in 128-row K-major panels
// ([dU ; dO], [K ; Q], [U ; V]), so a product whose A is a pair yields two
// results at once (lanes 0..63 and 64..127), and a 64-row A reads its partner
// tile (or a neighbouring buffer) as rows 64..127 whose result is ignored:
//   [dU ; dO] S0      -> -dW (lanes 0..63) and dO S0 (dO rows pre-scaled by
//                        scale e^{G_i}: the dq accumulator, lanes 64..127)
//   [U ; V] dS        -> etl .* (U dS) (U rows pre-scaled: the dk accumulator)
//   [K ; Q] K^T       -> K K^T, Q K^T       [dU ; dO] U^T -> dO U^T
//   [dU ; dO] V^T     -> dU V^T             [dW ; .] K^T  -> dW K^T
//   [dT ; .] T^T -> X,  [T^T ; .] X -> T^T X,  [T^T ; .] dW,  [T^T ; .] dU
//   dk += [dMM ; .] K + [dMM^T ; .] K + [sdPG^T ; .] Q,   dq += [. ; sdPG] K
// In every epilogue four warps share a TMEM lane quarter (one token row per
// thread) and split the row's columns; per-token sums meet in shared-memory
// atomics, and column sums over tokens go through a shared-memory transpose.
// One CTA of sixteen warps per chunk; thread 0 issues the loads and the MMAs.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace {
using namespace tc;

constexpr int BL_THREADS = 512;  // warp w: TMEM lane quarter w % 4, column group w / 4
constexpr int PAIR = 128 * 64;  // elements of one 128-row, 64-column panel
// tensor-memory columns
constexpr uint32_t TA = 0,     // [-dW ; dq accumulator]          128
    TB = 128,                  // [dk accumulator ; .]            128
    TC1 = 256,                 // [K K^T ; Q K^T]                  64  (then X)
    TC2 = 320,                 // [. ; dO U^T]                     64  (then T^T X)
    TW = 384,                  // [dW K^T ; .]                     64
    TU = 448,                  // [dU V^T ; .]                     64
    TKG = 256,                 // [T^T dW ; .]                    128 (phase E)
    TVB = 384,                 // [T^T dU ; .]                    128 (phase E)
    BL_TCOLS = 512;
constexpr uint32_t ID_N64 = tc5::idesc_bf16(128, 64, false, false);     // A, B K-major
constexpr uint32_t ID_N128_BMN = tc5::idesc_bf16(128, 128, false, true); // B MN-major
constexpr uint32_t ID_N64_AMN_BMN = tc5::idesc_bf16(128, 64, true, true);
constexpr uint32_t ID_N128_AMN_BMN = tc5::idesc_bf16(128, 128, true, true);

struct alignas(1024) BlSmem {
    __nv_bfloat16 R1[2 * PAIR];  // [dU | dO] panels; later dW in the dO rows
    __nv_bfloat16 R2[2 * PAIR];  // [K | Q]
    __nv_bfloat16 R3[2 * PAIR];  // [U | V]; later dMM in the U rows of panel 0
    __nv_bfloat16 R4[DV * DK];   // S0 (Kp<128>); later dT | X | M (fp32)
    __nv_bfloat16 R5[DV * DK];   // dS (Kp<128>); later . | sdPG | transpose scratch (fp32)
    // Swz<64> T, then 8 KB that the MN-major T^T operands read as their unused
    // rows 64..127
    __nv_bfloat16 T[2 * C * C];
    float G[C], beta[C];
    // Fixed-order partial sums (the dg and dbeta results are bit-reproducible):
    float pG[8][C];              // dG terms of a token's own rows, per (column group, lane half)
    float pB[4][C];              // dbeta terms, per column group
    float pC[8][C];              // column sums of hP and hA, per 8-row block
    float red[16], red2[16];     // per-warp sums: <dS, S0>; etl <dKt, k> (enters dG_last)
    float dgs[C];                // reverse-cumsum scratch
    uint64_t bar_ld, bar_mma;
    uint32_t tmem;
};

struct BlPtrs {
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

// 32 consecutive TMEM columns of this thread's lane into v[0..31].
GDN_DEV void ld_row32(float* v, uint32_t taddr) {
    tc5::ld32(*reinterpret_cast<float(*)[32]>(v), taddr);
}

// Scale the 64 elements of row r (0..127) of a pair region's panel by f.
GDN_DEV void scale_pair_row(__nv_bfloat16* R, int r, int panel, float f) {
    __nv_bfloat16* row = R + panel * PAIR + r * 64;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        const int j = (jj + r) & 7;  // per-row rotated order: lanes on different rows, different banks
        uint4 x = *reinterpret_cast<uint4*>(row + 8 * j);
        uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 v = unpack_bf16(w[i]);
            w[i] = pack_bf16(v.x * f, v.y * f);
        }
        *reinterpret_cast<uint4*>(row + 8 * j) = x;
    }
}

// sum_{c < 32} x[c] * R[r][c0 + c] for row r of a pair region (c0 a multiple
// of 32): four 16-byte loads of the row's swizzled chunks.
GDN_DEV float dot_row32(const float* x, const __nv_bfloat16* R, int r, int c0) {
    const __nv_bfloat16* base = R + (c0 >> 6) * PAIR;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(base + swz<64>(r, (c0 & 63) + 8 * j));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16(w[i]);
            acc = fmaf(x[8 * j + 2 * i], f.x, acc);
            acc = fmaf(x[8 * j + 2 * i + 1], f.y, acc);
        }
    }
    return acc;
}

__global__ void __launch_bounds__(BL_THREADS, 1) tc5_bwd_local_kernel(const __grid_constant__ BlPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BlSmem& s = *reinterpret_cast<BlSmem*>(align1k(smem_raw));
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
    if (warp == 0) {
        tc5::alloc(&s.tmem, BL_TCOLS);
        float g0 = lane < L ? p.g[row0 + lane * rs] : 0.f;
        float g1 = lane + 32 < L ? p.g[row0 + (lane + 32) * rs] : 0.f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float x0 = __shfl_up_sync(0xffffffffu, g0, o);
            const float x1 = __shfl_up_sync(0xffffffffu, g1, o);
            if (lane >= o) { g0 += x0; g1 += x1; }
        }
        g1 += __shfl_sync(0xffffffffu, g0, 31);
        s.G[lane] = g0;
        s.G[lane + 32] = g1;
        s.beta[lane] = lane < L ? p.beta[row0 + lane * rs] : 0.f;
        s.beta[lane + 32] = lane + 32 < L ? p.beta[row0 + (lane + 32) * rs] : 0.f;
    }
    if (tid < 16) s.red2[tid] = 0.f;
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;
    // TMEM lane quarter q, column group cg; row = this thread's token (lanes
    // 0..63: tokens of the lower half, lanes 64..127: of the upper half)
    const int q = warp & 3, cg = warp >> 2, row = 32 * (q & 1) + lane;
    const uint32_t trow = tm + ((uint32_t)(32 * q) << 16);  // this thread's TMEM lane
    const uint32_t sR1 = smem_u32(s.R1), sR2 = smem_u32(s.R2), sR3 = smem_u32(s.R3),
                   sR4 = smem_u32(s.R4), sR5 = smem_u32(s.R5), sT = smem_u32(s.T);
    constexpr uint32_t PB = PAIR * 2;  // bytes of one pair panel (the panel stride of pair regions)
    const float Gl = s.G[C - 1];
    uint32_t mph = 0;  // phase of bar_mma
    float myG = 0.f, myB = 0.f;  // this thread's (token, column group) share of dG / dbeta
    float myC = 0.f;             // this thread's (column, row block) share of the column sums
    // S0 / dS space, reused once both are dead
    float* Mf = reinterpret_cast<float*>(s.R4 + 2 * C * 64);   // M (fp32, [t][j], rotated columns)
    float* Xs = reinterpret_cast<float*>(s.R5 + 2 * C * 64);   // transpose scratch (fp32)
    __nv_bfloat16* dTt = s.R4;                                 // dT (Swz<64>)
    __nv_bfloat16* Xt = s.R4 + C * 64;                         // X (Swz<64>)
    __nv_bfloat16* sdPG = s.R5 + C * 64;                       // scale dP .* Gamma (Swz<64>)
    __nv_bfloat16* dMM = s.R3;                                 // dMM (Swz<64>), in the U rows
    bool ok = mbar_wait(&s.bar_ld, 0, p.status);
    if (__syncthreads_or(!ok)) goto done;
    // dO rows past the sequence end belong to the next sequence: zero them
    if (L < C) {
        for (int e = tid; e < (C - L) * 16; e += BL_THREADS) {
            const int r = L + (e >> 4), pc = e & 15;
            *reinterpret_cast<uint4*>(s.R1 + (pc >> 3) * PAIR + (C + r) * 64 + (pc & 7) * 8) =
                make_uint4(0, 0, 0, 0);
        }
        fence_async_smem();
    }
    __syncthreads();

    // ---- phase A1: products of the unscaled tiles ----------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)  // [dU ; dO] U^T
            tc5::mma(tm + TC2, tc5::kmajor<128>(sR1, kk), tc5::kmajor<128>(sR3, kk), ID_N64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)  // [K ; Q] K^T
            tc5::mma(tm + TC1, tc5::kmajor<128>(sR2, kk), tc5::kmajor<128>(sR2, kk), ID_N64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)  // [dU ; dO] V^T
            tc5::mma(tm + TU, tc5::kmajor<128>(sR1, kk), tc5::kmajor<128>(sR3 + C * 128, kk), ID_N64, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    // dO rows *= scale e^{G_i} (the dq rows), U rows *= e^{G_last - G_i} (the dk rows)
    if (tid < 256) {
        const int r = (tid >> 1) & 63, pn = tid & 1;
        if (tid < 128) scale_pair_row(s.R1, C + r, pn, p.scale * __expf(s.G[r]));
        else scale_pair_row(s.R3, r, pn, __expf(Gl - s.G[r]));
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    // ---- phase A2: [dU ; dO'] S0 and [U' ; V] dS -------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
            tc5::mma(tm + TA, tc5::kmajor<128>(sR1, kk), tc5::mnmajor(sR4, kk, 128 * 128), ID_N128_BMN, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk)
            tc5::mma(tm + TB, tc5::kmajor<128>(sR3, kk), tc5::mnmajor(sR5, kk, 128 * 128), ID_N128_BMN, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    {
        // ---- <dS, S0> (before S0 / dS space is reused) ------------------------
        float ss = 0.f;
        for (int e = tid; e < DV * DK / 8; e += BL_THREADS) {
            const uint4 x = reinterpret_cast<const uint4*>(s.R5)[e];
            const uint4 y = reinterpret_cast<const uint4*>(s.R4)[e];
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 a2 = unpack_bf16(xs[t]), b2 = unpack_bf16(ys[t]);
                ss += a2.x * b2.x + a2.y * b2.y;
            }
        }
        ss = warp_sum(ss);
        if (lane == 0) s.red[warp] = ss;
    }
    __syncthreads();  // S0 and dS are dead from here on
    {
        // ---- epilogue A -------------------------------------------------------
        if (q >= 2) {
            // token i: dP, Q K^T (columns 16cg..) -> sdPG and hP; <dO' S0, q_i> (columns 32cg..)
            const int i = row;
            const float Gi = s.G[i];
            float dp[16], qk[16], x[32];
            tc5::ld16(dp, trow + TC2 + 16 * cg);
            tc5::ld16(qk, trow + TC1 + 16 * cg);
            ld_row32(x, trow + TA + 32 * cg);
            tc5::wait_ld();
            float hrow = 0.f;
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int j = 16 * cg + c;
                const float g = j <= i ? p.scale * dp[c] * __expf(Gi - s.G[j]) : 0.f;  // scale dP .* Gamma
                const float hp = g * qk[c];                    // dP .* (scale Q K^T .* Gamma)
                hrow += hp;
                Xs[i * 64 + ((j + i) & 63)] = hp;              // column sums below
                dp[c] = g;
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) pk[c] = pack_bf16(dp[2 * c], dp[2 * c + 1]);
            *reinterpret_cast<uint4*>(sdPG + swz<64>(i, 16 * cg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(sdPG + swz<64>(i, 16 * cg + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            // scale e^{G_i} <dO S0 row i, q_i>, this thread's 32 columns
            const float dqq = dot_row32(x, s.R2, C + i, 32 * cg);
            myG += hrow + dqq;
        } else {
            // token t: -dW (columns 32cg..) -> dW (bf16, into the dO rows of R1);
            // M (columns 16cg..); <etl dKt row t, k_t> (columns 32cg..)
            const int t = row;
            const float Gt = s.G[t];
            float x[32], kk[16], y[32];
            ld_row32(x, trow + TA + 32 * cg);
            tc5::ld16(kk, trow + TC1 + 16 * cg);
            ld_row32(y, trow + TB + 32 * cg);
            tc5::wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(-x[2 * c], -x[2 * c + 1]);
            __nv_bfloat16* dst = s.R1 + (cg >> 1) * PAIR;  // panel of key columns 32cg..
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(dst + swz<64>(C + t, 32 * (cg & 1) + 8 * q4)) =
                    make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int j = 16 * cg + c;
                Mf[t * 64 + ((j + t) & 63)] = j < t ? kk[c] * __expf(Gt - s.G[j]) : 0.f;
            }
            float hk = dot_row32(y, s.R2, t, 32 * cg);
            myG -= hk;  // -etl_t <dKt_t, k_t>; the same enters dG_last
            hk = warp_sum(hk);
            if (lane == 0) s.red2[warp] = hk;
        }
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    {   // column sums of hP: dG_j -= sum_i hP_ij (eight row blocks per column)
        const int j = tid & 63, pb = tid >> 6;
#pragma unroll
        for (int i = 8 * pb; i < 8 * pb + 8; ++i) myC -= Xs[i * 64 + ((j + i) & 63)];
    }
    // ---- phase B: [dW ; .] K^T -----------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm + TW, tc5::kmajor<128>(sR1 + C * 128, kk), tc5::kmajor<128>(sR2, kk), ID_N64, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    // ---- epilogue B: dT row t = beta_j (e^{G_j} dW K^T + dU V^T)_tj -----------
    if (q < 2) {
        const int t = row;
        float tw[16], tu[16];
        tc5::ld16(tw, trow + TW + 16 * cg);
        tc5::ld16(tu, trow + TU + 16 * cg);
        tc5::wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int j0 = 16 * cg + 2 * c;
            const float d0 = s.beta[j0] * (__expf(s.G[j0]) * tw[2 * c] + tu[2 * c]);
            const float d1 = s.beta[j0 + 1] * (__expf(s.G[j0 + 1]) * tw[2 * c + 1] + tu[2 * c + 1]);
            pk[c] = pack_bf16(d0, d1);
        }
        *reinterpret_cast<uint4*>(dTt + swz<64>(t, 16 * cg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dTt + swz<64>(t, 16 * cg + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    // ---- phase C1: X = [dT ; .] T^T ---------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TC1, tc5::kmajor<128>(smem_u32(dTt), kk), tc5::kmajor<C>(sT, kk), ID_N64, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    if (q < 2) {
        const int t = row;
        float x[16];
        tc5::ld16(x, trow + TC1 + 16 * cg);
        tc5::wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) pk[c] = pack_bf16(x[2 * c], x[2 * c + 1]);
        *reinterpret_cast<uint4*>(Xt + swz<64>(t, 16 * cg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(Xt + swz<64>(t, 16 * cg + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    // ---- phase C2: T^T X ----------------------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TC2, tc5::mnmajor(sT, kk, C * 128), tc5::mnmajor(smem_u32(Xt), kk, C * 128),
                     ID_N64_AMN_BMN, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    // ---- epilogue D: dA = strict_lower(-T^T X); dMM; hA; dbeta and dG terms ----
    if (q < 2) {
        const int i = row;
        const float Gi = s.G[i], bi = s.beta[i];
        float x[16];
        tc5::ld16(x, trow + TC2 + 16 * cg);
        tc5::wait_ld();
        float hrow = 0.f, brow = 0.f;
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const int j = 16 * cg + c;
            const float dA = j < i ? -x[c] : 0.f;
            const float m = Mf[i * 64 + ((j + i) & 63)];  // K K^T .* Gamma (strict lower)
            brow += dA * m;
            const float hA = dA * bi * m;
            hrow += hA;
            Xs[i * 64 + ((j + i) & 63)] = hA;
            x[c] = j < i ? dA * bi * __expf(Gi - s.G[j]) : 0.f;  // dMM
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) pk[c] = pack_bf16(x[2 * c], x[2 * c + 1]);
        *reinterpret_cast<uint4*>(dMM + swz<64>(i, 16 * cg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dMM + swz<64>(i, 16 * cg + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        myG += hrow;
        myB += brow;
    }
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    {   // column sums of hA: dG_j -= sum_i hA_ij
        const int j = tid & 63, pb = tid >> 6;
#pragma unroll
        for (int i = 8 * pb; i < 8 * pb + 8; ++i) myC -= Xs[i * 64 + ((j + i) & 63)];
    }
    // ---- phase E: the remaining products --------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
        const uint32_t sdMM = smem_u32(dMM), ssdPG = smem_u32(sdPG);
        // dk += dMM K + dMM^T K + sdPG^T Q
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TB, tc5::kmajor<128>(sdMM, kk), tc5::mnmajor(sR2, kk, PB), ID_N128_BMN, true);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TB, tc5::mnmajor(sdMM, kk, C * 128), tc5::mnmajor(sR2, kk, PB), ID_N128_AMN_BMN, true);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TB, tc5::mnmajor(ssdPG, kk, C * 128), tc5::mnmajor(sR2 + C * 128, kk, PB),
                     ID_N128_AMN_BMN, true);
        // dq += [. ; sdPG] K   (rows 0..63 of the A view are the 8 KB before sdPG)
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TA, tc5::kmajor<128>(ssdPG - C * 128, kk), tc5::mnmajor(sR2, kk, PB), ID_N128_BMN, true);
        // T^T dW and T^T dU
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TKG, tc5::mnmajor(sT, kk, C * 128), tc5::mnmajor(sR1 + C * 128, kk, PB),
                     ID_N128_AMN_BMN, kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + TVB, tc5::mnmajor(sT, kk, C * 128), tc5::mnmajor(sR1, kk, PB), ID_N128_AMN_BMN, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();
    // ---- epilogue E: dk, dv, dq (columns 32cg..); dbeta / dG terms -------------------
    if (q < 2) {
        const int t = row;
        const float bt = s.beta[t], egt = __expf(s.G[t]);
        float a[32], kg[32];
        ld_row32(a, trow + TB + 32 * cg);
        ld_row32(kg, trow + TKG + 32 * cg);
        tc5::wait_ld();
        const float hk = dot_row32(kg, s.R2, t, 32 * cg);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; ++c) a[c] = fmaf(bt * egt, kg[c], a[c]);
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(a[2 * c], a[2 * c + 1]);
        if (t < L) {
            __nv_bfloat16* dkp = p.dk + (row0 + (size_t)t * rs) * DK + 32 * cg;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(dkp + 8 * q4) =
                    make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        ld_row32(a, trow + TVB + 32 * cg);
        tc5::wait_ld();
        const float hv = dot_row32(a, s.R3, C + t, 32 * cg);
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(bt * a[2 * c], bt * a[2 * c + 1]);
        if (t < L) {
            __nv_bfloat16* dvp = p.dv + (row0 + (size_t)t * rs) * DV + 32 * cg;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(dvp + 8 * q4) =
                    make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        myB += egt * hk + hv;
        myG += bt * egt * hk;
    } else {
        const int i = row;
        float a[32];
        ld_row32(a, trow + TA + 32 * cg);
        tc5::wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(a[2 * c], a[2 * c + 1]);
        if (i < L) {
            __nv_bfloat16* dqp = p.dq + (row0 + (size_t)i * rs) * DK + 32 * cg;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(dqp + 8 * q4) =
                    make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
    }
    // ---- per-token sums in a fixed order: dG (own-row terms + column terms),
    // dbeta; dg = reverse cumsum of dG -------------------------------------------
    s.pG[cg + 4 * (q >> 1)][row] = myG;
    if (q < 2) s.pB[cg][row] = myB;
    s.pC[tid >> 6][tid & 63] = myC;
    __syncthreads();
    if (warp < 2) {
        const int t = tid;
        float dG = 0.f, dB = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) dG += s.pG[k][t] + s.pC[k][t];
#pragma unroll
        for (int k = 0; k < 4; ++k) dB += s.pB[k][t];
        if (t == C - 1) {  // G_last: e^{G_last} <dS, S0> + sum_i etl_i <dKt_i, k_i>
            float ss = 0.f, la = 0.f;
#pragma unroll
            for (int w = 0; w < 16; ++w) { ss += s.red[w]; la += s.red2[w]; }
            dG += __expf(Gl) * ss + la;
        }
        float x = dG;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += y;
        }
        s.dgs[t] = x;  // per-warp suffix sums
        s.pB[0][t] = dB;
    }
    __syncthreads();
    if (tid < C) {
        const float x = s.dgs[tid] + (tid < 32 ? s.dgs[32] : 0.f);
        if (tid < L) {
            p.dg[row0 + (size_t)tid * rs] = x;
            p.dbeta[row0 + (size_t)tid * rs] = s.pB[0][tid];
        }
    }
done:
    tc5::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc5::fence_after();
        tc5::dealloc(tm, BL_TCOLS);
    }
}

}  // namespace

namespace tc {
bool launch_bwd_local5(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& cp, const void* dO,
                       void* dq, void* dk, void* dv, float* dg, float* dbeta, void* ws, cudaStream_t st) {
    BlPtrs lp{};
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
    const int smem = sizeof(BlSmem) + 1024;
    cudaFuncSetAttribute(tc5_bwd_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_bwd_local", st,
               tc5_bwd_local_kernel<<<(unsigned)L.nchunks, BL_THREADS, smem, st>>>(lp));
    return true;
}
}  // namespace tc
}  // namespace gdn
