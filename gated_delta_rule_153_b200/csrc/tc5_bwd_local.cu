// tc5_bwd_local.cu -- the chunkwise backward's local gradients on the
// fifth-generation tensor cores (scalar gate, bf16, dk = dv = 128, chunk 64).
//
// Reverse mode through the chunk equations of "Gated Delta Networks:
// Improving Mamba2 with Delta Rule" (paper review), section "Method" (the WY /
// UT-transform form; see tc_chunk.cu).  Given a chunk's entering state S0 and
// U (from the forward), its dS (gradient of the state leaving it) and dU
// (from the reverse walk), with Gamma_ij = e^{G_i - G_j}, etl_i =
// e^{G_last - G_i} and gamma = e^{G_last}:
//   dq  = scale e^G .* (dO S0) + sdPG K,        sdPG = scale lower(dO U^T) .* Gamma
//   dW  = -dU S0,   Gk = T^T dW,   Gv = T^T dU
//   dA  = strict_lower(-T^T dT T^T) = strict_lower(-(Gk W^T + Gv U~^T)),
//   dMM = dA .* beta_i .* Gamma
//   dk  = etl .* (U dS) + beta e^G .* Gk + dMM K + dMM^T K + sdPG^T Q
//   dv  = beta .* Gv
// and the gate and beta gradients from the matching row and column sums, with
// dg the reverse within-chunk cumsum of dG.  The dA line uses the WY factors
// themselves: dT = dW (beta e^G .* K)^T + dU (beta .* V)^T, so
// T^T dT T^T = Gk (T beta e^G K)^T + Gv (T beta V)^T = Gk W^T + Gv U~^T, and
// the W and U~ images of the forward's preparation serve as operands.  One
// product replaces the chain dT -> dT T^T -> T^T (dT T^T).
//
// Every product is one tcgen05 MMA group with M = 128 and an fp32 accumulator
// in tensor memory.  The 64-token tiles sit in pairs in 128-row K-major panels
// ([dU ; dO], [K ; Q]), so a product whose A is a pair yields two results at
// once (lanes 0..63 and 64..127), and a 64-row A reads its partner tile (or a
// neighbouring buffer) as rows 64..127 whose result is ignored:
//   A:  [dU ; dO] S0 -> -dW and dO S0 (the dq accumulator)
//       [U ; .] dS   -> U dS (the dk accumulator)
//       [dU ; dO] U^T -> dO U^T        [K ; Q] K^T -> K K^T, Q K^T
//   E1: [T^T ; .] dW -> Gk,  [T^T ; .] dU -> Gv,
//       dq += [. ; sdPG] K,  dk += [sdPG^T ; .] Q
//   C:  [Gk ; .] W^T + [Gv ; .] U~^T -> -dA (Gk and Gv as bf16 A operands in
//       tensor memory),  [K ; .] K^T again (for M = K K^T .* Gamma)
//   E2: dk += [dMM ; .] K + [dMM^T ; .] K
// The row scalings of the first products (scale e^{G_i} of the dq rows,
// e^{G_last - G_i} of the dk rows) are applied to the accumulators in the
// first epilogue (a TMEM load, scale, store), so every product of phase A
// reads the tiles as loaded and goes out in one group.  In every epilogue
// four warps share a TMEM lane quarter (one token row per thread) and split
// the row's columns; per-token sums meet in fixed-order shared-memory
// partials, and column sums over tokens go through a shared-memory transpose.
// Sixteen warps per CTA; thread 0 issues the MMAs, a lane of warp 2 the loads.
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
constexpr uint32_t TA = 0,     // [-dW ; dq accumulator]          128; after E1 its lanes
                               // 0..63 hold bf16 Gk (columns 0..63) and Gv (64..127)
    TB = 128,                  // [dk accumulator ; .]            128
    TC1 = 256,                 // [K K^T ; Q K^T]                  64
    TC2 = 320,                 // [. ; dO U^T]                     64
    TKG = 256,                 // [Gk = T^T dW ; .]               128 (after the first epilogue)
    TVB = 384,                 // [Gv = T^T dU ; .]               128 (after the first epilogue)
    TD = 384,                  // [Gk W^T + Gv U~^T ; .]           64 (after Gv is read)
    TKK = 448,                 // [K K^T ; .] again                64 (after Gv is read)
    BL_TCOLS = 512;
constexpr uint32_t ID_N64 = tc5::idesc_bf16(128, 64, false, false);     // A, B K-major
constexpr uint32_t ID_N64_BMN = tc5::idesc_bf16(128, 64, false, true);   // B MN-major
constexpr uint32_t ID_N128_BMN = tc5::idesc_bf16(128, 128, false, true); // B MN-major
constexpr uint32_t ID_N128_AMN_BMN = tc5::idesc_bf16(128, 128, true, true);

// Shared memory (one CTA per SM).  The CTA is persistent: it takes the chunks
// blockIdx.x, blockIdx.x + gridDim.x, ... and loads each buffer of the next
// chunk as soon as the current chunk is done with it (S0 and U after the
// first products, T, Q, dU and dO after E1, dS after the E1 epilogue, W and
// U~ after C, K after E2), so the loads of a chunk overlap the work of the
// one before.  Between the first products and the E1 epilogue the dS space
// holds this chunk's V tile (for <Gv_t, v_t>).
struct alignas(1024) BlSmem {
    __nv_bfloat16 R4[DV * DK];   // S0 (Kp<128>)
    __nv_bfloat16 R5[DV * DK];   // dS (Kp<128>); then V (Tma128) in its first 16 KB
    __nv_bfloat16 R1[2 * PAIR];  // [dU | dO] panels; dW in the dO rows
    __nv_bfloat16 R2[2 * PAIR];  // [K | Q]
    __nv_bfloat16 R3[2 * PAIR];  // [U | .]: U rows; sdPG in the other rows of panel 0, dMM in
                                 // those of panel 1
    // Swz<64> T; the MN-major T^T operands read the 8 KB after it (W) as their
    // unused rows 64..127
    __nv_bfloat16 T[C * C];
    __nv_bfloat16 W[C * DK];     // Tma128 image of W (two 64-key K-major panels)
    __nv_bfloat16 Ut[DV * C];    // Swz<64> image of U~^T (value rows x tokens)
    float Xs[C * C];             // transpose scratch for column sums (fp32, rotated columns)
    float G[2][C], beta[2][C];   // per chunk, alternating
    // Fixed-order partial sums (the dg and dbeta results are bit-reproducible):
    float pG[8][C];              // dG terms of a token's own rows, per (column group, lane half)
    float pB[4][C];              // dbeta terms, per column group
    float pC[8][C];              // column sums of hP and hA, per 8-row block
    float red[16], red2[16];     // per-warp sums: <dS, S0>; etl <dKt, k> (enters dG_last)
    float dgs[C];                // reverse-cumsum scratch
    // one load barrier per buffer group (one phase per chunk), one for the MMAs
    uint64_t bar_s, bar_ds, bar_u, bar_tq, bar_r1, bar_wu, bar_k, bar_v, bar_mma;
    uint32_t tmem;
};

struct BlPtrs {
    CUtensorMap qmap, kmap, vmap, dOmap;
    const float *g, *beta;
    const __nv_bfloat16 *v;
    const __nv_bfloat16 *S0, *U, *dS, *dU, *Tb, *W, *Ut;
    __nv_bfloat16 *dq, *dk, *dv;
    float *dg, *dbeta;
    unsigned int* status;
    int B, T, H, NT, nchunks;
    float scale;
    SeqMap seq;
};

// 32 consecutive TMEM columns of this thread's lane into v[0..31].
GDN_DEV void ld_row32(float* v, uint32_t taddr) {
    tc5::ld32(*reinterpret_cast<float(*)[32]>(v), taddr);
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

// The chunk of this CTA at or after c (grid stride) that holds tokens, or
// p.nchunks when none is left.
GDN_DEV int next_chunk(const BlPtrs& p, int c) {
    for (; c < p.nchunks; c += gridDim.x) {
        const int bh = c / p.NT;
        if (chunk_loc(p.seq, p.T, p.H, bh, c % p.NT).valid) break;
    }
    return c < p.nchunks ? c : p.nchunks;
}

struct BlChunk {
    int cid, h, tok, L;
    size_t row0;  // (first token of the chunk) * H + h
};

GDN_DEV BlChunk bl_chunk(const BlPtrs& p, int cid) {
    BlChunk c;
    c.cid = cid;
    const int bh = cid / p.NT;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, cid % p.NT);
    c.h = bh % p.H;
    c.tok = cl.tok;
    c.L = cl.L;
    c.row0 = (size_t)cl.tok * p.H + c.h;
    return c;
}

// Loads of one buffer group of chunk c (thread 0).
GDN_DEV void load_s0(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // S0
    mbar_arrive_expect(&s.bar_s, DV * DK * 2);
    bulk_g2s(s.R4, p.S0 + (size_t)c.cid * DV * DK, DV * DK * 2, &s.bar_s);
}
GDN_DEV void load_ds(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // dS
    mbar_arrive_expect(&s.bar_ds, DV * DK * 2);
    bulk_g2s(s.R5, p.dS + (size_t)c.cid * DV * DK, DV * DK * 2, &s.bar_ds);
}
GDN_DEV void load_u(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // U (rows 0..63 of R3)
    mbar_arrive_expect(&s.bar_u, C * DV * 2);
    bulk_g2s(s.R3, p.U + (size_t)c.cid * C * DV, C * 64 * 2, &s.bar_u);
    bulk_g2s(s.R3 + PAIR, p.U + (size_t)c.cid * C * DV + C * 64, C * 64 * 2, &s.bar_u);
}
GDN_DEV void load_tq(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // T, Q (rows 64..127 of R2)
    mbar_arrive_expect(&s.bar_tq, (C * C + C * DK) * 2);
    bulk_g2s(s.T, p.Tb + (size_t)c.cid * C * C, C * C * 2, &s.bar_tq);
    tma_load_3d(s.R2 + C * 64, &p.qmap, 0, c.h, c.tok, &s.bar_tq);
    tma_load_3d(s.R2 + PAIR + C * 64, &p.qmap, 64, c.h, c.tok, &s.bar_tq);
}
GDN_DEV void load_r1(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // dU, dO
    mbar_arrive_expect(&s.bar_r1, 2 * C * DV * 2);
    bulk_g2s(s.R1, p.dU + (size_t)c.cid * C * DV, C * 64 * 2, &s.bar_r1);
    bulk_g2s(s.R1 + PAIR, p.dU + (size_t)c.cid * C * DV + C * 64, C * 64 * 2, &s.bar_r1);
    tma_load_3d(s.R1 + C * 64, &p.dOmap, 0, c.h, c.tok, &s.bar_r1);
    tma_load_3d(s.R1 + PAIR + C * 64, &p.dOmap, 64, c.h, c.tok, &s.bar_r1);
}
GDN_DEV void load_wu(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // W, U~
    mbar_arrive_expect(&s.bar_wu, (C * DK + DV * C) * 2);
    bulk_g2s(s.W, p.W + (size_t)c.cid * C * DK, C * DK * 2, &s.bar_wu);
    bulk_g2s(s.Ut, p.Ut + (size_t)c.cid * DV * C, DV * C * 2, &s.bar_wu);
}
GDN_DEV void load_v(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // V (Tma128, in the dS space)
    mbar_arrive_expect(&s.bar_v, C * DV * 2);
    tma_load_3d(s.R5, &p.vmap, 0, c.h, c.tok, &s.bar_v);
    tma_load_3d(s.R5 + C * 64, &p.vmap, 64, c.h, c.tok, &s.bar_v);
}
GDN_DEV void load_k(BlSmem& s, const BlPtrs& p, const BlChunk& c) {  // K (rows 0..63 of R2)
    mbar_arrive_expect(&s.bar_k, C * DK * 2);
    tma_load_3d(s.R2, &p.kmap, 0, c.h, c.tok, &s.bar_k);
    tma_load_3d(s.R2 + PAIR, &p.kmap, 64, c.h, c.tok, &s.bar_k);
}
// The first buffers chunk c loads (U, S0, dS: 80 KB), into L2 a chunk ahead.
// The prefetches run on the TMA engine with the loads themselves; the rest of
// the chunk's buffers load late enough from DRAM (measured: prefetching the
// tiles and the other images as well is slower).
GDN_DEV void prefetch_chunk(const BlPtrs& p, const BlChunk& c) {
    bulk_prefetch_l2(p.U + (size_t)c.cid * C * DV, C * DV * 2);
    bulk_prefetch_l2(p.S0 + (size_t)c.cid * DV * DK, DV * DK * 2);
    bulk_prefetch_l2(p.dS + (size_t)c.cid * DV * DK, DV * DK * 2);
}

// G (within-chunk cumsum of g) and beta of chunk c into slot b (one warp).
GDN_DEV void load_gb(BlSmem& s, const BlPtrs& p, const BlChunk& c, int b) {
    const int lane = threadIdx.x & 31;
    const size_t rs = (size_t)p.H;
    float g0 = lane < c.L ? p.g[c.row0 + lane * rs] : 0.f;
    float g1 = lane + 32 < c.L ? p.g[c.row0 + (lane + 32) * rs] : 0.f;
    const float b0 = lane < c.L ? p.beta[c.row0 + lane * rs] : 0.f;
    const float b1 = lane + 32 < c.L ? p.beta[c.row0 + (lane + 32) * rs] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float x0 = __shfl_up_sync(0xffffffffu, g0, o);
        const float x1 = __shfl_up_sync(0xffffffffu, g1, o);
        if (lane >= o) { g0 += x0; g1 += x1; }
    }
    g1 += __shfl_sync(0xffffffffu, g0, 31);
    s.G[b][lane] = g0;
    s.G[b][lane + 32] = g1;
    s.beta[b][lane] = b0;
    s.beta[b][lane + 32] = b1;
}

// sum_{c < 32} x[c] * V[r][c0 + c] for row r of a Tma128 tile pair (two
// 64-column panels of 64 rows).
GDN_DEV float dot_tile32(const float* x, const __nv_bfloat16* V, int r, int c0) {
    const __nv_bfloat16* base = V + (c0 >> 6) * (C * 64);
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

// f * a[0..31] as bf16 to dst (this lane's row, 64 bytes at a 32-byte
// boundary) if ok.  Lanes 2i and 2i+1 hold neighbouring rows, pitch elements
// apart.  Each 32-byte sector is written by one instruction: the two lanes
// trade a 16-byte piece, so that in one store the pair writes both halves of
// the even row's sector and in the next both halves of the odd row's.  (A
// lane writing its own row alone fills every sector in two halves, which
// costs the store path twice.)  Called by all lanes of the warp.
GDN_DEV void store_row32(__nv_bfloat16* dst, size_t pitch, bool ok, const float* a, float f) {
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(f * a[2 * c], f * a[2 * c + 1]);
    const bool odd = threadIdx.x & 1;
    const bool pok = __shfl_xor_sync(0xffffffffu, ok, 1);
    __nv_bfloat16* const even_row = odd ? dst - pitch : dst;
    __nv_bfloat16* const odd_row = odd ? dst : dst + pitch;
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {  // sector hs: columns 16hs .. 16hs+15 (pieces 2hs, 2hs+1)
        uint32_t x[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) x[w] = __shfl_xor_sync(0xffffffffu, odd ? pk[8 * hs + w] : pk[8 * hs + 4 + w], 1);
        // the even row's sector: its piece 2hs from the even lane, 2hs+1 from the odd lane
        const uint4 ve = odd ? make_uint4(x[0], x[1], x[2], x[3])
                             : make_uint4(pk[8 * hs], pk[8 * hs + 1], pk[8 * hs + 2], pk[8 * hs + 3]);
        if (odd ? pok : ok) *reinterpret_cast<uint4*>(even_row + 16 * hs + (odd ? 8 : 0)) = ve;
        // the odd row's sector
        const uint4 vo = odd ? make_uint4(pk[8 * hs + 4], pk[8 * hs + 5], pk[8 * hs + 6], pk[8 * hs + 7])
                             : make_uint4(x[0], x[1], x[2], x[3]);
        if (odd ? ok : pok) *reinterpret_cast<uint4*>(odd_row + 16 * hs + (odd ? 8 : 0)) = vo;
    }
}

// Row t, columns c0..c0+31 (c0 a multiple of 32) of a pair region's panel, bf16.
GDN_DEV void put_pair_row32(__nv_bfloat16* R, int t, int c0, const float* a, float f) {
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(f * a[2 * c], f * a[2 * c + 1]);
    __nv_bfloat16* dst = R + (c0 >> 6) * PAIR;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint4*>(dst + swz<64>(t, (c0 & 63) + 8 * q4)) =
            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
}

// 32 fp32 values back into this thread's TMEM lane (two 16-column stores).
GDN_DEV void st_row32(uint32_t taddr, const float* a) {
    uint32_t r0[16], r1[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) { r0[c] = __float_as_uint(a[c]); r1[c] = __float_as_uint(a[16 + c]); }
    tc5::st16(taddr, r0);
    tc5::st16(taddr + 16, r1);
}

__global__ void __launch_bounds__(BL_THREADS, 1) tc5_bwd_local_kernel(const __grid_constant__ BlPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    BlSmem& s = *reinterpret_cast<BlSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int cid = next_chunk(p, blockIdx.x);
    if (cid >= p.nchunks) return;  // nothing for this CTA (before any barrier or TMEM)
    BlChunk ch = bl_chunk(p, cid);
    if (tid == 0) {
        mbar_init(&s.bar_s, 1);
        mbar_init(&s.bar_u, 1);
        mbar_init(&s.bar_ds, 1);
        mbar_init(&s.bar_tq, 1);
        mbar_init(&s.bar_r1, 1);
        mbar_init(&s.bar_wu, 1);
        mbar_init(&s.bar_k, 1);
        mbar_init(&s.bar_v, 1);
        mbar_init(&s.bar_mma, 1);
        fence_mbar_init();
        load_r1(s, p, ch);
        load_wu(s, p, ch);
        load_s0(s, p, ch);
        load_ds(s, p, ch);
        load_u(s, p, ch);
        load_k(s, p, ch);
        load_tq(s, p, ch);
    }
    if (warp == 0) {
        tc5::alloc(&s.tmem, BL_TCOLS);
        load_gb(s, p, ch, 0);
    }
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
    const size_t rs = (size_t)p.H;
    __nv_bfloat16* sdPG = s.R3 + C * 64;         // scale dP .* Gamma (Swz<64>), panel 0 rows 64..127
    __nv_bfloat16* dMM = s.R3 + PAIR + C * 64;   // dMM (Swz<64>), panel 1 rows 64..127
    float* Xs = s.Xs;
    uint32_t mph = 0;  // phase of bar_mma
    bool ok = true;
    // The next chunk's loads are issued by a lane of warp 2, whose epilogue
    // share is light or empty where they go out (thread 0 issues the MMAs).
    const bool loader = warp == 2 && lane == 0;
    for (int it = 0;; ++it) {
        const uint32_t lp = it & 1;  // phase of the load barriers for this chunk
        const int L = ch.L;
        const size_t row0 = ch.row0;
        const float* G = s.G[it & 1];
        const float* beta = s.beta[it & 1];
        const float Gl = G[C - 1];
        const int ncid = next_chunk(p, cid + gridDim.x);
        const bool has_next = ncid < p.nchunks;
        const BlChunk nch = bl_chunk(p, has_next ? ncid : cid);
        float myG = 0.f, myB = 0.f;  // this thread's (token, column group) share of dG / dbeta
        float myC = 0.f;             // this thread's (column, row block) share of the column sums
        if (loader && has_next) prefetch_chunk(p, nch);
        if (warp == 2 && has_next) {  // the next chunk's g and beta rows, into L2
            for (int t = lane; t < nch.L; t += 32) {
                prefetch_l2(p.g + nch.row0 + (size_t)t * rs);
                prefetch_l2(p.beta + nch.row0 + (size_t)t * rs);
            }
        }
        if (tid < 16) s.red2[tid] = 0.f;
        ok = mbar_wait(&s.bar_r1, lp, p.status) && mbar_wait(&s.bar_s, lp, p.status) &&
             mbar_wait(&s.bar_ds, lp, p.status) &&
             mbar_wait(&s.bar_u, lp, p.status) && mbar_wait(&s.bar_tq, lp, p.status);
        if (__syncthreads_or(!ok)) break;
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
        // ---- phase A: every product of the loaded tiles --------------------------------
        bool kfail = false;
        if (tid == 0) {
            tc5::fence_after();
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk)  // [dU ; dO] S0 -> [-dW ; dO S0]
                tc5::mma(tm + TA, tc5::kmajor<128>(sR1, kk), tc5::mnmajor(sR4, kk, 128 * 128), ID_N128_BMN,
                         kk > 0);
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk)  // [U ; .] dS
                tc5::mma(tm + TB, tc5::kmajor<128>(sR3, kk), tc5::mnmajor(sR5, kk, 128 * 128), ID_N128_BMN,
                         kk > 0);
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk)  // [dU ; dO] U^T
                tc5::mma(tm + TC2, tc5::kmajor<128>(sR1, kk), tc5::kmajor<128>(sR3, kk), ID_N64, kk > 0);
            if (mbar_wait(&s.bar_k, lp, p.status)) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)  // [K ; Q] K^T
                    tc5::mma(tm + TC1, tc5::kmajor<128>(sR2, kk), tc5::kmajor<128>(sR2, kk), ID_N64, kk > 0);
            } else {
                kfail = true;
            }
            tc5::commit(&s.bar_mma);
        }
        {   // <dS, S0> under the products (both are only read until the next chunk's loads),
            // by warps 1..15: warp 0 holds the thread that issues the products
            float ss = 0.f;
            for (int e = tid - 32; warp > 0 && e < DV * DK / 8; e += BL_THREADS - 32) {
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
        fence_async_smem();
        ok = mbar_wait(&s.bar_mma, mph, p.status);
        mph ^= 1;
        if (__syncthreads_or(!ok || kfail)) break;
        tc5::fence_after();
        // S0 and U are done with: this chunk's V, the next chunk's U
        if (loader) {
            load_v(s, p, ch);
            if (has_next) {
                load_u(s, p, nch);
                load_s0(s, p, nch);
            }
        }
        // ---- epilogue A --------------------------------------------------------------
        if (q >= 2) {
            // token i: dP, Q K^T (columns 16cg..) -> sdPG and hP; dq accumulator
            // (columns 32cg..) *= scale e^{G_i}, and <scale e^{G_i} dO S0 row i, q_i>
            const int i = row;
            const float Gi = G[i], fi = p.scale * __expf(Gi);
            float dp[16], qk[16], x[32];
            tc5::ld16(dp, trow + TC2 + 16 * cg);
            tc5::ld16(qk, trow + TC1 + 16 * cg);
            ld_row32(x, trow + TA + 32 * cg);
            tc5::wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] *= fi;
            st_row32(trow + TA + 32 * cg, x);
            float hrow = 0.f;
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int j = 16 * cg + c;
                const float g = j <= i ? p.scale * dp[c] * __expf(Gi - G[j]) : 0.f;  // scale dP .* Gamma
                const float hp = g * qk[c];                    // dP .* (scale Q K^T .* Gamma)
                hrow += hp;
                Xs[i * 64 + ((j + i) & 63)] = hp;              // column sums below
                dp[c] = g;
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) pk[c] = pack_bf16(dp[2 * c], dp[2 * c + 1]);
            *reinterpret_cast<uint4*>(sdPG + swz<64>(i, 16 * cg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(sdPG + swz<64>(i, 16 * cg + 8)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            const float dqq = dot_row32(x, s.R2, C + i, 32 * cg);
            myG += hrow + dqq;
        } else {
            // token t: -dW (columns 32cg..) -> dW (bf16, into the dO rows of R1); the dk
            // accumulator (U dS, columns 32cg..) *= etl_t, and <etl dKt row t, k_t>
            const int t = row;
            float x[32], y[32];
            ld_row32(x, trow + TA + 32 * cg);
            ld_row32(y, trow + TB + 32 * cg);
            tc5::wait_ld();
            const float et = __expf(Gl - G[t]);
#pragma unroll
            for (int c = 0; c < 32; ++c) y[c] *= et;
            st_row32(trow + TB + 32 * cg, y);
            put_pair_row32(s.R1 + C * 64, t, 32 * cg, x, -1.f);
            float hk = dot_row32(y, s.R2, t, 32 * cg);
            myG -= hk;  // -etl_t <dKt_t, k_t>; the same enters dG_last
            hk = warp_sum(hk);
            if (lane == 0) s.red2[warp] = hk;
        }
        tc5::wait_st();
        fence_async_smem();
        tc5::fence_before();
        __syncthreads();
        // ---- phase E1: Gk = T^T dW, Gv = T^T dU; dq += [. ; sdPG] K; dk += sdPG^T Q
        if (tid == 0) {
            tc5::fence_after();
            const uint32_t ssdPG = smem_u32(sdPG);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc5::mma(tm + TKG, tc5::mnmajor(sT, kk, C * 128), tc5::mnmajor(sR1 + C * 128, kk, PB),
                         ID_N128_AMN_BMN, kk > 0);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc5::mma(tm + TVB, tc5::mnmajor(sT, kk, C * 128), tc5::mnmajor(sR1, kk, PB), ID_N128_AMN_BMN,
                         kk > 0);
            // (rows 0..63 of this A view are the 8 KB before sdPG)
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc5::mma(tm + TA, tc5::kmajor<128>(ssdPG - C * 128, kk), tc5::mnmajor(sR2, kk, PB), ID_N128_BMN,
                         true);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc5::mma(tm + TB, tc5::mnmajor(ssdPG, kk, C * 128), tc5::mnmajor(sR2 + C * 128, kk, PB),
                         ID_N128_AMN_BMN, true);
            tc5::commit(&s.bar_mma);
        }
        {   // column sums of hP (under the E1 products): dG_j -= sum_i hP_ij (eight row
            // blocks per column)
            const int j = tid & 63, pb = tid >> 6;
#pragma unroll
            for (int i = 8 * pb; i < 8 * pb + 8; ++i) myC -= Xs[i * 64 + ((j + i) & 63)];
        }
        ok = mbar_wait(&s.bar_mma, mph, p.status);
        mph ^= 1;
        if (__syncthreads_or(!ok)) break;
        tc5::fence_after();
        if (loader && has_next) {  // T, Q, dU and dO are done with
            load_tq(s, p, nch);
            load_r1(s, p, nch);
        }
        // ---- epilogue E1: Gk, Gv -> bf16 A operands in TMEM (lanes 0..63 of TA); dv;
        // <Gk_t, k_t>, <Gv_t, v_t>; dq (complete after E1) -----------------------------
        if (q < 2) {
            const int t = row;
            const float bt = beta[t], egt = __expf(G[t]);
            float gk[32], gv[32];
            ld_row32(gk, trow + TKG + 32 * cg);
            ld_row32(gv, trow + TVB + 32 * cg);
            tc5::wait_ld();
            const float hk = dot_row32(gk, s.R2, t, 32 * cg);
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(gk[2 * c], gk[2 * c + 1]);
            tc5::st16(trow + TA + 16 * cg, pk);
#pragma unroll
            for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(gv[2 * c], gv[2 * c + 1]);
            tc5::st16(trow + TA + 64 + 16 * cg, pk);
            store_row32(p.dv + (row0 + (size_t)t * rs) * DV + 32 * cg, rs * DV, t < L, gv, bt);
            const bool vok = mbar_wait(&s.bar_v, lp, p.status);
            const float hv = vok ? dot_tile32(gv, s.R5, t, 32 * cg) : 0.f;
            ok = ok && vok;
            myB += egt * hk + hv;
            myG += bt * egt * hk;
        } else {
            const int i = row;
            float a[32];
            ld_row32(a, trow + TA + 32 * cg);
            tc5::wait_ld();
            store_row32(p.dq + (row0 + (size_t)i * rs) * DK + 32 * cg, rs * DK, i < L, a, 1.f);
        }
        tc5::wait_st();
        fence_async_smem();  // the V reads above, before the next chunk's S0 lands there
        tc5::fence_before();
        ok = ok && mbar_wait(&s.bar_wu, lp, p.status);
        if (__syncthreads_or(!ok)) break;
        if (loader && has_next) load_ds(s, p, nch);  // V (in the dS space) is done with
        // ---- phase C: [Gk ; .] W^T + [Gv ; .] U~^T = T^T dT T^T (A from TMEM); [K ; .] K^T
        if (tid == 0) {
            tc5::fence_after();
            const uint32_t sW = smem_u32(s.W), sUt = smem_u32(s.Ut);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                tc5::mma_ts(tm + TD, tm + TA + 8 * kk, tc5::kmajor<C>(sW, kk), ID_N64, kk > 0);
#pragma unroll
            for (int kk = 0; kk < DV / 16; ++kk)
                tc5::mma_ts(tm + TD, tm + TA + 64 + 8 * kk, tc5::mnmajor(sUt, kk, C * 128), ID_N64_BMN, true);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                tc5::mma(tm + TKK, tc5::kmajor<128>(sR2, kk), tc5::kmajor<128>(sR2, kk), ID_N64, kk > 0);
            tc5::commit(&s.bar_mma);
        }
        ok = mbar_wait(&s.bar_mma, mph, p.status);
        mph ^= 1;
        if (__syncthreads_or(!ok)) break;
        tc5::fence_after();
        if (loader && has_next) load_wu(s, p, nch);  // W and U~ are done with
        // ---- epilogue D: dA = strict_lower(-(Gk W^T + Gv U~^T)); M = K K^T .* Gamma;
        // dMM; hA; dbeta and dG terms --------------------------------------------------
        if (q < 2) {
            const int i = row;
            const float Gi = G[i], bi = beta[i];
            float x[16], kk[16];
            tc5::ld16(x, trow + TD + 16 * cg);
            tc5::ld16(kk, trow + TKK + 16 * cg);
            tc5::wait_ld();
            float hrow = 0.f, brow = 0.f;
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int j = 16 * cg + c;
                const float gam = j < i ? __expf(Gi - G[j]) : 0.f;
                const float dA = j < i ? -x[c] : 0.f;
                const float m = kk[c] * gam;  // K K^T .* Gamma (strict lower)
                brow += dA * m;
                const float hA = dA * bi * m;
                hrow += hA;
                Xs[i * 64 + ((j + i) & 63)] = hA;
                x[c] = dA * bi * gam;  // dMM
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
        // ---- phase E2: dk += dMM K + dMM^T K ---------------------------------------------
        if (tid == 0) {
            tc5::fence_after();
            const uint32_t sdMM = smem_u32(dMM);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc5::mma(tm + TB, tc5::kmajor<128>(sdMM, kk), tc5::mnmajor(sR2, kk, PB), ID_N128_BMN, true);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                tc5::mma(tm + TB, tc5::mnmajor(sdMM, kk, C * 128), tc5::mnmajor(sR2, kk, PB), ID_N128_AMN_BMN,
                         true);
            tc5::commit(&s.bar_mma);
        }
        {   // column sums of hA (under the E2 products): dG_j -= sum_i hA_ij
            const int j = tid & 63, pb = tid >> 6;
#pragma unroll
            for (int i = 8 * pb; i < 8 * pb + 8; ++i) myC -= Xs[i * 64 + ((j + i) & 63)];
        }
        ok = mbar_wait(&s.bar_mma, mph, p.status);
        mph ^= 1;
        if (__syncthreads_or(!ok)) break;
        tc5::fence_after();
        if (loader && has_next) load_k(s, p, nch);  // K is done with
        // ---- epilogue E2: dk = TB + beta e^G .* Gk; the next chunk's G and beta ----------
        if (q < 2) {
            const int t = row;
            const float f = beta[t] * __expf(G[t]);
            float a[32], kg[32];
            ld_row32(a, trow + TB + 32 * cg);
            ld_row32(kg, trow + TKG + 32 * cg);
            tc5::wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) a[c] = fmaf(f, kg[c], a[c]);
            store_row32(p.dk + (row0 + (size_t)t * rs) * DK + 32 * cg, rs * DK, t < L, a, 1.f);
        } else if (warp == 2 && has_next) {
            load_gb(s, p, nch, (it + 1) & 1);
        }
        // ---- per-token sums in a fixed order: dG (own-row terms + column terms),
        // dbeta; dg = reverse cumsum of dG ------------------------------------------------
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
        __syncthreads();  // the sums' scratch and this chunk's G are free
        if (!has_next) break;
        cid = ncid;
        ch = nch;
    }
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
    lp.g = cp.g; lp.beta = cp.beta; lp.v = cp.v; lp.status = cp.status;
    lp.S0 = (const __nv_bfloat16*)(base + L.S0);
    lp.U = (const __nv_bfloat16*)(base + L.U);
    lp.dS = (const __nv_bfloat16*)(base + L.dS);
    lp.dU = (const __nv_bfloat16*)(base + L.dU);
    lp.Tb = cp.Tb;
    lp.W = cp.W; lp.Ut = cp.Ut;
    lp.dq = (__nv_bfloat16*)dq; lp.dk = (__nv_bfloat16*)dk; lp.dv = (__nv_bfloat16*)dv;
    lp.dg = dg; lp.dbeta = dbeta;
    lp.B = d.B; lp.T = d.T; lp.H = d.H; lp.NT = L.NT; lp.scale = d.scale;
    lp.nchunks = (int)L.nchunks;
    lp.seq = cp.seq;
    if (L.nchunks == 0) return true;
    // persistent: one CTA per SM, each taking every gridDim.x-th chunk
    const unsigned grid = (unsigned)std::min<size_t>(L.nchunks, (size_t)sm_count());
    const int smem = sizeof(BlSmem) + 1024;
    cudaFuncSetAttribute(tc5_bwd_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_bwd_local", st, tc5_bwd_local_kernel<<<grid, BL_THREADS, smem, st>>>(lp));
    return true;
}
}  // namespace tc
}  // namespace gdn
