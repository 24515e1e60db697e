// tc5_prep.cu -- per-chunk WY preparation of the gated delta rule on the
// fifth-generation tensor cores (scalar gate, bf16, dk = dv = 128, chunk 64).
//
// For one chunk of one head, with G the within-chunk cumsum of the log-gate
// ("Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper review),
// section "Method": the gated delta rule in its chunkwise WY / UT-transform
// form):
//   A  = strict_lower(diag(beta) (K K^T .* D)),  D_ij = exp(G_i - G_j)
//   T  = (I + A)^{-1}                                 (UT transform)
//   W  = T (diag(beta e^G) K),   U~ = T (diag(beta) V)
//   P  = scale lower(Q K^T .* D)
// The products run as tcgen05 MMAs with fp32 accumulators in tensor memory:
//   [K K^T ; Q K^T] = [K ; Q] K^T           one M = 128, N = 64 product: rows
//                                           0..63 give A, rows 64..127 give P
//   W^T  = (beta e^G K)^T T^T               M = 128 (key), N = 64 (token)
//   U~^T = (beta V)^T T^T                   M = 128 (value), N = 64 (token)
// with K and Q stacked in one K-major operand (the TMA tiles of both land in
// the same 128-row panels), and the transposed products reading the K and V
// tiles as MN-major A operands, so no tile is copied or transposed in shared
// memory.  The row scales beta e^G of W and beta of U~ are applied to the K
// and V tiles in place once Q K^T and K K^T are done, so both transposed
// products share the B operand T.
// The triangular solve is the shared UT transform of tc5_solve.cuh.
//
// One CTA of eight warps per chunk; warps w and w + 4 share TMEM lane
// quarter w: in the first epilogue they split a row's columns, in the second
// one takes W^T and the other U~^T.
// Shared memory 74 KB and 128 TMEM columns, so three CTAs share an SM.
// Outputs (bulk stores into the workspace): the W image (Tma128), the U~^T
// image (Swz<64>, 128 value rows), P (Swz<64>), G, and optionally T (Swz<64>);
// the K~ = diag(e^{G_last - G}) K image (Tma128) goes out with plain 16-byte
// stores straight from the K tile, four whole 128-byte rows per warp store.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc5_solve.cuh"
#include "tc_common.cuh"

namespace gdn {
namespace {
using namespace tc;

constexpr int P5_THREADS = 256;  // warp w: TMEM lane quarter w % 4, column half w / 4
constexpr uint32_t P5_TCOLS = 128;  // D1 = [KK^T; QK^T] in 0..63; then W^T 0..63, U~^T 64..127
constexpr uint32_t ID_KQ = tc5::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_WU = tc5::idesc_bf16(128, 64, true, false);
constexpr int KQ_PANEL = 2 * C * 64;  // elements of one 128-row, 64-column panel

struct alignas(1024) P5Smem {
    // [K p0 | Q p0 | K p1 | Q p1], 8 KB each: panel p holds key columns 64p..64p+63
    // of the 64 K rows then the 64 Q rows.  Once the first product is done the
    // Q quarters hold the bf16 A (Swz<64>) and the fp32 diagonal blocks of A
    // with the solve's scratch; once the transposed products are done the
    // whole region holds the W image (16 KB) and the U~^T image (16 KB).
    __nv_bfloat16 KQ[2 * KQ_PANEL];
    __nv_bfloat16 V[C * DV];  // Tma128
    __nv_bfloat16 P[C * C];   // Swz<64>
    __nv_bfloat16 T[C * C];   // Swz<64>: T = (I + A)^{-1}
    float G[C];
    float beta[C];
    uint64_t bar_ld, bar_mma;
    uint32_t tmem;
};

// The q/k/v prologue of the block design ("Gated Delta Networks: Improving
// Mamba2 with Delta Rule" (paper review), section "Method": a short causal
// depthwise convolution, SiLU, and for q and k an L2 norm over the head's
// channels), applied in place to a raw 64-token tile in shared memory:
//   z_t[c] = sum_{j<K} w[h, c, j] x_{t-j}[c],  s = z sigmoid(z),
//   y = s / sqrt(sum_c s_c^2 + 1e-6)  (norm), else y = s.
// The tile's own raw rows give the history of its rows 3..63; the 3 rows
// before the chunk (zero at a sequence's first chunk) and the filter, 4 taps
// per channel (zero past K), were staged in shared memory while the tiles
// loaded.  Thread (row, 8-channel group); the norm's sum is a 16-lane
// reduction.  The caller reads every raw row of a tile (results in registers
// as bf16 pairs) before any is overwritten.
// Filtered rows of one tile into res (bf16 pairs): compute only, no write.
template <typename Off>
GDN_DEV void conv_rows(uint4 (&res)[4], const __nv_bfloat16* tile, Off off, const __nv_bfloat16* hal,
                       const float* wsm, int K, bool norm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = 8 * (lane & 15);
    float wr[8][4];  // [channel][tap]; wsm is [tap][channel]: a half-warp reads 512 contiguous bytes
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 a = *reinterpret_cast<const float4*>(wsm + j * DK + c0);
        const float4 b = *reinterpret_cast<const float4*>(wsm + j * DK + c0 + 4);
        wr[0][j] = a.x; wr[1][j] = a.y; wr[2][j] = a.z; wr[3][j] = a.w;
        wr[4][j] = b.x; wr[5][j] = b.y; wr[6][j] = b.z; wr[7][j] = b.w;
    }
#pragma unroll
    for (int ps = 0; ps < 4; ++ps) {
        const int r = 16 * ps + 2 * warp + (lane >> 4);
        float z[8] = {};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j >= K) break;
            const int rr = r - j;  // tile row of tap j
            const uint4 v = rr >= 0 ? *reinterpret_cast<const uint4*>(tile + off(rr, c0))
                                    : *reinterpret_cast<const uint4*>(hal + (3 + rr) * DK + c0);
            const uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = unpack_bf16(e[i]);
                z[2 * i] = fmaf(wr[2 * i][j], f.x, z[2 * i]);
                z[2 * i + 1] = fmaf(wr[2 * i + 1][j], f.y, z[2 * i + 1]);
            }
        }
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            z[i] = __fdividef(z[i], 1.f + __expf(-z[i]));
            ss += z[i] * z[i];
        }
        if (norm) {
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float inv = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int i = 0; i < 8; ++i) z[i] *= inv;
        }
        res[ps] = make_uint4(pack_bf16(z[0], z[1]), pack_bf16(z[2], z[3]), pack_bf16(z[4], z[5]),
                             pack_bf16(z[6], z[7]));
    }
}
// ... and their write-back into the tile and, for rows below L, to `out`.
template <typename Off>
GDN_DEV void conv_store(const uint4 (&res)[4], __nv_bfloat16* tile, Off off, __nv_bfloat16* out,
                        size_t row0, size_t rs, int L) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = 8 * (lane & 15);
#pragma unroll
    for (int ps = 0; ps < 4; ++ps) {
        const int r = 16 * ps + 2 * warp + (lane >> 4);
        *reinterpret_cast<uint4*>(tile + off(r, c0)) = res[ps];
        if (r < L) *reinterpret_cast<uint4*>(out + (row0 + (size_t)r * rs) * DK + c0) = res[ps];
    }
}

template <bool CONV>
__global__ void __launch_bounds__(P5_THREADS, 3) tc5_prep_kernel(const __grid_constant__ ChunkPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    P5Smem& s = *reinterpret_cast<P5Smem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, h = bh % p.H;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, n);
    if (!cl.valid) return;  // past the last chunk of a packed batch
    const int L = cl.L;
    const size_t row0 = (size_t)cl.tok * p.H + h;  // token-head index of row 0
    const size_t rs = (size_t)p.H;                 // token-head stride between rows

    if (tid == 0) {
        mbar_init(&s.bar_ld, 1);
        mbar_init(&s.bar_mma, 1);
        fence_mbar_init();
        // rows past L hold the next sequence's tokens (or zeros past the
        // tensor): finite, and annihilated by beta = 0 on those rows
        mbar_arrive_expect(&s.bar_ld, 3 * C * DK * 2);
        tma_load_3d(s.KQ, &p.kmap, 0, h, cl.tok, &s.bar_ld);
        tma_load_3d(s.KQ + C * 64, &p.qmap, 0, h, cl.tok, &s.bar_ld);
        tma_load_3d(s.KQ + KQ_PANEL, &p.kmap, 64, h, cl.tok, &s.bar_ld);
        tma_load_3d(s.KQ + KQ_PANEL + C * 64, &p.qmap, 64, h, cl.tok, &s.bar_ld);
        tma_load_tile(s.V, &p.vmap, h, cl.tok, &s.bar_ld);
    }
    if constexpr (CONV) {
        // the filters [tensor][tap][channel] fp32 in P's space and the 3
        // rows before the chunk [tensor][row][channel] bf16 in T's (both free
        // until the first epilogue), while the tiles load
        float* wsm = reinterpret_cast<float*>(s.P);
        __nv_bfloat16* hal = s.T;
        for (int e = tid; e < 3 * DK; e += P5_THREADS) {
            const int t = e / DK, c = e % DK;
            const float* src = (t == 0 ? p.conv.wk : t == 1 ? p.conv.wq : p.conv.wv) + ((size_t)h * DK + c) * p.conv.K;
#pragma unroll
            for (int j = 0; j < 4; ++j) wsm[(t * 4 + j) * DK + c] = j < p.conv.K ? src[j] : 0.f;
        }
        const int halo = n > 0 ? 3 : 0;  // a dense batch: one sequence per row b
        for (int e = tid; e < 3 * 3 * 16; e += P5_THREADS) {
            const int t = e / 48, j = (e / 16) % 3, c = 8 * (e % 16);  // row j: token tok - 3 + j
            uint4 v = make_uint4(0, 0, 0, 0);
            const __nv_bfloat16* xs = t == 0 ? p.conv.xk : t == 1 ? p.conv.xq : p.conv.xv;
            if (3 - j <= halo) v = *reinterpret_cast<const uint4*>(xs + (row0 - (size_t)(3 - j) * rs) * DK + c);
            *reinterpret_cast<uint4*>(hal + (t * 3 + j) * DK + c) = v;
        }
    }
    if (warp == 0) {
        tc5::alloc(&s.tmem, P5_TCOLS);
        // inclusive cumsum of the log-gate over the chunk (rows past L add 0)
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
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;
    const uint32_t sKQ = smem_u32(s.KQ);
    bool ok = true;

    if constexpr (CONV) {  // the tiles are raw projections: filter them in place
        ok = mbar_wait(&s.bar_ld, 0, p.status);
        if (__syncthreads_or(!ok)) goto done;
        const float* wsm = reinterpret_cast<const float*>(s.P);
        auto offk = [](int r, int c) { return (c >> 6) * KQ_PANEL + swz<64>(r, c & 63); };
        auto offq = [](int r, int c) { return (c >> 6) * KQ_PANEL + swz<64>(C + r, c & 63); };
        auto offv = [](int r, int c) { return (c >> 6) * (C * 64) + swz<64>(r, c & 63); };
        uint4 rr[4];  // a tile's raw rows are all read before any is overwritten
        conv_rows(rr, s.KQ, offk, s.T, wsm, p.conv.K, true);
        __syncthreads();
        conv_store(rr, s.KQ, offk, p.conv.kf, row0, rs, L);
        conv_rows(rr, s.KQ, offq, s.T + 3 * DK, wsm + 4 * DK, p.conv.K, true);
        __syncthreads();
        conv_store(rr, s.KQ, offq, p.conv.qf, row0, rs, L);
        conv_rows(rr, s.V, offv, s.T + 6 * DK, wsm + 8 * DK, p.conv.K, false);
        __syncthreads();
        conv_store(rr, s.V, offv, p.conv.vf, row0, rs, L);
        fence_async_smem();  // filtered tiles (generic writes) -> tensor-core reads
        tc5::fence_before();
        __syncthreads();
    }
    if (!CONV) {
        ok = mbar_wait(&s.bar_ld, 0, p.status);
        if (__syncthreads_or(!ok)) goto done;
    }
    // ---- [K K^T ; Q K^T] ---------------------------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm, tc5::kmajor<2 * C>(sKQ, kk), tc5::kmajor<2 * C>(sKQ, kk), ID_KQ, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    // ---- under the product: K~ = diag(e^{G_last - G}) K to the workspace (the
    // walks' B of the state update) from the K tile as loaded, and V <- diag(beta) V
    // in place (the row scale of U~; V is not read before the second product)
    if (tid < 128) {  // threads 0..127: K~ rows; 128..255: V rows
        // 16-byte piece e = tid + 128 it of the image: piece e & 7 of row e >> 4,
        // panel (e >> 3) & 1, so that every warp store writes four whole 128-byte
        // rows (a thread writing a row piece by piece fills each 32-byte sector
        // in two halves)
        __nv_bfloat16* kt = p.Kt + (size_t)cid * C * DK;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int e = tid + 128 * it, j = e & 7, pn = (e >> 3) & 1, r = e >> 4;
            const float dec = __expf(s.G[C - 1] - s.G[r]);
            // same swizzled position in the Tma128 image (panel pn at pn * 4096)
            const uint4 x = *reinterpret_cast<const uint4*>(s.KQ + pn * KQ_PANEL + r * 64 + 8 * j);
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            uint32_t wt[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f2 = unpack_bf16(w[i]);
                wt[i] = pack_bf16(f2.x * dec, f2.y * dec);
            }
            *reinterpret_cast<uint4*>(kt + pn * (C * 64) + r * 64 + 8 * j) = make_uint4(wt[0], wt[1], wt[2], wt[3]);
        }
    } else {
        const int r = (tid - 128) >> 1, pn = tid & 1;
        const float b = s.beta[r];
        __nv_bfloat16* vrow = s.V + pn * (C * 64) + r * 64;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const int j = (jj + r) & 7;
            uint4 x = *reinterpret_cast<uint4*>(vrow + 8 * j);
            uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f2 = unpack_bf16(w[i]);
                w[i] = pack_bf16(f2.x * b, f2.y * b);
            }
            *reinterpret_cast<uint4*>(vrow + 8 * j) = x;
        }
    }
    ok = mbar_wait(&s.bar_mma, 0, p.status);
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();

    // Q is dead: its first quarter holds the bf16 A, its second the fp32
    // diagonal blocks of A and each warp's 16x16 scratch of the solve.
    {
        __nv_bfloat16* Abf = s.KQ + C * 64;
        auto Ad = reinterpret_cast<float(*)[16][17]>(s.KQ + KQ_PANEL + C * 64);
        auto Xs = reinterpret_cast<__nv_bfloat16(*)[16 * 16]>(
            reinterpret_cast<unsigned char*>(s.KQ + KQ_PANEL + C * 64) + 4 * 16 * 17 * sizeof(float));

        // ---- epilogue 1: row r of [K K^T ; Q K^T] (TMEM lane), columns
        // 32 hf .. +31, two threads per row ----------------------------------
        {
            const int ql = warp & 3, hf = warp >> 2, lr = 32 * ql + lane;
            const uint32_t trow = tm + ((uint32_t)(32 * ql) << 16);
            const bool is_a = lr < C;
            const int r = is_a ? lr : lr - C, c0 = 32 * hf;
            float v[32];
            // rows 0..31 have their columns 32.. masked: no load, no exponentials
            const bool live = (ql & 1) || hf == 0;
            if (live) {
                tc5::ld32(v, trow + c0);
                tc5::wait_ld();
                const float Gr = s.G[r];
                // A row r: beta_r (k_r . k_c) e^{G_r - G_c} for c < r;
                // P row r: scale (q_r . k_c) e^{G_r - G_c} for c <= r (rows past L zero)
                const float f = is_a ? s.beta[r] : (r < L ? p.scale : 0.f);
                const int lim = is_a ? r : r + 1;
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] = (c0 + c < lim) ? f * v[c] * __expf(Gr - s.G[c0 + c]) : 0.f;
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] = 0.f;
            }
            __nv_bfloat16* dst = is_a ? Abf : s.P;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(dst + swz<C>(r, c0 + 8 * j)) =
                    make_uint4(pack_bf16(v[8 * j], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                               pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
            if (is_a && (r >> 5) == hf) {  // the row's diagonal 16x16 block of A, exact in fp32
                float* ad = &Ad[r >> 4][r & 15][0];
                if (r & 16) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) ad[c] = v[16 + c];
                } else {
#pragma unroll
                    for (int c = 0; c < 16; ++c) ad[c] = v[c];
                }
            }
        }
        fence_async_smem();  // P (generic writes) -> its bulk store
        tc5::fence_before();
        __syncthreads();
        if (tid == 0) {  // P and G are final: out now, under the solve
            bulk_s2g(p.P + (size_t)cid * C * C, s.P, C * C * 2);
            bulk_s2g(p.G + (size_t)cid * C, s.G, C * 4);
            bulk_commit();
        }

        // ---- K <- diag(beta e^G) K in place (the row scale of W): thread =
        // (row, quarter of the row's 128 channels)
        {
            const int r = tid >> 2, qc = tid & 3, pn = qc >> 1;
            const float e = s.beta[r] * __expf(s.G[r]);
            __nv_bfloat16* row = s.KQ + pn * KQ_PANEL + r * 64;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * (qc & 1) + ((jj + r) & 3);  // rotated order within the half row
                uint4 x = *reinterpret_cast<uint4*>(row + 8 * j);
                uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f2 = unpack_bf16(w[i]);
                    w[i] = pack_bf16(f2.x * e, f2.y * e);
                }
                *reinterpret_cast<uint4*>(row + 8 * j) = x;
            }
        }

        // ---- UT transform: T = (I + A)^{-1} ---------------------------------
        ut_solve(Ad, Abf, s.T, Xs);
    }

    // ---- W^T = (beta e^G K)^T T^T ; U~^T = (beta V)^T T^T -----------------------
    fence_async_smem();  // scaled K, V and T (generic writes) -> tensor-core reads
    tc5::fence_before();
    __syncthreads();
    if (tid == 0) {
        if (p.Tb) {  // T is final: out now, under the second product
            bulk_s2g(p.Tb + (size_t)cid * C * C, s.T, C * C * 2);
            bulk_commit();
        }
        tc5::fence_after();
        const uint32_t sT = smem_u32(s.T), sV = smem_u32(s.V);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm, tc5::mnmajor(sKQ, kk, KQ_PANEL * 2), tc5::kmajor<C>(sT, kk), ID_WU, kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + 64, tc5::mnmajor(sV, kk, C * 128), tc5::kmajor<C>(sT, kk), ID_WU, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, 1, p.status);
    if (__syncthreads_or(!ok)) goto done;
    tc5::fence_after();

    // ---- epilogue 2: warps 0..3 key rows of W^T, warps 4..7 value rows of U~^T
    {
        __nv_bfloat16* Wimg = s.KQ;             // Tma128, 16 KB
        __nv_bfloat16* Uimg = s.KQ + C * DK;    // Swz<64>, 128 rows x 64 tokens
        const int ql = warp & 3, row = 32 * ql + lane;
        const uint32_t trow = tm + ((uint32_t)(32 * ql) << 16);
        float x[32];
        if (warp < 4) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc5::ld32(x, trow + 32 * half);
                tc5::wait_ld();
#pragma unroll
                for (int t = 0; t < 32; ++t) Wimg[Tma128::off(32 * half + t, row)] = __float2bfloat16_rn(x[t]);
            }
        } else {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc5::ld32(x, trow + 64 + 32 * half);
                tc5::wait_ld();
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4*>(Uimg + swz<C>(row, 32 * half + 8 * j)) =
                        make_uint4(pack_bf16(x[8 * j], x[8 * j + 1]), pack_bf16(x[8 * j + 2], x[8 * j + 3]),
                                   pack_bf16(x[8 * j + 4], x[8 * j + 5]), pack_bf16(x[8 * j + 6], x[8 * j + 7]));
            }
        }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_s2g(p.W + (size_t)cid * C * DK, s.KQ, C * DK * 2);
        bulk_s2g(p.Ut + (size_t)cid * C * DV, s.KQ + C * DK, C * DV * 2);
        bulk_commit();
        bulk_wait_read<0>();
    }
done:
    tc5::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc5::fence_after();
        tc5::dealloc(tm, P5_TCOLS);
    }
}

}  // namespace

namespace tc {
void launch_prep5(const ChunkPtrs& p, size_t nchunks, cudaStream_t st) {
    const int smem = sizeof(P5Smem) + 1024;
    cudaFuncSetAttribute(tc5_prep_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_prep", st, tc5_prep_kernel<false><<<(unsigned)nchunks, P5_THREADS, smem, st>>>(p));
}
// The preparation with the q/k/v prologue fused into its load stage (p.conv set,
// the token maps over the raw projections).
void launch_prep5_conv(const ChunkPtrs& p, size_t nchunks, cudaStream_t st) {
    const int smem = sizeof(P5Smem) + 1024;
    cudaFuncSetAttribute(tc5_prep_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_prep_conv", st, tc5_prep_kernel<true><<<(unsigned)nchunks, P5_THREADS, smem, st>>>(p));
}
}  // namespace tc
}  // namespace gdn
