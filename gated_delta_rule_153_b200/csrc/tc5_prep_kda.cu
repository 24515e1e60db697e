// tc5_prep_kda.cu -- per-chunk WY preparation for the channel-wise gate
// (Kimi Delta Attention) on the fifth-generation tensor cores (bf16,
// dk = dv = 128, chunk 64).
//
// The recurrence is the gated delta rule with Diag(a_t) on the key index in
// place of the scalar a_t (the channel-gate reading of "Gated Delta Networks:
// Improving Mamba2 with Delta Rule" (paper review), section "Method"; the
// variant is named in "Linear Attention Architectures: Mechanisms,
// Trade-offs, and Cross-Layer Routing").  With G the per-channel within-chunk
// cumsum of the log-gate:
//   A_ij = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}       (j < i)
//   P_ij = scale sum_c q_ic k_jc e^{G_ic - G_jc}        (j <= i)
//   T = (I + A)^{-1},  W = T diag(beta) (K .* e^G),  U~ = T diag(beta) V
// and the walks take Qg = scale Q .* e^G, K~ = K .* e^{G_last - G} and the
// per-key chunk decay e^{G_last}.
//
// The decay sits inside the contraction over keys.  For the rows of 16-token
// block I (first row f) it splits about f:
//   e^{G_ic - G_jc} = EL_ic * R_I,jc,  EL_ic = e^{G_ic - G_fc} <= 1,
//                                      R_I,jc = e^{G_fc - G_jc},
// with R_I <= 1 on every column j < f.  Inside the block R_I is at most
// e^{span_I}, span_I = max_c (G_fc - G_{f+15,c}).  So the A and P rows of
// block I are one tcgen05 product
//   [K .* EL ; Q .* EL] (K .* R_I)^T      M = 128, N = 16 (I + 1), K = 128
// of which the 32 rows of block I are kept: four products per chunk, each
// with its own B operand.  R_I is formed as F_IJ * ER_j for j in block J < I
// (F_IJ = e^{G_fI - G_lJ}, ER_j = e^{G_lJ - G_j}, l the last row of J) and
// as e^{span} * ER_j inside the block, so the key tiles take two exponentials
// per element.  A block whose span exceeds 80 (e^80 is far inside the bf16 and
// fp32 range, e^88 is not) takes its diagonal 16x16 block from an exact
// elementwise sum instead.
// W^T and U~^T are the transposed products of the scalar-gate preparation:
//   W^T  = (beta e^G .* K)^T T^T,   U~^T = (beta V)^T T^T   (M = 128, N = 64)
// with the scaled key tile written next to the others while the tiles are
// built, so one pass over the loaded tiles makes every operand.
//
// One CTA of eight warps per chunk; about 110 KB of shared memory and 256
// TMEM columns, so two CTAs share an SM.  Outputs as the scalar-gate
// preparation: the W image (Tma128), the U~^T image (Swz<64>), P (Swz<64>),
// e^{G_last} per key (fp32), optionally T (Swz<64>); and the Qg and K~
// images (Tma128) with plain stores while the tiles are built.
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

constexpr int PK_THREADS = 256;
constexpr uint32_t PK_TCOLS = 256;  // D_0..D_3 in 0..159; then W^T 0..63, U~^T 64..127
constexpr int KQ_PANEL = 2 * C * 64;
// B operands R_I .* K: 16 (I + 1) rows each, K-major panels, 1024-aligned
GDN_DEV constexpr int b_base(int I) { return 1024 * I * (I + 1); }  // elements: 0, 2048, 6144, 12288
constexpr int B_ELEMS = 1024 * 4 * 5;                                 // 20480 elements, 40 KB
// TMEM column of the accumulator of row block I
GDN_DEV constexpr uint32_t d_col(int I) { return 8 * I * (I + 1); }    // 0, 16, 48, 96

struct alignas(1024) PkSmem {
    // [K p0 | Q p0 | K p1 | Q p1]: the TMA tiles, scaled in place to K .* EL
    // and Q .* EL (the A operand of the four products).  Afterwards: the
    // exact-block scratch, the fp32 diagonal blocks of A and the solve's
    // scratch; finally the W image (16 KB) and the U~^T image (16 KB).
    __nv_bfloat16 KQ[2 * KQ_PANEL];
    // B operands of the four products; afterwards P, bf16 A and T (Swz<64>)
    __nv_bfloat16 Bx[B_ELEMS];
    __nv_bfloat16 Kw[C * DK];  // Tma128: beta e^G .* K (MN-major A of W^T)
    __nv_bfloat16 V[C * DV];   // Tma128, scaled by beta in place
    float btot[4][DK];         // per-block sums of g, per key
    float Gf[4][DK], Gl[4][DK];  // G at the first and the last row of each block
    float gl[DK];              // e^{G_last}
    float beta[C];
    unsigned int span[4];      // max over keys of each block's span (float bits)
    uint64_t bar_ld, bar_mma;
    uint32_t tmem;
};
static_assert(sizeof(PkSmem) <= 112 * 1024, "two CTAs per SM");

// element offset of (row j, key c) in the B operand of row block I
GDN_DEV int b_off(int I, int j, int c) { return b_base(I) + (c >> 6) * (16 * (I + 1) * 64) + swz<64>(j, c & 63); }

__global__ void __launch_bounds__(PK_THREADS, 2) tc5_prep_kda_kernel(const __grid_constant__ ChunkPtrs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PkSmem& s = *reinterpret_cast<PkSmem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cid = blockIdx.x;
    const int bh = cid / p.NT, n = cid % p.NT, h = bh % p.H;
    const ChunkLoc cl = chunk_loc(p.seq, p.T, p.H, bh, n);
    if (!cl.valid) return;  // past the last chunk of a packed batch
    const int L = cl.L;
    const size_t row0 = (size_t)cl.tok * p.H + h;  // token-head index of row 0
    const size_t rs = (size_t)p.H;

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
    if (tid < 4) s.span[tid] = 0u;
    if (tid < C) s.beta[tid] = tid < L ? p.beta[row0 + tid * rs] : 0.f;
    // the per-key gate rows of the chunk a wave ahead (512 bytes each) into L2
    if (tid >= 64 && tid < 64 + C && p.pf_stride > 0 && cid + p.pf_stride < (int)gridDim.x) {
        const int pc = cid + p.pf_stride, pbh = pc / p.NT;
        const ChunkLoc pl = chunk_loc(p.seq, p.T, p.H, pbh, pc % p.NT);
        const int r = tid - 64;
        if (pl.valid && r < pl.L)
            bulk_prefetch_l2(p.g + (((size_t)pl.tok + r) * p.H + pbh % p.H) * DK, DK * 4);
    }
    if (warp == 0) tc5::alloc(&s.tmem, PK_TCOLS);

    // ---- per-key cumsum: thread (key pair kp, block bq) holds keys 2 kp and
    // 2 kp + 1 of the 16 rows of block bq (a warp: 32 key pairs of one block)
    const int kp = tid & 63, bq = tid >> 6, c = 2 * kp, i0 = 16 * bq;
    float G0[16], G1[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int i = i0 + r;
        float2 gv = make_float2(0.f, 0.f);  // rows past L add 0
        if (i < L) gv = *reinterpret_cast<const float2*>(p.g + (row0 + (size_t)i * rs) * DK + c);
        G0[r] = gv.x;
        G1[r] = gv.y;
    }
#pragma unroll
    for (int r = 1; r < 16; ++r) {
        G0[r] += G0[r - 1];
        G1[r] += G1[r - 1];
    }
    s.btot[bq][c] = G0[15];
    s.btot[bq][c + 1] = G1[15];
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;
    {
        float p0 = 0.f, p1 = 0.f;
        for (int t = 0; t < bq; ++t) {
            p0 += s.btot[t][c];
            p1 += s.btot[t][c + 1];
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            G0[r] += p0;
            G1[r] += p1;
        }
    }
    s.Gf[bq][c] = G0[0];
    s.Gf[bq][c + 1] = G1[0];
    s.Gl[bq][c] = G0[15];
    s.Gl[bq][c + 1] = G1[15];
    if (bq == 3) {
        s.gl[c] = __expf(G0[15]);
        s.gl[c + 1] = __expf(G1[15]);
    }
    {
        float sp = fmaxf(G0[0] - G0[15], G1[0] - G1[15]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sp = fmaxf(sp, __shfl_xor_sync(0xffffffffu, sp, o));
        // unsigned order of the float bits: negative spans and NaN compare above 80
        if (lane == 0) atomicMax(&s.span[bq], __float_as_uint(sp));
    }
    __syncthreads();
    if (__syncthreads_or(!mbar_wait(&s.bar_ld, 0, p.status))) goto done;

    // ---- every operand from one pass over the tiles (bf16 pairs) ------------
    {
        auto ld2 = [](const __nv_bfloat16* t, uint32_t o) {
            return unpack_bf16(*reinterpret_cast<const uint32_t*>(t + o));
        };
        auto st2 = [](__nv_bfloat16* t, uint32_t o, float x, float y) {
            *reinterpret_cast<uint32_t*>(t + o) = pack_bf16(x, y);
        };
        const float Gf0 = G0[0], Gl0 = G0[15], Gf1 = G1[0], Gl1 = G1[15];
        const float ef0 = __expf(Gf0), ef1 = __expf(Gf1);
        const float ekt0 = __expf(s.Gl[3][c] - Gl0), ekt1 = __expf(s.Gl[3][c + 1] - Gl1);
        const float esp0 = Gf0 - Gl0 <= 80.f ? __expf(Gf0 - Gl0) : 0.f;
        const float esp1 = Gf1 - Gl1 <= 80.f ? __expf(Gf1 - Gl1) : 0.f;
        float F0[4], F1[4];
#pragma unroll
        for (int I = 0; I < 4; ++I) {
            F0[I] = I > bq ? __expf(s.Gf[I][c] - Gl0) : 0.f;
            F1[I] = I > bq ? __expf(s.Gf[I][c + 1] - Gl1) : 0.f;
        }
        __nv_bfloat16* qg = p.Qg + (size_t)cid * C * DK;
        __nv_bfloat16* kt = p.Kt + (size_t)cid * C * DK;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int i = i0 + r;
            const float el0 = __expf(G0[r] - Gf0), er0 = __expf(Gl0 - G0[r]);
            const float el1 = __expf(G1[r] - Gf1), er1 = __expf(Gl1 - G1[r]);
            const uint32_t ok_ = Kp<128>::off(i, c), oq = Kp<128>::off(C + i, c), ot = Tma128::off(i, c);
            const float2 kv = ld2(s.KQ, ok_), qv = ld2(s.KQ, oq), vv = ld2(s.V, ot);
            const float bi = s.beta[i];
            st2(s.KQ, ok_, kv.x * el0, kv.y * el1);
            st2(s.KQ, oq, qv.x * el0, qv.y * el1);
            const float k0 = kv.x * er0, k1 = kv.y * er1;
            st2(s.Bx, b_off(bq, i, c), k0 * esp0, k1 * esp1);
#pragma unroll
            for (int I = 1; I < 4; ++I)
                if (I > bq) st2(s.Bx, b_off(I, i, c), k0 * F0[I], k1 * F1[I]);
            const float eg0 = el0 * ef0, eg1 = el1 * ef1;  // e^{G_i}
            st2(s.Kw, ot, kv.x * bi * eg0, kv.y * bi * eg1);
            st2(s.V, ot, vv.x * bi, vv.y * bi);
            st2(qg, ot, p.scale * qv.x * eg0, p.scale * qv.y * eg1);
            st2(kt, ot, k0 * ekt0, k1 * ekt1);
        }
    }
    fence_async_smem();  // generic writes -> tensor-core reads
    tc5::fence_before();
    __syncthreads();

    // ---- [A ; P] rows of block I = [K .* EL ; Q .* EL] (K .* R_I)^T ------------
    if (tid == 0) {
        tc5::fence_after();
        const uint32_t sKQ = smem_u32(s.KQ), sB = smem_u32(s.Bx);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm + d_col(0), tc5::kmajor<2 * C>(sKQ, kk), tc5::kmajor<16>(sB + 2 * b_base(0), kk),
                     tc5::idesc_bf16(128, 16, false, false), kk > 0);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm + d_col(1), tc5::kmajor<2 * C>(sKQ, kk), tc5::kmajor<32>(sB + 2 * b_base(1), kk),
                     tc5::idesc_bf16(128, 32, false, false), kk > 0);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm + d_col(2), tc5::kmajor<2 * C>(sKQ, kk), tc5::kmajor<48>(sB + 2 * b_base(2), kk),
                     tc5::idesc_bf16(128, 48, false, false), kk > 0);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
            tc5::mma(tm + d_col(3), tc5::kmajor<2 * C>(sKQ, kk), tc5::kmajor<64>(sB + 2 * b_base(3), kk),
                     tc5::idesc_bf16(128, 64, false, false), kk > 0);
        tc5::commit(&s.bar_mma);
    }
    if (__syncthreads_or(!mbar_wait(&s.bar_mma, 0, p.status))) goto done;
    tc5::fence_after();

    {
        __nv_bfloat16* P = s.Bx;              // Swz<64>
        __nv_bfloat16* Abf = s.Bx + C * C;    // Swz<64>
        __nv_bfloat16* T = s.Bx + 2 * C * C;  // Swz<64>, 1024-aligned
        auto Gs = reinterpret_cast<float(*)[DK]>(s.KQ);  // 16 x 128 fp32 scratch
        auto Ad = reinterpret_cast<float(*)[16][17]>(reinterpret_cast<unsigned char*>(s.KQ) + 16 * DK * 4);
        auto Xs = reinterpret_cast<__nv_bfloat16(*)[16 * 16]>(reinterpret_cast<unsigned char*>(s.KQ) +
                                                              16 * DK * 4 + 4 * 16 * 17 * 4);

        // ---- epilogue 1: warp (q, ch) reads TMEM lanes 32q.. and the column
        // blocks J = 2 ch, 2 ch + 1; lane = row of [A ; P], its block I ----------
        {
            const int q = warp & 3, ch = warp >> 2;
            const bool is_a = q < 2;
            const int i = 32 * (q & 1) + lane;  // token row
            const int I0 = 2 * (q & 1), I = i >> 4;
            const uint32_t trow = tm + ((uint32_t)(32 * q) << 16);
            const float f = is_a ? s.beta[i] : (i < L ? p.scale : 0.f);
            __nv_bfloat16* dst = is_a ? Abf : P;
#pragma unroll
            for (int jb = 0; jb < 2; ++jb) {
                const int J = 2 * ch + jb;
                float v[16];
                if (J > I0 + 1) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = 0.f;
                } else {
                    float v0[16], v1[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) v0[e] = 0.f;
                    if (J <= I0) tc5::ld16(v0, trow + d_col(I0) + 16 * J);
                    tc5::ld16(v1, trow + d_col(I0 + 1) + 16 * J);
                    tc5::wait_ld();
                    const bool hi = lane >= 16;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int j = 16 * J + e;
                        const bool live = is_a ? j < i : j <= i;
                        v[e] = live ? f * (hi ? v1[e] : v0[e]) : 0.f;
                    }
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    *reinterpret_cast<uint4*>(dst + swz<C>(i, 16 * J + 8 * hh)) =
                        make_uint4(pack_bf16(v[8 * hh], v[8 * hh + 1]), pack_bf16(v[8 * hh + 2], v[8 * hh + 3]),
                                   pack_bf16(v[8 * hh + 4], v[8 * hh + 5]),
                                   pack_bf16(v[8 * hh + 6], v[8 * hh + 7]));
                if (is_a && J == I) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) Ad[I][i & 15][e] = v[e];
                }
            }
        }
        tc5::fence_before();
        __syncthreads();

        // ---- exact diagonal blocks where the span is above 80 ---------------
        for (int b = 0; b < 4; ++b) {
            if (s.span[b] <= __float_as_uint(80.f)) continue;  // uniform over the CTA
            for (int e = tid; e < 16 * DK; e += PK_THREADS) {
                const int r = e / DK, cc = e % DK, i = 16 * b + r;
                Gs[r][cc] = i < L ? p.g[(row0 + (size_t)i * rs) * DK + cc] : 0.f;
            }
            __syncthreads();
            if (tid < DK) {
                for (int r = 1; r < 16; ++r) Gs[r][tid] += Gs[r - 1][tid];
            }
            __syncthreads();
            {
                const int r = tid >> 4, cc = tid & 15;  // pair (i, j) of the block
                const int i = 16 * b + r, j = 16 * b + cc;
                float sa = 0.f, sq = 0.f;
                if (cc <= r && i < L) {
                    const __nv_bfloat16* ki = p.k + (row0 + (size_t)i * rs) * DK;
                    const __nv_bfloat16* kj = p.k + (row0 + (size_t)j * rs) * DK;
                    const __nv_bfloat16* qi = p.q + (row0 + (size_t)i * rs) * DK;
                    for (int x = 0; x < DK; ++x) {
                        const float d = __expf(Gs[r][x] - Gs[cc][x]);
                        const float kjd = __bfloat162float(kj[x]) * d;
                        sa += __bfloat162float(ki[x]) * kjd;
                        sq += __bfloat162float(qi[x]) * kjd;
                    }
                }
                const float a = cc < r ? s.beta[i] * sa : 0.f;
                Ad[b][r][cc] = a;
                Abf[swz<C>(i, j)] = __float2bfloat16_rn(a);
                P[swz<C>(i, j)] = __float2bfloat16_rn(i < L ? p.scale * sq : 0.f);
            }
            __syncthreads();
        }

        // ---- UT transform: T = (I + A)^{-1} ---------------------------------
        ut_solve(Ad, Abf, T, Xs);
    }

    // ---- W^T = (beta e^G .* K)^T T^T ; U~^T = (beta V)^T T^T ---------------------
    fence_async_smem();
    tc5::fence_before();
    __syncthreads();
    if (tid == 0) {
        tc5::fence_after();
        const uint32_t sT = smem_u32(s.Bx + 2 * C * C), sKw = smem_u32(s.Kw), sV = smem_u32(s.V);
        constexpr uint32_t ID_WU = tc5::idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm, tc5::mnmajor(sKw, kk, C * 128), tc5::kmajor<C>(sT, kk), ID_WU, kk > 0);
#pragma unroll
        for (int kk = 0; kk < C / 16; ++kk)
            tc5::mma(tm + 64, tc5::mnmajor(sV, kk, C * 128), tc5::kmajor<C>(sT, kk), ID_WU, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    if (__syncthreads_or(!mbar_wait(&s.bar_mma, 1, p.status))) goto done;
    tc5::fence_after();

    // ---- epilogue 2: warps 0..3 key rows of W^T, warps 4..7 value rows of U~^T
    {
        const int q = warp & 3, row = 32 * q + lane;
        const uint32_t trow = tm + ((uint32_t)(32 * q) << 16);
        float x[32];
        if (warp < 4) {
            __nv_bfloat16* Wimg = s.KQ;  // Tma128, 16 KB
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc5::ld32(x, trow + 32 * half);
                tc5::wait_ld();
#pragma unroll
                for (int t = 0; t < 32; ++t) Wimg[Tma128::off(32 * half + t, row)] = __float2bfloat16_rn(x[t]);
            }
        } else {
            __nv_bfloat16* Uimg = s.KQ + C * DK;  // Swz<64>, 128 value rows x 64 tokens
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
        bulk_s2g(p.P + (size_t)cid * C * C, s.Bx, C * C * 2);
        bulk_s2g(p.G + (size_t)cid * DK, s.gl, DK * 4);
        if (p.Tb) bulk_s2g(p.Tb + (size_t)cid * C * C, s.Bx + 2 * C * C, C * C * 2);
        bulk_commit();
        bulk_wait_read<0>();
    }
done:
    tc5::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc5::fence_after();
        tc5::dealloc(tm, PK_TCOLS);
    }
}

}  // namespace

namespace tc {
void launch_prep5_kda(const ChunkPtrs& pin, size_t nchunks, cudaStream_t st) {
    ChunkPtrs p = pin;
    p.pf_stride = 2 * sm_count();  // two CTAs per SM
    const int smem = sizeof(PkSmem) + 1024;
    cudaFuncSetAttribute(tc5_prep_kda_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_prep_kda", st, tc5_prep_kda_kernel<<<(unsigned)nchunks, PK_THREADS, smem, st>>>(p));
}
}  // namespace tc
}  // namespace gdn
