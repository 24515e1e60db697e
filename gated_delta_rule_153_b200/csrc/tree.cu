// tree.cu -- draft-tree verification and commit for the gated delta rule.
//
// "TreeWY: Speculative Verification for Gated DeltaNet Hybrids" (the
// "Linked reviews" entry of the "Gated Delta Networks: Improving Mamba2
// with Delta Rule" review page): score every node of a speculative draft
// tree against the committed state with one triangular solve instead of one
// state snapshot per node, and rebuild only the accepted state on commit.
//
// A tree of M <= 64 nodes hangs below the committed state S0 of each
// (sequence, head); parent[i] in [-1, i) (-1: S0 itself).  Node i's output is
// the gated delta rule ("Gated Delta Networks: Improving Mamba2 with Delta
// Rule", section "Method") run from S0 over its root path.  With G_i the sum
// of g over the root path of i (inclusive) and anc(i) its strict ancestors,
// the chunkwise algebra of that review carries over with the causal mask
// replaced by the ancestor relation:
//     A_ij = beta_i e^{G_i - G_j} k_i.k_j        (j in anc(i), else 0)
//     T    = (I + A)^{-1}                         (lower triangular: parents first)
//     W    = T diag(beta e^G) K,   U~ = T diag(beta) V,   U = U~ - W S0^T
//     P_ij = scale e^{G_i - G_j} q_i.k_j          (j in anc(i) or j = i)
//     O    = scale diag(e^G) Q S0^T + P U.
// Row i of U is the delta-rule correction u_i of node i given the state at its
// parent, so O_i is exactly node i's read-out.  Commit runs the recurrent form
// along the accepted node's root path on the fp32 state: one read and one
// write of each state row.
#include <math.h>

#include <type_traits>

#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tma.cuh"

namespace gdn {
namespace {

constexpr int TD = 128;           // d_k = d_v
constexpr int TREE_THREADS = 256;  // 8 warps
constexpr int kMaxTreeNodes = 64;

// Verification on the fifth-generation tensor cores.  The node tiles (MP = 32
// or 64 rows) arrive by TMA, K and Q interleaved panel by panel so that one
// M = 128 product [K ; Q] K^T gives A's rows (lanes 0..MP-1) and P's rows
// (lanes MP..2MP-1).  W is never formed: with Tu = T diag(beta),
//   U = U~ - W S0^T = Tu (V - diag(e^G) K S0^T) = Tu Z,
// so the products that touch the state run transposed, the 128 value rows on
// the TMEM lanes (every warp has work in their epilogues):
//   [K ; Q] K^T                 lane = node    A and P (scalar gate)
//   S0 K^T                      lane = value   -> Z^T = V^T - (S0 K^T) diag(e^G),
//                                                 written over the V tile
//   U^T = Z^T Tu^T,  Y^T = S0 Q^T  lane = value
//   O^T = Y^T diag(scale e^G) + U^T P^T  lane = value
// The state enters as a bf16 A operand in tensor memory (each thread converts
// its own row), and so does U^T.  The ancestor masks, the decays and the
// level-by-level solve for T stay on CUDA cores: they are the tree's small
// dependent steps, not contractions.  Channel gate: A and P are sums over the
// keys pair by pair on CUDA cores, and K and Q are scaled by e^G per key in
// place before the state products (Z = V - (K .* e^G) S0^T, O = scale
// (Q .* e^G) S0^T + P U).
template <int MP, bool KDA>
struct alignas(1024) TreeSmem {
    __nv_bfloat16 KQ[2 * MP * TD];  // TMA tiles [K p0 | Q p0 | K p1 | Q p1]: 64-column panels of
                                    // MP node rows, 128-byte swizzle
    __nv_bfloat16 V[MP * TD];       // two 64-column panels of MP rows; then Z in place
    __nv_bfloat16 Tu[MP * 64];      // T diag(beta): [i][j] (K-major B: N = i)
    __nv_bfloat16 P[MP * 64];       // scale e^{G_i - G_j} q_i.k_j on ancestors and the diagonal
    float A[MP][MP + 1];            // masked, decayed beta K K^T
    float T[MP][MP + 1];            // (I + A)^{-1}
    float G[MP], g[MP], beta[MP];
    unsigned long long anc[MP];
    int par[MP], depth[MP];
    int maxdepth;
    uint64_t bar_ld, bar_mma;
    uint32_t tmem;
    alignas(16) float Gc[KDA ? MP : 1][TD];  // channel gate: per-key sums of g over each root path
};

struct TreePtrs {
    CUtensorMap qmap, kmap, vmap;  // [N, M, H, 128] node maps, boxes of MP rows
    int M, H;
    float scale;
    const int* parent;
    const float *g, *beta, *state;
    __nv_bfloat16* o;
    unsigned int* status;
};

GDN_DEV unsigned char* align_1k(unsigned char* p) {
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Elements (row, column) of K (Q at + MP * 64) in the interleaved tile, and of V.
template <int MP>
GDN_DEV int kqoff(int r, int c) { return (c >> 6) * (2 * MP * 64) + swz<64>(r, c & 63); }
template <int MP>
GDN_DEV int voff(int r, int c) { return (c >> 6) * (MP * 64) + swz<64>(r, c & 63); }

template <int MP>
GDN_DEV void ldcols(float* v, uint32_t taddr) {  // MP / 2 columns of this thread's lane
    if constexpr (MP == 32) tc5::ld16(*reinterpret_cast<float(*)[16]>(v), taddr);
    else tc5::ld32(*reinterpret_cast<float(*)[32]>(v), taddr);
}
template <int MP>
GDN_DEV void stcols(uint32_t taddr, const uint32_t* r) {  // MP / 2 32-bit columns
    if constexpr (MP == 32) {
        tc5::st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(r));
    } else {
        tc5::st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(r));
        tc5::st16(taddr + 16, *reinterpret_cast<const uint32_t(*)[16]>(r + 16));
    }
}

template <int MP, bool KDA>
GDN_DEV void verify_body(TreeSmem<MP, KDA>& s, const TreePtrs& p, uint32_t tm) {
    // tensor-memory columns: the bf16 state (64); then [K K^T ; Q K^T] and S0 K^T;
    // then U^T and Y^T (becoming O^T); U^T in bf16 takes the state's columns
    constexpr uint32_t TS0 = 0, TKQ = 64, TSK = 64 + MP, TU = 64, TY = 64 + MP, TUP = 0;
    constexpr uint32_t ID_NN = tc5::idesc_bf16(128, MP, false, false);
    constexpr uint32_t ID_MK = tc5::idesc_bf16(128, MP, true, false);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int M = p.M, H = p.H;
    const int nh = blockIdx.x, n = nh / H, h = nh % H;
    const size_t rs = (size_t)H * TD;                   // node row stride
    const size_t row0 = ((size_t)n * M * H + h) * TD;  // node 0 of (n, h)
    const float scale = p.scale;
    const uint32_t sKQ = smem_u32(s.KQ), sQ = sKQ + MP * 128, sV = smem_u32(s.V);
    const uint32_t sTu = smem_u32(s.Tu), sP = smem_u32(s.P);
    // epilogue thread roles on the 128 lanes: lane quarter warp % 4, column half warp / 4
    const int lr = 32 * (warp & 3) + lane, hh = warp >> 2, j0 = hh * (MP / 2);
    const uint32_t trow = tm + ((uint32_t)(32 * (warp & 3)) << 16);
    uint32_t mph = 0;

    if constexpr (KDA) {  // path sums, parents first: thread = key
        if (tid < TD)
            for (int i = 0; i < M; ++i)
                if (s.par[i] >= 0) s.Gc[i][tid] += s.Gc[s.par[i]][tid];
    }
    // ---- path sums of g and ancestor sets (parents precede children) ------
    if (tid < MP) {
        float Gi = s.g[tid];
        unsigned long long m = 0;
        for (int j = s.par[tid]; j >= 0; j = s.par[j]) {
            m |= 1ull << j;
            Gi += s.g[j];
        }
        s.G[tid] = Gi;
        s.anc[tid] = m;
        s.depth[tid] = __popcll(m);
        atomicMax(&s.maxdepth, __popcll(m));
    }
    bool ok = mbar_wait(&s.bar_ld, 0, p.status);
    if (__syncthreads_or(!ok)) return;

    if constexpr (KDA) {
        // ---- A and P: ancestor pairs (and, for P, the node itself) only; a
        // warp per pair, a lane per 4 keys; the decays e^{G_i - G_j} <= 1 key by key
        for (int e = tid; e < MP * MP; e += TREE_THREADS) {
            const int i = e / MP, j = e % MP;
            s.A[i][j] = 0.f;
            s.P[swz<64>(i, j)] = __float2bfloat16_rn(0.f);
        }
        __syncthreads();
        int pc = 0;
        const int c = 4 * lane;
        for (int i = 0; i < M; ++i) {
            for (unsigned long long m = s.anc[i] | (1ull << i); m; m &= m - 1ull, ++pc) {
                if ((pc & 7) != warp) continue;
                const int j = __ffsll((long long)m) - 1;
                const uint2 ki = *reinterpret_cast<const uint2*>(&s.KQ[kqoff<MP>(i, c)]);
                const uint2 kj = *reinterpret_cast<const uint2*>(&s.KQ[kqoff<MP>(j, c)]);
                const uint2 qi = *reinterpret_cast<const uint2*>(&s.KQ[MP * 64 + kqoff<MP>(i, c)]);
                const float2 ki0 = unpack_bf16(ki.x), ki1 = unpack_bf16(ki.y);
                const float2 kj0 = unpack_bf16(kj.x), kj1 = unpack_bf16(kj.y);
                const float2 qi0 = unpack_bf16(qi.x), qi1 = unpack_bf16(qi.y);
                const float d0 = __expf(s.Gc[i][c] - s.Gc[j][c]), d1 = __expf(s.Gc[i][c + 1] - s.Gc[j][c + 1]);
                const float d2 = __expf(s.Gc[i][c + 2] - s.Gc[j][c + 2]), d3 = __expf(s.Gc[i][c + 3] - s.Gc[j][c + 3]);
                const float w0 = kj0.x * d0, w1 = kj0.y * d1, w2 = kj1.x * d2, w3 = kj1.y * d3;
                float sa = ki0.x * w0 + ki0.y * w1 + ki1.x * w2 + ki1.y * w3;
                float sq = qi0.x * w0 + qi0.y * w1 + qi1.x * w2 + qi1.y * w3;
                sa = warp_sum(sa);
                sq = warp_sum(sq);
                if (lane == 0) {
                    if (j != i) s.A[i][j] = s.beta[i] * sa;
                    s.P[swz<64>(i, j)] = __float2bfloat16_rn(scale * sq);
                }
            }
        }
        __syncthreads();
        // K .* e^G (for Z) and Q .* e^G (the read-out), in place
        for (int e = tid; e < MP * TD / 2; e += TREE_THREADS) {
            const int i = e / (TD / 2), c2 = 2 * (e % (TD / 2));
            const float d0 = __expf(s.Gc[i][c2]), d1 = __expf(s.Gc[i][c2 + 1]);
            uint32_t* kp = reinterpret_cast<uint32_t*>(&s.KQ[kqoff<MP>(i, c2)]);
            uint32_t* qp = reinterpret_cast<uint32_t*>(&s.KQ[MP * 64 + kqoff<MP>(i, c2)]);
            const float2 kv = unpack_bf16(*kp), qv = unpack_bf16(*qp);
            *kp = pack_bf16(kv.x * d0, kv.y * d1);
            *qp = pack_bf16(qv.x * d0, qv.y * d1);
        }
        fence_async_smem();
        tc5::fence_before();
        __syncthreads();
    }
    // ---- [K ; Q] K^T (scalar gate) and S0 K^T -----------------------------------
    if (tid == 0) {
        tc5::fence_after();
        if constexpr (!KDA) {
#pragma unroll
            for (int kk = 0; kk < TD / 16; ++kk)
                tc5::mma(tm + TKQ, tc5::kmajor<2 * MP>(sKQ, kk), tc5::kmajor<2 * MP>(sKQ, kk), ID_NN, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < TD / 16; ++kk)
            tc5::mma_ts(tm + TSK, tm + TS0 + 8 * kk, tc5::kmajor<2 * MP>(sKQ, kk), ID_NN, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) return;
    tc5::fence_after();
    if constexpr (!KDA) {
        if (lr < MP) {  // A row i = lr, columns j0 ..
            const int i = lr;
            float kk[MP / 2];
            ldcols<MP>(kk, trow + TKQ + j0);
            tc5::wait_ld();
            const unsigned long long ai = s.anc[i];
            const float Gi = s.G[i], bi = s.beta[i];
#pragma unroll
            for (int c = 0; c < MP / 2; ++c) {
                const int j = j0 + c;
                s.A[i][j] = ((ai >> j) & 1ull) ? bi * __expf(Gi - s.G[j]) * kk[c] : 0.f;
            }
        } else if (lr < 2 * MP) {  // P row i = lr - MP
            const int i = lr - MP;
            float qk[MP / 2];
            ldcols<MP>(qk, trow + TKQ + j0);
            tc5::wait_ld();
            const unsigned long long ai = s.anc[i];
            const float Gi = s.G[i];
#pragma unroll
            for (int c = 0; c < MP / 2; ++c) {
                const int j = j0 + c;
                qk[c] = (((ai >> j) & 1ull) || j == i) ? scale * __expf(Gi - s.G[j]) * qk[c] : 0.f;
            }
#pragma unroll
            for (int c8 = 0; c8 < MP / 16; ++c8)
                *reinterpret_cast<uint4*>(&s.P[swz<64>(i, j0 + 8 * c8)]) =
                    make_uint4(pack_bf16(qk[8 * c8], qk[8 * c8 + 1]), pack_bf16(qk[8 * c8 + 2], qk[8 * c8 + 3]),
                               pack_bf16(qk[8 * c8 + 4], qk[8 * c8 + 5]), pack_bf16(qk[8 * c8 + 6], qk[8 * c8 + 7]));
        }
    }
    {   // Z^T = V^T - (S0 K^T) diag(e^G): value lr, nodes j0 .., over the V tile
        float sk[MP / 2];
        ldcols<MP>(sk, trow + TSK + j0);
        tc5::wait_ld();
#pragma unroll
        for (int c = 0; c < MP / 2; ++c) {
            __nv_bfloat16& vz = s.V[voff<MP>(j0 + c, lr)];
            const float f = KDA ? 1.f : __expf(s.G[j0 + c]);
            vz = __float2bfloat16_rn(__bfloat162float(vz) - f * sk[c]);
        }
    }
    tc5::fence_before();
    __syncthreads();

    // ---- T = (I + A)^{-1}, one tree level at a time --------------------------
    // Row i of T is e_i - sum over ancestors l of A_il T_l, and T_ic is non-zero
    // only for c an ancestor of i or i itself; so every node of one depth is
    // solved at once from the rows of shallower nodes (a chain: one per level).
    {   // thread = (node i, NC consecutive columns): fixed for every level
        constexpr int NC = MP * MP / TREE_THREADS;
        const int i = tid / (MP / NC), c0 = NC * (tid % (MP / NC));
        const unsigned long long ai = s.anc[i];
        const int di = s.depth[i], levels = s.maxdepth;
        for (int d = 0; d <= levels; ++d) {
            if (di == d) {
#pragma unroll
                for (int cc = 0; cc < NC; ++cc) {
                    const int c = c0 + cc;
                    float t = c == i ? 1.f : 0.f;
                    if ((ai >> c) & 1ull) {
                        float sum = 0.f;
                        for (unsigned long long m = ai & ~((1ull << c) - 1ull); m; m &= m - 1ull) {
                            const int l = __ffsll((long long)m) - 1;  // ancestors l >= c
                            sum += s.A[i][l] * s.T[l][c];
                        }
                        t = -sum;
                    }
                    s.T[i][c] = t;
                }
            }
            __syncthreads();
        }
    }
    for (int e = tid; e < MP * MP; e += TREE_THREADS) {
        const int i = e / MP, j = e % MP;
        s.Tu[swz<64>(i, j)] = __float2bfloat16_rn(s.T[i][j] * s.beta[j]);
    }
    fence_async_smem();  // Z, P and Tu (generic writes) -> tensor-core reads
    tc5::fence_before();
    __syncthreads();

    // ---- U^T = Z^T Tu^T,  Y^T = S0 Q^T (lane = value) ----------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < MP / 16; ++kk)
            tc5::mma(tm + TU, tc5::mnmajor(sV, kk, MP * 128), tc5::kmajor<MP>(sTu, kk), ID_MK, kk > 0);
#pragma unroll
        for (int kk = 0; kk < TD / 16; ++kk)
            tc5::mma_ts(tm + TY, tm + TS0 + 8 * kk, tc5::kmajor<2 * MP>(sQ, kk), ID_NN, kk > 0);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) return;
    tc5::fence_after();
    {   // U^T -> bf16 A operand (over the state's columns); Y^T columns *= scale e^{G_i}
        float u[MP / 2], y[MP / 2];
        ldcols<MP>(u, trow + TU + j0);
        ldcols<MP>(y, trow + TY + j0);
        tc5::wait_ld();
        uint32_t pk[MP / 4], yb[MP / 2];
#pragma unroll
        for (int c = 0; c < MP / 4; ++c) pk[c] = pack_bf16(u[2 * c], u[2 * c + 1]);
#pragma unroll
        for (int c = 0; c < MP / 2; ++c)
            yb[c] = __float_as_uint(y[c] * (KDA ? scale : scale * __expf(s.G[j0 + c])));
        if constexpr (MP == 32) tc5::st8(trow + TUP + j0 / 2, *reinterpret_cast<uint32_t(*)[8]>(pk));
        else tc5::st16(trow + TUP + j0 / 2, *reinterpret_cast<uint32_t(*)[16]>(pk));
        stcols<MP>(trow + TY + j0, yb);
        tc5::wait_st();
    }
    tc5::fence_before();
    __syncthreads();

    // ---- O^T = Y^T + U^T P^T (A from tensor memory) ------------------------------
    if (tid == 0) {
        tc5::fence_after();
#pragma unroll
        for (int kk = 0; kk < MP / 16; ++kk)
            tc5::mma_ts(tm + TY, tm + TUP + 8 * kk, tc5::kmajor<MP>(sP, kk), ID_NN, true);
        tc5::commit(&s.bar_mma);
    }
    ok = mbar_wait(&s.bar_mma, mph, p.status);
    mph ^= 1;
    if (__syncthreads_or(!ok)) return;
    tc5::fence_after();
    {   // O[i][v] for v = lr, nodes j0 ..: a warp writes 32 consecutive values of a
        // node, lane pairs trading halves so that each store is a 32-bit word
        float x[MP / 2];
        ldcols<MP>(x, trow + TY + j0);
        tc5::wait_ld();
#pragma unroll
        for (int g = 0; g < MP / 32; ++g) {
            uint32_t v[8], w[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) v[jj] = pack_bf16(x[16 * g + 2 * jj], x[16 * g + 2 * jj + 1]);
            pair_columns(v, w);  // w[jj]: values lr & ~1, +1 of node j0 + 16g + 2jj + (lane & 1)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int node = j0 + 16 * g + 2 * jj + (lane & 1);
                if (node < M) *reinterpret_cast<uint32_t*>(p.o + row0 + (size_t)node * rs + (lr & ~1)) = w[jj];
            }
        }
    }
}

// One CTA per (sequence n, head h), MP = 32 (four CTAs per SM; three with the
// channel gate's per-key path sums) or 64 node rows.
template <int MP, bool KDA>
__global__ void __launch_bounds__(TREE_THREADS, MP == 32 ? (KDA ? 3 : 4) : 1)
tree_verify_kernel(const __grid_constant__ TreePtrs p) {
    constexpr uint32_t TCOLS = MP == 32 ? 128 : 256;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    TreeSmem<MP, KDA>& s = *reinterpret_cast<TreeSmem<MP, KDA>*>(align_1k(smem_raw));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int M = p.M, H = p.H;
    const int nh = blockIdx.x, n = nh / H, h = nh % H;
    if (tid == 0) {
        mbar_init(&s.bar_ld, 1);
        mbar_init(&s.bar_mma, 1);
        fence_mbar_init();
        // rows past M hold the next sequence's nodes (or zeros past the
        // tensor): finite, and masked out of every product that reaches O
        mbar_arrive_expect(&s.bar_ld, 3 * MP * TD * 2);
        const int tok = n * M;
        tma_load_3d(s.KQ, &p.kmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.KQ + MP * 64, &p.qmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.KQ + 2 * MP * 64, &p.kmap, 64, h, tok, &s.bar_ld);
        tma_load_3d(s.KQ + 3 * MP * 64, &p.qmap, 64, h, tok, &s.bar_ld);
        tma_load_3d(s.V, &p.vmap, 0, h, tok, &s.bar_ld);
        tma_load_3d(s.V + MP * 64, &p.vmap, 64, h, tok, &s.bar_ld);
        s.maxdepth = 0;
    }
    if (warp == 0) tc5::alloc(&s.tmem, TCOLS);
    if (tid < MP) {
        int pa = -1;
        float gi = 0.f, bi = 0.f;
        if (tid < M) {
            pa = p.parent[(size_t)n * M + tid];
            if (pa < -1 || pa >= tid) {  // not a tree in topological order
                if (p.status) atomicOr(p.status, 2u);
                pa = -1;
            }
            if (!KDA) gi = p.g[((size_t)n * M + tid) * H + h];
            bi = p.beta[((size_t)n * M + tid) * H + h];
        }
        s.par[tid] = pa;
        s.g[tid] = gi;
        s.beta[tid] = bi;
    }
    if constexpr (KDA) {  // per-key gates of every node (zero past M)
        for (int e = tid; e < MP * TD / 4; e += TREE_THREADS) {
            const int i = e / (TD / 4), c4 = e % (TD / 4);
            cp_async16_zfill(&s.Gc[i][4 * c4], p.g + (((size_t)n * M + (i < M ? i : 0)) * H + h) * TD + 4 * c4,
                             i < M);
        }
        cp_async_commit();
    }
    // the state row of this thread's lane (value 32 (warp % 4) + lane), keys
    // 64 (warp / 4) .. +63, from fp32 to bf16 pairs.  The loads go through L1:
    // a warp's 16-byte loads touch half of each of 32 sectors, and the next
    // load of the same lanes finds the other half there ...
    uint32_t srow[32];
    {
        const float4* src = reinterpret_cast<const float4*>(
            p.state + ((size_t)nh * TD + 32 * (warp & 3) + (tid & 31)) * TD + 64 * (warp >> 2));
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float4 a = __ldg(src + j);
            srow[2 * j] = pack_bf16(a.x, a.y);
            srow[2 * j + 1] = pack_bf16(a.z, a.w);
        }
    }
    if constexpr (KDA) cp_async_wait<0>();
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;
    {   // ... into tensor memory as the A operand of the state products
        const uint32_t ta = tm + ((uint32_t)(32 * (warp & 3)) << 16) + 32 * (warp >> 2);
        tc5::st16(ta, *reinterpret_cast<uint32_t(*)[16]>(srow));
        tc5::st16(ta + 16, *reinterpret_cast<uint32_t(*)[16]>(srow + 16));
        tc5::wait_st();
    }
    verify_body<MP, KDA>(s, p, tm);
    tc5::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc5::fence_after();
        tc5::dealloc(tm, TCOLS);
    }
}

template <int MP, bool KDA>
bool launch_verify(int N, int M, int H, float scale, const int* parent, const void* q,
                   const void* k, const void* v, const float* g, const float* beta,
                   const float* state, void* o, unsigned int* status, cudaStream_t st) {
    TreePtrs tp{};
    if (!encode_token_map(&tp.qmap, q, N, M, H, 64, MP) || !encode_token_map(&tp.kmap, k, N, M, H, 64, MP) ||
        !encode_token_map(&tp.vmap, v, N, M, H, 64, MP))
        return false;
    tp.M = M; tp.H = H; tp.scale = scale;
    tp.parent = parent; tp.g = g; tp.beta = beta; tp.state = state;
    tp.o = (__nv_bfloat16*)o; tp.status = status;
    const int smem = sizeof(TreeSmem<MP, KDA>) + 1024;
    cudaFuncSetAttribute(tree_verify_kernel<MP, KDA>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tree_verify", st, (tree_verify_kernel<MP, KDA><<<(unsigned)(N * H), TREE_THREADS, smem, st>>>(tp)));
    return true;
}

// ---- commit: the recurrent form along the accepted node's root path --------
template <bool KDA>
struct CommitSmem {
    float k[kMaxTreeNodes][TD];  // keys of the path tokens, in path order
    float v[kMaxTreeNodes][TD];
    float alpha[kMaxTreeNodes][KDA ? TD : 1], beta[kMaxTreeNodes];  // decay per token (per key: channel gate)
    int path[kMaxTreeNodes];
    int len;
};

// One CTA per (n, h); a state row is covered by 8 lanes of 16 columns each
// (column 4*(sub + 8j) + e), and each thread keeps four rows in registers for
// the whole path: one streaming read and one streaming write per element.
template <bool KDA>
__global__ void __launch_bounds__(TREE_THREADS)
tree_commit_kernel(int M, int H, const int* __restrict__ parent, const int* __restrict__ accepted,
                   const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                   const float* __restrict__ g, const float* __restrict__ beta,
                   float* __restrict__ state, unsigned int* status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    CommitSmem<KDA>& s = *reinterpret_cast<CommitSmem<KDA>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nh = blockIdx.x, n = nh / H, h = nh % H;
    if (tid == 0) {
        int a = accepted[n];
        if (a < -1 || a >= M) {
            if (status) atomicOr(status, 2u);
            a = -1;
        }
        int len = 0;
        for (int j = a; j >= 0 && len < kMaxTreeNodes;) {  // leaf to root
            s.path[len++] = j;
            const int p = parent[(size_t)n * M + j];
            if (p < -1 || p >= j) {
                if (status) atomicOr(status, 2u);
                break;  // an invalid parent reads as -1, as in verification
            }
            j = p;
        }
        for (int x = 0; x < len / 2; ++x) {  // root to leaf
            const int t = s.path[x];
            s.path[x] = s.path[len - 1 - x];
            s.path[len - 1 - x] = t;
        }
        s.len = len;
    }
    __syncthreads();
    const int len = s.len;
    if (len == 0) return;  // nothing accepted: the state stays as it is
    for (int e = tid; e < len * TD; e += TREE_THREADS) {
        const int p = e / TD, c = e % TD;
        const size_t row = (((size_t)n * M + s.path[p]) * H + h) * TD;
        s.k[p][c] = __bfloat162float(k[row + c]);
        s.v[p][c] = __bfloat162float(v[row + c]);
    }
    if (tid < len) {
        const size_t i = ((size_t)n * M + s.path[tid]) * H + h;
        if (!KDA) s.alpha[tid][0] = __expf(g[i]);
        s.beta[tid] = beta[i];
    }
    if constexpr (KDA) {
        for (int e = tid; e < len * TD; e += TREE_THREADS) {
            const int p = e / TD, c = e % TD;
            s.alpha[p][c] = __expf(g[(((size_t)n * M + s.path[p]) * H + h) * TD + c]);
        }
    }
    float* S = state + (size_t)nh * TD * TD;
    const int sub = lane & 7, grp = lane >> 3;
    float4 st[4][4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const float4* src = reinterpret_cast<const float4*>(S + (size_t)(32 * rr + 4 * warp + grp) * TD);
#pragma unroll
        for (int j = 0; j < 4; ++j) st[rr][j] = __ldcs(src + sub + 8 * j);
    }
    __syncthreads();
    for (int p = 0; p < len; ++p) {
        float kr[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 x = *reinterpret_cast<const float4*>(&s.k[p][4 * (sub + 8 * j)]);
            kr[4 * j] = x.x; kr[4 * j + 1] = x.y; kr[4 * j + 2] = x.z; kr[4 * j + 3] = x.w;
        }
        float al[16];  // this thread's 16 key columns' decays
        if constexpr (KDA) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 x = *reinterpret_cast<const float4*>(&s.alpha[p][4 * (sub + 8 * j)]);
                al[4 * j] = x.x; al[4 * j + 1] = x.y; al[4 * j + 2] = x.z; al[4 * j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) al[j] = s.alpha[p][0];
        }
        const float be = s.beta[p];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                st[rr][j].x *= al[4 * j]; st[rr][j].y *= al[4 * j + 1];
                st[rr][j].z *= al[4 * j + 2]; st[rr][j].w *= al[4 * j + 3];
                dot += st[rr][j].x * kr[4 * j] + st[rr][j].y * kr[4 * j + 1] +
                       st[rr][j].z * kr[4 * j + 2] + st[rr][j].w * kr[4 * j + 3];
            }
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            dot += __shfl_xor_sync(0xffffffffu, dot, 4);
            const float u = be * (s.v[p][32 * rr + 4 * warp + grp] - dot);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                st[rr][j].x += u * kr[4 * j]; st[rr][j].y += u * kr[4 * j + 1];
                st[rr][j].z += u * kr[4 * j + 2]; st[rr][j].w += u * kr[4 * j + 3];
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        float4* dst = reinterpret_cast<float4*>(S + (size_t)(32 * rr + 4 * warp + grp) * TD);
#pragma unroll
        for (int j = 0; j < 4; ++j) __stcs(dst + sub + 8 * j, st[rr][j]);
    }
}

bool aligned(const void* p, unsigned a) { return ((uintptr_t)p & (a - 1)) == 0; }

gdn_status check_tree(int N, int M, int H, int dk, int dv, gdn_dtype dtype, gdn_gate gate) {
    if (N < 1 || H < 1 || M < 1) return GDN_ERR_INVALID_ARG;
    if ((long long)N * H > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (gate != GDN_GATE_SCALAR && gate != GDN_GATE_CHANNEL) return GDN_ERR_INVALID_ARG;
    if (M > kMaxTreeNodes) return GDN_ERR_UNSUPPORTED;
    if (dtype != GDN_BF16 || dk != TD || dv != TD) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

gdn_status launched() { return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace
}  // namespace gdn

extern "C" {

gdn_status gdn_tree_verify(int N, int M, int H, int dk, int dv, gdn_dtype dtype, gdn_gate gate,
                           float scale, const int* parent, const void* q, const void* k,
                           const void* v, const float* g, const float* beta, const float* state,
                           void* o, unsigned int* status, gdn_stream_t stream) {
    using namespace gdn;
    const gdn_status s = check_tree(N, M, H, dk, dv, dtype, gate);
    if (s != GDN_OK) return s;
    if (!isfinite(scale)) return GDN_ERR_INVALID_ARG;
    if (!parent || !q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(state, 16) ||
        !aligned(o, 16) || !aligned(parent, 4) || !aligned(g, 4) || !aligned(beta, 4) ||
        !aligned(status, 4))
        return GDN_ERR_INVALID_ARG;
    if (gate == GDN_GATE_CHANNEL && !aligned(g, 16)) return GDN_ERR_INVALID_ARG;  // 16-byte copies of g rows
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    auto run = [&](auto kda) {
        constexpr bool K = decltype(kda)::value;
        if (M <= 32) return launch_verify<32, K>(N, M, H, scale, parent, q, k, v, g, beta, state, o, status, st);
        return launch_verify<64, K>(N, M, H, scale, parent, q, k, v, g, beta, state, o, status, st);
    };
    const bool fine = gate == GDN_GATE_CHANNEL ? run(std::true_type{}) : run(std::false_type{});
    if (!fine) return GDN_ERR_CUDA;
    return launched();
}

gdn_status gdn_tree_commit(int N, int M, int H, int dk, int dv, gdn_dtype dtype, gdn_gate gate,
                           const int* parent, const int* accepted, const void* k, const void* v,
                           const float* g, const float* beta, float* state, unsigned int* status,
                           gdn_stream_t stream) {
    using namespace gdn;
    const gdn_status s = check_tree(N, M, H, dk, dv, dtype, gate);
    if (s != GDN_OK) return s;
    if (!parent || !accepted || !k || !v || !g || !beta || !state) return GDN_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(state, 16) || !aligned(parent, 4) ||
        !aligned(accepted, 4) || !aligned(g, 4) || !aligned(beta, 4) || !aligned(status, 4))
        return GDN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    auto run = [&](auto kda) {
        constexpr bool K = decltype(kda)::value;
        const int smem = sizeof(CommitSmem<K>);
        cudaFuncSetAttribute(tree_commit_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        GDN_LAUNCH("tree_commit", st,
                   (tree_commit_kernel<K><<<(unsigned)(N * H), TREE_THREADS, smem, st>>>(
                       M, H, parent, accepted, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, g,
                       beta, state, status)));
    };
    if (gate == GDN_GATE_CHANNEL) run(std::true_type{});
    else run(std::false_type{});
    return launched();
}

}  // extern "C"
