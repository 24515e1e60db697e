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

namespace gdn {
namespace {

constexpr int TD = 128;           // d_k = d_v
constexpr int TREE_THREADS = 256;  // 8 warps
constexpr int kMaxTreeNodes = 64;

template <int MP, bool KDA>
struct TreeSmem {
    __nv_bfloat16 K[MP * TD];  // Swz<128>; rows of U (value index as column) once W is built
    __nv_bfloat16 Q[MP * TD];
    __nv_bfloat16 V[MP * TD];
    union {
        float A[MP][MP + 1];          // masked, decayed beta K K^T
        __nv_bfloat16 Wn[MP * TD];    // -W, Swz<128>
    };
    float T[MP][MP + 1];              // (I + A)^{-1}
    alignas(128) __nv_bfloat16 Tw[MP * 64];  // T diag(beta e^G), Swz<64> (columns < MP used)
    __nv_bfloat16 Tu[MP * 64];        // T diag(beta)
    __nv_bfloat16 P[MP * 64];
    float G[MP], g[MP], beta[MP];
    unsigned long long anc[MP];
    int par[MP], depth[MP];
    int maxdepth;
    alignas(16) float Gc[KDA ? MP : 1][TD];  // channel gate: per-key sums of g over each root path (16-byte copies)
};

// One CTA per (sequence n, head h).  MB = number of 16-node blocks.
// Channel gate (KDA): g_i is a vector over the keys, G_i its sum over the root
// path, and every decay e^{G_i - G_j} (j an ancestor of i) carries the key
// index, so A and P sum k_i k_j e^{G_i - G_j} (q_i k_j e^{G_i - G_j}) over the
// keys pair by pair; W and the read-out take K .* e^G and Q .* e^G.
template <int MB, bool KDA>
__global__ void __launch_bounds__(TREE_THREADS, MB <= 2 ? 4 : 2)  // 4 CTAs per SM up to 32 nodes
tree_verify_kernel(int M, int H, float scale, const int* __restrict__ parent,
                   const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                   const float* __restrict__ beta, const float* __restrict__ state,
                   __nv_bfloat16* __restrict__ o, unsigned int* status) {
    constexpr int MP = 16 * MB;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    TreeSmem<MP, KDA>& s = *reinterpret_cast<TreeSmem<MP, KDA>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nh = blockIdx.x, n = nh / H, h = nh % H;
    const size_t rs = (size_t)H * TD;                        // token row stride
    const size_t row0 = ((size_t)n * M * H + h) * TD;       // node 0 of (n, h)

    // ---- loads: node tokens into shared tiles; the state is pulled into L2
    // now and read as MMA fragments in the last phase ------------------------
    const float* S0 = state + (size_t)nh * TD * TD;
    if (tid < 4) bulk_prefetch_l2(S0 + tid * (TD * TD / 4), TD * TD);  // 4 x 16 KiB
    if (tid == 0) s.maxdepth = 0;
    load_tile_async<TD>(s.K, k + row0, rs, MP, M, tid, TREE_THREADS);
    load_tile_async<TD>(s.Q, q + row0, rs, MP, M, tid, TREE_THREADS);
    load_tile_async<TD>(s.V, v + row0, rs, MP, M, tid, TREE_THREADS);
    cp_async_commit();
    if (tid < MP) {
        int p = -1;
        float gi = 0.f, bi = 0.f;
        if (tid < M) {
            p = parent[(size_t)n * M + tid];
            if (p < -1 || p >= tid) {  // not a tree in topological order
                if (status) atomicOr(status, 2u);
                p = -1;
            }
            if (!KDA) gi = g[((size_t)n * M + tid) * H + h];
            bi = beta[((size_t)n * M + tid) * H + h];
        }
        s.par[tid] = p;
        s.g[tid] = gi;
        s.beta[tid] = bi;
    }
    if constexpr (KDA) {  // per-key gates of every node (zero past M)
        for (int e = tid; e < MP * TD / 4; e += TREE_THREADS) {
            const int i = e / (TD / 4), c4 = e % (TD / 4);
            cp_async16_zfill(&s.Gc[i][4 * c4], g + (((size_t)n * M + (i < M ? i : 0)) * H + h) * TD + 4 * c4,
                             i < M);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
    __syncthreads();
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
    __syncthreads();

    // ---- A (warps 0-3) and P (warps 4-7): 16 node rows each -----------------
    if constexpr (KDA) {
        // ancestor pairs (and, for P, the node itself) only; a warp per pair,
        // a lane per 4 keys; the decays are e^{G_i - G_j} <= 1 key by key
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
                const uint2 ki = *reinterpret_cast<const uint2*>(&s.K[swz<TD>(i, c)]);
                const uint2 kj = *reinterpret_cast<const uint2*>(&s.K[swz<TD>(j, c)]);
                const uint2 qi = *reinterpret_cast<const uint2*>(&s.Q[swz<TD>(i, c)]);
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
    } else {
    {
        const int mat = warp >> 2, mb = warp & 3;
        if (mb < MB) {
            float acc[2 * MB][4];
#pragma unroll
            for (int t = 0; t < 2 * MB; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < TD / 16; ++kk) {
                uint32_t a[4];
                lda<TD>(a, mat ? s.Q : s.K, 16 * mb, 16 * kk);
#pragma unroll
                for (int np = 0; np < MB; ++np) {
                    uint32_t b[4];
                    ldb_nk<TD>(b, s.K, 16 * np, 16 * kk);
                    mma16816(acc[2 * np], a, b[0], b[1]);
                    mma16816(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int t = 0; t < 2 * MB; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 16 * mb + (lane >> 2) + 8 * (e >> 1);
                    const int j = 8 * t + 2 * (lane & 3) + (e & 1);
                    const bool is_anc = (s.anc[i] >> j) & 1ull;
                    if (mat == 0) {
                        s.A[i][j] = is_anc ? s.beta[i] * __expf(s.G[i] - s.G[j]) * acc[t][e] : 0.f;
                    } else {
                        const float pv = (is_anc || j == i) ? scale * __expf(s.G[i] - s.G[j]) * acc[t][e] : 0.f;
                        s.P[swz<64>(i, j)] = __float2bfloat16_rn(pv);
                    }
                }
        }
    }
    __syncthreads();

    }
    // ---- T = (I + A)^{-1}, one tree level at a time --------------------------
    // Row i of T is e_i - sum over ancestors l of A_il T_l, and T_ic is non-zero
    // only for c an ancestor of i or i itself; so every node of one depth is
    // solved at once from the rows of shallower nodes (a chain: one per level).
    {
        const int levels = s.maxdepth;
        for (int d = 0; d <= levels; ++d) {
            for (int e = tid; e < MP * MP; e += TREE_THREADS) {
                const int i = e / MP, c = e % MP;
                if (s.depth[i] != d) continue;
                const unsigned long long ai = s.anc[i];
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
            __syncthreads();
        }
    }
    for (int e = tid; e < MP * MP; e += TREE_THREADS) {
        const int i = e / MP, j = e % MP;
        const float t = s.T[i][j] * s.beta[j];
        s.Tw[swz<64>(i, j)] = __float2bfloat16_rn(KDA ? t : t * __expf(s.G[j]));
        s.Tu[swz<64>(i, j)] = __float2bfloat16_rn(t);
    }
    if constexpr (KDA) {  // K .* e^G (the rows of W) and Q .* e^G (the read-out), in place
        for (int e = tid; e < MP * TD / 2; e += TREE_THREADS) {
            const int i = e / (TD / 2), c = 2 * (e % (TD / 2));
            const float d0 = __expf(s.Gc[i][c]), d1 = __expf(s.Gc[i][c + 1]);
            uint32_t* kp = reinterpret_cast<uint32_t*>(&s.K[swz<TD>(i, c)]);
            uint32_t* qp = reinterpret_cast<uint32_t*>(&s.Q[swz<TD>(i, c)]);
            const float2 kv = unpack_bf16(*kp), qv = unpack_bf16(*qp);
            *kp = pack_bf16(kv.x * d0, kv.y * d1);
            *qp = pack_bf16(qv.x * d0, qv.y * d1);
        }
    }
    __syncthreads();

    // ---- -W = -T diag(beta e^G) K: 16 node rows x 64 key columns per warp ----
    {
        const int mb = warp & 3, c0 = 64 * (warp >> 2);
        if (mb < MB) {
            float acc[8][4];
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < MB; ++kk) {
                uint32_t a[4];
                lda<64>(a, s.Tw, 16 * mb, 16 * kk);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b[4];
                    ldb_kn<TD>(b, s.K, 16 * kk, c0 + 16 * np);
                    mma16816(acc[2 * np], a, b[0], b[1]);
                    mma16816(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float ng[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) ng[e] = -acc[t][e];
                st_c<TD>(s.Wn, 16 * mb, c0 + 8 * t, ng);
            }
        }
    }
    __syncthreads();  // K is read for the last time above; U takes its place

    // ---- U = U~ - W S0^T and O = scale e^G Q S0^T + P U, value rows a0..a0+15 ----
    const int a0 = 16 * warp;
    __nv_bfloat16* Ub = s.K;
    float accu[MB][2][4], acco[MB][2][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) { accu[mb][nt][e] = 0.f; acco[mb][nt][e] = 0.f; }
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int kk = 0; kk <= mb; ++kk) {  // T is lower triangular
            uint32_t a[4], b[4];
            lda<64>(a, s.Tu, 16 * mb, 16 * kk);
            ldb_kn<TD>(b, s.V, 16 * kk, a0);
            mma16816(accu[mb][0], a, b[0], b[1]);
            mma16816(accu[mb][1], a, b[2], b[3]);
        }
    // B fragments of S0^T (B[k = c][n = a] = S0[a][c]) straight from L2, one
    // K = 16 step at a time, shared by every node block.
    const float* srow0 = S0 + (size_t)(a0 + (lane >> 2)) * TD + 2 * (lane & 3);
    const float* srow1 = srow0 + 8 * TD;
#pragma unroll
    for (int kk = 0; kk < TD / 16; ++kk) {
        const float2 x0 = __ldcs(reinterpret_cast<const float2*>(srow0 + 16 * kk));
        const float2 y0 = __ldcs(reinterpret_cast<const float2*>(srow0 + 16 * kk + 8));
        const float2 x1 = __ldcs(reinterpret_cast<const float2*>(srow1 + 16 * kk));
        const float2 y1 = __ldcs(reinterpret_cast<const float2*>(srow1 + 16 * kk + 8));
        const uint32_t b00 = pack_bf16(x0.x, x0.y), b01 = pack_bf16(y0.x, y0.y);
        const uint32_t b10 = pack_bf16(x1.x, x1.y), b11 = pack_bf16(y1.x, y1.y);
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
            uint32_t a[4];
            lda<TD>(a, s.Wn, 16 * mb, 16 * kk);
            mma16816(accu[mb][0], a, b00, b01);
            mma16816(accu[mb][1], a, b10, b11);
            lda<TD>(a, s.Q, 16 * mb, 16 * kk);
            mma16816(acco[mb][0], a, b00, b01);
            mma16816(acco[mb][1], a, b10, b11);
        }
    }
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        st_c<TD>(Ub, 16 * mb, a0, accu[mb][0]);
        st_c<TD>(Ub, 16 * mb, a0 + 8, accu[mb][1]);
        const int r = 16 * mb + (lane >> 2);
        const float f0 = KDA ? scale : scale * __expf(s.G[r]), f1 = KDA ? scale : scale * __expf(s.G[r + 8]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            acco[mb][nt][0] *= f0; acco[mb][nt][1] *= f0;
            acco[mb][nt][2] *= f1; acco[mb][nt][3] *= f1;
        }
    }
    __syncwarp();  // this warp's U columns, written above, are all it reads below
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
#pragma unroll
        for (int kk = 0; kk <= mb; ++kk) {  // P is lower triangular
            uint32_t a[4], b[4];
            lda<64>(a, s.P, 16 * mb, 16 * kk);
            ldb_kn<TD>(b, Ub, 16 * kk, a0);
            mma16816(acco[mb][0], a, b[0], b[1]);
            mma16816(acco[mb][1], a, b[2], b[3]);
        }
        const int r = 16 * mb + (lane >> 2);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = a0 + 8 * nt + 2 * (lane & 3);
            if (r < M)
                *reinterpret_cast<uint32_t*>(o + row0 + (size_t)r * rs + col) =
                    pack_bf16(acco[mb][nt][0], acco[mb][nt][1]);
            if (r + 8 < M)
                *reinterpret_cast<uint32_t*>(o + row0 + (size_t)(r + 8) * rs + col) =
                    pack_bf16(acco[mb][nt][2], acco[mb][nt][3]);
        }
    }
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
    extern __shared__ __align__(128) unsigned char smem_raw[];
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

template <int MB, bool KDA>
void launch_verify(int N, int M, int H, float scale, const int* parent, const void* q,
                   const void* k, const void* v, const float* g, const float* beta,
                   const float* state, void* o, unsigned int* status, cudaStream_t st) {
    const int smem = sizeof(TreeSmem<16 * MB, KDA>);
    cudaFuncSetAttribute(tree_verify_kernel<MB, KDA>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tree_verify", st,
               (tree_verify_kernel<MB, KDA><<<(unsigned)(N * H), TREE_THREADS, smem, st>>>(
                   M, H, scale, parent, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                   (const __nv_bfloat16*)v, g, beta, state, (__nv_bfloat16*)o, status)));
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
        switch ((M + 15) / 16) {
            case 1: launch_verify<1, K>(N, M, H, scale, parent, q, k, v, g, beta, state, o, status, st); break;
            case 2: launch_verify<2, K>(N, M, H, scale, parent, q, k, v, g, beta, state, o, status, st); break;
            case 3: launch_verify<3, K>(N, M, H, scale, parent, q, k, v, g, beta, state, o, status, st); break;
            default: launch_verify<4, K>(N, M, H, scale, parent, q, k, v, g, beta, state, o, status, st); break;
        }
    };
    if (gate == GDN_GATE_CHANNEL) run(std::true_type{});
    else run(std::false_type{});
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
