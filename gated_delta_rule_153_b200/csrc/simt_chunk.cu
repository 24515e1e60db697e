// simt_chunk.cu -- chunkwise gated delta rule in plain fp32 SIMT arithmetic.
//
// This is the path for GDN_F32 (fp32 end to end, no tf32) and for head dims
// the tensor-core kernels do not cover.  One CTA walks one (b, h) stream
// chunk by chunk; every chunk-local matrix lives in a per-(b,h) slice of the
// caller's workspace.  The algebra is the chunkwise (WY / UT transform) form
// from "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper
// review), sections "Goal" and "Method"; per chunk of L tokens with S0 the
// state entering it and G the within-chunk cumsum of the log-gate:
//   A = strict_lower(diag(beta) (K K^T .* D)),  D_ij = exp(G_i - G_j)
//       (channel gate: the decay sits inside the contraction, per channel)
//   T = (I + A)^{-1}                      (forward substitution)
//   W = T diag(beta e^G) K,  U~ = T diag(beta) V,  U = U~ - W S0^T
//   O = (Q e^G) S0^T + lower(Q K^T .* D) U
//   S = e^{G_last} S0 + U^T (K e^{G_last - G})
// The backward is reverse-mode through exactly these equations.
#include "common.cuh"
#include "internal.h"

namespace gdn {
namespace {

enum Buf {
    bQ, bK, bV, bG, bBeta, bM, bA, bP, bT, bKg, bVb, bW, bUt, bU, bQg, bKt, bS, bO,
    // backward only
    bdO, bdU, bdP, bdQg, bdKt, bdW, bdS0, bdT, bdKg, bdVb, bdA, bTmp, bD, bdG, bdQ, bdK, bdB,
    bdS, NBUF
};

struct Lay {
    size_t off[NBUF + 1];
    size_t per_bh;  // floats per (b,h), chunk scratch only
};

__host__ __device__ inline Lay make_lay(int C, int dk, int dv, bool channel, bool bwd) {
    const size_t CC = (size_t)C * C, Cdk = (size_t)C * dk, Cdv = (size_t)C * dv,
                 S = (size_t)dv * dk, Cg = channel ? Cdk : (size_t)C;
    size_t sz[NBUF] = {Cdk, Cdk, Cdv, Cg, (size_t)C, CC, CC, CC, CC, Cdk, Cdv, Cdk, Cdv, Cdv,
                       Cdk, Cdk, S, Cdv,
                       Cdv, Cdv, CC, Cdk, Cdk, Cdk, S, CC, Cdk, Cdv, CC, CC, CC, Cg, Cdk, Cdk,
                       (size_t)C, S};
    Lay l;
    size_t o = 0;
    const int n = bwd ? NBUF : (int)bdO;
    for (int i = 0; i < NBUF; ++i) {
        l.off[i] = o;
        if (i < n) o += (sz[i] + 31) & ~(size_t)31;  // 128-byte aligned slices
    }
    l.off[NBUF] = o;
    l.per_bh = o;
    return l;
}

// out[m*ldo+n] = alpha * sum_k A(m,k) B(k,n) (+ out if acc); A(m,k) = ta ? a[k*lda+m] :
// a[m*lda+k], B(k,n) = tb ? b[n*ldb+k] : b[k*ldb+n].  `out` aliases neither input.
__device__ void mm(float* out, int ldo, const float* a, int lda, bool ta, const float* b,
                   int ldb, bool tb, int M, int N, int K, float alpha, bool acc) {
    for (int e = threadIdx.x; e < M * N; e += blockDim.x) {
        const int m = e / N, n = e % N;
        float s = 0.f;
        for (int kk = 0; kk < K; ++kk)
            s += (ta ? a[(size_t)kk * lda + m] : a[(size_t)m * lda + kk]) *
                 (tb ? b[(size_t)n * ldb + kk] : b[(size_t)kk * ldb + n]);
        out[(size_t)m * ldo + n] = alpha * s + (acc ? out[(size_t)m * ldo + n] : 0.f);
    }
    __syncthreads();
}

struct Args {
    int B, T, H, dk, dv, C, NT;
    float scale;
    const void *q, *k, *v, *dO;
    const float *g, *beta, *h0, *dhT;
    void *o, *dq, *dkk, *dvv;
    float *hT, *dg, *dbeta, *dh0;
    float* ws;       // past the status bytes
    float* s0all;    // backward: chunk-start states, [B*H][NT][dv*dk]
};

// Loads chunk n of stream (b,h) and builds every chunk-local matrix that
// depends only on the inputs and on S0 (the state entering the chunk).
// Returns L, the number of tokens in the chunk.
template <typename Tin, bool CH>
__device__ int chunk_prep(const Args& a, float* const* B, const float* S0, int b, int h, int n) {
    const int dk = a.dk, dv = a.dv, gd = CH ? dk : 1;
    const int t0 = n * a.C;
    const int L = min(a.C, a.T - t0);
    const int tid = threadIdx.x, nt = blockDim.x;
    const Tin* q = (const Tin*)a.q;
    const Tin* k = (const Tin*)a.k;
    const Tin* v = (const Tin*)a.v;
    for (int e = tid; e < L * dk; e += nt) {
        const int i = e / dk, c = e % dk;
        const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
        B[bQ][e] = a.scale * to_f(q[th * dk + c]);
        B[bK][e] = to_f(k[th * dk + c]);
        if (CH) B[bG][e] = a.g[th * dk + c];
    }
    for (int e = tid; e < L * dv; e += nt) {
        const int i = e / dv, c = e % dv;
        const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
        B[bV][e] = to_f(v[th * dv + c]);
    }
    for (int i = tid; i < L; i += nt) {
        const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
        B[bBeta][i] = a.beta[th];
        if (!CH) B[bG][i] = a.g[th];
    }
    __syncthreads();
    // within-chunk cumulative log-decay, one column per thread
    for (int c = tid; c < gd; c += nt)
        for (int i = 1; i < L; ++i) B[bG][i * gd + c] += B[bG][(i - 1) * gd + c];
    __syncthreads();
    const float* G = B[bG];
    // decayed products, pairwise exponent G_i - G_j <= 0 (never overflows)
    for (int e = tid; e < L * L; e += nt) {
        const int i = e / L, j = e % L;
        float m = 0.f, p = 0.f;
        if (j <= i) {
            if (CH) {
                for (int c = 0; c < dk; ++c) {
                    const float d = expf(G[i * dk + c] - G[j * dk + c]);
                    m += B[bK][i * dk + c] * B[bK][j * dk + c] * d;
                    p += B[bQ][i * dk + c] * B[bK][j * dk + c] * d;
                }
            } else {
                for (int c = 0; c < dk; ++c) {
                    m += B[bK][i * dk + c] * B[bK][j * dk + c];
                    p += B[bQ][i * dk + c] * B[bK][j * dk + c];
                }
                const float d = expf(G[i] - G[j]);
                m *= d;
                p *= d;
            }
        }
        B[bM][e] = (j < i) ? m : 0.f;
        B[bA][e] = (j < i) ? B[bBeta][i] * m : 0.f;
        B[bP][e] = p;
        B[bT][e] = (i == j) ? 1.f : 0.f;
    }
    __syncthreads();
    // UT transform: T = (I + A)^{-1} by forward substitution, row by row
    for (int i = 1; i < L; ++i) {
        for (int c = tid; c < i; c += nt) {
            float s = 0.f;
            for (int j = c; j < i; ++j) s += B[bA][i * L + j] * B[bT][j * L + c];
            B[bT][i * L + c] = -s;
        }
        __syncthreads();
    }
    for (int e = tid; e < L * dk; e += nt) {
        const int i = e / dk, c = e % dk;
        const float Gi = CH ? G[e] : G[i];
        const float Gl = CH ? G[(L - 1) * dk + c] : G[L - 1];
        const float eg = expf(Gi);
        B[bKg][e] = B[bBeta][i] * eg * B[bK][e];
        B[bQg][e] = eg * B[bQ][e];
        B[bKt][e] = expf(Gl - Gi) * B[bK][e];
    }
    for (int e = tid; e < L * dv; e += nt) B[bVb][e] = B[bBeta][e / dv] * B[bV][e];
    __syncthreads();
    mm(B[bW], dk, B[bT], L, false, B[bKg], dk, false, L, dk, L, 1.f, false);
    mm(B[bUt], dv, B[bT], L, false, B[bVb], dv, false, L, dv, L, 1.f, false);
    for (int e = tid; e < L * dv; e += nt) B[bU][e] = B[bUt][e];
    __syncthreads();
    mm(B[bU], dv, B[bW], dk, false, S0, dk, true, L, dv, dk, -1.f, true);  // U = U~ - W S0^T
    return L;
}

// S <- decay(S) + U^T Kt  (decay = e^{G_last} per key column)
template <bool CH>
__device__ void state_update(float* const* B, float* S, int L, int dk, int dv) {
    const float* G = B[bG];
    for (int e = threadIdx.x; e < dv * dk; e += blockDim.x) {
        const int c = e % dk;
        S[e] *= expf(CH ? G[(L - 1) * dk + c] : G[L - 1]);
    }
    __syncthreads();
    mm(S, dk, B[bU], dv, true, B[bKt], dk, false, dv, dk, L, 1.f, true);
}

template <typename Tin, bool CH>
__global__ void __launch_bounds__(256) simt_fwd_kernel(Args a) {
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int dk = a.dk, dv = a.dv;
    const Lay lay = make_lay(a.C, dk, dv, CH, false);
    float* base = a.ws + (size_t)bh * lay.per_bh;
    float* B[NBUF];
    for (int i = 0; i < NBUF; ++i) B[i] = base + lay.off[i];
    float* S = B[bS];
    for (int e = threadIdx.x; e < dv * dk; e += blockDim.x)
        S[e] = a.h0 ? a.h0[(size_t)bh * dv * dk + e] : 0.f;
    __syncthreads();
    Tin* o = (Tin*)a.o;
    for (int n = 0; n < a.NT; ++n) {
        const int L = chunk_prep<Tin, CH>(a, B, S, b, h, n);
        // O = Qg S0^T + P U
        mm(B[bO], dv, B[bQg], dk, false, S, dk, true, L, dv, dk, 1.f, false);
        mm(B[bO], dv, B[bP], L, false, B[bU], dv, false, L, dv, L, 1.f, true);
        for (int e = threadIdx.x; e < L * dv; e += blockDim.x) {
            const int i = e / dv, c = e % dv;
            const size_t th = ((size_t)b * a.T + n * a.C + i) * a.H + h;
            o[th * dv + c] = from_f<Tin>(B[bO][e]);
        }
        state_update<CH>(B, S, L, dk, dv);
    }
    if (a.hT)
        for (int e = threadIdx.x; e < dv * dk; e += blockDim.x)
            a.hT[(size_t)bh * dv * dk + e] = S[e];
}

template <typename Tin, bool CH>
__global__ void __launch_bounds__(256) simt_bwd_kernel(Args a) {
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int dk = a.dk, dv = a.dv, C = a.C, gd = CH ? dk : 1;
    const int tid = threadIdx.x, nt = blockDim.x;
    const Lay lay = make_lay(C, dk, dv, CH, true);
    float* base = a.ws + (size_t)bh * lay.per_bh;
    float* B[NBUF];
    for (int i = 0; i < NBUF; ++i) B[i] = base + lay.off[i];
    float* S0all = a.s0all + (size_t)bh * a.NT * dv * dk;
    const size_t SS = (size_t)dv * dk;

    // forward sweep: keep the state entering every chunk
    float* S = B[bS];
    for (size_t e = tid; e < SS; e += nt) S[e] = a.h0 ? a.h0[(size_t)bh * SS + e] : 0.f;
    __syncthreads();
    for (int n = 0; n < a.NT; ++n) {
        for (size_t e = tid; e < SS; e += nt) S0all[(size_t)n * SS + e] = S[e];
        __syncthreads();
        const int L = chunk_prep<Tin, CH>(a, B, S, b, h, n);
        state_update<CH>(B, S, L, dk, dv);
    }
    // reverse sweep
    float* dS = B[bdS];
    for (size_t e = tid; e < SS; e += nt) dS[e] = a.dhT ? a.dhT[(size_t)bh * SS + e] : 0.f;
    __syncthreads();
    const Tin* dO = (const Tin*)a.dO;
    for (int n = a.NT - 1; n >= 0; --n) {
        const float* S0 = S0all + (size_t)n * SS;
        const int L = chunk_prep<Tin, CH>(a, B, S0, b, h, n);
        const int t0 = n * C;
        const float* G = B[bG];
        for (int e = tid; e < L * dv; e += nt) {
            const int i = e / dv, c = e % dv;
            const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
            B[bdO][e] = to_f(dO[th * dv + c]);
        }
        for (int e = tid; e < L * gd; e += nt) B[bdG][e] = 0.f;
        for (int e = tid; e < L * dk; e += nt) { B[bdQ][e] = 0.f; B[bdK][e] = 0.f; }
        for (int i = tid; i < L; i += nt) B[bdB][i] = 0.f;
        __syncthreads();
        // O = Qg S0^T + P U ;  S_L = decay(S0) + U^T Kt ;  U = U~ - W S0^T
        mm(B[bdU], dv, B[bP], L, true, B[bdO], dv, false, L, dv, L, 1.f, false);
        mm(B[bdU], dv, B[bKt], dk, false, dS, dk, true, L, dv, dk, 1.f, true);
        mm(B[bdP], L, B[bdO], dv, false, B[bU], dv, true, L, L, dv, 1.f, false);
        mm(B[bdQg], dk, B[bdO], dv, false, S0, dk, false, L, dk, dv, 1.f, false);
        mm(B[bdKt], dk, B[bU], dv, false, dS, dk, false, L, dk, dv, 1.f, false);
        mm(B[bdW], dk, B[bdU], dv, false, S0, dk, false, L, dk, dv, -1.f, false);
        for (size_t e = tid; e < SS; e += nt) {
            const int c = (int)(e % dk);
            B[bdS0][e] = dS[e] * expf(CH ? G[(L - 1) * dk + c] : G[L - 1]);
        }
        __syncthreads();
        mm(B[bdS0], dk, B[bdO], dv, true, B[bQg], dk, false, dv, dk, L, 1.f, true);
        mm(B[bdS0], dk, B[bdU], dv, true, B[bW], dk, false, dv, dk, L, -1.f, true);
        // d G_last from the decay of S0: e^{G_last} <dS, S0> (per column for the channel gate)
        if (CH) {
            for (int c = tid; c < dk; c += nt) {
                float s = 0.f;
                for (int r = 0; r < dv; ++r) s += dS[(size_t)r * dk + c] * S0[(size_t)r * dk + c];
                B[bdG][(L - 1) * dk + c] += expf(G[(L - 1) * dk + c]) * s;
            }
        } else {
            __shared__ float red[32];
            float s = 0.f;
            for (size_t e = tid; e < SS; e += nt) s += dS[e] * S0[e];
            s = warp_sum(s);
            if ((tid & 31) == 0) red[tid >> 5] = s;
            __syncthreads();
            if (tid == 0) {
                float t = 0.f;
                for (int w = 0; w < (nt >> 5); ++w) t += red[w];
                B[bdG][L - 1] += expf(G[L - 1]) * t;
            }
        }
        __syncthreads();
        // W = T Kg ; U~ = T Vb
        mm(B[bdT], L, B[bdW], dk, false, B[bKg], dk, true, L, L, dk, 1.f, false);
        mm(B[bdT], L, B[bdU], dv, false, B[bVb], dv, true, L, L, dv, 1.f, true);
        mm(B[bdKg], dk, B[bT], L, true, B[bdW], dk, false, L, dk, L, 1.f, false);
        mm(B[bdVb], dv, B[bT], L, true, B[bdU], dv, false, L, dv, L, 1.f, false);
        // T = (I + A)^{-1}:  dA = strict_lower(-T^T dT T^T)
        mm(B[bTmp], L, B[bdT], L, false, B[bT], L, true, L, L, L, 1.f, false);
        mm(B[bdA], L, B[bT], L, true, B[bTmp], L, false, L, L, L, -1.f, false);
        for (int e = tid; e < L * L; e += nt) {
            const int i = e / L, j = e % L;
            if (j >= i) B[bdA][e] = 0.f;
            if (j > i) B[bdP][e] = 0.f;  // O uses lower(P) only
            if (!CH) B[bD][e] = (j <= i) ? expf(G[i] - G[j]) : 0.f;
        }
        __syncthreads();
        // per-token terms: dv, dbeta from V, and the row-scaled factors Kg, Qg, Kt
        Tin* dvp = (Tin*)a.dvv;
        for (int e = tid; e < L * dv; e += nt) {
            const int i = e / dv, c = e % dv;
            const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
            dvp[th * dv + c] = from_f<Tin>(B[bBeta][i] * B[bdVb][e]);
        }
        for (int i = tid; i < L; i += nt) {
            float s = 0.f, sA = 0.f;
            for (int c = 0; c < dv; ++c) s += B[bdVb][i * dv + c] * B[bV][i * dv + c];
            for (int j = 0; j < i; ++j) sA += B[bdA][i * L + j] * B[bM][i * L + j];
            B[bdB][i] += s + sA;
        }
        __syncthreads();
        for (int e = tid; e < L * dk; e += nt) {
            const int i = e / dk, c = e % dk;
            const float Gi = CH ? G[e] : G[i];
            const float Gl = CH ? G[(L - 1) * dk + c] : G[L - 1];
            const float eg = expf(Gi), et = expf(Gl - Gi), bi = B[bBeta][i];
            B[bdK][e] += bi * eg * B[bdKg][e] + et * B[bdKt][e];
            B[bdQ][e] += eg * B[bdQg][e];
            if (CH) {
                const float hk = B[bdKg][e] * B[bK][e] * eg;
                B[bdG][e] += bi * hk + eg * B[bdQg][e] * B[bQ][e] - et * B[bdKt][e] * B[bK][e];
            }
        }
        if (CH) {
            // beta gets sum_c dKg K e^G; G_last gets sum_i e^{G_last-G_i} dKt K per column
            __syncthreads();
            for (int i = tid; i < L; i += nt) {
                float s = 0.f;
                for (int c = 0; c < dk; ++c)
                    s += B[bdKg][i * dk + c] * B[bK][i * dk + c] * expf(G[i * dk + c]);
                B[bdB][i] += s;
            }
            for (int c = tid; c < dk; c += nt) {
                float s = 0.f;
                for (int i = 0; i < L; ++i)
                    s += expf(G[(L - 1) * dk + c] - G[i * dk + c]) * B[bdKt][i * dk + c] *
                         B[bK][i * dk + c];
                B[bdG][(L - 1) * dk + c] += s;
            }
        } else {
            __syncthreads();
            for (int i = tid; i < L; i += nt) {
                float hk = 0.f, hq = 0.f, ht = 0.f;
                for (int c = 0; c < dk; ++c) {
                    hk += B[bdKg][i * dk + c] * B[bK][i * dk + c];
                    hq += B[bdQg][i * dk + c] * B[bQ][i * dk + c];
                    ht += B[bdKt][i * dk + c] * B[bK][i * dk + c];
                }
                const float eg = expf(G[i]), et = expf(G[L - 1] - G[i]);
                B[bdB][i] += eg * hk;
                B[bdG][i] += B[bBeta][i] * eg * hk + eg * hq - et * ht;
                B[bTmp][i] = et * ht;  // collected into G_last below
            }
            __syncthreads();
            if (tid == 0) {
                float s = 0.f;
                for (int i = 0; i < L; ++i) s += B[bTmp][i];
                B[bdG][L - 1] += s;
            }
        }
        __syncthreads();
        // pair terms from A (via dA) and P (via dP); wA = dA .* beta_i
        for (int e = tid; e < L * dk; e += nt) {
            const int i = e / dk, c = e % dk;
            float dk_ = 0.f, dq_ = 0.f, dg_ = 0.f;
            const float Ki = B[bK][e], Qi = B[bQ][e];
            for (int j = 0; j < L; ++j) {
                const float Kj = B[bK][j * dk + c], Qj = B[bQ][j * dk + c];
                if (j <= i) {  // pairs (i, j): i is the later token
                    const float d = CH ? expf(G[e] - G[j * dk + c]) : B[bD][i * L + j];
                    const float wA = B[bdA][i * L + j] * B[bBeta][i];
                    const float dp = B[bdP][i * L + j];
                    dk_ += wA * Kj * d;
                    dq_ += dp * Kj * d;
                    dg_ += (wA * Ki * Kj + dp * Qi * Kj) * d;
                }
                if (j >= i) {  // pairs (j, i): i is the earlier token
                    const float d = CH ? expf(G[j * dk + c] - G[e]) : B[bD][j * L + i];
                    const float wA = B[bdA][j * L + i] * B[bBeta][j];
                    const float dp = B[bdP][j * L + i];
                    dk_ += (wA * Kj + dp * Qj) * d;
                    dg_ -= (wA * Kj * Ki + dp * Qj * Ki) * d;
                }
            }
            B[bdK][e] += dk_;
            B[bdQ][e] += dq_;
            if (CH) B[bdG][e] += dg_;
            else B[bdQg][e] = dg_;  // scalar gate: per-channel partials, summed below
        }
        __syncthreads();
        if (!CH) {
            for (int i = tid; i < L; i += nt) {
                float s = 0.f;
                for (int c = 0; c < dk; ++c) s += B[bdQg][i * dk + c];
                B[bdG][i] += s;
            }
            __syncthreads();
        }
        // write gradients; dg = reverse cumsum of dG inside the chunk
        Tin* dqp = (Tin*)a.dq;
        Tin* dkp = (Tin*)a.dkk;
        for (int e = tid; e < L * dk; e += nt) {
            const int i = e / dk, c = e % dk;
            const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
            dqp[th * dk + c] = from_f<Tin>(a.scale * B[bdQ][e]);
            dkp[th * dk + c] = from_f<Tin>(B[bdK][e]);
        }
        for (int i = tid; i < L; i += nt) {
            const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
            a.dbeta[th] = B[bdB][i];
        }
        for (int c = tid; c < gd; c += nt) {
            float run = 0.f;
            for (int i = L - 1; i >= 0; --i) {
                run += B[bdG][i * gd + c];
                const size_t th = ((size_t)b * a.T + t0 + i) * a.H + h;
                a.dg[th * gd + c] = run;
            }
        }
        for (size_t e = tid; e < SS; e += nt) dS[e] = B[bdS0][e];
        __syncthreads();
    }
    if (a.dh0)
        for (size_t e = tid; e < SS; e += nt) a.dh0[(size_t)bh * SS + e] = dS[e];
}

Args make_args(const gdn_dims& d, void* ws, bool bwd) {
    Args a{};
    a.B = d.B; a.T = d.T; a.H = d.H; a.dk = d.dk; a.dv = d.dv; a.C = d.chunk;
    a.NT = (d.T + d.chunk - 1) / d.chunk;
    a.scale = d.scale;
    const Lay lay = make_lay(d.chunk, d.dk, d.dv, d.gate == GDN_GATE_CHANNEL, bwd);
    a.ws = (float*)((char*)ws + kStatusBytes);
    a.s0all = a.ws + (size_t)d.B * d.H * lay.per_bh;
    return a;
}

}  // namespace

size_t simt_fwd_workspace(const gdn_dims& d) {
    const Lay lay = make_lay(d.chunk, d.dk, d.dv, d.gate == GDN_GATE_CHANNEL, false);
    return kStatusBytes + sizeof(float) * (size_t)d.B * d.H * lay.per_bh;
}

size_t simt_bwd_workspace(const gdn_dims& d) {
    const Lay lay = make_lay(d.chunk, d.dk, d.dv, d.gate == GDN_GATE_CHANNEL, true);
    const size_t NT = (d.T + d.chunk - 1) / d.chunk;
    return kStatusBytes + sizeof(float) * (size_t)d.B * d.H *
                              (lay.per_bh + NT * (size_t)d.dv * d.dk);
}

void launch_simt_fwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* h0, void* o, float* hT,
                     void* ws, cudaStream_t st) {
    Args a = make_args(d, ws, false);
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0; a.o = o; a.hT = hT;
    const int grid = d.B * d.H;
    const bool ch = d.gate == GDN_GATE_CHANNEL;
    if (d.dtype == GDN_BF16) {
        if (ch) GDN_LAUNCH("simt_fwd", st, simt_fwd_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(a));
        else GDN_LAUNCH("simt_fwd", st, simt_fwd_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(a));
    } else {
        if (ch) GDN_LAUNCH("simt_fwd", st, simt_fwd_kernel<float, true><<<grid, 256, 0, st>>>(a));
        else GDN_LAUNCH("simt_fwd", st, simt_fwd_kernel<float, false><<<grid, 256, 0, st>>>(a));
    }
}

void launch_simt_bwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* h0, const void* dO,
                     const float* dhT, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                     float* dh0, void* ws, cudaStream_t st) {
    Args a = make_args(d, ws, true);
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0; a.dO = dO; a.dhT = dhT;
    a.dq = dq; a.dkk = dk; a.dvv = dv; a.dg = dg; a.dbeta = dbeta; a.dh0 = dh0;
    const int grid = d.B * d.H;
    const bool ch = d.gate == GDN_GATE_CHANNEL;
    if (d.dtype == GDN_BF16) {
        if (ch) GDN_LAUNCH("simt_bwd", st, simt_bwd_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(a));
        else GDN_LAUNCH("simt_bwd", st, simt_bwd_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(a));
    } else {
        if (ch) GDN_LAUNCH("simt_bwd", st, simt_bwd_kernel<float, true><<<grid, 256, 0, st>>>(a));
        else GDN_LAUNCH("simt_bwd", st, simt_bwd_kernel<float, false><<<grid, 256, 0, st>>>(a));
    }
}

}  // namespace gdn
