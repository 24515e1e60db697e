// prologue.cu -- the q/k/v prologue of the layer: short causal convolution,
// SiLU and (for q and k) L2 normalisation, forward and backward.
//
// "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper review),
// section "Method": q and k pass through a short convolution and SiLU, then
// L2 normalisation; v takes the same path without the norm.  Read as a causal
// depthwise filter of K <= 4 taps per channel (zeros before the first token),
//     z_t[c] = sum_j w[c][j] x_{t-j}[c],   s = z sigmoid(z),
//     y = s / sqrt(sum_c s_c^2 + eps)   (over the d channels of one head).
// Backward, per token:  ds = (dy - y (y.dy)) / sqrt(|s|^2 + eps) (norm) or dy,
//     dz = ds sigmoid(z) (1 + z (1 - sigmoid(z))),
//     dx_t = sum_j w_j dz_{t+j},   dw_j = sum_t dz_t x_{t-j}.
//
// Both directions are single HBM passes.  A warp owns one head of a run of 8
// tokens (4 in the backward, which holds x and dy) with lane = d/32
// consecutive channels, and issues every load of the run (with its 3-token
// halos) before using any; the head's norm is a warp reduction.  The
// weight gradient is summed per run in registers, per CTA through shared
// memory in warp order, and over CTAs in a fixed order by a second kernel:
// deterministic, no atomics.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "mma.cuh"

namespace gdn {
namespace {

constexpr int KT = 4;          // taps held in registers (K <= KT; missing taps are zero)
constexpr int RUN_F = 8;       // tokens per warp, forward
constexpr int RUN_B = 4;       // tokens per warp, backward (it holds x and dy of a run)
constexpr int PW = 8;          // warps per CTA
constexpr float kNormEps = 1e-6f;

template <typename T, int CPL>
GDN_DEV void store_ch(T* p, const float (&v)[CPL]);
template <>
GDN_DEV void store_ch<__nv_bfloat16, 4>(__nv_bfloat16* p, const float (&v)[4]) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
}
template <>
GDN_DEV void store_ch<__nv_bfloat16, 2>(__nv_bfloat16* p, const float (&v)[2]) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16(v[0], v[1]);
}
template <>
GDN_DEV void store_ch<__nv_bfloat16, 1>(__nv_bfloat16* p, const float (&v)[1]) {
    *p = __float2bfloat16_rn(v[0]);
}
template <>
GDN_DEV void store_ch<float, 4>(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
GDN_DEV void store_ch<float, 2>(float* p, const float (&v)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}
template <>
GDN_DEV void store_ch<float, 1>(float* p, const float (&v)[1]) { *p = v[0]; }

// Work split: a CTA owns PW * RUNT consecutive tokens of one head (b, h); its
// warp w owns the run of RUNT tokens starting at tile start + w * RUNT.  All
// of a run's loads are issued before any of them is used.
struct Tile {
    int b, h, tile, t0, t1;  // t0 >= t1: this warp has no tokens
};
template <int RUNT>
GDN_DEV Tile tile_of(int H, int tiles, int Tn) {
    Tile r;
    r.h = (int)(blockIdx.x % H);
    const int bt = (int)(blockIdx.x / H);
    r.tile = bt % tiles;
    r.b = bt / tiles;
    r.t0 = r.tile * (PW * RUNT) + (threadIdx.x >> 5) * RUNT;
    r.t1 = min(Tn, r.t0 + RUNT);
    return r;
}

// A lane's CPL channels of one token, kept as loaded (bf16 pairs stay packed,
// halving the registers that hold a run in flight).
template <typename T, int CPL> struct Raw;
template <> struct Raw<__nv_bfloat16, 4> { using type = uint2; };
template <> struct Raw<__nv_bfloat16, 2> { using type = uint32_t; };
template <> struct Raw<__nv_bfloat16, 1> { using type = unsigned short; };
template <> struct Raw<float, 4> { using type = float4; };
template <> struct Raw<float, 2> { using type = float2; };
template <> struct Raw<float, 1> { using type = float; };

template <typename T, int CPL>
GDN_DEV typename Raw<T, CPL>::type load_raw(const T* p, bool ok) {
    using R = typename Raw<T, CPL>::type;
    if (ok) return *reinterpret_cast<const R*>(p);
    R z;
    memset(&z, 0, sizeof(R));
    return z;
}
GDN_DEV void unpack(float (&v)[4], uint2 r) {
    const float2 a = unpack_bf16(r.x), b = unpack_bf16(r.y);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
GDN_DEV void unpack(float (&v)[2], uint32_t r) {
    const float2 a = unpack_bf16(r);
    v[0] = a.x; v[1] = a.y;
}
GDN_DEV void unpack(float (&v)[1], unsigned short r) {
    v[0] = __bfloat162float(__ushort_as_bfloat16(r));
}
GDN_DEV void unpack(float (&v)[4], float4 r) { v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w; }
GDN_DEV void unpack(float (&v)[2], float2 r) { v[0] = r.x; v[1] = r.y; }
GDN_DEV void unpack(float (&v)[1], float r) { v[0] = r; }

// The lane's filters: CPL channels x K taps, contiguous in w; with K = KT and
// w 16-byte aligned they are CPL float4 loads, coalesced across the warp.
template <int CPL>
GDN_DEV void load_filters(float (&wr)[CPL][KT], const float* w, int K) {
    if (K == KT && ((uintptr_t)w & 15u) == 0) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(w) + i);
            wr[i][0] = f.x; wr[i][1] = f.y; wr[i][2] = f.z; wr[i][3] = f.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < CPL; ++i)
#pragma unroll
            for (int j = 0; j < KT; ++j) wr[i][j] = j < K ? __ldg(w + i * K + j) : 0.f;
    }
}

// z_t = sum_j w_j x_{t-j} from x_t and the window x_{t-1}, x_{t-2}, x_{t-3}.
template <int CPL>
GDN_DEV void conv_at(float (&z)[CPL], const float (&wr)[CPL][KT], const float (&xv)[CPL],
                     const float (&win)[KT - 1][CPL]) {
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        z[i] = wr[i][0] * xv[i] + wr[i][1] * win[0][i] + wr[i][2] * win[1][i] + wr[i][3] * win[2][i];
}
template <int CPL>
GDN_DEV void shift_in(float (&win)[KT - 1][CPL], const float (&xv)[CPL]) {
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        win[2][i] = win[1][i];
        win[1][i] = win[0][i];
        win[0][i] = xv[i];
    }
}

template <typename T, int CPL, bool NORM>
__global__ void __launch_bounds__(PW * 32, 3)
short_conv_fwd_kernel(int Tn, int H, int K, int tiles, const T* __restrict__ x,
                      const float* __restrict__ w, T* __restrict__ y) {
    using R = typename Raw<T, CPL>::type;
    constexpr int D = 32 * CPL;
    const int lane = threadIdx.x & 31, c0 = lane * CPL;
    constexpr int RUN = RUN_F;
    const Tile r = tile_of<RUN>(H, tiles, Tn);
    if (r.t0 >= r.t1) return;  // whole warps; no block-wide barrier below
    const size_t rs = (size_t)H * D;  // token stride
    const size_t base = ((size_t)r.b * Tn * H + r.h) * D + c0;
    R xs[KT - 1 + RUN];  // x_{t0-3} .. x_{t0+RUN-1}, all in flight at once
#pragma unroll
    for (int u = 0; u < KT - 1 + RUN; ++u) {
        const int t = r.t0 - (KT - 1) + u;
        xs[u] = load_raw<T, CPL>(x + base + (size_t)max(t, 0) * rs, t >= 0 && t < r.t1);
    }
    float wr[CPL][KT], win[KT - 1][CPL];
    load_filters<CPL>(wr, w + ((size_t)r.h * D + c0) * K, K);
#pragma unroll
    for (int j = 0; j < KT - 1; ++j) unpack(win[KT - 2 - j], xs[j]);  // win[0] = x_{t0-1}
    // Straight-line over the run, so the reductions of different tokens
    // overlap; tokens past the end are computed and not stored.
#pragma unroll
    for (int u = 0; u < RUN; ++u) {
        float xv[CPL], s[CPL];
        unpack(xv, xs[u + KT - 1]);
        conv_at<CPL>(s, wr, xv, win);
        shift_in<CPL>(win, xv);
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            s[i] = __fdividef(s[i], 1.f + __expf(-s[i]));
            ss += s[i] * s[i];
        }
        if (NORM) {
            const float inv = rsqrtf(warp_sum(ss) + kNormEps);
#pragma unroll
            for (int i = 0; i < CPL; ++i) s[i] *= inv;
        }
        if (r.t0 + u < r.t1) store_ch<T, CPL>(y + base + (size_t)(r.t0 + u) * rs, s);
    }
}

// dz_t from x_t, the window x_{t-1..t-3} and dy_t (a whole warp: the norm's
// sums are warp reductions).
template <int CPL, bool NORM, typename R>
GDN_DEV void dz_at(float (&dz)[CPL], const float (&wr)[CPL][KT], const float (&xv)[CPL],
                   const float (&win)[KT - 1][CPL], R dyraw) {
    float z[CPL], sg[CPL], sv[CPL], g[CPL];
    conv_at<CPL>(z, wr, xv, win);
    unpack(g, dyraw);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        sg[i] = __fdividef(1.f, 1.f + __expf(-z[i]));
        sv[i] = z[i] * sg[i];
        ss += sv[i] * sv[i];
    }
    if (NORM) {
        const float inv = rsqrtf(warp_sum(ss) + kNormEps);
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) dot += sv[i] * inv * g[i];
        dot = warp_sum(dot);
#pragma unroll
        for (int i = 0; i < CPL; ++i) g[i] = (g[i] - sv[i] * inv * dot) * inv;
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) dz[i] = g[i] * sg[i] * (1.f + z[i] * (1.f - sg[i]));
}

template <int CPL>
GDN_DEV void push_dz(float (&dzw)[KT][CPL], const float (&dz)[CPL]) {
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        dzw[3][i] = dzw[2][i];
        dzw[2][i] = dzw[1][i];
        dzw[1][i] = dzw[0][i];
        dzw[0][i] = dz[i];
    }
}

// dx_te = sum_j w_j dz_{te+j} once dz_{te+KT-1} is in dzw[0] (te in [t0, t1)).
template <typename T, int CPL>
GDN_DEV void emit_dx(T* dxb, size_t rs, const float (&wr)[CPL][KT], const float (&dzw)[KT][CPL],
                     int te, int t0, int t1) {
    if (te < t0 || te >= t1) return;
    float gx[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i)
        gx[i] = wr[i][0] * dzw[3][i] + wr[i][1] * dzw[2][i] + wr[i][2] * dzw[1][i] + wr[i][3] * dzw[0][i];
    store_ch<T, CPL>(dxb + (size_t)te * rs, gx);
}

// The backward: dz over the run and the KT-1 tokens after it (dx of the run
// needs dz_t .. dz_{t+KT-1}), x from KT-1 tokens before the run; dx of token
// t - (KT-1) is emitted once dz_t is known.
template <typename T, int CPL, bool NORM>
__global__ void __launch_bounds__(PW * 32, 2)
short_conv_bwd_kernel(int Tn, int H, int K, int tiles, const T* __restrict__ x,
                      const float* __restrict__ w, const T* __restrict__ dy, T* __restrict__ dx,
                      float* __restrict__ part) {
    using R = typename Raw<T, CPL>::type;
    constexpr int D = 32 * CPL;
    constexpr int RUN = RUN_B;
    constexpr int NZ = RUN + KT - 1;        // dz_{t0} .. dz_{t0+RUN+2}
    constexpr int NX = NZ + KT - 1;         // x_{t0-3} .. x_{t0+RUN+2}
    __shared__ float red[PW][KT][D];  // tap-major: a lane's CPL channels are contiguous
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, c0 = lane * CPL;
    const Tile r = tile_of<RUN>(H, tiles, Tn);
    const bool active = r.t0 < r.t1;  // uniform over the warp
    float wr[CPL][KT], dw[CPL][KT];
    load_filters<CPL>(wr, w + ((size_t)r.h * D + c0) * K, K);
#pragma unroll
    for (int i = 0; i < CPL; ++i)
#pragma unroll
        for (int j = 0; j < KT; ++j) dw[i][j] = 0.f;
    __shared__ float head[PW][KT - 1][D];  // each warp's first KT-1 dz, for the warp before it
    const size_t rs = (size_t)H * D;
    const size_t base = ((size_t)r.b * Tn * H + r.h) * D + c0;
    const bool last = warp == PW - 1;  // recomputes the KT-1 dz past the CTA's tokens
    R xs[NX], dys[NZ];
    float dzw[KT][CPL], win[KT - 1][CPL];  // dzw[j] = dz_{t-j}; win[j] = x_{t-1-j}
#pragma unroll
    for (int j = 0; j < KT; ++j)
#pragma unroll
        for (int i = 0; i < CPL; ++i) dzw[j][i] = 0.f;
    if (active) {
        const int tz = min(Tn, r.t1 + KT - 1);  // tokens that have a dz
#pragma unroll
        for (int u = 0; u < NX; ++u) {  // every load of the run in flight at once
            const int t = r.t0 - (KT - 1) + u;
            const bool need = u < RUN + KT - 1 || last;
            xs[u] = load_raw<T, CPL>(x + base + (size_t)max(t, 0) * rs, need && t >= 0 && t < tz);
        }
#pragma unroll
        for (int u = 0; u < NZ; ++u)
            dys[u] = load_raw<T, CPL>(dy + base + (size_t)(r.t0 + u) * rs,
                                      (u < RUN || last) && r.t0 + u < tz);
#pragma unroll
        for (int j = 0; j < KT - 1; ++j) unpack(win[KT - 2 - j], xs[j]);  // win[0] = x_{t0-1}
        // The run's own tokens, straight-line: past the end dy reads as zero,
        // which gives dz = 0 exactly, so nothing but stores is guarded.
#pragma unroll
        for (int u = 0; u < RUN; ++u) {
            float dz[CPL], xv[CPL];
            unpack(xv, xs[u + KT - 1]);
            dz_at<CPL, NORM>(dz, wr, xv, win, dys[u]);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                dw[i][0] += dz[i] * xv[i];
                dw[i][1] += dz[i] * win[0][i];
                dw[i][2] += dz[i] * win[1][i];
                dw[i][3] += dz[i] * win[2][i];
            }
            if (u < KT - 1) {
#pragma unroll
                for (int i = 0; i < CPL; ++i) head[warp][u][c0 + i] = dz[i];  // contiguous per lane
            }
            shift_in<CPL>(win, xv);
            push_dz<CPL>(dzw, dz);
            emit_dx<T, CPL>(dx + base, rs, wr, dzw, r.t0 + u - (KT - 1), r.t0, r.t1);
        }
    } else {
#pragma unroll
        for (int k = 0; k < KT - 1; ++k)
#pragma unroll
            for (int i = 0; i < CPL; ++i) head[warp][k][c0 + i] = 0.f;
    }
    __syncthreads();
    if (active) {  // dx of the run's last KT-1 tokens needs the next KT-1 dz
#pragma unroll
        for (int k = 0; k < KT - 1; ++k) {
            const int t = r.t0 + RUN + k;
            float dz[CPL];
            if (!last) {
#pragma unroll
                for (int i = 0; i < CPL; ++i) dz[i] = head[warp + 1][k][c0 + i];
            } else if (t < Tn) {  // uniform over the warp
                float xv[CPL];
                unpack(xv, xs[RUN + KT - 1 + k]);
                dz_at<CPL, NORM>(dz, wr, xv, win, dys[RUN + k]);
                shift_in<CPL>(win, xv);
            } else {
#pragma unroll
                for (int i = 0; i < CPL; ++i) dz[i] = 0.f;
            }
            push_dz<CPL>(dzw, dz);
            emit_dx<T, CPL>(dx + base, rs, wr, dzw, t - (KT - 1), r.t0, r.t1);
        }
    }
    // The CTA's weight-gradient partial: warps summed in a fixed order.
#pragma unroll
    for (int j = 0; j < KT; ++j)
#pragma unroll
        for (int i = 0; i < CPL; ++i) red[warp][j][c0 + i] = dw[i][j];
    __syncthreads();
    for (int e = threadIdx.x; e < D * K; e += PW * 32) {
        const int c = e / K, j = e % K;
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < PW; ++q) acc += red[q][j][c];
        part[(size_t)blockIdx.x * D * K + e] = acc;  // slot (b, tile, h) = blockIdx.x
    }
}

// dw[e] = sum over the (b, tile) partials of e, in a fixed order.  A CTA owns
// 32 consecutive e (one per lane); its RW warps take interleaved partials (a
// coalesced 128-byte row each), then their sums are added in warp order.
constexpr int RW = 32;
__global__ void __launch_bounds__(RW * 32)
short_conv_dw_reduce_kernel(const float* __restrict__ part, int nparts, int per,
                            float* __restrict__ dw) {
    __shared__ float red[RW][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    float acc = 0.f;
    if (e < per) {
#pragma unroll 4
        for (int p = warp; p < nparts; p += RW) acc += part[(size_t)p * per + e];
    }
    red[warp][lane] = acc;
    __syncthreads();
    if (warp == 0 && e < per) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < RW; ++q) t += red[q][lane];
        dw[e] = t;
    }
}

int tiles_of(int T, int run) { return (T + PW * run - 1) / (PW * run); }

template <typename T, int CPL>
void launch_fwd(int B, int Tn, int H, int K, bool norm, const void* x, const float* w, void* y,
                cudaStream_t st) {
    const int tiles = tiles_of(Tn, RUN_F);
    const unsigned grid = (unsigned)((long long)B * tiles * H);
    if (norm)
        GDN_LAUNCH("short_conv_fwd", st,
                   (short_conv_fwd_kernel<T, CPL, true><<<grid, PW * 32, 0, st>>>(
                       Tn, H, K, tiles, (const T*)x, w, (T*)y)));
    else
        GDN_LAUNCH("short_conv_fwd", st,
                   (short_conv_fwd_kernel<T, CPL, false><<<grid, PW * 32, 0, st>>>(
                       Tn, H, K, tiles, (const T*)x, w, (T*)y)));
}

template <typename T, int CPL>
void launch_bwd(int B, int Tn, int H, int K, bool norm, const void* x, const float* w,
                const void* dy, void* dx, float* part, cudaStream_t st) {
    const int tiles = tiles_of(Tn, RUN_B);
    const unsigned grid = (unsigned)((long long)B * tiles * H);
    if (norm)
        GDN_LAUNCH("short_conv_bwd", st,
                   (short_conv_bwd_kernel<T, CPL, true><<<grid, PW * 32, 0, st>>>(
                       Tn, H, K, tiles, (const T*)x, w, (const T*)dy, (T*)dx, part)));
    else
        GDN_LAUNCH("short_conv_bwd", st,
                   (short_conv_bwd_kernel<T, CPL, false><<<grid, PW * 32, 0, st>>>(
                       Tn, H, K, tiles, (const T*)x, w, (const T*)dy, (T*)dx, part)));
}

template <typename T>
void dispatch_fwd(int B, int Tn, int H, int d, int K, bool norm, const void* x, const float* w,
                  void* y, cudaStream_t st) {
    if (d == 32) launch_fwd<T, 1>(B, Tn, H, K, norm, x, w, y, st);
    else if (d == 64) launch_fwd<T, 2>(B, Tn, H, K, norm, x, w, y, st);
    else launch_fwd<T, 4>(B, Tn, H, K, norm, x, w, y, st);
}

template <typename T>
void dispatch_bwd(int B, int Tn, int H, int d, int K, bool norm, const void* x, const float* w,
                  const void* dy, void* dx, float* part, cudaStream_t st) {
    if (d == 32) launch_bwd<T, 1>(B, Tn, H, K, norm, x, w, dy, dx, part, st);
    else if (d == 64) launch_bwd<T, 2>(B, Tn, H, K, norm, x, w, dy, dx, part, st);
    else launch_bwd<T, 4>(B, Tn, H, K, norm, x, w, dy, dx, part, st);
}

gdn_status check_conv(int B, int T, int H, int d, int K, gdn_dtype dtype) {
    if (B < 1 || T < 1 || H < 1 || K < 1) return GDN_ERR_INVALID_ARG;
    if (dtype != GDN_BF16 && dtype != GDN_F32) return GDN_ERR_INVALID_ARG;
    if ((double)B * T * H * 128.0 > 9.0e18) return GDN_ERR_INVALID_ARG;
    if ((long long)B * tiles_of(T, RUN_B) * H > 0x7fffffffLL) return GDN_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 128) return GDN_ERR_UNSUPPORTED;
    if (K > KT) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

bool al(const void* p, unsigned a) { return ((uintptr_t)p & (a - 1)) == 0; }

size_t partial_bytes(int B, int T, int H, int d, int K) {
    return (size_t)B * tiles_of(T, RUN_B) * H * d * K * sizeof(float);
}

}  // namespace
}  // namespace gdn

extern "C" {

gdn_status gdn_short_conv_fwd(int B, int T, int H, int d, int K, gdn_dtype dtype, int l2norm,
                              const void* x, const float* w, void* y, gdn_stream_t stream) {
    using namespace gdn;
    const gdn_status s = check_conv(B, T, H, d, K, dtype);
    if (s != GDN_OK) return s;
    if (!x || !w || !y || x == y) return GDN_ERR_INVALID_ARG;
    if (!al(x, 16) || !al(y, 16) || !al(w, 4)) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    if (dtype == GDN_BF16) dispatch_fwd<__nv_bfloat16>(B, T, H, d, K, l2norm != 0, x, w, y, st);
    else dispatch_fwd<float>(B, T, H, d, K, l2norm != 0, x, w, y, st);
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_short_conv_bwd_workspace(int B, int T, int H, int d, int K) {
    using namespace gdn;
    if (check_conv(B, T, H, d, K, GDN_BF16) != GDN_OK) return 0;
    return partial_bytes(B, T, H, d, K);
}

gdn_status gdn_short_conv_bwd(int B, int T, int H, int d, int K, gdn_dtype dtype, int l2norm,
                              const void* x, const float* w, const void* dy, void* dx, float* dw,
                              void* ws, size_t ws_bytes, gdn_stream_t stream) {
    using namespace gdn;
    const gdn_status s = check_conv(B, T, H, d, K, dtype);
    if (s != GDN_OK) return s;
    if (!x || !w || !dy || !dx || !dw) return GDN_ERR_INVALID_ARG;
    if (dx == x || dx == dy) return GDN_ERR_INVALID_ARG;
    if (!al(x, 16) || !al(dy, 16) || !al(dx, 16) || !al(w, 4) || !al(dw, 4))
        return GDN_ERR_INVALID_ARG;
    if (!ws || ws_bytes < partial_bytes(B, T, H, d, K) || !al(ws, 256)) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    float* part = (float*)ws;
    if (dtype == GDN_BF16)
        dispatch_bwd<__nv_bfloat16>(B, T, H, d, K, l2norm != 0, x, w, dy, dx, part, st);
    else
        dispatch_bwd<float>(B, T, H, d, K, l2norm != 0, x, w, dy, dx, part, st);
    const int per = H * d * K;
    GDN_LAUNCH("short_conv_dw_reduce", st,
               (short_conv_dw_reduce_kernel<<<(per + 31) / 32, RW * 32, 0, st>>>(
                   part, B * tiles_of(T, RUN_B), per, dw)));
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"
