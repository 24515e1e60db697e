// tc_common.cuh -- shapes, workspace layout and pointer bundles shared by the
// tensor-core chunkwise kernels (tc_chunk.cu forward pieces, tc_bwd.cu).
#pragma once

#include "async.cuh"
#include "common.cuh"
#include "mma.cuh"
#include "tma.cuh"

namespace gdn {
namespace tc {

constexpr int C = 64, DK = 128, DV = 128;

struct TcLayout {
    int NT;
    size_t nchunks;
    // byte offsets into the workspace
    size_t W, Ut, P, G, Tb, S0, U, dS, dU, Qg, Kt, end;
};

inline TcLayout tc_layout(const gdn_dims& d, bool bwd) {
    TcLayout L{};
    L.NT = (d.T + C - 1) / C;
    L.nchunks = (size_t)d.B * d.H * L.NT;
    size_t o = kStatusBytes;
    auto take = [&](size_t bytes) { size_t r = o; o += (bytes + 255) & ~(size_t)255; return r; };
    L.W = take(L.nchunks * C * DK * 2);
    L.Ut = take(L.nchunks * C * DV * 2);
    L.P = take(L.nchunks * C * C * 2);
    L.G = take(L.nchunks * (d.gate == GDN_GATE_CHANNEL ? DK : C) * 4);
    if (d.gate == GDN_GATE_CHANNEL) {
        L.Qg = take(L.nchunks * C * DK * 2);
        L.Kt = take(L.nchunks * C * DK * 2);
    }
    if (bwd) {
        L.Tb = take(L.nchunks * C * C * 2);
        L.S0 = take(L.nchunks * DV * DK * 2);
        L.U = take(L.nchunks * C * DV * 2);
        L.dS = take(L.nchunks * DV * DK * 2);
        L.dU = take(L.nchunks * C * DV * 2);
    }
    L.end = o;
    return L;
}

// Workspace images (written by prep with bulk stores, read back the same way):
//   W   [chunk] Tma128 image of the 64x128 W (two 64-column K-major panels)
//   Ut  [chunk] Swz<64> image of U~^T: 128 value rows x 64 tokens, so any
//       16-row slice of the state is one contiguous 2 KB range
//   P   [chunk][64][64]  bf16, Swz<64> tile image (scale folded in)
//   G   [chunk][64] fp32 within-chunk cumsum of g (padding rows repeat the last);
//       channel gate: [chunk][128] fp32 e^{G_last,c}, the per-key decay of a chunk
//   Qg  channel gate only: [chunk] Tma128 image of scale * Q .* e^{G}
//   Kt  channel gate only: [chunk] Tma128 image of K .* e^{G_last - G}
//   Tb  [chunk][64][64]  bf16, Swz<64> tile image of T = (I + A)^{-1}
//   S0  [chunk][128][128] bf16, Swz<128> image of the chunk-start state
//   U   [chunk][64][128] bf16 row-major;  dS, dU likewise (backward)
struct ChunkPtrs {
    CUtensorMap qmap, kmap, vmap;  // token maps of q, k, v (see tma.cuh)
    const __nv_bfloat16 *q, *k, *v;
    const float *g, *beta;
    int B, T, H, NT;
    float scale;
    __nv_bfloat16 *W, *Ut, *P;
    float* G;
    __nv_bfloat16* Tb;  // optional: bf16 T = (I + A)^{-1} per chunk (backward)
    __nv_bfloat16 *Qg, *Kt;  // channel gate only
    unsigned int* status;
};

// Stage the W and U~ images from a warp's 16-row block of the W = T diag(.) K
// and U~ = T diag(beta) V accumulators (m16n8 fragments, 16 n-blocks of 8).
GDN_DEV void stage_w_ut(__nv_bfloat16* Wst, __nv_bfloat16* Ust, const float (&aw)[16][4],
                        const float (&au)[16][4], int m0) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        st_c<Tma128>(Wst, m0, 8 * j, aw[j]);
        const int r = m0 + (lane >> 2), c = 8 * j + 2 * (lane & 3);
        Ust[swz<C>(c, r)] = __float2bfloat16_rn(au[j][0]);
        Ust[swz<C>(c + 1, r)] = __float2bfloat16_rn(au[j][1]);
        Ust[swz<C>(c, r + 8)] = __float2bfloat16_rn(au[j][2]);
        Ust[swz<C>(c + 1, r + 8)] = __float2bfloat16_rn(au[j][3]);
    }
}

// The same for 8*NB of the 128 columns, starting at column n0.
template <int NB>
GDN_DEV void stage_w_ut_cols(__nv_bfloat16* Wst, __nv_bfloat16* Ust, const float (&aw)[NB][4],
                             const float (&au)[NB][4], int m0, int n0) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
        st_c<Tma128>(Wst, m0, n0 + 8 * j, aw[j]);
        const int r = m0 + (lane >> 2), c = n0 + 8 * j + 2 * (lane & 3);
        Ust[swz<C>(c, r)] = __float2bfloat16_rn(au[j][0]);
        Ust[swz<C>(c + 1, r)] = __float2bfloat16_rn(au[j][1]);
        Ust[swz<C>(c, r + 8)] = __float2bfloat16_rn(au[j][2]);
        Ust[swz<C>(c + 1, r + 8)] = __float2bfloat16_rn(au[j][3]);
    }
}

// Round a dynamic shared-memory pointer up to the 1024-byte alignment that
// 128-byte-swizzled TMA destinations need (launches request 1 KB extra).
GDN_DEV unsigned char* align1k(unsigned char* p) {
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace tc
}  // namespace gdn
