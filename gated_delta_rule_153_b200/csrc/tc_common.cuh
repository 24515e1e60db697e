// tc_common.cuh -- shapes, workspace layout and pointer bundles shared by the
// tensor-core chunkwise kernels (tc_chunk.cu forward pieces, tc_bwd.cu).
#pragma once

#include "common.cuh"
#include "mma.cuh"

namespace gdn {
namespace tc {

constexpr int C = 64, DK = 128, DV = 128;

struct TcLayout {
    int NT;
    size_t nchunks;
    // byte offsets into the workspace
    size_t W, Ut, P, G, Tb, S0, U, dS, dU, end;
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
    L.G = take(L.nchunks * C * 4);
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

struct ChunkPtrs {
    const __nv_bfloat16 *q, *k, *v;
    const float *g, *beta;
    int B, T, H, NT;
    float scale;
    __nv_bfloat16 *W, *Ut, *P;
    float* G;
    __nv_bfloat16* Tb;  // optional: bf16 T = (I + A)^{-1} per chunk (backward)
};

}  // namespace tc
}  // namespace gdn
