// product.cu -- the gated DeltaProduct on the chunkwise kernels.
//
// "DeltaProduct: Improving State-Tracking in Linear RNNs via Householder
// Products" (in the list of related papers of the "Linear Attention
// Architectures: Mechanisms, Trade-offs, and Cross-Layer Routing" summary
// page) and the "Gated Delta Networks: Improving Mamba2 with Delta Rule"
// review, section "Future work" (products of Householder matrices as an
// extension of the gated delta rule).  Each token t applies its gate once and
// then n delta-rule steps with its own keys, values and betas, in order, and
// is read out after the last:
//     S <- S D_t;   S <- S (I - b_tj k_tj k_tj^T) + b_tj v_tj k_tj^T,  j = 1..n;
//     o_t = S (scale q_t).
// That is the gated delta rule on the n*T sub-tokens (t, 1) .. (t, n) with
// g_t on the first sub-token (0 on the others) and q_t on the last (0 on the
// others), the output read at the last.  k [B,T,n,H,dk], v [B,T,n,H,dv] and
// beta [B,T,n,H] already are that sub-token sequence in memory; q and g are
// spread over it and o (dq, dg) gathered back by the two copy kernels below,
// and the chunkwise kernels run over T' = n*T.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace gdn {
namespace {

// dst row (r*n + j) = (j == pos ? src row r : 0), for r < rows; rows of `words`
// elements of type V.
template <typename V>
__global__ void expand_rows_kernel(V* __restrict__ dst, const V* __restrict__ src, long long rows,
                                   int n, int pos, int words) {
    const long long total = rows * n * words;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long drow = i / words;
        const int w = (int)(i - drow * words);
        const long long r = drow / n;
        const int j = (int)(drow - r * n);
        V x{};
        if (j == pos) x = src[r * words + w];
        dst[i] = x;
    }
}

// dst row r = src row (r*n + pos), for r < rows.
template <typename V>
__global__ void gather_rows_kernel(V* __restrict__ dst, const V* __restrict__ src, long long rows,
                                   int n, int pos, int words) {
    const long long total = rows * words;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long r = i / words;
        const int w = (int)(i - r * words);
        dst[i] = src[(r * n + pos) * words + w];
    }
}

unsigned grid_for(long long total) {
    return (unsigned)std::max(1LL, std::min((total + 255) / 256, 148LL * 16));
}

// Rows of `bytes` (a multiple of 4) each: 16-byte moves when the row and both
// pointers allow, 4-byte moves otherwise.
void expand_rows(void* dst, const void* src, long long rows, int n, int pos, size_t bytes,
                 cudaStream_t st) {
    if (bytes % 16 == 0 && ((uintptr_t)dst | (uintptr_t)src) % 16 == 0) {
        const int w = (int)(bytes / 16);
        GDN_LAUNCH("product_expand", st,
                   (expand_rows_kernel<uint4><<<grid_for(rows * n * w), 256, 0, st>>>(
                       (uint4*)dst, (const uint4*)src, rows, n, pos, w)));
    } else {
        const int w = (int)(bytes / 4);
        GDN_LAUNCH("product_expand", st,
                   (expand_rows_kernel<uint32_t><<<grid_for(rows * n * w), 256, 0, st>>>(
                       (uint32_t*)dst, (const uint32_t*)src, rows, n, pos, w)));
    }
}

void gather_rows(void* dst, const void* src, long long rows, int n, int pos, size_t bytes,
                 cudaStream_t st) {
    if (bytes % 16 == 0 && ((uintptr_t)dst | (uintptr_t)src) % 16 == 0) {
        const int w = (int)(bytes / 16);
        GDN_LAUNCH("product_gather", st,
                   (gather_rows_kernel<uint4><<<grid_for(rows * w), 256, 0, st>>>(
                       (uint4*)dst, (const uint4*)src, rows, n, pos, w)));
    } else {
        const int w = (int)(bytes / 4);
        GDN_LAUNCH("product_gather", st,
                   (gather_rows_kernel<uint32_t><<<grid_for(rows * w), 256, 0, st>>>(
                       (uint32_t*)dst, (const uint32_t*)src, rows, n, pos, w)));
    }
}

constexpr int kMaxProductSteps = 64;

size_t r256(size_t x) { return (x + 255) & ~(size_t)255; }

bool expanded_dims(const gdn_dims* d, int n, gdn_dims& e) {
    if (!d || n < 1 || n > kMaxProductSteps || d->T < 1) return false;
    if ((long long)d->T * n > 0x7fffffffLL) return false;
    e = *d;
    e.T = d->T * n;
    return true;
}

// Byte sizes of one token row (all heads) of q / o / g.
struct RowBytes {
    size_t qk, ov, g;
};
RowBytes row_bytes(const gdn_dims& d) {
    const size_t esz = d.dtype == GDN_BF16 ? 2 : 4;
    return {(size_t)d.H * d.dk * esz, (size_t)d.H * d.dv * esz,
            (size_t)d.H * (d.gate == GDN_GATE_CHANNEL ? d.dk : 1) * 4};
}

// Workspace: the inner call's workspace first (its status word at offset 0),
// then the spread q (and dO), g, and the sub-token o (or dq, dg).
struct ProductLayout {
    size_t inner, q, g, o, dO, dq, dg, total;
};
ProductLayout product_layout(const gdn_dims& e, long long sub_rows, bool bwd) {
    const RowBytes rb = row_bytes(e);
    ProductLayout L{};
    L.inner = bwd ? gdn_chunk_bwd_workspace(&e) : gdn_chunk_fwd_workspace(&e);
    size_t o = r256(L.inner);
    L.q = o; o += r256(sub_rows * rb.qk);
    L.g = o; o += r256(sub_rows * rb.g);
    if (bwd) {
        L.dO = o; o += r256(sub_rows * rb.ov);
        L.dq = o; o += r256(sub_rows * rb.qk);
        L.dg = o; o += r256(sub_rows * rb.g);
    } else {
        L.o = o; o += r256(sub_rows * rb.ov);
    }
    L.total = o;
    return L;
}

gdn_status finish() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace
}  // namespace gdn

extern "C" {

size_t gdn_product_fwd_workspace(const gdn_dims* d, int n) {
    gdn_dims e;
    if (!gdn::expanded_dims(d, n, e) || gdn_chunk_fwd_workspace(&e) == 0) return 0;
    return gdn::product_layout(e, (long long)e.B * e.T, false).total;
}

size_t gdn_product_bwd_workspace(const gdn_dims* d, int n) {
    gdn_dims e;
    if (!gdn::expanded_dims(d, n, e) || gdn_chunk_bwd_workspace(&e) == 0) return 0;
    return gdn::product_layout(e, (long long)e.B * e.T, true).total;
}

gdn_status gdn_product_fwd(const gdn_dims* d, int n, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* h0, void* o, float* hT,
                           void* ws, size_t ws_bytes, gdn_stream_t stream) {
    gdn_dims e;
    if (!gdn::expanded_dims(d, n, e)) return GDN_ERR_INVALID_ARG;
    if (!q || !g || !o) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_product_fwd_workspace(d, n);
    if (need == 0)  // dims the chunkwise forward rejects: report its reason
        return gdn_chunk_fwd(&e, q, k, v, g, beta, h0, o, hT, nullptr, 0, stream);
    if (!ws || ws_bytes < need) return GDN_ERR_WORKSPACE;
    if ((uintptr_t)ws & 255u) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    const long long rows = (long long)d->B * d->T;
    const gdn::RowBytes rb = gdn::row_bytes(*d);
    const gdn::ProductLayout L = gdn::product_layout(e, rows * n, false);
    char* w = (char*)ws;
    gdn::expand_rows(w + L.q, q, rows, n, n - 1, rb.qk, st);
    gdn::expand_rows(w + L.g, g, rows, n, 0, rb.g, st);
    if (gdn::finish() != GDN_OK) return GDN_ERR_CUDA;
    const gdn_status s = gdn_chunk_fwd(&e, w + L.q, k, v, (const float*)(w + L.g), beta, h0,
                                       w + L.o, hT, ws, L.inner, stream);
    if (s != GDN_OK) return s;
    gdn::gather_rows(o, w + L.o, rows, n, n - 1, rb.ov, st);
    return gdn::finish();
}

gdn_status gdn_product_bwd(const gdn_dims* d, int n, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const float* h0, const void* dO,
                           const float* dhT, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                           float* dh0, void* ws, size_t ws_bytes, gdn_stream_t stream) {
    gdn_dims e;
    if (!gdn::expanded_dims(d, n, e)) return GDN_ERR_INVALID_ARG;
    if (!q || !g || !dO || !dq || !dg) return GDN_ERR_INVALID_ARG;
    const size_t need = gdn_product_bwd_workspace(d, n);
    if (need == 0)  // dims the chunkwise backward rejects: report its reason
        return gdn_chunk_bwd(&e, q, k, v, g, beta, h0, dO, dhT, dq, dk, dv, dg, dbeta, dh0,
                             nullptr, 0, stream);
    if (!ws || ws_bytes < need) return GDN_ERR_WORKSPACE;
    if ((uintptr_t)ws & 255u) return GDN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaGetLastError();
    const long long rows = (long long)d->B * d->T;
    const gdn::RowBytes rb = gdn::row_bytes(*d);
    const gdn::ProductLayout L = gdn::product_layout(e, rows * n, true);
    char* w = (char*)ws;
    gdn::expand_rows(w + L.q, q, rows, n, n - 1, rb.qk, st);
    gdn::expand_rows(w + L.g, g, rows, n, 0, rb.g, st);
    gdn::expand_rows(w + L.dO, dO, rows, n, n - 1, rb.ov, st);
    if (gdn::finish() != GDN_OK) return GDN_ERR_CUDA;
    const gdn_status s = gdn_chunk_bwd(&e, w + L.q, k, v, (const float*)(w + L.g), beta, h0,
                                       w + L.dO, dhT, w + L.dq, dk, dv, (float*)(w + L.dg), dbeta,
                                       dh0, ws, L.inner, stream);
    if (s != GDN_OK) return s;
    gdn::gather_rows(dq, w + L.dq, rows, n, n - 1, rb.qk, st);
    gdn::gather_rows(dg, w + L.dg, rows, n, 0, rb.g, st);
    return gdn::finish();
}

}  // extern "C"
