// mma.cuh -- warp-level bf16 tensor-core helpers over swizzled shared tiles.
//
// Tiles: row-major bf16 [ROWS][COLS] (COLS = 64 or 128) whose 16-byte chunks
// are XOR-swizzled by (row % 8), so the eight row addresses one ldmatrix
// 8x8 block reads always fall in eight different bank groups.
//
// Fragments follow mma.m16n8k16 (bf16 in, fp32 accumulate):
//   A 16x16: a0 (m=l/4,   k=2(l%4)+{0,1}), a1 (m+8, same k), a2 (m, k+8), a3 (m+8, k+8)
//   B 16x8 : b0 (k=2(l%4)+{0,1}, n=l/4),   b1 (k+8, n)
//   C 16x8 : c0,c1 (m=l/4, n=2(l%4)+{0,1}), c2,c3 (m+8, same n)
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#define GDN_DEV __device__ __forceinline__

namespace gdn {

template <int COLS>
GDN_DEV uint32_t swz(int row, int col) {  // element offset inside a tile
    return row * COLS + ((((col >> 3) ^ (row & 7)) << 3) | (col & 7));
}

GDN_DEV uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

GDN_DEV void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

GDN_DEV void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

GDN_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (rows m0.., cols k0..) of a tile X with A[m][k] = X[m][k].
template <int COLS>
GDN_DEV void lda(uint32_t (&a)[4], const __nv_bfloat16* X, int m0, int k0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    const int row = m0 + (l & 7) + (idx & 1) * 8;
    const int col = k0 + (idx >> 1) * 8;
    ldsm_x4(a, smem_u32(X + swz<COLS>(row, col)));
}

// A fragment with A[m][k] = X[k][m] (X stored k-major).
template <int COLS>
GDN_DEV void lda_t(uint32_t (&a)[4], const __nv_bfloat16* X, int m0, int k0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    const int row = k0 + (l & 7) + (idx >> 1) * 8;
    const int col = m0 + (idx & 1) * 8;
    ldsm_x4_t(a, smem_u32(X + swz<COLS>(row, col)));
}

// B fragments for two n8 tiles (n0.., n0+8..) and k16 (k0..), B[k][n] = X[n][k].
// b[0],b[1] -> n-tile 0; b[2],b[3] -> n-tile 1.
template <int COLS>
GDN_DEV void ldb_nk(uint32_t (&b)[4], const __nv_bfloat16* X, int n0, int k0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    const int row = n0 + (l & 7) + (idx >> 1) * 8;
    const int col = k0 + (idx & 1) * 8;
    ldsm_x4(b, smem_u32(X + swz<COLS>(row, col)));
}

// Same with B[k][n] = X[k][n] (X stored n-contiguous).
template <int COLS>
GDN_DEV void ldb_kn(uint32_t (&b)[4], const __nv_bfloat16* X, int k0, int n0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    const int row = k0 + (l & 7) + (idx & 1) * 8;
    const int col = n0 + (idx >> 1) * 8;
    ldsm_x4_t(b, smem_u32(X + swz<COLS>(row, col)));
}

GDN_DEV uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

GDN_DEV float2 unpack_bf16(uint32_t x) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&x);
    return __bfloat1622float2(v);
}

// Store a C fragment (16x8 at m0, n0) into tile X as bf16, X[m][n].
template <int COLS>
GDN_DEV void st_c(__nv_bfloat16* X, int m0, int n0, const float (&c)[4]) {
    const int l = threadIdx.x & 31;
    const int r = m0 + (l >> 2), col = n0 + 2 * (l & 3);
    *reinterpret_cast<uint32_t*>(X + swz<COLS>(r, col)) = pack_bf16(c[0], c[1]);
    *reinterpret_cast<uint32_t*>(X + swz<COLS>(r + 8, col)) = pack_bf16(c[2], c[3]);
}

// Store a C fragment transposed: X[n][m] = C[m][n].
template <int COLS>
GDN_DEV void st_c_t(__nv_bfloat16* X, int m0, int n0, const float (&c)[4]) {
    const int l = threadIdx.x & 31;
    const int r = m0 + (l >> 2), col = n0 + 2 * (l & 3);
    X[swz<COLS>(col, r)] = __float2bfloat16_rn(c[0]);
    X[swz<COLS>(col + 1, r)] = __float2bfloat16_rn(c[1]);
    X[swz<COLS>(col, r + 8)] = __float2bfloat16_rn(c[2]);
    X[swz<COLS>(col + 1, r + 8)] = __float2bfloat16_rn(c[3]);
}

// Asynchronous 16-byte global -> shared copies.
GDN_DEV void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
GDN_DEV void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
    // src-size 0 fills the 16 bytes with zeros (used for rows past the sequence end)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 ::"r"(smem_u32(smem)), "l"(gmem), "r"(valid ? 16 : 0));
}
GDN_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
GDN_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Copy `rows` rows of a row-major global bf16 matrix (row stride `gstride`
// elements, COLS columns) into a swizzled tile; rows >= valid_rows are zeroed.
template <int COLS>
GDN_DEV void load_tile_async(__nv_bfloat16* X, const __nv_bfloat16* g, size_t gstride, int rows,
                             int valid_rows, int tid, int nthreads) {
    constexpr int CH = COLS / 8;
    for (int e = tid; e < rows * CH; e += nthreads) {
        const int r = e / CH, ch = e % CH;
        const bool ok = r < valid_rows;
        const __nv_bfloat16* src = g + (size_t)(ok ? r : 0) * gstride + ch * 8;
        cp_async16_zfill(X + swz<COLS>(r, ch * 8), src, ok);
    }
}

// Copy a tile image (a contiguous run of `bytes`, multiple of 16) verbatim.
GDN_DEV void load_image_async(void* X, const void* g, int bytes, int tid, int nthreads) {
    for (int e = tid; e < bytes / 16; e += nthreads)
        cp_async16((char*)X + 16 * e, (const char*)g + 16 * e);
}

}  // namespace gdn

namespace gdn {

// Layout classes: Swz<COLS> is the XOR-swizzled tile above; Pad<COLS> keeps
// each row's COLS elements contiguous and in order (so a row can be filled by
// one bulk copy) and pads the row pitch by 16 bytes, which also puts the
// eight rows of an ldmatrix block in eight different bank groups.
template <int COLS>
struct Swz {
    static constexpr int PITCH = COLS;
    GDN_DEV static uint32_t off(int r, int c) { return swz<COLS>(r, c); }
};
template <int COLS>
struct Pad {
    static constexpr int PITCH = COLS + 8;
    GDN_DEV static uint32_t off(int r, int c) { return r * PITCH + c; }
};

template <class LY>
GDN_DEV void lda(uint32_t (&a)[4], const __nv_bfloat16* X, int m0, int k0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    ldsm_x4(a, smem_u32(X + LY::off(m0 + (l & 7) + (idx & 1) * 8, k0 + (idx >> 1) * 8)));
}
template <class LY>
GDN_DEV void lda_t(uint32_t (&a)[4], const __nv_bfloat16* X, int m0, int k0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    ldsm_x4_t(a, smem_u32(X + LY::off(k0 + (l & 7) + (idx >> 1) * 8, m0 + (idx & 1) * 8)));
}
template <class LY>
GDN_DEV void ldb_nk(uint32_t (&b)[4], const __nv_bfloat16* X, int n0, int k0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    ldsm_x4(b, smem_u32(X + LY::off(n0 + (l & 7) + (idx >> 1) * 8, k0 + (idx & 1) * 8)));
}
template <class LY>
GDN_DEV void ldb_kn(uint32_t (&b)[4], const __nv_bfloat16* X, int k0, int n0) {
    const int l = threadIdx.x & 31, idx = l >> 3;
    ldsm_x4_t(b, smem_u32(X + LY::off(k0 + (l & 7) + (idx & 1) * 8, n0 + (idx >> 1) * 8)));
}
// Single n8 tile variants (x2): b[0], b[1] for n0..n0+7.
GDN_DEV void ldsm_x2(uint32_t (&r)[2], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
GDN_DEV void ldsm_x2_t(uint32_t (&r)[2], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
// B[k][n] = X[n][k], one n8 tile: lanes 0-7 rows n0.., k0; lanes 8-15 rows n0.., k0+8.
template <class LY>
GDN_DEV void ldb_nk1(uint32_t (&b)[2], const __nv_bfloat16* X, int n0, int k0) {
    const int l = threadIdx.x & 31, idx = (l >> 3) & 1;
    ldsm_x2(b, smem_u32(X + LY::off(n0 + (l & 7), k0 + idx * 8)));
}
// B[k][n] = X[k][n], one n8 tile: lanes 0-7 rows k0.., lanes 8-15 rows k0+8..
template <class LY>
GDN_DEV void ldb_kn1(uint32_t (&b)[2], const __nv_bfloat16* X, int k0, int n0) {
    const int l = threadIdx.x & 31, idx = (l >> 3) & 1;
    ldsm_x2_t(b, smem_u32(X + LY::off(k0 + (l & 7) + idx * 8, n0)));
}
template <class LY>
GDN_DEV void st_c(__nv_bfloat16* X, int m0, int n0, const float (&c)[4]) {
    const int l = threadIdx.x & 31;
    const int r = m0 + (l >> 2), col = n0 + 2 * (l & 3);
    *reinterpret_cast<uint32_t*>(X + LY::off(r, col)) = pack_bf16(c[0], c[1]);
    *reinterpret_cast<uint32_t*>(X + LY::off(r + 8, col)) = pack_bf16(c[2], c[3]);
}

}  // namespace gdn
