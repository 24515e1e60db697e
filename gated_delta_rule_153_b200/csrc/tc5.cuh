// tc5.cuh -- fifth-generation tensor-core (tcgen05) helpers for sm_100a:
// shared-memory matrix descriptors, the instruction descriptor of a
// bf16 x bf16 -> fp32 MMA, MMA issue and completion, tensor-memory
// allocation and loads.
//
// Operands live in shared memory in the canonical 128-byte-swizzle layouts:
//   K-major : rows of 64 bf16 (128 B), 16-byte chunk index XOR (row % 8),
//             8-row atoms of 1024 B; a K extent above 64 continues in a
//             further panel of the same shape.  (Kp<R> below; Swz<64> and
//             Tma128 are the 64-column and 64-row cases.)
//   MN-major: the same bytes read with rows along K: a row holds 64
//             consecutive M/N elements, panels of 64 step along M/N.
// The accumulator D of an M = 128 MMA occupies TMEM lanes 0..127 (lane = row)
// and N consecutive fp32 columns.
#pragma once
#include "common.cuh"
#include "mma.cuh"

namespace gdn {

// K-major panels: R rows, 64-column panels of 128-byte swizzled rows.
template <int R>
struct Kp {
    static constexpr int PITCH = 64;
    GDN_DEV static uint32_t off(int r, int c) { return (c >> 6) * (R * 64) + swz<64>(r, c & 63); }
};

// Transposed epilogue rows: a lane holds 16 consecutive rows r0 .. r0+15 of
// its own column c as bf16 pairs v[jj] = (row r0+2jj, row r0+2jj+1).  Lanes
// 2i and 2i+1 (columns c, c+1, c even) trade halves, so that w[jj] is the
// 32-bit word (column c, c+1) of row r0 + 2jj + (lane & 1): one store of it
// per row replaces two 2-byte stores.
GDN_DEV void pair_columns(const uint32_t (&v)[8], uint32_t (&w)[8]) {
    const bool odd = threadIdx.x & 1;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        const uint32_t o = __shfl_xor_sync(0xffffffffu, v[jj], 1);
        w[jj] = odd ? __byte_perm(o, v[jj], 0x7632) : __byte_perm(v[jj], o, 0x5410);
    }
}

namespace tc5 {

// Shared-memory descriptor: start address, leading and stride byte offsets,
// descriptor version 1 (sm_100), 128-byte swizzle.  The swizzle pattern is
// anchored at 1024-byte boundaries, so operand tiles start 1024-aligned and a
// K step inside a 128-byte row only moves the start address.
GDN_DEV uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: D fp32, A and B bf16, dense; a_mn / b_mn select the
// MN-major form of the operand.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B over one K = 16 step; issued by a single thread.
GDN_DEV void mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)acc));
}

// Same, with A read from tensor memory (K-major: lane = row, each 32-bit
// column holds two consecutive K elements, so a K = 16 step is 8 columns).
GDN_DEV void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"((uint32_t)acc));
}

// Arrive once on the mbarrier when every MMA issued so far by this thread is done.
GDN_DEV void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

GDN_DEV void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
GDN_DEV void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Generic-proxy shared-memory writes made visible to the tensor core's reads.
GDN_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Column allocation, by one whole warp; the TMEM address lands in *slot.
GDN_DEV void alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

GDN_DEV void dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 consecutive fp32 columns of this thread's lane (warp w reads lanes 32(w%4)..).
GDN_DEV void ld32(float (&v)[32], uint32_t taddr) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive fp32 columns of this thread's lane.
GDN_DEV void ld16(float (&v)[16], uint32_t taddr) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Store 8 / 16 consecutive 32-bit columns of this thread's lane.
GDN_DEV void st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
GDN_DEV void st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
GDN_DEV void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

GDN_DEV void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// TMEM address of (lane, column).
GDN_DEV uint32_t taddr(uint32_t base, int lane, int col) { return base + ((uint32_t)lane << 16) + (uint32_t)col; }

// Descriptors of the canonical operands (byte offsets from a 1024-aligned tile).
// K-major, R rows, K step kk of 16: within a 64-column panel the start moves
// 32 B per step; panels are R*128 B apart.
template <int R>
GDN_DEV uint64_t kmajor(uint32_t base, int kk) {
    return sdesc(base + (uint32_t)((kk >> 2) * (R * 128) + (kk & 3) * 32), 16, 1024);
}
// MN-major over a K-row tile: rows of 64 M/N elements, K step kk of 16 rows;
// panel stride along M/N is `panel` bytes.
GDN_DEV uint64_t mnmajor(uint32_t base, int kk, uint32_t panel) {
    return sdesc(base + (uint32_t)(kk * 16 * 128), panel, 1024);
}

}  // namespace tc5
}  // namespace gdn
