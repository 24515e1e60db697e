// tma.cuh -- TMA tensor-map loads of [token][head][d] tiles (sm_100a).
//
// q, k, v, dO are stored [B, T, H, d] (token-major).  A chunk tile of one
// head -- 64 consecutive tokens x 128 channels -- is a strided box, fetched
// by the TMA unit as two 64x64 boxes of a 3-D tensor map
//     dims {d, H, B*T}, strides {d*2 bytes, H*d*2 bytes}, box {64, 1, 64}
// with the hardware 128-byte swizzle.  In shared memory a tile is
// [2 halves][64 rows][64 channels], each half a 1024-byte-aligned 8 KB box
// whose 16-byte chunk j of row r sits at position j ^ (r % 8) -- the layout
// class Tma128 below.  Rows past the end of the tensor read as zero.
// Each load writes only the issuing CTA's own shared memory.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "mma.cuh"

namespace gdn {

struct Tma128 {
    static constexpr int PITCH = 64;
    GDN_DEV static uint32_t off(int r, int c) { return (c >> 6) * (64 * 64) + swz<64>(r, c & 63); }
};

GDN_DEV void tma_load_3d(void* smem, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(smem)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z),
          "r"(smem_u32(bar))
        : "memory");
}

// Both 64-channel halves of rows z .. z+63 of head y into a Tma128 tile.
GDN_DEV void tma_load_tile(__nv_bfloat16* tile, const CUtensorMap* map, int head, int token,
                           uint64_t* bar) {
    tma_load_3d(tile, map, 0, head, token, bar);
    tma_load_3d(tile + 64 * 64, map, 64, head, token, bar);
}

// Hint: pull box (x, y, z) of the map's tensor into L2 ahead of a load.
GDN_DEV void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Both 64-channel halves of rows token .. token+63 of head `head`.
GDN_DEV void tma_prefetch_tile(const CUtensorMap* map, int head, int token) {
    tma_prefetch_3d(map, 0, head, token);
    tma_prefetch_3d(map, 64, head, token);
}

// Host: encode the token map of a [B, T, H, 128] bf16 tensor.  box_cols 64
// gives 128-byte-swizzled boxes of box_rows x 64 (Tma128 tiles at 64 rows);
// box_cols 16 gives unswizzled box_rows x 16 boxes (32-byte rows).  Returns
// false if the driver entry point is unavailable or the encoder rejects the map.
bool encode_token_map(CUtensorMap* map, const void* base, int B, int T, int H,
                      int box_cols = 64, int box_rows = 64);

}  // namespace gdn
