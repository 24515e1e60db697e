// common.cuh -- small device helpers shared by the gdn kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

#define GDN_DEV __device__ __forceinline__

namespace gdn {

// Scalar conversions between the storage dtype of q/k/v/o and fp32.
template <typename T> GDN_DEV float to_f(T x);
template <> GDN_DEV float to_f<float>(float x) { return x; }
template <> GDN_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> GDN_DEV T from_f(float x);
template <> GDN_DEV float from_f<float>(float x) { return x; }
template <> GDN_DEV __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Bytes reserved at the start of every chunkwise workspace: word 0 is the
// device status word (non-zero after a bounded wait gave up).
constexpr size_t kStatusBytes = 256;

// Launch bracketing for gdn_profile_begin/end (no-ops unless enabled).
void prof_before(cudaStream_t st);
void prof_after(cudaStream_t st, const char* name);
#define GDN_LAUNCH(name, st, ...)          \
    do {                                   \
        ::gdn::prof_before(st);            \
        __VA_ARGS__;                       \
        ::gdn::prof_after(st, name);       \
    } while (0)

GDN_DEV float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace gdn
