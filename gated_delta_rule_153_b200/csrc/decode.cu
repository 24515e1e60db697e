// decode.cu -- single-token gated delta-rule update on N x H fp32 states.
//
// "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper review),
// sections "Background" and "Method": the recurrent form keeps a fixed-size
// matrix state per (sequence, head); one token applies
//     S <- S a (I - beta k k^T) + beta v k^T,   o = S (scale q)
// (channel gate: Diag(a) on the key index).  Written per value-row a of S:
//     sh_c = S_ac a_c,  p_a = sum_c sh_c k_c,  u_a = beta (v_a - p_a),
//     o_a = scale (sum_c sh_c q_c + u_a (k . q)),  S_ac <- sh_c + u_a k_c.
// Rows are independent, so each row is streamed through registers once:
// one 128-bit read and one 128-bit write per 4 state elements, nothing else
// touches HBM beyond q, k, v, g, beta and o (about 1 KiB per head).
//
// Thread layout: a row of DK floats is covered by L = DK/16 lanes, each lane
// owning 16 columns as four float4 at column offsets 4*(lane + L*j); the
// L lanes of a row read 16*L*4 = DK*4 contiguous bytes per float4 step, so a
// warp instruction touches 32*16 B = 512 B in whole 128-byte lines.
#include "common.cuh"
#include "internal.h"

namespace gdn {

template <int DK, typename T, bool CHANNEL, int ROWS_PER_THREAD>
__global__ void __launch_bounds__(256)
decode_step_kernel(int H, int dv, float scale, const T* __restrict__ q,
                   const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ g, const float* __restrict__ beta,
                   float* __restrict__ state, T* __restrict__ o) {
    constexpr int L = DK / 16;           // lanes per row
    constexpr int RPW = 32 / L;          // rows per warp per row-slot
    const int nh = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane % L;            // position inside the row group
    const int grp = lane / L;            // row group inside the warp
    const int nwarps = blockDim.x >> 5;

    // This lane's 16 columns of k, q and the decay.
    float kr[16], qr[16], ar[16];
    const T* kp = k + (size_t)nh * DK;
    const T* qp = q + (size_t)nh * DK;
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int c = 4 * (sub + L * j) + e;
            kr[4 * j + e] = to_f(kp[c]);
            qr[4 * j + e] = scale * to_f(qp[c]);
            kq += kr[4 * j + e] * qr[4 * j + e];
            if (CHANNEL) ar[4 * j + e] = expf(g[(size_t)nh * DK + c]);
        }
    }
#pragma unroll
    for (int o2 = L / 2; o2 > 0; o2 >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o2);
    float a_s = 1.f;
    if (!CHANNEL) a_s = expf(g[nh]);
    const float b = beta[nh];
    if (!CHANNEL) {
#pragma unroll
        for (int e = 0; e < 16; ++e) ar[e] = a_s;
    }

    float* S = state + (size_t)nh * dv * DK;
    const T* vp = v + (size_t)nh * dv;
    T* op = o + (size_t)nh * dv;
    const int rows_per_pass = nwarps * RPW * ROWS_PER_THREAD;
    for (int r0 = 0; r0 < dv; r0 += rows_per_pass) {
        int rows[ROWS_PER_THREAD];
        float4 s[ROWS_PER_THREAD][4];
#pragma unroll
        for (int rr = 0; rr < ROWS_PER_THREAD; ++rr) {
            rows[rr] = r0 + (warp * ROWS_PER_THREAD + rr) * RPW + grp;
            if (rows[rr] < dv) {
                const float4* src = reinterpret_cast<const float4*>(S + (size_t)rows[rr] * DK);
#pragma unroll
                for (int j = 0; j < 4; ++j) s[rr][j] = __ldcs(src + sub + L * j);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) s[rr][j] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int rr = 0; rr < ROWS_PER_THREAD; ++rr) {
            // every lane runs the shuffles below; only rows < dv are stored
            const bool valid = rows[rr] < dv;
            float sh[16];
            float p = 0.f, oq = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sh[4 * j + 0] = s[rr][j].x * ar[4 * j + 0];
                sh[4 * j + 1] = s[rr][j].y * ar[4 * j + 1];
                sh[4 * j + 2] = s[rr][j].z * ar[4 * j + 2];
                sh[4 * j + 3] = s[rr][j].w * ar[4 * j + 3];
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                p += sh[e] * kr[e];
                oq += sh[e] * qr[e];
            }
#pragma unroll
            for (int o2 = L / 2; o2 > 0; o2 >>= 1) {
                p += __shfl_xor_sync(0xffffffffu, p, o2);
                oq += __shfl_xor_sync(0xffffffffu, oq, o2);
            }
            if (!valid) continue;   // after the last shuffle of this row
            const float u = b * (to_f(vp[rows[rr]]) - p);
            float4* dst = reinterpret_cast<float4*>(S + (size_t)rows[rr] * DK);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 w;
                w.x = sh[4 * j + 0] + u * kr[4 * j + 0];
                w.y = sh[4 * j + 1] + u * kr[4 * j + 1];
                w.z = sh[4 * j + 2] + u * kr[4 * j + 2];
                w.w = sh[4 * j + 3] + u * kr[4 * j + 3];
                __stcs(dst + sub + L * j, w);
            }
            if (sub == 0) op[rows[rr]] = from_f<T>(oq + u * kq);
        }
    }
}

template <int DK, typename T, bool CHANNEL>
static void launch_decode(int N, int H, int dv, float scale, const void* q, const void* k,
                          const void* v, const float* g, const float* beta, float* state,
                          void* o, cudaStream_t st) {
    GDN_LAUNCH("decode_step", st,
               decode_step_kernel<DK, T, CHANNEL, 2><<<N * H, 256, 0, st>>>(
                   H, dv, scale, (const T*)q, (const T*)k, (const T*)v, g, beta, state,
                   (T*)o));
}

template <typename T, bool CHANNEL>
static void dispatch_dk(int N, int H, int dk, int dv, float scale, const void* q,
                        const void* k, const void* v, const float* g, const float* beta,
                        float* state, void* o, cudaStream_t st) {
    switch (dk) {
        case 16: launch_decode<16, T, CHANNEL>(N, H, dv, scale, q, k, v, g, beta, state, o, st); break;
        case 32: launch_decode<32, T, CHANNEL>(N, H, dv, scale, q, k, v, g, beta, state, o, st); break;
        case 64: launch_decode<64, T, CHANNEL>(N, H, dv, scale, q, k, v, g, beta, state, o, st); break;
        default: launch_decode<128, T, CHANNEL>(N, H, dv, scale, q, k, v, g, beta, state, o, st); break;
    }
}

void launch_recurrent_step(int N, int H, int dk, int dv, gdn_dtype dtype, gdn_gate gate,
                           float scale, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, float* state, void* o,
                           cudaStream_t st) {
    const bool ch = gate == GDN_GATE_CHANNEL;
    if (dtype == GDN_BF16) {
        if (ch) dispatch_dk<__nv_bfloat16, true>(N, H, dk, dv, scale, q, k, v, g, beta, state, o, st);
        else dispatch_dk<__nv_bfloat16, false>(N, H, dk, dv, scale, q, k, v, g, beta, state, o, st);
    } else {
        if (ch) dispatch_dk<float, true>(N, H, dk, dv, scale, q, k, v, g, beta, state, o, st);
        else dispatch_dk<float, false>(N, H, dk, dv, scale, q, k, v, g, beta, state, o, st);
    }
}

}  // namespace gdn
