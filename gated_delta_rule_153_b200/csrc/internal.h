// internal.h -- launchers shared between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/gdn.h"

namespace gdn {

void launch_recurrent_step(int N, int H, int dk, int dv, gdn_dtype dtype, gdn_gate gate,
                           float scale, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, float* state, void* o,
                           cudaStream_t st);

// Host-side argument checks of gdn_chunk_fwd (dims, required pointers,
// 16-byte alignment, h0/hT aliasing), without the workspace checks.
gdn_status validate_fwd_args(const gdn_dims* d, const void* q, const void* k, const void* v,
                             const float* g, const float* beta, const float* h0, const void* o,
                             const float* hT);

// Generic fp32-arithmetic chunkwise path (any supported dims, both dtypes).
size_t simt_fwd_workspace(const gdn_dims& d);
size_t simt_bwd_workspace(const gdn_dims& d);
void launch_simt_fwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* h0, void* o, float* hT,
                     void* ws, cudaStream_t st);
void launch_simt_bwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* h0, const void* dO,
                     const float* dhT, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                     float* dh0, void* ws, cudaStream_t st);

// Tensor-core path (bf16, dk = dv = 128, chunk = 64).
bool tc_supported(const gdn_dims& d);
bool tc_bwd_supported(const gdn_dims& d);
// nseq > 0: a packed batch of nseq sequences (d.B = 1, d.T tokens in all,
// device offsets cu[0..nseq]); states are [nseq, H, dv, dk].
size_t tc_fwd_workspace(const gdn_dims& d, int nseq = 0);
size_t tc_bwd_workspace(const gdn_dims& d, int nseq = 0);
// Return false if a TMA tensor map could not be encoded (nothing launched).
// wait_ns / stall_at: the bounded-wait limit and the stall test hook of the
// tcgen05 forward walk (defaults: 1 s, no stall).
bool launch_tc_fwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                   const float* g, const float* beta, const float* h0, void* o, float* hT,
                   void* ws, cudaStream_t st, const int* cu = nullptr, int nseq = 0,
                   unsigned long long wait_ns = 1000000000ull, int stall_at = -1);
// The forward of a training step: launch_tc_fwd's results, plus, in `ws` (a
// backward-layout workspace), what launch_tc_bwd(..., saved = true) reads
// back instead of recomputing it.
bool launch_tc_fwd_save(const gdn_dims& d, const void* q, const void* k, const void* v,
                        const float* g, const float* beta, const float* h0, void* o, float* hT,
                        void* ws, cudaStream_t st);
// The training pair with the q/k/v prologue (gdn_chunk_fwd_save_conv): after
// the `base` bytes of the saved chunk workspace come the filtered q, k, v,
// their gradients, and the prologue backward's workspace.
struct ConvLayout {
    size_t qf, kf, vf, dqf, dkf, dvf, cws, end;
};
ConvLayout conv_layout(const gdn_dims& d, int K, size_t base);
// The fused forward (scalar gate on the tensor-core shapes).
bool launch_tc_fwd_save_conv(const gdn_dims& d, int K, const void* xq, const void* xk, const void* xv,
                             const float* wq, const float* wk, const float* wv, const float* g,
                             const float* beta, const float* h0, void* o, float* hT, void* ws,
                             cudaStream_t st);
// True when the forward of these dims runs its chain on the tcgen05 whole-head walk.
bool tc_fwd_whole_head(const gdn_dims& d);
bool launch_tc_bwd(const gdn_dims& d, const void* q, const void* k, const void* v,
                   const float* g, const float* beta, const float* h0, const void* dO,
                   const float* dhT, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                   float* dh0, void* ws, cudaStream_t st, const int* cu = nullptr, int nseq = 0,
                   bool saved = false);
// Chunk offsets of a packed batch: cstart[s] = sum over s' < s of ceil(len_s' / 64).
// An offset table that is not non-decreasing from 0 to T sets status bit 1 and
// yields no chunks.
void launch_varlen_setup(const int* cu, int nseq, int T, int* cstart, unsigned int* status,
                         cudaStream_t st);

}  // namespace gdn
