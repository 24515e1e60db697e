/*
 * gdn.h -- C ABI of the gated delta-rule layer library (libgdn.so, sm_100a).
 *
 * The operation.  "Gated Delta Networks: Improving Mamba2 with Delta Rule"
 * (paper review), section "Method": per (sequence b, head h) a matrix state
 * S in R^{dv x dk} is updated token by token as
 *
 *     S_t = S_{t-1} a_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   a_t = exp(g_t),
 *
 * and read out as o_t = S_t (scale * q_t).  GDN_GATE_SCALAR takes one log-gate
 * g_t per (token, head); GDN_GATE_CHANNEL (the Kimi-Delta-Attention variant,
 * named in the same review's linked reviews and in the "Linear Attention
 * Architectures: Mechanisms, Trade-offs, and Cross-Layer Routing" abstract)
 * takes g_t in R^{dk} and uses Diag(a_t) on the key index in place of a_t.
 * The training calls compute the same values in the chunkwise-parallel form
 * built on the WY representation and the UT transform (same review, sections
 * "Goal" and "Method"); the decode call is the recurrent form, one token per
 * call ("Background": O(1)-memory inference with a fixed-size state).
 *
 * Layouts (all row-major and contiguous; element strides are implied):
 *   q, k          [B, T, H, dk]      q/k/v/o/dO/dq/dk/dv in `dtype`
 *   v, o          [B, T, H, dv]
 *   g             [B, T, H] (scalar gate) or [B, T, H, dk] (channel gate), fp32
 *   beta          [B, T, H] fp32
 *   h0, hT, dhT, dh0   [B, H, dv, dk] fp32 (row = value index, column = key index)
 * Gradients come back in the dtype of their primal; dg, dbeta, dh0 are fp32.
 *
 * Precision.  GDN_BF16: bf16 inputs/outputs, fp32 accumulation, fp32 gate
 * cumsums and an fp32 state.  GDN_F32: fp32 end to end (no tf32).
 *
 * Ownership and streams.  The caller owns every buffer, the workspace
 * included.  The library never allocates, frees or synchronises (except
 * gdn_query_device_status), keeps no state between calls, and enqueues all
 * work on the stream it is given.  All pointers other than the host-side
 * `dims` are device pointers.
 *
 * Errors.  Every argument is validated on the host before any launch; on
 * error nothing is launched and the outputs are untouched:
 *   GDN_ERR_INVALID_ARG  null required pointer, B/T/H < 1, bad enum, pointer
 *                        not 16-byte aligned, dh0 given without h0 or the
 *                        reverse, chunk not in {16, 32, 64}, scale not finite;
 *   GDN_ERR_UNSUPPORTED  dk or dv not in {16, 32, 64, 128};
 *   GDN_ERR_WORKSPACE    ws_bytes smaller than the *_workspace() size, or a
 *                        null workspace when that size is non-zero;
 *   GDN_ERR_CUDA         a launch failed (cudaGetLastError after launch).
 * Value preconditions are documented, not checked: g finite and <= 0,
 * beta in [0, 2].  beta in (1, 2] is the negative-eigenvalue transition that
 * "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper review),
 * section "Future work", names as an extension: I - beta k k^T then flips the
 * sign along a unit k (a reflection at beta = 2).  The arithmetic is the same;
 * both ranges are tested.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,
    GDN_ERR_UNSUPPORTED = 2,
    GDN_ERR_WORKSPACE = 3,
    GDN_ERR_CUDA = 4,
    GDN_ERR_DEVICE_TIMEOUT = 5
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;
typedef enum { GDN_GATE_SCALAR = 0, GDN_GATE_CHANNEL = 1 } gdn_gate;

/* Problem description shared by the chunkwise calls.
 * chunk: tokens per chunk of the chunkwise algorithm (16, 32 or 64); the
 * result does not depend on it beyond rounding.  T need not be a multiple of
 * chunk (the tail chunk is shorter).  scale multiplies q (1 = o_t = S_t q_t). */
typedef struct {
    int B, T, H, dk, dv, chunk;
    gdn_dtype dtype;
    gdn_gate gate;
    float scale;
} gdn_dims;

/* Bytes of device workspace gdn_chunk_fwd needs for `dims` (0 if dims are
 * invalid).  The workspace must be 256-byte aligned. */
size_t gdn_chunk_fwd_workspace(const gdn_dims *dims);

/* Chunkwise forward.  Reads q, k, v, g, beta and, if not NULL, the initial
 * state h0 (NULL = zero state).  Writes o and, if not NULL, the final state
 * hT.  h0 and hT may not alias.  Chunkwise algorithm: per chunk the gate
 * cumsum, the decayed K K^T, the UT transform T = (I + A)^{-1}, the WY
 * factors, the inter-chunk fp32 state recurrence and the output products. */
gdn_status gdn_chunk_fwd(const gdn_dims *dims, const void *q, const void *k,
                         const void *v, const float *g, const float *beta,
                         const float *h0, void *o, float *hT, void *ws,
                         size_t ws_bytes, gdn_stream_t stream);

/* Bytes of device workspace gdn_chunk_bwd needs for `dims`. */
size_t gdn_chunk_bwd_workspace(const gdn_dims *dims);

/* Chunkwise backward of L = <dO, o> + <dhT, hT> (dhT NULL = 0).  The call is
 * stateless: it recomputes what it needs from the primal inputs.  Writes dq,
 * dk, dv (primal dtype), dg (shape of g), dbeta, and dh0 (required exactly
 * when h0 is given; NULL otherwise). */
gdn_status gdn_chunk_bwd(const gdn_dims *dims, const void *q, const void *k,
                         const void *v, const float *g, const float *beta,
                         const float *h0, const void *dO, const float *dhT,
                         void *dq, void *dk, void *dv, float *dg, float *dbeta,
                         float *dh0, void *ws, size_t ws_bytes,
                         gdn_stream_t stream);

/* The forward and backward of a training step, with the forward's chunk
 * products kept for the backward instead of recomputed ("Gated Delta
 * Networks: Improving Mamba2 with Delta Rule" (paper review), section
 * "Method": the per-chunk WY factors, the UT transform T and the state
 * entering each chunk are functions of the forward's inputs alone).
 * gdn_chunk_fwd_save returns what gdn_chunk_fwd returns and leaves in `ws`
 * the prepared chunk images, T, and every chunk's entering state and U;
 * gdn_chunk_bwd_saved then returns what gdn_chunk_bwd returns for the same
 * primal inputs, reading those from `ws` instead of recomputing them.  Both
 * take the same workspace: ws_bytes >= max(gdn_chunk_bwd_workspace(dims),
 * gdn_chunk_fwd_workspace(dims)), 256-byte aligned; the caller owns it and
 * must keep it, and q, k, v, g, beta, h0, unchanged from the forward until
 * the backward has run (stream order suffices).  Arguments are otherwise those
 * of gdn_chunk_fwd / gdn_chunk_bwd, with the same error returns.  For shapes
 * outside the tensor-core path the backward recomputes, as gdn_chunk_bwd. */
gdn_status gdn_chunk_fwd_save(const gdn_dims *dims, const void *q, const void *k,
                              const void *v, const float *g, const float *beta,
                              const float *h0, void *o, float *hT, void *ws,
                              size_t ws_bytes, gdn_stream_t stream);
gdn_status gdn_chunk_bwd_saved(const gdn_dims *dims, const void *q, const void *k,
                               const void *v, const float *g, const float *beta,
                               const float *h0, const void *dO, const float *dhT,
                               void *dq, void *dk, void *dv, float *dg, float *dbeta,
                               float *dh0, void *ws, size_t ws_bytes,
                               gdn_stream_t stream);

/* The training pair with the block's q/k/v prologue ("Gated Delta Networks:
 * Improving Mamba2 with Delta Rule" (paper review), section "Method": q and k
 * pass through a short convolution, SiLU and L2 normalisation, v through the
 * convolution and SiLU; gdn_short_conv_fwd below defines the filter).  The
 * forward takes the raw projections xq, xk [B,T,H,dk] and xv [B,T,H,dv] (the
 * dtype of dims) and the filters wq, wk [H,dk,K], wv [H,dv,K] fp32 (1 <= K <=
 * 4), and returns o and hT of gdn_chunk_fwd applied to the filtered q, k, v;
 * the backward returns the gradients of <dO, o> + <dhT, hT> with respect to
 * xq, xk, xv (dtype of dims), wq, wk, wv (fp32, overwritten), g, beta and h0.
 * On the tensor-core shapes with the scalar gate the filter runs inside the
 * chunk preparation's load stage: it reads the raw tiles (and the 3 tokens
 * before each chunk), filters them in shared memory and writes the filtered
 * q, k, v once for the later kernels; elsewhere the prologue runs as its own
 * pass.  Both calls take the same caller-owned workspace of
 * gdn_chunk_conv_saved_workspace(dims, K) bytes (256-byte aligned), which
 * keeps the filtered tensors, the chunk products and the chunk states between
 * them; inputs must stay unchanged from the forward until the backward has
 * run.  The batch is dims->B sequences of dims->T tokens (the filter sees
 * zeros before each sequence's first token). */
size_t gdn_chunk_conv_saved_workspace(const gdn_dims *dims, int K);
gdn_status gdn_chunk_fwd_save_conv(const gdn_dims *dims, int K, const void *xq,
                                   const void *xk, const void *xv, const float *wq,
                                   const float *wk, const float *wv, const float *g,
                                   const float *beta, const float *h0, void *o,
                                   float *hT, void *ws, size_t ws_bytes,
                                   gdn_stream_t stream);
gdn_status gdn_chunk_bwd_saved_conv(const gdn_dims *dims, int K, const void *xq,
                                    const void *xk, const void *xv, const float *wq,
                                    const float *wk, const float *wv, const float *g,
                                    const float *beta, const float *h0, const void *dO,
                                    const float *dhT, void *dxq, void *dxk, void *dxv,
                                    float *dwq, float *dwk, float *dwv, float *dg,
                                    float *dbeta, float *dh0, void *ws, size_t ws_bytes,
                                    gdn_stream_t stream);

/* Packed variable-length batches.  Each sequence of a packed batch is its own
 * instance of the recurrence of "Gated Delta Networks: Improving Mamba2 with
 * Delta Rule" (paper review), section "Method": its state starts from its
 * own h0 (or zero) and no state crosses a sequence boundary, so the result
 * for sequence s equals gdn_chunk_fwd / gdn_chunk_bwd on that sequence alone.
 * The tokens of nseq sequences sit back to back in one row: dims->B must be 1
 * and dims->T is the total token count; sequence s holds tokens
 * cu_seqlens[s] .. cu_seqlens[s+1]-1 (a device array of nseq + 1 ints,
 * 4-byte aligned, cu_seqlens[0] = 0, non-decreasing, cu_seqlens[nseq] = T;
 * empty sequences are allowed and pass h0 through to hT).  q, k, v, g, beta,
 * o and their gradients take the [1, T, H, ...] layouts above; h0, hT, dhT,
 * dh0 are [nseq, H, dv, dk].  Chunks never straddle a boundary: each sequence
 * is cut into chunks of 64 from its own first token.
 * Tensor-core shapes only (GDN_BF16, dk = dv = 128, chunk = 64), else
 * GDN_ERR_UNSUPPORTED; nseq < 1 or B != 1 is GDN_ERR_INVALID_ARG.  The offsets
 * are device data and are checked on the device: offsets that break the rules
 * above leave the outputs unspecified and make gdn_query_device_status on
 * this workspace return GDN_ERR_INVALID_ARG.  The workspace depends on nseq. */
size_t gdn_chunk_fwd_varlen_workspace(const gdn_dims *dims, int nseq);
gdn_status gdn_chunk_fwd_varlen(const gdn_dims *dims, const int *cu_seqlens,
                                int nseq, const void *q, const void *k,
                                const void *v, const float *g,
                                const float *beta, const float *h0, void *o,
                                float *hT, void *ws, size_t ws_bytes,
                                gdn_stream_t stream);
size_t gdn_chunk_bwd_varlen_workspace(const gdn_dims *dims, int nseq);
gdn_status gdn_chunk_bwd_varlen(const gdn_dims *dims, const int *cu_seqlens,
                                int nseq, const void *q, const void *k,
                                const void *v, const float *g,
                                const float *beta, const float *h0,
                                const void *dO, const float *dhT, void *dq,
                                void *dk, void *dv, float *dg, float *dbeta,
                                float *dh0, void *ws, size_t ws_bytes,
                                gdn_stream_t stream);

/* The q/k/v prologue: "Gated Delta Networks: Improving Mamba2 with Delta
 * Rule" (paper review), section "Method": q and k pass through a short
 * convolution and SiLU, then L2 normalisation; v takes the same path without
 * the norm.  Read as a causal depthwise filter of K taps per channel with
 * zeros before each sequence's first token (no bias):
 *     z_t[c] = sum_{j<K} w[h, c, j] x_t-j[c],   s = z * sigmoid(z),
 *     y = s / sqrt(sum_c s_c^2 + 1e-6)  over the d channels of one head
 *     (l2norm != 0; otherwise y = s).
 * gdn_short_conv_fwd writes y; gdn_short_conv_bwd writes dx and dw for the
 * loss <dy, y> (dw is overwritten, not accumulated, and summed in a fixed
 * order, so it is deterministic).  Layouts (contiguous, device): x, y, dy, dx
 * [B, T, H, d] in `dtype` (bf16 or fp32); w, dw [H, d, K] fp32.  x and y may
 * not alias, nor dx and x or dy.  d in {32, 64, 128} and 1 <= K <= 4 (else
 * GDN_ERR_UNSUPPORTED / GDN_ERR_INVALID_ARG); x, y, dy, dx 16-byte aligned;
 * the backward workspace (gdn_short_conv_bwd_workspace bytes, 256-byte
 * aligned) holds one weight-gradient partial per 32-token tile of a head. */
gdn_status gdn_short_conv_fwd(int B, int T, int H, int d, int K, gdn_dtype dtype,
                              int l2norm, const void *x, const float *w, void *y,
                              gdn_stream_t stream);
size_t gdn_short_conv_bwd_workspace(int B, int T, int H, int d, int K);
gdn_status gdn_short_conv_bwd(int B, int T, int H, int d, int K, gdn_dtype dtype,
                              int l2norm, const void *x, const float *w,
                              const void *dy, void *dx, float *dw, void *ws,
                              size_t ws_bytes, gdn_stream_t stream);

/* Draft-tree verification and commit: "TreeWY: Speculative Verification for
 * Gated DeltaNet Hybrids" (the "Linked reviews" entry of the "Gated Delta
 * Networks: Improving Mamba2 with Delta Rule" review page).  Per (sequence n, head h) a speculative draft tree of M nodes hangs
 * below the committed state S = state[n, h]: node i carries one token and a
 * parent index parent[n, i] in [-1, i) (-1: the node follows S directly;
 * parents precede children).  Node i's output is the gated delta rule of
 * gdn_chunk_fwd run from S over the tokens of its root path, read out at i.
 * gdn_tree_verify computes all M outputs in one pass without any per-node
 * state: the chunkwise WY/UT algebra with the causal mask replaced by the
 * ancestor relation (one triangular solve per tree), reading S once.
 * gdn_tree_commit replaces S by the state after the root path of node
 * accepted[n] (-1 or nothing accepted: S is left untouched), by the
 * recurrent form along that path on the fp32 state.
 * Layouts (contiguous): parent [N, M] int32; accepted [N] int32; q, k
 * [N, M, H, dk]; v, o [N, M, H, dv]; g [N, M, H] fp32 (scalar gate) or
 * [N, M, H, dk] fp32 (channel gate: the decay of node t is Diag(e^{g_t}) on
 * the key index); beta [N, M, H] fp32; state [N, H, dv, dk] fp32 (row =
 * value index).  All device pointers.
 * Supported: GDN_BF16, either gate, dk = dv = 128, 1 <= M <= 64 (else
 * GDN_ERR_UNSUPPORTED); N, H, M < 1, null pointers or misalignment (16 bytes
 * for q, k, v, o, state and a channel-gate g; 4 for the rest) are
 * GDN_ERR_INVALID_ARG.
 * Tree indices are device data and are checked on the device: a parent out
 * of [-1, i) is read as -1 and an accepted index out of [-1, M) as -1; either
 * sets bit 1 (value 2) of the optional device word *status (may be NULL),
 * which gdn_query_device_status(status, stream) then reports as
 * GDN_ERR_INVALID_ARG.  state is read-only in gdn_tree_verify and updated in
 * place by gdn_tree_commit; q, k, v, g, beta may be shared by both calls. */
gdn_status gdn_tree_verify(int N, int M, int H, int dk, int dv, gdn_dtype dtype,
                           gdn_gate gate, float scale, const int *parent,
                           const void *q, const void *k, const void *v,
                           const float *g, const float *beta,
                           const float *state, void *o, unsigned int *status,
                           gdn_stream_t stream);
gdn_status gdn_tree_commit(int N, int M, int H, int dk, int dv, gdn_dtype dtype,
                           gdn_gate gate, const int *parent, const int *accepted,
                           const void *k, const void *v, const float *g,
                           const float *beta, float *state, unsigned int *status,
                           gdn_stream_t stream);

/* Gated DeltaProduct: "DeltaProduct: Improving State-Tracking in Linear RNNs
 * via Householder Products" (in the list of related papers of the "Linear
 * Attention Architectures: Mechanisms, Trade-offs, and Cross-Layer Routing"
 * summary page) with the gate of "Gated Delta Networks: Improving Mamba2
 * with Delta Rule" (paper review), whose section "Future work" names
 * products of Householder matrices as an extension.  The pages give no
 * equation; the reading: each token applies its gate once, then n delta-rule
 * steps with its own keys, values and betas in order j = 1..n, and is read
 * out after the last,
 *     S <- S D_t;  S <- S (I - b_tj k_tj k_tj^T) + b_tj v_tj k_tj^T;  o_t = S (scale q_t).
 * That is the gated delta rule on the n*T sub-tokens (t, 1) .. (t, n) with
 * g_t on the first and q_t read at the last, and it runs as exactly that:
 * gdn_chunk_fwd / gdn_chunk_bwd over T' = n*T, around device copies that
 * spread q, g (and dO) over the sub-tokens and gather o (dq, dg) back.
 * dims->T is the token count; 1 <= n <= 64 and n*T must fit an int.
 * Layouts (contiguous): q [B,T,H,dk]; k [B,T,n,H,dk]; v [B,T,n,H,dv];
 * beta [B,T,n,H] fp32; g, h0, hT as in gdn_chunk_fwd; o [B,T,H,dv].  The
 * gradients take the shapes of their primals.  The workspace holds the inner
 * call's workspace first, so gdn_query_device_status works on it.
 * Errors: GDN_ERR_INVALID_ARG for n out of range or a null q, g, o (dO, dq,
 * dg); otherwise those of gdn_chunk_fwd / gdn_chunk_bwd for T' = n*T. */
size_t gdn_product_fwd_workspace(const gdn_dims *dims, int n);
gdn_status gdn_product_fwd(const gdn_dims *dims, int n, const void *q,
                           const void *k, const void *v, const float *g,
                           const float *beta, const float *h0, void *o,
                           float *hT, void *ws, size_t ws_bytes,
                           gdn_stream_t stream);
size_t gdn_product_bwd_workspace(const gdn_dims *dims, int n);
gdn_status gdn_product_bwd(const gdn_dims *dims, int n, const void *q,
                           const void *k, const void *v, const float *g,
                           const float *beta, const float *h0, const void *dO,
                           const float *dhT, void *dq, void *dk, void *dv,
                           float *dg, float *dbeta, float *dh0, void *ws,
                           size_t ws_bytes, gdn_stream_t stream);

/* One decode token for N sequences x H heads, in place on the state.
 * q, k [N, H, dk]; v, o [N, H, dv] in `dtype`; g [N, H] (scalar) or
 * [N, H, dk] (channel) fp32; beta [N, H] fp32; state [N, H, dv, dk] fp32,
 * read once and written once.  o_t uses the updated state. */
gdn_status gdn_recurrent_step(int N, int H, int dk, int dv, gdn_dtype dtype,
                              gdn_gate gate, float scale, const void *q,
                              const void *k, const void *v, const float *g,
                              const float *beta, float *state, void *o,
                              gdn_stream_t stream);

/* Test hook for the bounded device waits (no counterpart in the paper): runs
 * gdn_chunk_fwd's tensor-core forward with the loads of chain step
 * `stall_at` (and after) never issued, so the waits on that step, which no
 * copy, MMA or thread will ever complete, give up after `wait_ns`
 * nanoseconds (1 .. 1e9).  Every role then stops; loads and MMAs already
 * issued are drained (those waits keep the 1 s limit), tensor memory is
 * freed, and the kernel returns with bit 0 of the workspace's status word
 * set, so gdn_query_device_status reports GDN_ERR_DEVICE_TIMEOUT.  o and hT
 * are then not valid.  Only shapes whose forward chain runs on the tcgen05
 * whole-head walk are accepted (bf16, dk = dv = 128, chunk 64, scalar or
 * channel gate, B*H*4 >= the SM count; GDN_ERR_UNSUPPORTED otherwise).
 * Arguments and workspace as gdn_chunk_fwd. */
gdn_status gdn_test_stalled_fwd(const gdn_dims *dims, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *h0, void *o, float *hT, void *ws,
                                size_t ws_bytes, int stall_at, unsigned long long wait_ns,
                                gdn_stream_t stream);

/* Synchronises `stream`, then reads and clears the status word kept in the
 * first bytes of a chunkwise workspace.  Each chunkwise call clears that word
 * (a 4-byte memset on its stream) before its kernels run, and a kernel whose
 * bounded device wait gives up sets it, so the answer covers the most recent
 * call on `ws`: GDN_ERR_DEVICE_TIMEOUT if a wait gave up, GDN_ERR_INVALID_ARG
 * if the offsets of a packed batch were invalid, else GDN_OK. */
gdn_status gdn_query_device_status(void *ws, gdn_stream_t stream);

/* Allocation-free chunkwise forward, for callers that cannot call
 * cudaMalloc (a fixed device-memory budget the allocator must not touch, a
 * runtime that provides no device allocation, or host code that must not
 * allocate between steps).  The paper has no counterpart: this is a
 * deployment variant of gdn_chunk_fwd.  Same arguments and results as
 * gdn_chunk_fwd minus the workspace: the workspace is a 64 MiB array built
 * into the library (a file-scope device variable that every GPU loading the
 * library holds until the process exits), so the caller passes only inputs
 * and outputs.  Supported shapes are those of the tensor-core path (bf16,
 * dk = dv = 128, chunk 64, scalar gate; GDN_ERR_UNSUPPORTED otherwise) whose
 * workspace, as gdn_chunk_fwd_workspace reports it, fits 64 MiB: about 72 KiB
 * per chunk-head, plus 192 KiB per run when few chains are cut into runs
 * (GDN_ERR_WORKSPACE otherwise, checked on the host before anything runs).
 * No cudaMalloc, cudaFree or other allocating call is made.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress),
 * so make that first call before any stream capture.  All calls share the
 * one array and a call leaves its contents behind: the call clears the word
 * that must start at zero itself, but calls that overlap on the GPU (other
 * streams, other host threads) race on the array and must be serialised by
 * the caller.  The array's address is looked up once per device and kept
 * for the life of the process, so these calls must not be used after
 * cudaDeviceReset (or anything else that destroys the device's primary
 * context) in the same process.  A device wait of these calls that gives up
 * is reported by gdn_noalloc_device_status, not by the return value. */
gdn_status gdn_chunk_fwd_noalloc(const gdn_dims *dims, const void *q, const void *k,
                                 const void *v, const float *g, const float *beta,
                                 const float *h0, void *o, float *hT,
                                 gdn_stream_t stream);

/* Companion of gdn_chunk_fwd_noalloc, with no counterpart in the paper
 * either: synchronises `stream`, then reads and clears the status word at
 * the start of the library's built-in array on the current device, exactly
 * as gdn_query_device_status does for a caller's workspace.  The answer
 * covers the most recent gdn_chunk_fwd_noalloc call on this device:
 * GDN_ERR_DEVICE_TIMEOUT if one of its bounded device waits gave up (its
 * o / hT are then not valid), else GDN_OK; GDN_ERR_CUDA if a CUDA call
 * failed.  Allocates nothing. */
gdn_status gdn_noalloc_device_status(gdn_stream_t stream);

/* Per-launch timing, a profiling aid (off by default; no compute happens in
 * these calls).  gdn_profile_begin(capacity) makes the calling host thread's
 * next `capacity` kernel launches by this library record a CUDA event before
 * and after each launch, on that launch's stream.  gdn_profile_end() stops
 * recording, waits for the recorded events, writes up to `capacity` launch
 * durations in milliseconds to `ms` and the kernel names (static strings) to
 * `names` (either may be NULL), and returns how many launches were made while
 * recording (may exceed what was stored), or -1 if recording was not on or a
 * CUDA call failed.  Events are created on the first begin and kept. */
gdn_status gdn_profile_begin(int capacity);
int gdn_profile_end(float *ms, const char **names, int capacity);

/* Static, human-readable name of a status code. */
const char *gdn_status_string(gdn_status status);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
