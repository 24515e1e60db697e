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
    int nseg, seglen;  // runs per chain of the segmented tcgen05 walks (1: unsegmented)
                       // and chunks per run (the last run may be shorter, never empty)
    // byte offsets into the workspace
    size_t W, Ut, P, G, Tb, S0, U, dS, dU, Qg, Kt, cstart, segE, segM, segN, end;
};

// Streaming multiprocessors of the current device (148 when it cannot be read).
inline int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
        return sms;
    cudaGetLastError();
    return 148;
}

// Runs per chain for the forward chain (and the backward's state recompute).
// With few chains, each chain of NT chunks can be cut into n runs: the maps
// of the runs (2n - 3 CTAs per chain, one per SM), a scan, then the runs
// themselves (n CTAs per chain, one per SM).  The estimate counts chain steps
// on the critical path, (waves of maps + waves of runs) x run length, plus
// half a step per scan step, against NT steps unsegmented; 3 .. 16 runs of at
// least 4 chunks are considered.
inline int seg_runs(int chains, int NT) {
    const int sms = sm_count();
    if (chains < 1) chains = 1;
    int best = 1;
    double best_cost = (double)NT * ((chains + sms - 1) / sms);
    for (int n = 3; n <= 16; ++n) {
        const int len = (NT + n - 1) / n;
        if (len < 4) break;
        const long long maps = (long long)chains * (2 * n - 3), runs = (long long)chains * n;
        const double cost = (double)len * ((maps + sms - 1) / sms + (runs + sms - 1) / sms) + 0.5 * (n - 2);
        if (cost < best_cost) { best_cost = cost; best = n; }
    }
    return best;
}

// nseq > 0: a packed batch of nseq sequences in one row of d.T tokens; the
// chunk count is bounded by ceil(T / C) + nseq.
inline TcLayout tc_layout(const gdn_dims& d, bool bwd, int nseq = 0) {
    TcLayout L{};
    L.NT = (d.T + C - 1) / C + nseq;
    L.nchunks = (size_t)(nseq ? 1 : d.B) * d.H * L.NT;
    L.nseg = nseq ? 1 : seg_runs(d.B * d.H, L.NT);
    L.seglen = (L.NT + L.nseg - 1) / L.nseg;
    L.nseg = (L.NT + L.seglen - 1) / L.seglen;
    size_t o = kStatusBytes;
    auto take = [&](size_t bytes) { size_t r = o; o += (bytes + 255) & ~(size_t)255; return r; };
    if (nseq) L.cstart = take((size_t)(nseq + 1) * 4);
    if (L.nseg > 1) {  // fp32 states: run entries E, and the maps M, N of each run
        const size_t seg = (size_t)d.B * d.H * L.nseg * DV * DK * 4;
        L.segE = take(seg);
        L.segM = take(seg);
        L.segN = take(seg);
    }
    L.W = take(L.nchunks * C * DK * 2);
    L.Ut = take(L.nchunks * C * DV * 2);
    L.P = take(L.nchunks * C * C * 2);
    L.G = take(L.nchunks * (d.gate == GDN_GATE_CHANNEL ? DK : C) * 4);
    L.Kt = take(L.nchunks * C * DK * 2);
    if (d.gate == GDN_GATE_CHANNEL) L.Qg = take(L.nchunks * C * DK * 2);
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

// Packed variable-length batches.  With `cu` null the batch is B sequences of
// T tokens and chunk n of (sequence b, head h) has image index (b*H + h)*NT + n.
// With `cu` set the tokens of N sequences are packed in one row of T tokens
// (sequence s = tokens cu[s] .. cu[s+1]-1), chunks are numbered over all
// sequences (cstart[s] = first chunk of s, cstart[N] = their count) and the
// image index is h*NT + n; NT bounds the chunk count.
struct SeqMap {
    const int* cu;      // [N+1] token offsets, or null
    const int* cstart;  // [N+1] chunk offsets (set on the device from cu)
    int N;
};

// Number of sequences the chains run over: B rows of T, or the N packed ones.
inline int chain_batches(int B, const SeqMap& m) { return m.cu ? m.N : B; }

// Token start and length of chunk n of image row bh, and its sequence.
struct ChunkLoc {
    int tok, L, seq;
    bool valid;
};
GDN_DEV ChunkLoc chunk_loc(const SeqMap& m, int T, int H, int bh, int n) {
    ChunkLoc c;
    if (!m.cu) {
        c.seq = bh / H;
        c.tok = c.seq * T + n * C;
        c.L = min(C, T - n * C);
        c.valid = true;
        return c;
    }
    c.valid = n < m.cstart[m.N];
    if (!c.valid) return c;
    int lo = 0, hi = m.N - 1;  // the last s with cstart[s] <= n
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (m.cstart[mid] <= n) lo = mid; else hi = mid - 1;
    }
    c.seq = lo;
    c.tok = m.cu[lo] + (n - m.cstart[lo]) * C;
    c.L = min(C, m.cu[lo + 1] - c.tok);
    return c;
}

// The chain of (sequence s, head h): its chunks n0 .. n1-1, their image row,
// and the first token.  The state of the chain is row s*H + h of h0 / hT.
struct Chain {
    int n0, n1, img, tok0, end;  // end: one past the chain's last token
};
GDN_DEV Chain chain_of(const SeqMap& m, int T, int H, int NT, int s, int h) {
    Chain c;
    if (!m.cu) {
        c.n0 = 0; c.n1 = NT; c.img = s * H + h; c.tok0 = s * T; c.end = (s + 1) * T;
    } else {
        c.n0 = m.cstart[s]; c.n1 = m.cstart[s + 1]; c.img = h; c.tok0 = m.cu[s]; c.end = m.cu[s + 1];
    }
    return c;
}

// Workspace images (written by prep with bulk stores, read back the same way):
//   W   [chunk] Tma128 image of the 64x128 W (two 64-column K-major panels)
//   Ut  [chunk] Swz<64> image of U~^T: 128 value rows x 64 tokens, so any
//       16-row slice of the state is one contiguous 2 KB range
//   P   [chunk][64][64]  bf16, Swz<64> tile image (scale folded in)
//   G   [chunk][64] fp32 within-chunk cumsum of g (padding rows repeat the last);
//       channel gate: [chunk][128] fp32 e^{G_last,c}, the per-key decay of a chunk
//   Qg  channel gate only: [chunk] Tma128 image of scale * Q .* e^{G}
//   Kt  [chunk] Tma128 image of K .* e^{G_last - G} (per key channel for the
//       channel gate, per token for the scalar gate)
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
    __nv_bfloat16 *Qg;  // channel gate only
    __nv_bfloat16* Kt;
    unsigned int* status;
    SeqMap seq;
    // bounded waits of the tcgen05 forward walks (see tc5_walk.cu)
    unsigned long long wait_ns = kWaitNs;
    int stall_at = -1;
    int pf_stride = 0;  // preparation: chunks a wave ahead whose gate rows go to L2 (0: none)
    // The q/k/v prologue fused into the preparation's load stage: the token
    // maps above then cover the raw projections, whose rows before a chunk
    // (the filter's history) are read from xq, xk, xv; the filtered tensors
    // ([B, T, H, 128] bf16) go to qf, kf, vf for the later kernels.
    struct Conv {
        const __nv_bfloat16 *xq, *xk, *xv;
        const float *wq, *wk, *wv;  // [H, 128, K] filters
        __nv_bfloat16 *qf, *kf, *vf;
        int K;
    } conv{};
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
