// tc5_walk.cu -- the forward's chunk chain on the fifth-generation tensor cores.
//
// One CTA carries one head's whole 128x128 state through its chunks (the
// chain of "Gated Delta Networks: Improving Mamba2 with Delta Rule" (paper
// review), section "Method": U = U~ - W S0^T, O = scale diag(e^G) Q S0^T + P U,
// S1 = e^{G_last} S0 + U^T diag(e^{G_last - G}) K), with every product on
// tcgen05 MMAs whose accumulators sit in tensor memory:
//   [X | Y] = -S0 [W ; Q]^T  (128 x 128, B negated in the instruction
//                             descriptor; one N = 128 MMA per K step)
//   X      += U~^T           (four N = 16 MMAs against a 16x16 identity), so X
//                             is U itself and Y = -S0 Q^T
//   D = U^T K~  (128 x 128, K~ = diag(e^{G_last - G}) K, an image from prep)
//   Z = U^T P^T (128 x 64)
// The A operands of the chain (the bf16 state and U) are written by the
// epilogue straight into tensor memory; U~^T arrives in shared memory with the
// chunk's other tiles and enters the accumulator through the identity, so the
// epilogue neither loads nor subtracts it.  The fp32 state lives in the
// epilogue threads' registers (thread = state row, 32 key columns each);
// every step they add D to it and store its bf16 copy as the next step's A
// operand, so the state itself never leaves fp32.
//
// Warp roles: warps 0..15 are the epilogue (TMEM lane quarter = warp % 4,
// column group = warp / 4); warp 16 allocates TMEM and its lane 0 issues
// every MMA; lane 0 of warp 17 issues the chunk loads into a three-stage
// ring as stages are released.  Per step the chain is
//   [X|Y], X += U~ -> U -> D -> S update + state image -> next [X|Y],
// with Z and the output store off the chain.  The epilogue reads X and Y
// together, so each accumulator needs only one buffer.
//
// MODE 1 (state recompute for the backward) has no output: it fetches
// neither Q nor P, runs X alone in place of [X|Y], skips Z, and stores each
// chunk's entering state (bf16, Kp<128> image: two 64-key panels of 128
// rows) and U (Tma128, token rows) for the backward kernels.  MODE 3 (the
// forward of a training step) does both: the outputs of MODE 0 and the
// stores of MODE 1, so the backward need not walk the chain again.
//
// Channel gate: Q arrives as the prepared image scale Q .* e^G, K~ is
// K .* e^{G_last - G} per key channel, G holds e^{G_last,c}, and the decay of
// the state is per key column.
#include "async.cuh"
#include "common.cuh"
#include "internal.h"
#include "mma.cuh"
#include "tc5.cuh"
#include "tc_common.cuh"

#include <type_traits>

namespace gdn {
namespace tc {
void launch_seg_scan(float* E, const float* Mmap, const float* Nmap, int nseg, int chains,
                     unsigned int* status, cudaStream_t st);
}
namespace {
using namespace tc;

constexpr int W5_EPI_WARPS = 16;
constexpr int W5_CTRL = W5_EPI_WARPS;      // MMA warp
constexpr int W5_PROD = W5_EPI_WARPS + 1;  // load warp
constexpr int W5_SAVE = W5_EPI_WARPS + 2;  // MODE 3: bulk stores of the chunk states
constexpr uint32_t NEG_B = 1u << 14;       // instruction descriptor: negate B
constexpr uint32_t ID_XY = tc5::idesc_bf16(128, 128, false, false) | NEG_B;
constexpr uint32_t ID_X = tc5::idesc_bf16(128, 64, false, false) | NEG_B;
constexpr uint32_t ID_UI = tc5::idesc_bf16(128, 16, false, false);
constexpr uint32_t ID_D = tc5::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_Z = tc5::idesc_bf16(128, 64, false, false);

// MODE 0: forward (O, hT).  MODE 1: state recompute for the backward (chunk
// states S0 and U stored).  MODE 2: a segment's affine map (final state only).
// MODE 3: forward that also stores S0 and U.
// Forward stage: [W p0 | Q p0 | W p1 | Q p1] (K-major B of [X|Y], 128 rows per
// 64-key panel, 8 KB each), K~, U~^T, P.
struct alignas(1024) W5Stage {
    __nv_bfloat16 WQ[2 * C * DK];
    __nv_bfloat16 K[C * DK];   // Tma128 image of K .* e^{G_last - G}: MN-major B of D
    __nv_bfloat16 Ut[DV * C];  // Swz<64> U~^T (value rows x tokens): K-major A of X += U~^T
    __nv_bfloat16 P[C * C];    // Swz<64>: K-major B of Z
};
// Stage without outputs: W (Tma128, K-major B of X), K~, U~^T.
struct alignas(1024) W5LeanStage {
    __nv_bfloat16 W[C * DK];
    __nv_bfloat16 K[C * DK];
    __nv_bfloat16 Ut[DV * C];
};

template <int MODE>
struct W5Cfg {
    static constexpr bool FULL = MODE == 0 || MODE == 3;  // outputs: Q, P, [X|Y], Z
    static constexpr bool SAVE = MODE == 1 || MODE == 3;  // S0 and U images stored
    // MODE 3 stages each chunk state in shared memory (two 32 KiB buffers) for
    // a bulk store by a warp of its own, so its ring has two stages
    static constexpr bool STAGED = MODE == 3;
    static constexpr int STAGES = MODE == 0 ? 3 : 2;
    static constexpr int THREADS = 32 * (W5_EPI_WARPS + 2 + (STAGED ? 1 : 0));
    // tensor-memory columns.  Forward: [X|Y] 0..127, D, Z (two buffers, by
    // step parity: a step's output is read during the next step), then the A
    // operands S (bf16 pairs) and U.  Lean: X and D share columns 0..127 (D is
    // issued only after the epilogue has read X), so two CTAs fit an SM.
    static constexpr int TXY = 0, TD = FULL ? 128 : 0, TZ = 256, TAS = FULL ? 320 : 128,
                         TAU = FULL ? 384 : 192, TZ2 = 448, TCOLS = FULL ? 512 : 256;
};

// The staged state images of MODE 3 and their hand-off barriers
template <bool STAGED>
struct W5Save {
    __nv_bfloat16 S0[2][DV * DK];  // Kp<128> image of the state entering a step
    uint64_t full[2], empty[2];
};
template <>
struct W5Save<false> {};

template <int MODE>
struct W5Smem {
    W5Save<W5Cfg<MODE>::STAGED> sv;
    using Stage = typename std::conditional<W5Cfg<MODE>::FULL, W5Stage, W5LeanStage>::type;
    Stage st[W5Cfg<MODE>::STAGES];
    __nv_bfloat16 I16[16 * 64];  // 16x16 identity, Swz<64> rows: B of X += U~^T
    float G[W5Cfg<MODE>::STAGES][DK];  // G (scalar gate, C used) or e^{G_last,c}
    uint64_t full[W5Cfg<MODE>::STAGES], empty[W5Cfg<MODE>::STAGES];
    uint64_t s_ready, u_ready, x_done, d_done, o_done[2], fin;
    uint32_t tmem;
};

struct W5Ptrs {
    CUtensorMap qmap;
    const float* h0;
    const __nv_bfloat16 *W, *Ut, *P, *Qg, *Kt;
    const float* G;
    __nv_bfloat16* o;
    float* hT;
    __nv_bfloat16 *S0out, *Uout;  // MODE 1 and 3
    unsigned int* status;
    int B, T, H, NT;
    float scale;
    SeqMap seq;
    // Segments: each chain of chunks is cut into nseg runs of seglen chunks
    // (nseg = 1: one run).  E[(bh*nseg + j)] holds the fp32 state entering
    // run j (j >= 1); MODE 2 writes E[..+1] from run 0 and the maps M, N of
    // runs 1 .. nseg-2 (state after the run from I without U~, from 0 with U~).
    int nseg, seglen;
    float *E, *Mmap, *Nmap;
    // Bounded waits: limit of every wait that does not guard a copy or an MMA
    // in flight at teardown (those use the default), and a test hook that
    // stops the loads before step stall_at (-1: never) so that the waits on
    // that stage, which nothing will complete, run out.
    unsigned long long wait_ns;
    int stall_at;
};

template <bool KDA, int MODE>
__device__ void w5_issue(typename W5Smem<MODE>::Stage& st, float* G, uint64_t* bar, const W5Ptrs& p,
                         const Chain& ch, int h, int n, bool use_u) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + n;  // step n of the chain
    constexpr int GW = KDA ? DK : C;
    constexpr int PANEL = C * 64;  // elements of one 64x64 panel
    const __nv_bfloat16* W = p.W + cid * C * DK;
    const int tok = ch.tok0 + n * C;
    if constexpr (W5Cfg<MODE>::FULL) {
        mbar_arrive_expect(bar, (3 * C * DK + DV * C + C * C) * 2 + GW * 4);  // W, Q, K~, U~^T, P
        bulk_g2s(st.WQ, W, PANEL * 2, bar);
        bulk_g2s(st.WQ + 2 * PANEL, W + PANEL, PANEL * 2, bar);
        if (KDA) {
            const __nv_bfloat16* Qg = p.Qg + cid * C * DK;
            bulk_g2s(st.WQ + PANEL, Qg, PANEL * 2, bar);
            bulk_g2s(st.WQ + 3 * PANEL, Qg + PANEL, PANEL * 2, bar);
        } else {
            tma_load_3d(st.WQ + PANEL, &p.qmap, 0, h, tok, bar);
            tma_load_3d(st.WQ + 3 * PANEL, &p.qmap, 64, h, tok, bar);
        }
        bulk_g2s(st.P, p.P + cid * C * C, C * C * 2, bar);
        bulk_g2s(st.Ut, p.Ut + cid * C * DV, DV * C * 2, bar);
    } else {
        mbar_arrive_expect(bar, (2 * C * DK + (use_u ? DV * C : 0)) * 2 + GW * 4);  // W, K~, U~^T
        bulk_g2s(st.W, W, C * DK * 2, bar);
        if (use_u) bulk_g2s(st.Ut, p.Ut + cid * C * DV, DV * C * 2, bar);
    }
    bulk_g2s(st.K, p.Kt + cid * C * DK, C * DK * 2, bar);
    bulk_g2s(G, p.G + cid * GW, GW * 4, bar);
}

// Warp-uniform bounded wait: every lane agrees on the outcome.
GDN_DEV bool wait_all(uint64_t* bar, uint32_t parity, unsigned int* status,
                      unsigned long long limit_ns) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, limit_ns));
}

// One arrival per warp, after all of its lanes' prior writes.
GDN_DEV void warp_arrive(uint64_t* bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// What one CTA walks: chain steps n_begin .. n_end-1 of state row bh, from
// `start` (kStartH0: h0 or zero; kStartE: the run's entry state; kStartI: the
// identity; kStartZero), with or without U~, ending in `out` (hT, E, M or N).
enum { kStartH0, kStartE, kStartI, kStartZero };
struct W5Job {
    int bh, n_begin, n_end, start;
    bool use_u;
    float* out;
};

template <int MODE>
GDN_DEV W5Job w5_job(const W5Ptrs& p, int nsteps_of_chain_unused) {
    W5Job jb;
    (void)nsteps_of_chain_unused;
    if constexpr (MODE == 2) {
        const int per = 2 * p.nseg - 3;  // run 0 from h0, then (M, N) of runs 1 .. nseg-2
        const int b = blockIdx.x / per, job = blockIdx.x % per;
        jb.bh = b;
        const int j = job == 0 ? 0 : 1 + (job - 1) / 2;
        jb.n_begin = j * p.seglen;
        jb.n_end = jb.n_begin + p.seglen;
        const size_t slot = ((size_t)b * p.nseg + j) * DV * DK;
        if (job == 0) {
            jb.start = kStartH0; jb.use_u = true; jb.out = p.E + slot + (size_t)DV * DK;
        } else if ((job - 1) % 2 == 0) {
            jb.start = kStartI; jb.use_u = false; jb.out = p.Mmap + slot;
        } else {
            jb.start = kStartZero; jb.use_u = true; jb.out = p.Nmap + slot;
        }
    } else {
        const int b = blockIdx.x / p.nseg, j = blockIdx.x % p.nseg;
        jb.bh = b;
        jb.n_begin = j * p.seglen;
        jb.n_end = (j + 1) * p.seglen;  // clipped to the chain below
        jb.start = j == 0 ? kStartH0 : kStartE;
        jb.use_u = true;
        jb.out = (W5Cfg<MODE>::FULL && j == p.nseg - 1 && p.hT) ? p.hT + (size_t)b * DV * DK : nullptr;
    }
    return jb;
}

// The same tiles of chain step n, pulled into L2 ahead of the ring (the saving
// forward with the scalar gate: 350M-scale forward 176.6 -> 174.3 us; with the
// channel gate it measured slower and is left out).
template <bool KDA, int MODE>
__device__ void w5_prefetch(const W5Ptrs& p, const Chain& ch, int h, int n) {
    const size_t cid = (size_t)ch.img * p.NT + ch.n0 + n;
    constexpr int GW = KDA ? DK : C;
    const int tok = ch.tok0 + n * C;
    bulk_prefetch_l2(p.W + cid * C * DK, C * DK * 2);
    if (KDA) bulk_prefetch_l2(p.Qg + cid * C * DK, C * DK * 2);
    else tma_prefetch_tile(&p.qmap, h, tok);
    bulk_prefetch_l2(p.P + cid * C * C, C * C * 2);
    bulk_prefetch_l2(p.Ut + cid * C * DV, DV * C * 2);
    bulk_prefetch_l2(p.Kt + cid * C * DK, C * DK * 2);
    bulk_prefetch_l2(p.G + cid * GW, GW * 4);
}
template <bool KDA, int MODE>
__global__ void __launch_bounds__(W5Cfg<MODE>::THREADS) tc5_walk_kernel(const __grid_constant__ W5Ptrs p) {
    using Cfg = W5Cfg<MODE>;
    using Smem = W5Smem<MODE>;
    constexpr int NST = Cfg::STAGES;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Smem& s = *reinterpret_cast<Smem*>(align1k(smem_raw));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    W5Job jb = w5_job<MODE>(p, 0);
    const int bh = jb.bh, h = bh % p.H;  // bh: state row (sequence * H + head)
    const Chain ch = chain_of(p.seq, p.T, p.H, p.NT, bh / p.H, h);
    const int n_begin = min(jb.n_begin, ch.n1 - ch.n0), n_end = min(jb.n_end, ch.n1 - ch.n0);
    const int nsteps = n_end - n_begin;  // steps of this CTA (chain steps n_begin ..)

    if (tid == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + W5_EPI_WARPS);
        }
        mbar_init(&s.s_ready, W5_EPI_WARPS);
        mbar_init(&s.u_ready, W5_EPI_WARPS);
        mbar_init(&s.x_done, 1);
        mbar_init(&s.d_done, 1);
        mbar_init(&s.o_done[0], 1);
        mbar_init(&s.o_done[1], 1);
        mbar_init(&s.fin, 1);
        if constexpr (Cfg::STAGED) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(&s.sv.full[i], W5_EPI_WARPS);
                mbar_init(&s.sv.empty[i], 1);
            }
        }
        fence_mbar_init();
    }
    // the 16x16 identity (rows of 64 elements, 128-byte swizzle)
    for (int e = tid; e < 16 * 64; e += Cfg::THREADS) {
        const int r = e >> 6, c = e & 63;
        s.I16[swz<64>(r, c)] = __float2bfloat16_rn(r == c ? 1.f : 0.f);
    }
    fence_async_smem();
    if (warp == W5_CTRL) tc5::alloc(&s.tmem, Cfg::TCOLS);
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem;

    if (warp == W5_PROD) {
        if (lane == 0) {
            int issued = 0;
            for (int n = 0; n < nsteps; ++n) {
                const int sn = n % NST;
                if (n == p.stall_at) break;  // test hook: leave this stage unloaded
                if (n >= NST && !mbar_wait(&s.empty[sn], ((n / NST) - 1) & 1, p.status, p.wait_ns)) break;
                w5_issue<KDA, MODE>(s.st[sn], s.G[sn], &s.full[sn], p, ch, h, n_begin + n, jb.use_u);
                if (MODE == 3 && !KDA && n + NST < nsteps) w5_prefetch<KDA, MODE>(p, ch, h, n_begin + n + NST);
                issued = n + 1;
            }
            // Leave no load in flight (returns at once for stages already consumed).
            for (int n = max(0, issued - NST); n < issued; ++n)
                mbar_wait(&s.full[n % NST], (n / NST) & 1, p.status);
        }
        __syncwarp();
    } else if (warp == W5_CTRL) {
        if (lane == 0) {
            const uint32_t sI = smem_u32(s.I16);
            for (int n = 0; n < nsteps; ++n) {
                const int sn = n % NST;
                auto& st = s.st[sn];
                if (!mbar_wait(&s.full[sn], (n / NST) & 1, p.status, p.wait_ns)) break;
                if (!mbar_wait(&s.s_ready, n & 1, p.status, p.wait_ns)) break;
                tc5::fence_after();
                const uint32_t sK = smem_u32(st.K), sU = smem_u32(st.Ut);
                // [X|Y] = -S0 [W;Q]^T (X alone without outputs), then X += U~^T:
                // X is U itself
                if constexpr (Cfg::FULL) {
                    const uint32_t sWQ = smem_u32(st.WQ);
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        tc5::mma_ts(tm + Cfg::TXY, tm + Cfg::TAS + 8 * kk, tc5::kmajor<2 * C>(sWQ, kk),
                                    ID_XY, kk > 0);
                } else {
                    const uint32_t sW = smem_u32(st.W);
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        tc5::mma_ts(tm + Cfg::TXY, tm + Cfg::TAS + 8 * kk, tc5::kmajor<C>(sW, kk), ID_X,
                                    kk > 0);
                }
                if (jb.use_u) {
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        tc5::mma(tm + Cfg::TXY + 16 * kk, tc5::kmajor<DV>(sU, kk), tc5::kmajor<16>(sI, 0),
                                 ID_UI, true);
                }
                tc5::commit(&s.x_done);
                if (!mbar_wait(&s.u_ready, n & 1, p.status, p.wait_ns)) break;
                tc5::fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    tc5::mma_ts(tm + Cfg::TD, tm + Cfg::TAU + 8 * kk, tc5::mnmajor(sK, kk, C * 128), ID_D,
                                kk > 0);
                tc5::commit(&s.d_done);
                if constexpr (Cfg::FULL) {  // onto -scale e^{G_i} Y, stored by the epilogue
                    const uint32_t sP = smem_u32(st.P), tz = tm + ((n & 1) ? Cfg::TZ2 : Cfg::TZ);
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        tc5::mma_ts(tz, tm + Cfg::TAU + 8 * kk, tc5::kmajor<C>(sP, kk), ID_Z, true);
                    tc5::commit(&s.o_done[n & 1]);
                }
                tc5::commit(&s.empty[sn]);
            }
            // Leave nothing in flight: every MMA retired.
            tc5::commit(&s.fin);
            mbar_wait(&s.fin, 0, p.status);
        }
        __syncwarp();
    } else if (warp == W5_SAVE) {
        // MODE 3: bulk-store each staged chunk state to its image, then hand the
        // buffer back (state m of this CTA in buffer m & 1)
        if constexpr (Cfg::STAGED) {
            if (lane == 0) {
                int issued = 0;
                for (int m = 0; m < nsteps; ++m) {
                    if (!mbar_wait(&s.sv.full[m & 1], (m >> 1) & 1, p.status, p.wait_ns)) break;
                    bulk_s2g(p.S0out + ((size_t)ch.img * p.NT + ch.n0 + n_begin + m) * DV * DK, s.sv.S0[m & 1],
                             DV * DK * 2);
                    bulk_commit();
                    issued = m + 1;
                    bulk_wait_read<0>();
                    mbar_arrive(&s.sv.empty[m & 1]);
                }
                (void)issued;
                bulk_wait<0>();  // every store complete before the CTA exits
            }
            __syncwarp();
        }
    } else {
        // ---- epilogue: thread = state row a; key columns 32*cg .. +31 of the
        // state, tokens 16*cg .. +15 of U and O ---------------------------------
        const int q = warp & 3, cg = warp >> 2, a = 32 * q + lane;
        const uint32_t trow = tm + ((uint32_t)(32 * q) << 16);
        const int t0 = 16 * cg;  // first token of this thread's U / O columns
        float S[32];
        {
            const float* src = nullptr;
            if (jb.start == kStartH0 && p.h0) src = p.h0 + (size_t)bh * DV * DK;
            if (jb.start == kStartE) src = p.E + ((size_t)bh * p.nseg + jb.n_begin / p.seglen) * DV * DK;
            if (src) src += (size_t)a * DK + 32 * cg;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
            }
            if (jb.start == kStartI) {
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = (32 * cg + j == a) ? 1.f : 0.f;
            }
        }
        auto store_state = [&]() {  // bf16 pairs of this thread's 32 key columns
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = pack_bf16(S[2 * j], S[2 * j + 1]);
            tc5::st16(trow + Cfg::TAS + 16 * cg, r);
            tc5::wait_st();
        };
        // MODE 1: bf16 state entering chain step n, Kp<128> image (64 bytes of a
        // row per thread, whole sectors per store).  MODE 3: the same image
        // staged in shared memory (buffer m & 1 for this CTA's m-th state,
        // m = n - n_begin) for the saver warp's bulk store.
        auto store_s0 = [&](int n) {
            __nv_bfloat16* dst = p.S0out + ((size_t)ch.img * p.NT + ch.n0 + n) * DV * DK;
            if constexpr (Cfg::STAGED) {
                const int m = n - n_begin;
                if (m >= 2 && !wait_all(&s.sv.empty[m & 1], ((m >> 1) - 1) & 1, p.status, p.wait_ns))
                    return false;
                dst = s.sv.S0[m & 1];
            }
            if constexpr (Cfg::STAGED) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = 32 * cg + 8 * j;
                    *reinterpret_cast<uint4*>(dst + Kp<DV>::off(a, c)) =
                        make_uint4(pack_bf16(S[8 * j], S[8 * j + 1]), pack_bf16(S[8 * j + 2], S[8 * j + 3]),
                                   pack_bf16(S[8 * j + 4], S[8 * j + 5]), pack_bf16(S[8 * j + 6], S[8 * j + 7]));
                }
            } else {
                // global memory: lanes 2i, 2i+1 (rows a, a+1 of one swizzle group) trade
                // a 16-byte piece so that each store covers whole 32-byte sectors
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) pk[j] = pack_bf16(S[2 * j], S[2 * j + 1]);
                const bool odd = lane & 1;
                const int re = odd ? a - 1 : a, ro = odd ? a : a + 1;
#pragma unroll
                for (int hs = 0; hs < 2; ++hs) {
                    uint32_t x[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        x[w] = __shfl_xor_sync(0xffffffffu, odd ? pk[8 * hs + w] : pk[8 * hs + 4 + w], 1);
                    const int c = 32 * cg + 16 * hs + (odd ? 8 : 0);
                    *reinterpret_cast<uint4*>(dst + Kp<DV>::off(re, c)) =
                        odd ? make_uint4(x[0], x[1], x[2], x[3])
                            : make_uint4(pk[8 * hs], pk[8 * hs + 1], pk[8 * hs + 2], pk[8 * hs + 3]);
                    *reinterpret_cast<uint4*>(dst + Kp<DV>::off(ro, c)) =
                        odd ? make_uint4(pk[8 * hs + 4], pk[8 * hs + 5], pk[8 * hs + 6], pk[8 * hs + 7])
                            : make_uint4(x[0], x[1], x[2], x[3]);
                }
            }
            if constexpr (Cfg::STAGED) {
                fence_async_smem();
                warp_arrive(&s.sv.full[(n - n_begin) & 1]);
            }
            return true;
        };
        // O^T of step m (tokens t0 .. t0+15 of value row a) from its Z buffer
        auto store_out = [&](int m) {
            if (!wait_all(&s.o_done[m & 1], (m >> 1) & 1, p.status, p.wait_ns)) return false;
            tc5::fence_after();
            const int cm = n_begin + m;
            const int Lm = min(C, ch.end - (ch.tok0 + cm * C));
            float z[16];
            tc5::ld16(z, trow + ((m & 1) ? Cfg::TZ2 : Cfg::TZ) + t0);
            tc5::wait_ld();
            uint32_t v[8], w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = pack_bf16(z[2 * j], z[2 * j + 1]);
            pair_columns(v, w);  // w[j]: values a & ~1, (a & ~1) + 1 of token t0 + 2j + (lane & 1)
            const int t1 = t0 + (lane & 1);
            __nv_bfloat16* o = p.o + (((size_t)ch.tok0 + cm * C + t1) * p.H + h) * DV + (a & ~1);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (t1 + 2 * j < Lm) *reinterpret_cast<uint32_t*>(o + (size_t)(2 * j) * p.H * DV) = w[j];
            return true;
        };
        int done_steps = 0;
        store_state();
        if (Cfg::SAVE && nsteps > 0) store_s0(n_begin);
        tc5::fence_before();
        warp_arrive(&s.s_ready);

        for (int n = 0; n < nsteps; ++n) {
            const int sn = n % NST;
            const float* G = s.G[sn];
            const int cn = n_begin + n;  // chain step
            const int L = min(C, ch.end - (ch.tok0 + cn * C));
            if (!wait_all(&s.full[sn], (n / NST) & 1, p.status, p.wait_ns)) break;
            // Scalar gate: the epilogue's only reads of the stage are two gate
            // factors; with them in registers it releases the stage at once (the
            // MMA thread releases it after the step's last product), so the next
            // loads need not wait for the output stores.
            float gam = 1.f, sce = 1.f;
            if constexpr (!KDA) {
                gam = __expf(G[C - 1]);
                sce = p.scale * __expf(G[t0 + (lane & 15)]);
                warp_arrive(&s.empty[sn]);
            }
            // ---- U = X (= U~ - S0 W^T); -scale e^{G_i} Y into this step's Z
            // buffer, onto which the MMA thread adds U^T P^T: the output ----------
            if (!wait_all(&s.x_done, n & 1, p.status, p.wait_ns)) break;
            tc5::fence_after();
            {
                float x[16], y[16];
                tc5::ld16(x, trow + Cfg::TXY + t0);
                if (Cfg::FULL) tc5::ld16(y, trow + Cfg::TXY + C + t0);
                tc5::wait_ld();
                uint32_t ru[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) ru[j] = pack_bf16(x[2 * j], x[2 * j + 1]);
                tc5::st8(trow + Cfg::TAU + 8 * cg, ru);
                if constexpr (Cfg::FULL) {
                    uint32_t ry[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float f = KDA ? 1.f : __shfl_sync(0xffffffffu, sce, j);
                        ry[j] = __float_as_uint(-f * y[j]);
                    }
                    tc5::st16(trow + ((n & 1) ? Cfg::TZ2 : Cfg::TZ) + t0, ry);
                }
                tc5::wait_st();
                tc5::fence_before();
                warp_arrive(&s.u_ready);
                if (Cfg::SAVE) {  // U image, Tma128 token rows (64 contiguous bytes per warp store)
                    __nv_bfloat16* dst = p.Uout + ((size_t)ch.img * p.NT + ch.n0 + cn) * C * DV;
                    uint32_t w[8];
                    pair_columns(ru, w);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint32_t*>(dst + Tma128::off(t0 + 2 * j + (lane & 1), a & ~1)) = w[j];
                }
            }
            // ---- the previous step's output, under this step's D product ----------
            if (Cfg::FULL && n > 0 && !store_out(n - 1)) break;
            // ---- S1 = gamma S0 + D, and the bf16 state image -------------------
            if (!wait_all(&s.d_done, n & 1, p.status, p.wait_ns)) break;
            tc5::fence_after();
            {
                float d[32];
                tc5::ld32(d, trow + Cfg::TD + 32 * cg);
                tc5::wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = fmaf(KDA ? G[32 * cg + j] : gam, S[j], d[j]);
            }
            store_state();
            tc5::fence_before();
            warp_arrive(&s.s_ready);
            if (KDA) warp_arrive(&s.empty[sn]);  // the per-key decays were its last stage reads
            if (Cfg::SAVE && n + 1 < nsteps && !store_s0(cn + 1)) break;
            done_steps = n + 1;
        }
        // the last step's output
        if (Cfg::FULL && done_steps == nsteps && nsteps > 0) store_out(nsteps - 1);
        if (jb.out) {
            float* out = jb.out + (size_t)a * DK + 32 * cg;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(out + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc5::fence_before();
    __syncthreads();
    if (warp == W5_CTRL) {
        tc5::fence_after();
        tc5::dealloc(tm, Cfg::TCOLS);
    }
}

// ---------------------------------------------------------------------------
// Scan over the runs of each chain: E_{j+1} = E_j M_j + N_j for j = 1 ..
// nseg-2, in fp32 (E_1 comes from run 0).  One CTA per (16-row block of the
// state, chain).  M_j (64 KB fp32) arrives in shared memory by two bulk copies
// on an mbarrier, the next step's map one step ahead (two buffers).
// ---------------------------------------------------------------------------
constexpr int SC_THREADS = 128, SC_ROWS = 16;
struct ScSmem {
    float M[2][DK * DK];   // double-buffered map
    float Er[SC_ROWS][DK]; // this CTA's rows of the entry state of the current run
    uint64_t bar[2];
};
// Thread t: rows 4 (t / 32) .. +3 and columns 4 (t % 32) .. +3 of the CTA's
// 16 x 128 block, so each map element read from shared memory feeds four rows
// (a warp reads 512 contiguous bytes of a map row; the state rows broadcast).
__global__ void __launch_bounds__(SC_THREADS) tc5_seg_scan_kernel(float* E, const float* Mmap,
                                                                  const float* Nmap, int nseg,
                                                                  unsigned int* status) {
    extern __shared__ __align__(128) unsigned char sc_raw[];
    ScSmem& s = *reinterpret_cast<ScSmem*>(sc_raw);
    const int tid = threadIdx.x;
    const int b = blockIdx.y, r0 = blockIdx.x * SC_ROWS;
    const int rg = 4 * (tid >> 5), c0 = (tid & 31) * 4;
    auto slot = [&](int j) { return ((size_t)b * nseg + j) * DV * DK; };
    auto fetch = [&](int j) {  // map of run j into buffer j & 1
        uint64_t* bar = &s.bar[j & 1];
        mbar_arrive_expect(bar, DK * DK * 4);
        bulk_g2s(s.M[j & 1], Mmap + slot(j), DK * DK * 2, bar);
        bulk_g2s(s.M[j & 1] + DK * DK / 2, Mmap + slot(j) + DK * DK / 2, DK * DK * 2, bar);
    };
    if (tid == 0) {
        mbar_init(&s.bar[0], 1);
        mbar_init(&s.bar[1], 1);
        fence_mbar_init();
        if (nseg > 2) fetch(1);
    }
    // E_1 (from run 0's walk), this CTA's rows
    for (int e = tid; e < SC_ROWS * DK / 4; e += SC_THREADS)
        reinterpret_cast<float4*>(&s.Er[0][0])[e] = reinterpret_cast<const float4*>(E + slot(1) + (size_t)r0 * DK)[e];
    __syncthreads();
    bool ok = true;
    for (int j = 1; j + 1 < nseg; ++j) {
        if (tid == 0 && j + 2 < nseg) fetch(j + 1);  // buffer of step j-1, released at its end
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 nv = reinterpret_cast<const float4*>(Nmap + slot(j) + (size_t)(r0 + rg + i) * DK)[c0 / 4];
            acc[i][0] = nv.x; acc[i][1] = nv.y; acc[i][2] = nv.z; acc[i][3] = nv.w;
        }
        ok = ok && mbar_wait(&s.bar[j & 1], ((j - 1) >> 1) & 1, status);
        if (__syncthreads_or(!ok)) break;
        const float* M = s.M[j & 1];
#pragma unroll 4
        for (int k = 0; k < DK; ++k) {
            const float4 m = *reinterpret_cast<const float4*>(M + k * DK + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float e = s.Er[rg + i][k];
                acc[i][0] = fmaf(e, m.x, acc[i][0]); acc[i][1] = fmaf(e, m.y, acc[i][1]);
                acc[i][2] = fmaf(e, m.z, acc[i][2]); acc[i][3] = fmaf(e, m.w, acc[i][3]);
            }
        }
        __syncthreads();  // every read of this step's entry rows and map done
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 v = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            reinterpret_cast<float4*>(&s.Er[rg + i][0])[c0 / 4] = v;
            reinterpret_cast<float4*>(E + slot(j + 1) + (size_t)(r0 + rg + i) * DK)[c0 / 4] = v;
        }
        __syncthreads();  // the next entry rows in place
    }
}

template <bool KDA, int MODE>
void launch_w5(const W5Ptrs& p, int grid, cudaStream_t st) {
    const int smem = sizeof(W5Smem<MODE>) + 1024;
    cudaFuncSetAttribute(tc5_walk_kernel<KDA, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH(MODE == 0 ? "tc5_walk_fwd" : MODE == 1 ? "tc5_walk_states" : MODE == 2 ? "tc5_seg_map"
                                                                             : "tc5_walk_fwd_save",
               st,
               (tc5_walk_kernel<KDA, MODE><<<grid, W5Cfg<MODE>::THREADS, smem, st>>>(p)));
}

W5Ptrs w5_ptrs(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0) {
    W5Ptrs w{};
    w.qmap = c.qmap;
    w.h0 = h0; w.W = c.W; w.Ut = c.Ut; w.P = c.P; w.G = c.G; w.Qg = c.Qg; w.Kt = c.Kt;
    w.status = c.status;
    w.wait_ns = c.wait_ns; w.stall_at = c.stall_at;
    w.B = chain_batches(d.B, c.seq); w.T = d.T; w.H = d.H; w.NT = L.NT; w.scale = d.scale;
    w.seq = c.seq;
    w.nseg = 1; w.seglen = L.NT;
    return w;
}

// Runs the segment maps and the scan, so that E holds every run's entry state.
template <bool KDA>
void run_segments(W5Ptrs& w, const TcLayout& L, void* ws, cudaStream_t st) {
    w.E = (float*)((char*)ws + L.segE);
    w.Mmap = (float*)((char*)ws + L.segM);
    w.Nmap = (float*)((char*)ws + L.segN);
    launch_w5<KDA, 2>(w, w.B * w.H * (2 * w.nseg - 3), st);
    if (w.nseg > 2) tc::launch_seg_scan(w.E, w.Mmap, w.Nmap, w.nseg, w.B * w.H, w.status, st);
}

}  // namespace

namespace tc {
void launch_seg_scan(float* E, const float* Mmap, const float* Nmap, int nseg, int chains,
                     unsigned int* status, cudaStream_t st) {
    const int smem = sizeof(ScSmem);
    cudaFuncSetAttribute(tc5_seg_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    GDN_LAUNCH("tc5_seg_scan", st,
               (tc5_seg_scan_kernel<<<dim3(DV / SC_ROWS, chains), SC_THREADS, smem, st>>>(
                   E, Mmap, Nmap, nseg, status)));
}

void launch_walk5_fwd(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0,
                      void* o, float* hT, void* ws, cudaStream_t st, bool save) {
    W5Ptrs w = w5_ptrs(d, L, c, h0);
    w.o = (__nv_bfloat16*)o; w.hT = hT;
    if (save) {  // a backward layout: keep the chunk states and U
        w.S0out = (__nv_bfloat16*)((char*)ws + L.S0);
        w.Uout = (__nv_bfloat16*)((char*)ws + L.U);
    }
    const bool kda = d.gate == GDN_GATE_CHANNEL;
    w.nseg = L.nseg;
    w.seglen = L.seglen;
    if (w.nseg > 1) {
        if (kda) run_segments<true>(w, L, ws, st);
        else run_segments<false>(w, L, ws, st);
    }
    if (save) {
        if (kda) launch_w5<true, 3>(w, w.B * w.H * w.nseg, st);
        else launch_w5<false, 3>(w, w.B * w.H * w.nseg, st);
    } else {
        if (kda) launch_w5<true, 0>(w, w.B * w.H * w.nseg, st);
        else launch_w5<false, 0>(w, w.B * w.H * w.nseg, st);
    }
}

void launch_walk5_states(const gdn_dims& d, const TcLayout& L, const ChunkPtrs& c, const float* h0,
                         void* ws, cudaStream_t st) {
    W5Ptrs w = w5_ptrs(d, L, c, h0);
    w.S0out = (__nv_bfloat16*)((char*)ws + L.S0);
    w.Uout = (__nv_bfloat16*)((char*)ws + L.U);
    const bool kda = d.gate == GDN_GATE_CHANNEL;
    w.nseg = L.nseg;
    w.seglen = L.seglen;
    if (w.nseg > 1) {
        if (kda) run_segments<true>(w, L, ws, st);
        else run_segments<false>(w, L, ws, st);
    }
    if (kda) launch_w5<true, 1>(w, w.B * w.H * w.nseg, st);
    else launch_w5<false, 1>(w, w.B * w.H * w.nseg, st);
}
}  // namespace tc
}  // namespace gdn
