// Tensor-core (tcgen05) WBMM forward and input-gradient kernel, window-major.
//
// The windows of a tile (128, or 512 as four M tiles when a window has at most
// 64 padded positions) are the GEMM's M dimension and the output positions of
// a window its N dimension:
//
//   D[n, (p, q)] = sum_{(r, s)} X[n, (r, s)] * M_c[(p, q), (r, s)]
//
// Positions are padded to RP = roundup(w, 8) slots per window row (position
// (p, q) at column p*RP + q, (r, s) at K slot r*RP + s).  One MMA K step of 16
// slots covers G = 16 / RP whole window rows r0 .. r0+G-1.  Because M_c is
// block-Toeplitz (its entry depends only on p - r and q - s), the B operand of
// every K step is a row window of ONE small per-channel matrix
//
//   Q[(delta + w - 1)*RP + q][u*RP + s] = T[delta - u + w - 1][q - s + w - 1]
//
// (delta = p - r0, u < G the row within the step): the step starting at row
// r0 reads Q from row (w - 1 - r0)*RP onwards.  Q is (2w - 1)*RP + NP - RP
// rows of 32 bytes, 13.5 KB at w = 14, so two channels' Q fit in shared
// memory and a channel change never stalls the tensor core.
//
// The windows (the A operand) live in tensor memory: the transform warps
// write them there with tcgen05.st (lane = window, one 32-bit column per pair
// of K slots), so shared memory holds only Q, the raw load ring and two
// output staging buffers, and a tile's input and output never share a buffer.
//
// Warp roles (608 threads):
//   warp 0       producer: bulk/TMA copies of half tiles (whole bands) into a
//                ring of raw slots
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warp 2       storer: stores a finished tile from its output buffer
//   warps 3..10  transform: two per TMEM lane quarter, each taking half of
//                the window rows; thread = window, raw band layout -> A rows
//                in TMEM (two A stages)
//   warps 11..18 epilogue: TMEM -> bf16 output rows -> band layout in an
//                output buffer.  They also write Q: the CTA's first two
//                channels up front, and Q of channel ci+1 right after the
//                first tile of channel ci, whose completion implies that
//                every MMA of channel ci-1 (the other buffer's user) has
//                finished.
//
// TMEM: A stages at columns 0 and 128 (M tile mt of a stage at mt*KP/2), the
// accumulator (single; M tile mt at 256 + mt*DSTEP).
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "wbmm_internal.h"

namespace wbmm {

template <int WS>
struct ToepCfg {
    static constexpr int D = WS * WS;
    static constexpr int RP = (WS + 7) / 8 * 8;            // slots per window row
    static constexpr int G = 16 / RP;                        // window rows per K step
    static constexpr int KSTEPS = (WS + G - 1) / G;
    static constexpr int KP = KSTEPS * 16;                   // K slots
    static constexpr int RROWS = KSTEPS * G;                 // window rows incl. zero rows
    static constexpr int NP = (WS * RP + 15) / 16 * 16;      // MMA N (output columns)
    static constexpr int QROWS = (WS - 1) * RP + NP;
    static constexpr int TSZ = (2 * WS - 1) * (2 * WS - 1);
    // 128-window M tiles per tile: four when a window is small (N <= 64), so
    // that the per-tile fixed costs cover four times the data
    static constexpr int MTW = NP <= 64 ? 4 : 1;
    static constexpr int DSTEP = NP <= 64 ? 64 : 256;        // accumulator columns per M tile
    static constexpr int TW = 128 * MTW;                     // windows per tile
    static constexpr int A_COLS = KP / 2;                    // TMEM columns per M tile of A
    static constexpr uint32_t Q_BYTES = (uint32_t)QROWS * 32;
    static constexpr uint32_t OUT_BYTES = (uint32_t)((TW * D * 2 + 127) / 128 * 128);
    static constexpr int LOADS = (NP + 31) / 32;             // 32-column TMEM loads per row
    static constexpr int RL = 32 / RP;                       // window rows per load
    static constexpr uint32_t IDESC = idesc_bf16(128, NP);
    // With one 128-window M tile (RP = 16), the accumulator is two halves of
    // output rows, [0, P0) and [P0, w), at TMEM columns 256 and 384: the MMAs
    // of one half run while the epilogue drains the other.
    static constexpr bool NSPLIT = MTW == 1;
    static constexpr int P0 = (WS + 1) / 2;
    static constexpr int N0 = NSPLIT ? P0 * RP : NP;
    static constexpr int N1 = NSPLIT ? WS * RP - N0 : 16;
    static constexpr uint32_t IDESC0 = idesc_bf16(128, N0);
    static constexpr uint32_t IDESC1 = idesc_bf16(128, N1);
    static_assert(MTW * A_COLS <= 128, "an A stage fits in 128 TMEM columns");
    static_assert((MTW - 1) * DSTEP + NP <= 256, "the accumulator fits in 256 TMEM columns");
    static_assert((WS - 1) * RP % 8 == 0, "Q row offsets must be whole core matrices");
    static_assert(!NSPLIT || (RP == 16 && N0 <= 128 && N1 <= 128 && N0 % 16 == 0 &&
                              N1 % 16 == 0 && N1 >= 16),
                  "each accumulator half fits in 128 TMEM columns");
};

constexpr int kToepRing = 8;
constexpr int kToepXformWarp0 = 3;
constexpr int kToepXformWarps = 8;
constexpr int kToepEpiWarp0 = kToepXformWarp0 + kToepXformWarps;
constexpr int kToepEpiWarps = 8;
constexpr int kToepThreads = (kToepEpiWarp0 + kToepEpiWarps) * 32;

struct TcToepParams {
    TmapBytes map_x;        // input planes, one box = a half tile (use_tmap)
    TmapBytes map_y;        // output planes, one box = a tile (use_tmap)
    const uint16_t* x;      // bf16 bits, [B][C][H][W]
    const uint16_t* T;      // bf16 table [C][(2w-1)^2]
    uint16_t* y;
    int C, H, W, nh, nw;
    int bpt;                // bands per tile
    int sb;                 // bands per half tile (raw slot)
    int tpc;                // tiles per channel
    int bands;              // bands per channel
    int items;              // C * tpc
    int R;                  // raw ring depth (half tiles)
    int nout;               // output buffers (1 or 2)
    uint32_t sub_bytes;     // raw slot stride
    int use_tmap;
    int kimg_sub;           // planes per half tile when use_tmap
    uint32_t off_out, off_q, off_raw, off_woff, off_bar, off_tst;
    int skip_seq;           // test only: CTA 0 skips this tile's load (-1: none)
    unsigned long long budget;
    int* status;
};

struct ToepBars {
    uint64_t raw_full[kToepRing];
    uint64_t raw_empty[kToepRing];
    uint64_t a_full[2];     // A stage written by the transform
    uint64_t a_empty[2];    // A stage's MMAs have completed
    uint64_t q_full[2];
    uint64_t acc_full[2];   // per accumulator half (one when not split)
    uint64_t acc_empty[2];
    uint64_t out_full[2];   // buffer holds the tile's output
    uint64_t out_empty[2];  // buffer has been read by the storer
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

__device__ __forceinline__ BandTile toep_tile(const TcToepParams& P, int it)
{
    BandTile t;
    t.c = it / P.tpc;
    t.band0 = (it - t.c * P.tpc) * P.bpt;
    const int left = P.bands - t.band0;
    t.nb = left < P.bpt ? left : P.bpt;
    return t;
}

// Half tile h of tile t: bands [band0 + h*sb, ...), possibly none.
__device__ __forceinline__ BandTile toep_half(const TcToepParams& P, const BandTile& t, int h)
{
    BandTile s;
    s.c = t.c;
    s.band0 = t.band0 + h * P.sb;
    const int left = t.nb - h * P.sb;
    s.nb = left <= 0 ? 0 : (left < P.sb ? left : P.sb);
    return s;
}

// Copies one channel's table into shared memory with coalesced loads: as
// stored for the forward, reversed end to end (the transposed matrix) for
// the input gradient.
template <int WS, int MODE>
__device__ __forceinline__ void stage_table(uint16_t* tst, const uint16_t* T, int tid,
                                            int nthreads)
{
    constexpr int TSZ = ToepCfg<WS>::TSZ;
    const unsigned short* src = reinterpret_cast<const unsigned short*>(T);
    for (int e = tid; e < TSZ; e += nthreads)
        tst[MODE == kTable ? e : TSZ - 1 - e] = __ldg(src + e);
}

// Writes Q for one channel from its staged table (layout: K-major, 8-row
// groups of 256 bytes, the two 8-slot core matrices of a row 128 bytes
// apart).  One thread per (row, 8-slot half).
template <int WS>
__device__ __forceinline__ void build_q(uint8_t* q, const uint16_t* tst, int tid, int nthreads)
{
    using F = ToepCfg<WS>;
    constexpr int L = 2 * WS - 1;
    for (int item = tid; item < F::QROWS * 2; item += nthreads) {
        const int rho = item >> 1, half = item & 1;
        const int delta = rho / F::RP - (WS - 1);
        const int ps = rho - (rho / F::RP) * F::RP;
        uint32_t wv[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint16_t v2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kk = half * 8 + 2 * m + e;
                const int u = kk / F::RP, s = kk - (kk / F::RP) * F::RP;
                const int a = delta - u + WS - 1, b = ps - s + WS - 1;
                uint16_t v = 0;
                if (ps < WS && s < WS && a >= 0 && a < L)
                    v = tst[a * L + b];
                v2[e] = v;
            }
            wv[m] = pack_bf16x2(v2[0], v2[1]);
        }
        *reinterpret_cast<uint4*>(q + (rho >> 3) * 256 + half * 128 + (rho & 7) * 16) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

// Rows [R0, R1) of one window -> its TMEM lane of an A stage: window row r
// at columns r*RP/2 .. (r+1)*RP/2 - 1 (slot pairs), rows w .. RROWS-1 zero.
template <int WS, int R0, int R1>
__device__ __forceinline__ void window_to_tmem(const uint16_t* src0, bool valid, int W,
                                               uint32_t acol)
{
    using F = ToepCfg<WS>;
#pragma unroll 2
    for (int r = R0; r < R1; ++r) {
        uint32_t wv[F::RP / 2];
        if (valid && r < WS) {
            const uint16_t* src = src0 + r * W;
            if (WS % 2 == 0) {
#pragma unroll
                for (int m = 0; m < F::RP / 2; ++m)
                    wv[m] = (2 * m < WS) ? reinterpret_cast<const uint32_t*>(src)[m] : 0u;
            } else {
#pragma unroll
                for (int m = 0; m < F::RP / 2; ++m) {
                    const uint16_t lo = (2 * m < WS) ? src[2 * m] : (uint16_t)0;
                    const uint16_t hi = (2 * m + 1 < WS) ? src[2 * m + 1] : (uint16_t)0;
                    wv[m] = pack_bf16x2(lo, hi);
                }
            }
        } else {
#pragma unroll
            for (int m = 0; m < F::RP / 2; ++m)
                wv[m] = 0u;
        }
        if constexpr (F::RP == 16)
            tmem_st8(acol + (uint32_t)(r * 8), wv);
        else
            tmem_st4(acol + (uint32_t)(r * 4), wv);
    }
}

__device__ __forceinline__ uint32_t bf16x2_rn(uint32_t lo, uint32_t hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <int WS, int MODE>
__global__ void __launch_bounds__(kToepThreads, 1)
    wbmm_tc_toep_kernel(const __grid_constant__ TcToepParams P)
{
    using F = ToepCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* out_base = smem + P.off_out;
    uint8_t* q_base = smem + P.off_q;
    uint8_t* raw_base = smem + P.off_raw;
    int* woff = reinterpret_cast<int*>(smem + P.off_woff);
    uint16_t* tst = reinterpret_cast<uint16_t*>(smem + P.off_tst);
    ToepBars& S = *reinterpret_cast<ToepBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R, NO = P.nout;

    // Contiguous, balanced range of items for this CTA.
    const int qn = P.items / (int)gridDim.x, rem = P.items % (int)gridDim.x;
    const int it0 = (int)blockIdx.x * qn + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem);
    const int n_it = qn + ((int)blockIdx.x < rem ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kToepRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], kToepXformWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.a_full[i], kToepXformWarps);
            mbar_init(&S.a_empty[i], 1);
            mbar_init(&S.q_full[i], kToepEpiWarps);
            mbar_init(&S.out_full[i], kToepEpiWarps);
            mbar_init(&S.out_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], kToepEpiWarps);
        }
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    for (int n = threadIdx.x; n < F::TW; n += kToepThreads) {
        const int k = n / P.nw, j = n - k * P.nw;
        woff[n] = k * WS * P.W + j * WS;
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_slot;
    // Everything above overlaps the previous kernel's tail; tensors are read
    // and written only after it has completed.
    grid_dep_wait();
    grid_dep_launch();

    if (warp == 0) {
        // ------------------------------------------------------ producer
        // The first tile's loads go out at once, beside the epilogue warps'
        // loads of the first two tables; the rest of the ring waits until
        // those tables have arrived, so that they are not queued behind every
        // CTA's ring fill (the first MMA needs Q).
        int issued = 0;
        bool go = true;
        for (int seq = 0; seq < n_it && go; ++seq) {
            const BandTile t = toep_tile(P, it0 + seq);
            for (int h = 0; h < 2; ++h) {
                const int ss = 2 * seq + h, s = ss % R;
                bool ok = !*abort;
                if (ss >= R)
                    ok = ok && mbar_wait(&S.raw_empty[s], ((ss / R) - 1) & 1, abort, P.budget,
                                         P.status);
                if (!__all_sync(0xffffffffu, ok)) {
                    go = false;
                    break;
                }
                const BandTile st = toep_half(P, t, h);
                uint8_t* slot = raw_base + (size_t)s * P.sub_bytes;
                if (seq == P.skip_seq && blockIdx.x == 0) {
                    // test only: the slot is never armed, so the transform's
                    // bounded wait for it runs out
                } else if (st.nb == 0) {
                    if (lane == 0)
                        mbar_arrive_expect_tx(&S.raw_full[s], 0);
                } else if (P.use_tmap) {
                    // whole planes; a box past the last image is zero-filled
                    // and still counts its full size
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&S.raw_full[s],
                                              (uint32_t)P.kimg_sub * WS * P.W * P.nh * 2);
                        tma_load_4d(slot, &P.map_x, 0, 0, st.c, st.band0 / P.nh, &S.raw_full[s]);
                    }
                } else {
                    if (lane == 0)
                        mbar_arrive_expect_tx(&S.raw_full[s], (uint32_t)st.nb * WS * P.W * 2);
                    __syncwarp();
                    const BandRuns runs = band_runs(st, P.nh);
                    for (int l = lane; l < runs.count; l += 32) {
                        long long goff;
                        uint32_t soff, nbytes;
                        band_run(st, runs, l, WS, P.W, P.H, P.C, P.nh, goff, soff, nbytes);
                        bulk_g2s(slot + soff, P.x + goff, nbytes, &S.raw_full[s]);
                    }
                }
                issued = ss + 1;
            }
            if (seq == 0)
                named_bar_sync(5, 32 + kToepEpiWarps * 32);
        }
        if (n_it == 0)
            named_bar_sync(5, 32 + kToepEpiWarps * 32);
        // Drain: every issued copy lands before the CTA can exit.
        if (lane == 0) {
            for (int s = 0; s < R && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / R) * R;
                mbar_wait_drain(&S.raw_full[s], (last / R) & 1, P.budget, P.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int cur_c = -1, ci = -1;
            for (int seq = 0; seq < n_it; ++seq) {
                const BandTile t = toep_tile(P, it0 + seq);
                const bool first = t.c != cur_c;
                if (first) {
                    cur_c = t.c;
                    ++ci;
                }
                const int st = seq & 1, qb = ci & 1;
                bool ok = !*abort;
                if (first)
                    ok = ok && mbar_wait(&S.q_full[qb], (ci >> 1) & 1, abort, P.budget, P.status);
                ok = ok && mbar_wait(&S.a_full[st], (seq >> 1) & 1, abort, P.budget, P.status);
                if (!ok)
                    continue;
                // K step k: A columns 8k .. 8k+7 of the M tile, Q rows from
                // (w - 1 - G*k)*RP: only the start-address field moves.
                const uint64_t qdesc0 = smem_desc(
                    smem_u32(q_base + (size_t)qb * F::Q_BYTES) + (uint32_t)((WS - 1) * F::RP * 32),
                    128, 256);
                if constexpr (F::NSPLIT) {
                    const uint32_t a0 = tmem + (uint32_t)(st * 128);
#pragma unroll
                    for (int hN = 0; hN < 2; ++hN) {
                        if (seq >= 1)
                            ok = ok && mbar_wait(&S.acc_empty[hN], (seq - 1) & 1, abort, P.budget,
                                                 P.status);
                        if (!ok)
                            break;
                        tc_fence_after();
                        // half hN: output rows from hN*P0, i.e. Q rows N0*hN on
                        const uint64_t qd = qdesc0 + (uint64_t)(hN * F::N0 * 2);
                        const uint32_t d = tmem + 256u + (uint32_t)(hN * 128);
#pragma unroll
                        for (int k = 0; k < F::KSTEPS; ++k)
                            mma_ts(d, a0 + (uint32_t)(k * 8),
                                   qd - (uint64_t)(k * F::G * F::RP * 2),
                                   hN ? F::IDESC1 : F::IDESC0, k > 0 ? 1u : 0u);
                        tc_commit(&S.acc_full[hN]);
                    }
                    if (ok)
                        tc_commit(&S.a_empty[st]);
                    continue;
                }
                if (seq >= 1)
                    ok = ok && mbar_wait(&S.acc_empty[0], (seq - 1) & 1, abort, P.budget, P.status);
                if (!ok)
                    continue;
                tc_fence_after();
#pragma unroll
                for (int mt = 0; mt < F::MTW; ++mt) {
                    const uint32_t a0 = tmem + (uint32_t)(st * 128 + mt * F::A_COLS);
                    const uint32_t d = tmem + 256u + (uint32_t)(mt * F::DSTEP);
#pragma unroll
                    for (int k = 0; k < F::KSTEPS; ++k)
                        mma_ts(d, a0 + (uint32_t)(k * 8),
                               qdesc0 - (uint64_t)(k * F::G * F::RP * 2), F::IDESC,
                               k > 0 ? 1u : 0u);
                }
                tc_commit(&S.a_empty[st]);
                tc_commit(&S.acc_full[0]);
            }
            // Drain: all issued MMAs complete before TMEM is released.
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ storer
        for (int seq = 0; seq < n_it; ++seq) {
            const int ob = seq % NO;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.out_full[ob], (seq / NO) & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const BandTile t = toep_tile(P, it0 + seq);
                const uint8_t* out = out_base + (size_t)ob * F::OUT_BYTES;
                if (P.use_tmap) {
                    // planes past the last image are clipped
                    if (lane == 0)
                        tma_store_4d(&P.map_y, 0, 0, t.c, t.band0 / P.nh, out);
                } else {
                    const BandRuns runs = band_runs(t, P.nh);
                    for (int l = lane; l < runs.count; l += 32) {
                        long long goff;
                        uint32_t soff, nbytes;
                        band_run(t, runs, l, WS, P.W, P.H, P.C, P.nh, goff, soff, nbytes);
                        bulk_s2g(P.y + goff, out + soff, nbytes);
                    }
                }
                bulk_commit();
                bulk_wait_read<0>();
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.out_empty[ob]);
        }
        bulk_wait<0>();
    } else if (warp < kToepEpiWarp0) {
        // ------------------------------------------------------ transform
        // Thread = window mt*128 + quarter*32 + lane; warp part 0 writes the
        // first half of the window rows, part 1 the rest.  tcgen05.st writes
        // all 32 lanes of the quarter, so a tile is written once both halves
        // of the tile have landed.
        constexpr int RH = (F::RROWS + 1) / 2;
        const int quarter = warp & 3;
        const int part = (warp - kToepXformWarp0) >> 2;
        const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = toep_tile(P, it0 + seq);
            const int st = seq & 1;
            bool ok = !*abort;
            if (seq >= 2)
                ok = ok && mbar_wait(&S.a_empty[st], ((seq >> 1) - 1) & 1, abort, P.budget,
                                     P.status);
            const int ss0 = 2 * seq, s0 = ss0 % R, s1 = (ss0 + 1) % R;
            ok = ok && mbar_wait(&S.raw_full[s0], (ss0 / R) & 1, abort, P.budget, P.status);
            ok = ok && mbar_wait(&S.raw_full[s1], ((ss0 + 1) / R) & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) {
                const int nwin = t.nb * P.nw;
                const int h0win = toep_half(P, t, 0).nb * P.nw;
#pragma unroll 1
                for (int mt = 0; mt < F::MTW; ++mt) {
                    const int n = mt * 128 + quarter * 32 + lane;
                    const bool valid = n < nwin;
                    const int h = n < h0win ? 0 : 1;
                    const uint16_t* raw = reinterpret_cast<const uint16_t*>(
                        raw_base + (size_t)(h ? s1 : s0) * P.sub_bytes);
                    const uint16_t* src0 = raw + (valid ? woff[h ? n - h0win : n] : 0);
                    const uint32_t acol = tmem + lanebase + (uint32_t)(st * 128 + mt * F::A_COLS);
                    if (part == 0)
                        window_to_tmem<WS, 0, RH>(src0, valid, P.W, acol);
                    else
                        window_to_tmem<WS, RH, F::RROWS>(src0, valid, P.W, acol);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0) {
                mbar_arrive(&S.raw_empty[s0]);
                mbar_arrive(&S.raw_empty[s1]);
                mbar_arrive(&S.a_full[st]);
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        // Two warps per TMEM lane quarter (32 windows); each takes every
        // other 32-column load, i.e. RL window rows of every window.
        const int quarter = warp & 3;
        const int hf = (warp - kToepEpiWarp0) >> 2;
        const int et = threadIdx.x - kToepEpiWarp0 * 32;
        const int c_first = toep_tile(P, it0).c;
        const int nch = toep_tile(P, it0 + n_it - 1).c - c_first + 1;
        // The tables of the CTA's first two channels, loaded into registers
        // before the producer may start: the rest of the tables are read
        // while Q of the channel before is in use.
        constexpr int TPT = (F::TSZ + kToepEpiWarps * 32 - 1) / (kToepEpiWarps * 32);
        uint16_t tpre[2][TPT];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int i = 0; i < TPT; ++i) {
                const int e = et + i * kToepEpiWarps * 32;
                tpre[j][i] = (j < nch && e < F::TSZ)
                                 ? __ldg(reinterpret_cast<const unsigned short*>(P.T) +
                                         (long long)(c_first + j) * F::TSZ + e)
                                 : (uint16_t)0;
            }
        named_bar_arrive(5, 32 + kToepEpiWarps * 32);
        // Every epilogue warp takes part in every build, whatever its wait
        // results, so the named barriers always see all 256 threads.
        auto build_for = [&](int ci) {
            named_bar_sync(2, kToepEpiWarps * 32);     // staged table fully read
            if (ci < 2) {
#pragma unroll
                for (int i = 0; i < TPT; ++i) {
                    const int e = et + i * kToepEpiWarps * 32;
                    if (e < F::TSZ)
                        tst[MODE == kTable ? e : F::TSZ - 1 - e] = tpre[ci][i];
                }
            } else {
                stage_table<WS, MODE>(tst, P.T + (long long)(c_first + ci) * F::TSZ, et,
                                      kToepEpiWarps * 32);
            }
            named_bar_sync(2, kToepEpiWarps * 32);
            build_q<WS>(q_base + (size_t)(ci & 1) * F::Q_BYTES, tst, et, kToepEpiWarps * 32);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&S.q_full[ci & 1]);
        };
        build_for(0);
        if (nch > 1)
            build_for(1);
        int cur_c = -1, ci = -1;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = toep_tile(P, it0 + seq);
            const int nwin = t.nb * P.nw;
            const int ob = seq % NO;
            bool ok = !*abort;
            if (seq >= NO)
                ok = ok && mbar_wait(&S.out_empty[ob], ((seq / NO) - 1) & 1, abort, P.budget,
                                     P.status);
            uint16_t* obuf = reinterpret_cast<uint16_t*>(out_base + (size_t)ob * F::OUT_BYTES);
            // Rows [pb, pe) of every window of M tile mt from the accumulator
            // columns at lbase (row pb at column 0), warp half hf taking every
            // other 32-column load; returns after the last TMEM read.
            auto drain = [&](int mt, uint32_t lbase, int pb, int pe) {
                const int n = mt * 128 + quarter * 32 + lane;
                if (!ok || mt * 128 + quarter * 32 >= nwin)
                    return;
                const bool valid = n < nwin;
                uint16_t* o0 = obuf + (valid ? woff[n] : 0);
                const uint32_t lrow = tmem + ((uint32_t)(quarter * 32) << 16) + lbase;
                const int nload = ((pe - pb) * F::RP + 31) / 32;
#pragma unroll 1
                for (int li = hf; li < nload; li += 2) {
                    uint32_t r[32];
                    tmem_ld32(lrow + (uint32_t)(li * 32), r);
                    tmem_wait_ld(r);
                    if (!valid)
                        continue;
#pragma unroll
                    for (int rr = 0; rr < F::RL; ++rr) {
                        const int pr = pb + li * F::RL + rr;
                        if (pr >= pe)
                            continue;
                        uint16_t* o = o0 + pr * P.W;
                        if (WS % 2 == 0) {
#pragma unroll
                            for (int m = 0; m < WS / 2; ++m)
                                reinterpret_cast<uint32_t*>(o)[m] =
                                    bf16x2_rn(r[rr * F::RP + 2 * m], r[rr * F::RP + 2 * m + 1]);
                        } else {
#pragma unroll
                            for (int s = 0; s < WS; ++s)
                                o[s] = __bfloat16_as_ushort(
                                    __float2bfloat16_rn(__uint_as_float(r[rr * F::RP + s])));
                        }
                    }
                }
            };
            if constexpr (F::NSPLIT) {
#pragma unroll 1
                for (int hN = 0; hN < 2; ++hN) {
                    ok = ok && mbar_wait(&S.acc_full[hN], seq & 1, abort, P.budget, P.status);
                    ok = __all_sync(0xffffffffu, ok);
                    tc_fence_after();
                    drain(0, 256u + (uint32_t)(hN * 128), hN ? F::P0 : 0, hN ? WS : F::P0);
                    tc_fence_before();
                    __syncwarp();
                    if (ok && lane == 0)
                        mbar_arrive(&S.acc_empty[hN]);
                }
            } else {
                ok = ok && mbar_wait(&S.acc_full[0], seq & 1, abort, P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();
#pragma unroll 1
                for (int mt = 0; mt < F::MTW; ++mt)
                    drain(mt, 256u + (uint32_t)(mt * F::DSTEP), 0, WS);
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) {
                if constexpr (!F::NSPLIT)
                    mbar_arrive(&S.acc_empty[0]);
                mbar_arrive(&S.out_full[ob]);
            }
            if (t.c != cur_c) {
                cur_c = t.c;
                ++ci;
                if (ci >= 1 && ci + 1 < nch)
                    build_for(ci + 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ host
namespace {

constexpr uint32_t kSmemMax = 232448;
constexpr uint32_t kMinSmem = 120 * 1024;

inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

struct ToepLayout {
    uint32_t off_out, off_q, off_raw, off_woff, off_bar, off_tst, total, sub_bytes;
    int R, bpt, sb, nout;
};

// Q (two channels) | output buffers | window offsets | staged table |
// barriers | raw ring.  Two output buffers when the ring still gets at least
// four half tiles, else one.
template <int WS>
bool toep_layout_n(const Geom& g, int nout, ToepLayout& L)
{
    using F = ToepCfg<WS>;
    if (g.nw < 1 || g.nw > F::TW)
        return false;
    L.nout = nout;
    L.bpt = F::TW / g.nw;
    L.sb = (L.bpt + 1) / 2;
    L.sub_bytes = align_up((uint32_t)L.sb * WS * g.W * 2, 128);
    uint32_t off = 0;
    L.off_q = off;
    off += 2 * F::Q_BYTES;
    L.off_out = align_up(off, 128);
    off = L.off_out + (uint32_t)nout * F::OUT_BYTES;
    L.off_woff = align_up(off, 16);
    off = L.off_woff + F::TW * 4;
    L.off_tst = align_up(off, 16);
    off = L.off_tst + (uint32_t)F::TSZ * 2;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(ToepBars);
    L.off_raw = align_up(off, 128);
    const uint32_t avail = kSmemMax - 1024 > L.off_raw ? kSmemMax - 1024 - L.off_raw : 0;
    int R = (int)(avail / L.sub_bytes);
    if (R > kToepRing)
        R = kToepRing;
    const int cap = debug_ring_cap();
    if (cap >= 2 && R > cap)
        R = cap;
    L.R = R;
    if (R < 2)
        return false;
    off = L.off_raw + (uint32_t)R * L.sub_bytes;
    L.total = align_up(off, 1024);
    // at least half the SM's shared memory: one CTA (and one 512-column TMEM
    // allocation) per SM
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L.total <= kSmemMax;
}

template <int WS>
bool toep_layout(const Geom& g, ToepLayout& L)
{
    if (toep_layout_n<WS>(g, 2, L) && L.R >= 4)
        return true;
    return toep_layout_n<WS>(g, 1, L);
}

template <int WS, int MODE>
cudaError_t toep_launch_ws(const Geom& g, const void* x, const void* T, void* y, const Launch& L)
{
    ToepLayout lay;
    if (!toep_layout<WS>(g, lay))
        return cudaErrorInvalidConfiguration;
    static int configured_smem[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_smem[dev & 63] < (int)lay.total) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_toep_kernel<WS, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMax);
        if (e != cudaSuccess)
            return e;
        configured_smem[dev & 63] = (int)kSmemMax;
    }
    TcToepParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.T = static_cast<const uint16_t*>(T);
    P.y = static_cast<uint16_t*>(y);
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = lay.bpt;
    P.sb = lay.sb;
    P.bands = (int)g.bands;
    P.tpc = (P.bands + P.bpt - 1) / P.bpt;
    P.items = g.C * P.tpc;
    P.R = lay.R;
    P.sub_bytes = lay.sub_bytes;
    P.use_tmap = 0;
    P.kimg_sub = 0;
    if (P.bpt % g.nh == 0 && P.sb % g.nh == 0) {
        const int ks = P.sb / g.nh, kt = P.bpt / g.nh;
        if (encode_plane_map(&P.map_x, x, g, ks) && encode_plane_map(&P.map_y, y, g, kt)) {
            P.use_tmap = 1;
            P.kimg_sub = ks;
        }
    }
    P.nout = lay.nout;
    P.off_out = lay.off_out; P.off_q = lay.off_q; P.off_raw = lay.off_raw;
    P.off_woff = lay.off_woff; P.off_bar = lay.off_bar; P.off_tst = lay.off_tst;
    P.budget = L.budget;
    P.status = L.status;
    P.skip_seq = debug_take_skip(0);
    int grid = L.num_sms;
    if (grid > P.items)
        grid = P.items;
    if (grid < 1)
        return cudaSuccess;
    cudaError_t e = launch_pdl(wbmm_tc_toep_kernel<WS, MODE>, dim3(grid), dim3(kToepThreads),
                               lay.total, L.stream, P);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

template <int WS>
cudaError_t toep_launch_mode(const Geom& g, AMode mode, const void* x, const void* T, void* y,
                             const Launch& L)
{
    if (mode == kTable)
        return toep_launch_ws<WS, kTable>(g, x, T, y, L);
    return toep_launch_ws<WS, kTableFlip>(g, x, T, y, L);
}

template <int WS>
bool toep_fits(const Geom& g)
{
    ToepLayout lay;
    return toep_layout<WS>(g, lay);
}

}  // namespace

bool tc_toep_supported(const Geom& g)
{
    if (g.w < 2 || g.w > 16)
        return false;
    // bulk copies move whole bands: 16-byte multiples
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    if (g.bands * (long long)g.C >= (1ll << 31))
        return false;
    switch (g.w) {
    case 2: return toep_fits<2>(g);
    case 3: return toep_fits<3>(g);
    case 4: return toep_fits<4>(g);
    case 5: return toep_fits<5>(g);
    case 6: return toep_fits<6>(g);
    case 7: return toep_fits<7>(g);
    case 8: return toep_fits<8>(g);
    case 9: return toep_fits<9>(g);
    case 10: return toep_fits<10>(g);
    case 11: return toep_fits<11>(g);
    case 12: return toep_fits<12>(g);
    case 13: return toep_fits<13>(g);
    case 14: return toep_fits<14>(g);
    case 15: return toep_fits<15>(g);
    default: return toep_fits<16>(g);
    }
}

cudaError_t tc_toep_launch(const Geom& g, AMode mode, const void* x, const void* T, void* y,
                           const Launch& L)
{
    if (mode == kCached)
        return cudaErrorInvalidValue;
    switch (g.w) {
    case 2: return toep_launch_mode<2>(g, mode, x, T, y, L);
    case 3: return toep_launch_mode<3>(g, mode, x, T, y, L);
    case 4: return toep_launch_mode<4>(g, mode, x, T, y, L);
    case 5: return toep_launch_mode<5>(g, mode, x, T, y, L);
    case 6: return toep_launch_mode<6>(g, mode, x, T, y, L);
    case 7: return toep_launch_mode<7>(g, mode, x, T, y, L);
    case 8: return toep_launch_mode<8>(g, mode, x, T, y, L);
    case 9: return toep_launch_mode<9>(g, mode, x, T, y, L);
    case 10: return toep_launch_mode<10>(g, mode, x, T, y, L);
    case 11: return toep_launch_mode<11>(g, mode, x, T, y, L);
    case 12: return toep_launch_mode<12>(g, mode, x, T, y, L);
    case 13: return toep_launch_mode<13>(g, mode, x, T, y, L);
    case 14: return toep_launch_mode<14>(g, mode, x, T, y, L);
    case 15: return toep_launch_mode<15>(g, mode, x, T, y, L);
    case 16: return toep_launch_mode<16>(g, mode, x, T, y, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
