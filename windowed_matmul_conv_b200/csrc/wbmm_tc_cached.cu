// Tensor-core (tcgen05) WBMM forward with a cached per-channel matrix,
// window-major.
//
// The windows of a tile (128) are the GEMM's M dimension and the output
// positions its N dimension:
//
//   D[n, (p, q)] = sum_{(r, s)} X[n, (r, s)] * M_c[(p, q), (r, s)]
//
// with positions padded to RP = roundup(w, 8) slots per window row, as in the
// table kernel.  A cached matrix has no Toeplitz structure, so the whole M_c^T
// (NP x KP bf16, 98 KB at w = 14) is the B operand, resident in shared memory
// for the channel; the windows are the A operand in tensor memory (lane n =
// window n, one 32-bit column per pair of K slots), written by the transform
// warps with tcgen05.st, which leaves shared memory for the load ring and an
// output staging buffer.
//
// Warp roles (608 threads):
//   warp 0       producer: bulk/TMA copies of half tiles into a ring of raw slots
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warp 2       storer: stores a tile from the output staging buffer
//   warps 3..10  transform: two per TMEM lane quarter, each half of the window
//                rows; thread = window, raw band layout -> A rows in TMEM (two
//                A stages)
//   warps 11..18 epilogue: TMEM -> bf16 output rows -> band layout in the
//                staging buffer; they also build B (M_c^T in the operand
//                layout) from HBM for the first channel and after the last
//                tile of each channel, whose completion implies that every
//                MMA reading the previous B has finished
//
// TMEM: A stages at columns 0 and 128; the accumulator at 256, in two halves
// of output positions (256 and 384) when there are more than 128 of them.
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include <type_traits>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "wbmm_internal.h"

namespace wbmm {

template <int WS>
struct CachedCfg {
    static constexpr int D = WS * WS;
    static constexpr int RP = (WS + 7) / 8 * 8;
    static constexpr int G = 16 / RP;                        // window rows per K step
    static constexpr int KSTEPS = (WS + G - 1) / G;
    static constexpr int KP = KSTEPS * 16;
    static constexpr int RROWS = KSTEPS * G;                 // window rows incl. zero rows
    static constexpr int KC = KP / 8;                        // core matrices along K
    static constexpr int NP = (D + 15) / 16 * 16;            // MMA N: output positions, dense
    static constexpr uint32_t LBO_B = 144;                   // core matrix stride along K
    static constexpr uint32_t SBO_B = (uint32_t)KC * LBO_B;  // bytes per 8-row group of B
    static constexpr uint32_t B_BYTES = (uint32_t)NP / 8 * SBO_B;
    static constexpr int A_COLS = KP / 2;                    // TMEM columns per A stage
    static constexpr int LOADS = (NP + 31) / 32;
    static constexpr uint32_t OUT_BYTES = (uint32_t)((128 * D * 2 + 127) / 128 * 128);
    static constexpr uint32_t IDESC = idesc_bf16(128, NP);
    static_assert(A_COLS <= 128 && NP <= 256, "TMEM plan: A stages at 0/128, D at 256");
    // With more than 128 output positions the accumulator is two halves of
    // positions, [0, N0) at TMEM column 256 and [N0, NP) at 384: the MMAs of
    // one half run while the epilogue drains the other.
    static constexpr bool NSPLIT = NP > 128;
    static constexpr int N0 = NSPLIT ? (NP / 2 + 15) / 16 * 16 : NP;
    static constexpr int N1 = NSPLIT ? NP - N0 : 16;
    static constexpr uint32_t IDESC0 = idesc_bf16(128, N0);
    static constexpr uint32_t IDESC1 = idesc_bf16(128, N1);
    static_assert(!NSPLIT || (N0 <= 128 && N1 <= 128 && N1 >= 16 && N0 % 16 == 0),
                  "each accumulator half fits in 128 TMEM columns");
};

constexpr int kCRing = 8;
constexpr int kCXformWarp0 = 3;
constexpr int kCXformWarps = 8;
constexpr int kCEpiWarp0 = kCXformWarp0 + kCXformWarps;
constexpr int kCEpiWarps = 8;
constexpr int kCThreads = (kCEpiWarp0 + kCEpiWarps) * 32;
constexpr int kCTileWindows = 128;

struct TcCachedParams {
    TmapBytes map_x;        // input planes, one box = a half tile (use_tmap)
    TmapBytes map_y;        // output planes, one box = a tile (use_tmap)
    const uint16_t* x;
    const uint16_t* M;      // [C][d][d] bf16, row u = p*w+q
    uint16_t* y;
    int C, H, W, nh, nw;
    int bpt, sb, tpc, bands, items, R;
    uint32_t sub_bytes;
    int use_tmap, kimg_sub;
    uint32_t off_b, off_out, off_raw, off_woff, off_bar;
    unsigned long long budget;
    int* status;
};

struct CachedBars {
    uint64_t raw_full[kCRing];
    uint64_t raw_empty[kCRing];
    uint64_t a_full[2];
    uint64_t a_empty[2];
    uint64_t b_full;
    uint64_t acc_full[2];   // per accumulator half (one when not split)
    uint64_t acc_empty[2];
    uint64_t out_full;
    uint64_t out_empty;
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

__device__ __forceinline__ BandTile cached_tile(const TcCachedParams& P, int it)
{
    BandTile t;
    t.c = it / P.tpc;
    t.band0 = (it - t.c * P.tpc) * P.bpt;
    const int left = P.bands - t.band0;
    t.nb = left < P.bpt ? left : P.bpt;
    return t;
}

__device__ __forceinline__ BandTile cached_half(const TcCachedParams& P, const BandTile& t, int h)
{
    BandTile s;
    s.c = t.c;
    s.band0 = t.band0 + h * P.sb;
    const int left = t.nb - h * P.sb;
    s.nb = left <= 0 ? 0 : (left < P.sb ? left : P.sb);
    return s;
}

// B = M_c^T in the K-major operand layout: row n = p*w + q (output position
// p, q; row n of M_c), K slot k = r*RP + s (input position r, s), the same K
// order as the table path, so both give identical bits.  Core matrices
// (8 rows x 16 bytes) lie LBO_B = 144 bytes apart along K and SBO_B apart
// along N: the 16 spare bytes put consecutive core matrices of one row on
// different bank groups, so copying rows of M_c in order writes shared
// memory almost without conflicts.  The whole image is zeroed once per
// launch (zero_b, then a barrier among the builders); a build rewrites only
// the d x d values.
template <int WS>
__device__ __forceinline__ void zero_b(uint8_t* b, int tid, int nthreads)
{
    using F = CachedCfg<WS>;
    for (int i = tid; i < (int)(F::B_BYTES / 16); i += nthreads)
        reinterpret_cast<uint4*>(b)[i] = make_uint4(0u, 0u, 0u, 0u);
}

// M_c is read in its own order, so a warp's loads are coalesced.  For even
// w a window row holds whole 32-bit pairs: one asynchronous 4-byte copy per
// pair, all of a thread's copies in flight at once.  For odd w pairs
// straddle window rows: 16-bit loads, eight per thread per pass, all loads
// of a pass issued before its stores.
template <int WS>
__device__ __forceinline__ void build_b_global(uint8_t* b, const uint16_t* Mc, int tid,
                                               int nthreads)
{
    using F = CachedCfg<WS>;
    if constexpr (WS % 2 == 0) {
        // Thread = one 32-bit pair column e of M_c and every RSTEP-th row u
        // from its phase: the destination column and the row step are fixed,
        // so each copy costs a few additions.
        constexpr int HALF = F::D / 2;   // 32-bit pairs per row of M_c
        const int rstep = nthreads / HALF;
        if (tid < rstep * HALF) {
            const int ep = tid % HALF, u0 = tid / HALF;
            const int e = 2 * ep;
            const int k = (e / WS) * F::RP + e % WS;
            const uint32_t col = smem_u32(b) + (uint32_t)(k >> 3) * F::LBO_B + (uint32_t)(k & 7) * 2;
            const uint16_t* src = Mc + (long long)u0 * F::D + e;
            for (int u = u0; u < F::D; u += rstep) {
                cp_async_4(col + (uint32_t)(u >> 3) * F::SBO_B + (uint32_t)(u & 7) * 16, src);
                src += rstep * F::D;
            }
        }
        cp_async_wait_all();
    } else {
        constexpr int BATCH = 8;
        constexpr int N = F::D * F::D;
        for (int base = tid; base < N; base += BATCH * nthreads) {
            uint16_t v[BATCH];
#pragma unroll
            for (int j = 0; j < BATCH; ++j) {
                const int e = base + j * nthreads;
                v[j] = e < N ? __ldg(reinterpret_cast<const unsigned short*>(Mc) + e)
                             : (uint16_t)0;
            }
#pragma unroll
            for (int j = 0; j < BATCH; ++j) {
                const int e = base + j * nthreads;
                if (e >= N)
                    continue;
                const int u = e / F::D, i = e - (e / F::D) * F::D;
                const int k = (i / WS) * F::RP + i % WS;
                *reinterpret_cast<uint16_t*>(b + (u >> 3) * F::SBO_B + (k >> 3) * F::LBO_B +
                                             (u & 7) * 16 + (k & 7) * 2) = v[j];
            }
        }
    }
}

__device__ __forceinline__ uint32_t cbf16x2_rn(uint32_t lo, uint32_t hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <int WS>
__global__ void __launch_bounds__(kCThreads, 1)
    wbmm_tc_cached_kernel(const __grid_constant__ TcCachedParams P)
{
    using F = CachedCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* b_base = smem + P.off_b;
    uint8_t* out_base = smem + P.off_out;
    uint8_t* raw_base = smem + P.off_raw;
    int* woff = reinterpret_cast<int*>(smem + P.off_woff);
    CachedBars& S = *reinterpret_cast<CachedBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R;

    const int qn = P.items / (int)gridDim.x, rem = P.items % (int)gridDim.x;
    const int it0 = (int)blockIdx.x * qn + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem);
    const int n_it = qn + ((int)blockIdx.x < rem ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kCRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], kCXformWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.a_full[i], kCXformWarps);
            mbar_init(&S.a_empty[i], 1);
        }
        mbar_init(&S.b_full, kCEpiWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], kCEpiWarps);
        }
        mbar_init(&S.out_full, kCEpiWarps);
        mbar_init(&S.out_empty, 1);
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    for (int n = threadIdx.x; n < kCTileWindows; n += kCThreads) {
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
        int issued = 0;
        bool go = true;
        for (int seq = 0; seq < n_it && go; ++seq) {
            const BandTile t = cached_tile(P, it0 + seq);
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
                const BandTile st = cached_half(P, t, h);
                uint8_t* slot = raw_base + (size_t)s * P.sub_bytes;
                if (st.nb == 0) {
                    if (lane == 0)
                        mbar_arrive_expect_tx(&S.raw_full[s], 0);
                } else if (P.use_tmap) {
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
        }
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
                const BandTile t = cached_tile(P, it0 + seq);
                const bool first = t.c != cur_c;
                if (first) {
                    cur_c = t.c;
                    ++ci;
                }
                const int st = seq & 1;
                bool ok = !*abort;
                if (first)
                    ok = ok && mbar_wait(&S.b_full, ci & 1, abort, P.budget, P.status);
                ok = ok && mbar_wait(&S.a_full[st], (seq >> 1) & 1, abort, P.budget, P.status);
                if (!ok)
                    continue;
                // K step k: A columns 8k .. 8k+7 of stage st, B core matrices 2k, 2k+1
                const uint64_t bdesc0 = smem_desc(smem_u32(b_base), F::LBO_B, F::SBO_B);
                const uint32_t a0 = tmem + (uint32_t)(st * 128);
                if constexpr (F::NSPLIT) {
#pragma unroll
                    for (int hN = 0; hN < 2; ++hN) {
                        if (seq >= 1)
                            ok = ok && mbar_wait(&S.acc_empty[hN], (seq - 1) & 1, abort, P.budget,
                                                 P.status);
                        if (!ok)
                            break;
                        tc_fence_after();
                        // half hN: B rows (output positions) from hN*N0, 8-row groups SBO_B apart
                        const uint64_t bd = bdesc0 + (uint64_t)(hN * (F::N0 / 8) * F::SBO_B / 16);
#pragma unroll
                        for (int k = 0; k < F::KSTEPS; ++k)
                            mma_ts(tmem + 256u + (uint32_t)(hN * 128), a0 + (uint32_t)(k * 8),
                                   bd + (uint64_t)(k * 2 * F::LBO_B / 16),
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
                for (int k = 0; k < F::KSTEPS; ++k)
                    mma_ts(tmem + 256u, a0 + (uint32_t)(k * 8),
                           bdesc0 + (uint64_t)(k * 2 * F::LBO_B / 16),
                           F::IDESC, k > 0 ? 1u : 0u);
                tc_commit(&S.a_empty[st]);
                tc_commit(&S.acc_full[0]);
            }
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ storer
        for (int seq = 0; seq < n_it; ++seq) {
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.out_full, seq & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const BandTile t = cached_tile(P, it0 + seq);
                if (P.use_tmap) {
                    if (lane == 0)
                        tma_store_4d(&P.map_y, 0, 0, t.c, t.band0 / P.nh, out_base);
                } else {
                    const BandRuns runs = band_runs(t, P.nh);
                    for (int l = lane; l < runs.count; l += 32) {
                        long long goff;
                        uint32_t soff, nbytes;
                        band_run(t, runs, l, WS, P.W, P.H, P.C, P.nh, goff, soff, nbytes);
                        bulk_s2g(P.y + goff, out_base + soff, nbytes);
                    }
                }
                bulk_commit();
                bulk_wait_read<0>();
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.out_empty);
        }
        bulk_wait<0>();
    } else if (warp < kCEpiWarp0) {
        // ------------------------------------------------------ transform
        // Thread = window n of the warp's lane quarter; warp part 0 writes
        // the first half of the window rows, part 1 the rest.  tcgen05.st
        // writes all 32 lanes, so a tile is written once both halves of the
        // tile have landed.
        constexpr int RH = (F::RROWS + 1) / 2;
        const int quarter = warp & 3;
        const int part = (warp - kCXformWarp0) >> 2;
        const int r_lo = part ? RH : 0, r_hi = part ? F::RROWS : RH;
        const int n = quarter * 32 + lane;
        const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = cached_tile(P, it0 + seq);
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
                const int h0win = cached_half(P, t, 0).nb * P.nw;
                const bool valid = n < nwin;
                const int h = n < h0win ? 0 : 1;
                const uint16_t* raw = reinterpret_cast<const uint16_t*>(
                    raw_base + (size_t)(h ? s1 : s0) * P.sub_bytes);
                const uint16_t* src0 = raw + (valid ? woff[h ? n - h0win : n] : 0);
                const uint32_t acol = tmem + lanebase + (uint32_t)(st * 128);
#pragma unroll 2
                for (int r = r_lo; r < r_hi; ++r) {
                    uint32_t wv[F::RP / 2];
                    if (valid && r < WS) {
                        const uint16_t* src = src0 + r * P.W;
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
        const int quarter = warp & 3;
        const int hf = (warp - kCEpiWarp0) >> 2;
        const int et = threadIdx.x - kCEpiWarp0 * 32;
        const int n = quarter * 32 + lane;
        const int c_first = cached_tile(P, it0).c;
        // B of channel c, read straight from HBM/L2.  All epilogue warps take
        // part in every build whatever their wait results.
        auto build_for = [&](int c) {
            build_b_global<WS>(b_base, P.M + (long long)c * F::D * F::D, et, kCEpiWarps * 32);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&S.b_full);
        };
        zero_b<WS>(b_base, et, kCEpiWarps * 32);
        named_bar_sync(1, kCEpiWarps * 32);
        build_for(c_first);
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = cached_tile(P, it0 + seq);
            const int nwin = t.nb * P.nw;
            bool ok = !*abort;
            if (seq >= 1)
                ok = ok && mbar_wait(&S.out_empty, (seq - 1) & 1, abort, P.budget, P.status);
            const bool valid = n < nwin;
            uint16_t* o0 = reinterpret_cast<uint16_t*>(out_base) + (valid ? woff[n] : 0);
            // output positions [E0, E1) from the accumulator columns at lbase
            // (position E0 at column 0); warp half hf takes every other
            // 32-column load.  Positions are compile-time constants, so the
            // (row, column) of each is too.
            auto drain = [&](uint32_t lbase, auto e0c, auto e1c) {
                constexpr int E0 = decltype(e0c)::value, E1 = decltype(e1c)::value;
                if (!ok || quarter * 32 >= nwin)
                    return;
                const uint32_t lrow = tmem + ((uint32_t)(quarter * 32) << 16) + lbase;
                constexpr int NLOAD = (E1 - E0 + 31) / 32;
#pragma unroll
                for (int li = 0; li < NLOAD; ++li) {
                    if ((li & 1) != hf)
                        continue;
                    uint32_t r[32];
                    tmem_ld32(lrow + (uint32_t)(li * 32), r);
                    tmem_wait_ld(r);
                    if (!valid)
                        continue;
                    // accumulator column c is output position e0 + c = (e / w, e % w)
                    if (WS % 2 == 0) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const int e = E0 + li * 32 + j;
                            if (e < E1 && e < F::D)
                                *reinterpret_cast<uint32_t*>(o0 + (e / WS) * P.W + e % WS) =
                                    cbf16x2_rn(r[j], r[j + 1]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int e = E0 + li * 32 + j;
                            if (e < E1 && e < F::D)
                                o0[(e / WS) * P.W + e % WS] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
                        }
                    }
                }
            };
            if constexpr (F::NSPLIT) {
#pragma unroll
                for (int hN = 0; hN < 2; ++hN) {
                    ok = ok && mbar_wait(&S.acc_full[hN], seq & 1, abort, P.budget, P.status);
                    ok = __all_sync(0xffffffffu, ok);
                    tc_fence_after();
                    if (hN == 0)
                        drain(256u, std::integral_constant<int, 0>{},
                              std::integral_constant<int, F::N0>{});
                    else
                        drain(384u, std::integral_constant<int, F::N0>{},
                              std::integral_constant<int, F::NP>{});
                    tc_fence_before();
                    __syncwarp();
                    if (ok && lane == 0)
                        mbar_arrive(&S.acc_empty[hN]);
                }
            } else {
                ok = ok && mbar_wait(&S.acc_full[0], seq & 1, abort, P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();
                drain(256u, std::integral_constant<int, 0>{}, std::integral_constant<int, F::NP>{});
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) {
                if constexpr (!F::NSPLIT)
                    mbar_arrive(&S.acc_empty[0]);
                mbar_arrive(&S.out_full);
            }
            // the channel's last tile is done: every MMA that read B has
            // completed (acc_full), so B can take the next channel's matrix
            if (seq + 1 < n_it && cached_tile(P, it0 + seq + 1).c != t.c)
                build_for(t.c + 1);
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

struct CachedLayout {
    uint32_t off_b, off_out, off_raw, off_woff, off_bar, total, sub_bytes;
    int R, bpt, sb;
};

template <int WS>
bool cached_layout(const Geom& g, CachedLayout& L)
{
    using F = CachedCfg<WS>;
    if (g.nw < 1 || g.nw > kCTileWindows)
        return false;
    L.bpt = kCTileWindows / g.nw;
    L.sb = (L.bpt + 1) / 2;
    L.sub_bytes = align_up((uint32_t)L.sb * WS * g.W * 2, 128);
    uint32_t off = 0;
    L.off_b = off;                                   // 1024-aligned
    off += F::B_BYTES;
    L.off_out = align_up(off, 128);
    off = L.off_out + F::OUT_BYTES;
    L.off_woff = align_up(off, 16);
    off = L.off_woff + kCTileWindows * 4;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(CachedBars);
    L.off_raw = align_up(off, 128);
    const uint32_t avail = kSmemMax - 1024 > L.off_raw ? kSmemMax - 1024 - L.off_raw : 0;
    int R = (int)(avail / L.sub_bytes);
    if (R > kCRing)
        R = kCRing;
    L.R = R;
    if (R < 2)
        return false;
    L.total = align_up(L.off_raw + (uint32_t)R * L.sub_bytes, 1024);
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L.total <= kSmemMax;
}

template <int WS>
cudaError_t cached_launch_ws(const Geom& g, const void* x, const void* M, void* y, const Launch& L)
{
    CachedLayout lay;
    if (!cached_layout<WS>(g, lay))
        return cudaErrorInvalidConfiguration;
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_cached_kernel<WS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMax);
        if (e != cudaSuccess)
            return e;
        configured[dev & 63] = 1;
    }
    TcCachedParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.M = static_cast<const uint16_t*>(M);
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
    P.off_b = lay.off_b; P.off_out = lay.off_out; P.off_raw = lay.off_raw;
    P.off_woff = lay.off_woff; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    int grid = L.num_sms;
    if (grid > P.items)
        grid = P.items;
    if (grid < 1)
        return cudaSuccess;
    cudaError_t e = launch_pdl(wbmm_tc_cached_kernel<WS>, dim3(grid), dim3(kCThreads), lay.total,
                               L.stream, P);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

template <int WS>
bool cached_fits(const Geom& g)
{
    CachedLayout lay;
    return cached_layout<WS>(g, lay);
}

}  // namespace

bool tc_cached_supported(const Geom& g)
{
    if (g.w < 2 || g.w > 15)
        return false;
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    if (g.bands * (long long)g.C >= (1ll << 31))
        return false;
    switch (g.w) {
    case 2: return cached_fits<2>(g);
    case 3: return cached_fits<3>(g);
    case 4: return cached_fits<4>(g);
    case 5: return cached_fits<5>(g);
    case 6: return cached_fits<6>(g);
    case 7: return cached_fits<7>(g);
    case 8: return cached_fits<8>(g);
    case 9: return cached_fits<9>(g);
    case 10: return cached_fits<10>(g);
    case 11: return cached_fits<11>(g);
    case 12: return cached_fits<12>(g);
    case 13: return cached_fits<13>(g);
    case 14: return cached_fits<14>(g);
    default: return cached_fits<15>(g);
    }
}

cudaError_t tc_cached_launch(const Geom& g, const void* x, const void* M, void* y, const Launch& L)
{
    switch (g.w) {
    case 2: return cached_launch_ws<2>(g, x, M, y, L);
    case 3: return cached_launch_ws<3>(g, x, M, y, L);
    case 4: return cached_launch_ws<4>(g, x, M, y, L);
    case 5: return cached_launch_ws<5>(g, x, M, y, L);
    case 6: return cached_launch_ws<6>(g, x, M, y, L);
    case 7: return cached_launch_ws<7>(g, x, M, y, L);
    case 8: return cached_launch_ws<8>(g, x, M, y, L);
    case 9: return cached_launch_ws<9>(g, x, M, y, L);
    case 10: return cached_launch_ws<10>(g, x, M, y, L);
    case 11: return cached_launch_ws<11>(g, x, M, y, L);
    case 12: return cached_launch_ws<12>(g, x, M, y, L);
    case 13: return cached_launch_ws<13>(g, x, M, y, L);
    case 14: return cached_launch_ws<14>(g, x, M, y, L);
    case 15: return cached_launch_ws<15>(g, x, M, y, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
