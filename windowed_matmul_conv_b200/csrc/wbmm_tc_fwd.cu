// Tensor-core (tcgen05) WBMM forward, input-gradient and cached-matrix kernel.
//
// One persistent CTA per SM walks a contiguous range of work items; an item is
// (channel c, tile of whole bands).  For every channel the CTA writes the
// d x d matrix M_c (or its transpose, for the input gradient) into tensor
// memory once; it is the A operand of every MMA of that channel and is never
// written to HBM.  Windows stream through as the GEMM's N dimension:
//
//   D[u, n] = sum_k A[u, k] * X[k, n]     u = p*w+q output position (lane),
//                                         k = r*RP+s padded input position,
//                                         n the windows of the tile
//
// Warp roles (640 threads):
//   warp 0        producer: bulk-copies the tile's bands (contiguous NCHW
//                 strips, w rows x W) into a ring of raw shared-memory
//                 slots, one run of bands per lane
//   warp 1        MMA issuer (one thread) and TMEM owner
//   warp 2        storer: bulk-stores finished output slots to NCHW
//   warps 3..7    transform: raw band layout -> K-major operand, one window
//                 row per thread as whole 16-byte core-matrix rows
//   warps 8..11   A builders: on a channel change they write M_c into TMEM,
//                 one tcgen05.st per (row u, window row r) from contiguous
//                 table slices; loads and transforms keep running meanwhile
//   warps 12..19  epilogue: TMEM -> registers -> bf16 (round to nearest
//                 even) -> band layout in shared memory
//
// Pipeline: raw ring (R slots) -> operand stages (2) -> accumulators (2)
// -> output slots (2).
//
// Fused 3x3 (cached matrices only): the work is split in units of whole image
// planes (one plane of several tiles, or one tile of several planes), the
// epilogue writes bf16 y into a buffer for the unit that replaces the output
// slots, and after the unit's last tile the epilogue warps apply the 3x3
// mixing to each of its planes from shared memory (zero outside the plane)
// and store z; y never reaches HBM.
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include "dw_common.cuh"
#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "wbmm_internal.h"

namespace wbmm {

template <int WS>
struct FwdCfg : PadCfg<WS> {
    using P = PadCfg<WS>;
    static constexpr int MT = (P::D + 127) / 128;          // 128-row M tiles
    static constexpr int NT = (MT == 1) ? 128 : 64;        // windows per tile (MMA N)
    static constexpr int KSTEPS = P::KP / 16;
    static constexpr int A_COLS = MT * P::KP / 2;          // TMEM columns of bf16 pairs
    static constexpr int D_COL0 = 256;                     // accumulators at [256, 512)
    static constexpr uint32_t RAW_BYTES = (uint32_t)((NT * P::D * 2 + 127) / 128 * 128);
    static constexpr uint32_t B_BYTES = (uint32_t)(NT * P::KP * 2);
    static constexpr uint32_t SBO_B = (uint32_t)(P::KP * 16);   // bytes per 8-window group
    static constexpr int TROW = 2 * WS;                          // table copy row stride
    static constexpr uint32_t TCOPY_BYTES = (uint32_t)(((2 * WS - 1) * TROW * 2 + 15) / 16 * 16);
    static constexpr uint32_t IDESC = idesc_bf16(128, NT);
    static_assert(A_COLS <= D_COL0, "A operand must fit below the accumulators");
    static_assert(2 * MT * NT <= 256, "two accumulators must fit in 256 columns");
};

constexpr int kMaxRing = 8;
// warp roles: 0 producer, 1 MMA, 2 storer, 3..7 transform, 8..11 A builders,
// 12..19 epilogue
constexpr int kTransformWarps = 5;
constexpr int kBuildWarp0 = 3 + kTransformWarps;
constexpr int kEpiWarp0 = kBuildWarp0 + 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;

struct TcFwdParams {
    TmapBytes map_x;        // whole-plane tensor maps (used when use_tmap)
    TmapBytes map_y;
    const uint16_t* x;      // bf16 bits, [B][C][H][W]
    const uint16_t* src;    // table [C][tsz] or matrices [C][d][d]
    uint16_t* y;            // output map
    int C, H, W, nh, nw;
    int bpt;                // bands per tile
    int tpc;                // tiles per channel
    int bands;              // bands per channel
    int items;              // C * tpc
    int R;                  // raw ring depth
    int use_tmap;           // tiles are whole planes: one 4-D TMA per tile
    int kimg;               // planes per tile (bpt / nh) when use_tmap
    uint32_t off_raw, off_b, off_out, off_tbl, off_woff, off_bar;
    unsigned long long budget;
    int* status;
    int fused;              // 3x3 mixing applied to y in shared memory
    int ub;                 // bands per work unit (fused: whole planes)
    int tpp;                // tiles per work unit (fused), else 1
    const uint16_t* dw;     // 3x3 weights [C][9] (fused)
    uint16_t* z;            // mixed output map (fused)
};

struct Bars {
    uint64_t raw_full[kMaxRing];
    uint64_t raw_empty[kMaxRing];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t out_full[2];
    uint64_t out_empty[2];
    uint64_t a_full[2];     // per M tile
    uint64_t a_empty[2];
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

__device__ __forceinline__ BandTile tile_of(const TcFwdParams& P, int it)
{
    BandTile t;
    t.c = it / P.tpc;
    t.band0 = (it - t.c * P.tpc) * P.bpt;
    const int left = P.bands - t.band0;
    t.nb = left < P.bpt ? left : P.bpt;
    return t;
}

// Loads the table rows the A builders slice from: copy 0 is the source table
// with rows padded to 2w entries, copy 1 the same shifted left by one entry,
// so a slice starting at any column is read as aligned 32-bit words.  The
// forward (M_c[u][v]) reads rows reversed; the input gradient (M_c[v][u])
// reads them as stored.
template <int WS, int MODE>
__device__ __forceinline__ void load_tables(uint16_t* c0, uint16_t* c1, const uint16_t* T,
                                            int tid, int nthreads)
{
    using F = FwdCfg<WS>;
    constexpr int L = 2 * WS - 1;
    for (int e = tid; e < L * F::TROW; e += nthreads) {
        const int a = e / F::TROW, col = e - a * F::TROW;
        auto src = [&](int cc) -> uint16_t {
            if (cc >= L)
                return 0;
            return T[a * L + (MODE == kTable ? (L - 1 - cc) : cc)];
        };
        c0[e] = src(col);
        c1[e] = src(col + 1);
    }
}

// Writes this warp's 32 lanes (rows u) of M tile `mt` of the A operand into
// TMEM: for each window row r the RP/2 columns holding slots r*RP .. +RP-1.
template <int WS, int MODE>
__device__ __forceinline__ void build_a(uint32_t tmem, const uint16_t* c0, const uint16_t* c1,
                                        const uint16_t* Mc, int quarter, int lane, int mt)
{
    using F = FwdCfg<WS>;
    const int u = mt * 128 + quarter * 32 + lane;
    const bool uval = u < F::D;
    const int p = uval ? u / WS : 0, q = uval ? u - (u / WS) * WS : 0;
    const int col0 = WS - 1 - q;                       // first table column of a slice
    const uint16_t* tcopy = (col0 & 1) ? c1 : c0;
    const int cbase = col0 & ~1;
    const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * (F::KP / 2));
#pragma unroll 2
    for (int r = 0; r < WS; ++r) {
        uint32_t wv[F::RP / 2];
        if (MODE == kCached) {
            const uint16_t* row = Mc + (long long)u * F::D + r * WS;
#pragma unroll
            for (int m = 0; m < F::RP / 2; ++m) {
                uint32_t v = 0;
                if (uval && 2 * m < WS) {
                    if (WS % 2 == 0) {
                        v = __ldg(reinterpret_cast<const unsigned int*>(row) + m);
                    } else {
                        const uint16_t lo = row[2 * m];
                        const uint16_t hi = (2 * m + 1 < WS) ? row[2 * m + 1] : (uint16_t)0;
                        v = pack_bf16x2(lo, hi);
                    }
                }
                wv[m] = v;
            }
        } else {
            const int a = (MODE == kTable) ? (p - r + WS - 1) : (r - p + WS - 1);
            const uint32_t* srow = reinterpret_cast<const uint32_t*>(tcopy + a * F::TROW + cbase);
#pragma unroll
            for (int m = 0; m < F::RP / 2; ++m) {
                uint32_t v = (uval && 2 * m < WS) ? srow[m] : 0u;
                if (WS % 2 == 1 && 2 * m + 1 == WS)
                    v &= 0xFFFFu;
                wv[m] = v;
            }
        }
        if constexpr (F::RP == 16) {
            tmem_st8(taddr + (uint32_t)(r * 8), wv);
        } else {
            tmem_st4(taddr + (uint32_t)(r * 4), wv);
        }
    }
    if (F::KP > F::K) {
        // zero the K columns past the last window row (odd small w)
        const uint32_t z[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int cc = F::K / 2; cc < F::KP / 2; cc += 4)
            tmem_st4(taddr + (uint32_t)cc, z);
    }
}

template <int WS, int MODE>
__global__ void __launch_bounds__(kThreads, 1) wbmm_tc_fwd_kernel(const __grid_constant__ TcFwdParams P)
{
    using F = FwdCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t* raw_base = smem + P.off_raw;
    uint8_t* b_base = smem + P.off_b;
    uint8_t* out_base = smem + P.off_out;
    uint16_t* tc0 = reinterpret_cast<uint16_t*>(smem + P.off_tbl);
    uint16_t* tc1 = reinterpret_cast<uint16_t*>(smem + P.off_tbl + F::TCOPY_BYTES);
    int* woff = reinterpret_cast<int*>(smem + P.off_woff);
    Bars& S = *reinterpret_cast<Bars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R;

    // Contiguous, balanced range of items for this CTA, in units of tpp
    // tiles (whole image planes when fused).
    const int units = P.items / P.tpp;
    const int q = units / (int)gridDim.x, rem = units % (int)gridDim.x;
    const int it0 = ((int)blockIdx.x * q + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem)) * P.tpp;
    const int n_it = (q + ((int)blockIdx.x < rem ? 1 : 0)) * P.tpp;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], kTransformWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.b_full[i], kTransformWarps);
            mbar_init(&S.b_empty[i], 1);
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], kEpiWarps);
            mbar_init(&S.out_full[i], kEpiWarps);
            mbar_init(&S.out_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.a_full[i], 4);
            mbar_init(&S.a_empty[i], 1);
        }
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    for (int n = threadIdx.x; n < F::NT; n += kThreads) {
        const int k = n / P.nw, j = n - k * P.nw;
        woff[n] = k * WS * P.W + j * WS;
    }
    // Operand stages start as zeros: K slots past the last window row are
    // never written by the transform.
    for (uint32_t e = threadIdx.x; e < 2 * F::B_BYTES / 16; e += kThreads)
        reinterpret_cast<uint4*>(b_base)[e] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
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
        // Lane 0 arms the slot's barrier; the lanes issue one run each.
        int issued = 0;
        for (int seq = 0; seq < n_it; ++seq) {
            const int s = seq % R;
            bool ok = !*abort;
            if (seq >= R)
                ok = ok && mbar_wait(&S.raw_empty[s], ((seq / R) - 1) & 1, abort, P.budget,
                                     P.status);
            if (!__all_sync(0xffffffffu, ok))
                break;
            const BandTile t = tile_of(P, it0 + seq);
            uint8_t* slot = raw_base + (size_t)s * F::RAW_BYTES;
            if (P.use_tmap) {
                // whole planes: one request; a box past the last image is
                // zero-filled and still counts its full size
                if (lane == 0) {
                    mbar_arrive_expect_tx(&S.raw_full[s], (uint32_t)P.kimg * WS * P.W * P.nh * 2);
                    tma_load_4d(slot, &P.map_x, 0, 0, t.c, t.band0 / P.nh, &S.raw_full[s]);
                }
                issued = seq + 1;
                continue;
            }
            if (lane == 0)
                mbar_arrive_expect_tx(&S.raw_full[s], (uint32_t)t.nb * WS * P.W * 2);
            __syncwarp();
            const BandRuns runs = band_runs(t, P.nh);
            for (int l = lane; l < runs.count; l += 32) {
                long long goff;
                uint32_t soff, nbytes;
                band_run(t, runs, l, WS, P.W, P.H, P.C, P.nh, goff, soff, nbytes);
                bulk_g2s(slot + soff, P.x + goff, nbytes, &S.raw_full[s]);
            }
            issued = seq + 1;
        }
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
            int cur_c = -1, ci = 0;
            for (int seq = 0; seq < n_it; ++seq) {
                const BandTile t = tile_of(P, it0 + seq);
                bool ok = !*abort;
                const bool first_of_channel = t.c != cur_c;
                if (first_of_channel) {
                    cur_c = t.c;
                    ++ci;
                }
                const int bs = seq & 1, ab = seq & 1;
                ok = ok && mbar_wait(&S.b_full[bs], (seq >> 1) & 1, abort, P.budget, P.status);
                if (seq >= 2)
                    ok = ok && mbar_wait(&S.acc_empty[ab], ((seq >> 1) - 1) & 1, abort, P.budget,
                                         P.status);
                const bool last_of_channel =
                    (seq == n_it - 1) || (tile_of(P, it0 + seq + 1).c != t.c);
                // Descriptors differ per K step only in the start-address
                // field (+256 bytes = +16 in 16-byte units); the loop is fully
                // unrolled so each MMA issues with a couple of integer adds.
                // M tiles are handed over one at a time: the A builders may
                // refill tile 0 while tile 1's last MMAs of a channel run.
                const uint64_t bdesc0 =
                    smem_desc(smem_u32(b_base + (size_t)bs * F::B_BYTES), 128, F::SBO_B);
                const uint32_t d0 = tmem + F::D_COL0 + (uint32_t)(ab * F::MT * F::NT);
#pragma unroll
                for (int mt = 0; mt < F::MT; ++mt) {
                    if (first_of_channel)
                        ok = ok && mbar_wait(&S.a_full[mt], (ci - 1) & 1, abort, P.budget, P.status);
                    if (!ok)
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < F::KSTEPS; ++k)
                        mma_ts(d0 + (uint32_t)(mt * F::NT), tmem + (uint32_t)(mt * (F::KP / 2) + k * 8),
                               bdesc0 + (uint64_t)(k * 16), F::IDESC, k > 0 ? 1u : 0u);
                    if (last_of_channel)
                        tc_commit(&S.a_empty[mt]);
                }
                if (!ok)
                    continue;
                tc_commit(&S.b_empty[bs]);
                tc_commit(&S.acc_full[ab]);
            }
            // Drain: all issued MMAs complete before TMEM is released.
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ storer
        // Bulk-stores each finished output slot (one run per lane), waits
        // until the copies have read shared memory, then frees the slot.
        // Idle when fused: the epilogue warps write z themselves.
        for (int seq = 0; seq < (P.fused ? 0 : n_it); ++seq) {
            const int os = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.out_full[os], (seq >> 1) & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const BandTile t = tile_of(P, it0 + seq);
                const BandRuns runs = band_runs(t, P.nh);
                const uint8_t* out = out_base + (size_t)os * F::RAW_BYTES;
                if (P.use_tmap && lane == 0)       // planes past the last image are clipped
                    tma_store_4d(&P.map_y, 0, 0, t.c, t.band0 / P.nh, out);
                for (int l = P.use_tmap ? runs.count : lane; l < runs.count; l += 32) {
                    long long goff;
                    uint32_t soff, nbytes;
                    band_run(t, runs, l, WS, P.W, P.H, P.C, P.nh, goff, soff, nbytes);
                    bulk_s2g(P.y + goff, out + soff, nbytes);
                }
                bulk_commit();
                bulk_wait_read<0>();
            }
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.out_empty[os]);
        }
        bulk_wait<0>();
    } else if (warp < 3 + kTransformWarps) {
        // ------------------------------------------------------ transform
        const int tt = threadIdx.x - 3 * 32;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = tile_of(P, it0 + seq);
            const int s = seq % R, bs = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.raw_full[s], (seq / R) & 1, abort, P.budget, P.status);
            if (seq >= 2)
                ok = ok && mbar_wait(&S.b_empty[bs], ((seq >> 1) - 1) & 1, abort, P.budget,
                                     P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const uint16_t* raw =
                    reinterpret_cast<const uint16_t*>(raw_base + (size_t)s * F::RAW_BYTES);
                const int nwin = t.nb * P.nw;
                transform_rows<WS>(raw, b_base + (size_t)bs * F::B_BYTES, F::SBO_B, nwin, nwin,
                                   woff, P.W, tt, kTransformWarps * 32);
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (ok && lane == 0) {
                mbar_arrive(&S.b_full[bs]);
                mbar_arrive(&S.raw_empty[s]);
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------ A builders
        const int quarter = warp & 3;
        const int at = threadIdx.x - kBuildWarp0 * 32;  // 0..127
        int cur_c = -1, ci = 0;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = tile_of(P, it0 + seq);
            if (t.c == cur_c)
                continue;
            const uint16_t* Mc = nullptr;
            if (MODE == kCached) {
                Mc = P.src + (long long)t.c * F::D * F::D;
            } else {
                // the tables live in shared memory: they can be refilled
                // before the previous channel's MMAs release TMEM
                named_bar_sync(1, 128);   // previous channel's slices all read
                load_tables<WS, MODE>(tc0, tc1, P.src + (long long)t.c * F::TSZ, at, 128);
                named_bar_sync(1, 128);
            }
            bool ok = !*abort;
#pragma unroll 1
            for (int mt = 0; mt < F::MT; ++mt) {
                if (ci > 0)
                    ok = ok && mbar_wait(&S.a_empty[mt], (ci - 1) & 1, abort, P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();
                if (ok) {
                    build_a<WS, MODE>(tmem, tc0, tc1, Mc, quarter, lane, mt);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0)
                    mbar_arrive(&S.a_full[mt]);
            }
            cur_c = t.c;
            ++ci;
        }
    } else {
        // ------------------------------------------------------ epilogue
        // Eight warps: two per TMEM lane quarter.  Each takes every other
        // 32-window chunk of the tile, loads that chunk of both M tiles with
        // one wait, and writes bf16 outputs into the band-layout slot.
        const int quarter = warp & 3;
        const int half = (warp - kEpiWarp0) >> 2;
        constexpr int NCH = F::NT / 32;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = tile_of(P, it0 + seq);
            const int nwin = t.nb * P.nw;
            const int ab = seq & 1, os = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.acc_full[ab], (seq >> 1) & 1, abort, P.budget, P.status);
            if (seq >= 2 && !P.fused)
                ok = ok && mbar_wait(&S.out_empty[os], ((seq >> 1) - 1) & 1, abort, P.budget,
                                     P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            uint16_t* out = P.fused
                ? reinterpret_cast<uint16_t*>(out_base) + (long long)(t.band0 % P.ub) * WS * P.W
                : reinterpret_cast<uint16_t*>(out_base + (size_t)os * F::RAW_BYTES);
            if (ok) {
                const uint32_t lrow = tmem + ((uint32_t)(quarter * 32) << 16) + F::D_COL0 +
                                      (uint32_t)(ab * F::MT * F::NT);
#pragma unroll 1
                for (int ch = half; ch < NCH; ch += 2) {
                    const int c0 = ch * 32;
                    if (c0 >= nwin)
                        break;
                    uint32_t r[F::MT][32];
#pragma unroll
                    for (int mt = 0; mt < F::MT; ++mt)
                        tmem_ld32(lrow + (uint32_t)(mt * F::NT + c0), r[mt]);
#pragma unroll
                    for (int mt = 0; mt < F::MT; ++mt)
                        tmem_wait_ld(r[mt]);
                    int pos[F::MT];
                    bool uval[F::MT];
#pragma unroll
                    for (int mt = 0; mt < F::MT; ++mt) {
                        const int u = mt * 128 + quarter * 32 + lane;
                        uval[mt] = u < F::D;
                        pos[mt] = (u / WS) * P.W + (u - (u / WS) * WS);
                    }
                    // window offsets walked in registers: band k, column j
                    int wk = c0 / P.nw, wj = c0 - wk * P.nw;
                    int wo = wk * WS * P.W + wj * WS;
                    const int band_step = WS * P.W - (P.nw - 1) * WS;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int n = c0 + jj;
                        if (n < nwin) {
                            uint16_t* o = out + wo;
#pragma unroll
                            for (int mt = 0; mt < F::MT; ++mt)
                                if (uval[mt])
                                    o[pos[mt]] = __bfloat16_as_ushort(
                                        __float2bfloat16_rn(__uint_as_float(r[mt][jj])));
                        }
                        if (++wj == P.nw) {
                            wj = 0;
                            wo += band_step;
                        } else {
                            wo += WS;
                        }
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) {
                mbar_arrive(&S.acc_empty[ab]);
                if (!P.fused)
                    mbar_arrive(&S.out_full[os]);
            }
            if (P.fused && (seq + 1) % P.tpp == 0) {
                // the unit's last tile: y of its planes is complete in shared memory
                named_bar_sync(4, kEpiWarps * 32);
                const int et = threadIdx.x - kEpiWarp0 * 32;
                const int ub0 = t.band0 - t.band0 % P.ub;
                const int left = P.bands - ub0;
                const int planes = (left < P.ub ? left : P.ub) / P.nh;
                const int b0 = ub0 / P.nh;
                uint64_t kw[9];
                dw_weights(P.dw + t.c * 9, kw);
                const int nvec = P.W / 8, per_plane = P.H * nvec;
                for (int o = et; o < planes * per_plane; o += kEpiWarps * 32) {
                    const int j = o / per_plane, r = o - j * per_plane;
                    const int h = r / nvec, v = r - (r / nvec) * nvec;
                    const uint16_t* mid = reinterpret_cast<const uint16_t*>(out_base) +
                                          ((long long)j * P.H + h) * P.W + 8 * v;
                    const uint16_t* rows[3] = {h > 0 ? mid - P.W : nullptr, mid,
                                               h + 1 < P.H ? mid + P.W : nullptr};
                    uint4* zp = reinterpret_cast<uint4*>(
                        P.z + (((long long)(b0 + j) * P.C + t.c) * P.H) * P.W);
                    zp[r] = dw3x3_row8(rows, v, nvec, kw);
                }
                named_bar_sync(4, kEpiWarps * 32);   // read before the buffer is rewritten
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

struct FwdLayout {
    uint32_t off_raw, off_b, off_out, off_tbl, off_woff, off_bar, total;
    int R;
};

// out_bytes: the output region, two band slots, or one image plane when the
// 3x3 mixing is fused.
template <int WS>
FwdLayout fwd_layout(uint32_t out_bytes)
{
    using F = FwdCfg<WS>;
    FwdLayout L;
    const uint32_t fixed = 2 * F::B_BYTES + out_bytes + 2 * F::TCOPY_BYTES + F::NT * 4 +
                           align_up(sizeof(Bars), 16) + 3 * 1024;
    if (fixed >= kSmemMax) {
        L.R = 0;
        L.total = kSmemMax + 1;
        return L;
    }
    int R = (int)((kSmemMax - fixed) / F::RAW_BYTES);
    if (R > kMaxRing)
        R = kMaxRing;
    L.R = R;
    uint32_t off = 0;
    L.off_b = off;                       // operand stages first: 1024-aligned
    off += 2 * F::B_BYTES;
    L.off_raw = align_up(off, 128);
    off = L.off_raw + (uint32_t)R * F::RAW_BYTES;
    L.off_out = align_up(off, 128);
    off = L.off_out + out_bytes;
    L.off_tbl = align_up(off, 16);
    off = L.off_tbl + 2 * F::TCOPY_BYTES;
    L.off_woff = align_up(off, 16);
    off = L.off_woff + F::NT * 4;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(Bars);
    L.total = align_up(off, 1024);
    // at least half the SM's shared memory: one CTA (and one 512-column TMEM
    // allocation) per SM
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L;
}

// Bands per fused work unit: one plane of several tiles or one tile of
// several planes; 0 when neither divides the other.
int fused_unit_bands(const Geom& g, int bpt)
{
    if (g.nh % bpt == 0)
        return g.nh;
    if (bpt % g.nh == 0)
        return bpt;
    return 0;
}

template <int WS>
uint32_t out_region_bytes(const Geom& g, bool fused)
{
    if (!fused)
        return 2 * FwdCfg<WS>::RAW_BYTES;
    const int ub = fused_unit_bands(g, FwdCfg<WS>::NT / g.nw);
    return align_up((uint32_t)((long long)ub * WS * g.W * 2), 128);
}

// y: the output map (z when fused); dw: the 3x3 weights when fused, else null.
template <int WS, int MODE>
cudaError_t launch_ws(const Geom& g, const void* x, const void* src, void* y, const void* dw,
                      const Launch& L)
{
    using F = FwdCfg<WS>;
    const bool fused = dw != nullptr;
    const FwdLayout lay = fwd_layout<WS>(out_region_bytes<WS>(g, fused));
    if (lay.R < 2 || lay.total > kSmemMax)
        return cudaErrorInvalidConfiguration;
    static int configured_smem[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_smem[dev & 63] < (int)kSmemMax) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_fwd_kernel<WS, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMax);
        if (e != cudaSuccess)
            return e;
        configured_smem[dev & 63] = (int)kSmemMax;
    }
    TcFwdParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.src = static_cast<const uint16_t*>(src);
    P.y = static_cast<uint16_t*>(y);
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = F::NT / g.nw;
    P.bands = (int)g.bands;
    P.tpc = (P.bands + P.bpt - 1) / P.bpt;
    P.items = g.C * P.tpc;
    P.R = lay.R;
    P.fused = fused ? 1 : 0;
    P.ub = fused ? fused_unit_bands(g, P.bpt) : P.bpt;
    P.tpp = fused ? P.ub / P.bpt : 1;
    P.dw = static_cast<const uint16_t*>(dw);
    P.z = fused ? static_cast<uint16_t*>(y) : nullptr;
    P.use_tmap = 0;
    P.kimg = 0;
    if (P.bpt % g.nh == 0) {
        const int k = P.bpt / g.nh;
        if (encode_plane_map(&P.map_x, x, g, k) && encode_plane_map(&P.map_y, y, g, k)) {
            P.use_tmap = 1;
            P.kimg = k;
        }
    }
    P.off_raw = lay.off_raw; P.off_b = lay.off_b; P.off_out = lay.off_out;
    P.off_tbl = lay.off_tbl; P.off_woff = lay.off_woff; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    int grid = L.num_sms;
    if (grid > P.items / P.tpp)
        grid = P.items / P.tpp;
    if (grid < 1)
        return cudaSuccess;
    cudaError_t e = launch_pdl(wbmm_tc_fwd_kernel<WS, MODE>, dim3(grid), dim3(kThreads),
                               lay.total, L.stream, P);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

template <int WS>
cudaError_t launch_mode(const Geom& g, AMode mode, const void* x, const void* src, void* y,
                        const void* dw, const Launch& L)
{
    switch (mode) {
    case kTable: return launch_ws<WS, kTable>(g, x, src, y, nullptr, L);
    case kTableFlip: return launch_ws<WS, kTableFlip>(g, x, src, y, nullptr, L);
    default: return launch_ws<WS, kCached>(g, x, src, y, dw, L);
    }
}

template <int WS>
bool fused_fits(const Geom& g)
{
    const FwdLayout lay = fwd_layout<WS>(out_region_bytes<WS>(g, true));
    return lay.R >= 2 && lay.total <= kSmemMax;
}

int nt_for(int w)
{
    const int d = w * w;
    return ((d + 127) / 128 == 1) ? 128 : 64;
}

}  // namespace

bool tc_fwd_supported(const Geom& g, bool fused)
{
    if (g.w < 2 || g.w > 16)
        return false;
    if (g.nw > nt_for(g.w))
        return false;
    // bulk copies move whole bands: 16-byte multiples
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    // 32-bit tile bookkeeping
    if (g.bands * (long long)g.C >= (1ll << 31))
        return false;
    if (fused) {
        // tiles are whole bands of one plane, planes whole 16-byte rows, and
        // one plane of y fits in shared memory beside the pipeline
        if (g.W % 8 != 0 || fused_unit_bands(g, nt_for(g.w) / g.nw) == 0)
            return false;
        switch (g.w) {
        case 2: return fused_fits<2>(g);
        case 3: return fused_fits<3>(g);
        case 4: return fused_fits<4>(g);
        case 5: return fused_fits<5>(g);
        case 6: return fused_fits<6>(g);
        case 7: return fused_fits<7>(g);
        case 8: return fused_fits<8>(g);
        case 9: return fused_fits<9>(g);
        case 10: return fused_fits<10>(g);
        case 11: return fused_fits<11>(g);
        case 12: return fused_fits<12>(g);
        case 13: return fused_fits<13>(g);
        case 14: return fused_fits<14>(g);
        case 15: return fused_fits<15>(g);
        default: return fused_fits<16>(g);
        }
    }
    return true;
}

cudaError_t tc_fwd_launch(const Geom& g, AMode mode, const void* x, const void* src, void* y,
                          const void* dw, const Launch& L)
{
    switch (g.w) {
    case 2: return launch_mode<2>(g, mode, x, src, y, dw, L);
    case 3: return launch_mode<3>(g, mode, x, src, y, dw, L);
    case 4: return launch_mode<4>(g, mode, x, src, y, dw, L);
    case 5: return launch_mode<5>(g, mode, x, src, y, dw, L);
    case 6: return launch_mode<6>(g, mode, x, src, y, dw, L);
    case 7: return launch_mode<7>(g, mode, x, src, y, dw, L);
    case 8: return launch_mode<8>(g, mode, x, src, y, dw, L);
    case 9: return launch_mode<9>(g, mode, x, src, y, dw, L);
    case 10: return launch_mode<10>(g, mode, x, src, y, dw, L);
    case 11: return launch_mode<11>(g, mode, x, src, y, dw, L);
    case 12: return launch_mode<12>(g, mode, x, src, y, dw, L);
    case 13: return launch_mode<13>(g, mode, x, src, y, dw, L);
    case 14: return launch_mode<14>(g, mode, x, src, y, dw, L);
    case 15: return launch_mode<15>(g, mode, x, src, y, dw, L);
    case 16: return launch_mode<16>(g, mode, x, src, y, dw, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
