// Tensor-core (tcgen05) WBMM forward, input-gradient and cached-matrix kernel.
//
// One persistent CTA per SM walks a contiguous range of work items; an item is
// (channel c, tile of whole bands).  For every channel the CTA writes the
// d x d matrix M_c (or its transpose, for the input gradient) into tensor
// memory once; it is the A operand of every MMA of that channel and is never
// written to HBM.  Windows stream through as the GEMM's N dimension:
//
//   D[u, n] = sum_v A[u, v] * X[v, n]        u, v in-window positions,
//                                            n the windows of the tile
//
// Warp roles (320 threads):
//   warp 0      producer: bulk-copies the tile's bands (contiguous NCHW
//               strips, w rows x W) into a ring of raw shared-memory slots
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warps 2..5  transform: raw band layout -> K-major UMMA operand (no
//               swizzle, 8x16B core matrices); on a channel change they
//               expand the table (or load the cached matrix) into TMEM
//   warps 6..9  epilogue: TMEM -> registers -> bf16 (round to nearest even)
//               -> band layout in shared memory -> bulk store to NCHW
//
// Pipeline: raw ring (R slots) -> operand stages (2) -> accumulators (2).
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "wbmm_internal.h"

namespace wbmm {

template <int WS>
struct FwdCfg {
    static constexpr int D = WS * WS;
    static constexpr int KP = (D + 15) / 16 * 16;          // K padded to the MMA K step
    static constexpr int MT = (D + 127) / 128;             // 128-row M tiles
    static constexpr int NT = (MT == 1) ? 128 : 64;        // windows per tile (MMA N)
    static constexpr int KSTEPS = KP / 16;
    static constexpr int TSZ = (2 * WS - 1) * (2 * WS - 1);
    static constexpr int A_COLS = MT * KP / 2;             // TMEM columns of bf16 pairs
    static constexpr int D_COL0 = 256;                     // accumulators at [256, 512)
    static constexpr uint32_t RAW_BYTES = (uint32_t)((NT * D * 2 + 127) / 128 * 128);
    static constexpr uint32_t B_BYTES = (uint32_t)(NT * KP * 2);
    static constexpr uint32_t SBO_B = (uint32_t)(KP * 16);  // bytes per 8-window group
    static constexpr uint32_t TBL_BYTES = (uint32_t)((TSZ * 2 + 15) / 16 * 16);
    static constexpr uint32_t IDESC = idesc_bf16(128, NT);
    static_assert(A_COLS <= D_COL0, "A operand must fit below the accumulators");
    static_assert(2 * MT * NT <= 256, "two accumulators must fit in 256 columns");
};

constexpr int kMaxRing = 8;
constexpr int kThreads = 320;

struct TcFwdParams {
    const uint16_t* x;      // bf16 bits, [B][C][H][W]
    const uint16_t* src;    // table [C][tsz] or matrices [C][d][d]
    uint16_t* y;            // output map
    int C, H, W, nh, nw;
    int bpt;                // bands per tile
    int tpc;                // tiles per channel
    long long bands;        // bands per channel
    long long items;        // C * tpc
    int R;                  // raw ring depth
    uint32_t off_raw, off_b, off_out, off_tbl, off_woff, off_bar;
    unsigned long long budget;
    int* status;
};

struct Bars {
    uint64_t raw_full[kMaxRing];
    uint64_t raw_empty[kMaxRing];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t a_full;
    uint64_t a_empty;
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

struct TileRef {
    int c;
    long long band0;
    int nb;
};

__device__ __forceinline__ TileRef tile_ref(const TcFwdParams& P, long long it)
{
    TileRef t;
    t.c = (int)(it / P.tpc);
    const int ti = (int)(it - (long long)t.c * P.tpc);
    t.band0 = (long long)ti * P.bpt;
    const long long left = P.bands - t.band0;
    t.nb = (int)(left < P.bpt ? left : P.bpt);
    return t;
}

// Calls f(global element offset, byte offset in the slot, bytes) for each
// contiguous run of bands (bands of one image plane are adjacent in NCHW).
template <int WS, typename F>
__device__ __forceinline__ void for_each_run(const TcFwdParams& P, const TileRef& t, F&& f)
{
    const long long band_elems = (long long)WS * P.W;
    long long g = t.band0;
    const long long g_end = t.band0 + t.nb;
    uint32_t soff = 0;
    while (g < g_end) {
        const long long b = g / P.nh;
        const int i = (int)(g - b * P.nh);
        long long run = P.nh - i;
        if (run > g_end - g)
            run = g_end - g;
        const long long goff = ((b * P.C + t.c) * (long long)P.H + (long long)i * WS) * P.W;
        const uint32_t bytes = (uint32_t)(run * band_elems * 2);
        f(goff, soff, bytes);
        soff += bytes;
        g += run;
    }
}

// Relative-table entry of M_c[u][v] (or of M_c[v][u] when flipped).
template <int WS, int MODE>
__device__ __forceinline__ uint16_t a_elem(const uint16_t* tbl, const uint16_t* Mc, int u, int p,
                                           int q, int v)
{
    constexpr int D = WS * WS;
    constexpr int TSZ = (2 * WS - 1) * (2 * WS - 1);
    if (v >= D)
        return 0;
    if (MODE == kCached)
        return Mc[(long long)u * D + v];
    const int r = v / WS, s = v - (v / WS) * WS;
    const int idx = (p - r + WS - 1) * (2 * WS - 1) + (q - s + WS - 1);
    return tbl[MODE == kTableFlip ? (TSZ - 1 - idx) : idx];
}

// Writes the A operand (rows u = lanes, K pairs packed in 32-bit columns)
// of this warp's 32-lane quarter into TMEM.
template <int WS, int MODE>
__device__ __forceinline__ void expand_a(uint32_t tmem, const uint16_t* tbl, const uint16_t* Mc,
                                         int quarter, int lane)
{
    using Cfg = FwdCfg<WS>;
#pragma unroll 1
    for (int mt = 0; mt < Cfg::MT; ++mt) {
        const int u = mt * 128 + quarter * 32 + lane;
        const bool uval = u < Cfg::D;
        const int p = u / WS, q = u - (u / WS) * WS;
#pragma unroll 1
        for (int c8 = 0; c8 < Cfg::KP / 2; c8 += 8) {
            uint32_t r[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int v0 = 2 * (c8 + jj);
                uint16_t lo = 0, hi = 0;
                if (uval) {
                    lo = a_elem<WS, MODE>(tbl, Mc, u, p, q, v0);
                    hi = a_elem<WS, MODE>(tbl, Mc, u, p, q, v0 + 1);
                }
                r[jj] = pack_bf16x2(lo, hi);
            }
            tmem_st8(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * (Cfg::KP / 2) + c8),
                     r);
        }
    }
}

// Raw band layout -> K-major operand.  One warp instruction writes one
// 8-window x 8-position core matrix (128 contiguous bytes, conflict free).
template <int WS>
__device__ __forceinline__ void transform_tile(const uint16_t* raw, uint8_t* bst, int nwin,
                                               const int* woff, int W, int tw, int lane)
{
    using Cfg = FwdCfg<WS>;
    constexpr int KG = Cfg::KP / 8;
    constexpr int NG = Cfg::NT / 8;
    const int nl = lane & 7, pair = lane >> 3;
#pragma unroll 1
    for (int g8 = tw; g8 < NG; g8 += 4) {
        if (g8 * 8 >= nwin)
            break;
        const int n = g8 * 8 + nl;
        const bool nval = n < nwin;
        const int wo = nval ? woff[n] : 0;
        uint32_t* dst = reinterpret_cast<uint32_t*>(bst + g8 * Cfg::SBO_B + nl * 16 + pair * 4);
#pragma unroll 2
        for (int vg = 0; vg < KG; ++vg) {
            const int v = vg * 8 + pair * 2;
            uint32_t word = 0;
            if (nval && v < Cfg::D) {
                if (WS % 2 == 0) {
                    const int r = v / WS, s = v - (v / WS) * WS;
                    word = *reinterpret_cast<const uint32_t*>(raw + wo + r * W + s);
                } else {
                    const int r0 = v / WS, s0 = v - r0 * WS;
                    const uint16_t lo = raw[wo + r0 * W + s0];
                    uint16_t hi = 0;
                    if (v + 1 < Cfg::D) {
                        const int r1 = (v + 1) / WS, s1 = (v + 1) - r1 * WS;
                        hi = raw[wo + r1 * W + s1];
                    }
                    word = pack_bf16x2(lo, hi);
                }
            }
            dst[vg * 32] = word;
        }
    }
}

template <int WS, int MODE>
__global__ void __launch_bounds__(kThreads, 1) wbmm_tc_fwd_kernel(const TcFwdParams P)
{
    using Cfg = FwdCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t* raw_base = smem + P.off_raw;
    uint8_t* b_base = smem + P.off_b;
    uint8_t* out_base = smem + P.off_out;
    int* woff = reinterpret_cast<int*>(smem + P.off_woff);
    Bars& S = *reinterpret_cast<Bars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R;

    // Contiguous, balanced range of items for this CTA.
    const long long q = P.items / gridDim.x, rem = P.items % gridDim.x;
    const long long it0 = blockIdx.x * q + (blockIdx.x < rem ? blockIdx.x : rem);
    const int n_it = (int)(q + (blockIdx.x < rem ? 1 : 0));

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.b_full[i], 4);
            mbar_init(&S.b_empty[i], 1);
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], 4);
        }
        mbar_init(&S.a_full, 4);
        mbar_init(&S.a_empty, 1);
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    for (int n = threadIdx.x; n < Cfg::NT; n += kThreads) {
        const int k = n / P.nw, j = n - (n / P.nw) * P.nw;
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

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int seq = 0; seq < n_it; ++seq) {
                const int s = seq % R;
                if (*abort)
                    break;
                if (seq >= R && !mbar_wait(&S.raw_empty[s], ((seq / R) - 1) & 1, abort, P.budget,
                                           P.status))
                    break;
                const TileRef t = tile_ref(P, it0 + seq);
                const uint32_t bytes = (uint32_t)t.nb * WS * P.W * 2;
                mbar_arrive_expect_tx(&S.raw_full[s], bytes);
                uint8_t* slot = raw_base + (size_t)s * Cfg::RAW_BYTES;
                for_each_run<WS>(P, t, [&](long long goff, uint32_t soff, uint32_t nbytes) {
                    bulk_g2s(slot + soff, P.x + goff, nbytes, &S.raw_full[s]);
                });
                issued = seq + 1;
            }
            // Drain: every issued copy lands before the CTA can exit.
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
                const TileRef t = tile_ref(P, it0 + seq);
                bool ok = !*abort;
                if (t.c != cur_c) {
                    ok = ok && mbar_wait(&S.a_full, ci & 1, abort, P.budget, P.status);
                    cur_c = t.c;
                    ++ci;
                }
                const int bs = seq & 1, ab = seq & 1;
                ok = ok && mbar_wait(&S.b_full[bs], (seq >> 1) & 1, abort, P.budget, P.status);
                if (seq >= 2)
                    ok = ok && mbar_wait(&S.acc_empty[ab], ((seq >> 1) - 1) & 1, abort, P.budget,
                                         P.status);
                if (!ok)
                    continue;
                tc_fence_after();
                const uint32_t b_addr = smem_u32(b_base + (size_t)bs * Cfg::B_BYTES);
#pragma unroll
                for (int mt = 0; mt < Cfg::MT; ++mt) {
                    const uint32_t d_tmem =
                        tmem + Cfg::D_COL0 + (uint32_t)(ab * Cfg::MT * Cfg::NT + mt * Cfg::NT);
                    const uint32_t a_tmem = tmem + (uint32_t)(mt * (Cfg::KP / 2));
#pragma unroll 1
                    for (int k = 0; k < Cfg::KSTEPS; ++k) {
                        const uint64_t bdesc = smem_desc(b_addr + k * 256, 128, Cfg::SBO_B);
                        mma_ts(d_tmem, a_tmem + (uint32_t)(k * 8), bdesc, Cfg::IDESC, k > 0);
                    }
                }
                tc_commit(&S.b_empty[bs]);
                tc_commit(&S.acc_full[ab]);
                const bool last_of_channel =
                    (seq == n_it - 1) || (tile_ref(P, it0 + seq + 1).c != t.c);
                if (last_of_channel)
                    tc_commit(&S.a_empty);
            }
            // Drain: all issued MMAs complete before TMEM is released.
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------ transform
        const int tw = warp - 2;
        const int quarter = warp & 3;
        uint16_t* tbl = reinterpret_cast<uint16_t*>(smem + P.off_tbl + tw * Cfg::TBL_BYTES);
        int cur_c = -1, ci = 0;
        for (int seq = 0; seq < n_it; ++seq) {
            const TileRef t = tile_ref(P, it0 + seq);
            if (t.c != cur_c) {
                bool ok = !*abort;
                if (ci > 0)
                    ok = ok && mbar_wait(&S.a_empty, (ci - 1) & 1, abort, P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();
                const uint16_t* Mc = nullptr;
                if (MODE == kCached) {
                    Mc = P.src + (long long)t.c * Cfg::D * Cfg::D;
                } else {
                    for (int i = lane; i < Cfg::TSZ; i += 32)
                        tbl[i] = P.src[(long long)t.c * Cfg::TSZ + i];
                    __syncwarp();
                }
                if (ok) {
                    expand_a<WS, MODE>(tmem, tbl, Mc, quarter, lane);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0)
                    mbar_arrive(&S.a_full);
                cur_c = t.c;
                ++ci;
            }
            const int s = seq % R, bs = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.raw_full[s], (seq / R) & 1, abort, P.budget, P.status);
            if (seq >= 2)
                ok = ok && mbar_wait(&S.b_empty[bs], ((seq >> 1) - 1) & 1, abort, P.budget,
                                     P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const uint16_t* raw =
                    reinterpret_cast<const uint16_t*>(raw_base + (size_t)s * Cfg::RAW_BYTES);
                transform_tile<WS>(raw, b_base + (size_t)bs * Cfg::B_BYTES, t.nb * P.nw, woff, P.W,
                                   tw, lane);
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (ok && lane == 0) {
                mbar_arrive(&S.b_full[bs]);
                mbar_arrive(&S.raw_empty[s]);
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int et = threadIdx.x - 6 * 32;  // 0..127
        for (int seq = 0; seq < n_it; ++seq) {
            const TileRef t = tile_ref(P, it0 + seq);
            const int nwin = t.nb * P.nw;
            const int ab = seq & 1, os = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.acc_full[ab], (seq >> 1) & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (et == 0)
                bulk_wait_read<1>();
            named_bar_sync(2, 128);
            uint16_t* out = reinterpret_cast<uint16_t*>(out_base + (size_t)os * Cfg::RAW_BYTES);
            if (ok) {
#pragma unroll 1
                for (int mt = 0; mt < Cfg::MT; ++mt) {
                    const int u = mt * 128 + quarter * 32 + lane;
                    const int pos = (u / WS) * P.W + (u - (u / WS) * WS);
                    const uint32_t dcol =
                        tmem + ((uint32_t)(quarter * 32) << 16) + Cfg::D_COL0 +
                        (uint32_t)(ab * Cfg::MT * Cfg::NT + mt * Cfg::NT);
#pragma unroll 1
                    for (int c0 = 0; c0 < Cfg::NT; c0 += 32) {
                        if (c0 >= nwin)
                            break;
                        uint32_t r[32];
                        tmem_ld32(dcol + (uint32_t)c0, r);
                        tmem_wait_ld(r);
                        if (u < Cfg::D) {
#pragma unroll
                            for (int jj = 0; jj < 32; ++jj) {
                                const int n = c0 + jj;
                                if (n < nwin)
                                    out[woff[n] + pos] = __bfloat16_as_ushort(
                                        __float2bfloat16_rn(__uint_as_float(r[jj])));
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.acc_empty[ab]);
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            if (et == 0 && ok && !*abort) {
                for_each_run<WS>(P, t, [&](long long goff, uint32_t soff, uint32_t nbytes) {
                    bulk_s2g(P.y + goff, reinterpret_cast<const uint8_t*>(out) + soff, nbytes);
                });
                bulk_commit();
            }
        }
        if (et == 0)
            bulk_wait<0>();
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

template <int WS>
struct FwdLayout {
    uint32_t off_raw, off_b, off_out, off_tbl, off_woff, off_bar, total;
    int R;
};

constexpr uint32_t kSmemMax = 232448;
constexpr uint32_t kMinSmem = 120 * 1024;

inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

template <int WS>
FwdLayout<WS> fwd_layout()
{
    using Cfg = FwdCfg<WS>;
    FwdLayout<WS> L;
    const uint32_t fixed = 2 * Cfg::B_BYTES + 2 * Cfg::RAW_BYTES + 4 * Cfg::TBL_BYTES +
                           Cfg::NT * 4 + align_up(sizeof(Bars), 16) + 3 * 1024;
    int R = (int)((kSmemMax - fixed) / Cfg::RAW_BYTES);
    if (R > kMaxRing)
        R = kMaxRing;
    L.R = R;
    uint32_t off = 0;
    L.off_b = off;                       // operand stages first: 1024-aligned
    off += 2 * Cfg::B_BYTES;
    L.off_raw = align_up(off, 128);
    off = L.off_raw + (uint32_t)R * Cfg::RAW_BYTES;
    L.off_out = align_up(off, 128);
    off = L.off_out + 2 * Cfg::RAW_BYTES;
    L.off_tbl = align_up(off, 16);
    off = L.off_tbl + 4 * Cfg::TBL_BYTES;
    L.off_woff = align_up(off, 16);
    off = L.off_woff + Cfg::NT * 4;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(Bars);
    L.total = align_up(off, 1024);
    // at least half the SM's shared memory: one CTA (and one 512-column
    // TMEM allocation) per SM
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L;
}

template <int WS, int MODE>
cudaError_t launch_ws(const Geom& g, const void* x, const void* src, void* y, const Launch& L)
{
    using Cfg = FwdCfg<WS>;
    const FwdLayout<WS> lay = fwd_layout<WS>();
    if (lay.R < 2 || lay.total > kSmemMax)
        return cudaErrorInvalidConfiguration;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(configured & (1ull << (dev & 63)))) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_fwd_kernel<WS, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)lay.total);
        if (e != cudaSuccess)
            return e;
        configured |= 1ull << (dev & 63);
    }
    TcFwdParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.src = static_cast<const uint16_t*>(src);
    P.y = static_cast<uint16_t*>(y);
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = Cfg::NT / g.nw;
    P.bands = g.bands;
    P.tpc = (int)((g.bands + P.bpt - 1) / P.bpt);
    P.items = (long long)g.C * P.tpc;
    P.R = lay.R;
    P.off_raw = lay.off_raw; P.off_b = lay.off_b; P.off_out = lay.off_out;
    P.off_tbl = lay.off_tbl; P.off_woff = lay.off_woff; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    long long grid = L.num_sms;
    if (grid > P.items)
        grid = P.items;
    if (grid < 1)
        return cudaSuccess;
    wbmm_tc_fwd_kernel<WS, MODE><<<(unsigned)grid, kThreads, lay.total, L.stream>>>(P);
    note_launches(1);
    return cudaGetLastError();
}

template <int WS>
cudaError_t launch_mode(const Geom& g, AMode mode, const void* x, const void* src, void* y,
                        const Launch& L)
{
    switch (mode) {
    case kTable: return launch_ws<WS, kTable>(g, x, src, y, L);
    case kTableFlip: return launch_ws<WS, kTableFlip>(g, x, src, y, L);
    default: return launch_ws<WS, kCached>(g, x, src, y, L);
    }
}

int nt_for(int w)
{
    const int d = w * w;
    return ((d + 127) / 128 == 1) ? 128 : 64;
}

}  // namespace

bool tc_fwd_supported(const Geom& g, bool fused)
{
    if (fused)
        return false;
    if (g.w < 2 || g.w > 16)
        return false;
    if (g.nw > nt_for(g.w))
        return false;
    // bulk copies move whole bands: 16-byte multiples
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    return true;
}

cudaError_t tc_fwd_launch(const Geom& g, AMode mode, const void* x, const void* src, void* y,
                          const void* dw, const Launch& L)
{
    (void)dw;
    switch (g.w) {
    case 2: return launch_mode<2>(g, mode, x, src, y, L);
    case 3: return launch_mode<3>(g, mode, x, src, y, L);
    case 4: return launch_mode<4>(g, mode, x, src, y, L);
    case 5: return launch_mode<5>(g, mode, x, src, y, L);
    case 6: return launch_mode<6>(g, mode, x, src, y, L);
    case 7: return launch_mode<7>(g, mode, x, src, y, L);
    case 8: return launch_mode<8>(g, mode, x, src, y, L);
    case 9: return launch_mode<9>(g, mode, x, src, y, L);
    case 10: return launch_mode<10>(g, mode, x, src, y, L);
    case 11: return launch_mode<11>(g, mode, x, src, y, L);
    case 12: return launch_mode<12>(g, mode, x, src, y, L);
    case 13: return launch_mode<13>(g, mode, x, src, y, L);
    case 14: return launch_mode<14>(g, mode, x, src, y, L);
    case 15: return launch_mode<15>(g, mode, x, src, y, L);
    case 16: return launch_mode<16>(g, mode, x, src, y, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
