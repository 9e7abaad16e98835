// Tensor-core (tcgen05) WBMM table gradient.
//
// For one channel, G = dY X^T is a d x d matrix summed over windows:
//   G[u, v] = sum_n dY[u, n] X[v, n]        (u, v in-window positions)
// and the table gradient is its sum along constant relative offset:
//   dT[(p-r+w-1)(2w-1) + (q-s+w-1)] = sum over (u=(p,q), v=(r,s)) of G[u, v].
//
// Work item = (channel, fixed chunk of tiles).  The chunk split depends only
// on the shape, every sum runs in a fixed order, and each item writes its own
// fp32 partial table, so the result is bit-identical from run to run and for
// any grid size; a second kernel adds the partials in chunk order.
//
// Per tile (64 windows = the MMA's K for this GEMM) the producer bulk-copies
// the dY and x bands into a raw slot; the transform warps write both as
// K-major operands (rows = positions, K = windows); one thread issues
// 128 x NP x 16 MMAs into G held in TMEM (two 128-row halves for d > 128).
// After the item's last tile the epilogue warps read G from TMEM and add each
// entry into a per-warp bin array in shared memory (within one TMEM column
// every lane maps to a different bin, so the adds never collide), then sum the
// four warp arrays in warp order into the item's partial table.
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "wbmm_internal.h"

namespace wbmm {

template <int WS>
struct DtCfg {
    static constexpr int D = WS * WS;
    static constexpr int MT = (D + 127) / 128;
    static constexpr int NP = (D + 15) / 16 * 16;           // MMA N (positions of x)
    static constexpr int NT = 64;                           // windows per tile = K per stage
    static constexpr int KSTEPS = NT / 16;
    static constexpr int TSZ = (2 * WS - 1) * (2 * WS - 1);
    static constexpr uint32_t SBO = NT * 16;                // bytes per 8-row group
    static constexpr int RG = (D + 7) / 8;                  // written 8-row groups
    // Rows of the A tile past D are never stored; the MMA may read them from
    // the B tile that follows (their products land in ignored rows of G).
    static constexpr int A_GROUPS = ((MT * 128 - RG * 8) <= NP) ? RG : MT * 16;
    static constexpr uint32_t A_BYTES = A_GROUPS * SBO;
    static constexpr uint32_t B_BYTES = (NP / 8) * SBO;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t RAW_HALF = (uint32_t)((NT * D * 2 + 127) / 128 * 128);
    static constexpr uint32_t RAW_BYTES = 2 * RAW_HALF;    // dY tile, then x tile
    static constexpr uint32_t IDESC = idesc_bf16(128, NP);
    static_assert(MT * 256 <= 512 || MT == 1, "G must fit in TMEM");
};

constexpr int kDtThreads = 320;
constexpr int kDtRing = 2;

struct TcDtParams {
    const uint16_t* x;
    const uint16_t* dy;
    float* partials;        // [C][chunks][tsz]
    int C, H, W, nh, nw;
    int bpt;
    int tpc;                // tiles per channel
    int ch;                 // tiles per chunk
    int chunks;             // chunks per channel
    long long bands;
    long long items;        // C * chunks
    uint32_t off_raw, off_stage, off_bins, off_woff, off_bar;
    unsigned long long budget;
    int* status;
};

struct DtBars {
    uint64_t raw_full[kDtRing];
    uint64_t raw_empty[kDtRing];
    uint64_t st_full[2];
    uint64_t st_empty[2];
    uint64_t g_full;
    uint64_t g_empty;
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

struct DtTile {
    int c;
    long long band0;
    int nb;
    bool first, last;   // first / last tile of its item
};

// The flattened tile sequence of a CTA: items blockIdx.x, +grid, ...; within
// an item its tiles in order.  Every role walks the same sequence.
struct DtWalker {
    long long item;
    int tile;       // tile index within the channel
    int tile_end;
    __device__ __forceinline__ bool valid(const TcDtParams& P) const { return item < P.items; }
    __device__ __forceinline__ void start(const TcDtParams& P)
    {
        item = blockIdx.x;
        set_item(P);
    }
    __device__ __forceinline__ void set_item(const TcDtParams& P)
    {
        if (item >= P.items)
            return;
        const int chunk = (int)(item % P.chunks);
        tile = chunk * P.ch;
        tile_end = tile + P.ch < P.tpc ? tile + P.ch : P.tpc;
    }
    __device__ __forceinline__ DtTile get(const TcDtParams& P) const
    {
        DtTile t;
        t.c = (int)(item / P.chunks);
        t.band0 = (long long)tile * P.bpt;
        const long long left = P.bands - t.band0;
        t.nb = (int)(left < P.bpt ? left : P.bpt);
        const int chunk = (int)(item % P.chunks);
        t.first = tile == chunk * P.ch;
        t.last = tile + 1 == tile_end;
        return t;
    }
    __device__ __forceinline__ void next(const TcDtParams& P)
    {
        if (++tile >= tile_end) {
            item += gridDim.x;
            set_item(P);
        }
    }
};

template <int WS, typename F>
__device__ __forceinline__ void dt_runs(const TcDtParams& P, const DtTile& t, F&& f)
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

// One operand (rows = positions of `raw`, K = windows) -> K-major core matrices.
template <int WS>
__device__ __forceinline__ void dt_transform(const uint16_t* raw, uint8_t* dst, int nwin,
                                             const int* woff, int W, int tw, int lane)
{
    using Cfg = DtCfg<WS>;
    constexpr int NG = Cfg::NT / 8;
    const int rl = lane & 7, pair = lane >> 3;
#pragma unroll 1
    for (int cm = tw; cm < Cfg::RG * NG; cm += 4) {
        const int rg = cm / NG, ng = cm - (cm / NG) * NG;
        const int row = rg * 8 + rl;
        const int n0 = ng * 8 + pair * 2;
        uint16_t lo = 0, hi = 0;
        if (row < Cfg::D) {
            const int pos = (row / WS) * W + (row - (row / WS) * WS);
            if (n0 < nwin)
                lo = raw[woff[n0] + pos];
            if (n0 + 1 < nwin)
                hi = raw[woff[n0 + 1] + pos];
        }
        *reinterpret_cast<uint32_t*>(dst + rg * Cfg::SBO + ng * 128 + rl * 16 + pair * 4) =
            pack_bf16x2(lo, hi);
    }
}

template <int WS>
__global__ void __launch_bounds__(kDtThreads, 1) wbmm_tc_dt_kernel(const TcDtParams P)
{
    using Cfg = DtCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* raw_base = smem + P.off_raw;
    uint8_t* st_base = smem + P.off_stage;
    float* bins = reinterpret_cast<float*>(smem + P.off_bins);
    int* woff = reinterpret_cast<int*>(smem + P.off_woff);
    DtBars& S = *reinterpret_cast<DtBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDtRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.st_full[i], 4);
            mbar_init(&S.st_empty[i], 1);
        }
        mbar_init(&S.g_full, 1);
        mbar_init(&S.g_empty, 4);
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    for (int n = threadIdx.x; n < Cfg::NT; n += kDtThreads) {
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
            int issued = 0, seq = 0;
            DtWalker it;
            for (it.start(P); it.valid(P); it.next(P), ++seq) {
                const int s = seq % kDtRing;
                if (*abort)
                    break;
                if (seq >= kDtRing && !mbar_wait(&S.raw_empty[s], ((seq / kDtRing) - 1) & 1,
                                                 abort, P.budget, P.status))
                    break;
                const DtTile t = it.get(P);
                const uint32_t bytes = (uint32_t)t.nb * WS * P.W * 2;
                mbar_arrive_expect_tx(&S.raw_full[s], 2 * bytes);
                uint8_t* slot = raw_base + (size_t)s * Cfg::RAW_BYTES;
                dt_runs<WS>(P, t, [&](long long goff, uint32_t soff, uint32_t nbytes) {
                    bulk_g2s(slot + soff, P.dy + goff, nbytes, &S.raw_full[s]);
                    bulk_g2s(slot + Cfg::RAW_HALF + soff, P.x + goff, nbytes, &S.raw_full[s]);
                });
                issued = seq + 1;
            }
            for (int s = 0; s < kDtRing && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / kDtRing) * kDtRing;
                mbar_wait_drain(&S.raw_full[s], (last / kDtRing) & 1, P.budget, P.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int seq = 0, item_seq = 0;
            bool ok_item = true;
            DtWalker it;
            for (it.start(P); it.valid(P); it.next(P), ++seq) {
                const DtTile t = it.get(P);
                const int bs = seq & 1;
                bool ok = !*abort;
                if (t.first && item_seq > 0)
                    ok = ok && mbar_wait(&S.g_empty, (item_seq - 1) & 1, abort, P.budget,
                                         P.status);
                ok = ok && mbar_wait(&S.st_full[bs], (seq >> 1) & 1, abort, P.budget, P.status);
                ok_item = ok;
                if (ok) {
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(st_base + (size_t)bs * Cfg::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
                    for (int mt = 0; mt < Cfg::MT; ++mt) {
#pragma unroll
                        for (int k = 0; k < Cfg::KSTEPS; ++k) {
                            const uint64_t adesc =
                                smem_desc(a_addr + mt * 16 * Cfg::SBO + k * 256, 128, Cfg::SBO);
                            const uint64_t bdesc = smem_desc(b_addr + k * 256, 128, Cfg::SBO);
                            mma_ss(tmem + (uint32_t)(mt * 256), adesc, bdesc, Cfg::IDESC,
                                   (t.first && k == 0) ? 0u : 1u);
                        }
                    }
                    tc_commit(&S.st_empty[bs]);
                }
                if (t.last) {
                    if (ok_item)
                        tc_commit(&S.g_full);
                    ++item_seq;
                }
            }
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------ transform
        const int tw = warp - 2;
        int seq = 0;
        DtWalker it;
        for (it.start(P); it.valid(P); it.next(P), ++seq) {
            const DtTile t = it.get(P);
            const int s = seq % kDtRing, bs = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.raw_full[s], (seq / kDtRing) & 1, abort, P.budget, P.status);
            if (seq >= 2)
                ok = ok && mbar_wait(&S.st_empty[bs], ((seq >> 1) - 1) & 1, abort, P.budget,
                                     P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const uint16_t* raw =
                    reinterpret_cast<const uint16_t*>(raw_base + (size_t)s * Cfg::RAW_BYTES);
                uint8_t* stage = st_base + (size_t)bs * Cfg::STAGE_BYTES;
                const int nwin = t.nb * P.nw;
                dt_transform<WS>(raw, stage, nwin, woff, P.W, tw, lane);
                dt_transform<WS>(raw + Cfg::RAW_HALF / 2, stage + Cfg::A_BYTES, nwin, woff, P.W,
                                 tw, lane);
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (ok && lane == 0) {
                mbar_arrive(&S.st_full[bs]);
                mbar_arrive(&S.raw_empty[s]);
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int ew = warp - 6;
        const int et = threadIdx.x - 6 * 32;
        float* mybins = bins + ew * Cfg::TSZ;
        int item_seq = 0;
        for (long long item = blockIdx.x; item < P.items; item += gridDim.x, ++item_seq) {
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.g_full, item_seq & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            for (int i = lane; i < Cfg::TSZ; i += 32)
                mybins[i] = 0.0f;
            __syncwarp();
            if (ok) {
#pragma unroll 1
                for (int mt = 0; mt < Cfg::MT; ++mt) {
                    const int u = mt * 128 + quarter * 32 + lane;
                    const int p = u / WS, q = u - (u / WS) * WS;
                    const int base = (p + WS - 1) * (2 * WS - 1) + (q + WS - 1);
                    const uint32_t gcol =
                        tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * 256);
#pragma unroll 1
                    for (int c0 = 0; c0 < Cfg::NP; c0 += 32) {
                        uint32_t r[32];
                        tmem_ld32(gcol + (uint32_t)c0, r);
                        tmem_wait_ld(r);
                        // Column v is the same for all lanes: lanes add into
                        // distinct bins; __syncwarp orders columns.
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int v = c0 + jj;
                            if (v < Cfg::D && u < Cfg::D) {
                                const int rr = v / WS, ss = v - (v / WS) * WS;
                                const int bin = base - rr * (2 * WS - 1) - ss;
                                mybins[bin] += __uint_as_float(r[jj]);
                            }
                            __syncwarp();
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.g_empty);
            named_bar_sync(3, 128);
            if (ok) {
                float* out = P.partials + item * Cfg::TSZ;
                for (int i = et; i < Cfg::TSZ; i += 128) {
                    float acc = bins[i];
                    acc += bins[Cfg::TSZ + i];
                    acc += bins[2 * Cfg::TSZ + i];
                    acc += bins[3 * Cfg::TSZ + i];
                    out[i] = acc;
                }
            }
            named_bar_sync(3, 128);
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

struct DtLayout {
    uint32_t off_raw, off_stage, off_bins, off_woff, off_bar, total;
};

template <int WS>
DtLayout dt_layout()
{
    using Cfg = DtCfg<WS>;
    DtLayout L;
    uint32_t off = 0;
    L.off_stage = off;
    off += 2 * Cfg::STAGE_BYTES;
    L.off_raw = align_up(off, 128);
    off = L.off_raw + kDtRing * Cfg::RAW_BYTES;
    L.off_bins = align_up(off, 16);
    off = L.off_bins + 4 * Cfg::TSZ * 4;
    L.off_woff = align_up(off, 16);
    off = L.off_woff + Cfg::NT * 4;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(DtBars);
    L.total = align_up(off, 1024);
    // at least half the SM's shared memory: one CTA (and one 512-column
    // TMEM allocation) per SM
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L;
}

// Tiles per chunk: a fixed function of the shape (never of the grid).
int chunk_tiles(int tpc)
{
    return tpc < 2 ? 1 : 2;
}

template <int WS>
cudaError_t dt_launch_ws(const Geom& g, const void* x, const void* dy, float* partials,
                         const Launch& L)
{
    using Cfg = DtCfg<WS>;
    const DtLayout lay = dt_layout<WS>();
    if (lay.total > kSmemMax)
        return cudaErrorInvalidConfiguration;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(configured & (1ull << (dev & 63)))) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_dt_kernel<WS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)lay.total);
        if (e != cudaSuccess)
            return e;
        configured |= 1ull << (dev & 63);
    }
    TcDtParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.dy = static_cast<const uint16_t*>(dy);
    P.partials = partials;
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = Cfg::NT / g.nw;
    P.bands = g.bands;
    P.tpc = (int)((g.bands + P.bpt - 1) / P.bpt);
    P.ch = chunk_tiles(P.tpc);
    P.chunks = (P.tpc + P.ch - 1) / P.ch;
    P.items = (long long)g.C * P.chunks;
    P.off_raw = lay.off_raw; P.off_stage = lay.off_stage; P.off_bins = lay.off_bins;
    P.off_woff = lay.off_woff; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    long long grid = L.num_sms;
    if (grid > P.items)
        grid = P.items;
    if (grid < 1)
        return cudaSuccess;
    wbmm_tc_dt_kernel<WS><<<(unsigned)grid, kDtThreads, lay.total, L.stream>>>(P);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool tc_dt_supported(const Geom& g)
{
    if (g.w < 2 || g.w > 16)
        return false;
    if (g.nw > 64)
        return false;
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    return true;
}

int tc_dt_chunks(const Geom& g)
{
    const int bpt = 64 / g.nw;
    const int tpc = (int)((g.bands + bpt - 1) / bpt);
    const int ch = chunk_tiles(tpc);
    return (tpc + ch - 1) / ch;
}

cudaError_t tc_dt_launch(const Geom& g, const void* x, const void* dy, float* partials,
                         const Launch& L)
{
    switch (g.w) {
    case 2: return dt_launch_ws<2>(g, x, dy, partials, L);
    case 3: return dt_launch_ws<3>(g, x, dy, partials, L);
    case 4: return dt_launch_ws<4>(g, x, dy, partials, L);
    case 5: return dt_launch_ws<5>(g, x, dy, partials, L);
    case 6: return dt_launch_ws<6>(g, x, dy, partials, L);
    case 7: return dt_launch_ws<7>(g, x, dy, partials, L);
    case 8: return dt_launch_ws<8>(g, x, dy, partials, L);
    case 9: return dt_launch_ws<9>(g, x, dy, partials, L);
    case 10: return dt_launch_ws<10>(g, x, dy, partials, L);
    case 11: return dt_launch_ws<11>(g, x, dy, partials, L);
    case 12: return dt_launch_ws<12>(g, x, dy, partials, L);
    case 13: return dt_launch_ws<13>(g, x, dy, partials, L);
    case 14: return dt_launch_ws<14>(g, x, dy, partials, L);
    case 15: return dt_launch_ws<15>(g, x, dy, partials, L);
    case 16: return dt_launch_ws<16>(g, x, dy, partials, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
