// Tensor-core (tcgen05) WBMM forward and input gradient for large windows
// (w = 28: d = 784), windows as the GEMM's N dimension.
//
// At this size neither a tile of windows nor the matrix M_c fits beside the
// other in one SM, and the MMA is the bound (arithmetic intensity ~d/2 = 392
// FLOP/B, above the ridge), so the kernel is organised around the tensor
// core instead of around HBM:
//
//   D[(p, q), n] = sum_{(r, s)} M_c[(p, q), (r, s)] * X[n, (r, s)]
//
// with output positions padded to 32 slots per window row (u = p*32 + q, M
// tiles of 128 = four output rows) and the K dimension walked one half window
// row (16 slots s) at a time.  M_c depends only on (p - r, q - s), so the A
// operand of M tile m and K step (r, half h) is a row window of one per-
// channel matrix per half,
//
//   Q_h[(delta + w - 1)*32 + q][s'] = T[delta][q - (16h + s') + w - 1],
//
// starting at row 128m + (w - 1 - r)*32: Q (two halves, 110 KB at w = 28) is
// built in shared memory once per channel and only the descriptors' start
// addresses move.  The B operand is 64 windows of one channel (K-major, 16-
// slot K steps), produced four window rows at a time: the producer copies the
// four image rows of every band of the tile with bulk copies, the transform
// rearranges them into the K-major layout (zeros beyond w), and the MMA warp
// runs the 7 x 8 MMAs of the chunk (M = 128, N = 64, K = 16) into a TMEM
// accumulator of 7 x 64 columns.  Each MMA reads its 4 KB A block from shared
// memory, so N = 64 (not 32) keeps the tensor core's operand reads from
// bounding it.  The epilogue reads one output row per warp lane quarter
// (lane = q, 32 registers = 32 windows, two loads) and stores bf16 straight
// to the output map: 28 consecutive elements per warp store.
//
// Warp roles (576 threads):
//   warp 0       producer: bulk copies of four-row chunks into a raw ring
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warps 2..9   transform: raw chunk -> B chunk (thread = window, row);
//                after a tile's chunks, half of the accumulator drain
//   warps 10..17 epilogue, and Q for each channel (after the channel's last
//                accumulator is complete, so no MMA still reads the old Q)
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "wbmm_internal.h"

namespace wbmm {

template <int WS>
struct BigCfg {
    static constexpr int RP = 32;                            // slots per window row
    static constexpr int L = 2 * WS - 1;
    static constexpr int TSZ = L * L;
    static constexpr int MT = (WS * RP + 127) / 128;         // 128-row M tiles
    static constexpr int NW = 64;                            // windows per tile (MMA N)
    static constexpr int CR = 4;                             // window rows per chunk
    static constexpr int NCH = (WS + CR - 1) / CR;           // chunks per tile
    static constexpr int KCH = CR * 2;                       // K steps per chunk
    static constexpr int QROWS = (WS - 1) * RP + MT * 128;   // rows of each Q half
    static constexpr uint32_t QH_BYTES = (uint32_t)QROWS * 32;
    static constexpr uint32_t KSTEP_BYTES = (NW / 8) * 256;  // one K step of B
    static constexpr uint32_t BCH_BYTES = KCH * KSTEP_BYTES; // one chunk of B
    static constexpr uint32_t IDESC = idesc_bf16(128, NW);
    static_assert(MT * NW <= 512, "the accumulator fits in TMEM");
    static_assert(QROWS % 8 == 0 && ((WS - 1) * RP) % 8 == 0, "Q rows in whole core matrices");
};

constexpr int kBigRawRing = 8;
constexpr int kBigBRing = 3;
constexpr int kBigXformWarp0 = 2;
constexpr int kBigXformWarps = 8;
constexpr int kBigEpiWarp0 = kBigXformWarp0 + kBigXformWarps;
constexpr int kBigEpiWarps = 8;
constexpr int kBigThreads = (kBigEpiWarp0 + kBigEpiWarps) * 32;
// warps that drain the accumulator: the epilogue's and the transform's
constexpr int kBigEpilogueThreads = (kBigEpiWarps + kBigXformWarps) * 32;

struct TcBigParams {
    const uint16_t* x;      // bf16 bits, [B][C][H][W]
    const uint16_t* T;      // bf16 table [C][(2w-1)^2]
    uint16_t* y;
    int C, H, W, nh, nw;
    int bpt;                // bands per tile
    int tpc;                // tiles per channel
    int bands;              // bands per channel
    int items;              // C * tpc
    int R;                  // raw ring depth (chunks)
    uint32_t raw_bytes;     // raw chunk slot stride
    uint32_t off_q, off_b, off_raw, off_tst, off_wb, off_bar;
    unsigned long long budget;
    int* status;
};

struct BigBars {
    uint64_t raw_full[kBigRawRing];
    uint64_t raw_empty[kBigRawRing];
    uint64_t b_full[kBigBRing];
    uint64_t b_empty[kBigBRing];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t q_full;
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

__device__ __forceinline__ BandTile big_tile(const TcBigParams& P, int it)
{
    BandTile t;
    t.c = it / P.tpc;
    t.band0 = (it - t.c * P.tpc) * P.bpt;
    const int left = P.bands - t.band0;
    t.nb = left < P.bpt ? left : P.bpt;
    return t;
}

// Global element offset of image row `row` (0 .. w-1) of band g of channel c.
__device__ __forceinline__ long long big_row_offset(const TcBigParams& P, int WS, int c, int g,
                                                    int row)
{
    const int b = g / P.nh, i = g - (g / P.nh) * P.nh;
    return (((long long)b * P.C + c) * P.H + (long long)i * WS + row) * P.W;
}

// Q for one channel from its staged table (K-major, 8-row groups of 256
// bytes, the two 8-slot core matrices of a row 128 bytes apart).  One thread
// per (half, row, 8-slot core).
template <int WS>
__device__ __forceinline__ void big_build_q(uint8_t* q, const uint16_t* tst, int tid, int nthreads)
{
    using F = BigCfg<WS>;
    for (int item = tid; item < 2 * F::QROWS * 2; item += nthreads) {
        const int h = item / (F::QROWS * 2);
        const int rem = item - h * (F::QROWS * 2);
        const int rho = rem >> 1, core = rem & 1;
        const int dl = rho / F::RP;                    // delta + w - 1
        const int qq = rho - dl * F::RP;
        uint32_t wv[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint16_t v2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int s = 16 * h + 8 * core + 2 * m + e;
                uint16_t v = 0;
                if (qq < WS && s < WS && dl < F::L)
                    v = tst[dl * F::L + (qq - s + WS - 1)];
                v2[e] = v;
            }
            wv[m] = pack_bf16x2(v2[0], v2[1]);
        }
        *reinterpret_cast<uint4*>(q + (size_t)h * F::QH_BYTES + (rho >> 3) * 256 + core * 128 +
                                  (rho & 7) * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

// Windows 16*idx .. 16*idx+15 of the tile, every output row of the warp's
// lane quarter: in M tile m the quarter holds output row p = 4m + quarter,
// lane q its column, and accumulator columns m*NW + n are window n (wb: the
// windows' output bases, read once).  Stores bf16 straight to y, 28
// consecutive elements per warp store.
template <int WS>
__device__ __forceinline__ void big_drain(const TcBigParams& P, uint32_t tmem, int quarter,
                                          int lane, int idx, int nwin, const long long* wb)
{
    using F = BigCfg<WS>;
    const int n0 = 16 * idx;
    if (n0 >= nwin)
        return;
    long long base[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        base[i] = wb[n0 + i] + lane;
#pragma unroll 1
    for (int m = 0; m < F::MT; ++m) {
        const int p = 4 * m + quarter;
        if (p >= WS)
            break;
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(m * F::NW + n0), r);
        tmem_wait_ld(r);
        if (lane >= WS)
            continue;
        const long long off = (long long)p * P.W;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (n0 + i < nwin)
                P.y[base[i] + off] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[i])));
    }
}

template <int WS, int MODE>
__global__ void __launch_bounds__(kBigThreads, 1)
    wbmm_tc_big_kernel(const __grid_constant__ TcBigParams P)
{
    using F = BigCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* q_base = smem + P.off_q;
    uint8_t* b_base = smem + P.off_b;
    uint8_t* raw_base = smem + P.off_raw;
    uint16_t* tst = reinterpret_cast<uint16_t*>(smem + P.off_tst);
    long long* wbase = reinterpret_cast<long long*>(smem + P.off_wb);   // [2][NW]
    BigBars& S = *reinterpret_cast<BigBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R;

    const int qn = P.items / (int)gridDim.x, rem = P.items % (int)gridDim.x;
    const int it0 = (int)blockIdx.x * qn + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem);
    const int n_it = qn + ((int)blockIdx.x < rem ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kBigRawRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], kBigXformWarps);
        }
        for (int i = 0; i < kBigBRing; ++i) {
            mbar_init(&S.b_full[i], kBigXformWarps);
            mbar_init(&S.b_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.acc_full[i], 1);
            mbar_init(&S.acc_empty[i], kBigEpiWarps + kBigXformWarps);
        }
        mbar_init(&S.q_full, kBigEpiWarps);
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_slot;
    grid_dep_wait();
    grid_dep_launch();

    if (warp == 0) {
        // ------------------------------------------------------ producer
        // Chunk ch of tile seq: image rows 4ch .. 4ch+3 of each band of the
        // tile, band k at slot offset k*CR*W (rows past w are not copied).
        int issued = 0;
        bool go = true;
        for (int seq = 0; seq < n_it && go; ++seq) {
            const BandTile t = big_tile(P, it0 + seq);
            for (int ch = 0; ch < F::NCH; ++ch) {
                const int ss = seq * F::NCH + ch, s = ss % R;
                bool ok = !*abort;
                if (ss >= R)
                    ok = ok && mbar_wait(&S.raw_empty[s], ((ss / R) - 1) & 1, abort, P.budget,
                                         P.status);
                if (!__all_sync(0xffffffffu, ok)) {
                    go = false;
                    break;
                }
                const int r0 = ch * F::CR;
                const int nr = (WS - r0) < F::CR ? (WS - r0) : F::CR;
                const uint32_t bytes = (uint32_t)nr * P.W * 2;
                uint8_t* slot = raw_base + (size_t)s * P.raw_bytes;
                if (lane == 0)
                    mbar_arrive_expect_tx(&S.raw_full[s], bytes * (uint32_t)t.nb);
                __syncwarp();
                for (int k = lane; k < t.nb; k += 32)
                    bulk_g2s(slot + (size_t)k * F::CR * P.W * 2,
                             P.x + big_row_offset(P, WS, t.c, t.band0 + k, r0), bytes,
                             &S.raw_full[s]);
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
                const BandTile t = big_tile(P, it0 + seq);
                const bool first = t.c != cur_c;
                if (first) {
                    cur_c = t.c;
                    ++ci;
                }
                bool ok = !*abort;
                if (first)
                    ok = ok && mbar_wait(&S.q_full, ci & 1, abort, P.budget, P.status);
                if (seq >= 1)
                    ok = ok && mbar_wait(&S.acc_empty[0], (seq - 1) & 1, abort, P.budget,
                                         P.status);
                const uint32_t q0 = smem_u32(q_base);
                const uint32_t d0 = tmem;
                for (int ch = 0; ch < F::NCH; ++ch) {
                    const int ss = seq * F::NCH + ch, bs = ss % kBigBRing;
                    ok = ok && mbar_wait(&S.b_full[bs], (ss / kBigBRing) & 1, abort, P.budget,
                                         P.status);
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t bch = smem_u32(b_base + (size_t)bs * F::BCH_BYTES);
#pragma unroll 1
                    for (int kk = 0; kk < F::KCH; ++kk) {
                        const int r = ch * F::CR + (kk >> 1), h = kk & 1;
                        if (r >= WS)
                            break;
                        const uint64_t bdesc =
                            smem_desc(bch + (uint32_t)kk * F::KSTEP_BYTES, 128, 256);
                        const uint32_t qh = q0 + (uint32_t)h * F::QH_BYTES +
                                            (uint32_t)((WS - 1 - r) * F::RP / 8) * 256;
#pragma unroll
                        for (int m = 0; m < F::MT; ++m) {
                            const uint64_t adesc = smem_desc(qh + (uint32_t)m * 16 * 256, 128, 256);
                            mma_ss(d0 + (uint32_t)(m * F::NW), adesc, bdesc, F::IDESC,
                                   (ch > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(&S.b_empty[bs]);
                }
                if (ok)
                    tc_commit(&S.acc_full[0]);
            }
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp < kBigEpiWarp0) {
        // ------------------------------------------------------ transform
        // Thread = (window n, chunk row rr): the window's 16-slot halves of
        // that row as two pairs of 16-byte core-matrix rows (zeros past w and
        // for windows past the tile's last band).
        const int tid = threadIdx.x - kBigXformWarp0 * 32;
        const int n = tid % F::NW, rr = tid / F::NW;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = big_tile(P, it0 + seq);
            const int nwin = t.nb * P.nw;
            const int k = n / P.nw, j = n - (n / P.nw) * P.nw;
            for (int ch = 0; ch < F::NCH; ++ch) {
                const int ss = seq * F::NCH + ch, s = ss % R, bs = ss % kBigBRing;
                bool ok = !*abort;
                ok = ok && mbar_wait(&S.raw_full[s], (ss / R) & 1, abort, P.budget, P.status);
                if (ss >= kBigBRing)
                    ok = ok && mbar_wait(&S.b_empty[bs], ((ss / kBigBRing) - 1) & 1, abort,
                                         P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                if (ok) {
                    const int r = ch * F::CR + rr;
                    const bool valid = n < nwin && r < WS;
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(
                        raw_base + (size_t)s * P.raw_bytes +
                        ((size_t)(k * F::CR + rr) * P.W + (size_t)j * WS) * 2);
                    uint32_t wv[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        wv[m] = (valid && 2 * m < WS) ? src[m] : 0u;
                    uint8_t* bch = b_base + (size_t)bs * F::BCH_BYTES;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int core = 0; core < 2; ++core) {
                            const int w0 = 8 * h + 4 * core;
                            *reinterpret_cast<uint4*>(
                                bch + (size_t)(rr * 2 + h) * F::KSTEP_BYTES + (n >> 3) * 256 +
                                core * 128 + (n & 7) * 16) =
                                make_uint4(wv[w0], wv[w0 + 1], wv[w0 + 2], wv[w0 + 3]);
                        }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (ok && lane == 0) {
                    mbar_arrive(&S.b_full[bs]);
                    mbar_arrive(&S.raw_empty[s]);
                }
            }
            // then take two of the four warps per lane quarter that drain
            // this tile's accumulator (windows 32 .. 63; the MMAs of the next
            // tile wait for it)
            named_bar_sync(3, kBigEpilogueThreads);       // window bases written
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.acc_full[0], seq & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok)
                big_drain<WS>(P, tmem, warp & 3, lane, 2 + ((warp - kBigXformWarp0) >> 2), nwin,
                              wbase + (seq & 1) * F::NW);
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.acc_empty[0]);
        }
    } else {
        // ------------------------------------------------------ epilogue
        // Two warps per TMEM lane quarter, with the transform's two: warp
        // half hf drains windows 16hf .. 16hf+15 (big_drain).
        const int quarter = warp & 3;
        const int hf = (warp - kBigEpiWarp0) >> 2;
        const int et = threadIdx.x - kBigEpiWarp0 * 32;
        constexpr int EPT = kBigEpiWarps * 32;
        const int c_first = big_tile(P, it0).c;
        // Q of channel c.  Every epilogue warp takes part whatever its wait
        // results, so the named barriers always see all of them.
        auto build_for = [&](int c) {
            named_bar_sync(2, EPT);                       // staged table fully read
            const unsigned short* src = reinterpret_cast<const unsigned short*>(P.T) +
                                        (long long)c * F::TSZ;
            for (int e = et; e < F::TSZ; e += EPT)
                tst[MODE == kTable ? e : F::TSZ - 1 - e] = __ldg(src + e);
            named_bar_sync(2, EPT);
            big_build_q<WS>(q_base, tst, et, EPT);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&S.q_full);
        };
        if (n_it > 0)
            build_for(c_first);
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = big_tile(P, it0 + seq);
            const int nwin = t.nb * P.nw;
            const int a = seq & 1;          // window-base buffer
            // output base of each window of the tile (row 0, column 0)
            if (et < F::NW) {
                long long v = 0;
                if (et < nwin) {
                    const int k = et / P.nw, j = et - (et / P.nw) * P.nw;
                    v = big_row_offset(P, WS, t.c, t.band0 + k, 0) + (long long)j * WS;
                }
                wbase[a * F::NW + et] = v;
            }
            named_bar_sync(3, kBigEpilogueThreads);
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.acc_full[0], seq & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok)
                big_drain<WS>(P, tmem, quarter, lane, hf, nwin, wbase + a * F::NW);
            tc_fence_before();
            __syncwarp();
            if (ok && lane == 0)
                mbar_arrive(&S.acc_empty[0]);
            // the channel's last tile is complete (acc_full): no MMA reads Q
            if (seq + 1 < n_it && big_tile(P, it0 + seq + 1).c != t.c)
                build_for(big_tile(P, it0 + seq + 1).c);
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

inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

struct BigLayout {
    uint32_t off_q, off_b, off_raw, off_tst, off_wb, off_bar, total, raw_bytes;
    int R, bpt;
};

// Q (two halves) | B ring | table | window bases | barriers | raw ring.
template <int WS>
bool big_layout(const Geom& g, BigLayout& L)
{
    using F = BigCfg<WS>;
    if (g.nw < 1 || g.nw > F::NW)
        return false;
    L.bpt = F::NW / g.nw;
    L.raw_bytes = align_up((uint32_t)L.bpt * F::CR * g.W * 2, 128);
    uint32_t off = 0;
    L.off_q = off;
    off += 2 * F::QH_BYTES;
    L.off_b = align_up(off, 1024);
    off = L.off_b + kBigBRing * F::BCH_BYTES;
    L.off_tst = align_up(off, 16);
    off = L.off_tst + (uint32_t)F::TSZ * 2;
    L.off_wb = align_up(off, 16);
    off = L.off_wb + 2 * F::NW * 8;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(BigBars);
    L.off_raw = align_up(off, 128);
    const uint32_t avail = kSmemMax - 1024 > L.off_raw ? kSmemMax - 1024 - L.off_raw : 0;
    int R = (int)(avail / L.raw_bytes);
    if (R > kBigRawRing)
        R = kBigRawRing;
    L.R = R;
    if (R < 2)
        return false;
    L.total = align_up(L.off_raw + (uint32_t)R * L.raw_bytes, 1024);
    return L.total <= kSmemMax;
}

template <int WS, int MODE>
cudaError_t big_launch_ws(const Geom& g, const void* x, const void* T, void* y, const Launch& L)
{
    BigLayout lay;
    if (!big_layout<WS>(g, lay))
        return cudaErrorInvalidConfiguration;
    static bool configured[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_big_kernel<WS, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMax);
        if (e != cudaSuccess)
            return e;
        configured[dev & 63] = true;
    }
    TcBigParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.T = static_cast<const uint16_t*>(T);
    P.y = static_cast<uint16_t*>(y);
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = lay.bpt;
    P.bands = (int)g.bands;
    P.tpc = (P.bands + P.bpt - 1) / P.bpt;
    P.items = g.C * P.tpc;
    P.R = lay.R;
    P.raw_bytes = lay.raw_bytes;
    P.off_q = lay.off_q; P.off_b = lay.off_b; P.off_raw = lay.off_raw;
    P.off_tst = lay.off_tst; P.off_wb = lay.off_wb; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    int grid = L.num_sms;
    if (grid > P.items)
        grid = P.items;
    if (grid < 1)
        return cudaSuccess;
    cudaError_t e = launch_pdl(wbmm_tc_big_kernel<WS, MODE>, dim3(grid), dim3(kBigThreads),
                               lay.total, L.stream, P);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool tc_big_supported(const Geom& g)
{
    if (g.w != 28)
        return false;
    // bulk copies of whole image rows: 16-byte aligned starts and sizes
    if (g.W % 8 != 0)
        return false;
    if (g.bands * (long long)g.C >= (1ll << 31))
        return false;
    BigLayout lay;
    return big_layout<28>(g, lay);
}

cudaError_t tc_big_launch(const Geom& g, AMode mode, const void* x, const void* T, void* y,
                          const Launch& L)
{
    if (g.w != 28 || mode == kCached)
        return cudaErrorInvalidValue;
    if (mode == kTable)
        return big_launch_ws<28, kTable>(g, x, T, y, L);
    return big_launch_ws<28, kTableFlip>(g, x, T, y, L);
}

}  // namespace wbmm
