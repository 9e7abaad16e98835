// Tensor-core (tcgen05) WBMM forward and input gradient for large windows
// (w = 28: d = 784).
//
// At this size neither a tile of windows nor the matrix M_c fits beside the
// other in one SM, and the MMA is the bound (arithmetic intensity ~d/2 = 392
// FLOP/B, above the ridge), so the kernel is organised around the tensor
// core instead of around HBM:
//
//   D[n, (p, q)] = sum_{(r, s)} X[n, (r, s)] * M_c[(p, q), (r, s)]
//
// with the tile's 128 windows as the MMA's M dimension, held as the A
// operand in tensor memory (lane = window, one 32-bit column per pair of the
// 32 K slots of a window row: 448 columns), and output positions as N, two
// output rows (64 slots, u = p*32 + q) per MMA.  M_c depends only on
// (p - r, q - s), so the B operand of output rows 2m, 2m+1 and K step (input
// row r, half h) is a 64-row window of one per-channel matrix per half,
//
//   Q_h[(delta + w - 1)*32 + q][s'] = T[delta][q - (16h + s') + w - 1],
//
// starting at row 64m + (w - 1 - r)*32: Q (two halves, 110 KB at w = 28) is
// built in shared memory once per channel and only the descriptors' start
// addresses move.  Per MMA only the 2 KB B block comes from shared memory.
// (An earlier kernel with the table as A, M = output positions, and 64
// windows as N read a 4 KB A block and a 2 KB window block per MMA of the
// same size and kept its 7 x 64-column accumulator until a tile's epilogue
// had drained it: 308 us on the 112 x 112 sweep against 271 us here.)
//
// The 64 remaining TMEM columns hold one accumulator (N = 64): the epilogue
// warps read one output row per warp half into registers, release the
// accumulator for the next chunk's MMAs, then convert and store.  A is
// written four window rows at a time as the raw chunks arrive; per chunk an
// mbarrier hands those rows to the MMAs (which start the first output chunk
// at once) and another, committed after the tile's last output chunk has
// read those rows, hands them back to the transform of the next tile.
//
// Warp roles (576 threads):
//   warp 0       producer: bulk copies of four-row chunks into a raw ring
//   warp 1       MMA issuer (one thread) and TMEM owner
//   warps 2..9   transform: two per TMEM lane quarter (thread = window), each
//                two of the chunk's four window rows -> A columns
//   warps 10..17 epilogue: accumulator -> bf16 -> y (one output row per
//                warp half); Q for each channel after its last chunk
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "wbmm_internal.h"

namespace wbmm {

// The per-channel Toeplitz stack Q (two halves of 16 K slots each): rows
// (delta + w - 1)*32 + q, enough of them for every output chunk's window.
template <int WS>
struct BigCfg {
    static constexpr int RP = 32;                            // slots per window row
    static constexpr int L = 2 * WS - 1;
    static constexpr int TSZ = L * L;
    static constexpr int MT = (WS * RP + 127) / 128;         // 128-row groups of positions
    static constexpr int QROWS = (WS - 1) * RP + MT * 128;   // rows of each Q half
    static constexpr uint32_t QH_BYTES = (uint32_t)QROWS * 32;
    static_assert(QROWS % 8 == 0 && ((WS - 1) * RP) % 8 == 0, "Q rows in whole core matrices");
};

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
    uint32_t band_bytes;    // stride of a band's rows in a raw slot (padded)
    uint32_t off_q, off_raw, off_bar;
    unsigned long long budget;
    int* status;
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

// Q for one channel from its table Tc in global memory, read reversed for
// dX (flip) (K-major, 8-row groups of 256 bytes, the two 8-slot core
// matrices of a row 128 bytes apart).  One thread per (half, row, 8-slot
// core).
template <int WS>
__device__ __forceinline__ void big_build_q(uint8_t* q, const uint16_t* Tc, bool flip, int tid,
                                            int nthreads)
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
                if (qq < WS && s < WS && dl < F::L) {
                    const int e = dl * F::L + (qq - s + WS - 1);
                    v = __ldg(reinterpret_cast<const unsigned short*>(Tc) +
                              (flip ? F::TSZ - 1 - e : e));
                }
                v2[e] = v;
            }
            wv[m] = pack_bf16x2(v2[0], v2[1]);
        }
        *reinterpret_cast<uint4*>(q + (size_t)h * F::QH_BYTES + (rho >> 3) * 256 + core * 128 +
                                  (rho & 7) * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

template <int WS>
struct BigWmCfg {
    static constexpr int RP = 32;                            // K slots per window row
    static constexpr int L = 2 * WS - 1;
    static constexpr int TSZ = L * L;
    static constexpr int NT = 128;                           // windows per tile (MMA M)
    static constexpr int ACOLS = WS * RP / 2;                // TMEM columns of A
    static constexpr int NCH = (WS + 1) / 2;                 // output chunks of two rows
    static constexpr int CR = 4;                             // window rows per raw chunk
    static constexpr int NRC = (WS + CR - 1) / CR;           // raw chunks per tile
    static constexpr uint32_t IDESC = idesc_bf16(128, 64);
    static_assert(ACOLS + 64 <= 512, "A and one accumulator fit in TMEM");
    static_assert(NRC <= 8, "per-chunk barriers");
    // B rows 64m + (w-1-r)*32 .. +64 stay inside the Q stack of the table-as-A
    // kernel (QROWS = (w-1)*32 + MT*128 rows)
    static_assert(64 * NCH <= BigCfg<WS>::MT * 128, "Q covers every output chunk");
};

__device__ __forceinline__ uint32_t wm_bf16x2(uint32_t lo, uint32_t hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
    return *reinterpret_cast<const uint32_t*>(&v);
}

constexpr int kWmRawRing = 8;
constexpr int kWmXformWarp0 = 2;
constexpr int kWmXformWarps = 8;
constexpr int kWmEpiWarp0 = kWmXformWarp0 + kWmXformWarps;
constexpr int kWmEpiWarps = 8;
constexpr int kWmThreads = (kWmEpiWarp0 + kWmEpiWarps) * 32;

struct WmBars {
    uint64_t raw_full[kWmRawRing];
    uint64_t raw_empty[kWmRawRing];
    uint64_t a_full[8];     // per raw chunk: its window rows are in TMEM
    uint64_t a_empty[8];    // per raw chunk: the tile's MMAs are done with them
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t q_full;
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
};

template <int WS, int MODE>
__global__ void __launch_bounds__(kWmThreads, 1)
    wbmm_tc_bigwm_kernel(const __grid_constant__ TcBigParams P)
{
    using F = BigWmCfg<WS>;
    using Q = BigCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* q_base = smem + P.off_q;
    uint8_t* raw_base = smem + P.off_raw;
    WmBars& S = *reinterpret_cast<WmBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R;

    const int qn = P.items / (int)gridDim.x, rem = P.items % (int)gridDim.x;
    const int it0 = (int)blockIdx.x * qn + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem);
    const int n_it = qn + ((int)blockIdx.x < rem ? 1 : 0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWmRawRing; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], kWmXformWarps);
        }
        for (int i = 0; i < 8; ++i) {
            mbar_init(&S.a_full[i], kWmXformWarps);
            mbar_init(&S.a_empty[i], 1);
        }
        mbar_init(&S.acc_full, 1);
        mbar_init(&S.acc_empty, kWmEpiWarps);
        mbar_init(&S.q_full, kWmEpiWarps);
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
        // tile, band k at slot offset k*band_bytes (rows past w are not
        // copied).
        int issued = 0;
        bool go = true;
        for (int seq = 0; seq < n_it && go; ++seq) {
            const BandTile t = big_tile(P, it0 + seq);
            for (int ch = 0; ch < F::NRC; ++ch) {
                const int ss = seq * F::NRC + ch, s = ss % R;
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
                    bulk_g2s(slot + (size_t)k * P.band_bytes,
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
        // Output chunk m of tile seq: K steps (r, h) in order; the first
        // chunk of a tile waits for each raw chunk's rows, the last one hands
        // each raw chunk's rows back once its MMAs have completed.
        if (lane == 0) {
            int cur_c = -1, ci = -1, gc = 0;
            const uint32_t q0 = smem_u32(q_base);
            bool ok = true;
            for (int seq = 0; seq < n_it && ok; ++seq) {
                const BandTile t = big_tile(P, it0 + seq);
                ok = !*abort;
                if (t.c != cur_c) {
                    cur_c = t.c;
                    ++ci;
                    ok = ok && mbar_wait(&S.q_full, ci & 1, abort, P.budget, P.status);
                }
                for (int m = 0; m < F::NCH && ok; ++m, ++gc) {
                    if (gc >= 1)
                        ok = ok && mbar_wait(&S.acc_empty, (gc - 1) & 1, abort, P.budget, P.status);
                    for (int ch = 0; ch < F::NRC && ok; ++ch) {
                        if (m == 0)
                            ok = ok && mbar_wait(&S.a_full[ch], seq & 1, abort, P.budget,
                                                 P.status);
                        if (!ok)
                            break;
                        tc_fence_after();
                        // K steps (4ch + rr, h): the B window moves back 32 Q
                        // rows (64 descriptor units of 16 bytes) per input row
                        // and to the other Q half with h; A moves 16 columns
                        // per row and 8 per half: compile-time offsets from
                        // the chunk's first step.
                        const uint64_t bd0 = smem_desc(
                            q0 + (uint32_t)(8 * m + 4 * (WS - 1 - ch * F::CR)) * 256, 128, 256);
                        const uint32_t a0 = tmem + (uint32_t)(16 * ch * F::CR);
                        const uint32_t d = tmem + (uint32_t)F::ACOLS;
                        if (ch * F::CR + F::CR <= WS) {
                            mma_ts(d, a0, bd0, F::IDESC, ch > 0 ? 1u : 0u);
#pragma unroll
                            for (int kk = 1; kk < 2 * F::CR; ++kk) {
                                const int rr = kk >> 1, h = kk & 1;
                                mma_ts(d, a0 + (uint32_t)(16 * rr + 8 * h),
                                       bd0 - (uint64_t)(rr * 64) +
                                           (uint64_t)(h * (Q::QH_BYTES >> 4)),
                                       F::IDESC, 1u);
                            }
                        } else {
                            for (int kk = 0; kk < 2 * (WS - ch * F::CR); ++kk) {
                                const int rr = kk >> 1, h = kk & 1;
                                mma_ts(d, a0 + (uint32_t)(16 * rr + 8 * h),
                                       bd0 - (uint64_t)(rr * 64) +
                                           (uint64_t)(h * (Q::QH_BYTES >> 4)),
                                       F::IDESC, (ch > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        if (m == F::NCH - 1)
                            tc_commit(&S.a_empty[ch]);
                    }
                    if (ok)
                        tc_commit(&S.acc_full);
                }
            }
            // Drain: all issued MMAs complete before TMEM is released.
            tc_commit(&S.fin);
            mbar_wait_drain(&S.fin, 0, P.budget, P.status);
        }
    } else if (warp < kWmEpiWarp0) {
        // ------------------------------------------------------ transform
        // Thread = window n of the warp's lane quarter; warp part `part`
        // writes window rows 2part, 2part+1 of each raw chunk: 32 K slots per
        // row (zeros past w and for windows past the tile's last band) as
        // 16 columns.
        const int quarter = warp & 3;
        const int part = (warp - kWmXformWarp0) >> 2;
        const int n = quarter * 32 + lane;
        const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = big_tile(P, it0 + seq);
            const bool valid = n < t.nb * P.nw;
            const int k = n / P.nw, j = n - (n / P.nw) * P.nw;
            for (int ch = 0; ch < F::NRC; ++ch) {
                const int ss = seq * F::NRC + ch, s = ss % R;
                bool ok = !*abort;
                if (seq >= 1)
                    ok = ok && mbar_wait(&S.a_empty[ch], (seq - 1) & 1, abort, P.budget,
                                         P.status);
                ok = ok && mbar_wait(&S.raw_full[s], (ss / R) & 1, abort, P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();
                if (ok) {
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int rl = 2 * part + rr;
                        const int r = ch * F::CR + rl;
                        if (r >= WS)
                            break;
                        uint32_t lo[8], hi[8];
                        const uint32_t* src = reinterpret_cast<const uint32_t*>(
                            raw_base + (size_t)s * P.raw_bytes + (size_t)k * P.band_bytes +
                            ((size_t)rl * P.W + (size_t)j * WS) * 2);
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            lo[m] = (valid && 2 * m < WS) ? src[m] : 0u;
                            hi[m] = (valid && 2 * (m + 8) < WS) ? src[m + 8] : 0u;
                        }
                        tmem_st8(tmem + lanebase + (uint32_t)(16 * r), lo);
                        tmem_st8(tmem + lanebase + (uint32_t)(16 * r + 8), hi);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0) {
                    mbar_arrive(&S.raw_empty[s]);
                    mbar_arrive(&S.a_full[ch]);
                }
            }
        }
    } else {
        // ------------------------------------------------------ epilogue
        // Warp half hf drains output row 2m + hf of every window of its lane
        // quarter (lane = window, 32 columns = the row's slots) and stores
        // its w bf16 values, 8 bytes at a time.
        static_assert(WS % 4 == 0, "output rows in whole 8-byte stores");
        const int quarter = warp & 3;
        const int hf = (warp - kWmEpiWarp0) >> 2;
        const int et = threadIdx.x - kWmEpiWarp0 * 32;
        constexpr int EPT = kWmEpiWarps * 32;
        const int n = quarter * 32 + lane;
        const uint32_t lanebase = (uint32_t)(quarter * 32) << 16;
        // Q of channel c, built by all epilogue warps; each arrives on q_full.
        auto build_for = [&](int c) {
            big_build_q<WS>(q_base, P.T + (long long)c * F::TSZ, MODE != kTable, et, EPT);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&S.q_full);
        };
        if (n_it > 0)
            build_for(big_tile(P, it0).c);
        int gc = 0;
        for (int seq = 0; seq < n_it; ++seq) {
            const BandTile t = big_tile(P, it0 + seq);
            const bool valid = n < t.nb * P.nw;
            long long base = 0;
            if (valid) {
                const int k = n / P.nw, j = n - (n / P.nw) * P.nw;
                base = big_row_offset(P, WS, t.c, t.band0 + k, 0) + (long long)j * WS;
            }
            for (int m = 0; m < F::NCH; ++m, ++gc) {
                bool ok = !*abort;
                ok = ok && mbar_wait(&S.acc_full, gc & 1, abort, P.budget, P.status);
                ok = __all_sync(0xffffffffu, ok);
                tc_fence_after();
                const int p = 2 * m + hf;
                uint32_t r[32];
                if (ok) {
                    tmem_ld32(tmem + lanebase + (uint32_t)(F::ACOLS + 32 * hf), r);
                    tmem_wait_ld(r);
                }
                // the row is in registers: the next chunk's MMAs may start
                tc_fence_before();
                __syncwarp();
                if (ok && lane == 0)
                    mbar_arrive(&S.acc_empty);
                if (ok && valid && p < WS) {
                    uint2* dst = reinterpret_cast<uint2*>(P.y + base + (long long)p * P.W);
#pragma unroll
                    for (int i = 0; i < WS / 4; ++i)
                        dst[i] = make_uint2(wm_bf16x2(r[4 * i], r[4 * i + 1]),
                                            wm_bf16x2(r[4 * i + 2], r[4 * i + 3]));
                }
            }
            // the channel's last chunk is complete (acc_full): no MMA reads Q
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

struct BigWmLayout {
    uint32_t off_q, off_bar, off_raw, total, raw_bytes, band_bytes;
    int R, bpt;
};

// Q (two halves) | barriers | raw ring.
template <int WS>
bool bigwm_layout(const Geom& g, BigWmLayout& L)
{
    using F = BigWmCfg<WS>;
    using Q = BigCfg<WS>;
    if (g.nw < 1 || g.nw > F::NT)
        return false;
    L.bpt = F::NT / g.nw;
    // A band's four rows (4*W*2 bytes, a multiple of 64) plus 16 bytes: the
    // transform's threads (one window each, several bands per warp) then
    // read shared memory with 2-way instead of 8-way bank conflicts.
    L.band_bytes = (uint32_t)F::CR * g.W * 2 + 16;
    L.raw_bytes = (uint32_t)L.bpt * L.band_bytes;
    L.raw_bytes = (L.raw_bytes + 127) / 128 * 128;
    uint32_t off = 0;
    L.off_q = off;
    off += 2 * Q::QH_BYTES;
    L.off_bar = (off + 15) / 16 * 16;
    off = L.off_bar + sizeof(WmBars);
    L.off_raw = (off + 127) / 128 * 128;
    const uint32_t smax = 232448;
    const uint32_t avail = smax > L.off_raw ? smax - L.off_raw : 0;
    int R = (int)(avail / L.raw_bytes);
    if (R > kWmRawRing)
        R = kWmRawRing;
    L.R = R;
    if (R < 2)
        return false;
    L.total = L.off_raw + (uint32_t)R * L.raw_bytes;
    return L.total <= smax;
}

template <int WS, int MODE>
cudaError_t bigwm_launch_ws(const Geom& g, const void* x, const void* T, void* y, const Launch& L)
{
    BigWmLayout lay;
    if (!bigwm_layout<WS>(g, lay))
        return cudaErrorInvalidConfiguration;
    static bool configured[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_bigwm_kernel<WS, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
        if (e != cudaSuccess)
            return e;
        configured[dev & 63] = true;
    }
    TcBigParams P{};
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
    P.band_bytes = lay.band_bytes;
    P.off_q = lay.off_q; P.off_raw = lay.off_raw; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    int grid = L.num_sms;
    if (grid > P.items)
        grid = P.items;
    if (grid < 1)
        return cudaSuccess;
    cudaError_t e = launch_pdl(wbmm_tc_bigwm_kernel<WS, MODE>, dim3(grid), dim3(kWmThreads),
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
    BigWmLayout wm;
    return bigwm_layout<28>(g, wm);
}

cudaError_t tc_big_launch(const Geom& g, AMode mode, const void* x, const void* T, void* y,
                          const Launch& L)
{
    if (g.w != 28 || mode == kCached)
        return cudaErrorInvalidValue;
    return mode == kTable ? bigwm_launch_ws<28, kTable>(g, x, T, y, L)
                          : bigwm_launch_ws<28, kTableFlip>(g, x, T, y, L);
}

}  // namespace wbmm
