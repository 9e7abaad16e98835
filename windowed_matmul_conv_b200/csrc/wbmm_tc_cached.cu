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
// Fused 3x3 mixing (FUSE, the inter-block depthwise step that follows the
// cached forward): the CTA ranges are whole image planes; after each tile's
// drain the transform and epilogue warps (16 workers) apply the 3x3 to the
// bf16 y rows in the staging buffer, carrying the two rows at a tile edge
// inside a plane to the next tile, and store z from registers; the storer
// idles and y never reaches HBM.  Bit-identical to the cached forward
// followed by the standalone 3x3 kernel.
//
// TMEM: A stages at columns 0 and 128; the accumulator at 256, in two halves
// of output positions (256 and 384) when there are more than 128 of them.
// Every wait is bounded; a wait that runs out raises the CTA's abort flag and
// the device status word, and every role then runs its loop without doing
// work so that all threads reach the drain and the TMEM release.
#include <cuda_bf16.h>

#include <type_traits>

#include "dw_common.cuh"
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
// fused 3x3: the transform and epilogue warps share each tile's stencil
constexpr int kFuseWorkers = kCXformWarps + kCEpiWarps;
constexpr int kCTileWindows = 128;

struct TcCachedParams {
    TmapBytes map_x;        // input planes, one box = a half tile (use_tmap)
    TmapBytes map_y;        // output planes, one box = a tile (use_tmap)
    const uint16_t* x;
    const uint16_t* M;      // [C][d][d] bf16, row u = p*w+q
    uint16_t* y;            // y, or z = 3x3(y) when fused
    const uint16_t* dw;     // fused: [C][3][3] bf16 weights
    int C, H, W, nh, nw;
    int bpt, sb, tpc, bands, items, R;
    int unit;               // tiles per unit of the CTA ranges (fused: whole planes)
    uint32_t sub_bytes;
    int use_tmap, kimg_sub;
    uint32_t off_b, off_out, off_raw, off_bar, off_halo;
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

// Fused 3x3 mixing of one tile, run by the transform and epilogue warps
// once the tile's bf16 y rows are in the output buffer (row R = k*w + r of
// the tile's bands, W elements, i.e. image rows in order).  Rows R = -2, -1
// are the previous tile's last two rows (a halo buffer), valid when the tile
// starts inside a plane; that tile's last output row waits for this tile's
// first row and is made here (R = -1).  Likewise this tile's last row is left
// to the next tile when the plane continues.  Worker k of nworkers takes a
// contiguous range of output rows; lane = 16-byte vector of a row.  The
// worker streams the input rows once, in order: input row i adds its taps
// of kernel row a = 0 to output i+1, a = 1 to output i and a = 2 to output
// i-1, so every output receives the standalone kernel's fp32 fused
// multiply-adds in the same (a, e) order (dw3x3_pairs8).  Taps that would
// read across a plane edge are left out instead of multiplying zeros: an
// accumulator that starts at +0 never holds -0, so adding a zero product
// never changes it and the bits are the same.  z goes to HBM straight from
// registers.
template <int WS>
__device__ __forceinline__ void fused_dw_rows(const TcCachedParams& P, const BandTile& t,
                                              const uint16_t* ybuf, const uint16_t* halo,
                                              int worker, int nworkers, int lane)
{
    const int W = P.W, nv = W >> 3, H = P.nh * WS;
    const int nbw = t.nb * WS;
    const int pr0 = (t.band0 % P.nh) * WS;          // plane row of the tile's row 0
    const bool next_cont = (t.band0 + t.nb) % P.nh != 0;
    const int r_lo = pr0 != 0 ? -1 : 0, r_hi = next_cont ? nbw - 1 : nbw;
    const int cnt = r_hi - r_lo;
    const int rs = r_lo + worker * cnt / nworkers, re = r_lo + (worker + 1) * cnt / nworkers;
    if (rs >= re)
        return;
    float k[9];
#pragma unroll
    for (int m = 0; m < 9; ++m)
        k[m] = __bfloat162float(__ushort_as_bfloat16(P.dw[(long long)t.c * 9 + m]));
    // plane row and image of input row rs - 1 (plane row -1: the row above
    // the tile when the tile starts a plane, which belongs to no output)
    int p1, b1;
    if (rs - 1 < 0) {
        p1 = pr0 + rs - 1;
        b1 = t.band0 / P.nh;
    } else {
        const int gb = t.band0 + (rs - 1) / WS;
        b1 = gb / P.nh;
        p1 = (gb - b1 * P.nh) * WS + (rs - 1) % WS;
    }
    const long long plane_step = (long long)P.C * H * W;   // next image, same channel
    for (int v = lane; v < nv; v += 32) {
        int pi = p1;                                // plane row of input row i
        // z addresses of rows i (zc) and i - 1 (zo); row -1 of an image is
        // the address one row before its row 0
        uint16_t* zc = P.y + (((long long)b1 * P.C + t.c) * H + p1) * W + 8 * v;
        uint16_t* zo = zc;
        const uint16_t* yrow = (rs - 1 >= 0 ? ybuf + (size_t)(rs - 1) * W
                                            : halo + (size_t)(rs + 1) * W) + 8 * v;
        // Input row i: X holds output i-1 (kernel row 2, then stored), Y
        // output i (kernel row 1), Z output i+1 (started here, kernel row 0).
        float X[8], Y[8], Z[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            X[j] = Y[j] = 0.0f;
        for (int i = rs - 1; i <= re; ++i) {
            const bool c_up = i + 1 >= rs && i + 1 < re && pi >= 0 && pi + 1 < H;
            const bool c_mid = i >= rs && i < re;
            const bool c_dn = i - 1 >= rs && i - 1 < re && pi > 0;
            float u[10];
            if (c_up || c_mid || c_dn) {
                const uint4 q = *reinterpret_cast<const uint4*>(yrow);
                u[0] = v > 0 ? __uint_as_float((uint32_t)yrow[-1] << 16) : 0.0f;
                u[9] = v + 1 < nv ? __uint_as_float((uint32_t)yrow[8] << 16) : 0.0f;
                const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    u[1 + 2 * j] = __uint_as_float(w4[j] << 16);
                    u[2 + 2 * j] = __uint_as_float(w4[j] & 0xFFFF0000u);
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                Z[j] = 0.0f;
            if (c_up) {
#pragma unroll
                for (int e = 0; e < 3; ++e)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        Z[j] = __fmaf_rn(k[e], u[j + e], Z[j]);
            }
            if (c_mid) {
#pragma unroll
                for (int e = 0; e < 3; ++e)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        Y[j] = __fmaf_rn(k[3 + e], u[j + e], Y[j]);
            }
            if (c_dn) {
#pragma unroll
                for (int e = 0; e < 3; ++e)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        X[j] = __fmaf_rn(k[6 + e], u[j + e], X[j]);
            }
            if (i - 1 >= rs && i - 1 < re) {
                uint32_t packed[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(X[2 * m], X[2 * m + 1]);
                    packed[m] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(zo) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
            // advance to row i + 1: the halo rows are followed by the tile's
            // row 0, and the next plane starts one image later
            yrow = i == -1 ? ybuf + 8 * v : yrow + W;
            zo = zc;
            zc += W;
            if (++pi == H) {
                pi = 0;
                zc += plane_step - (long long)H * W;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                X[j] = Y[j];
                Y[j] = Z[j];
            }
        }
    }
}

template <int WS, bool FUSE>
__global__ void __launch_bounds__(kCThreads, 1)
    wbmm_tc_cached_kernel(const __grid_constant__ TcCachedParams P)
{
    using F = CachedCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* b_base = smem + P.off_b;
    uint8_t* out_base = smem + P.off_out;
    uint8_t* raw_base = smem + P.off_raw;
    // offset of window m of a band-layout buffer (band k = m / nw, column j)
    auto woff = [&](int m) { return (m / P.nw) * WS * P.W + (m % P.nw) * WS; };
    CachedBars& S = *reinterpret_cast<CachedBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;
    const int R = P.R;

    // a contiguous, balanced range of units (P.unit tiles each) per CTA
    const int units = P.items / P.unit;
    const int qn = units / (int)gridDim.x, rem = units % (int)gridDim.x;
    const int it0 = ((int)blockIdx.x * qn + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem)) * P.unit;
    const int n_it = (qn + ((int)blockIdx.x < rem ? 1 : 0)) * P.unit;

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
    if (warp == 1) {
        tmem_alloc(&S.tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_slot;
    // Fused 3x3 of tile sq (FUSE): every transform and epilogue thread calls
    // this once per tile, in tile order, whatever its wait results.  The
    // first barrier is reached by the epilogue warps after draining tile sq
    // and by the transform warps after writing the A operand of tile sq + 1;
    // the stencil reads the halo buffer (sq + 1) & 1, and the epilogue threads
    // keep the tile's last two rows in buffer sq & 1 for the next tile.
    auto fused_stage = [&](int sq, int worker, bool epi) {
        const BandTile ft = cached_tile(P, it0 + sq);
        const uint16_t* ybuf = reinterpret_cast<const uint16_t*>(out_base);
        uint16_t* halo = reinterpret_cast<uint16_t*>(smem + P.off_halo);
        const size_t hsz = 2 * (size_t)P.W;
        named_bar_sync(2, kFuseWorkers * 32);       // y rows of tile sq written
        if (!*abort)
            fused_dw_rows<WS>(P, ft, ybuf, halo + ((sq + 1) & 1) * hsz, worker, kFuseWorkers,
                              lane);
        if (epi && (ft.band0 + ft.nb) % P.nh != 0) {
            const int nvec2 = 2 * (P.W >> 3);
            const uint4* src = reinterpret_cast<const uint4*>(ybuf + (size_t)(ft.nb * WS - 2) * P.W);
            uint4* dst = reinterpret_cast<uint4*>(halo + (sq & 1) * hsz);
            for (int i = (int)threadIdx.x - kCEpiWarp0 * 32; i < nvec2; i += kCEpiWarps * 32)
                dst[i] = src[i];
        }
        named_bar_sync(2, kFuseWorkers * 32);       // the buffer and halo rows are read
    };
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
        // (fused: the stencil workers store z themselves)
        for (int seq = 0; seq < (FUSE ? 0 : n_it); ++seq) {
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
                const uint16_t* src0 = raw + (valid ? woff(h ? n - h0win : n) : 0);
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
            if constexpr (FUSE) {
                if (seq >= 1)
                    fused_stage(seq - 1, warp - kCXformWarp0, false);
            }
        }
        if constexpr (FUSE) {
            if (n_it >= 1)
                fused_stage(n_it - 1, warp - kCXformWarp0, false);
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
            if (!FUSE && seq >= 1)
                ok = ok && mbar_wait(&S.out_empty, (seq - 1) & 1, abort, P.budget, P.status);
            const bool valid = n < nwin;
            uint16_t* o0 = reinterpret_cast<uint16_t*>(out_base) + (valid ? woff(n) : 0);
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
                if constexpr (!FUSE)
                    mbar_arrive(&S.out_full);
            }
            // the channel's last tile is done: every MMA that read B has
            // completed (acc_full), so B can take the next channel's matrix
            if (seq + 1 < n_it && cached_tile(P, it0 + seq + 1).c != t.c)
                build_for(t.c + 1);
            if constexpr (FUSE)
                fused_stage(seq, kCXformWarps + warp - kCEpiWarp0, true);
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
    uint32_t off_b, off_out, off_raw, off_bar, off_halo, total, sub_bytes;
    int R, bpt, sb, unit;
};

// fuse: the 3x3 runs in the epilogue; it needs whole 16-byte vectors per
// row and tiles that hold whole planes or planes of whole tiles (the CTA
// ranges are then whole planes), plus two halo rows of shared memory.
template <int WS>
bool cached_layout(const Geom& g, CachedLayout& L, bool fuse)
{
    using F = CachedCfg<WS>;
    if (g.nw < 1 || g.nw > kCTileWindows)
        return false;
    L.bpt = kCTileWindows / g.nw;
    L.unit = 1;
    if (fuse) {
        if (g.W % 8 != 0)
            return false;
        if (L.bpt >= g.nh) {
            L.bpt = L.bpt / g.nh * g.nh;            // whole planes per tile
        } else {
            while (g.nh % L.bpt != 0)               // planes of whole tiles
                --L.bpt;
            L.unit = g.nh / L.bpt;
        }
    }
    L.sb = (L.bpt + 1) / 2;
    L.sub_bytes = align_up((uint32_t)L.sb * WS * g.W * 2, 128);
    uint32_t off = 0;
    L.off_b = off;                                   // 1024-aligned
    off += F::B_BYTES;
    L.off_out = align_up(off, 128);
    off = L.off_out + F::OUT_BYTES;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(CachedBars);
    L.off_halo = align_up(off, 16);
    if (fuse)
        off = L.off_halo + 2u * 2u * (uint32_t)g.W * 2u;     // two halo buffers of two rows
    L.off_raw = align_up(off, 128);
    // the fused layout is not rounded up to 1 KB, which keeps a third ring
    // slot at 224 x 224
    const uint32_t reserve = fuse ? 0u : 1024u;
    const uint32_t avail = kSmemMax - reserve > L.off_raw ? kSmemMax - reserve - L.off_raw : 0;
    int R = (int)(avail / L.sub_bytes);
    if (R > kCRing)
        R = kCRing;
    L.R = R;
    if (R < 2)
        return false;
    L.total = align_up(L.off_raw + (uint32_t)R * L.sub_bytes, fuse ? 128u : 1024u);
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L.total <= kSmemMax;
}

template <int WS>
cudaError_t cached_launch_ws(const Geom& g, const void* x, const void* M, const void* dw, void* y,
                             const Launch& L)
{
    const bool fuse = dw != nullptr;
    CachedLayout lay;
    if (!cached_layout<WS>(g, lay, fuse))
        return cudaErrorInvalidConfiguration;
    static int configured[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_cached_kernel<WS, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMax);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(wbmm_tc_cached_kernel<WS, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax);
        if (e != cudaSuccess)
            return e;
        configured[dev & 63] = 1;
    }
    TcCachedParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.M = static_cast<const uint16_t*>(M);
    P.y = static_cast<uint16_t*>(y);
    P.dw = static_cast<const uint16_t*>(dw);
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = lay.bpt;
    P.sb = lay.sb;
    P.unit = lay.unit;
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
    P.off_bar = lay.off_bar; P.off_halo = lay.off_halo;
    P.budget = L.budget;
    P.status = L.status;
    int grid = L.num_sms;
    if (grid > P.items / P.unit)
        grid = P.items / P.unit;
    if (grid < 1)
        return cudaSuccess;
    cudaError_t e = fuse ? launch_pdl(wbmm_tc_cached_kernel<WS, true>, dim3(grid), dim3(kCThreads),
                                      lay.total, L.stream, P)
                         : launch_pdl(wbmm_tc_cached_kernel<WS, false>, dim3(grid),
                                      dim3(kCThreads), lay.total, L.stream, P);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

template <int WS>
bool cached_fits(const Geom& g, bool fuse)
{
    CachedLayout lay;
    return cached_layout<WS>(g, lay, fuse);
}

}  // namespace

bool tc_cached_supported(const Geom& g, bool fuse)
{
    if (g.w < 2 || g.w > 15)
        return false;
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    if (g.bands * (long long)g.C >= (1ll << 31))
        return false;
    switch (g.w) {
    case 2: return cached_fits<2>(g, fuse);
    case 3: return cached_fits<3>(g, fuse);
    case 4: return cached_fits<4>(g, fuse);
    case 5: return cached_fits<5>(g, fuse);
    case 6: return cached_fits<6>(g, fuse);
    case 7: return cached_fits<7>(g, fuse);
    case 8: return cached_fits<8>(g, fuse);
    case 9: return cached_fits<9>(g, fuse);
    case 10: return cached_fits<10>(g, fuse);
    case 11: return cached_fits<11>(g, fuse);
    case 12: return cached_fits<12>(g, fuse);
    case 13: return cached_fits<13>(g, fuse);
    case 14: return cached_fits<14>(g, fuse);
    default: return cached_fits<15>(g, fuse);
    }
}

cudaError_t tc_cached_launch(const Geom& g, const void* x, const void* M, const void* dw, void* y,
                             const Launch& L)
{
    switch (g.w) {
    case 2: return cached_launch_ws<2>(g, x, M, dw, y, L);
    case 3: return cached_launch_ws<3>(g, x, M, dw, y, L);
    case 4: return cached_launch_ws<4>(g, x, M, dw, y, L);
    case 5: return cached_launch_ws<5>(g, x, M, dw, y, L);
    case 6: return cached_launch_ws<6>(g, x, M, dw, y, L);
    case 7: return cached_launch_ws<7>(g, x, M, dw, y, L);
    case 8: return cached_launch_ws<8>(g, x, M, dw, y, L);
    case 9: return cached_launch_ws<9>(g, x, M, dw, y, L);
    case 10: return cached_launch_ws<10>(g, x, M, dw, y, L);
    case 11: return cached_launch_ws<11>(g, x, M, dw, y, L);
    case 12: return cached_launch_ws<12>(g, x, M, dw, y, L);
    case 13: return cached_launch_ws<13>(g, x, M, dw, y, L);
    case 14: return cached_launch_ws<14>(g, x, M, dw, y, L);
    case 15: return cached_launch_ws<15>(g, x, M, dw, y, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
