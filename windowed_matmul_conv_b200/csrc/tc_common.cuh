// Pieces shared by the tensor-core WBMM kernels: the padded in-window K
// layout, band/tile bookkeeping and the raw-band -> UMMA operand transform.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace wbmm {

// In-window positions as an MMA operand dimension: window row r occupies
// RP = roundup(w, 8) slots (position s of the row at slot r*RP + s, slots
// s >= w hold zero), so every window row is a whole number of 16-byte core
// matrix rows and needs no element shuffling.
template <int WS>
struct PadCfg {
    static constexpr int D = WS * WS;
    static constexpr int RP = (WS + 7) / 8 * 8;
    static constexpr int K = WS * RP;                  // padded positions
    static constexpr int KP = (K + 15) / 16 * 16;      // rounded to the MMA K step
    static constexpr int TSZ = (2 * WS - 1) * (2 * WS - 1);
};

// Bands of one tile: bands [band0, band0 + nb) of channel c; the bands of one
// image plane are adjacent in NCHW, so a tile is a few contiguous runs.
struct BandTile {
    int c;
    int band0;
    int nb;
};

// The contiguous runs of a tile, addressable one by one so that the lanes of
// a warp can issue their copies in parallel.  Run 0 starts at band0 and ends at the end
// of its image plane (or of the tile); every later run is one whole plane or
// the tile's tail.
struct BandRuns {
    int r0;      // bands in run 0
    int count;   // number of runs
};

__device__ __forceinline__ BandRuns band_runs(const BandTile& t, int nh)
{
    BandRuns R;
    const int i0 = t.band0 % nh;
    R.r0 = (nh - i0) < t.nb ? (nh - i0) : t.nb;
    R.count = 1 + (t.nb - R.r0 + nh - 1) / nh;
    return R;
}

// Global element offset, byte offset in the slot and bytes of run l.
__device__ __forceinline__ void band_run(const BandTile& t, const BandRuns& R, int l, int ws,
                                         int W, int H, int C, int nh, long long& goff,
                                         uint32_t& soff, uint32_t& bytes)
{
    const int first = (l == 0) ? 0 : R.r0 + (l - 1) * nh;   // band index within the tile
    int len = (l == 0) ? R.r0 : t.nb - first;
    if (len > nh)
        len = nh;
    const int g = t.band0 + first;
    const int b = g / nh, i = g - (g / nh) * nh;
    const uint32_t band_bytes = (uint32_t)ws * W * 2;
    goff = (((long long)b * C + t.c) * H + (long long)i * ws) * W;
    soff = (uint32_t)first * band_bytes;
    bytes = (uint32_t)len * band_bytes;
}

// Raw band layout -> operand tile with rows = windows n (8-row groups
// `sbo` bytes apart) and columns = padded positions (core matrices of 8
// slots, 128 bytes apart).  A warp takes one group of NWIN windows (8 or
// 16): lane (nl, rs) = (lane % NWIN, lane / NWIN) handles window NWIN*g + nl
// and window rows rs, rs + 32/NWIN, ...; all of a lane's rows are read
// before any is written, so its loads overlap.  Eight consecutive lanes take
// eight consecutive windows, so each quarter-warp store is one contiguous
// 128-byte line.  At w = 14, 16 windows x 2 rows per load instruction hit 32
// different banks for every plane width W = 28k (8 x 4 hit some banks twice);
// other window sizes keep 8 x 4.  Rows nwin <= n < nend are written as zeros;
// rows past that are left as they are.
template <int WS>
struct TransformCfg {
    static constexpr int NWIN = WS == 14 ? 16 : 8;      // windows per group
};

template <int WS>
__device__ __forceinline__ void transform_group(const uint16_t* raw, uint8_t* dst, uint32_t sbo,
                                                int gi, int nwin, int nend, const int* woff,
                                                int W, int lane)
{
    using P = PadCfg<WS>;
    constexpr int NWIN = TransformCfg<WS>::NWIN;
    constexpr int NROW = 32 / NWIN;
    constexpr int RQ = (WS + NROW - 1) / NROW;
    const int nl = lane % NWIN, rs = lane / NWIN;
    const int n = gi * NWIN + nl;
    if (n >= nend)
        return;
    const uint16_t* base = raw + woff[n < nwin ? n : 0];
    uint32_t wv[RQ][P::RP / 2];
#pragma unroll
    for (int q = 0; q < RQ; ++q) {
        const int r = q * NROW + rs;
        const uint16_t* src = base + r * W;
        if (n >= nwin || r >= WS) {
#pragma unroll
            for (int m = 0; m < P::RP / 2; ++m)
                wv[q][m] = 0u;
        } else if (WS % 2 == 0) {
#pragma unroll
            for (int m = 0; m < P::RP / 2; ++m)
                wv[q][m] = (2 * m < WS) ? reinterpret_cast<const uint32_t*>(src)[m] : 0u;
        } else {
#pragma unroll
            for (int m = 0; m < P::RP / 2; ++m) {
                const uint16_t lo = (2 * m < WS) ? src[2 * m] : (uint16_t)0;
                const uint16_t hi = (2 * m + 1 < WS) ? src[2 * m + 1] : (uint16_t)0;
                wv[q][m] = pack_bf16x2(lo, hi);
            }
        }
    }
    uint8_t* d0 = dst + (n >> 3) * sbo + (n & 7) * 16;
#pragma unroll
    for (int q = 0; q < RQ; ++q) {
        const int r = q * NROW + rs;
        if (r >= WS)
            continue;
#pragma unroll
        for (int c = 0; c < P::RP / 8; ++c)
            *reinterpret_cast<uint4*>(d0 + (r * P::RP / 8 + c) * 128) =
                make_uint4(wv[q][4 * c], wv[q][4 * c + 1], wv[q][4 * c + 2], wv[q][4 * c + 3]);
    }
}

// One tile: windows [0, nwin), zero rows up to nzero.  Warps take groups.
template <int WS>
__device__ __forceinline__ void transform_rows(const uint16_t* raw, uint8_t* dst, uint32_t sbo,
                                               int nwin, int nzero, const int* woff, int W,
                                               int tid, int nthreads)
{
    constexpr int NWIN = TransformCfg<WS>::NWIN;
    const int lane = tid & 31, wid = tid >> 5, nwarps = nthreads >> 5;
    const int nend = nzero > nwin ? nzero : nwin;
    const int groups = (nend + NWIN - 1) / NWIN;
    for (int gi = wid; gi < groups; gi += nwarps)
        transform_group<WS>(raw, dst, sbo, gi, nwin, nend, woff, W, lane);
}

// Two tiles of the same windows (from two tensors) in one pass: warps take
// the groups of both, so small tiles still keep every warp busy.
template <int WS>
__device__ __forceinline__ void transform_rows_pair(const uint16_t* raw0, uint8_t* dst0,
                                                    const uint16_t* raw1, uint8_t* dst1,
                                                    uint32_t sbo, int nwin, int nzero,
                                                    const int* woff, int W, int tid, int nthreads)
{
    constexpr int NWIN = TransformCfg<WS>::NWIN;
    const int lane = tid & 31, wid = tid >> 5, nwarps = nthreads >> 5;
    const int nend = nzero > nwin ? nzero : nwin;
    const int groups = (nend + NWIN - 1) / NWIN;
    for (int it = wid; it < 2 * groups; it += nwarps) {
        const bool second = it >= groups;
        transform_group<WS>(second ? raw1 : raw0, second ? dst1 : dst0, sbo,
                            second ? it - groups : it, nwin, nend, woff, W, lane);
    }
}

}  // namespace wbmm
