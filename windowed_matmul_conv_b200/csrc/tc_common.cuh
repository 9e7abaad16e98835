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

// Calls f(global element offset, byte offset in the slot, bytes) for every
// contiguous run of the tile (32-bit index math; host checks the ranges).
template <typename F>
__device__ __forceinline__ void for_each_band_run(int ws, int W, int H, int C, int nh,
                                                  const BandTile& t, F&& f)
{
    const uint32_t band_bytes = (uint32_t)ws * W * 2;
    int b = t.band0 / nh;
    int i = t.band0 - b * nh;
    int left = t.nb;
    uint32_t soff = 0;
    while (left > 0) {
        const int run = (nh - i) < left ? (nh - i) : left;
        const long long goff = (((long long)b * C + t.c) * H + (long long)i * ws) * W;
        f(goff, soff, (uint32_t)run * band_bytes);
        soff += (uint32_t)run * band_bytes;
        left -= run;
        ++b;
        i = 0;
    }
}

// The same runs, addressable one by one so that the lanes of a warp can
// issue their copies in parallel.  Run 0 starts at band0 and ends at the end
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
// slots, 128 bytes apart).  Work item = (window n, window row r); one thread
// reads the row and writes RP/8 16-byte core-matrix rows.  Eight consecutive
// lanes take eight consecutive windows, so each quarter-warp store is one
// contiguous 128-byte line.  Rows nwin <= n < nzero are written as zeros;
// rows past that are left as they are.
template <int WS>
__device__ __forceinline__ void transform_rows(const uint16_t* raw, uint8_t* dst, uint32_t sbo,
                                               int nwin, int nzero, const int* woff, int W,
                                               int tid, int nthreads)
{
    using P = PadCfg<WS>;
    constexpr int R4 = (WS + 3) / 4;
    const int lane = tid & 31, wid = tid >> 5, nwarps = nthreads >> 5;
    const int nl = lane & 7, rs = lane >> 3;
    const int nend = nzero > nwin ? nzero : nwin;
    const int groups = (nend + 7) >> 3;
    for (int it = wid; it < groups * R4; it += nwarps) {
        const int g8 = it / R4, r = (it - g8 * R4) * 4 + rs;
        const int n = g8 * 8 + nl;
        if (r >= WS || n >= nend)
            continue;
        const uint16_t* src = raw + woff[n < nwin ? n : 0] + r * W;
        uint8_t* d0 = dst + g8 * sbo + (r * P::RP / 8) * 128 + nl * 16;
        uint32_t wv[P::RP / 2];
        if (n >= nwin) {
#pragma unroll
            for (int m = 0; m < P::RP / 2; ++m)
                wv[m] = 0u;
        } else if (WS % 2 == 0) {
#pragma unroll
            for (int m = 0; m < P::RP / 2; ++m)
                wv[m] = (2 * m < WS) ? reinterpret_cast<const uint32_t*>(src)[m] : 0u;
        } else {
#pragma unroll
            for (int m = 0; m < P::RP / 2; ++m) {
                const uint16_t lo = (2 * m < WS) ? src[2 * m] : (uint16_t)0;
                const uint16_t hi = (2 * m + 1 < WS) ? src[2 * m + 1] : (uint16_t)0;
                wv[m] = pack_bf16x2(lo, hi);
            }
        }
#pragma unroll
        for (int c = 0; c < P::RP / 8; ++c) {
            uint4 v = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
            *reinterpret_cast<uint4*>(d0 + c * 128) = v;
        }
    }
}

}  // namespace wbmm
