// CUDA-core kernels: the fp32 WBMM path (tensor-core tf32 cannot meet the
// fp32 accuracy bound), bf16 shapes outside the tensor-core kernels' limits,
// the table-gradient finaliser, matrix caching, the standalone 3x3 depthwise
// mixing and the bounded-wait self-test.
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include <utility>

#include "dw_common.cuh"
#include "ptx_sm100.cuh"
#include "wbmm_internal.h"

namespace wbmm {

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// ------------------------------------------------------------- forward
// One block per band (plane b*C+c, window row i): the band's w rows and the
// channel's table sit in shared memory as fp32; each thread computes outputs
// (window j, position u) with an fp32 sum in fixed (r, s) order.
template <typename TIn>
__global__ void simt_fwd_kernel(const TIn* __restrict__ x, const TIn* __restrict__ src,
                                TIn* __restrict__ y, int C, int H, int W, int w, int nh, int nw,
                                int mode)
{
    extern __shared__ float sm[];
    const int tsz = (2 * w - 1) * (2 * w - 1), d = w * w;
    grid_dep_wait();
    grid_dep_launch();
    const long long blk = blockIdx.x;
    const long long bc = blk / nh;
    const int i = (int)(blk - bc * nh);
    const int c = (int)(bc % C);
    float* tbl = sm;
    float* band = sm + (mode == kCached ? 0 : tsz);
    if (mode != kCached)
        for (int k = threadIdx.x; k < tsz; k += blockDim.x)
            tbl[k] = to_f(src[(long long)c * tsz + k]);
    const TIn* xb = x + (bc * H + (long long)i * w) * W;
    for (int k = threadIdx.x; k < w * W; k += blockDim.x)
        band[k] = to_f(xb[k]);
    __syncthreads();
    TIn* yb = y + (bc * H + (long long)i * w) * W;
    const TIn* Mc = src + (long long)c * d * d;
    for (int o = threadIdx.x; o < nw * d; o += blockDim.x) {
        const int j = o / d, u = o - (o / d) * d;
        const int p = u / w, q = u - (u / w) * w;
        float acc = 0.0f;
        for (int r = 0; r < w; ++r) {
            const float* xr = band + r * W + j * w;
            const int rowi = (p - r + w - 1) * (2 * w - 1) + (q + w - 1);
            for (int s = 0; s < w; ++s) {
                float coef;
                if (mode == kCached)
                    coef = to_f(Mc[(long long)u * d + r * w + s]);
                else if (mode == kTableFlip)
                    coef = tbl[tsz - 1 - (rowi - s)];
                else
                    coef = tbl[rowi - s];
                acc = __fmaf_rn(coef, xr[s], acc);
            }
        }
        yb[p * W + j * w + q] = from_f<TIn>(acc);
    }
}

// ------------------------------------------------ forward, cached matrices
// Register-tiled form of the cached-matrix sums (d = w*w <= 196): a block
// holds M_c^T (rows v, d padded to DP = roundup(d, 8) columns u) and a tile
// of whole bands (at most 64 windows) X[v][n] in shared memory as fp32, the
// tile stored with a row stride of 68 floats so that the transposing writes
// of the band loads meet few bank conflicts; thread (ug, ng) keeps the 8 x 4
// outputs (u = 8ug.., n = 4ng..) in registers and, for each v, loads two
// float4 of M and one of X for 32 fused multiply-adds.  Loads and stores
// walk band rows, one lane per element.  Each output is one fp32 sum in
// v = (r, s) order, as in simt_fwd_kernel, so the results are bit-identical
// to it.  Blocks take contiguous runs of one channel's tiles, so M_c is
// loaded once per run.
constexpr int kCachedNT = 64;       // windows per tile, at most
constexpr int kCachedXS = 68;       // row stride of the tile in shared memory
constexpr size_t kCachedSmemMax = 232448;       // the per-block maximum on sm_100

template <typename TIn>
__global__ void __launch_bounds__(400, 1)
    simt_cached_kernel(const TIn* __restrict__ x, const TIn* __restrict__ M, TIn* __restrict__ y,
                       int C, int H, int W, int w, int nh, int nw, long long bands, int bpt,
                       int ntiles, int tpb, int G)
{
    extern __shared__ __align__(16) float smc[];
    const int d = w * w, DP = (d + 7) / 8 * 8;
    float* MT = smc;                              // [d][DP]
    float* XS = smc + (size_t)d * DP;             // [d][kCachedXS], then Y[u][n]
    grid_dep_wait();
    grid_dep_launch();
    const int c = blockIdx.x / G, gidx = blockIdx.x - (blockIdx.x / G) * G;
    const int t0 = gidx * tpb, t1 = t0 + tpb < ntiles ? t0 + tpb : ntiles;
    if (t0 >= t1)
        return;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    const TIn* Mc = M + (long long)c * d * d;
    // fp32 operands go to shared memory as asynchronous 4-byte copies, all of
    // a tile's in flight at once; bf16 ones are widened through registers
    constexpr bool kAsync = std::is_same<TIn, float>::value;
    for (int e = tid; e < d * d; e += nthr) {
        const int u = e / d, v = e - (e / d) * d;
        if constexpr (kAsync)
            cp_async_4(smem_u32(MT + v * DP + u), Mc + e);
        else
            MT[v * DP + u] = to_f(Mc[e]);
    }
    const int ug = tid >> 4, ng = tid & 15;
    const bool active = 8 * ug < d;
    for (int t = t0; t < t1; ++t) {
        const long long g0 = (long long)t * bpt;
        const int nb = bands - g0 < bpt ? (int)(bands - g0) : bpt;
        __syncthreads();        // M_c written; the previous tile's outputs stored
        // zero the windows past the tile's last band (read by the register
        // tiles, never stored)
        for (int e = tid; e < d * kCachedNT; e += nthr) {
            const int v = e >> 6, n = e & (kCachedNT - 1);
            if (n >= nb * nw)
                XS[v * kCachedXS + n] = 0.0f;
        }
        for (int row = warp; row < nb * w; row += nwarps) {
            const int kb = row / w, r = row - (row / w) * w;
            const long long gb = g0 + kb;
            const long long b = gb / nh;
            const int i = (int)(gb - b * nh);
            const TIn* src = x + ((b * C + c) * H + (long long)i * w + r) * W;
            for (int col = lane; col < W; col += 32) {
                const int j = col / w, sidx = col - (col / w) * w;
                float* dst = XS + (r * w + sidx) * kCachedXS + kb * nw + j;
                if constexpr (kAsync)
                    cp_async_4(smem_u32(dst), src + col);
                else
                    *dst = to_f(src[col]);
            }
        }
        if constexpr (kAsync)
            cp_async_wait_all();
        __syncthreads();
        float acc[8][4];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int bq = 0; bq < 4; ++bq)
                acc[a][bq] = 0.0f;
        if (active) {
            // the operands of v + 1 are loaded while the 32 multiply-adds of
            // v run, so the shared-memory latency is not exposed
            const float* mp = MT + 8 * ug;
            const float* xp = XS + 4 * ng;
            float4 m0 = *reinterpret_cast<const float4*>(mp);
            float4 m1 = *reinterpret_cast<const float4*>(mp + 4);
            float4 xv = *reinterpret_cast<const float4*>(xp);
#pragma unroll 2
            for (int v = 0; v < d; ++v) {
                const int vn = v + 1 < d ? v + 1 : v;
                const float4 n0 = *reinterpret_cast<const float4*>(mp + vn * DP);
                const float4 n1 = *reinterpret_cast<const float4*>(mp + vn * DP + 4);
                const float4 nx = *reinterpret_cast<const float4*>(xp + vn * kCachedXS);
                const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
                const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int bq = 0; bq < 4; ++bq)
                        acc[a][bq] = __fmaf_rn(mv[a], xs[bq], acc[a][bq]);
                m0 = n0;
                m1 = n1;
                xv = nx;
            }
        }
        __syncthreads();        // every thread is done reading XS
        if (active) {
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int u = 8 * ug + a;
                if (u < d)
                    *reinterpret_cast<float4*>(XS + u * kCachedXS + 4 * ng) =
                        make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
            }
        }
        __syncthreads();
        for (int row = warp; row < nb * w; row += nwarps) {
            const int kb = row / w, p = row - (row / w) * w;
            const long long gb = g0 + kb;
            const long long b = gb / nh;
            const int i = (int)(gb - b * nh);
            TIn* dst = y + ((b * C + c) * H + (long long)i * w + p) * W;
            for (int col = lane; col < W; col += 32) {
                const int j = col / w, q = col - (col / w) * w;
                dst[col] = from_f<TIn>(XS[(p * w + q) * kCachedXS + kb * nw + j]);
            }
        }
    }
}

// ------------------------------------------------ forward, table modes
// Register-tiled form of the same sums for the table modes and w <= 32: a
// thread computes QC consecutive outputs (p, q0 .. q0+QC-1) of one window.
// For each input row r it loads the QC + w - 1 table entries of row p - r
// that those outputs use, then for each input s one x value feeds QC fused
// multiply-adds with static indices; shared-memory loads per FMA drop from 2
// to about 2/QC.  Each output is still one fp32 sum in (r, s) order, so the
// result is bit-identical to simt_fwd_kernel.  A block takes `rb`
// consecutive bands of one channel; the table (reversed end to end for the
// input gradient) and the bands sit in shared memory as fp32.
template <int WS>
struct RowCfg {
    static constexpr int QC = WS <= 16 ? WS : (WS + 1) / 2;   // outputs per thread
    static constexpr int NQ = (WS + QC - 1) / QC;
    static constexpr int L = 2 * WS - 1;
    static constexpr int TSZ = L * L;
    static constexpr int TPAD = (TSZ + QC + 3) / 4 * 4;        // table + overhang of the last chunk
};

template <typename TIn, int WS, bool FLIP>
__global__ void __launch_bounds__(256) simt_fwd_rows_kernel(const TIn* __restrict__ x,
                                                            const TIn* __restrict__ T,
                                                            TIn* __restrict__ y, int C, int H,
                                                            int W, int nh, int nw, int bands,
                                                            int rb, int groups)
{
    using F = RowCfg<WS>;
    extern __shared__ float sm[];
    grid_dep_wait();
    grid_dep_launch();
    float* tbl = sm;
    float* sb = sm + F::TPAD;
    const int c = (int)(blockIdx.x / groups);
    const int g0 = (int)(blockIdx.x - c * groups) * rb;
    const int nb = bands - g0 < rb ? bands - g0 : rb;
    for (int k = threadIdx.x; k < F::TPAD; k += blockDim.x)
        tbl[k] = k < F::TSZ ? to_f(T[(long long)c * F::TSZ + (FLIP ? F::TSZ - 1 - k : k)]) : 0.0f;
    const int band_elems = WS * W;
    for (int e = threadIdx.x; e < nb * band_elems; e += blockDim.x) {
        const int k = e / band_elems, off = e - k * band_elems;
        const int g = g0 + k, b = g / nh, i = g - (g / nh) * nh;
        sb[e] = to_f(x[(((long long)b * C + c) * H + (long long)i * WS) * W + off]);
    }
    __syncthreads();
    const int items = nb * nw * F::NQ * WS;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int p = it % WS;
        int rest = it / WS;
        const int qc = rest % F::NQ;
        rest /= F::NQ;
        const int j = rest % nw, k = rest / nw;
        const int q0 = qc * F::QC;
        const float* xw = sb + k * band_elems + j * WS;
        float acc[F::QC];
#pragma unroll
        for (int qq = 0; qq < F::QC; ++qq)
            acc[qq] = 0.0f;
#pragma unroll 1
        for (int r = 0; r < WS; ++r) {
            const float* trow = tbl + (p - r + WS - 1) * F::L + q0;
            float tv[F::QC + WS - 1];
#pragma unroll
            for (int m = 0; m < F::QC + WS - 1; ++m)
                tv[m] = trow[m];
            const float* xr = xw + r * W;
#pragma unroll
            for (int s2 = 0; s2 < WS; ++s2) {
                const float xv = xr[s2];
#pragma unroll
                for (int qq = 0; qq < F::QC; ++qq)
                    acc[qq] = __fmaf_rn(tv[qq - s2 + WS - 1], xv, acc[qq]);
            }
        }
        const int g = g0 + k, b = g / nh, i = g - (g / nh) * nh;
        TIn* yr = y + (((long long)b * C + c) * H + (long long)i * WS + p) * W + j * WS + q0;
#pragma unroll
        for (int qq = 0; qq < F::QC; ++qq)
            if (q0 + qq < WS)
                yr[qq] = from_f<TIn>(acc[qq]);
    }
}

// ------------------------------------------- reparameterisation merge
// One thread per matrix entry: the w-window table entry plus, inside the
// same k x k sub-window, the k-window table entry; fp32 sum, one rounding.
template <typename E>
__global__ void reparam_kernel(const E* __restrict__ Tw, const E* __restrict__ Tk,
                               E* __restrict__ M, int C, int w, int k)
{
    grid_dep_wait();
    grid_dep_launch();
    const int d = w * w, Lw = 2 * w - 1, Lk = 2 * k - 1;
    const long long total = (long long)C * d * d;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(e / ((long long)d * d));
        const int rem = (int)(e - (long long)c * d * d);
        const int u = rem / d, v = rem - (rem / d) * d;
        const int p = u / w, q = u - (u / w) * w, r = v / w, s = v - (v / w) * w;
        float val = to_f(Tw[(long long)c * Lw * Lw + (p - r + w - 1) * Lw + (q - s + w - 1)]);
        if (p / k == r / k && q / k == s / k)
            val += to_f(Tk[(long long)c * Lk * Lk + (p % k - r % k + k - 1) * Lk +
                           (q % k - s % k + k - 1)]);
        M[e] = from_f<E>(val);
    }
}

// ------------------------------------------------------- table gradient
// One block per (channel, chunk of kSimtChunkBands bands); each thread owns
// table bins and sums dy[p,q] * x[p-dp, q-dq] over the chunk's windows in a
// fixed order.  Partials go to [C][chunks][tsz].
constexpr int kSimtChunkBands = 8;
constexpr int kSimtMaxBinsPerThread = 16;

template <typename TIn>
__global__ void simt_dt_kernel(const TIn* __restrict__ x, const TIn* __restrict__ dy,
                               float* __restrict__ part, int C, int H, int W, int w, int nh,
                               int nw, long long bands, int chunks)
{
    extern __shared__ float sm[];
    grid_dep_wait();
    grid_dep_launch();
    const int tsz = (2 * w - 1) * (2 * w - 1);
    const int c = blockIdx.x / chunks, k = blockIdx.x - (blockIdx.x / chunks) * chunks;
    float* xb = sm;
    float* gb = sm + w * W;
    float acc[kSimtMaxBinsPerThread];
    for (int m = 0; m < kSimtMaxBinsPerThread; ++m)
        acc[m] = 0.0f;
    const long long g0 = (long long)k * kSimtChunkBands;
    const long long g1 = g0 + kSimtChunkBands < bands ? g0 + kSimtChunkBands : bands;
    for (long long g = g0; g < g1; ++g) {
        const long long b = g / nh;
        const int i = (int)(g - b * nh);
        const long long off = ((b * C + c) * H + (long long)i * w) * W;
        __syncthreads();
        for (int e = threadIdx.x; e < w * W; e += blockDim.x) {
            xb[e] = to_f(x[off + e]);
            gb[e] = to_f(dy[off + e]);
        }
        __syncthreads();
        for (int m = 0; m < kSimtMaxBinsPerThread; ++m) {
            const int t = threadIdx.x + m * blockDim.x;
            if (t >= tsz)
                break;
            const int dp = t / (2 * w - 1) - (w - 1), dq = t % (2 * w - 1) - (w - 1);
            const int p0 = dp > 0 ? dp : 0, p1 = dp > 0 ? w : w + dp;
            const int q0 = dq > 0 ? dq : 0, q1 = dq > 0 ? w : w + dq;
            float a = acc[m];
            for (int j = 0; j < nw; ++j)
                for (int p = p0; p < p1; ++p)
                    for (int q = q0; q < q1; ++q)
                        a = __fmaf_rn(gb[p * W + j * w + q], xb[(p - dp) * W + j * w + (q - dq)],
                                      a);
            acc[m] = a;
        }
    }
    for (int m = 0; m < kSimtMaxBinsPerThread; ++m) {
        const int t = threadIdx.x + m * blockDim.x;
        if (t < tsz)
            part[((long long)c * chunks + k) * tsz + t] = acc[m];
    }
}

// Table gradient for 4 <= w <= 14 as G = dY X^T (positions x positions,
// summed over windows) and diagonal sums: dT[dp, dq] adds G[(p, q),
// (p - dp, q - dq)] over the positions where both are inside the window,
// the same products the table-bin loop above forms.
//
// The tiles (whole bands, at most 64 windows) of all channels, channel by
// channel, are split into gridDim.x contiguous ranges of equal size to
// within one tile, one per block.  Per tile the dY and x windows sit in
// shared memory as fp32 rows [window][position] (row stride DP = roundup(d,
// 4*NCG); rows past the tile's windows are zero), two tiles deep so that the
// next tile's copies overlap this tile's arithmetic; the copies go out in
// units of V elements (V = 2 when w and W are even), every thread stepping
// through the tile's rows and columns by a fixed stride without divisions.
// Thread (ug, vg) accumulates G at rows 8ug .. 8ug+7 and columns k*CP +
// 4vg .. k*CP + 4vg+3, k < NCG (CP = DP / NCG), over the windows in order:
// 32*NCG fused multiply-adds per 2 + NCG 16-byte shared loads, and a warp
// reads consecutive 16-byte words of the x rows.  Where its range leaves a channel, the block
// puts G in shared memory; a warp per pair of window rows (p, p') sums the
// 2w - 1 diagonals of that w x w block of G, lane by lane, then every bin
// adds its (p, p - dp) sums in order of p into the partial table
// [c][slot][tsz] (slot = block - first block of the channel).  The block of
// slot 0 zeroes the slots the channel does not use, and the finaliser adds
// all S slots in order.
constexpr int kDtgSMs = 148;                // SMs of a B200
constexpr int kDtgMaxCols = kCachedNT * 14; // window columns of a row, at most
// Two column groups (8 x 8 thread tiles, 625 threads at w = 14) ran faster
// than four (8 x 16, 325 threads): more warps cover the FMA latencies.
constexpr int kDtgNCG = 2;                  // column groups of 4 per thread tile
constexpr int kDtgMaxThreads = 640;         // thread tiles at w = 14, in whole warps

template <typename TIn, int V>
__global__ void __launch_bounds__(kDtgMaxThreads, 1)
    simt_dtg_kernel(const TIn* __restrict__ x, const TIn* __restrict__ dy, float* __restrict__ part,
                    int C, int H, int W, int w, int nh, int nw, long long bands, int bpt,
                    int ntiles, int S)
{
    extern __shared__ __align__(16) float sgm[];
    constexpr int NCG = kDtgNCG, TV = 4 * NCG;
    const int d = w * w, DP = (d + TV - 1) / TV * TV, CP = DP / NCG;
    const int UG = (d + 7) / 8, VG = CP / 4;
    const int L = 2 * w - 1, tsz = L * L;
    const int stage_floats = 2 * kCachedNT * DP;  // dY rows, then x rows
    int* colmap = reinterpret_cast<int*>(sgm + 2 * stage_floats);
    // tile indices fit in 32 bits (the host checks C * ntiles < 2^31)
    const long long G = gridDim.x, Ttot = (long long)C * ntiles;
    const int T0 = (int)(blockIdx.x * Ttot / G), T1 = (int)((blockIdx.x + 1) * Ttot / G);
    auto block_of = [&](int f) { return (int)((((long long)f + 1) * G - 1) / Ttot); };
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
    const int ug = tid / VG, vg = tid - (tid / VG) * VG;
    const bool active = ug < UG;
    // copy units of an image row: unit cu holds columns V*cu .. V*cu + V-1
    // of window j, at offset j*DP + (position in the window row)
    const int upr = nw * w / V;
    for (int cu = tid; cu < upr; cu += nthr) {
        const int col = cu * V, j = col / w;
        colmap[cu] = j * DP + (col - j * w);
    }
    // this thread's first unit (row0, cu0) of a tile and its step: drow
    // rows and dcu units (one more row when the unit index wraps)
    const int row0 = tid / upr, cu0 = tid - (tid / upr) * upr;
    const int drow = nthr / upr, dcu = nthr - (nthr / upr) * upr;
    const int kb0 = row0 / w, r0 = row0 - (row0 / w) * w;
    grid_dep_wait();
    grid_dep_launch();
    __syncthreads();
    constexpr bool kAsync = std::is_same<TIn, float>::value;
    // Tile f (flattened over channels) into stage st: asynchronous copies
    // for fp32 (one commit group per tile), widened through registers for
    // bf16.
    auto load_tile = [&](int f, int st) {
        float* GS = sgm + (size_t)st * stage_floats;
        float* XS = GS + kCachedNT * DP;
        const int c = f / ntiles;
        const int g0 = (f - c * ntiles) * bpt;                  // bands < 2^31 (host)
        const int nb = (int)bands - g0 < bpt ? (int)bands - g0 : bpt;
        for (int e = tid; e < (kCachedNT - nb * nw) * DP; e += nthr) {
            GS[nb * nw * DP + e] = 0.0f;
            XS[nb * nw * DP + e] = 0.0f;
        }
        // band kb0 of the tile: image b, band i of that image
        const int gb = g0 + kb0;
        int b = gb / nh;
        int i = gb - b * nh;
        int kb = kb0, r = r0, cu = cu0;
        while (kb < nb) {
            const long long off =
                ((long long)(b * C + c) * H + i * w + r) * W + (long long)cu * V;
            const int o = kb * nw * DP + r * w + colmap[cu];
            if constexpr (kAsync) {
                if constexpr (V == 2) {
                    cp_async_8(smem_u32(GS + o), dy + off);
                    cp_async_8(smem_u32(XS + o), x + off);
                } else {
                    cp_async_4(smem_u32(GS + o), dy + off);
                    cp_async_4(smem_u32(XS + o), x + off);
                }
            } else {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    GS[o + v] = to_f(dy[off + v]);
                    XS[o + v] = to_f(x[off + v]);
                }
            }
            cu += dcu;
            int rinc = drow;
            if (cu >= upr) {
                cu -= upr;
                ++rinc;
            }
            r += rinc;
            while (r >= w) {
                r -= w;
                ++kb;
                if (++i == nh) {
                    i = 0;
                    ++b;
                }
            }
        }
        if constexpr (kAsync)
            cp_async_commit();
    };
    float acc[8][TV];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < TV; ++b)
            acc[a][b] = 0.0f;
    int st = 0;
    if (T0 < T1)
        load_tile(T0, 0);
    for (int f = T0; f < T1; ++f) {
        const int c = f / ntiles;
        const bool same_next = f + 1 < T1 && (f + 1) / ntiles == c;
        // stage st ^ 1 was last read by the previous tile, before the barrier
        // that closed its iteration
        if (same_next)
            load_tile(f + 1, st ^ 1);
        if constexpr (kAsync) {
            if (same_next)
                cp_async_wait_group<1>();
            else
                cp_async_wait_group<0>();
        }
        __syncthreads();
        if (active) {
            const float* ap = sgm + (size_t)st * stage_floats + 8 * ug;
            const float* bp = sgm + (size_t)st * stage_floats + kCachedNT * DP + 4 * vg;
#pragma unroll 2
            for (int n = 0; n < kCachedNT; ++n) {
                const float4 a0 = *reinterpret_cast<const float4*>(ap + n * DP);
                const float4 a1 = *reinterpret_cast<const float4*>(ap + n * DP + 4);
                float bv[TV];
#pragma unroll
                for (int k = 0; k < NCG; ++k) {
                    const float4 bk = *reinterpret_cast<const float4*>(bp + n * DP + k * CP);
                    bv[4 * k] = bk.x;
                    bv[4 * k + 1] = bk.y;
                    bv[4 * k + 2] = bk.z;
                    bv[4 * k + 3] = bk.w;
                }
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < TV; ++b)
                        acc[a][b] = __fmaf_rn(av[a], bv[b], acc[a][b]);
            }
        }
        __syncthreads();
        if (same_next) {
            st ^= 1;
            continue;
        }
        // ------------------------------------------- channel c's partial
        // G[u][v] to shared memory (the operand stages are dead); rows u >= d
        // are not written, columns v >= d are written but never read.  The
        // diagonal sums R[p][p'][dq + w - 1] follow G.
        float* GM = sgm;
        float* RS = sgm + (size_t)d * DP;
        if (active) {
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int u = 8 * ug + a;
                if (u < d) {
#pragma unroll
                    for (int k = 0; k < NCG; ++k)
                        *reinterpret_cast<float4*>(GM + u * DP + k * CP + 4 * vg) =
                            make_float4(acc[a][4 * k], acc[a][4 * k + 1], acc[a][4 * k + 2],
                                        acc[a][4 * k + 3]);
                }
            }
        }
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < TV; ++b)
                acc[a][b] = 0.0f;
        __syncthreads();
        // block (p, p') of G: rows p*w + q, columns p'*w + q'; lane l sums
        // its diagonal q - q' = l - (w - 1) in order of q
        for (int pr = warp; pr < d; pr += nwarps) {
            const int p = pr / w, p2 = pr - (pr / w) * w;
            if (lane < L) {
                const int dq = lane - (w - 1);
                const int q0 = dq > 0 ? dq : 0, q1 = dq > 0 ? w : w + dq;
                const float* gp = GM + (p * w + q0) * DP + p2 * w + (q0 - dq);
                float sum = 0.0f;
                for (int q = q0; q < q1; ++q, gp += DP + 1)
                    sum += *gp;
                RS[pr * L + lane] = sum;
            }
        }
        __syncthreads();
        const int first = block_of(c * ntiles);
        const int slot = (int)blockIdx.x - first;
        float* out = part + ((long long)c * S + slot) * tsz;
        for (int bin = tid; bin < tsz; bin += nthr) {
            const int dpi = bin / L, dqi = bin - (bin / L) * L;
            const int dp = dpi - (w - 1);
            const int p0 = dp > 0 ? dp : 0, p1 = dp > 0 ? w : w + dp;
            float sum = 0.0f;
            for (int p = p0; p < p1; ++p)
                sum += RS[(p * w + p - dp) * L + dqi];
            out[bin] = sum;
        }
        if (slot == 0) {
            const int used = block_of(c * ntiles + ntiles - 1) - first + 1;
            for (int e = used * tsz + tid; e < S * tsz; e += nthr)
                part[(long long)c * S * tsz + e] = 0.0f;
        }
        __syncthreads();        // RS read before the next tile's copies land
        if (f + 1 < T1)
            load_tile(f + 1, 0);
        st = 0;
    }
}

// Fixed-order sum of the partial tables.
__global__ void dt_finalize_kernel(const float* __restrict__ part, float* __restrict__ dT, int C,
                                   int tsz, int chunks)
{
    grid_dep_wait();
    grid_dep_launch();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)C * tsz)
        return;
    const long long c = i / tsz, t = i - (i / tsz) * tsz;
    float acc = 0.0f;
    for (int k = 0; k < chunks; ++k)
        acc += part[(c * chunks + k) * tsz + t];
    dT[i] = acc;
}

// M[c][u][v] = T[c][idx(u, v)]: a bit copy of table entries.
template <typename E>
__global__ void cache_kernel(const E* __restrict__ T, E* __restrict__ M, int C, int w)
{
    grid_dep_wait();
    grid_dep_launch();
    const int d = w * w, tsz = (2 * w - 1) * (2 * w - 1);
    const long long total = (long long)C * d * d;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const long long c = e / ((long long)d * d);
        const int rem = (int)(e - c * d * d);
        const int u = rem / d, v = rem - (rem / d) * d;
        const int p = u / w, q = u - (u / w) * w, r = v / w, s = v - (v / w) * w;
        M[e] = T[c * tsz + (p - r + w - 1) * (2 * w - 1) + (q - s + w - 1)];
    }
}

// --------------------------------------------------------- 3x3 mixing
// Tile of kDwTH x kDwTW outputs with a one-pixel halo (zero outside the
// image) in shared memory; fp32 sum in fixed (a, e) order.
constexpr int kDwTH = 16, kDwTW = 64;

template <typename TIn>
__global__ void dw3x3_kernel(const TIn* __restrict__ y, const TIn* __restrict__ K,
                             TIn* __restrict__ z, int C, int H, int W, int tiles_y, int tiles_x)
{
    grid_dep_wait();
    grid_dep_launch();
    __shared__ float tile[(kDwTH + 2) * (kDwTW + 2)];
    const long long blk = blockIdx.x;
    const long long bc = blk / ((long long)tiles_y * tiles_x);
    const int rem = (int)(blk - bc * tiles_y * tiles_x);
    const int ty = rem / tiles_x, tx = rem - (rem / tiles_x) * tiles_x;
    const int c = (int)(bc % C);
    float k[9];
#pragma unroll
    for (int m = 0; m < 9; ++m)
        k[m] = to_f(K[c * 9 + m]);
    const int h0 = ty * kDwTH, x0 = tx * kDwTW;
    const TIn* yp = y + bc * H * (long long)W;
    for (int e = threadIdx.x; e < (kDwTH + 2) * (kDwTW + 2); e += blockDim.x) {
        const int hh = h0 - 1 + e / (kDwTW + 2), xx = x0 - 1 + e % (kDwTW + 2);
        tile[e] = (hh >= 0 && hh < H && xx >= 0 && xx < W) ? to_f(yp[(long long)hh * W + xx])
                                                            : 0.0f;
    }
    __syncthreads();
    TIn* zp = z + bc * H * (long long)W;
    for (int o = threadIdx.x; o < kDwTH * kDwTW; o += blockDim.x) {
        const int oh = o / kDwTW, ox = o - (o / kDwTW) * kDwTW;
        const int h = h0 + oh, xw = x0 + ox;
        if (h >= H || xw >= W)
            continue;
        float acc = 0.0f;
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int e = 0; e < 3; ++e)
                acc = __fmaf_rn(k[a * 3 + e], tile[(oh + a) * (kDwTW + 2) + ox + e], acc);
        zp[(long long)h * W + xw] = from_f<TIn>(acc);
    }
}

// bf16 maps whose rows are whole 16-byte vectors (W % 8 == 0), streamed.
// Lane = one 16-byte vector of a 32-vector chunk (256 columns) of a plane; a
// warp walks down rows.  The flattened row space (plane-chunk, row) is cut
// into one contiguous, balanced range per warp, so every warp streams the
// same number of rows.  Each lane keeps its own column of the next kDwRing
// input rows in flight with 16-byte asynchronous copies into a ring in shared
// memory (rows outside the image are zero-filled by the copy); a row is read
// back once, unpacked into fp32 pairs (its left and right neighbour values
// from the adjacent lanes by shuffles, or a 2-byte load at a chunk edge inside
// the row), and its slot is refilled at once.  The three live rows stay
// unpacked in registers.  The per-output arithmetic is dw3x3_f8: the fp32
// fused multiply-adds of dw3x3_pairs8 (the fused epilogue's, two outputs per
// instruction) one output at a time in the same order, so both give the same
// bits.
constexpr int kDwRing = 16;
constexpr int kDwWarps = 4;
constexpr int kDwBlocksPerSm = 6;
constexpr size_t kDwSmem = (size_t)kDwWarps * kDwRing * 32 * 16;
static_assert((kDwRing & (kDwRing - 1)) == 0, "ring slots advance by masking");

__global__ void __launch_bounds__(kDwWarps * 32, kDwBlocksPerSm) dw3x3_bf16_rows_kernel(
    const uint16_t* __restrict__ y, const uint16_t* __restrict__ K, uint16_t* __restrict__ z,
    int C, int H, int W, int chunks, long long total_rows)
{
    extern __shared__ uint4 dw_ring[];
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const uint32_t ring0 = smem_u32(dw_ring + (threadIdx.x >> 5) * kDwRing * 32 + lane);
    const uint4* ringp = dw_ring + (threadIdx.x >> 5) * kDwRing * 32 + lane;
    const long long gw = (long long)blockIdx.x * kDwWarps + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * kDwWarps;
    const long long qn = total_rows / nwarps, rem = total_rows % nwarps;
    long long r = gw * qn + (gw < rem ? gw : rem);
    const long long r1 = r + qn + (gw < rem ? 1 : 0);
    const int nvec = W / 8;
    while (r < r1) {
        const long long pc = r / H;
        const int hs = (int)(r - pc * H);
        const int he = (int)((r1 - r) < (long long)(H - hs) ? hs + (r1 - r) : H);
        r += he - hs;
        const long long bc = pc / chunks;
        const int chunk = (int)(pc - bc * chunks);
        const int c = (int)(bc % C);
        const int v = chunk * 32 + lane;
        const bool act = v < nvec;
        const uint4* yp = reinterpret_cast<const uint4*>(y) + bc * H * (long long)nvec;
        const uint16_t* y16 = y + bc * H * (long long)W;
        uint4* zp = reinterpret_cast<uint4*>(z) + bc * H * (long long)nvec;
        float k[9];
#pragma unroll
        for (int m = 0; m < 9; ++m)
            k[m] = __bfloat162float(__ushort_as_bfloat16(__ldg(K + c * 9 + m)));
        // Input rows hs-1 .. he are needed; those inside the image are
        // [xlo, xhi].  Row x goes to ring slot (x - hs + 1) mod kDwRing; the
        // fetch and take positions advance one row at a time.
        const int xlo = hs - 1 > 0 ? hs - 1 : 0, xhi = he < H - 1 ? he : H - 1;
        int fx = hs - 1;                                    // next row to fetch
        uint32_t fslot = 0;
        const uint4* fsrc = yp + (long long)(hs - 1) * nvec + v;
        auto fetch = [&]() {
            const bool ok = act && fx >= xlo && fx <= xhi;
            cp_async_16z(ring0 + fslot * (32u * 16u), ok ? fsrc : yp, ok ? 16u : 0u);
            cp_async_commit();
            ++fx;
            fslot = (fslot + 1) & (kDwRing - 1);
            fsrc += nvec;
        };
        int tx = hs - 1;                                    // next row to take
        uint32_t tslot = 0;
        const bool edges = chunks > 1;      // a row's chunks need 2-byte edge loads
        // row tx -> fp32 values (after its copy completed), then its slot is refilled
        auto take = [&](DwRowF& u) {
            cp_async_wait_group<kDwRing - 1>();
            const uint4 vec = ringp[tslot * 32];
            uint32_t lf = __shfl_up_sync(0xffffffffu, vec.w, 1) & 0xFFFF0000u;
            uint32_t rt = __shfl_down_sync(0xffffffffu, vec.x, 1) << 16;
            if (lane == 0)
                lf = 0u;
            if (v + 1 >= nvec)
                rt = 0u;
            if (edges) {
                const bool hv = tx >= xlo && tx <= xhi;
                if (lane == 0 && act && hv && v > 0)
                    lf = (uint32_t)__ldg(y16 + (long long)tx * W + 8 * v - 1) << 16;
                if (lane == 31 && act && hv && v + 1 < nvec)
                    rt = (uint32_t)__ldg(y16 + (long long)tx * W + 8 * v + 8) << 16;
            }
            dw_unpack_f(vec, lf, rt, u);
            ++tx;
            tslot = (tslot + 1) & (kDwRing - 1);
            fetch();
        };
        uint4* zrow = zp + (long long)hs * nvec + v;
        auto emit = [&](const DwRowF& u0, const DwRowF& u1, const DwRowF& u2) {
            const uint4 out = dw3x3_f8(u0, u1, u2, k);
            if (act)
                *zrow = out;
            zrow += nvec;
        };
        for (int i = 0; i < kDwRing; ++i)
            fetch();
        DwRowF ua, ub, uc;
        take(ua);
        take(ub);
        // three rows per pass, the unpacked rows rotating through ua, ub, uc
        for (int h = hs; h < he; h += 3) {
            take(uc);
            emit(ua, ub, uc);
            if (h + 1 >= he)
                break;
            take(ua);
            emit(ub, uc, ua);
            if (h + 2 >= he)
                break;
            take(ub);
            emit(uc, ua, ub);
        }
        cp_async_wait_group<0>();   // the ring is free before the next segment
    }
}

// ------------------------------------------------ bounded-wait self-test
__global__ void wait_selftest_kernel(unsigned long long cycles, int* status)
{
    grid_dep_wait();
    grid_dep_launch();
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: the wait must give up after `cycles`.
    if (threadIdx.x == 0)
        mbar_wait(&bar, 0, &abort_flag, cycles, status);
}

// ------------------------------------------------------------------ host
namespace {

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes)
{
    if (bytes <= 48 * 1024)
        return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

constexpr size_t kSimtSmemMax = 200 * 1024;

}  // namespace

namespace {

// one thread per 8 x 4*kDtgNCG block of G, in whole warps
int dtg_threads(const Geom& g)
{
    const int d = g.w * g.w, TV = 4 * kDtgNCG;
    return ((d + 7) / 8 * ((d + TV - 1) / TV) + 31) / 32 * 32;
}

size_t dtg_smem(const Geom& g)
{
    const int d = g.w * g.w, DP = (d + 4 * kDtgNCG - 1) / (4 * kDtgNCG) * (4 * kDtgNCG);
    // two stages of dY and x rows (G and the diagonal row sums fit in them),
    // then the column map
    return (size_t)4 * kCachedNT * DP * 4 + (size_t)kDtgMaxCols * 4;
}

// The register-tiled table gradient's plan: whole bands per tile, tiles per
// channel, blocks, and partial-table slots per channel.  A channel's tiles
// span at most 2 + (ntiles - 2) / (fewest tiles of a block) blocks: every
// block strictly inside the span covers that many of the channel's tiles.
// Returns false when the shape takes the table-bin kernel instead.
struct DtgPlan {
    int bpt, ntiles, grid, slots;
};

bool dtg_plan(const Geom& g, DtgPlan& pl)
{
    if (g.w < 4 || g.w > 14 || g.nw < 1 || g.nw > kCachedNT || g.bands < 1 || g.C < 1 ||
        g.nw * g.w > kDtgMaxCols || g.bands >= (1ll << 31) ||
        g.bands / g.nh * (long long)g.C >= (1ll << 31))
        return false;
    pl.bpt = kCachedNT / g.nw;
    const long long nt = (g.bands + pl.bpt - 1) / pl.bpt;
    const long long total = nt * g.C;
    if (nt > (1 << 30) || total >= (1ll << 31))
        return false;
    pl.ntiles = (int)nt;
    // blocks resident per SM, by shared memory (233472 bytes per SM, 1 KB
    // reserved per block), threads and registers (at most the launch
    // bound's share of 65536 per thread)
    const int threads = dtg_threads(g);
    const int regs = 65536 / kDtgMaxThreads / 8 * 8;
    int bps = (int)(233472 / (dtg_smem(g) + 1024));
    bps = std::min(bps, 2048 / threads);
    bps = std::max(1, std::min(bps, 65536 / (threads * regs)));
    const long long want = (long long)kDtgSMs * bps;
    pl.grid = (int)(total < want ? total : want);
    const long long fewest = total / pl.grid;
    const long long span = nt == 1 ? 1 : 2 + (nt - 2) / fewest;
    pl.slots = (int)(span < nt ? span : nt);
    return true;
}

}  // namespace

int simt_dt_chunks(const Geom& g)
{
    DtgPlan pl;
    if (dtg_plan(g, pl))
        return pl.slots;
    return (int)((g.bands + kSimtChunkBands - 1) / kSimtChunkBands);
}

namespace {

template <typename E, int WS, bool FLIP>
cudaError_t rows_launch_t(const Geom& g, const void* x, const void* T, void* y, const Launch& L)
{
    using F = RowCfg<WS>;
    const size_t band_bytes = (size_t)WS * g.W * 4;
    int rb = (int)((96 * 1024) / band_bytes);
    if (rb > 4)
        rb = 4;
    if (rb < 1)
        return cudaErrorInvalidConfiguration;
    const size_t smem = (size_t)F::TPAD * 4 + (size_t)rb * band_bytes;
    const int bands = (int)g.bands;
    const int groups = (bands + rb - 1) / rb;
    const long long blocks = (long long)g.C * groups;
    if (blocks == 0)
        return cudaSuccess;
    if (blocks > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    cudaError_t e = set_smem(simt_fwd_rows_kernel<E, WS, FLIP>, smem);
    if (e == cudaSuccess)
        e = launch_pdl(simt_fwd_rows_kernel<E, WS, FLIP>, dim3((unsigned)blocks), dim3(256), smem,
                       L.stream, static_cast<const E*>(x), static_cast<const E*>(T),
                       static_cast<E*>(y), g.C, g.H, g.W, g.nh, g.nw, bands, rb, groups);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

template <int WS>
cudaError_t rows_launch_w(const Geom& g, bool flip, bool is_bf16, const void* x, const void* T,
                          void* y, const Launch& L)
{
    if (is_bf16)
        return flip ? rows_launch_t<__nv_bfloat16, WS, true>(g, x, T, y, L)
                    : rows_launch_t<__nv_bfloat16, WS, false>(g, x, T, y, L);
    return flip ? rows_launch_t<float, WS, true>(g, x, T, y, L)
                : rows_launch_t<float, WS, false>(g, x, T, y, L);
}

// w = Is + 1 for Is = 0 .. 31
template <int... Is>
cudaError_t rows_dispatch(std::integer_sequence<int, Is...>, const Geom& g, bool flip,
                          bool is_bf16, const void* x, const void* T, void* y, const Launch& L)
{
    cudaError_t e = cudaErrorInvalidValue;
    ((g.w == Is + 1 ? (e = rows_launch_w<Is + 1>(g, flip, is_bf16, x, T, y, L), true) : false) ||
     ...);
    return e;
}

}  // namespace

cudaError_t simt_fwd_launch(const Geom& g, AMode mode, bool is_bf16, const void* x,
                            const void* src, void* y, const Launch& L)
{
    if (mode != kCached && g.w >= 1 && g.w <= 32 && (size_t)g.w * g.W * 4 <= 96 * 1024) {
        cudaError_t e = rows_dispatch(std::make_integer_sequence<int, 32>{}, g, mode == kTableFlip,
                                      is_bf16, x, src, y, L);
        if (e != cudaErrorInvalidValue)
            return e;
    }
    if (mode == kCached && g.w >= 3 && g.w <= 14 && g.nw <= kCachedNT) {
        const int d = g.d, DP = (d + 7) / 8 * 8;
        const size_t csmem = ((size_t)d * DP + (size_t)d * kCachedXS) * 4;
        const int bpt = kCachedNT / g.nw;         // whole bands per tile
        const int ntiles = (int)((g.bands + bpt - 1) / bpt);
        if (csmem <= kCachedSmemMax && ntiles > 0) {
            // about two blocks' worth of runs per SM, M_c loaded once per run
            int G = (2 * L.num_sms + g.C - 1) / g.C;
            if (G > ntiles)
                G = ntiles;
            const int tpb = (ntiles + G - 1) / G;
            const dim3 grid((unsigned)(g.C * G)), block((unsigned)(DP / 8 * 16));
            cudaError_t e;
            if (is_bf16) {
                using E = __nv_bfloat16;
                e = set_smem(simt_cached_kernel<E>, csmem);
                if (e == cudaSuccess)
                    e = launch_pdl(simt_cached_kernel<E>, grid, block, csmem, L.stream,
                                   static_cast<const E*>(x), static_cast<const E*>(src),
                                   static_cast<E*>(y), g.C, g.H, g.W, g.w, g.nh, g.nw, g.bands,
                                   bpt, ntiles, tpb, G);
            } else {
                e = set_smem(simt_cached_kernel<float>, csmem);
                if (e == cudaSuccess)
                    e = launch_pdl(simt_cached_kernel<float>, grid, block, csmem, L.stream,
                                   static_cast<const float*>(x), static_cast<const float*>(src),
                                   static_cast<float*>(y), g.C, g.H, g.W, g.w, g.nh, g.nw, g.bands,
                                   bpt, ntiles, tpb, G);
            }
            if (e != cudaSuccess)
                return e;
            note_launches(1);
            return cudaGetLastError();
        }
    }
    const size_t smem = ((mode == kCached ? 0 : (size_t)g.tsz) + (size_t)g.w * g.W) * 4;
    if (smem > kSimtSmemMax)
        return cudaErrorInvalidConfiguration;
    const long long blocks = (long long)g.B * g.C * g.nh;
    if (blocks == 0)
        return cudaSuccess;
    if (blocks > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)blocks), block(256);
    cudaError_t e;
    if (is_bf16) {
        using E = __nv_bfloat16;
        e = set_smem(simt_fwd_kernel<E>, smem);
        if (e == cudaSuccess)
            e = launch_pdl(simt_fwd_kernel<E>, grid, block, smem, L.stream,
                           static_cast<const E*>(x), static_cast<const E*>(src),
                           static_cast<E*>(y), g.C, g.H, g.W, g.w, g.nh, g.nw, (int)mode);
    } else {
        e = set_smem(simt_fwd_kernel<float>, smem);
        if (e == cudaSuccess)
            e = launch_pdl(simt_fwd_kernel<float>, grid, block, smem, L.stream,
                           static_cast<const float*>(x), static_cast<const float*>(src),
                           static_cast<float*>(y), g.C, g.H, g.W, g.w, g.nh, g.nw, (int)mode);
    }
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t simt_dt_launch(const Geom& g, bool is_bf16, const void* x, const void* dy,
                           float* partials, const Launch& L)
{
    DtgPlan pl;
    if (dtg_plan(g, pl)) {
        const int threads = dtg_threads(g);
        const size_t smem = dtg_smem(g);
        const dim3 grid((unsigned)pl.grid), block(threads);
        // two-element copies need even w and W and 8-byte aligned fp32 rows
        const bool pairs = g.w % 2 == 0 && g.W % 2 == 0 &&
                           ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy)) & 7) == 0;
        cudaError_t e;
        if (is_bf16) {
            using E = __nv_bfloat16;
            e = set_smem(simt_dtg_kernel<E, 1>, smem);
            if (e == cudaSuccess)
                e = launch_pdl(simt_dtg_kernel<E, 1>, grid, block, smem, L.stream,
                               static_cast<const E*>(x), static_cast<const E*>(dy), partials, g.C,
                               g.H, g.W, g.w, g.nh, g.nw, g.bands, pl.bpt, pl.ntiles, pl.slots);
        } else {
            auto kern = pairs ? simt_dtg_kernel<float, 2> : simt_dtg_kernel<float, 1>;
            e = set_smem(kern, smem);
            if (e == cudaSuccess)
                e = launch_pdl(kern, grid, block, smem, L.stream, static_cast<const float*>(x),
                               static_cast<const float*>(dy), partials, g.C, g.H, g.W, g.w, g.nh,
                               g.nw, g.bands, pl.bpt, pl.ntiles, pl.slots);
        }
        if (e != cudaSuccess)
            return e;
        note_launches(1);
        return cudaGetLastError();
    }
    const size_t smem = (size_t)2 * g.w * g.W * 4;
    // each thread owns up to kSimtMaxBinsPerThread table entries: 256 threads
    // cover w <= 32, 1024 threads every w the library accepts (<= 64)
    const int threads = g.tsz <= 256 * kSimtMaxBinsPerThread ? 256 : 1024;
    if (smem > kSimtSmemMax || g.tsz > threads * kSimtMaxBinsPerThread)
        return cudaErrorInvalidConfiguration;
    const int chunks = simt_dt_chunks(g);
    const long long blocks = (long long)g.C * chunks;
    if (blocks == 0)
        return cudaSuccess;
    const dim3 grid((unsigned)blocks), block(threads);
    cudaError_t e;
    if (is_bf16) {
        using E = __nv_bfloat16;
        e = set_smem(simt_dt_kernel<E>, smem);
        if (e == cudaSuccess)
            e = launch_pdl(simt_dt_kernel<E>, grid, block, smem, L.stream,
                           static_cast<const E*>(x), static_cast<const E*>(dy), partials, g.C,
                           g.H, g.W, g.w, g.nh, g.nw, g.bands, chunks);
    } else {
        e = set_smem(simt_dt_kernel<float>, smem);
        if (e == cudaSuccess)
            e = launch_pdl(simt_dt_kernel<float>, grid, block, smem, L.stream,
                           static_cast<const float*>(x), static_cast<const float*>(dy), partials,
                           g.C, g.H, g.W, g.w, g.nh, g.nw, g.bands, chunks);
    }
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t dt_finalize_launch(int C, int tsz, int chunks, const float* partials, float* dT,
                               const Launch& L)
{
    const long long n = (long long)C * tsz;
    if (n == 0)
        return cudaSuccess;
    cudaError_t e = launch_pdl(dt_finalize_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256),
                               0, L.stream, partials, dT, C, tsz, chunks);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t cache_matrices_launch(int C, int w, bool is_bf16, const void* T, void* M,
                                  const Launch& L)
{
    const long long total = (long long)C * w * w * w * w;
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)L.num_sms * 32)
        blocks = (long long)L.num_sms * 32;
    if (blocks < 1)
        return cudaSuccess;
    const dim3 grid((unsigned)blocks), block(256);
    cudaError_t e;
    if (is_bf16)
        e = launch_pdl(cache_kernel<uint16_t>, grid, block, 0, L.stream,
                       static_cast<const uint16_t*>(T), static_cast<uint16_t*>(M), C, w);
    else
        e = launch_pdl(cache_kernel<uint32_t>, grid, block, 0, L.stream,
                       static_cast<const uint32_t*>(T), static_cast<uint32_t*>(M), C, w);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t reparam_merge_launch(int C, int w, int k, bool is_bf16, const void* Tw,
                                 const void* Tk, void* M, const Launch& L)
{
    const long long total = (long long)C * w * w * w * w;
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)L.num_sms * 32)
        blocks = (long long)L.num_sms * 32;
    if (blocks < 1)
        return cudaSuccess;
    const dim3 grid((unsigned)blocks), block(256);
    cudaError_t e;
    if (is_bf16) {
        using E = __nv_bfloat16;
        e = launch_pdl(reparam_kernel<E>, grid, block, 0, L.stream, static_cast<const E*>(Tw),
                       static_cast<const E*>(Tk), static_cast<E*>(M), C, w, k);
    } else {
        e = launch_pdl(reparam_kernel<float>, grid, block, 0, L.stream,
                       static_cast<const float*>(Tw), static_cast<const float*>(Tk),
                       static_cast<float*>(M), C, w, k);
    }
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t dw3x3_launch(const Geom& g, bool is_bf16, const void* y, const void* K, void* z,
                         const Launch& L)
{
    if (is_bf16 && g.W % 8 == 0 && reinterpret_cast<uintptr_t>(y) % 16 == 0 &&
        reinterpret_cast<uintptr_t>(z) % 16 == 0) {
        const int chunks = (g.W / 8 + 31) / 32;
        const long long total_rows = (long long)g.B * g.C * chunks * g.H;
        // one pass of warps over the SMs; at least 8 rows per warp
        long long blocks = (long long)L.num_sms * kDwBlocksPerSm;
        const long long need = (total_rows + 8 * kDwWarps - 1) / (8 * kDwWarps);
        if (blocks > need)
            blocks = need;
        if (blocks > 0) {
            cudaError_t e = launch_pdl(dw3x3_bf16_rows_kernel, dim3((unsigned)blocks),
                                       dim3(kDwWarps * 32), kDwSmem, L.stream,
                                       static_cast<const uint16_t*>(y),
                                       static_cast<const uint16_t*>(K), static_cast<uint16_t*>(z),
                                       g.C, g.H, g.W, chunks, total_rows);
            if (e != cudaSuccess)
                return e;
            note_launches(1);
            return cudaGetLastError();
        }
    }
    const int ty = (g.H + kDwTH - 1) / kDwTH, tx = (g.W + kDwTW - 1) / kDwTW;
    const long long blocks = (long long)g.B * g.C * ty * tx;
    if (blocks == 0)
        return cudaSuccess;
    if (blocks > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)blocks), block(256);
    cudaError_t e;
    if (is_bf16) {
        using E = __nv_bfloat16;
        e = launch_pdl(dw3x3_kernel<E>, grid, block, 0, L.stream, static_cast<const E*>(y),
                       static_cast<const E*>(K), static_cast<E*>(z), g.C, g.H, g.W, ty, tx);
    } else {
        e = launch_pdl(dw3x3_kernel<float>, grid, block, 0, L.stream,
                       static_cast<const float*>(y), static_cast<const float*>(K),
                       static_cast<float*>(z), g.C, g.H, g.W, ty, tx);
    }
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t wait_selftest_launch(unsigned long long cycles, const Launch& L)
{
    cudaError_t e = launch_pdl(wait_selftest_kernel, dim3(1), dim3(32), 0, L.stream, cycles,
                               L.status);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace wbmm
