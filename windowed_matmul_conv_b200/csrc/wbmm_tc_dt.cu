// Tensor-core (tcgen05) WBMM table gradient.
//
// For one channel, G = dY X^T is a matrix over in-window positions summed
// over windows:
//   G[u, v] = sum_n dY[u, n] X[v, n]        (u, v in-window positions)
// and the table gradient is its sum along constant relative offset:
//   dT[(p-r+w-1)(2w-1) + (q-s+w-1)] = sum over (u=(p,q), v=(r,s)) of G[u, v].
//
// The channels' tiles, in channel order, are split into one contiguous,
// balanced range per CTA: of whole channels when that gives no CTA more tiles
// than a split at tile granularity, else of tiles.  A segment is the part of a
// CTA's range inside one channel; each segment ends with one reduction of G
// into its own fp32 partial table.  A channel inside one CTA's range is
// written to dT directly.  A channel split between CTAs k0 < ... < k1 is
// finished by whichever of them arrives last: each writes its segment's
// partial table (at index c + k of the workspace's tables: ranges are
// ordered, so the index is unique) and then adds one to the channel's arrival
// counter
// (acquire-release, device scope); the CTA that sees the count reach
// k1 - k0 + 1 adds the partial tables in CTA order k0, ..., k1 into dT and
// sets the counter back to zero.  No CTA ever waits for another, so the grid
// need not be co-resident, and a counter can only reach its final count
// within one launch: a re-launch with the same arguments (a replayed graph)
// never sees the previous launch's partials as ready.  Every counter starts
// at zero (the workspace's counter region must be zero before its first use)
// and every launch leaves it zero, the aborted ones included, since each CTA
// arrives once per split channel whether or not its waits succeeded.  Every
// sum runs in a fixed order, so the result is bit-identical from run to run
// for a given grid (the device's SM count).
//
// Per tile the producer bulk-copies the dY and x bands into a raw slot; the
// transform warps write both tiles in the layout of the forward kernel's
// operand (rows = windows, 16-byte rows of 8 padded positions); warps 2..9 do this.  Read as an
// MN-major operand that layout has positions as M (or N) and windows as K,
// so one thread issues 128 x NPOS x 16 MMAs (A = dY tile, B = x tile) into G
// in TMEM (two 128-row halves when the padded positions exceed 128).  After
// the segment's last tile eight epilogue warps reduce G one 128-row half at a
// time: every (p, r) block of G (image rows p and r, RP x RP entries) is
// summed along its diagonals q - s in registers and written once to a
// staging array [p][r][q - s]; the half is then released to the next segment's
// MMAs, and each thread adds the staged sums of the table entries it owns
// (fixed p order) into registers.  The last half's sums are the segment's
// partial table.
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "wbmm.h"
#include "tc_common.cuh"
#include "wbmm_internal.h"

namespace wbmm {

constexpr uint32_t kSmemMax = 232448;
constexpr int kDtRingMax = 8;
constexpr int kDtXformWarps = 8;                 // warps 2..9
constexpr int kDtEpiWarp0 = 2 + kDtXformWarps;  // warps 10..17
constexpr int kDtEpiWarps = 8;
constexpr int kDtEpiThreads = kDtEpiWarps * 32;
constexpr int kDtThreads = (kDtEpiWarp0 + kDtEpiWarps) * 32;

// Image rows p of G per 128-row half, and the staging array of one half:
// fp32 [p][r][2*RP] with diagonal q - s = b at slot b + RP; the row of each p
// is padded so that the 32/RP image rows a warp holds start RP banks apart
// and one store instruction of the warp never conflicts.
__host__ __device__ constexpr int dt_rows_per_half(int ws)
{
    const int pl = 128 / ((ws + 7) / 8 * 8);
    return pl < ws ? pl : ws;
}
__host__ __device__ constexpr int dt_stg_stride(int ws)
{
    const int rp = (ws + 7) / 8 * 8;
    return ws * 2 * rp + (rp - (ws * 2 * rp) % 32 + 32) % 32;
}
constexpr uint32_t dt_stg_bytes(int ws)
{
    return (uint32_t)(128 / ((ws + 7) / 8 * 8)) * dt_stg_stride(ws) * 4;
}

// Windows per tile (the MMA K of one stage): 64, or 32 for w = 16 where two
// 64-window stages and two raw slots do not fit.  (Measured at w = 14: 32-
// window tiles with a six-deep ring run ~10% slower than 64-window tiles.)
constexpr int dt_nt_for(int ws) { return ws >= 15 ? 32 : 64; }

template <int WS>
struct DtCfg : PadCfg<WS> {
    using P = PadCfg<WS>;
    static constexpr int NT = dt_nt_for(WS);               // windows per tile = K per stage
    static constexpr int MT = (P::K + 127) / 128;           // 128-row halves of G
    static constexpr int NPOS = P::KP;                      // MMA N: padded positions of x
    static constexpr uint32_t SBO_T = (uint32_t)(P::KP * 16);   // 8-window group stride
    static constexpr uint32_t TILE_BYTES = (uint32_t)(NT * P::KP * 2);
    static constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;     // dY tile, then x tile
    static constexpr uint32_t RAW_HALF = (uint32_t)((NT * P::D * 2 + 127) / 128 * 128);
    static constexpr uint32_t RAW_BYTES = 2 * RAW_HALF;
    // kind::f16, bf16 A and B, both MN-major (positions contiguous), fp32 D
    static constexpr uint32_t IDESC = idesc_bf16(128, NPOS) | (1u << 15) | (1u << 16);
    static_assert(NPOS <= 256 && MT <= 2, "G must fit in TMEM");
};

struct TcDtParams {
    TmapBytes map_x;        // whole-plane tensor maps (used when use_tmap)
    TmapBytes map_dy;
    const uint16_t* x;
    const uint16_t* dy;
    float* partials;        // [C + grid - 1][tsz], segment (c, k) at c + k
    unsigned int* counters; // [C] segments of channel c written so far (zero between launches)
    float* dT;              // [C][tsz]
    int C, H, W, nh, nw;
    int bpt;
    int tpc;                // tiles per channel
    int bands;
    int rq, rr;             // range split: CTA k gets rq + (k < rr) units
    int unit;               // tiles per unit: 1, or tpc (whole channels)
    int dep_wait;           // 1: wait for the previous kernel before any load;
                            // 0: the previous kernel is the same call's input
                            // gradient, which writes nothing this one touches,
                            // so the wait moves to the end of the kernel
    int use_tmap;           // tiles are whole planes: one 4-D TMA per tensor
    int kimg;               // planes per tile when use_tmap
    int R;                  // raw ring depth (tiles)
    uint32_t off_raw, off_stage, off_stg, off_woff, off_bar;
    int skip_seq;           // test only: CTA 0 skips this tile's load (-1: none)
    unsigned long long budget;
    int* status;
};

struct DtBars {
    uint64_t raw_full[kDtRingMax];
    uint64_t raw_empty[kDtRingMax];
    uint64_t st_full[2];
    uint64_t st_empty[2];
    uint64_t g_full;
    uint64_t g_empty[2];    // per 128-row half of G
    uint64_t fin;
    uint32_t tmem_slot;
    int abort;
    int last;               // this CTA is the last to arrive at the current split channel
};

struct DtTile {
    BandTile bt;
    bool first, last;   // first / last tile of its segment
};

// The CTA whose range holds tile t (inverse of dt_range).
__device__ __forceinline__ int dt_cta_of(const TcDtParams& P, long long t)
{
    const long long u = t / P.unit;
    const long long big = (long long)P.rr * (P.rq + 1);
    return (int)(u < big ? u / (P.rq + 1) : P.rr + (u - big) / P.rq);
}

// The tile range of a CTA: [t0, t1) of the channel-major tile sequence.
__device__ __forceinline__ void dt_range(const TcDtParams& P, int& t0, int& t1)
{
    const int k = (int)blockIdx.x;
    t0 = (k * P.rq + (k < P.rr ? k : P.rr)) * P.unit;
    t1 = t0 + (P.rq + (k < P.rr ? 1 : 0)) * P.unit;
}

// Every role walks the CTA's range in the same order.
struct DtWalker {
    int t, t0, t1;
    __device__ __forceinline__ bool valid(const TcDtParams&) const { return t < t1; }
    __device__ __forceinline__ void start(const TcDtParams& P)
    {
        dt_range(P, t0, t1);
        t = t0;
    }
    __device__ __forceinline__ DtTile get(const TcDtParams& P) const
    {
        DtTile d;
        d.bt.c = t / P.tpc;
        const int tile = t - d.bt.c * P.tpc;
        d.bt.band0 = tile * P.bpt;
        const int left = P.bands - d.bt.band0;
        d.bt.nb = left < P.bpt ? left : P.bpt;
        d.first = t == t0 || tile == 0;
        d.last = t + 1 == t1 || tile + 1 == P.tpc;
        return d;
    }
    __device__ __forceinline__ void next(const TcDtParams&) { ++t; }
};

template <int WS>
__global__ void __launch_bounds__(kDtThreads, 1) wbmm_tc_dt_kernel(const __grid_constant__ TcDtParams P)
{
    using F = DtCfg<WS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* raw_base = smem + P.off_raw;
    uint8_t* st_base = smem + P.off_stage;
    float* stg = reinterpret_cast<float*>(smem + P.off_stg);
    int* woff = reinterpret_cast<int*>(smem + P.off_woff);
    DtBars& S = *reinterpret_cast<DtBars*>(smem + P.off_bar);
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDtRingMax; ++i) {
            mbar_init(&S.raw_full[i], 1);
            mbar_init(&S.raw_empty[i], kDtXformWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.st_full[i], kDtXformWarps);
            mbar_init(&S.st_empty[i], 1);
        }
        mbar_init(&S.g_full, 1);
        mbar_init(&S.g_empty[0], kDtEpiWarps);
        mbar_init(&S.g_empty[1], kDtEpiWarps);
        mbar_init(&S.fin, 1);
        S.abort = 0;
        fence_mbar_init();
    }
    for (int n = threadIdx.x; n < F::NT; n += kDtThreads) {
        const int k = n / P.nw, j = n - k * P.nw;
        woff[n] = k * WS * P.W + j * WS;
    }
    // Operand stages start as zeros (padding slots are never written).
    for (uint32_t e = threadIdx.x; e < 2 * F::STAGE_BYTES / 16; e += kDtThreads)
        reinterpret_cast<uint4*>(st_base)[e] = make_uint4(0u, 0u, 0u, 0u);
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
    // and written only after it has completed.  The input-gradient kernel of
    // the same backward call is the exception: it signals this launch only
    // after its own wait, so whatever produced dY and x is complete, and it
    // writes nothing this kernel touches.
    if (P.dep_wait)
        grid_dep_wait();
    grid_dep_launch();

    if (warp == 0) {
        // ------------------------------------------------------ producer
        // Lane 0 arms the slot's barrier; the lanes issue one run each.
        int issued = 0, seq = 0;
        DtWalker it;
        for (it.start(P); it.valid(P); it.next(P), ++seq) {
            const int s = seq % P.R;
            bool ok = !*abort;
            if (seq >= P.R)
                ok = ok && mbar_wait(&S.raw_empty[s], ((seq / P.R) - 1) & 1, abort, P.budget,
                                     P.status);
            if (!__all_sync(0xffffffffu, ok))
                break;
            const DtTile t = it.get(P);
            uint8_t* slot = raw_base + (size_t)s * F::RAW_BYTES;
            if (seq == P.skip_seq && blockIdx.x == 0) {
                // test only: the slot is never armed, so the transform's
                // bounded wait for it runs out
                issued = seq + 1;
                continue;
            }
            if (P.use_tmap) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&S.raw_full[s], 2u * P.kimg * WS * P.W * P.nh * 2);
                    tma_load_4d(slot, &P.map_dy, 0, 0, t.bt.c, t.bt.band0 / P.nh, &S.raw_full[s]);
                    tma_load_4d(slot + F::RAW_HALF, &P.map_x, 0, 0, t.bt.c, t.bt.band0 / P.nh,
                                &S.raw_full[s]);
                }
                issued = seq + 1;
                continue;
            }
            if (lane == 0)
                mbar_arrive_expect_tx(&S.raw_full[s], 2u * t.bt.nb * WS * P.W * 2);
            __syncwarp();
            const BandRuns runs = band_runs(t.bt, P.nh);
            for (int l = lane; l < runs.count; l += 32) {
                long long goff;
                uint32_t soff, nbytes;
                band_run(t.bt, runs, l, WS, P.W, P.H, P.C, P.nh, goff, soff, nbytes);
                bulk_g2s(slot + soff, P.dy + goff, nbytes, &S.raw_full[s]);
                bulk_g2s(slot + F::RAW_HALF + soff, P.x + goff, nbytes, &S.raw_full[s]);
            }
            issued = seq + 1;
        }
        if (lane == 0) {
            for (int s = 0; s < P.R && s < issued; ++s) {
                const int last = s + ((issued - 1 - s) / P.R) * P.R;
                mbar_wait_drain(&S.raw_full[s], (last / P.R) & 1, P.budget, P.status);
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
                if (t.first)
                    ok_item = true;
                ok = ok && mbar_wait(&S.st_full[bs], (seq >> 1) & 1, abort, P.budget, P.status);
                ok_item = ok_item && ok;
                if (ok) {
                    const uint32_t a_addr = smem_u32(st_base + (size_t)bs * F::STAGE_BYTES);
                    const uint32_t b_addr = a_addr + F::TILE_BYTES;
                    const int nwin = t.bt.nb * P.nw;
                    const int ksteps = (nwin + 15) >> 4;
#pragma unroll
                    for (int mt = 0; mt < F::MT; ++mt) {
                        // the previous item's reduction hands G over one
                        // 128-row half at a time
                        if (t.first && item_seq > 0)
                            ok = ok && mbar_wait(&S.g_empty[mt], (item_seq - 1) & 1, abort,
                                                 P.budget, P.status);
                        if (!ok)
                            break;
                        tc_fence_after();
#pragma unroll 1
                        for (int k = 0; k < ksteps; ++k) {
                            // MN-major: LBO = window-group stride, SBO = position-group stride
                            const uint64_t adesc =
                                smem_desc(a_addr + mt * 16 * 128 + k * 2 * F::SBO_T, F::SBO_T, 128);
                            const uint64_t bdesc =
                                smem_desc(b_addr + k * 2 * F::SBO_T, F::SBO_T, 128);
                            mma_ss(tmem + (uint32_t)(mt * 256), adesc, bdesc, F::IDESC,
                                   (t.first && k == 0) ? 0u : 1u);
                        }
                    }
                    if (ok)
                        tc_commit(&S.st_empty[bs]);
                    ok_item = ok_item && ok;
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
    } else if (warp < kDtEpiWarp0) {
        // ------------------------------------------------------ transform
        const int tt = threadIdx.x - 64;
        int seq = 0;
        DtWalker it;
        for (it.start(P); it.valid(P); it.next(P), ++seq) {
            const DtTile t = it.get(P);
            const int s = seq % P.R, bs = seq & 1;
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.raw_full[s], (seq / P.R) & 1, abort, P.budget, P.status);
            if (seq >= 2)
                ok = ok && mbar_wait(&S.st_empty[bs], ((seq >> 1) - 1) & 1, abort, P.budget,
                                     P.status);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                const uint16_t* raw =
                    reinterpret_cast<const uint16_t*>(raw_base + (size_t)s * F::RAW_BYTES);
                uint8_t* stage = st_base + (size_t)bs * F::STAGE_BYTES;
                const int nwin = t.bt.nb * P.nw;
                const int nzero = (nwin + 15) & ~15;    // last MMA K step reads up to here
                transform_rows_pair<WS>(raw, stage, raw + F::RAW_HALF / 2, stage + F::TILE_BYTES,
                                        F::SBO_T, nwin, nzero, woff, P.W, tt,
                                        kDtXformWarps * 32);
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
        // Two warps per TMEM lane quarter; warp half h takes the 32-column
        // chunks h, h+2, ... of its 32 rows of G.  With positions padded to
        // RP slots per image row, the 32 lanes are 32/RP segments of one image
        // row p each, and a chunk is 32/RP blocks of one column row r each.
        // The diagonal sums of an RP x RP block (fixed p, r) come from
        // width-RP shuffles: lane L takes column s from lane (L+s)%RP, an
        // entry of diagonal q - s = L (no wrap) or L - RP (wrap), and adds it
        // to one of two sums in ascending s; both sums are staged with
        // unconditional stores (slots of invalid diagonals are never read).
        // Columns s >= w are zero padding and are skipped.
        constexpr int RP = F::RP;
        constexpr int NB = 32 / RP;                  // blocks (r values) per chunk
        constexpr int NCH = (F::NPOS + 31) / 32;     // chunks per row (last may overhang)
        constexpr int L2 = 2 * WS - 1;
        constexpr int PL = dt_rows_per_half(WS);     // image rows p per half
        constexpr int SP = dt_stg_stride(WS);        // staging floats per image row p
        constexpr int NBT = (F::TSZ + kDtEpiThreads - 1) / kDtEpiThreads;
        const int quarter = warp & 3;
        const int h = (warp - kDtEpiWarp0) >> 2;
        const int et = threadIdx.x - kDtEpiWarp0 * 32;
        const int L = lane & (RP - 1);
        int t0, t1;
        dt_range(P, t0, t1);
        const int c_first = t0 / P.tpc, c_last = (t1 - 1) / P.tpc;
        int item_seq = 0;
        for (int c = c_first; c <= c_last; ++c, ++item_seq) {
            bool ok = !*abort;
            ok = ok && mbar_wait(&S.g_full, item_seq & 1, abort, P.budget, P.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            const int k = (int)blockIdx.x;
            const int k0 = dt_cta_of(P, (long long)c * P.tpc);
            const int k1 = dt_cta_of(P, (long long)c * P.tpc + P.tpc - 1);
            float acc[NBT];
#pragma unroll
            for (int i = 0; i < NBT; ++i)
                acc[i] = 0.0f;
#pragma unroll 1
            for (int mt = 0; mt < F::MT; ++mt) {
                const int ubase = mt * 128 + quarter * 32;
                // warp-uniform: rows past the last image row are padding
                if (ok && ubase / RP < WS && h < NCH) {
                    const uint32_t gcol =
                        tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(mt * 256);
#pragma unroll 1
                    for (int ch = h; ch < NCH; ch += 2) {
                        uint32_t r[32];
                        tmem_ld32(gcol + (uint32_t)(ch * 32), r);
                        tmem_wait_ld(r);
                        float v[32];
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            v[jj] = __uint_as_float(r[jj]);
#pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            const int rr = ch * NB + b;
                            if (rr < WS) {
                                float a = 0.0f, wrap = 0.0f;
#pragma unroll
                                for (int s = 0; s < WS; ++s) {
                                    const float g = __shfl_sync(0xffffffffu, v[b * RP + s],
                                                                (L + s) & (RP - 1), RP);
                                    if (L + s < RP)
                                        a += g;
                                    else
                                        wrap += g;
                                }
                                float* row = stg + ((ubase - mt * 128 + lane) / RP) * SP + rr * 2 * RP;
                                row[L + RP] = a;
                                row[L] = wrap;
                            }
                        }
                    }
                }
                // this half of G has been read: the next item's MMAs may
                // overwrite it while the staged sums are added up
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&S.g_empty[mt]);
                named_bar_sync(3, kDtEpiThreads);
                if (ok) {
                    // the thread's bins are independent chains: interleave them
                    int da[NBT], off[NBT];
#pragma unroll
                    for (int i = 0; i < NBT; ++i) {
                        const int bin = et + i * kDtEpiThreads;
                        const int bb = bin < F::TSZ ? bin : 0;
                        da[i] = bin < F::TSZ ? bb / L2 - (WS - 1) : 4 * WS;   // out of range: no adds
                        off[i] = bb - (bb / L2) * L2 - (WS - 1) + RP;
                    }
                    const int p0 = mt * PL;
#pragma unroll
                    for (int j = 0; j < PL; ++j) {
                        const int pp = p0 + j;
                        if (pp < WS) {
#pragma unroll
                            for (int i = 0; i < NBT; ++i) {
                                const int rr = pp - da[i];
                                if (rr >= 0 && rr < WS)
                                    acc[i] += stg[j * SP + rr * 2 * RP + off[i]];
                            }
                        }
                    }
                }
                named_bar_sync(3, kDtEpiThreads);
            }
            if (k0 == k1) {
                // the whole channel is in this CTA's range
                if (ok) {
                    float* out = P.dT + (long long)c * F::TSZ;
#pragma unroll
                    for (int i = 0; i < NBT; ++i) {
                        const int bin = et + i * kDtEpiThreads;
                        if (bin < F::TSZ)
                            out[bin] = acc[i];
                    }
                }
                continue;
            }
            // a channel split between CTAs: publish this segment's partial
            // table, then count it; the last CTA to arrive adds all of them
            {
                float* out = P.partials + (long long)(c + k) * F::TSZ;
#pragma unroll
                for (int i = 0; i < NBT; ++i) {
                    const int bin = et + i * kDtEpiThreads;
                    if (bin < F::TSZ)
                        out[bin] = acc[i];
                }
            }
            __threadfence();
            named_bar_sync(3, kDtEpiThreads);
            if (et == 0) {
                const unsigned int prev = atom_add_acq_rel_u32(P.counters + c, 1u);
                const int last = prev == (unsigned int)(k1 - k0);
                if (last)
                    atomicExch(P.counters + c, 0u);   // zero again for the next launch
                S.last = last;
            }
            named_bar_sync(3, kDtEpiThreads);
            if (S.last && ok) {
                __threadfence();
#pragma unroll
                for (int i = 0; i < NBT; ++i) {
                    const int bin = et + i * kDtEpiThreads;
                    if (bin < F::TSZ) {
                        const float* pc = P.partials + (long long)c * F::TSZ + bin;
                        float sum = k0 == k ? acc[i] : __ldcg(pc + (long long)k0 * F::TSZ);
                        for (int kk = k0 + 1; kk <= k1; ++kk)
                            sum += kk == k ? acc[i] : __ldcg(pc + (long long)kk * F::TSZ);
                        P.dT[(long long)c * F::TSZ + bin] = sum;
                    }
                }
            }
            named_bar_sync(3, kDtEpiThreads);   // S.last is rewritten next
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
    // Without the wait at the start, this grid could finish before the
    // input-gradient kernel launched ahead of it; a later kernel in the
    // stream that waits only for this grid would then see dX incomplete.
    // Waiting here makes this grid's completion imply the earlier one's.
    if (!P.dep_wait)
        grid_dep_wait();
}

// ------------------------------------------------------------------ host
namespace {

constexpr uint32_t kMinSmem = 120 * 1024;
inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

struct DtLayout {
    uint32_t off_raw, off_stage, off_stg, off_woff, off_bar, total;
    int R;
};

// Operand stages | staging array | window offsets | barriers | raw ring,
// as many raw slots as fit (at most kDtRingMax).
template <int WS>
DtLayout dt_layout()
{
    using F = DtCfg<WS>;
    DtLayout L;
    uint32_t off = 0;
    L.off_stage = off;
    off += 2 * F::STAGE_BYTES;
    L.off_stg = align_up(off, 16);
    off = L.off_stg + dt_stg_bytes(WS);
    L.off_woff = align_up(off, 16);
    off = L.off_woff + F::NT * 4;
    L.off_bar = align_up(off, 16);
    off = L.off_bar + sizeof(DtBars);
    L.off_raw = align_up(off, 128);
    const uint32_t avail = kSmemMax - 1024 > L.off_raw ? kSmemMax - 1024 - L.off_raw : 0;
    int R = (int)(avail / F::RAW_BYTES);
    L.R = R < kDtRingMax ? R : kDtRingMax;
    const int cap = debug_ring_cap();
    if (cap >= 2 && L.R > cap)
        L.R = cap;
    off = L.off_raw + (uint32_t)L.R * F::RAW_BYTES;
    L.total = align_up(off, 1024);
    // at least half the SM's shared memory: one CTA (and one 512-column TMEM
    // allocation) per SM
    if (L.total < kMinSmem)
        L.total = kMinSmem;
    return L;
}

// Largest grid of the table-gradient kernel: bounds the number of partial
// tables (C + grid - 1) without knowing the device.
constexpr int kDtMaxGrid = 256;

long long tc_dt_partials_impl(const Geom& g);

int dt_tiles_per_channel(const Geom& g)
{
    const int bpt = dt_nt_for(g.w) / g.nw;
    return (int)((g.bands + bpt - 1) / bpt);
}

long long tc_dt_partials_impl(const Geom& g)
{
    const long long tiles = (long long)g.C * dt_tiles_per_channel(g);
    return g.C + (tiles < kDtMaxGrid ? tiles : kDtMaxGrid) - 1;
}

template <int WS>
cudaError_t dt_launch_ws(const Geom& g, const void* x, const void* dy, float* workspace,
                         float* dT, bool after_dx, const Launch& L)
{
    using F = DtCfg<WS>;
    const DtLayout lay = dt_layout<WS>();
    if (lay.total > kSmemMax || lay.R < 2)
        return cudaErrorInvalidConfiguration;
    static unsigned long long configured = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(configured & (1ull << (dev & 63)))) {
        cudaError_t e = cudaFuncSetAttribute(wbmm_tc_dt_kernel<WS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemMax);
        if (e != cudaSuccess)
            return e;
        configured |= 1ull << (dev & 63);
    }
    TcDtParams P;
    P.x = static_cast<const uint16_t*>(x);
    P.dy = static_cast<const uint16_t*>(dy);
    P.counters = reinterpret_cast<unsigned int*>(workspace);
    P.partials = workspace + WBMM_DT_COUNTER_WORDS;
    P.dT = dT;
    P.C = g.C; P.H = g.H; P.W = g.W; P.nh = g.nh; P.nw = g.nw;
    P.bpt = F::NT / g.nw;
    P.bands = (int)g.bands;
    P.tpc = (P.bands + P.bpt - 1) / P.bpt;
    const int tiles = g.C * P.tpc;
    int grid = L.num_sms < kDtMaxGrid ? L.num_sms : kDtMaxGrid;
    if (grid > tiles)
        grid = tiles;
    if (grid < 1)
        return cudaSuccess;
    // Ranges of whole channels when that costs a CTA no more tiles than the
    // tile-granular split (no channel is then shared between CTAs: one
    // reduction of G per channel, no partial tables), else tile ranges.
    const int per_tile = (tiles + grid - 1) / grid;
    const int per_chan = (g.C + grid - 1) / grid * P.tpc;
    if (g.C >= grid && per_chan <= per_tile) {
        P.unit = P.tpc;
        P.rq = g.C / grid;
        P.rr = g.C - P.rq * grid;
    } else {
        P.unit = 1;
        P.rq = tiles / grid;
        P.rr = tiles - P.rq * grid;
    }
    P.dep_wait = after_dx ? 0 : 1;
    P.use_tmap = 0;
    P.kimg = 0;
    if (P.bpt % g.nh == 0) {
        const int k = P.bpt / g.nh;
        if (encode_plane_map(&P.map_x, x, g, k) && encode_plane_map(&P.map_dy, dy, g, k)) {
            P.use_tmap = 1;
            P.kimg = k;
        }
    }
    P.R = lay.R;
    P.off_raw = lay.off_raw; P.off_stage = lay.off_stage; P.off_stg = lay.off_stg;
    P.off_woff = lay.off_woff; P.off_bar = lay.off_bar;
    P.budget = L.budget;
    P.status = L.status;
    P.skip_seq = debug_take_skip(1);
    cudaError_t e = launch_pdl(wbmm_tc_dt_kernel<WS>, dim3(grid), dim3(kDtThreads), lay.total,
                               L.stream, P);
    if (e != cudaSuccess)
        return e;
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

bool tc_dt_supported(const Geom& g)
{
    if (g.w < 2 || g.w > 16)
        return false;
    if (g.nw > dt_nt_for(g.w))
        return false;
    if (((long long)g.w * g.W * 2) % 16 != 0)
        return false;
    if (g.bands * (long long)g.C >= (1ll << 31))
        return false;
    if (g.C > WBMM_DT_COUNTER_WORDS)
        return false;
    return true;
}

long long tc_dt_partials(const Geom& g)
{
    return tc_dt_partials_impl(g);
}

long long tc_dt_tiles(const Geom& g)
{
    return (long long)g.C * dt_tiles_per_channel(g);
}

long long tc_dt_workspace_floats(const Geom& g)
{
    // a fixed region of arrival counters (one per channel, the same words for
    // every shape, so a workspace shared by calls of different shapes keeps
    // them zero), then the partial tables
    return WBMM_DT_COUNTER_WORDS + tc_dt_partials(g) * g.tsz;
}

cudaError_t tc_dt_launch(const Geom& g, const void* x, const void* dy, float* partials, float* dT,
                         bool after_dx, const Launch& L)
{
    switch (g.w) {
    case 2: return dt_launch_ws<2>(g, x, dy, partials, dT, after_dx, L);
    case 3: return dt_launch_ws<3>(g, x, dy, partials, dT, after_dx, L);
    case 4: return dt_launch_ws<4>(g, x, dy, partials, dT, after_dx, L);
    case 5: return dt_launch_ws<5>(g, x, dy, partials, dT, after_dx, L);
    case 6: return dt_launch_ws<6>(g, x, dy, partials, dT, after_dx, L);
    case 7: return dt_launch_ws<7>(g, x, dy, partials, dT, after_dx, L);
    case 8: return dt_launch_ws<8>(g, x, dy, partials, dT, after_dx, L);
    case 9: return dt_launch_ws<9>(g, x, dy, partials, dT, after_dx, L);
    case 10: return dt_launch_ws<10>(g, x, dy, partials, dT, after_dx, L);
    case 11: return dt_launch_ws<11>(g, x, dy, partials, dT, after_dx, L);
    case 12: return dt_launch_ws<12>(g, x, dy, partials, dT, after_dx, L);
    case 13: return dt_launch_ws<13>(g, x, dy, partials, dT, after_dx, L);
    case 14: return dt_launch_ws<14>(g, x, dy, partials, dT, after_dx, L);
    case 15: return dt_launch_ws<15>(g, x, dy, partials, dT, after_dx, L);
    case 16: return dt_launch_ws<16>(g, x, dy, partials, dT, after_dx, L);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace wbmm
