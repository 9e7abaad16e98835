// Host-side interface between the C ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

namespace wbmm {

// Geometry of one call.  Bands are the w-row strips of one image plane: band
// g = b*nh + i of channel c holds windows (b, i, 0..nw-1) and is w*W
// contiguous elements of the NCHW map.
struct Geom {
    int B, C, H, W, w;
    int nh, nw, d, tsz;
    long long bands;     // B * nh bands per channel
};

inline Geom make_geom(int B, int C, int H, int W, int w)
{
    Geom g;
    g.B = B; g.C = C; g.H = H; g.W = W; g.w = w;
    g.nh = H / w; g.nw = W / w; g.d = w * w; g.tsz = (2 * w - 1) * (2 * w - 1);
    g.bands = (long long)B * g.nh;
    return g;
}

// How the tensor-core kernel builds its A operand (the per-channel matrix).
enum AMode : int {
    kTable = 0,      // M_c[u][v] from the table (forward)
    kTableFlip = 1,  // M_c[v][u] from the table (input gradient)
    kCached = 2,     // M_c read from a [C][d][d] matrix in global memory
};

struct Launch {
    cudaStream_t stream;
    int num_sms;
    int* status;                  // device status word
    unsigned long long budget;    // bounded-wait budget, SM cycles
};

// Opaque storage for a CUtensorMap (128 bytes, 64-byte aligned), so kernel
// parameter structs can hold one without including the driver header.
struct alignas(64) TmapBytes {
    unsigned char b[128];
};

// Tensor maps (see wbmm_tmap.cu).  `map` points at a 64-byte aligned
// 128-byte CUtensorMap.  Returns false when the shape cannot use one.
int plane_row_elems(const Geom& g);
bool encode_plane_map(void* map, const void* base, const Geom& g, int k_images);

// tcgen05 forward family (x: bf16 map; src: table or matrices; dw: fused 3x3
// weights or null).  *_supported() must be checked before launching.
bool tc_fwd_supported(const Geom& g, bool fused);
cudaError_t tc_fwd_launch(const Geom& g, AMode mode, const void* x, const void* src, void* y,
                          const void* dw, const Launch& L);

// tcgen05 forward / input gradient from the table, windows as the MMA's M
// dimension (mode kTable or kTableFlip only).
bool tc_toep_supported(const Geom& g);
cudaError_t tc_toep_launch(const Geom& g, AMode mode, const void* x, const void* T, void* y,
                           const Launch& L);

// tcgen05 forward / input gradient for w = 28 from the table, windows as the
// MMA's N dimension and a per-channel Toeplitz stack as A (mode kTable or
// kTableFlip only).
bool tc_big_supported(const Geom& g);
cudaError_t tc_big_launch(const Geom& g, AMode mode, const void* x, const void* T, void* y,
                          const Launch& L);

// tcgen05 forward with a cached [C][d][d] matrix, windows as the MMA's M
// dimension; with dw (fuse) the epilogue applies the 3x3 mixing and y is z.
bool tc_cached_supported(const Geom& g, bool fuse);
cudaError_t tc_cached_launch(const Geom& g, const void* x, const void* M, const void* dw, void* y,
                             const Launch& L);

// tcgen05 table gradient: one contiguous tile range per CTA.  The workspace
// (tc_dt_workspace_floats floats) starts with WBMM_DT_COUNTER_WORDS 32-bit
// arrival counters (one per channel; zero before the first launch, and every
// launch leaves them zero), followed by the fp32 partial tables of channels
// split between CTAs.
// after_dx: the previous launch on the stream is the same backward call's
// input-gradient kernel (which reads dY and T and writes only dX), so the
// kernel need not wait for it to finish.  The grid is min(L.num_sms, 256,
// tiles); tc_dt_tiles is the number of 64-window (32 at w >= 15) tiles.
bool tc_dt_supported(const Geom& g);
long long tc_dt_partials(const Geom& g);
long long tc_dt_tiles(const Geom& g);
long long tc_dt_workspace_floats(const Geom& g);
cudaError_t tc_dt_launch(const Geom& g, const void* x, const void* dy, float* workspace, float* dT,
                         bool after_dx, const Launch& L);

// CUDA-core kernels.  is_bf16 selects the element type of every map/table.
int simt_dt_chunks(const Geom& g);
cudaError_t simt_fwd_launch(const Geom& g, AMode mode, bool is_bf16, const void* x,
                            const void* src, void* y, const Launch& L);
cudaError_t simt_dt_launch(const Geom& g, bool is_bf16, const void* x, const void* dy,
                           float* partials, const Launch& L);
cudaError_t dt_finalize_launch(int C, int tsz, int chunks, const float* partials, float* dT,
                               const Launch& L);
cudaError_t cache_matrices_launch(int C, int w, bool is_bf16, const void* T, void* M,
                                  const Launch& L);
cudaError_t reparam_merge_launch(int C, int w, int k, bool is_bf16, const void* Tw,
                                 const void* Tk, void* M, const Launch& L);
cudaError_t dw3x3_launch(const Geom& g, bool is_bf16, const void* y, const void* K, void* z,
                         const Launch& L);
cudaError_t wait_selftest_launch(unsigned long long cycles, const Launch& L);

void note_launches(int n);

// Launches `kernel` with programmatic stream serialization: it may begin its
// prologue while the previous kernel in the stream drains, and every library
// kernel calls grid_dep_wait() before reading or writing tensors.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch settings (stream, SM count, status word, wait budget) for the
// current device; returns a wbmm_status code (0 on success).
int launch_for_stream(void* stream, Launch* L);

// Test-only settings of wbmm_debug_set.  debug_take_skip(family) returns the
// tile (in CTA 0's order) whose load the next launch of the family skips and
// clears it (-1: none; family 0 = window-major forward / input gradient,
// 1 = table gradient); debug_ring_cap() caps the load ring (0: no cap).
int debug_take_skip(int family);
int debug_ring_cap();

}  // namespace wbmm
