// Table gradient without caller-provided or library-allocated scratch.
//
// Some callers cannot allocate device memory at the point where they need
// the table gradient: hosts with a fixed device-memory budget set at start-up
// (real-time or embedded deployments), plugins running inside a framework that
// owns every device allocation, and code paths where a cudaMalloc would
// synchronise the device.  wbmm_backward_dt_static serves them: it computes
// the same dT as wbmm_backward, with its per-chunk partial tables in a
// file-scope device array instead of a workspace argument.
//
// The array is kStaticPartials floats (4 MiB), laid out like a workspace of
// wbmm_backward: its first words are the tensor-core path's per-channel
// arrival counters, which start at zero (a __device__ array is zero-filled
// when the library loads) and which every call leaves at zero; the partial
// tables after them are overwritten before they are read.  Every GPU that
// loads this library holds it until the process exits.  All calls share it,
// so calls whose work overlaps on the GPU (different streams, or devices
// sharing nothing but the host thread) race on it and must be ordered by the
// caller.
#include <cuda_runtime.h>

#include <mutex>

#include "wbmm.h"
#include "wbmm_internal.h"

namespace wbmm {

namespace {

constexpr size_t kStaticPartials = 1u << 20;   // floats (4 MiB)
constexpr int kMaxDev = 64;

static __device__ __align__(256) float g_static_partials[kStaticPartials];

std::mutex g_static_mu;
float* g_static_ptr[kMaxDev] = {};

// Device address of g_static_partials on the current device.  The array's
// name in host code is a host-side stand-in, not a device address, so the
// address is fetched once per device with that device current.
wbmm_status static_partials(float** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev)
        return WBMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_partials) != cudaSuccess || p == nullptr)
            return WBMM_ERR_CUDA;
        g_static_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_static_ptr[dev];
    return WBMM_OK;
}

}  // namespace

}  // namespace wbmm

using namespace wbmm;

extern "C" WBMM_API wbmm_status wbmm_backward_dt_static(const void* x, const void* dY, float* dT,
                                                        int B, int C, int H, int W, int w,
                                                        wbmm_dtype dt, void* stream)
{
    if (dt != WBMM_F32 && dt != WBMM_BF16)
        return WBMM_ERR_DTYPE;
    if (!x || !dY || !dT || B <= 0 || C <= 0 || H <= 0 || W <= 0 || w <= 0)
        return WBMM_ERR_INVALID_ARG;
    if (H % w != 0 || W % w != 0)
        return WBMM_ERR_SHAPE;
    if (w > 64)
        return WBMM_ERR_UNSUPPORTED;
    const uintptr_t align = dt == WBMM_BF16 ? 16 : 4;
    if (reinterpret_cast<uintptr_t>(x) % align || reinterpret_cast<uintptr_t>(dY) % align ||
        reinterpret_cast<uintptr_t>(dT) % 4)
        return WBMM_ERR_ALIGNMENT;
    const Geom g = make_geom(B, C, H, W, w);
    const size_t esz = dt == WBMM_BF16 ? 2 : 4;
    const size_t mb = (size_t)B * C * H * W * esz;
    const uintptr_t t0 = reinterpret_cast<uintptr_t>(dT), t1 = t0 + (size_t)C * g.tsz * 4;
    for (const void* in : {x, dY}) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(in), a1 = a0 + mb;
        if (t0 < a1 && a0 < t1)
            return WBMM_ERR_INVALID_ARG;
    }
    // Same partial-table split as wbmm_backward, checked against the array.
    const bool tc = dt == WBMM_BF16 && tc_dt_supported(g);
    const long long need = tc ? tc_dt_workspace_floats(g)
                              : WBMM_DT_COUNTER_WORDS + (long long)C * simt_dt_chunks(g) * g.tsz;
    if ((unsigned long long)need > kStaticPartials)
        return WBMM_ERR_WORKSPACE;

    float* part = nullptr;
    wbmm_status st = static_partials(&part);
    if (st != WBMM_OK)
        return st;
    Launch L;
    if ((st = static_cast<wbmm_status>(launch_for_stream(stream, &L))) != WBMM_OK)
        return st;

    cudaError_t e;
    if (tc) {
        e = tc_dt_launch(g, x, dY, part, dT, false, L);
    } else {
        // the CUDA-core path's partial tables also sit after the counters
        float* chunks = part + WBMM_DT_COUNTER_WORDS;
        e = simt_dt_launch(g, dt == WBMM_BF16, x, dY, chunks, L);
        if (e == cudaSuccess)
            e = dt_finalize_launch(C, g.tsz, simt_dt_chunks(g), chunks, dT, L);
    }
    if (e == cudaErrorInvalidConfiguration)
        return WBMM_ERR_UNSUPPORTED;
    return e == cudaSuccess ? WBMM_OK : WBMM_ERR_CUDA;
}
