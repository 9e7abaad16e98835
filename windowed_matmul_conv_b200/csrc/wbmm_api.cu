// C ABI of libwbmm.so: argument checks, kernel selection and launches.
// Declarations and the contract of every entry point are in include/wbmm.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "wbmm.h"
#include "wbmm_internal.h"

namespace wbmm {

// Device status word: kernels OR in kStatusTimeout when a bounded wait runs
// out.  One copy per device; host code reaches it through its symbol address.
__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultBudget = 4000000000ull;  // ~2 s of SM cycles

struct DevInfo {
    bool ready = false;
    bool sm100 = false;
    int num_sms = 0;
    int* status = nullptr;
};

std::mutex g_mu;
DevInfo g_dev[kMaxDevices];
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_budget{kDefaultBudget};
// Test-only settings (wbmm_debug_set): a tile whose load the producer of
// CTA 0 skips in the next launch of a kernel family (-1: none), and a cap on
// the load ring's depth (0: none).
std::atomic<int> g_dbg_skip_toep{-1};
std::atomic<int> g_dbg_skip_dt{-1};
std::atomic<int> g_dbg_ring_cap{0};
thread_local int t_last_path = 0;

wbmm_status dev_info(DevInfo** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return WBMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
            return WBMM_ERR_CUDA;
        d.sm100 = (prop.major == 10 && prop.minor == 0);
        d.num_sms = prop.multiProcessorCount;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess)
            return WBMM_ERR_CUDA;
        d.status = static_cast<int*>(p);
        d.ready = true;
    }
    *out = &d;
    return WBMM_OK;
}

wbmm_status make_launch(void* stream, Launch* L)
{
    DevInfo* d = nullptr;
    wbmm_status st = dev_info(&d);
    if (st != WBMM_OK)
        return st;
    if (!d->sm100)
        return WBMM_ERR_UNSUPPORTED;  // kernels are built for sm_100a only
    L->stream = static_cast<cudaStream_t>(stream);
    L->num_sms = d->num_sms;
    L->status = d->status;
    L->budget = g_budget.load();
    return WBMM_OK;
}

wbmm_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess)
        return WBMM_OK;
    if (e == cudaErrorInvalidConfiguration)
        return WBMM_ERR_UNSUPPORTED;
    return WBMM_ERR_CUDA;
}

size_t elem_size(wbmm_dtype dt) { return dt == WBMM_BF16 ? 2 : 4; }

bool dtype_ok(wbmm_dtype dt) { return dt == WBMM_F32 || dt == WBMM_BF16; }

bool aligned(const void* p, wbmm_dtype dt)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return dt == WBMM_BF16 ? (a % 16 == 0) : (a % 4 == 0);
}

struct Span {
    const void* p;
    size_t bytes;
};

bool overlap(Span a, Span b)
{
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0)
        return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

wbmm_status check_map(int B, int C, int H, int W, int w)
{
    if (B <= 0 || C <= 0 || H <= 0 || W <= 0 || w <= 0)
        return WBMM_ERR_INVALID_ARG;
    if (H % w != 0 || W % w != 0)
        return WBMM_ERR_SHAPE;
    if (w > 64)
        return WBMM_ERR_UNSUPPORTED;
    return WBMM_OK;
}

size_t map_bytes(const Geom& g, wbmm_dtype dt)
{
    return (size_t)g.B * g.C * g.H * g.W * elem_size(dt);
}

// Workspace floats the backward will use for this shape and dtype.  Every
// workspace starts with the tensor-core path's counter region, so a buffer
// shared by calls of both paths never has its counters overwritten.
long long dt_workspace_floats(const Geom& g, wbmm_dtype dt)
{
    if (dt == WBMM_BF16 && tc_dt_supported(g))
        return tc_dt_workspace_floats(g);
    return WBMM_DT_COUNTER_WORDS + (long long)g.C * simt_dt_chunks(g) * g.tsz;
}

}  // namespace

void note_launches(int n) { g_launches.fetch_add((unsigned long long)n); }

int debug_take_skip(int family)
{
    return (family == 0 ? g_dbg_skip_toep : g_dbg_skip_dt).exchange(-1);
}

int debug_ring_cap() { return g_dbg_ring_cap.load(); }

int launch_for_stream(void* stream, Launch* L) { return (int)make_launch(stream, L); }

}  // namespace wbmm

using namespace wbmm;

extern "C" {

const char* wbmm_status_string(wbmm_status s)
{
    switch (s) {
    case WBMM_OK: return "WBMM_OK";
    case WBMM_ERR_INVALID_ARG: return "WBMM_ERR_INVALID_ARG: null pointer, bad size or overlap";
    case WBMM_ERR_SHAPE: return "WBMM_ERR_SHAPE: H and W must be multiples of w";
    case WBMM_ERR_DTYPE: return "WBMM_ERR_DTYPE: unknown dtype";
    case WBMM_ERR_ALIGNMENT: return "WBMM_ERR_ALIGNMENT: pointer not aligned";
    case WBMM_ERR_UNSUPPORTED: return "WBMM_ERR_UNSUPPORTED: size beyond a kernel limit or no sm_100 device";
    case WBMM_ERR_WORKSPACE: return "WBMM_ERR_WORKSPACE: workspace missing or too small";
    case WBMM_ERR_CUDA: return "WBMM_ERR_CUDA: CUDA runtime error";
    case WBMM_ERR_TIMEOUT: return "WBMM_ERR_TIMEOUT: a bounded device wait expired";
    }
    return "WBMM: unknown status";
}

void wbmm_set_wait_budget(unsigned long long cycles)
{
    g_budget.store(cycles ? cycles : kDefaultBudget);
}

unsigned long long wbmm_launch_count(void) { return g_launches.load(); }

wbmm_status wbmm_debug_set(int what, int value)
{
    switch (what) {
    case WBMM_DEBUG_SKIP_LOAD_WINDOW_MAJOR: g_dbg_skip_toep.store(value < 0 ? -1 : value); return WBMM_OK;
    case WBMM_DEBUG_SKIP_LOAD_TABLE_GRAD: g_dbg_skip_dt.store(value < 0 ? -1 : value); return WBMM_OK;
    case WBMM_DEBUG_RING_CAP: g_dbg_ring_cap.store(value < 0 ? 0 : value); return WBMM_OK;
    }
    return WBMM_ERR_INVALID_ARG;
}

int wbmm_last_path(void) { return t_last_path; }

wbmm_status wbmm_forward(const void* x, const void* T, void* y, int B, int C, int H, int W,
                         int w, wbmm_dtype dt, void* stream)
{
    if (!dtype_ok(dt))
        return WBMM_ERR_DTYPE;
    if (!x || !T || !y)
        return WBMM_ERR_INVALID_ARG;
    wbmm_status st = check_map(B, C, H, W, w);
    if (st != WBMM_OK)
        return st;
    if (!aligned(x, dt) || !aligned(T, dt) || !aligned(y, dt))
        return WBMM_ERR_ALIGNMENT;
    const Geom g = make_geom(B, C, H, W, w);
    const Span ys{y, map_bytes(g, dt)};
    if (overlap(ys, Span{x, map_bytes(g, dt)}) ||
        overlap(ys, Span{T, (size_t)C * g.tsz * elem_size(dt)}))
        return WBMM_ERR_INVALID_ARG;
    Launch L;
    if ((st = make_launch(stream, &L)) != WBMM_OK)
        return st;
    if (dt == WBMM_BF16 && tc_toep_supported(g)) {
        st = from_cuda(tc_toep_launch(g, kTable, x, T, y, L));
        if (st == WBMM_OK)
            t_last_path = 1;
        return st;
    }
    if (dt == WBMM_BF16 && tc_fwd_supported(g, false)) {
        st = from_cuda(tc_fwd_launch(g, kTable, x, T, y, nullptr, L));
        if (st == WBMM_OK)
            t_last_path = 1;
        return st;
    }
    if (dt == WBMM_BF16 && tc_big_supported(g)) {
        st = from_cuda(tc_big_launch(g, kTable, x, T, y, L));
        if (st == WBMM_OK)
            t_last_path = 1;
        return st;
    }
    st = from_cuda(simt_fwd_launch(g, kTable, dt == WBMM_BF16, x, T, y, L));
    if (st == WBMM_OK)
        t_last_path = 2;
    return st;
}

size_t wbmm_backward_workspace_bytes(int B, int C, int H, int W, int w, wbmm_dtype dt)
{
    if (!dtype_ok(dt) || check_map(B, C, H, W, w) != WBMM_OK)
        return 0;
    const Geom g = make_geom(B, C, H, W, w);
    return (size_t)dt_workspace_floats(g, dt) * sizeof(float);
}

wbmm_status wbmm_backward(const void* x, const void* T, const void* dY, void* dX, float* dT,
                          void* workspace, size_t ws_bytes, int B, int C, int H, int W, int w,
                          wbmm_dtype dt, void* stream)
{
    if (!dtype_ok(dt))
        return WBMM_ERR_DTYPE;
    if (!dY || (dX && !T) || (dT && !x))
        return WBMM_ERR_INVALID_ARG;
    wbmm_status st = check_map(B, C, H, W, w);
    if (st != WBMM_OK)
        return st;
    if (!aligned(dY, dt) || (dX && !aligned(dX, dt)) || (dX && !aligned(T, dt)) ||
        (dT && !aligned(x, dt)) || (dT && reinterpret_cast<uintptr_t>(dT) % 4 != 0))
        return WBMM_ERR_ALIGNMENT;
    const Geom g = make_geom(B, C, H, W, w);
    const size_t mb = map_bytes(g, dt);
    const size_t tb = (size_t)C * g.tsz * elem_size(dt);
    const size_t need_ws = wbmm_backward_workspace_bytes(B, C, H, W, w, dt);
    if (dX) {
        const Span s{dX, mb};
        if (overlap(s, Span{dY, mb}) || overlap(s, Span{x, x ? mb : 0}) || overlap(s, Span{T, tb}))
            return WBMM_ERR_INVALID_ARG;
    }
    if (dT) {
        const Span s{dT, (size_t)C * g.tsz * 4};
        if (overlap(s, Span{dY, mb}) || overlap(s, Span{x, mb}) ||
            overlap(s, Span{dX, dX ? mb : 0}) || overlap(s, Span{workspace, ws_bytes}))
            return WBMM_ERR_INVALID_ARG;
        if (!workspace || ws_bytes < need_ws)
            return WBMM_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0)
            return WBMM_ERR_ALIGNMENT;
        const Span wsp{workspace, need_ws};
        if (overlap(wsp, Span{dY, mb}) || overlap(wsp, Span{x, mb}) ||
            overlap(wsp, Span{dX, dX ? mb : 0}))
            return WBMM_ERR_INVALID_ARG;
    }
    Launch L;
    if ((st = make_launch(stream, &L)) != WBMM_OK)
        return st;
    const bool tc_dt = dT && dt == WBMM_BF16 && tc_dt_supported(g);
    // Both gradients on tensor cores and enough tiles to fill the device: the
    // two kernels run at the same time on disjoint SMs (2/5 for dX, the rest
    // for dT, the measured balance at w = 14), each walking the channels in
    // the same order, so the second read of each dY tile is served from L2
    // and one kernel's ramp and tail overlap the other's steady state.  The
    // dT kernel's grid (and so its fixed summation order) is a function of
    // the shape and the SM count only.
    Launch Lx = L, Lt = L;
    if (dX && tc_dt && tc_toep_supported(g) && tc_dt_tiles(g) >= 2LL * L.num_sms &&
        L.num_sms >= 5) {
        Lx.num_sms = (2 * L.num_sms + 2) / 5;
        Lt.num_sms = L.num_sms - Lx.num_sms;
    }
    if (dX) {
        if (dt == WBMM_BF16 && tc_toep_supported(g)) {
            st = from_cuda(tc_toep_launch(g, kTableFlip, dY, T, dX, Lx));
            t_last_path = 1;
        } else if (dt == WBMM_BF16 && tc_fwd_supported(g, false)) {
            st = from_cuda(tc_fwd_launch(g, kTableFlip, dY, T, dX, nullptr, L));
            t_last_path = 1;
        } else if (dt == WBMM_BF16 && tc_big_supported(g)) {
            st = from_cuda(tc_big_launch(g, kTableFlip, dY, T, dX, L));
            t_last_path = 1;
        } else {
            st = from_cuda(simt_fwd_launch(g, kTableFlip, dt == WBMM_BF16, dY, T, dX, L));
            t_last_path = 2;
        }
        if (st != WBMM_OK)
            return st;
    }
    if (dT) {
        float* part = static_cast<float*>(workspace);
        if (tc_dt) {
            // dX, when requested, was the launch just before this one (every
            // library kernel signals its dependents only after its own wait)
            const bool after_dx = dX != nullptr;
            st = from_cuda(tc_dt_launch(g, x, dY, part, dT, after_dx, Lt));
        } else {
            float* chunks = part + WBMM_DT_COUNTER_WORDS;
            st = from_cuda(simt_dt_launch(g, dt == WBMM_BF16, x, dY, chunks, L));
            if (st != WBMM_OK)
                return st;
            st = from_cuda(dt_finalize_launch(C, g.tsz, simt_dt_chunks(g), chunks, dT, L));
        }
    }
    return st;
}

wbmm_status wbmm_cache_matrices(const void* T, void* M, int C, int w, wbmm_dtype dt,
                                void* stream)
{
    if (!dtype_ok(dt))
        return WBMM_ERR_DTYPE;
    if (!T || !M || C <= 0 || w <= 0)
        return WBMM_ERR_INVALID_ARG;
    if (w > 64)
        return WBMM_ERR_UNSUPPORTED;
    if (!aligned(T, dt) || !aligned(M, dt))
        return WBMM_ERR_ALIGNMENT;
    const size_t d = (size_t)w * w, tsz = (size_t)(2 * w - 1) * (2 * w - 1);
    if (overlap(Span{M, (size_t)C * d * d * elem_size(dt)}, Span{T, C * tsz * elem_size(dt)}))
        return WBMM_ERR_INVALID_ARG;
    Launch L;
    wbmm_status st = make_launch(stream, &L);
    if (st != WBMM_OK)
        return st;
    return from_cuda(cache_matrices_launch(C, w, dt == WBMM_BF16, T, M, L));
}

wbmm_status wbmm_reparam_merge(const void* Tw, const void* Tk, void* M, int C, int w, int k,
                               wbmm_dtype dt, void* stream)
{
    if (!dtype_ok(dt))
        return WBMM_ERR_DTYPE;
    if (!Tw || !Tk || !M || C <= 0 || w <= 0 || k <= 0 || w % k != 0)
        return WBMM_ERR_INVALID_ARG;
    if (w > 64)
        return WBMM_ERR_UNSUPPORTED;
    if (!aligned(Tw, dt) || !aligned(Tk, dt) || !aligned(M, dt))
        return WBMM_ERR_ALIGNMENT;
    const size_t d = (size_t)w * w;
    const size_t tw = (size_t)(2 * w - 1) * (2 * w - 1), tk = (size_t)(2 * k - 1) * (2 * k - 1);
    const Span ms{M, (size_t)C * d * d * elem_size(dt)};
    if (overlap(ms, Span{Tw, C * tw * elem_size(dt)}) ||
        overlap(ms, Span{Tk, C * tk * elem_size(dt)}))
        return WBMM_ERR_INVALID_ARG;
    Launch L;
    wbmm_status st = make_launch(stream, &L);
    if (st != WBMM_OK)
        return st;
    return from_cuda(reparam_merge_launch(C, w, k, dt == WBMM_BF16, Tw, Tk, M, L));
}

wbmm_status wbmm_forward_cached(const void* x, const void* M, const void* dw3x3, void* out,
                                int B, int C, int H, int W, int w, wbmm_dtype dt, void* stream)
{
    if (!dtype_ok(dt))
        return WBMM_ERR_DTYPE;
    if (!x || !M || !out)
        return WBMM_ERR_INVALID_ARG;
    wbmm_status st = check_map(B, C, H, W, w);
    if (st != WBMM_OK)
        return st;
    if (!aligned(x, dt) || !aligned(M, dt) || !aligned(out, dt) || (dw3x3 && !aligned(dw3x3, dt)))
        return WBMM_ERR_ALIGNMENT;
    const Geom g = make_geom(B, C, H, W, w);
    const Span os{out, map_bytes(g, dt)};
    if (overlap(os, Span{x, map_bytes(g, dt)}) ||
        overlap(os, Span{M, (size_t)C * g.d * g.d * elem_size(dt)}) ||
        overlap(os, Span{dw3x3, dw3x3 ? (size_t)C * 9 * elem_size(dt) : 0}))
        return WBMM_ERR_INVALID_ARG;
    Launch L;
    if ((st = make_launch(stream, &L)) != WBMM_OK)
        return st;
    const bool fused = dw3x3 != nullptr;
    if (dt == WBMM_BF16 && tc_cached_supported(g, fused)) {
        st = from_cuda(tc_cached_launch(g, x, M, dw3x3, out, L));
        if (st == WBMM_OK)
            t_last_path = 1;
        return st;
    }
    if (dt == WBMM_BF16 && tc_fwd_supported(g, fused)) {
        st = from_cuda(tc_fwd_launch(g, kCached, x, M, out, dw3x3, L));
        if (st == WBMM_OK)
            t_last_path = 1;
        return st;
    }
    if (fused)
        return WBMM_ERR_UNSUPPORTED;
    st = from_cuda(simt_fwd_launch(g, kCached, dt == WBMM_BF16, x, M, out, L));
    if (st == WBMM_OK)
        t_last_path = 2;
    return st;
}

wbmm_status wbmm_dw3x3(const void* y, const void* K, void* z, int B, int C, int H, int W,
                       wbmm_dtype dt, void* stream)
{
    if (!dtype_ok(dt))
        return WBMM_ERR_DTYPE;
    if (!y || !K || !z || B <= 0 || C <= 0 || H <= 0 || W <= 0)
        return WBMM_ERR_INVALID_ARG;
    if (!aligned(y, dt) || !aligned(K, dt) || !aligned(z, dt))
        return WBMM_ERR_ALIGNMENT;
    const Geom g = make_geom(B, C, H, W, 1);
    const Span zs{z, map_bytes(g, dt)};
    if (overlap(zs, Span{y, map_bytes(g, dt)}) || overlap(zs, Span{K, (size_t)C * 9 * elem_size(dt)}))
        return WBMM_ERR_INVALID_ARG;
    Launch L;
    wbmm_status st = make_launch(stream, &L);
    if (st != WBMM_OK)
        return st;
    return from_cuda(dw3x3_launch(g, dt == WBMM_BF16, y, K, z, L));
}

wbmm_status wbmm_get_device_status(void* stream)
{
    DevInfo* d = nullptr;
    wbmm_status st = dev_info(&d);
    if (st != WBMM_OK)
        return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return WBMM_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return WBMM_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(d->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return WBMM_ERR_CUDA;
        return WBMM_ERR_TIMEOUT;
    }
    return WBMM_OK;
}

wbmm_status wbmm_wait_selftest(unsigned long long cycles, void* stream)
{
    Launch L;
    wbmm_status st = make_launch(stream, &L);
    if (st != WBMM_OK)
        return st;
    return from_cuda(wait_selftest_launch(cycles, L));
}

}  // extern "C"
