/*
 * wbmm.h -- C ABI of libwbmm.so, Windowed Batch Matrix Multiplication (WBMM)
 * on NVIDIA B200 (sm_100a).
 *
 * The operator (arXiv 2607.02097, "WBMM: Windowed Batch Matrix
 * Multiplication for Efficient Large Receptive Field Convolution"):
 * an NCHW feature map x[B,C,H,W] is cut into non-overlapping w x w windows
 * (d = w*w positions each; reading notes, section "Method", first point).
 * Each channel c owns a compact relative-position table T_c of (2w-1)^2
 * entries, indexed into a d x d matrix shared by every window of every image
 * (reading notes, section "Core Idea"; the abstract: a small table of
 * relative-offset weights is indexed to form each channel's matrix, and all
 * windows then go through one batched matrix multiplication):
 *
 *     M_c[(p,q),(r,s)] = T_c[(p-r+w-1)(2w-1) + (q-s+w-1)]
 *     y[b,c,i*w+p,j*w+q] = sum_{r,s} M_c[(p,q),(r,s)] x[b,c,i*w+r,j*w+s]
 *
 * (p,q) is the output and (r,s) the input position inside window (i,j); the
 * in-window position index is u = p*w + q.  H and W must be multiples of w.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, contiguous, row-major (NCHW for feature maps) and live
 *     in device memory of the current CUDA device, unless an argument says
 *     otherwise.  The caller owns every buffer; the library keeps no pointer
 *     after a call returns.
 *   - dtype WBMM_BF16: x, y, T, M, dY, dX and 3x3 weights are bfloat16,
 *     products accumulate in fp32 and outputs round to nearest even.
 *     dtype WBMM_F32: the same tensors are fp32 and accumulate in fp32.
 *     The table gradient dT is fp32 for both dtypes.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Argument errors are reported synchronously and
 *     launch nothing.  A bounded device-side wait that expires is reported by
 *     wbmm_get_device_status().
 *   - Outputs must not overlap inputs.  bf16 pointers must be 16-byte
 *     aligned (WBMM_ERR_ALIGNMENT otherwise); fp32 pointers 4-byte aligned.
 *   - The library allocates no device memory per call.
 *   - Not thread-safe per stream: one caller per stream at a time.
 */
#ifndef WBMM_H
#define WBMM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WBMM_API __attribute__((visibility("default")))
#else
#define WBMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WBMM_OK = 0,
    WBMM_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, overlap   */
    WBMM_ERR_SHAPE = 2,        /* H or W not a multiple of w, shape mismatch */
    WBMM_ERR_DTYPE = 3,        /* unknown dtype                              */
    WBMM_ERR_ALIGNMENT = 4,    /* pointer not aligned as stated above        */
    WBMM_ERR_UNSUPPORTED = 5,  /* size beyond a kernel limit, or no sm_100   */
    WBMM_ERR_WORKSPACE = 6,    /* workspace missing or too small             */
    WBMM_ERR_CUDA = 7,         /* a CUDA runtime call or launch failed       */
    WBMM_ERR_TIMEOUT = 8       /* a bounded device wait expired              */
} wbmm_status;

typedef enum { WBMM_F32 = 0, WBMM_BF16 = 1 } wbmm_dtype;

/*
 * Forward pass, y = WBMM(x; T).
 *   x  [B,C,H,W]       input map, dtype dt
 *   T  [C,(2w-1)^2]    relative-position table, dtype dt
 *   y  [B,C,H,W]       output map, dtype dt (overwritten)
 * M_c is expanded from T_c on chip and never written to memory.
 * Errors: INVALID_ARG, SHAPE (H % w or W % w), DTYPE, ALIGNMENT, UNSUPPORTED
 * (w > 64), CUDA.
 */
WBMM_API wbmm_status wbmm_forward(const void *x, const void *T, void *y,
                         int B, int C, int H, int W, int w,
                         wbmm_dtype dt, void *stream);

/*
 * Size of the arrival-counter region at the start of a table-gradient
 * workspace, in 32-bit words (see wbmm_backward_workspace_bytes).
 */
#define WBMM_DT_COUNTER_WORDS 65536

/*
 * Bytes of device workspace wbmm_backward needs for the table gradient.
 * bf16 on the tensor-core kernels (C <= WBMM_DT_COUNTER_WORDS): the workspace
 * starts with WBMM_DT_COUNTER_WORDS 32-bit arrival counters (256 KiB; word c
 * counts the CTAs that have finished their part of channel c), followed by
 * fp32 partial tables of the channels whose windows are split between CTAs.
 * Zero-fill the workspace once before its first use (cudaMemset,
 * torch.zeros).  Every call leaves the counters at zero again, a call that
 * ends in WBMM_ERR_TIMEOUT included, and no call writes a counter word for
 * anything else, so one workspace serves any number of later calls of any
 * shape it is large enough for, graph replays included.  A call that ends in
 * WBMM_ERR_CUDA may leave it dirty: zero it again.
 * fp32 (and bf16 shapes outside the tensor-core kernels): the same counter
 * region (left untouched), then fp32 partial tables, one per (channel, fixed
 * chunk of windows), whose prior content does not matter.
 * The split depends only on the shape, the device's SM count and whether dX
 * is computed in the same call, so dT is bit-identical from run to run.
 * Calls that share a workspace must not overlap on the GPU.
 * Returns 0 for invalid shapes.
 */
WBMM_API size_t wbmm_backward_workspace_bytes(int B, int C, int H, int W, int w, wbmm_dtype dt);

/*
 * Training backward.
 *   dX_c = M_c^T dY_c  (equal to WBMM of dY with the 180-degree rotated table)
 *   dT_c[(dp+w-1)(2w-1)+(dq+w-1)] = sum over windows n and position pairs with
 *       p-r = dp, q-s = dq of dY[n,(p,q)] * x[n,(r,s)]  (the diagonal sums of
 *       dY_c X_c^T along constant relative offset)
 *   x, dY [B,C,H,W] dtype dt;  T [C,(2w-1)^2] dtype dt
 *   dX [B,C,H,W] dtype dt, or NULL to skip it (overwritten)
 *   dT [C,(2w-1)^2] fp32, or NULL to skip it (overwritten, not accumulated)
 *   workspace: device buffer of at least wbmm_backward_workspace_bytes()
 *   bytes, 16-byte aligned; needed only when dT != NULL.
 * With both outputs on a large enough bf16 problem the two gradient kernels
 * run at the same time on disjoint SMs (dX on 2/5 of them); dT then sums in
 * a different fixed order than a dT-only call, so the two differ by rounding
 * (each deterministic).  The call's work is complete when its last kernel is.
 * Errors: as wbmm_forward, plus WORKSPACE.
 */
WBMM_API wbmm_status wbmm_backward(const void *x, const void *T, const void *dY,
                          void *dX, float *dT, void *workspace, size_t ws_bytes,
                          int B, int C, int H, int W, int w,
                          wbmm_dtype dt, void *stream);

/*
 * Inference caching (reading notes, "Method": caching M removes the index
 * construction cost): M[c][u][v] = M_c[u,v], an exact copy of table entries.
 *   T [C,(2w-1)^2] dtype dt;  M [C,d,d] dtype dt, row-major, u = p*w+q.
 * Errors: INVALID_ARG, DTYPE, ALIGNMENT, UNSUPPORTED, CUDA.
 */
WBMM_API wbmm_status wbmm_cache_matrices(const void *T, void *M, int C, int w,
                                wbmm_dtype dt, void *stream);

/*
 * Hierarchical window reparameterisation folded for inference (reading
 * notes, "Method", fourth point: a k x k local structure overlaid on the
 * w x w window at no inference cost).  Read as a second WBMM branch of window
 * k (k divides w) on the same input, whose k-windows tile every w-window; the
 * two branches sum to one w-window map whose per-channel matrix is
 *   M[c][(p,q),(r,s)] = Tw[c, (p-r+w-1)(2w-1) + (q-s+w-1)]
 *     + (p/k == r/k and q/k == s/k) * Tk[c, (p%k-r%k+k-1)(2k-1) + (q%k-s%k+k-1)]
 * (rows and columns u = p*w+q), summed in fp32 and rounded once to dt.  Pass
 * M to wbmm_forward_cached.
 *   Tw [C,(2w-1)^2], Tk [C,(2k-1)^2], M [C,w*w,w*w]; dtype dt.
 * Errors: INVALID_ARG (null pointer, C, w or k <= 0, k not dividing w, M
 * overlapping a table), UNSUPPORTED (w > 64), DTYPE, ALIGNMENT, CUDA.
 */
WBMM_API wbmm_status wbmm_reparam_merge(const void *Tw, const void *Tk, void *M, int C, int w,
                                        int k, wbmm_dtype dt, void *stream);

/*
 * Cached-matrix forward, optionally followed by the inter-block 3x3 depthwise
 * mixing (reading notes, "Method", third point):
 *   y = M_c X_c per window (M as written by wbmm_cache_matrices, or any
 *       caller-built [C,d,d] matrix, e.g. a merged reparameterisation);
 *   out = y                           when dw3x3 == NULL
 *   out = dw3x3(y; K) (see wbmm_dw3x3) when dw3x3 != NULL, in one fused launch:
 *       y is rounded to dt exactly as a separate wbmm_forward_cached call
 *       would store it, so the fused result equals the two-call result.
 *   x [B,C,H,W], M [C,d,d], dw3x3 [C,1,3,3] or NULL, out [B,C,H,W]; dtype dt.
 * Errors: as wbmm_forward; UNSUPPORTED for a fused call the fused kernel
 * does not cover: fp32 maps, W not a multiple of 8, a tile of window rows
 * that does not divide the image's window rows (the kernel processes whole
 * image planes), or a plane of H*W bf16 elements beyond the per-SM buffer
 * (about 100 KB beside the pipeline at w = 14).  out must not overlap x, M or
 * dw3x3.
 */
WBMM_API wbmm_status wbmm_forward_cached(const void *x, const void *M, const void *dw3x3,
                                void *out, int B, int C, int H, int W, int w,
                                wbmm_dtype dt, void *stream);

/*
 * Standalone inter-block 3x3 depthwise mixing:
 *   z[b,c,h,x] = sum_{a,e in 0..2} K[c,0,a,e] * y[b,c,h+a-1,x+e-1],
 * y taken as zero outside the image (cross-correlation, zero padding 1, no
 * bias); fp32 accumulation.  y, z [B,C,H,W], K [C,1,3,3]; dtype dt.
 * Errors: INVALID_ARG, DTYPE, ALIGNMENT, CUDA.
 */
WBMM_API wbmm_status wbmm_dw3x3(const void *y, const void *K, void *z,
                       int B, int C, int H, int W, wbmm_dtype dt, void *stream);

/*
 * Table gradient for callers that cannot allocate device memory: the dT of
 * wbmm_backward called with dX = NULL (same kernels, same bits), with the
 * fp32 partial tables kept in a fixed 4 MiB array inside the library instead
 * of a workspace argument.
 * The paper has no counterpart to this entry point; it exists for hosts with a
 * fixed device-memory budget, plugins inside frameworks that own all device
 * allocations, and paths where cudaMalloc would synchronise the device.
 *   x, dY [B,C,H,W] dtype dt;  dT [C,(2w-1)^2] fp32 (overwritten)
 * Allocates nothing and frees nothing.  The first call on a device looks up
 * the array's device address (cudaGetSymbolAddress); make that first call
 * before any stream capture.  Every device holds the array until exit.  All
 * calls share it, so calls whose work overlaps on the GPU race and must be
 * ordered by the caller.  The array starts zeroed and every call leaves its
 * arrival counters at zero (see wbmm_backward_workspace_bytes).  Returns
 * WBMM_ERR_WORKSPACE, before any launch, when the workspace that
 * wbmm_backward_workspace_bytes reports for the same shape and a dT-only call
 * exceeds the array's 2^20 floats (4 MiB).
 */
WBMM_API wbmm_status wbmm_backward_dt_static(const void *x, const void *dY, float *dT,
                                             int B, int C, int H, int W, int w,
                                             wbmm_dtype dt, void *stream);

/*
 * Synchronises `stream`, then reports and clears the device status word that
 * kernels set when a bounded wait expires (WBMM_ERR_TIMEOUT), or returns
 * WBMM_ERR_CUDA for a sticky CUDA error.  WBMM_OK otherwise.
 */
WBMM_API wbmm_status wbmm_get_device_status(void *stream);

/* Static, human-readable name of a status code. */
WBMM_API const char *wbmm_status_string(wbmm_status s);

/*
 * Device-side wait budget, in SM clock cycles, applied to every bounded
 * mbarrier wait of later launches on this process (default 4e9, about two
 * seconds).  0 restores the default.
 */
WBMM_API void wbmm_set_wait_budget(unsigned long long cycles);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a
 * shared-memory barrier that nothing completes, with `cycles` as the budget.
 * The kernel gives up, records WBMM_ERR_TIMEOUT in the device status word and
 * returns; wbmm_get_device_status() then reports it.  No other state changes.
 */
WBMM_API wbmm_status wbmm_wait_selftest(unsigned long long cycles, void *stream);

/*
 * Number of kernels this library has launched in the process so far (all
 * devices, all entry points).  Used to count launches inside a timed region.
 */
WBMM_API unsigned long long wbmm_launch_count(void);

/*
 * Test-only settings, off by default, for exercising failure handling
 * without faulting the GPU (the library's own tests use them; a normal
 * caller never needs them).  No counterpart in the paper.
 *   WBMM_DEBUG_SKIP_LOAD_WINDOW_MAJOR, value t >= 0: in the next launch of
 *     the window-major tensor-core kernel (wbmm_forward, or the input
 *     gradient of wbmm_backward, w <= 16), the load producer of CTA 0 skips
 *     its t-th tile; the consumer's bounded wait for it runs out, the kernel
 *     abandons its work, drains its copies and MMAs, releases its tensor
 *     memory and returns, and wbmm_get_device_status() reports
 *     WBMM_ERR_TIMEOUT.  The outputs of that call are undefined.  Consumed by
 *     that launch; value < 0 clears it.
 *   WBMM_DEBUG_SKIP_LOAD_TABLE_GRAD: the same for the next launch of the
 *     tensor-core table-gradient kernel.
 *   WBMM_DEBUG_RING_CAP, value n: the window-major and table-gradient
 *     kernels use at most n load slots (0 restores the default, as many as
 *     fit); results do not depend on it.
 * Pair a skip with a short wait budget (wbmm_set_wait_budget).  Process-wide;
 * not for concurrent use.  Returns WBMM_ERR_INVALID_ARG for an unknown `what`.
 */
#define WBMM_DEBUG_SKIP_LOAD_WINDOW_MAJOR 1
#define WBMM_DEBUG_SKIP_LOAD_TABLE_GRAD 2
#define WBMM_DEBUG_RING_CAP 3
WBMM_API wbmm_status wbmm_debug_set(int what, int value);

/*
 * Kernel family used by the most recent successful wbmm_forward,
 * wbmm_backward (input-gradient part) or wbmm_forward_cached call on this
 * host thread: 1 = tcgen05 tensor-core kernel, 2 = CUDA-core (SIMT) kernel.
 */
WBMM_API int wbmm_last_path(void);

#ifdef __cplusplus
}
#endif

#endif /* WBMM_H */
