/*
 * WBMM oracle: test infrastructure, not part of the product path.
 *
 * A plain, slow, obviously correct CPU statement of what the Windowed Batch
 * Matrix Multiplication operator computes, in fp64, written as the direct
 * loop form of each definition.  Only tests/, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this file's library.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * Source: "WBMM: Windowed Batch Matrix Multiplication for Efficient Large
 * Receptive Field Convolution" (arXiv 2607.02097), as described by
 *   - the paper.gecl.asia reading notes, sections "Core Idea" and "Method"
 *     (window partition, relative-position table indexed into a per-channel
 *     d x d matrix shared by all windows, Toeplitz structure restricted to
 *     the window, inter-block 3x3 depthwise mixing, inference caching);
 *   - the arxivdaily.com English abstract (contiguous windows, compact
 *     relative position bias table, batched matrix multiplication).
 * The pages print no formula.  The index convention used here (offset =
 * output minus input position, row-major over the two offsets) is
 *   M_c[(p,q),(r,s)] = T_c[(p-r+w-1)(2w-1) + (q-s+w-1)],
 * with (p,q) the output and (r,s) the input position inside one window.
 *
 * Layouts: every feature map is dense NCHW; T is [C][(2w-1)^2] row-major
 * over (dp, dq); M is [C][d][d] with in-window position u = p*w + q.
 * H and W must be multiples of w (the caller checks).
 *
 * Parallelism: OpenMP over independent (image, channel) planes, or over
 * channels for the table gradient; every inner sum runs in a fixed order.
 */
#include <stddef.h>

/* Offset (dp, dq) = (p-r, q-s) -> position in the relative table. */
static long rel_index(int w, int dp, int dq)
{
    return (long)(dp + w - 1) * (2 * w - 1) + (dq + w - 1);
}

/*
 * Forward: y[b,c,i*w+p,j*w+q] = sum_{r,s} T[c, idx(p-r,q-s)] * x[b,c,i*w+r,j*w+s].
 * (reading notes, "Core Idea": each window is multiplied by the channel's
 * d x d matrix built from the table; no term crosses a window border.)
 */
void oracle_forward(const double *x, const double *T, double *y,
                    int B, int C, int H, int W, int w)
{
    const long tsz = (long)(2 * w - 1) * (2 * w - 1);
    const int nh = H / w, nw = W / w;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < C; ++c) {
            const double *xp = x + ((long)b * C + c) * H * W;
            double *yp = y + ((long)b * C + c) * H * W;
            const double *Tc = T + (long)c * tsz;
            for (int i = 0; i < nh; ++i)
                for (int j = 0; j < nw; ++j)
                    for (int p = 0; p < w; ++p)
                        for (int q = 0; q < w; ++q) {
                            double acc = 0.0;
                            for (int r = 0; r < w; ++r)
                                for (int s = 0; s < w; ++s)
                                    acc += Tc[rel_index(w, p - r, q - s)] *
                                           xp[(long)(i * w + r) * W + j * w + s];
                            yp[(long)(i * w + p) * W + j * w + q] = acc;
                        }
        }
    }
}

/*
 * Input gradient: dX_c = M_c^T dY_c, i.e.
 * dx[b,c,i*w+r,j*w+s] = sum_{p,q} T[c, idx(p-r,q-s)] * dy[b,c,i*w+p,j*w+q].
 */
void oracle_backward_dx(const double *dy, const double *T, double *dx,
                        int B, int C, int H, int W, int w)
{
    const long tsz = (long)(2 * w - 1) * (2 * w - 1);
    const int nh = H / w, nw = W / w;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < C; ++c) {
            const double *gp = dy + ((long)b * C + c) * H * W;
            double *op = dx + ((long)b * C + c) * H * W;
            const double *Tc = T + (long)c * tsz;
            for (int i = 0; i < nh; ++i)
                for (int j = 0; j < nw; ++j)
                    for (int r = 0; r < w; ++r)
                        for (int s = 0; s < w; ++s) {
                            double acc = 0.0;
                            for (int p = 0; p < w; ++p)
                                for (int q = 0; q < w; ++q)
                                    acc += Tc[rel_index(w, p - r, q - s)] *
                                           gp[(long)(i * w + p) * W + j * w + q];
                            op[(long)(i * w + r) * W + j * w + s] = acc;
                        }
        }
    }
}

/*
 * Table gradient: every pair (output (p,q), input (r,s)) of every window
 * adds dy[p,q] * x[r,s] to the table entry it reads, idx(p-r, q-s).
 * dT is overwritten.  One thread owns one channel, so each entry is summed
 * in the fixed order (b, i, j, p, q, r, s).
 */
void oracle_backward_dt(const double *x, const double *dy, double *dT,
                        int B, int C, int H, int W, int w)
{
    const long tsz = (long)(2 * w - 1) * (2 * w - 1);
    const int nh = H / w, nw = W / w;
#pragma omp parallel for schedule(static)
    for (int c = 0; c < C; ++c) {
        double *g = dT + (long)c * tsz;
        for (long k = 0; k < tsz; ++k)
            g[k] = 0.0;
        for (int b = 0; b < B; ++b) {
            const double *xp = x + ((long)b * C + c) * H * W;
            const double *gp = dy + ((long)b * C + c) * H * W;
            for (int i = 0; i < nh; ++i)
                for (int j = 0; j < nw; ++j)
                    for (int p = 0; p < w; ++p)
                        for (int q = 0; q < w; ++q) {
                            const double gy = gp[(long)(i * w + p) * W + j * w + q];
                            for (int r = 0; r < w; ++r)
                                for (int s = 0; s < w; ++s)
                                    g[rel_index(w, p - r, q - s)] +=
                                        gy * xp[(long)(i * w + r) * W + j * w + s];
                        }
        }
    }
}

/*
 * Matrix expansion (the cached-inference matrices):
 * M[c][(p*w+q)*d + (r*w+s)] = T[c, idx(p-r, q-s)], an exact copy.
 */
void oracle_expand(const double *T, double *M, int C, int w)
{
    const long tsz = (long)(2 * w - 1) * (2 * w - 1);
    const long d = (long)w * w;
    for (int c = 0; c < C; ++c)
        for (int p = 0; p < w; ++p)
            for (int q = 0; q < w; ++q)
                for (int r = 0; r < w; ++r)
                    for (int s = 0; s < w; ++s)
                        M[(long)c * d * d + (long)(p * w + q) * d + (r * w + s)] =
                            T[(long)c * tsz + rel_index(w, p - r, q - s)];
}

/*
 * Hierarchical window reparameterisation folded for inference (reading
 * notes, "Method", fourth point: a k x k local structure overlaid on the
 * w x w window, with no inference cost).  Read as a second WBMM branch of
 * window k (k divides w) on the same input, whose windows tile each w-window
 * 2-D; the sum of the branches is one w-window map with matrix
 *   M[c][(p,q),(r,s)] = T_w[c, idx_w(p-r, q-s)]
 *                       + [p/k == r/k and q/k == s/k] T_k[c, idx_k(p%k - r%k, q%k - s%k)].
 */
void oracle_reparam_merge(const double *Tw, const double *Tk, double *M, int C, int w, int k)
{
    const long tw = (long)(2 * w - 1) * (2 * w - 1), tk = (long)(2 * k - 1) * (2 * k - 1);
    const long d = (long)w * w;
    for (int c = 0; c < C; ++c)
        for (int p = 0; p < w; ++p)
            for (int q = 0; q < w; ++q)
                for (int r = 0; r < w; ++r)
                    for (int s = 0; s < w; ++s) {
                        double v = Tw[(long)c * tw + rel_index(w, p - r, q - s)];
                        if (p / k == r / k && q / k == s / k)
                            v += Tk[(long)c * tk + rel_index(k, p % k - r % k, q % k - s % k)];
                        M[(long)c * d * d + (long)(p * w + q) * d + (r * w + s)] = v;
                    }
}

/*
 * Inter-block 3x3 depthwise mixing (reading notes, "Method", third point):
 * z[b,c,h,x] = sum_{a,e in 0..2} K[c,a,e] * y[b,c,h+a-1,x+e-1], with y taken
 * as zero outside the image (cross-correlation, zero padding 1, no bias).
 */
void oracle_dw3x3(const double *y, const double *K, double *z,
                  int B, int C, int H, int W)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < C; ++c) {
            const double *yp = y + ((long)b * C + c) * H * W;
            double *zp = z + ((long)b * C + c) * H * W;
            const double *Kc = K + (long)c * 9;
            for (int h = 0; h < H; ++h)
                for (int x0 = 0; x0 < W; ++x0) {
                    double acc = 0.0;
                    for (int a = 0; a < 3; ++a)
                        for (int e = 0; e < 3; ++e) {
                            const int hh = h + a - 1, xx = x0 + e - 1;
                            if (hh < 0 || hh >= H || xx < 0 || xx >= W)
                                continue;
                            acc += Kc[a * 3 + e] * yp[(long)hh * W + xx];
                        }
                    zp[(long)h * W + x0] = acc;
                }
        }
    }
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
