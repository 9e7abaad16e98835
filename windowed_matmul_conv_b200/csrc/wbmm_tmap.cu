// Host-side encoding of the 4-D tensor maps that let one TMA request move a
// run of whole image planes of one channel: NCHW viewed as
//   {I, H*W/I, C, B}  (I elements per row, rows per plane, channel, image),
// box {I, H*W/I, 1, k}: k consecutive images of channel c land in shared
// memory as k contiguous planes -- the raw band layout of the tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "wbmm_internal.h"

namespace wbmm {

namespace {

std::mutex g_enc_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
bool g_encode_tried = false;

PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    std::lock_guard<std::mutex> lk(g_enc_mu);
    if (!g_encode_tried) {
        g_encode_tried = true;
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    return g_encode;
}

}  // namespace

int plane_row_elems(const Geom& g)
{
    const long long hw = (long long)g.H * g.W;
    for (int cand = 256; cand >= 8; cand -= 8)
        if (hw % cand == 0 && hw / cand <= 256)
            return cand;
    return 0;
}

bool encode_plane_map(void* map, const void* base, const Geom& g, int k_images)
{
    const int I = plane_row_elems(g);
    if (I == 0 || k_images < 1 || k_images > 256)
        return false;
    const long long hw = (long long)g.H * g.W;
    if ((hw * 2) % 16 != 0 || reinterpret_cast<uintptr_t>(base) % 16 != 0)
        return false;
    PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc)
        return false;
    cuuint64_t dims[4] = {(cuuint64_t)I, (cuuint64_t)(hw / I), (cuuint64_t)g.C, (cuuint64_t)g.B};
    cuuint64_t strides[3] = {(cuuint64_t)I * 2, (cuuint64_t)hw * 2, (cuuint64_t)g.C * hw * 2};
    cuuint32_t box[4] = {(cuuint32_t)I, (cuuint32_t)(hw / I), 1u, (cuuint32_t)k_images};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = enc(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                     const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace wbmm
