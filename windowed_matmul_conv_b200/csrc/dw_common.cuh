// The inter-block 3x3 depthwise mixing of one 16-byte vector of a bf16 row:
// eight consecutive outputs from three input rows.  Shared by the standalone
// kernel and the cached forward's fused epilogue so that both perform the
// same fp32 fused multiply-adds in the same order (a outer, e inner, from 0,
// zero padding included) and give the same bits.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace wbmm {

// rows[a] points at element 8*v of input row h-1+a, or is null for a row
// outside the image (read as zeros); v is the vector index in the row and
// nvec the vectors per row (W / 8).  k: the channel's 3x3 weights, row-major.
__device__ __forceinline__ uint4 dw3x3_row8(const uint16_t* const (&rows)[3], int v, int nvec,
                                            const float (&k)[9])
{
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        acc[j] = 0.0f;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const uint16_t* row = rows[a];
        float vals[10];
        if (row != nullptr) {
            vals[0] = v > 0 ? __bfloat162float(__ushort_as_bfloat16(row[-1])) : 0.0f;
            const uint4 mid = *reinterpret_cast<const uint4*>(row);
            const uint32_t w4[4] = {mid.x, mid.y, mid.z, mid.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                vals[1 + 2 * j] = __uint_as_float(w4[j] << 16);
                vals[2 + 2 * j] = __uint_as_float(w4[j] & 0xFFFF0000u);
            }
            vals[9] = v + 1 < nvec ? __bfloat162float(__ushort_as_bfloat16(row[8])) : 0.0f;
        } else {
#pragma unroll
            for (int j = 0; j < 10; ++j)
                vals[j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int e = 0; e < 3; ++e)
                acc[j] = __fmaf_rn(k[a * 3 + e], vals[j + e], acc[j]);
    }
    uint32_t packed[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * j]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * j + 1]));
        packed[j] = lo | (hi << 16);
    }
    return make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

}  // namespace wbmm
