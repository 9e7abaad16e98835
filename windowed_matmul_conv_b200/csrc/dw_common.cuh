// The inter-block 3x3 depthwise mixing of one 16-byte vector of a bf16 row:
// eight consecutive outputs from three input rows.  Shared by the standalone
// kernels and the cached forward's fused epilogue so that all perform the
// same fp32 fused multiply-adds in the same order (a outer, e inner, from 0,
// zero padding included) and give the same bits.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace wbmm {

__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

// acc = a * b + acc on both fp32 halves, each rounded to nearest even like
// __fmaf_rn (one packed instruction for two outputs).
__device__ __forceinline__ void f32x2_fma(uint64_t& acc, uint64_t a, uint64_t b)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// The ten input values of one input row around eight consecutive outputs,
// v[0] = left neighbour, v[1..8] = the 16-byte vector, v[9] = right
// neighbour (zeros outside the image), as fp32 pairs: E[m] = (v[2m], v[2m+1])
// and O[m] = (v[2m+1], v[2m+2]).  Output pair m, tap e reads E[m] (e = 0),
// O[m] (e = 1) or E[m+1] (e = 2).
struct DwRowPairs {
    uint64_t E[5];
    uint64_t O[4];
};

// lf, rt: the neighbour values as fp32 bits.
__device__ __forceinline__ void dw_unpack(const uint4& vec, uint32_t lf, uint32_t rt,
                                          DwRowPairs& u)
{
    const uint32_t w4[4] = {vec.x, vec.y, vec.z, vec.w};
    float v[10];
    v[0] = __uint_as_float(lf);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[1 + 2 * j] = __uint_as_float(w4[j] << 16);
        v[2 + 2 * j] = __uint_as_float(w4[j] & 0xFFFF0000u);
    }
    v[9] = __uint_as_float(rt);
#pragma unroll
    for (int m = 0; m < 5; ++m)
        u.E[m] = f32x2_pack(v[2 * m], v[2 * m + 1]);
#pragma unroll
    for (int m = 0; m < 4; ++m)
        u.O[m] = f32x2_pack(v[2 * m + 1], v[2 * m + 2]);
}

// The channel's 3x3 weights (row-major), each duplicated into both halves.
__device__ __forceinline__ void dw_weights(const uint16_t* Kc, uint64_t (&k2)[9])
{
#pragma unroll
    for (int m = 0; m < 9; ++m) {
        const float kv = __bfloat162float(__ushort_as_bfloat16(Kc[m]));
        k2[m] = f32x2_pack(kv, kv);
    }
}

// Eight consecutive outputs from input rows h-1, h, h+1 (u[0], u[1], u[2]).
// Per output the fp32 sum runs over (a, e) in lexicographic order from 0;
// the result is rounded to bf16 (nearest even).
__device__ __forceinline__ uint4 dw3x3_pairs8(const DwRowPairs (&u)[3], const uint64_t (&k2)[9])
{
    uint64_t acc[4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
        acc[m] = 0ull;
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int e = 0; e < 3; ++e)
#pragma unroll
            for (int m = 0; m < 4; ++m)
                f32x2_fma(acc[m], k2[a * 3 + e],
                          e == 0 ? u[a].E[m] : (e == 1 ? u[a].O[m] : u[a].E[m + 1]));
    uint32_t packed[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float lo, hi;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[m]));
        const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        packed[m] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// The same ten input values of one row as plain fp32 (v[0] = left
// neighbour, v[1..8] = the vector, v[9] = right neighbour).
struct DwRowF {
    float v[10];
};

__device__ __forceinline__ void dw_unpack_f(const uint4& vec, uint32_t lf, uint32_t rt, DwRowF& u)
{
    const uint32_t w4[4] = {vec.x, vec.y, vec.z, vec.w};
    u.v[0] = __uint_as_float(lf);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        u.v[1 + 2 * j] = __uint_as_float(w4[j] << 16);
        u.v[2 + 2 * j] = __uint_as_float(w4[j] & 0xFFFF0000u);
    }
    u.v[9] = __uint_as_float(rt);
}

// dw3x3_pairs8 with one fp32 fused multiply-add per instruction: the same
// operations on every output in the same order, so the same bits.
__device__ __forceinline__ uint4 dw3x3_f8(const DwRowF& u0, const DwRowF& u1, const DwRowF& u2,
                                          const float (&k)[9])
{
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        acc[j] = 0.0f;
    const DwRowF* rows[3] = {&u0, &u1, &u2};
#pragma unroll
    for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int e = 0; e < 3; ++e)
#pragma unroll
            for (int j = 0; j < 8; ++j)
                acc[j] = __fmaf_rn(k[a * 3 + e], rows[a]->v[j + e], acc[j]);
    uint32_t packed[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * m], acc[2 * m + 1]);
        packed[m] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// rows[a] points at element 8*v of input row h-1+a, or is null for a row
// outside the image (read as zeros); v is the vector index in the row and
// nvec the vectors per row (W / 8).
__device__ __forceinline__ uint4 dw3x3_row8(const uint16_t* const (&rows)[3], int v, int nvec,
                                            const uint64_t (&k2)[9])
{
    DwRowPairs u[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
        const uint16_t* row = rows[a];
        if (row != nullptr) {
            const uint32_t lf = v > 0 ? (uint32_t)row[-1] << 16 : 0u;
            const uint32_t rt = v + 1 < nvec ? (uint32_t)row[8] << 16 : 0u;
            dw_unpack(*reinterpret_cast<const uint4*>(row), lf, rt, u[a]);
        } else {
            dw_unpack(make_uint4(0, 0, 0, 0), 0u, 0u, u[a]);
        }
    }
    return dw3x3_pairs8(u, k2);
}

}  // namespace wbmm
