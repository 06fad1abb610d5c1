// Row helpers shared by the row-moving kernels (permute/combine and their
// expert-parallel forms): eight bf16 values per 16-byte vector, fp32 math.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ void fma_bf16x8(float *acc, float w, const uint4 &v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xffff0000u), acc[2 * i + 1]);
    }
}

__device__ __forceinline__ void add_bf16x8(float *acc, const uint4 &v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(u[i] << 16);
        acc[2 * i + 1] += __uint_as_float(u[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float *acc) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        u[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
}

}  // namespace moe
