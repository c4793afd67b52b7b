// Rotary-embedding arithmetic shared by kv_rope_append and the fused
// rotate + append + decode launch: 16-byte vectors of bf16 / fp16 / fp32
// unpacked to fp32 and packed back with round-to-nearest-even, and the pair
// rotation with every product and sum rounded to fp32 on its own.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "kvpaged.h"

namespace kvp {

template <int DT>
struct RopeVec;

template <>
struct RopeVec<KV_DTYPE_BF16> {
    static constexpr int kN = 8;
    __device__ static void load(const uint4& v, float* x) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static uint4 store(const float* x) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat16 lo = __float2bfloat16_rn(x[2 * i]);
            const __nv_bfloat16 hi = __float2bfloat16_rn(x[2 * i + 1]);
            w[i] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct RopeVec<KV_DTYPE_F16> {
    static constexpr int kN = 8;
    __device__ static void load(const uint4& v, float* x) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xffffu)));
            x[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
        }
    }
    __device__ static uint4 store(const float* x) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half lo = __float2half_rn(x[2 * i]);
            const __half hi = __float2half_rn(x[2 * i + 1]);
            w[i] = static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct RopeVec<KV_DTYPE_F32> {
    static constexpr int kN = 4;
    __device__ static void load(const uint4& v, float* x) {
        x[0] = __uint_as_float(v.x);
        x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z);
        x[3] = __uint_as_float(v.w);
    }
    __device__ static uint4 store(const float* x) {
        return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
    }
};

// x_i' = x_i c - x_j s, x_j' = x_j c + x_i s, each operation rounded to fp32.
__device__ __forceinline__ void rotate_pair(float& xi, float& xj, float c, float s) {
    const float a = __fsub_rn(__fmul_rn(xi, c), __fmul_rn(xj, s));
    const float b = __fadd_rn(__fmul_rn(xj, c), __fmul_rn(xi, s));
    xi = a;
    xj = b;
}

}  // namespace kvp
