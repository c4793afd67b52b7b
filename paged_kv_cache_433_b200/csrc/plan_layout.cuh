// Layout constants of the device work plans (written by the plan kernels,
// read by the decode and combine kernels and sized by the host).
#pragma once

#include <cstdint>

namespace kvp {

constexpr int kPlanHdr = 4;  // header words before the per-sequence arrays

// Balanced plan (paged_plan_stream_kernel): [0] kPlanStream, [1] G | v << 16,
// [2], [3] T (int64), [4 ..] S_b (int64, B + 1 entries), then cta_row[G].
constexpr int32_t kPlanStream = -2;

__host__ __device__ __forceinline__ int32_t plan_stream_G(const int32_t* plan) { return plan[1] & 0xffff; }
__host__ __device__ __forceinline__ int32_t plan_stream_v(const int32_t* plan) {
    return static_cast<int32_t>(static_cast<uint32_t>(plan[1]) >> 16);
}
__host__ __device__ __forceinline__ int64_t plan_stream_T(const int32_t* plan) {
    return static_cast<int64_t>(static_cast<uint32_t>(plan[2])) | (static_cast<int64_t>(plan[3]) << 32);
}

__host__ __device__ __forceinline__ int64_t* plan_stream_prefix(int32_t* plan) {
    return reinterpret_cast<int64_t*>(plan + kPlanHdr);
}
__host__ __device__ __forceinline__ const int64_t* plan_stream_prefix(const int32_t* plan) {
    return reinterpret_cast<const int64_t*>(plan + kPlanHdr);
}
__host__ __device__ __forceinline__ int64_t plan_stream_words(int32_t B, int64_t grid) {
    return kPlanHdr + 2LL * (B + 1) + grid;
}
// first CTA (of G) whose range holds page x (0 <= x < T): the largest c with floor(c T / G) <= x
__host__ __device__ __forceinline__ int32_t plan_stream_cta(int64_t x, int64_t T, int32_t G) {
    return static_cast<int32_t>(((x + 1) * G - 1) / T);
}

}  // namespace kvp
