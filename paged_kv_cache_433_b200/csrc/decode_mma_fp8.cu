// Compiled tensor-core decode instances for E4M3 K/V (q in bf16 or fp16).
#include "decode_launch.cuh"

namespace kvp {

cudaError_t launch_mma_fp8(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int q_dtype, int DH,
                           int P, dim3 grid, cudaStream_t st) {
    return q_dtype == KV_DTYPE_BF16 ? launch_mma_dt<KV_DTYPE_FP8_E4M3, KV_DTYPE_BF16>(p, tk, tv, DH, P, grid, st)
                                    : launch_mma_dt<KV_DTYPE_FP8_E4M3, KV_DTYPE_F16>(p, tk, tv, DH, P, grid, st);
}

}  // namespace kvp
