// Compiled tensor-core decode instances for one storage dtype.
#include "decode_launch.cuh"

namespace kvp {

cudaError_t launch_mma_bf16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P, dim3 grid,
                          cudaStream_t st) {
    return launch_mma_dt<KV_DTYPE_BF16, KV_DTYPE_BF16>(p, tk, tv, DH, P, grid, st);
}

cudaError_t launch_prefill_bf16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P,
                                dim3 grid, cudaStream_t st) {
    return launch_prefill_dt<KV_DTYPE_BF16>(p, tk, tv, DH, P, grid, st);
}

}  // namespace kvp
