// Compiled tensor-core decode instances for one storage dtype.
#include "decode_launch.cuh"

namespace kvp {

cudaError_t launch_mma_f16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P, dim3 grid,
                          cudaStream_t st) {
    return launch_mma_dt<KV_DTYPE_F16, KV_DTYPE_F16>(p, tk, tv, DH, P, grid, st);
}

cudaError_t launch_prefill_f16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P,
                                dim3 grid, cudaStream_t st) {
    return launch_prefill_dt<KV_DTYPE_F16>(p, tk, tv, DH, P, grid, st);
}

}  // namespace kvp
