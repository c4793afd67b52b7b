// Compiled decode-kernel instances for one storage dtype (split per dtype so
// the instances build in parallel).
#include "decode_launch.cuh"

namespace kvp {

cudaError_t launch_decode_f16(const DecodeParams& p, int DH, int P, int GW, int NW, dim3 grid, cudaStream_t st) {
    return launch_decode_dt<KV_DTYPE_F16>(p, DH, P, GW, NW, grid, st);
}

}  // namespace kvp
