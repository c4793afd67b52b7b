// Compiled instances of the tcgen05 multi-token query kernel (Dh = 128;
// bf16 and fp16 K/V; page size 16 and 32) and their launch.
#include <atomic>

#include "decode_launch.cuh"
#include "prefill_tc.cuh"

namespace kvp {

template <int KT, int P>
cudaError_t launch_prefill_tc_inst(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, dim3 grid,
                                   cudaStream_t st) {
    using C = PfCfg<128, P>;
    auto* kern = paged_prefill_tc_kernel<KT, 128, P>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        // the kernel moves registers between its warpgroups (setmaxnreg): the shares must fit in what a CTA
        // is launched with, or the warpgroup asking for more would wait for ever
        cudaFuncAttributes fa{};
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        const long long pool = static_cast<long long>(fa.numRegs) * C::kThreads;
        const long long need = 128LL * C::kRegsLow + 256LL * C::kRegsHigh;
        if (need > pool) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(kern, grid, dim3(C::kThreads), C::kSmem, st, p, tk, tv);
}

cudaError_t launch_prefill_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int dtype, int P,
                              dim3 grid, cudaStream_t st) {
    if (dtype == KV_DTYPE_BF16)
        return P == 16 ? launch_prefill_tc_inst<KV_DTYPE_BF16, 16>(p, tk, tv, grid, st)
                       : launch_prefill_tc_inst<KV_DTYPE_BF16, 32>(p, tk, tv, grid, st);
    return P == 16 ? launch_prefill_tc_inst<KV_DTYPE_F16, 16>(p, tk, tv, grid, st)
                   : launch_prefill_tc_inst<KV_DTYPE_F16, 32>(p, tk, tv, grid, st);
}

}  // namespace kvp
