// Compiled instances of the tcgen05 decode kernel (GQA groups of 4, 8, 16 and
// 32 heads, Dh = 128; bf16 and fp16 K/V; page size 16 and 32) and their launch.
#include <atomic>

#include "decode_launch.cuh"
#include "decode_tc.cuh"

namespace kvp {

template <int KT, int P, int G>
cudaError_t launch_tc_inst(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                           int n_work, int grid, cudaStream_t st) {
    using C = TcCfg<128, P, G>;
    auto* kern = paged_decode_tc_kernel<KT, 128, P, G>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        // the kernel moves registers between its warpgroups (setmaxnreg): the shares must fit in what a CTA
        // is launched with, or a warpgroup asking for more would wait for ever
        cudaFuncAttributes fa{};
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        const long long pool = static_cast<long long>(fa.numRegs) * C::kThreads;
        const long long need = 128LL * (C::kRegsLow + C::kRegsSoftmax + C::kRegsEpi);
        if (need > pool) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmem, st, p, tk, tv, tq, n_work);
}

template <int KT, int G>
cudaError_t launch_tc_page(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                           int P, int n_work, int grid, cudaStream_t st) {
    return P == 16 ? launch_tc_inst<KT, 16, G>(p, tk, tv, tq, n_work, grid, st)
                   : launch_tc_inst<KT, 32, G>(p, tk, tv, tq, n_work, grid, st);
}

template <int KT>
cudaError_t launch_tc_dt(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                         int P, int n_work, int grid, cudaStream_t st) {
    switch (p.g) {
        case 4: return launch_tc_page<KT, 4>(p, tk, tv, tq, P, n_work, grid, st);
        case 8: return launch_tc_page<KT, 8>(p, tk, tv, tq, P, n_work, grid, st);
        case 16: return launch_tc_page<KT, 16>(p, tk, tv, tq, P, n_work, grid, st);
        default: return launch_tc_page<KT, 32>(p, tk, tv, tq, P, n_work, grid, st);
    }
}

cudaError_t launch_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                      int dtype, int P, int n_work, int grid, cudaStream_t st) {
    return dtype == KV_DTYPE_BF16 ? launch_tc_dt<KV_DTYPE_BF16>(p, tk, tv, tq, P, n_work, grid, st)
                                  : launch_tc_dt<KV_DTYPE_F16>(p, tk, tv, tq, P, n_work, grid, st);
}

}  // namespace kvp
