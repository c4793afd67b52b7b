// Compiled instances of the tcgen05 decode kernel over E4M3 K/V
// (decode_tc_fp8.cuh: GQA groups of 4, 8 and 16 heads, Dh = 128; q in bf16 or
// fp16; page size 16 and 32) and their launch.
#include <atomic>

#include "decode_launch.cuh"
#include "decode_tc_fp8.cuh"

namespace kvp {

template <int QT, int P, int G>
cudaError_t launch_tc_fp8_inst(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int n_work,
                               int grid, cudaStream_t st) {
    using C = TcF8Cfg<P, G>;
    auto* kern = paged_decode_tc_fp8_kernel<QT, P, G>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        // the warpgroups' register shares (setmaxnreg) must fit in what a CTA is launched with, or a
        // warpgroup asking for more would wait for ever
        cudaFuncAttributes fa{};
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        const long long pool = static_cast<long long>(fa.numRegs) * C::kThreads;
        const long long need = 128LL * (C::kRegsLow + C::kRegsSoftmax + C::kRegsEpi + C::kRegsConvK + C::kRegsConvV);
        if (need > pool) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(kern, dim3(grid), dim3(C::kThreads), C::kSmem, st, p, tk, tv, n_work);
}

template <int QT, int G>
cudaError_t launch_tc_fp8_page(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int P, int n_work,
                               int grid, cudaStream_t st) {
    return P == 16 ? launch_tc_fp8_inst<QT, 16, G>(p, tk, tv, n_work, grid, st)
                   : launch_tc_fp8_inst<QT, 32, G>(p, tk, tv, n_work, grid, st);
}

template <int QT>
cudaError_t launch_tc_fp8_q(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int P, int n_work,
                            int grid, cudaStream_t st) {
    switch (p.g) {
        case 4: return launch_tc_fp8_page<QT, 4>(p, tk, tv, P, n_work, grid, st);
        case 8: return launch_tc_fp8_page<QT, 8>(p, tk, tv, P, n_work, grid, st);
        default: return launch_tc_fp8_page<QT, 16>(p, tk, tv, P, n_work, grid, st);
    }
}

cudaError_t launch_tc_fp8(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int q_dtype, int P,
                          int n_work, int grid, cudaStream_t st) {
    return q_dtype == KV_DTYPE_BF16 ? launch_tc_fp8_q<KV_DTYPE_BF16>(p, tk, tv, P, n_work, grid, st)
                                    : launch_tc_fp8_q<KV_DTYPE_F16>(p, tk, tv, P, n_work, grid, st);
}

}  // namespace kvp
