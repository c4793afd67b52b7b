// Template dispatch for the decode kernels: maps the runtime shape (Dh, page
// size, heads per warp GW, consumer warps NW) onto a compiled instance, sets
// its shared-memory limit once per device, and launches it.
#pragma once

#include <atomic>
#include <utility>

#include "decode_kernel.cuh"

namespace kvp {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream finishes; every kernel of this
// library starts with griddepcontrol.wait, so nothing is read early.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int DT, int DH, int P, int GW, int NW>
cudaError_t launch_decode_inst(const DecodeParams& p, dim3 grid, cudaStream_t st) {
    using C = DecodeCfg<DT, DH, P, GW, NW>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(paged_decode_kernel<DT, DH, P, GW, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(paged_decode_kernel<DT, DH, P, GW, NW>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(paged_decode_kernel<DT, DH, P, GW, NW>, grid, dim3(C::kThreads), C::kSmem, st, p);
}

template <int DT, int DH, int P>
cudaError_t launch_decode_gw(const DecodeParams& p, int GW, int NW, dim3 grid, cudaStream_t st) {
    if (NW == 4) {
        if (GW == 4) return launch_decode_inst<DT, DH, P, 4, 4>(p, grid, st);
        if (GW == 2) return launch_decode_inst<DT, DH, P, 2, 4>(p, grid, st);
        return launch_decode_inst<DT, DH, P, 1, 4>(p, grid, st);
    }
    if (GW == 4) return launch_decode_inst<DT, DH, P, 4, 8>(p, grid, st);
    if (GW == 2) return launch_decode_inst<DT, DH, P, 2, 8>(p, grid, st);
    return launch_decode_inst<DT, DH, P, 1, 8>(p, grid, st);
}

template <int DT>
cudaError_t launch_decode_dt(const DecodeParams& p, int DH, int P, int GW, int NW, dim3 grid, cudaStream_t st) {
    if (DH == 128) {
        return P == 16 ? launch_decode_gw<DT, 128, 16>(p, GW, NW, grid, st)
                       : launch_decode_gw<DT, 128, 32>(p, GW, NW, grid, st);
    }
    return P == 16 ? launch_decode_gw<DT, 64, 16>(p, GW, NW, grid, st) : launch_decode_gw<DT, 64, 32>(p, GW, NW, grid, st);
}

// Defined in decode_f32.cu / decode_bf16.cu / decode_f16.cu.
cudaError_t launch_decode_f32(const DecodeParams& p, int DH, int P, int GW, int NW, dim3 grid, cudaStream_t st);
cudaError_t launch_decode_bf16(const DecodeParams& p, int DH, int P, int GW, int NW, dim3 grid, cudaStream_t st);
cudaError_t launch_decode_f16(const DecodeParams& p, int DH, int P, int GW, int NW, dim3 grid, cudaStream_t st);

}  // namespace kvp

// ---- tensor-core variant (bf16 / fp16) ------------------------------------
#include "decode_mma.cuh"

namespace kvp {

template <int KT, int QT, int DH, int P, bool LO, bool QM = false>
cudaError_t launch_mma_inst(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, dim3 grid,
                            cudaStream_t st) {
    constexpr int NW = 4;
    // E4M3 pages of 16 tokens are half the bytes of a 16-bit page: two of them share a stage
    constexpr int PPS = (KT == KV_DTYPE_FP8_E4M3 && P == 16) ? 2 : 1;
    using C = MmaCfg<DH, P, NW, KT == KV_DTYPE_FP8_E4M3 ? 1 : 2, PPS>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    auto* kern = paged_decode_mma_kernel<KT, QT, DH, P, NW, LO, PPS, QM>;
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    return launch_pdl(kern, grid, dim3(C::kThreads), C::kSmem, st, p, tk, tv);
}

// Groups of at most 8 heads take the instance that carries the probability
// residual in the MMA's padding rows.
template <int KT, int QT, int DH, int P>
cudaError_t launch_mma_group(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, dim3 grid,
                             cudaStream_t st) {
    return p.g <= 8 ? launch_mma_inst<KT, QT, DH, P, true>(p, tk, tv, grid, st)
                    : launch_mma_inst<KT, QT, DH, P, false>(p, tk, tv, grid, st);
}

template <int KT, int QT>
cudaError_t launch_mma_dt(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P, dim3 grid,
                          cudaStream_t st) {
    if (DH == 128)
        return P == 16 ? launch_mma_group<KT, QT, 128, 16>(p, tk, tv, grid, st)
                       : launch_mma_group<KT, QT, 128, 32>(p, tk, tv, grid, st);
    return P == 16 ? launch_mma_group<KT, QT, 64, 16>(p, tk, tv, grid, st)
                   : launch_mma_group<KT, QT, 64, 32>(p, tk, tv, grid, st);
}

// Multi-token query (chunk of new tokens per sequence, causal within it).
template <int KT>
cudaError_t launch_prefill_dt(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P,
                              dim3 grid, cudaStream_t st) {
    if (DH == 128)
        return P == 16 ? launch_mma_inst<KT, KT, 128, 16, false, true>(p, tk, tv, grid, st)
                       : launch_mma_inst<KT, KT, 128, 32, false, true>(p, tk, tv, grid, st);
    return P == 16 ? launch_mma_inst<KT, KT, 64, 16, false, true>(p, tk, tv, grid, st)
                   : launch_mma_inst<KT, KT, 64, 32, false, true>(p, tk, tv, grid, st);
}

// Defined in decode_mma_bf16.cu / decode_mma_f16.cu / decode_mma_fp8.cu.
cudaError_t launch_prefill_bf16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P,
                                dim3 grid, cudaStream_t st);
cudaError_t launch_prefill_f16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P,
                               dim3 grid, cudaStream_t st);
cudaError_t launch_mma_bf16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P, dim3 grid,
                            cudaStream_t st);
cudaError_t launch_mma_f16(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int DH, int P, dim3 grid,
                           cudaStream_t st);
// tcgen05 kernel (decode_tc.cu): g = 32, Dh = 128, bf16 / fp16 K/V; n_work items over `grid` persistent CTAs.
cudaError_t launch_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                      int dtype, int P, int n_work, int grid, cudaStream_t st);
// tcgen05 multi-token query kernel (prefill_tc.cu): Dh = 128, 128 % g == 0, bf16 / fp16 K/V.
cudaError_t launch_prefill_tc(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int dtype, int P,
                              dim3 grid, cudaStream_t st);
// tcgen05 kernel over E4M3 K/V (decode_tc_fp8.cu): g in {4, 8, 16}, Dh = 128, q of type q_dtype (bf16 or
// fp16); n_work items over `grid` persistent CTAs.
cudaError_t launch_tc_fp8(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int q_dtype, int P,
                          int n_work, int grid, cudaStream_t st);
// E4M3 K/V with q of type q_dtype (bf16 or fp16).
cudaError_t launch_mma_fp8(const DecodeParams& p, const CUtensorMap& tk, const CUtensorMap& tv, int q_dtype, int DH,
                           int P, dim3 grid, cudaStream_t st);

}  // namespace kvp
