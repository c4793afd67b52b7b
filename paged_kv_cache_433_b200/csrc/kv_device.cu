// Device entry points of the C ABI: kv_append and paged_decode_attention
// (argument checks, split-KV planning, launches). The kernels themselves are
// in decode_kernel.cuh; see include/kvpaged.h for the contract.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "combine_kernel.cuh"
#include "decode_launch.cuh"
#include "fp8.cuh"
#include "kvpaged.h"
#include "plan_kernel.cuh"

namespace kvp {

// New token's K/V rows -> their slots ("07｜KV Cache、FlashAttention与
// PagedAttention的内部过程", Q025: the new K/V are appended to the layer's
// cache before the query attends). One thread moves 16 bytes; the first
// `rows * vpr` threads copy K, the next ones V.
__global__ void __launch_bounds__(256) kv_append_kernel(uint4* __restrict__ k_pages, uint4* __restrict__ v_pages,
                                                        const uint4* __restrict__ k_new,
                                                        const uint4* __restrict__ v_new,
                                                        const int64_t* __restrict__ slots, int64_t rows, int32_t H_kv,
                                                        int32_t vpr, int32_t P, int64_t num_slots, int* err) {
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t per = rows * vpr;
    if (i >= 2 * per) return;
    const bool is_v = i >= per;
    if (is_v) i -= per;
    const int64_t row = i / vpr;
    const int32_t c = static_cast<int32_t>(i - row * vpr);
    const int64_t b = row / H_kv;
    const int32_t h = static_cast<int32_t>(row - b * H_kv);
    const int64_t slot = slots[b];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (!is_v && h == 0 && c == 0 && err) atomicOr(err, KV_DEV_ERR_SLOT);
        return;
    }
    const int64_t page = slot / P, off = slot - page * P;
    const int64_t dst = ((page * H_kv + h) * P + off) * vpr + c;
    if (is_v)
        v_pages[dst] = v_new[i];
    else
        k_pages[dst] = k_new[i];
}

// Whole-page copy for copy-on-write: pair i copies page src[i] to dst[i] in
// both pools (all H_kv heads, all P slots). One thread moves 16 bytes;
// threads run over (pair, K/V, 16-byte word).
__global__ void __launch_bounds__(256) kv_copy_pages_kernel(uint4* __restrict__ k_pages, uint4* __restrict__ v_pages,
                                                            const int32_t* __restrict__ src,
                                                            const int32_t* __restrict__ dst, int32_t n,
                                                            int64_t words_per_page, int32_t num_pages, int* err) {
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    const int64_t total = 2 * (int64_t)n * words_per_page;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t pair_w = i % (n * words_per_page);
        const bool is_v = i >= n * words_per_page;
        const int32_t k = static_cast<int32_t>(pair_w / words_per_page);
        const int64_t w = pair_w - (int64_t)k * words_per_page;
        const int32_t s = src[k], d = dst[k];
        if (s < 0 || s >= num_pages || d < 0 || d >= num_pages) {
            if (w == 0 && !is_v && err) atomicOr(err, KV_DEV_ERR_PAGE_RANGE);
            continue;
        }
        uint4* base = is_v ? v_pages : k_pages;
        base[(int64_t)d * words_per_page + w] = base[(int64_t)s * words_per_page + w];
    }
}

// Quantising append for E4M3 pools: code = E4M3(x / scale[h]) with the
// division in IEEE fp32 and round-to-nearest-even, saturating at +-448. One
// thread converts 16 elements of one row (16 output bytes); the first half of
// the threads serve K, the rest V.
template <int SRC>
__global__ void __launch_bounds__(256) kv_append_fp8_kernel(uint4* __restrict__ k_pages, uint4* __restrict__ v_pages,
                                                            const void* __restrict__ k_new,
                                                            const void* __restrict__ v_new,
                                                            const float* __restrict__ k_scale,
                                                            const float* __restrict__ v_scale,
                                                            const int64_t* __restrict__ slots, int64_t B, int32_t H_kv,
                                                            int32_t cpr, int32_t P, int64_t num_slots, int* err) {
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t per = B * H_kv * cpr;
    if (i >= 2 * per) return;
    const bool is_v = i >= per;
    if (is_v) i -= per;
    const int64_t row = i / cpr;
    const int32_t c = static_cast<int32_t>(i - row * cpr);
    const int64_t b = row / H_kv;
    const int32_t h = static_cast<int32_t>(row - b * H_kv);
    const int64_t slot = slots[b];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (!is_v && h == 0 && c == 0 && err) atomicOr(err, KV_DEV_ERR_SLOT);
        return;
    }
    float x[16];
    if constexpr (SRC == KV_DTYPE_F32) {
        const float4* src = static_cast<const float4*>(is_v ? v_new : k_new) + i * 4;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 f = src[k];
            x[4 * k] = f.x, x[4 * k + 1] = f.y, x[4 * k + 2] = f.z, x[4 * k + 3] = f.w;
        }
    } else {
        const uint4* src = static_cast<const uint4*>(is_v ? v_new : k_new) + i * 2;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint4 u = src[k];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if constexpr (SRC == KV_DTYPE_BF16) {
                    x[8 * k + 2 * j] = __uint_as_float(w[j] << 16);
                    x[8 * k + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
                } else {
                    x[8 * k + 2 * j] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] & 0xffffu)));
                    x[8 * k + 2 * j + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] >> 16)));
                }
            }
        }
    }
    const float sc = (is_v ? v_scale : k_scale)[h];
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t lo = f32x2_to_e4m3x2(__fdiv_rn(x[4 * j], sc), __fdiv_rn(x[4 * j + 1], sc));
        const uint32_t hi = f32x2_to_e4m3x2(__fdiv_rn(x[4 * j + 2], sc), __fdiv_rn(x[4 * j + 3], sc));
        out[j] = lo | (hi << 16);
    }
    const int64_t page = slot / P, off = slot - page * P;
    const int64_t dst = ((page * H_kv + h) * P + off) * cpr + c;
    (is_v ? v_pages : k_pages)[dst] = make_uint4(out[0], out[1], out[2], out[3]);
}

namespace {

int elem_bytes(int32_t dtype) {
    switch (dtype) {
        case KV_DTYPE_F32: return 4;
        case KV_DTYPE_BF16: return 2;
        case KV_DTYPE_F16: return 2;
        case KV_DTYPE_FP8_E4M3: return 1;
        default: return 0;
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    int v = cached[dev & 63].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cached[dev & 63].store(v, std::memory_order_relaxed);
    return v;
}

// The plan and combine kernels run between decode kernels that use most of shared memory: they ask for
// the same L1 / shared-memory split, so an SM need not reconfigure between them (once per device).
int keep_shared_carveout() {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return 0;
    const int c = cudaSharedmemCarveoutMaxShared;
    const auto a = cudaFuncAttributePreferredSharedMemoryCarveout;
    cudaError_t e = cudaFuncSetAttribute(paged_plan_stream_kernel, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_plan_kernel, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_combine_stream_kernel<128>, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_combine_stream_kernel<64>, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_combine_kernel<128, 1>, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_combine_kernel<128, kCombineWarps>, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_combine_kernel<64, 1>, a, c);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(paged_combine_kernel<64, kCombineWarps>, a, c);
    if (e != cudaSuccess) return -1;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return 0;
}

// Heads per consumer warp and consumer warps per CTA for a GQA group of g.
bool plan_group(int32_t g, int* GW, int* HS, int* NW, int* WP) {
    int gw = (g % 4 == 0) ? 4 : (g % 2 == 0) ? 2 : 1;
    int hs = g / gw;
    if (hs > 8) return false;
    int nw = hs <= 4 ? 4 : 8;
    *GW = gw;
    *HS = hs;
    *NW = nw;
    *WP = nw / hs;
    return true;
}

// Split count. Explicit requests are honoured (capped at max_blocks). For
// num_splits == 0, with `slots` = 2 CTAs per SM resident:
//  * B == 1 (every row has the same length): one full wave, S = slots / H_kv;
//  * otherwise (lengths unknown on the host and usually unequal): about six
//    CTAs per slot so late short CTAs even out long ones, S = ceil(6 slots /
//    (B H_kv)), with at least 16 pages per split; S = 1 once rows alone are
//    that many.
//  * E4M3 K/V (kv_bytes == 1): a CTA moves half the bytes per page, so half
//    as many CTAs per slot (8B-shaped layer: S = 2 / 3 / 4 / 6 -> 0.65 /
//    0.64 / 0.62 / 0.58 of the copy peak).
int resolve_splits(int32_t B, int32_t H_kv, int32_t max_blocks, int32_t num_splits, int32_t* S_out, int32_t* C_out,
                   int kv_bytes = 2) {
    int32_t S = num_splits;
    if (S <= 0) {
        int sms = sm_count();
        if (sms <= 0) return KV_ERR_CUDA;
        const int64_t rows = static_cast<int64_t>(B) * H_kv;
        const int64_t slots = 2LL * sms;
        if (B == 1) {
            // one wave, with an eighth of the slots left free: launched early, the CTAs of the previous step's
            // combine still hold registers on some SMs when this launch starts, and a split that filled every
            // slot would send its last CTAs to a second wave (32K context, 32 layers: 878.7 us a step at S = 32,
            // 906.4 at S = 37 = all slots)
            const int64_t free_slots = slots - slots / 8;
            S = static_cast<int32_t>(free_slots / rows > 1 ? free_slots / rows : 1);
        } else {
            const int64_t per_slot = kv_bytes == 1 ? 3 : 6;
            S = static_cast<int32_t>((per_slot * slots + rows - 1) / rows);
            const int32_t cap = max_blocks / 16 > 1 ? max_blocks / 16 : 1;
            if (S > cap) S = cap;
        }
    }
    if (S > max_blocks) S = max_blocks;
    if (S < 1) S = 1;
    const int32_t C = (max_blocks + S - 1) / S;
    S = (max_blocks + C - 1) / C;
    *S_out = S;
    *C_out = C;
    return KV_OK;
}

std::atomic<int> g_kernel_kind{KV_DECODE_KERNEL_AUTO};

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
// Looked up once; the function-local static makes concurrent first calls from
// several host threads safe.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

// A K or V pool [num_pages][H_kv][P][Dh] seen as a 2-D tensor of
// num_pages * H_kv * P rows of Dh elements; boxes of P rows x 128 bytes with
// the 128-byte swizzle (64 elements of 16 bits, or 128 E4M3 codes), or, for
// E4M3 rows of 64 bytes, P rows x 64 bytes with the 64-byte swizzle.
bool make_pool_map(CUtensorMap* m, const void* base, int32_t dtype, int64_t rows, int32_t Dh, int32_t P) {
    auto enc = tensor_map_encoder();
    if (!enc || rows >= (1LL << 32)) return false;
    const int eb = elem_bytes(dtype);
    const int row_bytes = Dh * eb;
    const int box_bytes = row_bytes < 128 ? row_bytes : 128;
    cuuint64_t gdim[2] = {static_cast<cuuint64_t>(Dh), static_cast<cuuint64_t>(rows)};
    cuuint64_t gstride[1] = {static_cast<cuuint64_t>(row_bytes)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes / eb), static_cast<cuuint32_t>(P)};
    cuuint32_t estride[2] = {1, 1};
    const CUtensorMapDataType t = dtype == KV_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                  : dtype == KV_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                          : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    const CUtensorMapSwizzle sw = box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = enc(m, t, 2, const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor cores for 16-bit K/V when the GQA group fits 4 slices of 16 rows.
// E4M3 K/V exist only on the tensor-core kernel.
bool use_mma(int32_t dtype, int32_t g) {
    const int kind = g_kernel_kind.load(std::memory_order_relaxed);
    if (dtype == KV_DTYPE_F32) return false;
    if (kind == KV_DECODE_KERNEL_SIMT && dtype != KV_DTYPE_FP8_E4M3) return false;
    return g <= 64;
}

// The tcgen05 kernel (decode_tc.cuh): 16-bit K/V, Dh = 128, no fused rotation,
// GQA groups of 4, 8, 16 or 32 heads when selected explicitly; the automatic
// selection takes it for groups of 32 (MQA-shaped), where the warp-MMA
// kernel is bound by its per-page MMA work.
// The automatic choice takes the tcgen05 kernel for 32-head groups (MQA-shaped), and for groups of 4, 8
// and 16 when the balanced plan has many rows to even out (B H_kv above four per SM): there it beats the
// warp-MMA kernel's grid split (8B-shaped GQA, B = 256: 0.98 vs 0.91 of the copy peak); with fewer rows
// (B = 64) the two are level and the warp-MMA kernel, which needs no plan, is kept.
// E4M3 K/V (decode_tc_fp8.cuh: pages widened to fp16 on the SM) for groups of 4, 8 and 16 when selected
// explicitly: its sixteen N = 16 MMAs per 128-token stage take ~0.8 us on the tensor pipe, longer than the
// stage's 32 KB take from HBM, and the warp-MMA kernel stays faster (8B-shaped layer, B = 64: 68 vs 115 us).
bool tc_ok(int32_t dtype, int32_t g, int32_t Dh, bool rope, int32_t B, int32_t H_kv, int32_t num_splits) {
    const int kind = g_kernel_kind.load(std::memory_order_relaxed);
    if (dtype == KV_DTYPE_FP8_E4M3)
        return kind == KV_DECODE_KERNEL_TCGEN05 && Dh == 128 && !rope && (g == 4 || g == 8 || g == 16);
    if ((dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_F16) || Dh != 128 || rope) return false;
    const bool shape = g == 4 || g == 8 || g == 16 || g == 32;
    if (kind == KV_DECODE_KERNEL_TCGEN05) return shape;
    if (kind != KV_DECODE_KERNEL_AUTO || !shape) return false;
    if (g == 32) return true;
    const int sms = sm_count();
    return num_splits == 0 && B > 1 && sms > 0 && static_cast<int64_t>(B) * H_kv > 4LL * sms;
}

size_t workspace_for(int32_t B, int32_t H_q, int32_t Dh, int32_t S) {
    if (S <= 1) return 0;
    const size_t rows = static_cast<size_t>(B) * H_q * S;
    return rows * Dh * sizeof(float) + rows * sizeof(float2);
}

// Planned launches (tensor-core kernel, num_splits == 0, B > 1): the grid is
// an upper bound on the plan's chunk count -- 4 chunks per resident slot plus
// one tail chunk per row.
int64_t planned_grid(int32_t B, int32_t H_kv) {
    const int sms = sm_count();
    if (sms <= 0) return -1;
    return 4LL * 2 * sms + static_cast<int64_t>(B) * H_kv;
}

struct PlannedLayout {
    size_t plan_off, items_off, u_off, ml_off, total;
};

PlannedLayout planned_layout(int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int64_t grid) {
    auto r16 = [](size_t x) { return (x + 15) / 16 * 16; };
    const size_t g = static_cast<size_t>(H_q / H_kv);
    PlannedLayout L{};
    L.plan_off = 0;
    L.items_off = r16(sizeof(int32_t) * (kPlanHdr + static_cast<size_t>(B) + 1));
    L.u_off = L.items_off + r16(sizeof(int4) * static_cast<size_t>(grid));
    L.ml_off = L.u_off + r16(sizeof(float) * static_cast<size_t>(grid) * g * Dh);
    L.total = L.ml_off + r16(sizeof(float2) * static_cast<size_t>(grid) * g);
    return L;
}

// Balanced plan of the persistent tcgen05 kernel (paged_plan_stream_kernel):
// the plan words, then two partial slots per CTA.
PlannedLayout stream_layout(int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int64_t grid) {
    auto r16 = [](size_t x) { return (x + 15) / 16 * 16; };
    const size_t g = static_cast<size_t>(H_q / H_kv);
    PlannedLayout L{};
    L.plan_off = 0;
    L.items_off = r16(sizeof(int32_t) * static_cast<size_t>(plan_stream_words(B, grid)));
    L.u_off = L.items_off;  // no item list
    L.ml_off = L.u_off + r16(sizeof(float) * 2 * static_cast<size_t>(grid) * g * Dh);
    L.total = L.ml_off + r16(sizeof(float2) * 2 * static_cast<size_t>(grid) * g);
    return L;
}

// Automatic split choice between the two launch forms. With no more
// (sequence, KV head) rows than two waves of resident CTAs, the grid rule
// splits every row into equal ranges of the longest possible row and keeps
// up (measured on the 8B-shaped B=64 layer and the shared-prefix batch);
// beyond that it cannot split rows at all (S = 1), and in a skewed batch a
// few long rows end the launch alone -- there the plan, which chunks rows by
// their actual lengths on the device, is used.
bool planned_ok(bool mma, int32_t B, int32_t H_q, int32_t H_kv, int32_t num_splits) {
    const int sms = sm_count();
    return mma && num_splits == 0 && B > 1 && B <= kPlanThreads * kPlanRowsPerThread && (H_q / H_kv) <= 64 &&
           sms > 0 && static_cast<int64_t>(B) * H_kv > 4LL * sms;
}

// The tcgen05 kernel is persistent (one CTA per SM walking work items), so it
// takes the device plan for every multi-row batch with the automatic split:
// chunks follow the actual lengths instead of the table width.
bool planned_tc(int32_t B, int32_t num_splits) {
    return num_splits == 0 && B > 1 && B <= kPlanThreads * kPlanRowsPerThread;
}

// A q tensor [rows][Dh] (16-bit) seen as boxes of `box_rows` rows x 128 bytes, 128-byte swizzle.
bool make_q_map(CUtensorMap* m, const void* q, int32_t dtype, int64_t rows, int32_t Dh, int32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc || rows >= (1LL << 32)) return false;
    cuuint64_t gdim[2] = {static_cast<cuuint64_t>(Dh), static_cast<cuuint64_t>(rows)};
    cuuint64_t gstride[1] = {static_cast<cuuint64_t>(Dh) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estride[2] = {1, 1};
    const CUtensorMapDataType t =
        dtype == KV_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = enc(m, t, 2, const_cast<void*>(q), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int check_shape(int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t dtype) {
    if (H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return KV_ERR_ARG;
    if (elem_bytes(dtype) == 0) return KV_ERR_ARG;
    if (Dh != 64 && Dh != 128) return KV_ERR_UNSUPPORTED;
    if (page_size != 16 && page_size != 32) return KV_ERR_UNSUPPORTED;
    int a, b, c, d;
    if (dtype == KV_DTYPE_FP8_E4M3) return use_mma(dtype, H_q / H_kv) ? KV_OK : KV_ERR_UNSUPPORTED;
    if (!use_mma(dtype, H_q / H_kv) && !plan_group(H_q / H_kv, &a, &b, &c, &d)) return KV_ERR_UNSUPPORTED;
    return KV_OK;
}

}  // namespace
}  // namespace kvp

using namespace kvp;

extern "C" {

int kv_append(void* k_pages, void* v_pages, const void* k_new, const void* v_new, const int64_t* slot_mapping,
              int32_t B, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, int32_t dtype, int* err_flag,
              void* stream) {
    const int eb = elem_bytes(dtype);
    if (B < 0 || H_kv <= 0 || Dh <= 0 || page_size <= 0 || num_pages <= 0 || eb == 0) return KV_ERR_ARG;
    if ((static_cast<int64_t>(Dh) * eb) % 16 != 0) return KV_ERR_UNSUPPORTED;
    if (B == 0) return KV_OK;
    if (!k_pages || !v_pages || !k_new || !v_new || !slot_mapping) return KV_ERR_ARG;
    if (!aligned16(k_pages) || !aligned16(v_pages) || !aligned16(k_new) || !aligned16(v_new)) return KV_ERR_ARG;
    const int32_t vpr = Dh * eb / 16;
    const int64_t rows = static_cast<int64_t>(B) * H_kv;
    const int64_t threads = 2 * rows * vpr;
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return KV_ERR_UNSUPPORTED;
    cudaError_t e = launch_pdl(kv_append_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                               static_cast<cudaStream_t>(stream), static_cast<uint4*>(k_pages),
                               static_cast<uint4*>(v_pages), static_cast<const uint4*>(k_new),
                               static_cast<const uint4*>(v_new), slot_mapping, rows, H_kv, vpr, page_size,
                               static_cast<int64_t>(num_pages) * page_size, err_flag);
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

int kv_copy_pages(void* k_pages, void* v_pages, const int32_t* src_pages, const int32_t* dst_pages, int32_t n,
                  int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, int32_t dtype, int* err_flag,
                  void* stream) {
    const int eb = elem_bytes(dtype);
    if (n < 0 || H_kv <= 0 || Dh <= 0 || page_size <= 0 || num_pages <= 0 || eb == 0) return KV_ERR_ARG;
    const int64_t page_bytes = static_cast<int64_t>(H_kv) * page_size * Dh * eb;
    if (page_bytes % 16 != 0) return KV_ERR_UNSUPPORTED;
    if (n == 0) return KV_OK;
    if (!k_pages || !v_pages || !src_pages || !dst_pages || !aligned16(k_pages) || !aligned16(v_pages)) return KV_ERR_ARG;
    const int64_t words = page_bytes / 16;
    const int64_t total = 2 * static_cast<int64_t>(n) * words;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 65535LL * 16) blocks = 65535LL * 16;
    cudaError_t e = launch_pdl(kv_copy_pages_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                               static_cast<cudaStream_t>(stream), static_cast<uint4*>(k_pages),
                               static_cast<uint4*>(v_pages), src_pages, dst_pages, n, words, num_pages, err_flag);
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

int paged_decode_set_kernel(int32_t kind) {
    if (kind != KV_DECODE_KERNEL_AUTO && kind != KV_DECODE_KERNEL_SIMT && kind != KV_DECODE_KERNEL_MMA &&
        kind != KV_DECODE_KERNEL_TCGEN05)
        return KV_ERR_ARG;
    g_kernel_kind.store(kind, std::memory_order_relaxed);
    return KV_OK;
}

int paged_decode_num_splits(int32_t B, int32_t H_kv, int32_t max_blocks, int32_t page_size, int32_t num_splits,
                            int32_t* out) {
    if (!out || B < 0 || H_kv <= 0 || max_blocks <= 0 || page_size <= 0 || num_splits < 0) return KV_ERR_ARG;
    int32_t S, C;
    int rc = resolve_splits(B, H_kv, max_blocks, num_splits, &S, &C);
    if (rc == KV_OK) *out = planned_ok(true, B, /*H_q=*/H_kv, H_kv, num_splits) ? 0 : S;
    return rc;
}

int paged_decode_workspace_bytes(int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t max_blocks,
                                 int32_t page_size, int32_t num_splits, size_t* out) {
    if (!out || B < 0 || H_q <= 0 || H_kv <= 0 || Dh <= 0 || max_blocks <= 0 || page_size <= 0 || num_splits < 0)
        return KV_ERR_ARG;
    int32_t S, C;
    int rc = resolve_splits(B, H_kv, max_blocks, num_splits, &S, &C);
    if (rc != KV_OK) return rc;
    size_t need = workspace_for(B, H_q, Dh, S);
    // the pool dtype is not known here: cover the tcgen05 kernel's balanced plan (16-bit pools) and the
    // chunked plan of the warp-MMA kernel (the other dtypes) wherever either may be chosen
    const bool tc = H_q % H_kv == 0 && (tc_ok(KV_DTYPE_BF16, H_q / H_kv, Dh, false, B, H_kv, num_splits) ||
                                        tc_ok(KV_DTYPE_FP8_E4M3, H_q / H_kv, Dh, false, B, H_kv, num_splits));
    if (tc && planned_tc(B, num_splits)) {
        const int sms = sm_count();
        if (sms <= 0) return KV_ERR_CUDA;
        const size_t pl = stream_layout(B, H_q, H_kv, Dh, sms).total;
        if (pl > need) need = pl;
    }
    if (planned_ok(true, B, H_q, H_kv, num_splits)) {
        const int64_t grid = planned_grid(B, H_kv);
        if (grid < 0) return KV_ERR_CUDA;
        const size_t pl = planned_layout(B, H_q, H_kv, Dh, grid).total;
        if (pl > need) need = pl;
    }
    *out = need;
    return KV_OK;
}

int paged_decode_launch_info(int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t max_blocks, int32_t page_size,
                             int32_t dtype, int32_t num_splits, int32_t* splits, int32_t* kernel) {
    if (!splits || !kernel || B < 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0 || Dh <= 0 || max_blocks <= 0 ||
        page_size <= 0 || num_splits < 0 || elem_bytes(dtype) == 0)
        return KV_ERR_ARG;
    const int32_t g = H_q / H_kv;
    int32_t S, C;
    int rc = resolve_splits(B, H_kv, max_blocks, num_splits, &S, &C, elem_bytes(dtype));
    if (rc != KV_OK) return rc;
    const bool mma = use_mma(dtype, g);
    const bool tc = mma && tc_ok(dtype, g, Dh, false, B, H_kv, num_splits);
    *kernel = tc ? KV_DECODE_KERNEL_TCGEN05 : (mma ? KV_DECODE_KERNEL_MMA : KV_DECODE_KERNEL_SIMT);
    *splits = (tc ? planned_tc(B, num_splits) : planned_ok(mma, B, H_q, H_kv, num_splits)) ? 0 : S;
    return KV_OK;
}

}  // extern "C"

namespace kvp {
namespace {

// dtype: the K/V pools' type; q_dtype: q's (the same for 16-bit and fp32
// K/V; bf16 or fp16 with E4M3 K/V, which also need k_scale / v_scale).
int decode_impl(float* out, const void* q, const void* k_new, const void* v_new, const void* k_pages,
                const void* v_pages, const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t B,
                int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, float scale, int32_t dtype,
                int32_t num_splits, void* workspace, size_t ws_bytes, int* err_flag, void* stream,
                int32_t q_dtype = -1, const float* k_scale = nullptr, const float* v_scale = nullptr,
                const float* cos_sin = nullptr, int32_t max_pos = 0, int32_t rope_style = 0) {
    int rc = check_shape(H_q, H_kv, Dh, page_size, dtype);
    if (rc != KV_OK) return rc;
    if (q_dtype < 0) q_dtype = dtype;
    if (dtype == KV_DTYPE_FP8_E4M3) {
        if (q_dtype != KV_DTYPE_BF16 && q_dtype != KV_DTYPE_F16) return KV_ERR_ARG;
        if (k_new != nullptr || v_new != nullptr) return KV_ERR_UNSUPPORTED;  // quantising append: kv_append_fp8
        if (B > 0 && (!k_scale || !v_scale)) return KV_ERR_ARG;
    } else if (q_dtype != dtype) {
        return KV_ERR_ARG;
    }
    if (B < 0 || max_blocks <= 0 || num_pages <= 0 || num_splits < 0) return KV_ERR_ARG;
    if (B == 0) return KV_OK;
    if (B > 65535 || H_kv > 65535) return KV_ERR_UNSUPPORTED;
    if (!out || !q || !k_pages || !v_pages || !block_tables || !seq_lens) return KV_ERR_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages)) return KV_ERR_ARG;
    const int32_t g = H_q / H_kv;
    // TMA row coordinates are int32: very large pools stay on the CUDA-core kernel.
    const bool mma = use_mma(dtype, g) && static_cast<int64_t>(num_pages) * H_kv * page_size < (1LL << 31);
    if (dtype == KV_DTYPE_FP8_E4M3 && !mma) return KV_ERR_UNSUPPORTED;
    int GW = 0, HS, NW, WP;
    if (mma) {
        HS = (g + 15) / 16;
        NW = 4;
        WP = NW / HS;
    } else {
        plan_group(g, &GW, &HS, &NW, &WP);
    }
    int32_t S, C;
    rc = resolve_splits(B, H_kv, max_blocks, num_splits, &S, &C, elem_bytes(dtype));
    if (rc != KV_OK) return rc;
    const bool tc = mma && tc_ok(dtype, g, Dh, cos_sin != nullptr, B, H_kv, num_splits);
    const bool planned = tc ? planned_tc(B, num_splits) : planned_ok(mma, B, H_q, H_kv, num_splits);

    DecodeParams p{};
    p.out = out;
    p.q = q;
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_pages = k_pages;
    p.v_pages = v_pages;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = err_flag;
    p.max_blocks = max_blocks;
    p.B = B;
    p.H_q = H_q;
    p.H_kv = H_kv;
    p.num_pages = num_pages;
    p.g = H_q / H_kv;
    p.HS = HS;
    p.WP = WP;
    p.num_splits = S;
    p.pages_per_split = C;
    p.scale_log2 = scale * kLog2e;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.cos_sin = cos_sin;
    p.max_pos = max_pos;
    p.rope_style = rope_style;
    if (cos_sin != nullptr && !mma) return KV_ERR_UNSUPPORTED;  // the fused rotation lives in the tensor-core kernel
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dim3 grid(static_cast<unsigned>(S), static_cast<unsigned>(H_kv), static_cast<unsigned>(B));
    cudaError_t e;
    int64_t pgrid = 0;
    const int sms_all = sm_count();
    if (sms_all <= 0 || keep_shared_carveout() != 0) return KV_ERR_CUDA;
    if (planned && tc) {
        // balanced plan: one persistent CTA per SM, each streaming the same number of pages
        pgrid = sms_all;
        const PlannedLayout L = stream_layout(B, H_q, H_kv, Dh, pgrid);
        if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return KV_ERR_WORKSPACE;
        char* w = static_cast<char*>(workspace);
        int32_t* plan = reinterpret_cast<int32_t*>(w + L.plan_off);
        p.plan = plan;
        p.stream_plan = 1;
        p.items = nullptr;
        p.part_u = reinterpret_cast<float*>(w + L.u_off);
        p.part_ml = reinterpret_cast<float2*>(w + L.ml_off);
        p.num_splits = 0;
        // at least two stages of 128 keys per CTA; a work item's fixed cost counted as one stage of pages, three
        // at g = 32, whose items pay CTA-wide reductions over 32 heads (log-normal batch, B = 256: MQA 68.4 vs
        // 72.2 us at P = 16, 69.2 vs 74.1 at P = 32; GQA best at one stage: 8B-shaped B = 64 108.0 vs 110.9 us)
        const int32_t stage_pages = std::max<int32_t>(1, 128 / page_size);
        const int32_t item_pages = stage_pages * (H_q / H_kv >= 32 ? 3 : 1);
        e = launch_pdl(paged_plan_stream_kernel, dim3(1), dim3(kPlanThreads), 0, st, seq_lens, B, H_kv, page_size,
                       max_blocks, static_cast<int32_t>(pgrid), 2 * stage_pages, item_pages, plan, out, H_q, Dh,
                       err_flag);
        if (e != cudaSuccess) return KV_ERR_CUDA;
    } else if (planned) {
        pgrid = planned_grid(B, H_kv);
        if (pgrid < 0) return KV_ERR_CUDA;
        if (pgrid > 0x7fffffffLL) return KV_ERR_UNSUPPORTED;
        const PlannedLayout L = planned_layout(B, H_q, H_kv, Dh, pgrid);
        if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return KV_ERR_WORKSPACE;
        char* w = static_cast<char*>(workspace);
        int32_t* plan = reinterpret_cast<int32_t*>(w + L.plan_off);
        int4* items = reinterpret_cast<int4*>(w + L.items_off);
        p.plan = plan;
        p.items = items;
        p.part_u = reinterpret_cast<float*>(w + L.u_off);
        p.part_ml = reinterpret_cast<float2*>(w + L.ml_off);
        p.num_splits = 0;
        // chunk floor: a chunk's partial (g x (Dh + 2) fp32) at most ~6 % of its K/V bytes
        const int64_t chunk_bytes_per_page = 2LL * page_size * Dh * elem_bytes(dtype);
        const int64_t partial_bytes = static_cast<int64_t>(H_q / H_kv) * (Dh + 2) * 4;
        const int32_t c_floor = static_cast<int32_t>(std::max<int64_t>(8, (16 * partial_bytes + chunk_bytes_per_page - 1) /
                                                                                chunk_bytes_per_page));
        // resident CTAs of the warp-MMA kernel: two per SM
        const int32_t slots = static_cast<int32_t>(2 * sms_all);
        e = launch_pdl(paged_plan_kernel, dim3(1), dim3(kPlanThreads), 0, st, seq_lens, B, H_kv, page_size, max_blocks,
                       slots, static_cast<int32_t>(pgrid), c_floor, plan, items, err_flag);
        if (e != cudaSuccess) return KV_ERR_CUDA;
        grid = dim3(static_cast<unsigned>(pgrid), 1, 1);
    } else if (S > 1) {
        const size_t need = workspace_for(B, H_q, Dh, S);
        if (!workspace || ws_bytes < need || !aligned16(workspace)) return KV_ERR_WORKSPACE;
        const size_t rows = static_cast<size_t>(B) * H_q * S;
        p.part_u = static_cast<float*>(workspace);
        p.part_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) + rows * Dh * sizeof(float));
    }
    if (tc) {
        CUtensorMap tk, tv, tq;
        const int64_t rows = static_cast<int64_t>(num_pages) * H_kv * page_size;
        if (!make_pool_map(&tk, k_pages, dtype, rows, Dh, page_size) ||
            !make_pool_map(&tv, v_pages, dtype, rows, Dh, page_size))
            return KV_ERR_CUDA;
        const int64_t n_work = planned ? pgrid : static_cast<int64_t>(S) * H_kv * B;
        if (n_work > 0x7fffffffLL) return KV_ERR_UNSUPPORTED;
        const int tc_grid = static_cast<int>(std::min<int64_t>(n_work, sms_all));
        if (dtype == KV_DTYPE_FP8_E4M3) {
            e = launch_tc_fp8(p, tk, tv, q_dtype, page_size, static_cast<int>(n_work), tc_grid, st);
        } else {
            if (!make_q_map(&tq, q, dtype, static_cast<int64_t>(B) * H_q, Dh, g)) return KV_ERR_CUDA;
            e = launch_tc(p, tk, tv, tq, dtype, page_size, static_cast<int>(n_work), tc_grid, st);
        }
    } else if (mma) {
        CUtensorMap tk, tv;
        const int64_t rows = static_cast<int64_t>(num_pages) * H_kv * page_size;
        if (!make_pool_map(&tk, k_pages, dtype, rows, Dh, page_size) ||
            !make_pool_map(&tv, v_pages, dtype, rows, Dh, page_size))
            return KV_ERR_CUDA;
        e = dtype == KV_DTYPE_BF16   ? launch_mma_bf16(p, tk, tv, Dh, page_size, grid, st)
            : dtype == KV_DTYPE_F16 ? launch_mma_f16(p, tk, tv, Dh, page_size, grid, st)
                                    : launch_mma_fp8(p, tk, tv, q_dtype, Dh, page_size, grid, st);
    } else {
        switch (dtype) {
            case KV_DTYPE_F32: e = launch_decode_f32(p, Dh, page_size, GW, NW, grid, st); break;
            case KV_DTYPE_BF16: e = launch_decode_bf16(p, Dh, page_size, GW, NW, grid, st); break;
            default: e = launch_decode_f16(p, Dh, page_size, GW, NW, grid, st); break;
        }
    }
    if (e != cudaSuccess) return KV_ERR_CUDA;
    if (planned && tc) {
        // balanced plan: one CTA per range boundary merges the row cut there (if any)
        const dim3 blocks(static_cast<unsigned>(pgrid)), threads(32 * kCombineStreamWarps);
        e = Dh == 128 ? launch_pdl(paged_combine_stream_kernel<128>, blocks, threads, 0, st, out, p.part_u, p.part_ml,
                                   static_cast<const int32_t*>(p.plan), B, H_q, H_kv)
                      : launch_pdl(paged_combine_stream_kernel<64>, blocks, threads, 0, st, out, p.part_u, p.part_ml,
                                   static_cast<const int32_t*>(p.plan), B, H_q, H_kv);
        if (e != cudaSuccess) return KV_ERR_CUDA;
    } else if (planned || S > 1) {
        // one warp per row when a single round of 8 loads per lane covers the splits (and for
        // planned launches, where rows have different chunk counts), else 8 warps per row
        const int64_t rows = static_cast<int64_t>(B) * H_q;
        const bool narrow = planned || S <= 8;
        const int32_t* plan = planned ? p.plan : nullptr;
        const int64_t rows_per_cta = narrow ? kCombineWarps : 1;
        const dim3 blocks(static_cast<unsigned>((rows + rows_per_cta - 1) / rows_per_cta));
        const dim3 threads(32 * kCombineWarps);
        const float2* ml = p.part_ml;
        const float* pu = p.part_u;
        if (Dh == 128)
            e = narrow ? launch_pdl(paged_combine_kernel<128, 1>, blocks, threads, 0, st, out, pu, ml, seq_lens, B, H_q,
                                    S, C, page_size, max_blocks, plan, H_kv)
                       : launch_pdl(paged_combine_kernel<128, kCombineWarps>, blocks, threads, 0, st, out, pu, ml,
                                    seq_lens, B, H_q, S, C, page_size, max_blocks, plan, H_kv);
        else
            e = narrow ? launch_pdl(paged_combine_kernel<64, 1>, blocks, threads, 0, st, out, pu, ml, seq_lens, B, H_q, S,
                                    C, page_size, max_blocks, plan, H_kv)
                       : launch_pdl(paged_combine_kernel<64, kCombineWarps>, blocks, threads, 0, st, out, pu, ml,
                                    seq_lens, B, H_q, S, C, page_size, max_blocks, plan, H_kv);
        if (e != cudaSuccess) return KV_ERR_CUDA;
    }
    return KV_OK;
}

}  // namespace
}  // namespace kvp

extern "C" {

int paged_decode_attention(float* out, const void* q, const void* k_pages, const void* v_pages,
                           const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t B,
                           int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, float scale,
                           int32_t dtype, int32_t num_splits, void* workspace, size_t ws_bytes, int* err_flag,
                           void* stream) {
    return decode_impl(out, q, nullptr, nullptr, k_pages, v_pages, block_tables, max_blocks, seq_lens, B, H_q, H_kv, Dh,
                       page_size, num_pages, scale, dtype, num_splits, workspace, ws_bytes, err_flag, stream);
}

int paged_decode_attention_append(float* out, const void* q, const void* k_new, const void* v_new, void* k_pages,
                                  void* v_pages, const int32_t* block_tables, int32_t max_blocks,
                                  const int32_t* seq_lens, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh,
                                  int32_t page_size, int32_t num_pages, float scale, int32_t dtype, int32_t num_splits,
                                  void* workspace, size_t ws_bytes, int* err_flag, void* stream) {
    if (B > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))) return KV_ERR_ARG;
    return decode_impl(out, q, k_new, v_new, k_pages, v_pages, block_tables, max_blocks, seq_lens, B, H_q, H_kv, Dh,
                       page_size, num_pages, scale, dtype, num_splits, workspace, ws_bytes, err_flag, stream);
}

int paged_decode_attention_fp8(float* out, const void* q, int32_t q_dtype, const void* k_pages, const void* v_pages,
                               const float* k_scale, const float* v_scale, const int32_t* block_tables,
                               int32_t max_blocks, const int32_t* seq_lens, int32_t B, int32_t H_q, int32_t H_kv,
                               int32_t Dh, int32_t page_size, int32_t num_pages, float scale, int32_t num_splits,
                               void* workspace, size_t ws_bytes, int* err_flag, void* stream) {
    return decode_impl(out, q, nullptr, nullptr, k_pages, v_pages, block_tables, max_blocks, seq_lens, B, H_q, H_kv, Dh,
                       page_size, num_pages, scale, KV_DTYPE_FP8_E4M3, num_splits, workspace, ws_bytes, err_flag,
                       stream, q_dtype, k_scale, v_scale);
}

int paged_decode_attention_rope_append(float* out, const void* q, const void* k_new, const void* v_new,
                                       void* k_pages, void* v_pages, const int32_t* block_tables, int32_t max_blocks,
                                       const int32_t* seq_lens, const float* cos_sin, int32_t max_pos,
                                       int32_t rope_style, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh,
                                       int32_t page_size, int32_t num_pages, float scale, int32_t dtype,
                                       int32_t num_splits, void* workspace, size_t ws_bytes, int* err_flag,
                                       void* stream) {
    if (dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_F16) return dtype == KV_DTYPE_F32 ? KV_ERR_UNSUPPORTED : KV_ERR_ARG;
    if (rope_style != KV_ROPE_HALF && rope_style != KV_ROPE_INTERLEAVED) return KV_ERR_ARG;
    if (B > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) || !cos_sin || max_pos <= 0))
        return KV_ERR_ARG;
    return decode_impl(out, q, k_new, v_new, k_pages, v_pages, block_tables, max_blocks, seq_lens, B, H_q, H_kv, Dh,
                       page_size, num_pages, scale, dtype, num_splits, workspace, ws_bytes, err_flag, stream, dtype,
                       nullptr, nullptr, cos_sin, max_pos, rope_style);
}

int paged_prefill_attention(float* out, const void* q, const int32_t* q_start, int32_t max_q_len,
                            const void* k_pages, const void* v_pages, const int32_t* block_tables, int32_t max_blocks,
                            const int32_t* seq_lens, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh,
                            int32_t page_size, int32_t num_pages, float scale, int32_t dtype, int* err_flag,
                            void* stream) {
    if (dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_F16) return dtype == KV_DTYPE_F32 ? KV_ERR_UNSUPPORTED : KV_ERR_ARG;
    if (H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return KV_ERR_ARG;
    if (Dh != 64 && Dh != 128) return KV_ERR_UNSUPPORTED;
    if (page_size != 16 && page_size != 32) return KV_ERR_UNSUPPORTED;
    const int32_t g = H_q / H_kv;
    if (g > 64) return KV_ERR_UNSUPPORTED;
    if (B < 0 || max_q_len < 0 || max_blocks <= 0 || num_pages <= 0) return KV_ERR_ARG;
    if (B == 0 || max_q_len == 0) return KV_OK;
    if (B > 65535 || H_kv > 65535) return KV_ERR_UNSUPPORTED;
    if (!out || !q || !q_start || !k_pages || !v_pages || !block_tables || !seq_lens) return KV_ERR_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages)) return KV_ERR_ARG;
    if (static_cast<int64_t>(num_pages) * H_kv * page_size >= (1LL << 31)) return KV_ERR_UNSUPPORTED;
    // tcgen05 kernel: 128 MMA rows per CTA (128 / g chunk tokens x g heads); warp-MMA kernel: 64 rows
    // (64 / g tokens, four 16-row slices)
    const int kind = g_kernel_kind.load(std::memory_order_relaxed);
    const bool tc = (kind == KV_DECODE_KERNEL_AUTO || kind == KV_DECODE_KERNEL_TCGEN05) && Dh == 128 && 128 % g == 0;
    const int32_t q_tile = tc ? 128 / g : 64 / g;
    DecodeParams p{};
    p.out = out;
    p.q = q;
    p.k_pages = k_pages;
    p.v_pages = v_pages;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = err_flag;
    p.max_blocks = max_blocks;
    p.B = B;
    p.H_q = H_q;
    p.H_kv = H_kv;
    p.num_pages = num_pages;
    p.g = g;
    p.HS = (q_tile * g + 15) / 16;
    p.WP = 4 / p.HS;
    p.num_splits = 1;
    p.pages_per_split = max_blocks;
    p.scale_log2 = scale * kLog2e;
    p.q_start = q_start;
    p.q_tile = q_tile;
    CUtensorMap tk, tv;
    const int64_t rows = static_cast<int64_t>(num_pages) * H_kv * page_size;
    if (!make_pool_map(&tk, k_pages, dtype, rows, Dh, page_size) || !make_pool_map(&tv, v_pages, dtype, rows, Dh, page_size))
        return KV_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>((max_q_len + q_tile - 1) / q_tile), static_cast<unsigned>(H_kv),
                    static_cast<unsigned>(B));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = tc                       ? launch_prefill_tc(p, tk, tv, dtype, page_size, grid, st)
                          : dtype == KV_DTYPE_BF16 ? launch_prefill_bf16(p, tk, tv, Dh, page_size, grid, st)
                                                   : launch_prefill_f16(p, tk, tv, Dh, page_size, grid, st);
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

int kv_append_fp8(void* k_pages, void* v_pages, const void* k_new, const void* v_new, int32_t src_dtype,
                  const float* k_scale, const float* v_scale, const int64_t* slot_mapping, int32_t B, int32_t H_kv,
                  int32_t Dh, int32_t page_size, int32_t num_pages, int* err_flag, void* stream) {
    const int eb = elem_bytes(src_dtype);
    if (B < 0 || H_kv <= 0 || Dh <= 0 || page_size <= 0 || num_pages <= 0 || eb == 0 || src_dtype == KV_DTYPE_FP8_E4M3)
        return KV_ERR_ARG;
    if (Dh % 16 != 0) return KV_ERR_UNSUPPORTED;
    if (B == 0) return KV_OK;
    if (!k_pages || !v_pages || !k_new || !v_new || !slot_mapping || !k_scale || !v_scale) return KV_ERR_ARG;
    if (!aligned16(k_pages) || !aligned16(v_pages) || !aligned16(k_new) || !aligned16(v_new)) return KV_ERR_ARG;
    const int32_t cpr = Dh / 16;  // 16-code groups per row
    const int64_t threads = 2LL * B * H_kv * cpr;
    int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return KV_ERR_UNSUPPORTED;
    auto* kern = src_dtype == KV_DTYPE_BF16  ? kv_append_fp8_kernel<KV_DTYPE_BF16>
                 : src_dtype == KV_DTYPE_F16 ? kv_append_fp8_kernel<KV_DTYPE_F16>
                                             : kv_append_fp8_kernel<KV_DTYPE_F32>;
    cudaError_t e = launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, static_cast<cudaStream_t>(stream),
                               static_cast<uint4*>(k_pages), static_cast<uint4*>(v_pages), k_new, v_new, k_scale,
                               v_scale, slot_mapping, static_cast<int64_t>(B), H_kv, cpr, page_size,
                               static_cast<int64_t>(num_pages) * page_size, err_flag);
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

}  // extern "C"
