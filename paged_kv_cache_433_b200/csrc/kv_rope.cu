// Rotary position embedding fused with the KV append ("06 KV Cache、Prefix
// Cache、PagedAttention 与 vLLM", 6.1: a new token's q and k are rotated by
// its position before k and v are appended and q attends).
//
// A thread owns one pair of 16-byte vectors of a row: for the split-halves
// pairing the vector at element e (< Dh/2) and the one at e + Dh/2, for the
// interleaved pairing two adjacent vectors. Both cover the same run of pair
// indices k, so the thread loads those cos / sin entries of the token's table
// row as float4s. Rows are, per token: H_q query heads (rotated into q_out),
// H_kv key heads (rotated into the K page slot) and H_kv value heads (copied
// into the V page slot). The rotation is done in fp32 with every product and
// sum rounded on its own (__fmul_rn / __fadd_rn / __fsub_rn, which the
// compiler never contracts into an FMA), then rounded to the storage dtype
// with round-to-nearest-even: the stored bits are fully determined.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "decode_launch.cuh"
#include "kvpaged.h"
#include "rope.cuh"

namespace kvp {
namespace {

// Thread t of a CTA owns unit t of a token (row r = t / upr, vector pair u;
// loops when a token has more units than the CTA has threads) and walks the
// tokens blockIdx.x, + gridDim.x, ...: the unit's row, vectors and pair
// indices are computed once, the token loop holds no division.
template <int DT>
__global__ void __launch_bounds__(384, 3) kv_rope_append_kernel(
    uint4* __restrict__ k_pages, uint4* __restrict__ v_pages, uint4* q_out, const uint4* q,
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, const int64_t* __restrict__ slots,
    const int32_t* __restrict__ positions, const float* __restrict__ cos_sin, int32_t max_pos, int32_t style, int64_t B,
    int32_t H_q, int32_t H_kv, int32_t Dh, int32_t P, int64_t num_slots, int* err) {
    using V = RopeVec<DT>;
    constexpr int N = V::kN;  // elements per 16-byte vector
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    const int32_t vpr = Dh / N;          // vectors per row
    const int32_t upr = vpr / 2;         // units (vector pairs) per row
    const int32_t q_rows = q_out != nullptr ? H_q : 0;
    const int32_t units = (q_rows + 2 * H_kv) * upr;  // per token
    for (int32_t rem = threadIdx.x; rem < units; rem += blockDim.x) {
        const int32_t r = rem / upr, u = rem - r * upr;
        const bool is_q = r < q_rows;
        const bool is_v = !is_q && r >= q_rows + H_kv;
        const int32_t h = is_q ? r : r - q_rows - (is_v ? H_kv : 0);
        // the two vectors of this unit and the first pair index they hold
        const int32_t va = style == KV_ROPE_HALF ? u : 2 * u;
        const int32_t vb = style == KV_ROPE_HALF ? u + upr : 2 * u + 1;
        const int32_t k0 = u * N;  // pairs k0 .. k0 + N - 1
        const uint4* src0 = (is_q ? q : (is_v ? v_new : k_new)) + (int64_t)h * vpr;
        const int64_t src_stride = (int64_t)(is_q ? H_q : H_kv) * vpr;  // per token
        for (int64_t b = blockIdx.x; b < B; b += gridDim.x) {
            const int32_t pos = positions[b];
            if (pos < 0 || pos >= max_pos) {
                if (rem == 0 && err) atomicOr(err, KV_DEV_ERR_POSITION);
                continue;
            }
            uint4* dst;
            if (is_q) {
                dst = q_out + (b * H_q + h) * vpr;
            } else {
                const int64_t slot = slots[b];
                if (slot < 0) continue;
                if (slot >= num_slots) {
                    if (h == 0 && u == 0 && !is_v && err) atomicOr(err, KV_DEV_ERR_SLOT);
                    continue;
                }
                const int64_t page = slot / P, off = slot - page * P;
                dst = (is_v ? v_pages : k_pages) + ((page * H_kv + h) * P + off) * vpr;
            }
            const uint4* src = src0 + b * src_stride;
            const uint4 a = src[va], bv = src[vb];
            if (is_v) {
                dst[va] = a;
                dst[vb] = bv;
                continue;
            }
            float xa[N], xb[N];
            V::load(a, xa);
            V::load(bv, xb);
            const float* crow = cos_sin + (int64_t)pos * Dh;
            float c[N], s[N];
#pragma unroll
            for (int i = 0; i < N; i += 4) {
                const float4 cc = *reinterpret_cast<const float4*>(crow + k0 + i);
                const float4 ss = *reinterpret_cast<const float4*>(crow + Dh / 2 + k0 + i);
                c[i] = cc.x, c[i + 1] = cc.y, c[i + 2] = cc.z, c[i + 3] = cc.w;
                s[i] = ss.x, s[i + 1] = ss.y, s[i + 2] = ss.z, s[i + 3] = ss.w;
            }
            if (style == KV_ROPE_HALF) {
                // pair k0 + i = (element i of a, element i of b)
#pragma unroll
                for (int i = 0; i < N; ++i) rotate_pair(xa[i], xb[i], c[i], s[i]);
            } else {
                // a holds pairs k0 .. k0 + N/2 - 1, b the next N/2, as (2i, 2i + 1)
#pragma unroll
                for (int i = 0; i < N / 2; ++i) {
                    rotate_pair(xa[2 * i], xa[2 * i + 1], c[i], s[i]);
                    rotate_pair(xb[2 * i], xb[2 * i + 1], c[N / 2 + i], s[N / 2 + i]);
                }
            }
            dst[va] = V::store(xa);
            dst[vb] = V::store(xb);
        }
    }
}

int elem_size(int32_t dtype) {
    return dtype == KV_DTYPE_F32 ? 4 : (dtype == KV_DTYPE_BF16 || dtype == KV_DTYPE_F16) ? 2 : 0;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace kvp

using namespace kvp;

extern "C" int kv_rope_append(void* k_pages, void* v_pages, void* q_out, const void* q, const void* k_new,
                              const void* v_new, const int64_t* slot_mapping, const int32_t* positions,
                              const float* cos_sin, int32_t max_pos, int32_t rope_style, int32_t B, int32_t H_q,
                              int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, int32_t dtype,
                              int* err_flag, void* stream) {
    const int eb = elem_size(dtype);
    if (B < 0 || H_kv <= 0 || Dh <= 0 || page_size <= 0 || num_pages <= 0 || eb == 0 || max_pos <= 0) return KV_ERR_ARG;
    if (rope_style != KV_ROPE_HALF && rope_style != KV_ROPE_INTERLEAVED) return KV_ERR_ARG;
    if ((q == nullptr) != (q_out == nullptr) || (q != nullptr && H_q <= 0)) return KV_ERR_ARG;
    if ((static_cast<int64_t>(Dh) * eb) % 32 != 0) return KV_ERR_UNSUPPORTED;  // whole vector pairs per row
    if (B == 0) return KV_OK;
    if (!k_pages || !v_pages || !k_new || !v_new || !slot_mapping || !positions || !cos_sin) return KV_ERR_ARG;
    if (!al16(k_pages) || !al16(v_pages) || !al16(k_new) || !al16(v_new) || !al16(cos_sin)) return KV_ERR_ARG;
    if (q != nullptr && (!al16(q) || !al16(q_out))) return KV_ERR_ARG;
    const int32_t vpr = Dh * eb / 16;
    const int64_t rows = (q != nullptr ? H_q : 0) + 2LL * H_kv;
    const int64_t units = rows * (vpr / 2);  // per token: one thread each
    const int threads = static_cast<int>(std::min<int64_t>(384, (units + 31) / 32 * 32));
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(B, sms * std::max<int64_t>(1, 1152 / threads)));  // resident CTAs
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t num_slots = static_cast<int64_t>(num_pages) * page_size;
    cudaError_t e;
    auto args = [&](auto kernel) {
        return launch_pdl(kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, st, static_cast<uint4*>(k_pages),
                          static_cast<uint4*>(v_pages), static_cast<uint4*>(q_out), static_cast<const uint4*>(q),
                          static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping, positions,
                          cos_sin, max_pos, rope_style, static_cast<int64_t>(B), H_q, H_kv, Dh, page_size, num_slots,
                          err_flag);
    };
    if (dtype == KV_DTYPE_BF16)
        e = args(kv_rope_append_kernel<KV_DTYPE_BF16>);
    else if (dtype == KV_DTYPE_F16)
        e = args(kv_rope_append_kernel<KV_DTYPE_F16>);
    else
        e = args(kv_rope_append_kernel<KV_DTYPE_F32>);
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}
