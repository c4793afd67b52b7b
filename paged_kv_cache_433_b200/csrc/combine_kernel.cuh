// Split-KV combine kernel (K4): merges the per-split (m, l, u) partials
// written by the decode kernels into the output rows.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "plan_layout.cuh"
#include "ptx.cuh"

namespace kvp {

// Merge split partials (the same (m, l, u) rule over the splits of one row):
// m* = max_s m_s, o = sum_s 2^{m_s - m*} u_s / sum_s 2^{m_s - m*} l_s.
// CTAs of kCombineWarps warps; WPR warps per (sequence, query head) row, so
// a CTA covers kCombineWarps / WPR rows (WPR = 1 for few splits, 8 for
// many). The kernel is latency-bound, so every load of a round is issued
// before any is used: each warp of a row holds up to kPer of its splits in
// registers while the lanes also fetch all m_s for m*; then weights, sums,
// and (WPR > 1) a shared-memory sum over the row's warps, all relative to the
// same m*.
constexpr int kCombineWarps = 8;

// Planned launches (plan != nullptr, WPR == 1 only): the row's chunk size and
// first item come from the plan; rows with one chunk were written by the
// decode kernel and are skipped, empty rows are zeroed here; partial s of
// (b, query head h) sits at item t0 + s, row h of that item's [g][Dh] block.
// Balanced plans (plan[0] == kPlanStream): the row's pages lie in the ranges
// of CTAs c0 .. c1; its first piece left its partial in slot 2 c0 + 1, piece
// s >= 1 in slot 2 (c0 + s).
template <int DH, int WPR>
__global__ void __launch_bounds__(32 * kCombineWarps) paged_combine_kernel(
    float* __restrict__ out, const float* __restrict__ part_u, const float2* __restrict__ part_ml,
    const int32_t* __restrict__ seq_lens, int32_t B, int32_t H_q, int32_t S, int32_t pages_per_split, int32_t P,
    int32_t max_blocks, const int32_t* __restrict__ plan, int32_t H_kv) {
    constexpr int kD = DH / 32;  // dims per lane
    constexpr int kPer = 8;      // splits per warp per round
    constexpr int kRound = WPR * kPer;
    constexpr int kRows = kCombineWarps / WPR;
    __shared__ float red_u[kCombineWarps][DH];
    __shared__ float red_l[kCombineWarps];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rw = warp % WPR;  // warp within its row
    const int64_t item = (int64_t)blockIdx.x * kRows + warp / WPR;
    grid_dependency_wait();  // the decode kernel's partials
    if (threadIdx.x == 0) grid_launch_dependents();
    bool live = item < (int64_t)B * H_q;
    int ns = 0;
    int64_t base = item * S, stride = 1, first = 0;  // partial s at base + (s == 0 ? first : s * stride)
    if (live) {
        const int b = static_cast<int>(item / H_q);
        int len = seq_lens[b];
        if (len < 0 || len > max_blocks * P) len = 0;
        const int n_pages = (len + P - 1) / P;
        if (plan != nullptr && plan[0] == kPlanStream) {
            const int G = plan[1];
            const long long T = static_cast<long long>(static_cast<uint32_t>(plan[2])) |
                                (static_cast<long long>(plan[3]) << 32);
            const int64_t* pre = plan_stream_prefix(plan);
            const int g = H_q / H_kv;
            const int hq = static_cast<int>(item % H_q);
            const long long s0 = pre[b], n = pre[b + 1] - s0;
            if (n > 0 && G > 0) {
                const long long r0 = (long long)H_kv * s0 + (long long)(hq / g) * n;
                const int c0 = plan_stream_cta(r0, T, G), c1 = plan_stream_cta(r0 + n - 1, T, G);
                if (c0 == c1) {
                    live = false;  // the decode kernel wrote this row
                } else {
                    ns = c1 - c0 + 1;
                    base = 2LL * g * c0 + hq % g;
                    stride = 2LL * g;
                    first = g;
                }
            }
        } else if (plan != nullptr) {
            const int C = plan[0];
            const int items_b = (n_pages + C - 1) / C;
            const int g = H_q / H_kv;
            const int hq = static_cast<int>(item % H_q);
            if (items_b == 1) live = false;  // the decode kernel wrote this row
            ns = items_b > 1 ? items_b : 0;
            const int64_t t0 = (int64_t)H_kv * plan[kPlanHdr + b] + (int64_t)(hq / g) * items_b;
            base = t0 * g + hq % g;
            stride = g;
        } else {
            ns = min(S, (n_pages + pages_per_split - 1) / pages_per_split);
        }
    }
    const float2* ml = part_ml + base;
    const float* pu = part_u + base * DH + lane * kD;

    float acc[kD];
#pragma unroll
    for (int i = 0; i < kD; ++i) acc[i] = 0.f;
    float L = 0.f;
    float mstar = -INFINITY;
    for (int r0 = 0; r0 < ns; r0 += kRound) {
        float2 st[kPer];
        float v[kPer][kD];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int s = r0 + rw + j * WPR;
            if (s < ns) {
                const int64_t off = s == 0 ? first : (int64_t)s * stride;
                st[j] = ml[off];
                const float* src = pu + off * DH;
                if constexpr (kD == 4) {
                    const float4 x = *reinterpret_cast<const float4*>(src);
                    v[j][0] = x.x; v[j][1] = x.y; v[j][2] = x.z; v[j][3] = x.w;
                } else {
#pragma unroll
                    for (int i = 0; i < kD; ++i) v[j][i] = src[i];
                }
            } else {
                st[j] = make_float2(-INFINITY, 0.f);
#pragma unroll
                for (int i = 0; i < kD; ++i) v[j][i] = 0.f;
            }
        }
        if (r0 == 0) {
            for (int s = lane; s < ns; s += 32) mstar = fmaxf(mstar, ml[s == 0 ? first : (int64_t)s * stride].x);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
        }
        if (mstar != -INFINITY) {
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                if (st[j].x == -INFINITY) continue;
                const float w = exp2f(st[j].x - mstar);
                L += w * st[j].y;
#pragma unroll
                for (int i = 0; i < kD; ++i) acc[i] += w * v[j][i];
            }
        }
    }
    if constexpr (WPR == 1) {
        if (live) {
            const float inv = (L > 0.f) ? 1.f / L : 0.f;
            float* dst = out + item * DH + lane * kD;
            if constexpr (kD == 4) {
                *reinterpret_cast<float4*>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
            } else {
#pragma unroll
                for (int i = 0; i < kD; ++i) dst[i] = acc[i] * inv;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < kD; ++i) red_u[warp][lane * kD + i] = acc[i];
        if (lane == 0) red_l[warp] = L;
        __syncthreads();
        const int row_w0 = (warp / WPR) * WPR;
        if (live && rw == 0) {
            for (int d = lane; d < DH; d += 32) {
                float U = 0.f, Lt = 0.f;
#pragma unroll
                for (int w = 0; w < WPR; ++w) {
                    U += red_u[row_w0 + w][d];
                    Lt += red_l[row_w0 + w];
                }
                out[item * DH + d] = (Lt > 0.f) ? U / Lt : 0.f;
            }
        }
    }
}

}  // namespace kvp
