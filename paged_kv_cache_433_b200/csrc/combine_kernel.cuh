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
// before any is used (in a grid split the first round goes out together with
// the row's length): each warp of a row holds up to kPer of its splits in
// registers and folds them in relative to its own maximum m_w; with WPR > 1
// the row's warps then meet in shared memory, each scaled by 2^{m_w - m*}.
constexpr int kCombineWarps = 8;

// Planned launches (plan != nullptr, WPR == 1 only): the row's chunk size and
// first item come from the plan; rows with one chunk were written by the
// decode kernel and are skipped, empty rows are zeroed here; partial s of
// (b, query head h) sits at item t0 + s, row h of that item's [g][Dh] block.
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
    __shared__ float red_l[kCombineWarps], red_m[kCombineWarps];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rw = warp % WPR;  // warp within its row
    const int64_t item = (int64_t)blockIdx.x * kRows + warp / WPR;
    bool live = item < (int64_t)B * H_q;
    // The lengths and a plan were written before the decode kernel this one follows could start (it waits for
    // its predecessors before it lets this one launch, and writes neither), so they are read before the wait
    // for the partials, from L2 (ld.global.cg), never from a line an earlier kernel left in this SM's L1.
    int len = 0;
    if (live) len = __ldcg(seq_lens + item / H_q);
    int ns = plan != nullptr ? 0 : S;  // splits loaded (grid split: the row's own count masks them after)
    int64_t base = item * S, stride = 1;
    if (live && plan != nullptr) {
        const int b = static_cast<int>(item / H_q);
        if (len < 0 || len > max_blocks * P) len = 0;
        const int n_pages = (len + P - 1) / P;
        const int C = __ldcg(plan);
        const int items_b = (n_pages + C - 1) / C;
        const int g = H_q / H_kv;
        const int hq = static_cast<int>(item % H_q);
        if (items_b == 1) live = false;  // the decode kernel wrote this row
        ns = items_b > 1 ? items_b : 0;
        const int64_t t0 = (int64_t)H_kv * __ldcg(plan + kPlanHdr + b) + (int64_t)(hq / g) * items_b;
        base = t0 * g + hq % g;
        stride = g;
    }
    grid_dependency_wait();  // the decode kernel's partials
    if (threadIdx.x == 0) grid_launch_dependents();
    if (!live) ns = 0;
    const float2* ml = part_ml + base;
    const float* pu = part_u + base * DH + lane * kD;

    // this warp's splits folded in with their own reference maximum m_w (moved per round as needed); the
    // warps of a row then meet relative to the largest m_w
    float acc[kD];
#pragma unroll
    for (int i = 0; i < kD; ++i) acc[i] = 0.f;
    float L = 0.f;
    float mw = -INFINITY;
    int nrow = ns;  // the row's splits
    for (int r0 = 0; r0 < ns; r0 += kRound) {
        float2 st[kPer];
        float v[kPer][kD];
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int s = r0 + rw + j * WPR;
            if (s < ns) {
                st[j] = ml[s * stride];
                const float* src = pu + (int64_t)s * stride * DH;
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
        if (plan == nullptr && r0 == 0) {
            if (len < 0 || len > max_blocks * P) len = 0;
            const int n_pages = (len + P - 1) / P;
            nrow = min(S, (n_pages + pages_per_split - 1) / pages_per_split);
        }
        float mr = -INFINITY;
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (r0 + rw + j * WPR >= nrow) st[j].x = -INFINITY;  // a split with no pages of this row
#pragma unroll
        for (int j = 0; j < kPer; ++j) mr = fmaxf(mr, st[j].x);
        if (mr > mw) {
            const float a = mw == -INFINITY ? 0.f : exp2f(mw - mr);
            L *= a;
#pragma unroll
            for (int i = 0; i < kD; ++i) acc[i] *= a;
            mw = mr;
        }
        if (mw != -INFINITY) {
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                if (st[j].x == -INFINITY) continue;
                const float w = exp2f(st[j].x - mw);
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
        if (lane == 0) red_l[warp] = L, red_m[warp] = mw;
        __syncthreads();
        const int row_w0 = (warp / WPR) * WPR;
        if (live && rw == 0) {
            float ms = -INFINITY;
#pragma unroll
            for (int w = 0; w < WPR; ++w) ms = fmaxf(ms, red_m[row_w0 + w]);
            float sc[WPR];
            float Lt = 0.f;
#pragma unroll
            for (int w = 0; w < WPR; ++w) {
                sc[w] = red_m[row_w0 + w] == -INFINITY ? 0.f : exp2f(red_m[row_w0 + w] - ms);
                Lt += sc[w] * red_l[row_w0 + w];
            }
            for (int d = lane; d < DH; d += 32) {
                float U = 0.f;
#pragma unroll
                for (int w = 0; w < WPR; ++w) U += sc[w] * red_u[row_w0 + w][d];
                out[item * DH + d] = (Lt > 0.f) ? U / Lt : 0.f;
            }
        }
    }
}

// Combine of a balanced plan (paged_plan_stream_kernel): only rows cut by a
// CTA boundary have partials, at most one per boundary, so CTA c of the grid
// merges the row whose real pages start in CTA c's range and run past its end
// (if any): its first piece is in slot 2c + 1, piece s >= 1 in slot 2 (c + s).
// One warp per head of the row's GQA group (g <= 32); lane s holds piece s's
// (m, l) and weight, then every lane sums DH / 32 dims over the pieces with
// all loads of a round issued before any is used. Rows inside one range were
// written by the decode kernel, rows without pages by the plan kernel.
constexpr int kCombineStreamWarps = 32;

template <int DH>
__global__ void __launch_bounds__(32 * kCombineStreamWarps) paged_combine_stream_kernel(
    float* __restrict__ out, const float* __restrict__ part_u, const float2* __restrict__ part_ml,
    const int32_t* __restrict__ plan, int32_t B, int32_t H_q, int32_t H_kv) {
    constexpr int kD = DH / 32;
    constexpr int kRound = 4;  // pieces whose dims are loaded together
    const int h = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = H_q / H_kv;
    const int c = blockIdx.x;
    // The row this CTA merges comes from the plan alone. The plan kernel completed before the decode kernel
    // this one follows let it launch (that kernel waits for the plan before it triggers), so the row is found
    // before the wait for the partials; the plan is read from L2 (ld.global.cg), never from a line an
    // earlier kernel left in this SM's L1.
    int ns = 0, b = 0, kvh = 0;
    if (h < g) {
        const int32_t w1 = __ldcg(plan + 1);
        const int G = w1 & 0xffff, v = static_cast<int>(static_cast<uint32_t>(w1) >> 16);
        const long long T = static_cast<long long>(static_cast<uint32_t>(__ldcg(plan + 2))) |
                            (static_cast<long long>(__ldcg(plan + 3)) << 32);
        if (c + 1 < G) {  // the last range ends the line
            const long long lo = T * c / G, hi = T * (c + 1) / G;
            // the row whose span holds position hi: its sequence starts CTA c + 1's range
            const int bb = __ldcg(plan + kPlanHdr + 2 * (B + 1) + c + 1);
            const long long* pre = reinterpret_cast<const long long*>(plan + kPlanHdr);
            const long long s0 = __ldcg(pre + bb), d = __ldcg(pre + bb + 1) - s0;
            if (d > 0) {
                const int kv = static_cast<int>((hi - (long long)H_kv * s0) / d);
                const long long r0 = (long long)H_kv * s0 + (long long)kv * d + v, n = d - v;  // its real pages
                // cut at this boundary when its real pages start inside this range (they then run past hi)
                if (r0 < hi && r0 >= lo) {
                    ns = plan_stream_cta(r0 + n - 1, T, G) - c + 1;
                    b = bb;
                    kvh = kv;
                }
            }
        }
    }
    grid_dependency_wait();  // the decode kernel's partials
    if (threadIdx.x == 0) grid_launch_dependents();
    if (ns <= 0) return;
    auto slot = [&](int s) { return (s == 0 ? 2LL * c + 1 : 2LL * (c + s)) * g + h; };
    // first round: piece `lane`'s (m, l) and the dims of the first kRound pieces go out together
    float2 st0 = make_float2(-INFINITY, 0.f);
    if (lane < ns) st0 = part_ml[slot(lane)];
    float v0[kRound][kD];
#pragma unroll
    for (int q = 0; q < kRound; ++q) {
        if (q < ns) {
            const float* src = part_u + slot(q) * DH + lane * kD;
#pragma unroll
            for (int i = 0; i < kD; ++i) v0[q][i] = src[i];
        } else {
#pragma unroll
            for (int i = 0; i < kD; ++i) v0[q][i] = 0.f;
        }
    }
    float mstar = st0.x;
    for (int s = lane + 32; s < ns; s += 32) mstar = fmaxf(mstar, part_ml[slot(s)].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, o));
    float acc[kD];
#pragma unroll
    for (int i = 0; i < kD; ++i) acc[i] = 0.f;
    float L = 0.f;
    // passes of 32 pieces (lane s: piece base + s's weight); a piece of weight 0 contributes 0, whatever its
    // dims hold
    for (int base = 0; base < ns && mstar != -INFINITY; base += 32) {
        const int s_l = base + lane;
        float2 st = st0;
        if (base > 0) st = s_l < ns ? part_ml[slot(s_l)] : make_float2(-INFINITY, 0.f);
        float w = 0.f;
        if (s_l < ns && st.x != -INFINITY) {
            w = exp2f(st.x - mstar);
            L += w * st.y;
        }
        const int cnt = min(32, ns - base);
        for (int s = 0; s < cnt; s += kRound) {
            float v[kRound][kD];
            float ws[kRound];
#pragma unroll
            for (int q = 0; q < kRound; ++q) {
                ws[q] = __shfl_sync(0xffffffffu, w, (s + q) & 31);
                if (base == 0 && s == 0) {
#pragma unroll
                    for (int i = 0; i < kD; ++i) v[q][i] = v0[q][i];
                } else if (s + q < cnt) {
                    const float* src = part_u + slot(base + s + q) * DH + lane * kD;
#pragma unroll
                    for (int i = 0; i < kD; ++i) v[q][i] = src[i];
                } else {
#pragma unroll
                    for (int i = 0; i < kD; ++i) v[q][i] = 0.f;
                }
            }
#pragma unroll
            for (int q = 0; q < kRound; ++q)
#pragma unroll
                for (int i = 0; i < kD; ++i) acc[i] += ws[q] != 0.f ? ws[q] * v[q][i] : 0.f;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    const float inv = L > 0.f ? 1.f / L : 0.f;
    float* dst = out + ((int64_t)b * H_q + (int64_t)kvh * g + h) * DH + lane * kD;
#pragma unroll
    for (int i = 0; i < kD; ++i) dst[i] = acc[i] * inv;
}

}  // namespace kvp
