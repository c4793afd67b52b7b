// Work plan for a planned decode launch: splits every (sequence, KV head)
// row into chunks of C pages; full chunks are listed from the front of the
// grid and the shorter tail chunks from the back, so the hardware block
// scheduler -- which starts CTAs in index order -- ends on small pieces
// (the CTAs in between find no work and exit). C is chosen from the actual
// lengths, which the host does not see: every row the same length -> one
// wave (chunks ~ `slots`); otherwise about four chunks per resident slot;
// never below `c_floor` (keeps each chunk's (m, l, u) partial small next to
// its K/V). One CTA of 1024 threads; each thread keeps its rows' page counts
// in registers, so the lengths are read once.
//
// Plan layout (int32, in the workspace):
//   [0] C (pages per chunk)   [1] total items   [2], [3] unused
//   [4 .. 4+B] S_b: exclusive prefix over b of ceil(n_pages_b / C) -- the
//   canonical item id t of (b, kvh, chunk) is H_kv * S_b + kvh * items_b +
//   chunk, and indexes the partials.
// Item list (int4 [grid]): {b, kvh, chunk, t} per CTA; b = -1: no work.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "kvpaged.h"
#include "plan_layout.cuh"
#include "ptx.cuh"

namespace kvp {

constexpr int kPlanThreads = 1024;
constexpr int kPlanRowsPerThread = 8;  // rows held in registers per thread (B <= 8192)

// Block-wide exclusive scan of one 64-bit value per thread; returns the block total.
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v, unsigned long long* warp_sums,
                                                                   unsigned long long& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        unsigned long long w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    total = warp_sums[(blockDim.x >> 5) - 1];
    const unsigned long long before = (warp > 0) ? warp_sums[warp - 1] : 0ull;
    __syncthreads();
    return before + x - v;
}

__global__ void __launch_bounds__(kPlanThreads) paged_plan_kernel(const int32_t* __restrict__ seq_lens, int32_t B,
                                                                  int32_t H_kv, int32_t P, int32_t max_blocks,
                                                                  int32_t slots, int32_t grid, int32_t c_floor,
                                                                  int32_t* __restrict__ plan, int4* __restrict__ items,
                                                                  int* err) {
    __shared__ unsigned long long warp_sums[32];
    __shared__ int s_min, s_max;
    __shared__ unsigned long long s_total;
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_min = 0x7fffffff;
        s_max = 0;
        s_total = 0;
    }
    // rows tid, tid + 1024, ...: page counts in registers
    int n[kPlanRowsPerThread];
    unsigned long long local = 0;
    int mn = 0x7fffffff, mx = 0;
#pragma unroll
    for (int r = 0; r < kPlanRowsPerThread; ++r) {
        const int b = tid + r * kPlanThreads;
        n[r] = 0;
        if (b < B) {
            int len = seq_lens[b];
            if (len < 0 || len > max_blocks * P) {
                if (err) atomicOr(err, KV_DEV_ERR_SEQ_LEN);
                len = 0;
            }
            n[r] = (len + P - 1) / P;
            local += n[r];
            mn = min(mn, n[r]);
            mx = max(mx, n[r]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        local += __shfl_xor_sync(0xffffffffu, local, o);
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    __syncthreads();
    if ((tid & 31) == 0) {
        atomicAdd(&s_total, local);
        atomicMin(&s_min, mn);
        atomicMax(&s_max, mx);
    }
    __syncthreads();
    const long long T = static_cast<long long>(s_total) * H_kv;  // (page, KV head) pairs of the launch
    const int target = (s_min == s_max) ? slots : 4 * slots;
    long long c = (T + target - 1) / target;
    if (c < c_floor) c = c_floor;
    const int C = static_cast<int>(c);
    // chunks per row (it) and whether the last one is short (tail), packed
    // into one scan: it in the high word, tail in the low word
    long long carry_it = 0, carry_tail = 0;
#pragma unroll
    for (int r = 0; r < kPlanRowsPerThread; ++r) {
        if (r * kPlanThreads >= B) break;
        const int b = tid + r * kPlanThreads;
        const int it = (n[r] + C - 1) / C;
        const int full = n[r] / C;
        const int tail = it - full;
        unsigned long long tot;
        const unsigned long long pre =
            block_exclusive_scan((static_cast<unsigned long long>(it) << 32) | static_cast<unsigned>(tail), warp_sums, tot);
        const long long pre_it = carry_it + static_cast<long long>(pre >> 32);
        const long long pre_tail = carry_tail + static_cast<long long>(pre & 0xffffffffull);
        const long long pre_full = pre_it - pre_tail;
        if (b < B) {
            plan[kPlanHdr + b] = static_cast<int32_t>(pre_it);
            for (int kvh = 0; kvh < H_kv; ++kvh) {
                const long long t0 = H_kv * pre_it + (long long)kvh * it;
                for (int cc = 0; cc < full; ++cc) {
                    const long long pos = pre_full * H_kv + (long long)kvh * full + cc;
                    if (pos < grid) items[pos] = make_int4(b, kvh, cc, static_cast<int>(t0 + cc));
                }
                if (tail) {
                    const long long pos = grid - 1 - (pre_tail * H_kv + kvh);
                    if (pos >= 0) items[pos] = make_int4(b, kvh, full, static_cast<int>(t0 + full));
                }
            }
        }
        carry_it += static_cast<long long>(tot >> 32);
        carry_tail += static_cast<long long>(tot & 0xffffffffull);
    }
    const long long total = carry_it * H_kv;
    const long long n_full = (carry_it - carry_tail) * H_kv, n_tail = carry_tail * H_kv;
    if (tid == 0) {
        plan[0] = C;
        plan[1] = static_cast<int32_t>(total);
        plan[2] = 0;
        plan[3] = 0;
        plan[kPlanHdr + B] = static_cast<int32_t>(carry_it);
        if (total > grid && err) atomicOr(err, KV_DEV_ERR_PIPELINE);  // the host sizes the grid so this cannot happen
    }
    for (long long pos = n_full + tid; pos < grid - n_tail; pos += kPlanThreads) items[pos] = make_int4(-1, 0, 0, 0);
}

// Balanced ("stream") plan for the persistent tcgen05 decode kernel. The
// (sequence, KV head) rows are laid end to end in (b, kvh) order, each
// preceded by v virtual pages that stand for the fixed cost of a work item
// (its Q tile, the first stage's maximum, the hand-over to the epilogue):
// with D_b = n_b + v for a sequence with pages (0 without), row (b, kvh)
// spans [H_kv S_b + kvh D_b, + D_b) of a line of T = H_kv sum_b D_b, its
// real pages the last n_b of the span. CTA c of G takes the line positions
// [floor(c T / G), floor((c + 1) T / G)): every CTA carries the same cost
// (+-1 page), whatever the length mix. A row cut by a CTA boundary is
// processed in pieces by consecutive CTAs; a piece leaves its (m, l, u)
// partial in one of two slots of its CTA -- slot 2c + 1 when the row starts
// inside the CTA's range (the CTA's last piece), slot 2c when it started
// before (the CTA's first piece) -- and the combine kernel merges them. Rows
// inside one CTA's range are written to the output directly.
// G = min(grid, ceil(T / min_pages)) keeps at least `min_pages` per CTA.
// Output rows of sequences without pages are zeroed here (no CTA visits them).
//
// Plan layout (int32 words): [0] kPlanStream, [1] G | v << 16, [2], [3] T
// (int64), [4 ..] S_b (int64, B + 1 entries: exclusive prefix of D_b), then
// cta_row[G]: the sequence whose rows' spans hold position floor(c T / G).

__global__ void __launch_bounds__(kPlanThreads) paged_plan_stream_kernel(const int32_t* __restrict__ seq_lens,
                                                                         int32_t B, int32_t H_kv, int32_t P,
                                                                         int32_t max_blocks, int32_t grid,
                                                                         int32_t min_pages, int32_t v,
                                                                         int32_t* __restrict__ plan,
                                                                         float* __restrict__ out, int32_t H_q,
                                                                         int32_t Dh, int* err) {
    __shared__ unsigned long long warp_sums[32];
    __shared__ int empties[kPlanThreads];
    __shared__ int n_empty;
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    const int tid = threadIdx.x;
    int64_t* pre = plan_stream_prefix(plan);
    int32_t* cta_row = plan + kPlanHdr + 2 * (B + 1);
    // rows tid, tid + 1024, ...: page counts, spans D_b = n_b + v (0 without pages) and their exclusive
    // prefix in registers
    int n[kPlanRowsPerThread];
    long long s[kPlanRowsPerThread];
    long long carry = 0;
#pragma unroll
    for (int r = 0; r < kPlanRowsPerThread; ++r) {
        const int b = tid + r * kPlanThreads;
        n[r] = 0;
        s[r] = 0;
        if (r * kPlanThreads >= B) continue;  // uniform over the block
        if (b < B) {
            int len = seq_lens[b];
            if (len < 0 || len > max_blocks * P) {
                if (err) atomicOr(err, KV_DEV_ERR_SEQ_LEN);
                len = 0;
            }
            n[r] = (len + P - 1) / P;
        }
        unsigned long long tot;
        const long long span = n[r] > 0 ? n[r] + v : 0;
        const unsigned long long ex = block_exclusive_scan(static_cast<unsigned long long>(span), warp_sums, tot);
        s[r] = carry + static_cast<long long>(ex);
        if (b < B) pre[b] = s[r];
        carry += static_cast<long long>(tot);
    }
    // sequences without pages (empty, or a length the table cannot hold): the decode kernel never visits
    // their rows, so their output rows are zeroed here, one round of 1024 sequences at a time
    const long long row_floats = static_cast<long long>(H_q) * Dh;
    for (int r = 0; r < kPlanRowsPerThread && r * kPlanThreads < B; ++r) {
        if (tid == 0) n_empty = 0;
        __syncthreads();
        const int b = tid + r * kPlanThreads;
        if (b < B && n[r] == 0) empties[atomicAdd(&n_empty, 1)] = b;
        __syncthreads();
        const long long ne = n_empty;
        for (long long i = tid; i < ne * row_floats; i += kPlanThreads)
            out[static_cast<long long>(empties[i / row_floats]) * row_floats + i % row_floats] = 0.f;
        __syncthreads();
    }
    const long long T = carry * H_kv;
    long long G = min_pages > 0 ? (T + min_pages - 1) / min_pages : T;
    if (G > grid) G = grid;
    if (tid == 0) {
        plan[0] = kPlanStream;
        plan[1] = static_cast<int32_t>(G | (static_cast<long long>(v) << 16));
        plan[2] = static_cast<int32_t>(T & 0xffffffffLL);
        plan[3] = static_cast<int32_t>(T >> 32);
        pre[B] = carry;
    }
    if (G <= 0) return;
    // CTA c starts in the rows of sequence b when floor(c T / G) lies in [H_kv S_b, H_kv S_{b+1}), i.e.
    // c in [ceil(H_kv S_b G / T), ceil(H_kv S_{b+1} G / T)); sequences without pages span nothing
#pragma unroll
    for (int r = 0; r < kPlanRowsPerThread; ++r) {
        const int b = tid + r * kPlanThreads;
        if (b >= B || n[r] == 0) continue;
        const long long a0 = s[r] * H_kv, a1 = (s[r] + n[r] + v) * H_kv;
        const long long c0 = (a0 * G + T - 1) / T, c1 = (a1 * G + T - 1) / T;
        for (long long c = c0; c < c1; ++c) cta_row[c] = b;
    }
}

}  // namespace kvp
