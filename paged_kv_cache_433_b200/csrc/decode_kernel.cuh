// Paged decode attention kernels for sm_100a (CUDA cores, bulk-copy pipeline).
//
// What is computed, per sequence b and query head h (one new query each):
//   out[b][h] = softmax(scale * q[b][h] . K_t) V_t over t < seq_lens[b],
// with K_t / V_t of KV head h / g (g = H_q / H_kv) read through the block
// table ("04. 注意力与 KV 缓存" and "03. KV Cache：用显存换计算", attention
// formula sections; "07｜KV Cache、FlashAttention与PagedAttention的内部过程",
// Q028 block-table walk). Pages are folded in with the online (m, l, u) merge
// of the same handbook page, Q027: m_new = max(m_old, m_block),
// alpha = exp(m_old - m_new), l = alpha l + sum e^{s - m_new},
// u = alpha u + sum e^{s - m_new} v, o = u / l. Scores are kept in base-2
// units (q is pre-multiplied by scale * log2 e), so every exp is an exp2;
// the merge is unchanged.
//
// CTA = one (sequence, KV head[, split]) holding all g query heads of the GQA
// group, so each K/V byte is read from HBM once:
//   warp 0       producer: reads the block-table slice (32 entries per load)
//                and, per page, issues two 1-D bulk copies (the contiguous
//                P x Dh K chunk and V chunk of that (page, head)) into a ring
//                of NS shared-memory stages, completing on a full-barrier.
//   warps 1..NW  consumers. Consumer warp c serves head slice c % HS (GW heads)
//                for pages i with i % WP == c / HS. Lane = (token group tg =
//                lane / 8, column j = lane % 8): it owns tokens tg, tg+4, ...
//                of a page and 16-byte chunks j, j+8, ... of each row (Dh / 8
//                dims), so a quarter-warp reads 128 contiguous bytes of one row.
// Scores: per-lane partial dot products (packed f32x2 FMAs) are reduced over
// the 8 lanes of a row group by a halving exchange (each step ships half the
// values), which leaves every lane with whole scores of one head. The page
// maximum and alpha are warp-uniform per head; probabilities reach the lanes
// that own the V rows through a small per-warp shared buffer.
// Finalize: token groups are summed with shuffles, then the page-warps of a
// head slice are merged in shared memory with the same (m, l, u) rule. In a
// split launch the merged (m, l, u) of the CTA's page range is written to the
// workspace instead, and paged_combine_kernel merges the splits.
//
// Every wait is bounded (KV_DEV_ERR_TIMEOUT); a block-table entry outside
// [0, num_pages) is never dereferenced (KV_DEV_ERR_PAGE_RANGE, page skipped).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kvpaged.h"
#include "ptx.cuh"

namespace kvp {

constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s per wait
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
    float* out;                 // [B][H_q][Dh]
    const void* q;              // [B][H_q][Dh]
    const void* k_pages;        // [num_pages][H_kv][P][Dh]
    const void* v_pages;
    const int32_t* block_tables;  // [B][max_blocks]
    const int32_t* seq_lens;      // [B]
    const void* k_new;          // nullable: fused append of the token at position len - 1, [B][H_kv][Dh]
    const void* v_new;
    float* part_u;              // split: [B][H_q][S][Dh]; planned: [item][g][Dh]
    float2* part_ml;            // split: [B][H_q][S]; planned: [item][g] (m in log2 units, l)
    const int4* items;          // planned launch: {b, kvh, chunk, item} per CTA (nullable)
    const float* k_scale;       // E4M3 K/V: per-KV-head scales (read value = code * scale)
    const float* v_scale;
    const float* cos_sin;       // fused rotary embedding (nullable): fp32 [max_pos][Dh], cos then sin
    int32_t max_pos, rope_style;
    const int32_t* q_start;     // multi-token query: rows of sequence b are q_start[b] .. q_start[b+1]-1
    int32_t q_tile;             // multi-token query: chunk tokens per CTA
    const int32_t* plan;        // planned launch: [0] pages per chunk, [4 + b] item prefix
    int32_t stream_plan;        // 1: `plan` is the balanced plan of the persistent tcgen05 kernel
    int* err;
    int32_t max_blocks, B, H_q, H_kv, num_pages;
    int32_t g, HS, WP;          // GQA group, head slices, page-warps
    int32_t num_splits, pages_per_split;
    float scale_log2;           // scale * log2(e)
};

// ---- storage formats ------------------------------------------------------
template <int DT>
struct Fmt;
template <>
struct Fmt<KV_DTYPE_F32> {
    static constexpr int kElem = 4;
    // 16 bytes -> 2 float2
    static __device__ __forceinline__ void unpack(const uint4& c, float2 (&f)[2]) {
        f[0] = make_float2(__uint_as_float(c.x), __uint_as_float(c.y));
        f[1] = make_float2(__uint_as_float(c.z), __uint_as_float(c.w));
    }
};
template <>
struct Fmt<KV_DTYPE_BF16> {
    static constexpr int kElem = 2;
    static __device__ __forceinline__ float2 pair(uint32_t w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ void unpack(const uint4& c, float2 (&f)[4]) {
        f[0] = pair(c.x); f[1] = pair(c.y); f[2] = pair(c.z); f[3] = pair(c.w);
    }
};
template <>
struct Fmt<KV_DTYPE_F16> {
    static constexpr int kElem = 2;
    static __device__ __forceinline__ float2 pair(uint32_t w) {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        return __half22float2(h);
    }
    static __device__ __forceinline__ void unpack(const uint4& c, float2 (&f)[4]) {
        f[0] = pair(c.x); f[1] = pair(c.y); f[2] = pair(c.z); f[3] = pair(c.w);
    }
};

__device__ __forceinline__ void raise_err(int* err, int bit) {
    if (err) atomicOr(err, bit);
}

// Fused append ("07｜KV Cache、FlashAttention与PagedAttention的内部过程", Q025:
// the new token's K/V join the layer's cache before the query attends). The
// CTA whose page range ends at the sequence's last page writes the new
// token's K and V rows for its KV head into position len - 1 (slot
// table[(len-1)/P] * P + (len-1) % P), before its producer loads that page.
// Each lane fences its stores against the async proxy and the warp syncs, so
// the bulk / TMA reads issued afterwards see them. Called by one whole warp.
__device__ __forceinline__ void append_new_token(const DecodeParams& p, int b, int kvh, int len, int P,
                                                 int row_bytes, int lane) {
    const int pos = len - 1;
    const int32_t page = p.block_tables[(int64_t)b * p.max_blocks + pos / P];
    if (page >= 0 && page < p.num_pages) {
        const int nch = row_bytes / 16;
        const int64_t dst_row = ((int64_t)page * p.H_kv + kvh) * P + pos % P;
        const int64_t src_row = (int64_t)b * p.H_kv + kvh;
        for (int c = lane; c < 2 * nch; c += 32) {
            const bool is_v = c >= nch;
            const int cc = is_v ? c - nch : c;
            const uint4* src = static_cast<const uint4*>(is_v ? p.v_new : p.k_new) + src_row * nch + cc;
            uint4* dst = static_cast<uint4*>(const_cast<void*>(is_v ? p.v_pages : p.k_pages)) + dst_row * nch + cc;
            *dst = *src;
        }
        fence_proxy_async_global();
    } else if (lane == 0) {
        raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
    }
    __syncwarp();
}

template <int DT, int DH, int P, int GW, int NW>
struct DecodeCfg {
    static constexpr int kElem = Fmt<DT>::kElem;
    static constexpr int kVec = 16 / kElem;          // elements per 16-byte chunk
    static constexpr int kPairs = kVec / 2;          // float2 per chunk
    static constexpr int kRowB = DH * kElem;         // bytes per token row
    static constexpr int kNch = kRowB / 16;          // chunks per row
    static constexpr int kCpl = kNch / 8;            // chunks per lane
    static constexpr int kDpl = kCpl * kVec;         // dims per lane (= DH / 8)
    static constexpr int kR = P / 4;                 // tokens per lane per page
    static constexpr int kN = GW * kR;               // score values per lane before reduction
    static constexpr int kLogN = (kN >= 32) ? 5 : (kN >= 16) ? 4 : (kN >= 8) ? 3 : (kN >= 4) ? 2 : (kN >= 2) ? 1 : 0;
    static constexpr int kNH = (kN >= 8) ? kN / 8 : 1;  // scores held per lane after reduction
    static constexpr int kLH = (kN >= 8) ? 8 / GW : 8;   // lanes (per row group) holding one head
    static constexpr int kDup = (kN >= 8) ? 1 : 8 / kN;  // copies of each held score in a group
    static constexpr int kChunk = P * kRowB;         // bytes of one (page, head) chunk
    static constexpr int kStage = 2 * kChunk;        // K + V
    static constexpr int kStageBudget = (NW <= 4) ? 96 * 1024 : 160 * 1024;
    // Stage i % NS of page i is consumed by page-warp i % WP. NS must be a
    // multiple of WP (<= 4 when NW == 4, 1 when NW == 8): then every stage is
    // always drained by the same warp, which waits on each of its phases in
    // order, so a parity wait can never match a phase two fills old.
    static constexpr int kWPMax = (NW <= 4) ? 4 : 1;
    static constexpr int kNS0 = (kStageBudget / kStage) / kWPMax * kWPMax;
    static constexpr int kNS = kNS0 > 16 ? 16 : (kNS0 < kWPMax ? kWPMax : (kNS0 < 2 ? 2 : kNS0));
    static constexpr int kThreads = 32 * (NW + 1);
    // shared memory layout (bytes)
    static constexpr int kOffBars = kNS * kStage;                      // full[NS], empty[NS] (8 B each)
    static constexpr int kOffValid = kOffBars + 16 * kNS;              // int[NS]: page index held, -1 = skipped
    static constexpr int kOffPbuf = kOffValid + 4 * kNS;               // NW x (4 x kN + GW) floats
    static constexpr int kPbufFloats = 4 * kN + GW;
    static constexpr int kOffMerge = ((kOffPbuf + 4 * NW * kPbufFloats) + 15) / 16 * 16;  // NW x GW x (DH + 2)
    static constexpr int kSmem = kOffMerge + 4 * NW * GW * (DH + 2);
    static_assert(kNch % 8 == 0, "row must be a multiple of 128 bytes");
    static_assert(kNS % kWPMax == 0, "stage ring must be a multiple of the page-warps");
    static_assert(P % 4 == 0, "page size must be a multiple of 4");
};

// Halving exchange over the 8 lanes of a row group (xor 4, 2, 1): afterwards
// v[0 .. NH) hold complete sums for indices [base, base + NH), where
// base = j * NH for N >= 8 (j = lane % 8); for N < 8 every index is held by
// 8 / N lanes (base = j >> (3 - log2 N)).
template <int N>
__device__ __forceinline__ void group_reduce(float (&v)[N], int lane) {
    constexpr int n1 = N >= 2 ? N / 2 : 1;
    constexpr int n2 = n1 >= 2 ? n1 / 2 : 1;
#pragma unroll
    for (int step = 0; step < 3; ++step) {
        const int o = 4 >> step;
        const int n = step == 0 ? N : (step == 1 ? n1 : n2);
        const bool upper = (lane & o) != 0;
        if (n >= 2) {
            const int half = n / 2;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                if (i < half) {
                    float a = v[i], b = v[i + half];
                    float send = upper ? a : b;
                    float keep = upper ? b : a;
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
        }
    }
}

template <int DT, int DH, int P, int GW, int NW>
// Two CTAs of NW = 4 consumers per SM: 10 warps spread over 4 sub-partitions
// put 3 warps on some, so registers are capped at 16384 / (3 * 32) = 168.
__global__ void __launch_bounds__(32 * (NW + 1), (NW <= 4) ? 2 : 1) paged_decode_kernel(const DecodeParams p) {
    using C = DecodeCfg<DT, DH, P, GW, NW>;
    extern __shared__ __align__(128) unsigned char smem[];

    const int split = blockIdx.x;
    const int kvh = blockIdx.y;
    const int b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool split_mode = p.num_splits > 1;

    grid_dependency_wait();  // inputs may come from the previous kernel in the stream
    if (threadIdx.x == 0) grid_launch_dependents();
    int len = p.seq_lens[b];
    if (len < 0 || len > p.max_blocks * P) {
        if (threadIdx.x == 0 && split == 0) raise_err(p.err, KV_DEV_ERR_SEQ_LEN);
        len = 0;
    }
    const int n_pages = (len + P - 1) / P;
    const int first = split_mode ? split * p.pages_per_split : 0;
    int n_local = split_mode ? min(p.pages_per_split, n_pages - first) : n_pages;
    if (n_local <= 0) {
        if (!split_mode) {  // empty sequence: zero output rows of this group
            for (int e = threadIdx.x; e < p.g * DH; e += blockDim.x)
                p.out[((int64_t)b * p.H_q + (int64_t)kvh * p.g) * DH + e] = 0.f;
        }
        return;  // split ranges past the end are skipped by the combine kernel
    }

    const uint32_t sbase = smem_u32(smem);
    const uint32_t full_bar = sbase + C::kOffBars;
    const uint32_t empty_bar = full_bar + 8 * C::kNS;
    volatile int* stage_valid = reinterpret_cast<volatile int*>(smem + C::kOffValid);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kNS; ++s) {
            mbar_init(full_bar + 8 * s, 1);
            mbar_init(empty_bar + 8 * s, p.HS);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (p.k_new != nullptr && first + n_local == n_pages) append_new_token(p, b, kvh, len, P, C::kRowB, lane);
        const int32_t* row = p.block_tables + (int64_t)b * p.max_blocks + first;
        const char* kbase = static_cast<const char*>(p.k_pages);
        const char* vbase = static_cast<const char*>(p.v_pages);
        bool ok = true;
        int issued = 0;
        for (int base = 0; base < n_local && ok; base += 32) {
            int my = (base + lane < n_local) ? row[base + lane] : 0;
            const int cnt = min(32, n_local - base);
            for (int k = 0; k < cnt; ++k) {
                const int pg = __shfl_sync(0xffffffffu, my, k);
                const int i = base + k;
                if (lane == 0) {
                    const int s = i % C::kNS;
                    if (i >= C::kNS && !mbar_wait_bounded(empty_bar + 8 * s, ((i / C::kNS) - 1) & 1, kWaitLimitNs)) {
                        raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                        ok = false;
                    } else {
                        const uint32_t dst = sbase + s * C::kStage;
                        if (pg >= 0 && pg < p.num_pages) {
                            stage_valid[s] = i;
                            const int64_t off = ((int64_t)pg * p.H_kv + kvh) * (int64_t)C::kChunk;
                            mbar_arrive_expect_tx(full_bar + 8 * s, C::kStage);
                            bulk_g2s(dst, kbase + off, C::kChunk, full_bar + 8 * s);
                            bulk_g2s(dst + C::kChunk, vbase + off, C::kChunk, full_bar + 8 * s);
                        } else {
                            raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
                            stage_valid[s] = -1 - i;
                            mbar_arrive(full_bar + 8 * s);
                        }
                        ++issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        // Never leave with a copy in flight: wait for the last round of stages.
        if (lane == 0) {
            for (int i = max(0, issued - C::kNS); i < issued; ++i)
                if (!mbar_wait_bounded(full_bar + 8 * (i % C::kNS), (i / C::kNS) & 1, kWaitLimitNs))
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int cw = warp - 1;
    const int hs = cw % p.HS;
    const int wp = cw / p.HS;
    const bool active = wp < p.WP;
    const int tg = lane >> 3;
    const int j = lane & 7;
    const int h0 = kvh * p.g + hs * GW;  // first query head of this warp's slice

    // Held-score bookkeeping after group_reduce.
    constexpr int kLogN = C::kLogN;
    const int base = (C::kN >= 8) ? j * C::kNH : (j >> (3 - kLogN));
    const int hl = base / C::kR;  // head (within the slice) of the held scores
    const int r0 = base % C::kR;

    // q in registers: my dims of GW heads, pre-scaled to log2 units.
    float2 q2[GW][C::kCpl][C::kPairs];
    {
        const char* qb = static_cast<const char*>(p.q);
#pragma unroll
        for (int h = 0; h < GW; ++h) {
#pragma unroll
            for (int k = 0; k < C::kCpl; ++k) {
                const int64_t off = ((int64_t)b * p.H_q + h0 + h) * C::kRowB + (j + 8 * k) * 16;
                uint4 raw = *reinterpret_cast<const uint4*>(qb + off);
                float2 f[C::kPairs];
                Fmt<DT>::unpack(raw, f);
#pragma unroll
                for (int e = 0; e < C::kPairs; ++e)
                    q2[h][k][e] = make_float2(f[e].x * p.scale_log2, f[e].y * p.scale_log2);
            }
        }
    }

    float2 u2[GW][C::kCpl][C::kPairs];
#pragma unroll
    for (int h = 0; h < GW; ++h)
#pragma unroll
        for (int k = 0; k < C::kCpl; ++k)
#pragma unroll
            for (int e = 0; e < C::kPairs; ++e) u2[h][k][e] = make_float2(0.f, 0.f);
    float m_run = -INFINITY;  // running max (log2 units) of head hl; warp-uniform per head
    float l_run = 0.f;        // lane-partial sum of exp2 for head hl

    float* pbuf = reinterpret_cast<float*>(smem + C::kOffPbuf) + cw * C::kPbufFloats;
    bool ok = true;

    if (active) {
        for (int i = wp; i < n_local; i += p.WP) {
            const int s = i % C::kNS;
            if (!mbar_wait_bounded(full_bar + 8 * s, (i / C::kNS) & 1, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                ok = false;
            }
            if (!__all_sync(0xffffffffu, ok)) break;
            // The stage must hold page i (a page the producer skipped is tagged -1 - i).
            const int tag = stage_valid[s];
            if (tag != i && tag != -1 - i) {
                if (lane == 0) raise_err(p.err, KV_DEV_ERR_PIPELINE);
                break;
            }
            const bool valid = tag == i;
            const int pos0 = (first + i) * P;
            const int nvalid = valid ? min(P, len - pos0) : 0;
            const uint32_t sK = sbase + s * C::kStage;
            const uint32_t sV = sK + C::kChunk;

            // ---- scores: partial dots over my dims, then group reduction
            float sc[C::kN];
#pragma unroll
            for (int r = 0; r < C::kR; ++r) {
                const int t = tg + 4 * r;
                float2 acc[GW];
#pragma unroll
                for (int h = 0; h < GW; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < C::kCpl; ++k) {
                    float2 kf[C::kPairs];
                    Fmt<DT>::unpack(lds128(sK + t * C::kRowB + (j + 8 * k) * 16), kf);
#pragma unroll
                    for (int h = 0; h < GW; ++h)
#pragma unroll
                        for (int e = 0; e < C::kPairs; ++e) acc[h] = ffma2(q2[h][k][e], kf[e], acc[h]);
                }
#pragma unroll
                for (int h = 0; h < GW; ++h) sc[h * C::kR + r] = acc[h].x + acc[h].y;
            }
            group_reduce<C::kN>(sc, lane);

            // ---- mask, page max per head (lanes of one head: xor < LH, groups xor 8, 16)
            float mx = -INFINITY;
#pragma unroll
            for (int v = 0; v < C::kNH; ++v) {
                const int t = tg + 4 * (r0 + v);
                if (t >= nvalid) sc[v] = -INFINITY;
                mx = fmaxf(mx, sc[v]);
            }
#pragma unroll
            for (int o = 1; o < C::kLH; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run, mx);
            const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
            m_run = m_new;
            float psum = 0.f;
            __syncwarp();  // previous page's readers are done with pbuf
#pragma unroll
            for (int v = 0; v < C::kNH; ++v) {
                const float pv = (sc[v] == -INFINITY) ? 0.f : exp2f(sc[v] - m_new);
                psum += pv;
                pbuf[tg * C::kN + base + v] = pv;
            }
            l_run = l_run * alpha + psum;
            if (tg == 0 && (j % C::kLH) == 0) pbuf[4 * C::kN + hl] = alpha;
            __syncwarp();

            // ---- rescale accumulators when a head's maximum moved
            float a[GW];
#pragma unroll
            for (int h = 0; h < GW; ++h) a[h] = pbuf[4 * C::kN + h];
#pragma unroll
            for (int h = 0; h < GW; ++h) {
                if (a[h] != 1.f) {
                    const float2 a2 = make_float2(a[h], a[h]);
#pragma unroll
                    for (int k = 0; k < C::kCpl; ++k)
#pragma unroll
                        for (int e = 0; e < C::kPairs; ++e) u2[h][k][e] = fmul2(u2[h][k][e], a2);
                }
            }

            // ---- u += p * V over my tokens
#pragma unroll
            for (int r = 0; r < C::kR; ++r) {
                const int t = tg + 4 * r;
                if (t < nvalid) {
                    float2 pr[GW];
#pragma unroll
                    for (int h = 0; h < GW; ++h) {
                        const float pv = pbuf[tg * C::kN + h * C::kR + r];
                        pr[h] = make_float2(pv, pv);
                    }
#pragma unroll
                    for (int k = 0; k < C::kCpl; ++k) {
                        float2 vf[C::kPairs];
                        Fmt<DT>::unpack(lds128(sV + t * C::kRowB + (j + 8 * k) * 16), vf);
#pragma unroll
                        for (int h = 0; h < GW; ++h)
#pragma unroll
                            for (int e = 0; e < C::kPairs; ++e) u2[h][k][e] = ffma2(pr[h], vf[e], u2[h][k][e]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar + 8 * s);
        }
    }

    // ---- finalize: sum token groups (same max within the warp)
#pragma unroll
    for (int h = 0; h < GW; ++h)
#pragma unroll
        for (int k = 0; k < C::kCpl; ++k)
#pragma unroll
            for (int e = 0; e < C::kPairs; ++e) {
                float2 v = u2[h][k][e];
                v.x += __shfl_xor_sync(0xffffffffu, v.x, 8);
                v.y += __shfl_xor_sync(0xffffffffu, v.y, 8);
                v.x += __shfl_xor_sync(0xffffffffu, v.x, 16);
                v.y += __shfl_xor_sync(0xffffffffu, v.y, 16);
                u2[h][k][e] = v;
            }
    float lsum = l_run;
#pragma unroll
    for (int o = 1; o < C::kLH; o <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
    lsum *= 1.f / C::kDup;

    float* merge = reinterpret_cast<float*>(smem + C::kOffMerge);  // [NW][GW][DH + 2]
    if (active && tg == 0) {
#pragma unroll
        for (int h = 0; h < GW; ++h) {
            float* dst = merge + (cw * GW + h) * (DH + 2);
#pragma unroll
            for (int k = 0; k < C::kCpl; ++k)
#pragma unroll
                for (int e = 0; e < C::kPairs; ++e) {
                    const int d = (j + 8 * k) * C::kVec + 2 * e;
                    dst[d] = u2[h][k][e].x;
                    dst[d + 1] = u2[h][k][e].y;
                }
        }
        if ((j % C::kLH) == 0) {
            float* dst = merge + (cw * GW + hl) * (DH + 2);
            dst[DH] = m_run;
            dst[DH + 1] = lsum;
        }
    }
    named_bar_sync(1, 32 * NW);

    // ---- merge page-warps of each head slice; write output or split partials
    const int tid = threadIdx.x - 32;
    for (int e = tid; e < p.g * DH; e += 32 * NW) {
        const int hh = e / DH;  // head within the GQA group
        const int d = e % DH;
        const int slice = hh / GW, hw = hh % GW;
        float mstar = -INFINITY;
        for (int w = 0; w < p.WP; ++w) mstar = fmaxf(mstar, merge[((w * p.HS + slice) * GW + hw) * (DH + 2) + DH]);
        float L = 0.f, U = 0.f;
        if (mstar != -INFINITY) {
            for (int w = 0; w < p.WP; ++w) {
                const float* src = merge + ((w * p.HS + slice) * GW + hw) * (DH + 2);
                const float mw = src[DH];
                if (mw == -INFINITY) continue;
                const float sw = exp2f(mw - mstar);
                L += sw * src[DH + 1];
                U += sw * src[d];
            }
        }
        const int64_t hq = (int64_t)b * p.H_q + (int64_t)kvh * p.g + hh;
        if (!split_mode) {
            p.out[hq * DH + d] = (L > 0.f) ? U / L : 0.f;
        } else {
            const int64_t ps = hq * p.num_splits + split;
            p.part_u[ps * DH + d] = U;
            if (d == 0) p.part_ml[ps] = make_float2(mstar, L);
        }
    }
}

}  // namespace kvp
