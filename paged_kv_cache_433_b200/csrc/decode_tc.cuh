// Paged decode attention for large GQA groups (MQA: g = 32 query heads per
// KV head) on the fifth-generation tensor cores (tcgen05), sm_100a.
//
// Same contract and the same online (m, l, u) merge as decode_kernel.cuh
// ("07｜KV Cache、FlashAttention与PagedAttention的内部过程", Q027: blocks are
// folded in with m_new = max, alpha = exp(m_old - m_new), l and u rescaled;
// the attention formula of "04. 注意力与 KV 缓存"); the block table is walked
// as in Q028 of the same handbook page.
//
// With one query token and g = 32 heads the natural MMA row count (heads) is
// far below the 128 rows of a tcgen05 MMA, so the products are taken
// transposed, with the 128 tokens of a stage as the rows:
//   S^T[128 tokens x g] = K_stage[128 x Dh] . Q^T[Dh x g]     (K-major A and B)
//   O^T[Dh x g]        += V_stage^T[Dh x 128] . P^T[128 x g]  (MN-major A and B)
// S^T and O^T live in tensor memory (fp32); thread t of the four softmax
// warps owns token row t of S^T (all g scores of one token) and dimension
// row t of O^T. P^T goes to shared memory as a bf16 (fp16) pair hi + lo:
// hi = RN(p), lo = RN(p - hi); the second P.V MMA on lo carries p to ~2^-16
// relative, so short rows keep the accuracy of the fp32 softmax.
//
// Reference maximum (log2 units, per head, shared by the whole CTA): it moves
// only when some score of a stage exceeds it by more than 2^8; then the stage
// maximum is reduced over the CTA, and O^T and the partial row sums are
// rescaled (o = u / l holds for any common reference).
//
// Warp roles (192 threads, one CTA per SM, persistent over work items):
//   warp 0     producer: Q tile (2-D TMA, 128-byte swizzle) and, per stage,
//              the K then the V boxes of its pages (P rows x 128 bytes each)
//              into a ring of six 32 KB entries (K and V of three stages);
//              fused append of the new token when the item owns the last page.
//   warp 1     allocates tensor memory; lane 0 issues QK(j) then PV(j - 1),
//              committing each onto the mbarriers the other roles wait on.
//   warps 2-5  softmax and epilogue (tensor-memory lane quarter = warp % 4).
// A work item is (sequence, KV head, chunk of pages): from the device plan
// (planned launch) or from the grid rule (split); partials use the layout of
// decode_mma.cuh, so paged_combine_kernel merges them.
//
// Every wait is bounded (KV_DEV_ERR_TIMEOUT, then the CTA winds down); a
// block-table entry outside [0, num_pages) is never loaded (its tokens are
// masked, KV_DEV_ERR_PAGE_RANGE).
#pragma once

#include <cuda.h>

#include "decode_kernel.cuh"
#include "tc05.cuh"

namespace kvp {

template <int DH, int P, int G>
struct TcCfg {
    static constexpr int kTP = 128;              // tokens per stage = MMA rows
    static constexpr int kPPS = kTP / P;         // pages per stage
    static constexpr int kBoxCols = DH / 64;     // 128-byte box columns per token row
    static constexpr int kBoxB = kTP * 128;      // one box column of an entry
    static constexpr int kEntry = kBoxCols * kBoxB;  // K (or V) of one stage
    static constexpr int kRing = 6;              // entries: K, V of three stages
    static constexpr int kQB = kBoxCols * G * 128;
    static constexpr int kPB = kTP * G * 2;      // one P^T tile (hi or lo)
    static constexpr int kOffQ = kRing * kEntry;
    static constexpr int kOffP = kOffQ + kQB;
    static constexpr int kOffRed = kOffP + 2 * kPB;          // 2 x [G][4] floats
    static constexpr int kOffFlag = kOffRed + 2 * G * 4 * 4;  // 2 x 4 ints
    static constexpr int kOffBad = kOffFlag + 32;             // int per ring entry
    static constexpr int kOffBar = (kOffBad + 4 * kRing + 7) / 8 * 8;
    // full[6], empty[6], q_full, q_empty, s_full[2], s_empty[2], p_full, p_empty, o_full, o_empty, done
    static constexpr int kNumBars = 2 * kRing + 2 + 4 + 4 + 1;
    static constexpr int kOffTmem = kOffBar + 8 * kNumBars;
    static constexpr int kSmem = 1024 + kOffTmem + 16;
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 128;   // S^T x 2 (2g) + O^T (g)
    static_assert(G == 32 && DH == 128, "instance: g = 32, Dh = 128");
    static_assert(kPPS * kBoxCols <= 32, "one TMA box per lane");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct TcWork {
    int b, kvh, split, item, first, n_local, len, n_pages;
    bool split_mode, bad_len;
};

// Work item w: planned (items list) or grid (split, KV head, sequence).
__device__ __forceinline__ bool tc_work(const DecodeParams& p, int w, int P, TcWork& k) {
    int chunk_pages;
    if (p.items != nullptr) {
        const int4 it = p.items[w];
        if (it.x < 0) return false;
        k.b = it.x;
        k.kvh = it.y;
        k.split = it.z;
        k.item = it.w;
        chunk_pages = p.plan[0];
    } else {
        k.split = w % p.num_splits;
        const int rest = w / p.num_splits;
        k.kvh = rest % p.H_kv;
        k.b = rest / p.H_kv;
        k.item = 0;
        chunk_pages = p.pages_per_split;
    }
    const bool chunked = p.items != nullptr || p.num_splits > 1;
    k.first = chunked ? k.split * chunk_pages : 0;
    int len = p.seq_lens[k.b];
    k.bad_len = len < 0 || len > p.max_blocks * P;
    if (k.bad_len) len = 0;
    k.len = len;
    k.n_pages = (len + P - 1) / P;
    k.n_local = chunked ? min(chunk_pages, k.n_pages - k.first) : k.n_pages;
    k.split_mode = p.items != nullptr ? k.n_pages > chunk_pages : p.num_splits > 1;
    return true;
}

// Per-head reduction over the 32 lanes of a warp: afterwards lane l holds the
// reduction of x[l] (halving exchange: each step ships half of the values).
template <bool MAX>
__device__ __forceinline__ float warp_heads_reduce(float (&x)[32], int lane) {
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int off = 16 >> k;
        const int half = 16 >> k;
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? x[i] : x[i + half];
            const float keep = up ? x[i + half] : x[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            x[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    return x[0];
}

// The same reduction over the four softmax warps (128 threads, named barrier
// 1); every thread receives all 32 results. `buf` alternates between calls.
template <bool MAX>
__device__ __forceinline__ void cta_heads_reduce(float (&x)[32], float* red, int sw, int lane, int& buf) {
    const float v = warp_heads_reduce<MAX>(x, lane);
    float* r = red + buf * 32 * 4;
    r[lane * 4 + sw] = v;
    named_bar_sync(1, 128);
    const float4* r4 = reinterpret_cast<const float4*>(r);
#pragma unroll
    for (int h = 0; h < 32; ++h) {
        const float4 a = r4[h];
        x[h] = MAX ? fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)) : (a.x + a.y) + (a.z + a.w);
    }
    buf ^= 1;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int KT, int DH, int P, int G>
__global__ void __launch_bounds__(192, 1)
    paged_decode_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_q,
                           int n_work) {
    using C = TcCfg<DH, P, G>;
    constexpr bool kBF16 = KT == KV_DTYPE_BF16;
    constexpr uint32_t kIdescQK = idesc_f16(kBF16, 128, G, false, false);
    constexpr uint32_t kIdescPV = idesc_f16(kBF16, 128, G, true, true);
    extern __shared__ __align__(1024) unsigned char smem_raw[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_q);
    }
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + C::kOffBar;
    auto full = [&](int e) { return bar0 + 8u * e; };
    auto empty = [&](int e) { return bar0 + 8u * (C::kRing + e); };
    const uint32_t q_full = bar0 + 8u * (2 * C::kRing);
    const uint32_t q_empty = q_full + 8;
    auto s_full = [&](int i) { return q_full + 16u + 8u * i; };
    auto s_empty = [&](int i) { return q_full + 32u + 8u * i; };
    const uint32_t p_full = q_full + 48;
    const uint32_t p_empty = q_full + 56;
    const uint32_t o_full = q_full + 64;
    const uint32_t o_empty = q_full + 72;
    const uint32_t done_bar = q_full + 80;
    volatile int* stage_bad = reinterpret_cast<volatile int*>(smem + C::kOffBad);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmem);

    if (threadIdx.x == 0) {
        for (int e = 0; e < C::kRing; ++e) {
            mbar_init(full(e), 1);
            mbar_init(empty(e), 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 1);
            mbar_init(s_empty(i), 4);
        }
        mbar_init(p_full, 4);
        mbar_init(p_empty, 1);
        mbar_init(o_full, 1);
        mbar_init(o_empty, 4);
        mbar_init(done_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem;           // S^T buffers: columns [0, 2g)
    const uint32_t tO = tmem + 2 * G;   // O^T: columns [2g, 3g)
    const uint32_t ring = sbase;
    const uint32_t sQ = sbase + C::kOffQ;
    const uint32_t sPhi = sbase + C::kOffP;
    const uint32_t sPlo = sPhi + C::kPB;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        uint32_t fill = 0;
        int item_i = 0;
        for (int w = blockIdx.x; w < n_work && ok; w += gridDim.x) {
            TcWork wk;
            if (!tc_work(p, w, P, wk) || wk.n_local <= 0) continue;
            if (p.k_new != nullptr && wk.first + wk.n_local == wk.n_pages)
                append_new_token(p, wk.b, wk.kvh, wk.len, P, DH * 2, lane);
            if (lane == 0) {
                if (item_i > 0 && !mbar_wait_bounded(q_empty, (item_i - 1) & 1, kWaitLimitNs)) {
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                    ok = false;
                } else {
                    mbar_arrive_expect_tx(q_full, C::kQB);
#pragma unroll
                    for (int bb = 0; bb < C::kBoxCols; ++bb)
                        tma_load_2d(sQ + bb * G * 128, &tmap_q, bb * 64, wk.b * p.H_q + wk.kvh * G, q_full);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++item_i;
            const int32_t* row = p.block_tables + (int64_t)wk.b * p.max_blocks + wk.first;
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            for (int j = 0; j < n_st && ok; ++j) {
                const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                const int pg = lane < np ? row[j * C::kPPS + lane] : -1;
                const bool good = lane < np && pg >= 0 && pg < p.num_pages;
                if (lane < np && !good) raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
                const unsigned gmask = __ballot_sync(0xffffffffu, good);
                const int box_page = lane / C::kBoxCols, bb = lane % C::kBoxCols;
                const int pgl = __shfl_sync(0xffffffffu, pg, box_page & 31);
#pragma unroll 1
                for (int half = 0; half < 2 && ok; ++half) {
                    const int e = fill % C::kRing;
                    if (lane == 0) {
                        if (fill >= (uint32_t)C::kRing &&
                            !mbar_wait_bounded(empty(e), ((fill / C::kRing) - 1) & 1, kWaitLimitNs)) {
                            raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                            ok = false;
                        } else {
                            stage_bad[e] = (int)(~gmask & ((1u << np) - 1u));
                            mbar_arrive_expect_tx(full(e), __popc(gmask) * C::kBoxCols * P * 128);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    if (box_page < np && ((gmask >> box_page) & 1u)) {
                        const uint32_t dst = ring + e * C::kEntry + bb * C::kBoxB + box_page * P * 128;
                        tma_load_2d(dst, half ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k),
                                    bb * 64, (pgl * p.H_kv + wk.kvh) * P, full(e));
                    }
                    ++fill;
                }
            }
        }
        if (lane == 0) {  // let every copy in flight land before the CTA exits
            for (uint32_t i = fill > (uint32_t)C::kRing ? fill - C::kRing : 0; i < fill; ++i)
                if (!mbar_wait_bounded(full(i % C::kRing), (i / C::kRing) & 1, kWaitLimitNs))
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
            if (item_i > 0 && !mbar_wait_bounded(q_full, (item_i - 1) & 1, kWaitLimitNs))
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            bool ok = true;
            uint32_t fbase = 0;  // ring fills of the earlier items
            uint32_t J = 0;      // stages issued so far (all items)
            int item_i = 0;
            auto wait = [&](uint32_t bar, uint32_t parity) {
                if (ok && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                    ok = false;
                }
                return ok;
            };
            // P.V of stage jj (global stage JJ) of the current item
            auto pv = [&](int jj, uint32_t JJ) {
                const uint32_t f = fbase + 2 * jj + 1;
                const int e = f % C::kRing;
                if (!wait(full(e), (f / C::kRing) & 1)) return;
                if (!wait(p_full, JJ & 1)) return;
                if (jj == 0 && item_i > 0 && !wait(o_empty, (item_i - 1) & 1)) return;
                tc_fence_after();
                const uint32_t sV = ring + e * C::kEntry;
#pragma unroll
                for (int kk = 0; kk < C::kTP / 16; ++kk) {
                    const uint64_t a = smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128);
                    umma_ss(tO, a, smem_desc(sPhi + kk * 16 * 64, C::kTP * 64, 512, kSwz64), kIdescPV,
                            (jj > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < C::kTP / 16; ++kk) {
                    const uint64_t a = smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128);
                    umma_ss(tO, a, smem_desc(sPlo + kk * 16 * 64, C::kTP * 64, 512, kSwz64), kIdescPV, 1u);
                }
                umma_commit(empty(e));
                umma_commit(p_empty);
            };
            for (int w = blockIdx.x; w < n_work && ok; w += gridDim.x) {
                TcWork wk;
                if (!tc_work(p, w, P, wk) || wk.n_local <= 0) continue;
                const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
                if (!wait(q_full, item_i & 1)) break;
                for (int j = 0; j < n_st && ok; ++j) {
                    const uint32_t f = fbase + 2 * j;
                    const int e = f % C::kRing;
                    const int sb = J & 1;
                    if (!wait(full(e), (f / C::kRing) & 1)) break;
                    if (J >= 2 && !wait(s_empty(sb), ((J >> 1) - 1) & 1)) break;
                    tc_fence_after();
                    const uint32_t sK = ring + e * C::kEntry;
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        const uint32_t koff = (kk >> 2) * C::kBoxB + (kk & 3) * 32;
                        const uint32_t qoff = (kk >> 2) * G * 128 + (kk & 3) * 32;
                        umma_ss(tS + sb * G, smem_desc(sK + koff, 16, 1024, kSwz128),
                                smem_desc(sQ + qoff, 16, 1024, kSwz128), kIdescQK, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(s_full(sb));
                    umma_commit(empty(e));
                    if (j == n_st - 1) umma_commit(q_empty);
                    if (j > 0) pv(j - 1, J - 1);
                    ++J;
                }
                if (!ok) break;
                pv(n_st - 1, J - 1);
                umma_commit(o_full);
                fbase += 2 * n_st;
                ++item_i;
            }
            // every MMA issued has completed before tensor memory is released
            umma_commit(done_bar);
            if (!mbar_wait_bounded(done_bar, 0, kWaitLimitNs)) raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // Named barrier 1 (these 128 threads) is only ever reached by all four warps together: a
        // failed wait is shared at the next flag exchange and every warp then stops at once.
        const int sw = warp - 2;           // softmax warp 0..3
        const int quarter = warp & 3;      // tensor-memory lane quarter of this warp
        const int r = quarter * 32 + lane;  // token row of S^T, dimension row of O^T
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        float* red = reinterpret_cast<float*>(smem + C::kOffRed);
        volatile int* flags = reinterpret_cast<volatile int*>(smem + C::kOffFlag);
        int rbuf = 0, fbuf = 0;
        bool ok = true;  // equal in the four warps at every flag exchange
        uint32_t fbase = 0, J = 0;
        int item_i = 0;
        // warp-uniform outcome: the tensor-memory loads and stores after a wait are warp-collective
        auto wait = [&](bool& okl, uint32_t bar, uint32_t parity) {
            if (okl && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                okl = false;
            }
            okl = __all_sync(0xffffffffu, okl);
            return okl;
        };
        // OR of `bits` over the four warps (bit 1: a wait failed)
        auto exchange = [&](int bits) {
            bits = __reduce_or_sync(0xffffffffu, bits);
            if (lane == 0) flags[fbuf * 4 + sw] = bits;
            named_bar_sync(1, 128);
            const int all = flags[fbuf * 4] | flags[fbuf * 4 + 1] | flags[fbuf * 4 + 2] | flags[fbuf * 4 + 3];
            fbuf ^= 1;
            return all;
        };
        auto zero_rows = [&](const TcWork& wk) {
            if (!wk.split_mode)
                for (int h = 0; h < G; ++h) p.out[((int64_t)wk.b * p.H_q + wk.kvh * G + h) * DH + r] = 0.f;
        };
        for (int w = blockIdx.x; w < n_work; w += gridDim.x) {
            TcWork wk;
            if (!tc_work(p, w, P, wk)) continue;
            if (wk.bad_len && r == 0 && wk.split == 0 && p.items == nullptr) raise_err(p.err, KV_DEV_ERR_SEQ_LEN);
            if (wk.n_local <= 0 || !ok) {
                zero_rows(wk);
                continue;
            }
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            float m_ref[G], lp[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY, lp[h] = 0.f;
            for (int j = 0; j < n_st; ++j) {
                bool okl = ok;
                const int sb = J & 1;
                float s[G];
#pragma unroll
                for (int h = 0; h < G; ++h) s[h] = -INFINITY;
                if (wait(okl, s_full(sb), (J >> 1) & 1)) {
                    tc_fence_after();
                    uint32_t a[16], b2[16];
                    tmem_ld16(tS + sb * G + lane_addr, a);
                    tmem_ld16(tS + sb * G + 16 + lane_addr, b2);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 16; ++h) s[h] = __uint_as_float(a[h]), s[16 + h] = __uint_as_float(b2[h]);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_empty(sb));
                }
                // the stage's V entry (and its skipped-page mask) must have landed
                const uint32_t fv = fbase + 2 * j + 1;
                const int ev = fv % C::kRing;
                bool valid = false;
                if (wait(okl, full(ev), (fv / C::kRing) & 1)) {
                    const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                    const int bad = stage_bad[ev];
                    const int pg_in = r / P;
                    valid = (wk.first + j * C::kPPS) * P + r < wk.len && pg_in < np && !((bad >> pg_in) & 1);
                }
#pragma unroll
                for (int h = 0; h < G; ++h) s[h] = valid ? s[h] * p.scale_log2 : -INFINITY;
                // reference maximum: moves only when a score exceeds it by more than 2^8
                bool need = false;
#pragma unroll
                for (int h = 0; h < G; ++h) need |= s[h] > m_ref[h] + 8.f;
                const int all = exchange((need ? 1 : 0) | (okl ? 0 : 2));
                if (all & 2) {
                    ok = false;
                    break;
                }
                float alpha[G];
                bool rescale_o = false;
                if (all & 1) {
                    float mx[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) mx[h] = s[h];
                    cta_heads_reduce<true>(mx, red, sw, lane, rbuf);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float mn = fmaxf(m_ref[h], mx[h]);
                        alpha[h] = (mn == m_ref[h]) ? 1.f : exp2f(m_ref[h] - mn);
                        m_ref[h] = mn;
                        lp[h] *= alpha[h];
                    }
                    rescale_o = j > 0;
                }
                // P.V of the previous stage has finished: the P^T tiles are free and O^T is settled
                if (J > 0 && !wait(okl, p_empty, (J - 1) & 1)) {
                    ok = false;  // the next flag exchange stops every warp
                    ++J;
                    continue;
                }
                if (rescale_o) {
                    tc_fence_after();
                    uint32_t a[16], b2[16];
                    tmem_ld16(tO + lane_addr, a);
                    tmem_ld16(tO + 16 + lane_addr, b2);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        a[h] = __float_as_uint(__uint_as_float(a[h]) * alpha[h]);
                        b2[h] = __float_as_uint(__uint_as_float(b2[h]) * alpha[16 + h]);
                    }
                    tmem_st16(tO + lane_addr, a);
                    tmem_st16(tO + 16 + lane_addr, b2);
                    tmem_wait_st();
                }
                // probabilities -> P^T row r (hi and residual lo), 64-byte swizzle
                uint32_t hi[G / 2], lo[G / 2];
#pragma unroll
                for (int i = 0; i < G / 2; ++i) {
                    const float p0 = s[2 * i] == -INFINITY ? 0.f : exp2f(s[2 * i] - m_ref[2 * i]);
                    const float p1 = s[2 * i + 1] == -INFINITY ? 0.f : exp2f(s[2 * i + 1] - m_ref[2 * i + 1]);
                    lp[2 * i] += p0;
                    lp[2 * i + 1] += p1;
                    pack2_split<kBF16>(p0, p1, hi[i], lo[i]);
                }
#pragma unroll
                for (int c = 0; c < G / 8; ++c) {
                    const uint32_t off = r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
                    sts128(sPhi + off, hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                    sts128(sPlo + off, lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                }
                // a masked token's V row may hold stale bytes (even NaN): zero it before P.V
                if (!valid) {
                    const uint32_t vrow = ring + ev * C::kEntry + r * 128;
#pragma unroll
                    for (int bb = 0; bb < C::kBoxCols; ++bb)
#pragma unroll
                        for (int c = 0; c < 8; ++c) sts128_zero(vrow + bb * C::kBoxB + c * 16);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
                ++J;
            }
            // ---- epilogue: O^T row r, row sums over the CTA, output or partials
            bool okl = ok;
            if (wait(okl, o_full, item_i & 1)) {
                tc_fence_after();
            }
            if (exchange(okl ? 0 : 2) & 2) ok = false;
            if (!ok) {
                zero_rows(wk);
                continue;
            }
            fbase += 2 * n_st;
            float o[G];
            {
                uint32_t a[16], b2[16];
                tmem_ld16(tO + lane_addr, a);
                tmem_ld16(tO + 16 + lane_addr, b2);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 16; ++h) o[h] = __uint_as_float(a[h]), o[16 + h] = __uint_as_float(b2[h]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_empty);
            ++item_i;
            cta_heads_reduce<false>(lp, red, sw, lane, rbuf);
            const int64_t hq0 = (int64_t)wk.b * p.H_q + (int64_t)wk.kvh * G;
            if (!wk.split_mode) {
#pragma unroll
                for (int h = 0; h < G; ++h) p.out[(hq0 + h) * DH + r] = lp[h] > 0.f ? o[h] / lp[h] : 0.f;
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const int64_t ps = p.items != nullptr ? (int64_t)wk.item * G + h : (hq0 + h) * p.num_splits + wk.split;
                    p.part_u[ps * DH + r] = o[h];
                    if (r == 0) p.part_ml[ps] = make_float2(m_ref[h], lp[h]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace kvp
