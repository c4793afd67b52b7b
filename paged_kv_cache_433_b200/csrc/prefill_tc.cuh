// Multi-token query (chunked prefill) over the paged cache on the
// fifth-generation tensor cores (tcgen05), sm_100a.
//
// What is computed: row i of sequence b's chunk sits at position
// p_i = seq_lens[b] - n_b + i and attends to the keys at positions 0 .. p_i
// (causal within the chunk, "04. 注意力与 KV 缓存" and
// "07｜KV Cache、FlashAttention与PagedAttention的内部过程" Q025), read through
// the block table (Q028) and folded in with the online (m, l, u) merge of Q027.
// Chunked prefill itself is the workload of "06 KV Cache、Prefix Cache、
// PagedAttention 与 vLLM", 6.2 / 6.6.
//
// Tile: 128 MMA rows = 128 / g chunk tokens x the g query heads of one KV
// head, so every K/V byte staged in shared memory serves the whole GQA group
// of 128 / g tokens. Per stage of 128 keys:
//   S[128 x 128]  = Q[128 x Dh] . K_stage^T             (SS: both K-major)
//   O[128 x Dh]  += P[128 x 128] . V_stage               (TS: P in tensor memory,
//                                                          V MN-major)
// S is triple-buffered in tensor memory (3 x 128 columns) and O takes the
// last 128 columns. Each row is owned by two threads of the eight softmax
// warps (warps w and w + 4 share a tensor-memory lane quarter; one takes
// columns 0..63, the other 64..127): exponentials and partial sums stay in
// registers, the two halves of a row meet once per stage in shared memory to
// agree on the row maximum. P is
// written back over its own S columns as a 16-bit pair: hi in columns 0..63,
// the residual lo = p - hi in 64..127 (bf16: both truncated with integer
// operations; fp16: rounded); the P.V MMA runs on both, so the probabilities
// carry ~2^-14 relative precision into the product.
// The reference maximum of a row moves only when a score exceeds it by more
// than 2^8; the row's O and l are then rescaled (o = u / l for any common
// reference).
//
// Warps (384 threads = three warpgroups, one CTA per SM by tensor memory and
// shared memory):
//   warps 0, 2 producers: per stage warp 0 the K boxes, warp 2 the V boxes
//              of its pages (P rows x 128 bytes, 128-byte swizzle) into three
//              K and two V entries of 32 KB (a K entry is refilled once its
//              QK has run);
//   warp 1     tensor memory allocation; lane 0 issues the QK(j);
//   warp 3     lane 0 issues the P.V(j); each issuer is paced only by its own
//              barriers (in different warps, so one's wait never holds up
//              the other);
//   warps 4-11 load the Q tile (swizzled stores), softmax, epilogue; each pair
//              of warps of one lane quarter syncs on its own named barrier.
// The first warpgroup gives registers back (setmaxnreg) to the two softmax
// warpgroups, which hold a 64-score half row each.
// Every wait is bounded (KV_DEV_ERR_TIMEOUT); block-table entries outside
// [0, num_pages) are never loaded (their keys are masked,
// KV_DEV_ERR_PAGE_RANGE).
#pragma once

#include <cuda.h>

#include "decode_kernel.cuh"
#include "tc05.cuh"

namespace kvp {

template <int DH, int P>
struct PfCfg {
    static constexpr int kTP = 128;              // keys per stage
    static constexpr int kPPS = kTP / P;         // pages per stage
    static constexpr int kBoxCols = DH / 64;
    static constexpr int kBoxB = kTP * 128;      // one 128-byte box column of an entry
    static constexpr int kEntry = kBoxCols * kBoxB;
    // entries 0..2 hold K of stages j % 3, entries 3..4 V of stages j % 2: a K entry is refilled as soon
    // as its QK has run, independently of the P.V of older stages
    static constexpr int kKSlots = 3, kVSlots = 2;
    static constexpr int kRing = kKSlots + kVSlots;
    static constexpr int kQB = 128 * DH * 2;     // Q tile: 128 rows
    static constexpr int kOffQ = kRing * kEntry;
    static constexpr int kOffX = kOffQ + kQB;   // row exchange: [2][2][128] floats + ints
    static constexpr int kOffBar = kOffX + 2 * 2 * 128 * 4 * 2;
    // full[R], empty[R], q_full, s_full[3], p_full[3], p_empty[3], o_full, done (QK), done (PV)
    static constexpr int kNumBars = 2 * kRing + 1 + 3 + 3 + 3 + 3;
    static constexpr int kOffTmem = kOffBar + 8 * kNumBars;
    static constexpr int kSmem = 1024 + kOffTmem + 16;
    static constexpr int kThreads = 384;
    static constexpr int kVWarp = 2;             // the V producer (warp 0 produces K)
    static constexpr int kPVWarp = 3;            // issues P.V (warp 1 issues QK)
    static constexpr int kFirstSoftmaxWarp = 4;
    // registers per thread after the split: warpgroup 0 (producers, issuers) and warpgroups 1-2 (softmax);
    // 128 x kRegsLow + 256 x kRegsHigh must not exceed the launch's 384 x (registers per thread), which the
    // host checks before the first launch
    static constexpr uint32_t kRegsLow = 64, kRegsHigh = 216;
    static constexpr int kSoftmaxWarps = 8;
    static constexpr uint32_t kTmemCols = 512;   // S x 3 (384) + O (128)
    static_assert(DH == 128, "instance: Dh = 128");
    static_assert(kPPS * kBoxCols <= 32, "one TMA box per lane");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int KT, int DH, int P>
__global__ void __launch_bounds__(384, 1)
    paged_prefill_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v) {
    using C = PfCfg<DH, P>;
    constexpr bool kBF16 = KT == KV_DTYPE_BF16;
    constexpr uint32_t kIdescQK = idesc_f16(kBF16, 128, C::kTP, false, false);
    constexpr uint32_t kIdescPV = idesc_f16(kBF16, 128, DH, false, true);
    extern __shared__ __align__(1024) unsigned char smem_raw[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();

    // ---- this CTA's tile: chunk tokens t0 .. t0 + nt - 1 of sequence b, KV head kvh
    const int kvh = blockIdx.y, b = blockIdx.z;
    const int g = p.g;
    const int qs0 = p.q_start[b];
    const int n_q = p.q_start[b + 1] - qs0;
    const int t0 = blockIdx.x * p.q_tile;
    if (t0 >= n_q) return;
    const int nt = min(p.q_tile, n_q - t0);
    int len = p.seq_lens[b];
    if (len < 0 || len > p.max_blocks * P || n_q > len) {
        if (threadIdx.x == 0 && t0 == 0 && kvh == 0) raise_err(p.err, KV_DEV_ERR_SEQ_LEN);
        // rows of this tile are zero
        for (int e = threadIdx.x; e < nt * g * DH; e += blockDim.x) {
            const int rr = e / DH;
            p.out[((int64_t)(qs0 + t0 + rr / g) * p.H_q + (int64_t)kvh * g + rr % g) * DH + e % DH] = 0.f;
        }
        return;
    }
    const int pos0 = len - n_q + t0;          // position of the tile's first token
    const int key_end = pos0 + nt;            // keys 0 .. key_end - 1 are seen by some row
    const int n_pages = (key_end + P - 1) / P;
    const int n_st = (key_end + C::kTP - 1) / C::kTP;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + C::kOffBar;
    auto full = [&](int e) { return bar0 + 8u * e; };
    auto empty = [&](int e) { return bar0 + 8u * (C::kRing + e); };
    auto kslot = [](int j) { return j % C::kKSlots; };
    auto vslot = [](int j) { return C::kKSlots + j % C::kVSlots; };
    auto kphase = [](int j) { return static_cast<uint32_t>((j / C::kKSlots) & 1); };
    auto vphase = [](int j) { return static_cast<uint32_t>((j / C::kVSlots) & 1); };
    const uint32_t q_full = bar0 + 8u * (2 * C::kRing);
    auto s_full = [&](int i) { return q_full + 8u + 8u * i; };
    // P of stage j is announced on p_full(j % 3) by all eight softmax warps. The warps of different lane
    // quarters do not wait for one another, and none waits for V, so one may arrive for stage j + 2 while
    // another is still writing P(j): with two barriers that early arrival would complete stage j's phase.
    // Stage j + 3 needs S(j + 3), hence QK(j + 3), hence P.V(j) done, hence every stage-j arrival: three
    // barriers keep each phase's arrivals to its own stage.
    auto p_full = [&](int i) { return q_full + 32u + 8u * i; };
    // P.V(j) completion is announced on p_empty(j % 3), the barrier of the S columns it read
    auto p_empty = [&](int i) { return q_full + 56u + 8u * i; };
    const uint32_t o_full = q_full + 80;
    const uint32_t done_qk = q_full + 88;
    const uint32_t done_pv = q_full + 96;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmem);

    if (threadIdx.x == 0) {
        for (int e = 0; e < C::kRing; ++e) {
            mbar_init(full(e), 1);
            mbar_init(empty(e), 1);
        }
        mbar_init(q_full, C::kSoftmaxWarps);
        for (int i = 0; i < 3; ++i) mbar_init(s_full(i), 1);
        for (int i = 0; i < 3; ++i) mbar_init(p_full(i), C::kSoftmaxWarps);
        for (int i = 0; i < 3; ++i) mbar_init(p_empty(i), 1);
        mbar_init(o_full, 1);
        mbar_init(done_qk, 1);
        mbar_init(done_pv, 1);
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
    const uint32_t tO = tmem + 3 * C::kTP;
    const uint32_t ring = sbase;
    const uint32_t sQ = sbase + C::kOffQ;

    // the register split sits at the top of each warpgroup's branch, so every code path after it is
    // compiled for its own budget
    if (warp < C::kFirstSoftmaxWarp) {
    regs_dec<C::kRegsLow>();
    if (warp == 0 || warp == C::kVWarp) {
        // ------------------------------------------------------------ producers
        // warp 0 issues the K boxes of every stage, warp kVWarp the V boxes: two streams of TMA requests
        const int half = warp == 0 ? 0 : 1;
        bool ok = true;
        int kfills = 0, vfills = 0;  // stages whose K / V boxes were issued
        const int32_t* row = p.block_tables + (int64_t)b * p.max_blocks;
        int tab_cur = lane < n_pages ? row[lane] : -1, tab_nxt = -1;
        for (int j = 0; j < n_st && ok; ++j) {
            const int np = min(C::kPPS, n_pages - j * C::kPPS);
            // block-table entries come 32 at a time, one per lane, the next 32 fetched while these are used
            // (stages never straddle a group: 32 is a multiple of the pages per stage)
            if (((j * C::kPPS) & 31) == 0) {
                const int base = j * C::kPPS;
                tab_cur = base == 0 ? tab_cur : tab_nxt;
                tab_nxt = (base + 32 + lane < n_pages) ? row[base + 32 + lane] : -1;
            }
            const int pg_all = __shfl_sync(0xffffffffu, tab_cur, (j * C::kPPS + lane) & 31);
            const int pg = lane < np ? pg_all : -1;
            const bool good = lane < np && pg >= 0 && pg < p.num_pages;
            if (lane < np && !good) raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
            const unsigned gmask = __ballot_sync(0xffffffffu, good);
            const int box_page = lane / C::kBoxCols, bb = lane % C::kBoxCols;
            const int pgl = __shfl_sync(0xffffffffu, pg, box_page & 31);
            {
                const int e = half ? vslot(j) : kslot(j);
                const int use = half ? j / C::kVSlots : j / C::kKSlots;  // earlier fills of this entry
                if (lane == 0) {
                    if (use > 0 && !mbar_wait_bounded(empty(e), (use - 1) & 1, kWaitLimitNs)) {
                        raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                        ok = false;
                    } else {
                        mbar_arrive_expect_tx(full(e), __popc(gmask) * C::kBoxCols * P * 128);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (box_page < np && ((gmask >> box_page) & 1u)) {
                    const uint32_t dst = ring + e * C::kEntry + bb * C::kBoxB + box_page * P * 128;
                    tma_load_2d(dst, half ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k),
                                bb * 64, (pgl * p.H_kv + kvh) * P, full(e));
                }
                if (half) vfills = j + 1;
                else kfills = j + 1;
            }
        }
        if (lane == 0) {  // the last fill of every entry has landed before the CTA exits
            if (half == 0) {
                for (int j = max(0, kfills - C::kKSlots); j < kfills; ++j)
                    if (!mbar_wait_bounded(full(kslot(j)), kphase(j), kWaitLimitNs))
                        raise_err(p.err, KV_DEV_ERR_TIMEOUT);
            } else {
                for (int j = max(0, vfills - C::kVSlots); j < vfills; ++j)
                    if (!mbar_wait_bounded(full(vslot(j)), vphase(j), kWaitLimitNs))
                        raise_err(p.err, KV_DEV_ERR_TIMEOUT);
            }
        }
    } else {
        // ------------------------------------------------------------ MMA issue
        // Warp 1 issues QK(j) once K(j) has landed and P.V(j - 3) has released S columns j % 3; the P.V
        // warp issues P.V(j) once the softmax has written P(j). Neither waits on the other's barriers.
        const bool qk = warp == 1;
        if (lane == 0) {
            bool ok = true;
            auto wait = [&](uint32_t bar, uint32_t parity) {
                if (ok && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                    ok = false;
                }
                return ok;
            };
            if (qk) {
                if (wait(q_full, 0)) {
                    for (int j = 0; j < n_st; ++j) {
                        const int e = kslot(j);
                        if (!wait(full(e), kphase(j))) break;
                        if (j >= 3 && !wait(p_empty(j % 3), ((j - 3) / 3) & 1)) break;
                        tc_fence_after();
                        const uint32_t sK = ring + e * C::kEntry;
                        const uint32_t tS = tmem + (j % 3) * C::kTP;
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * C::kBoxB + (kk & 3) * 32;
                            umma_ss(tS, smem_desc(sQ + off, 16, 1024, kSwz128), smem_desc(sK + off, 16, 1024, kSwz128),
                                    kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(s_full(j % 3));
                        umma_commit(empty(e));
                    }
                }
            } else {
                for (int j = 0; j < n_st; ++j) {
                    const int e = vslot(j);
                    if (!wait(full(e), vphase(j))) break;
                    if (!wait(p_full(j % 3), (j / 3) & 1)) break;
                    tc_fence_after();
                    const uint32_t sV = ring + e * C::kEntry;
                    const uint32_t tP = tmem + (j % 3) * C::kTP;
#pragma unroll
                    for (int kk = 0; kk < C::kTP / 16; ++kk)
                        umma_ts(tO, tP + kk * 8, smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128), kIdescPV,
                                (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < C::kTP / 16; ++kk)
                        umma_ts(tO, tP + C::kTP / 2 + kk * 8, smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128),
                                kIdescPV, 1u);
                    umma_commit(empty(e));
                    umma_commit(p_empty(j % 3));
                }
                if (ok) umma_commit(o_full);
            }
            const uint32_t done = qk ? done_qk : done_pv;
            umma_commit(done);
            if (!mbar_wait_bounded(done, 0, kWaitLimitNs)) raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    }
    } else {
        regs_inc<C::kRegsHigh>();
        // ------------------------------------------------------------ Q tile, softmax, epilogue
        const int quarter = warp & 3;
        const int half = (warp - C::kFirstSoftmaxWarp) >> 2;  // key columns [64 half, 64 half + 64) of S, dims of O likewise
        const int r = quarter * 32 + lane;   // MMA row: chunk token t0 + r / g, head kvh * g + r % g
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t pair_bar = 1 + quarter;  // named barrier of the two warps that share row r
        const int tr = r / g;
        const bool row_valid = tr < nt;
        const int pos = pos0 + tr;           // this row sees keys 0 .. pos
        const int64_t qrow = ((int64_t)(qs0 + t0 + tr) * p.H_q + (int64_t)kvh * g + r % g);
        float* xm = reinterpret_cast<float*>(smem + C::kOffX);        // [buf][half][row] partial maxima / sums
        int* xok = reinterpret_cast<int*>(smem + C::kOffX) + 2 * 2 * 128;
        int xbuf = 0;
        // this thread's half of Q row r -> box column `half` of the swizzled K-major tile
        {
            const uint4* src = static_cast<const uint4*>(p.q) + qrow * (DH / 8) + half * 8;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (row_valid) v = src[c];
                const uint32_t dst = sQ + half * (128 * 128) + r * 128 + ((c ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z),
                             "r"(v.w)
                             : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_full);
        }
        bool ok = true;
        // warp-uniform outcome: the tensor-memory loads and stores after a wait are warp-collective
        auto wait = [&](bool& okl, uint32_t bar, uint32_t parity) {
            if (okl && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                okl = false;
            }
            okl = __all_sync(0xffffffffu, okl);
            return okl;
        };
        // the two halves of row r meet: returns the partner's value; `okl` becomes the AND of both
        auto meet = [&](float v, bool& okl) {
            xm[(xbuf * 2 + half) * 128 + r] = v;
            xok[(xbuf * 2 + half) * 128 + r] = okl ? 1 : 0;
            named_bar_sync(pair_bar, 64);
            const float other = xm[(xbuf * 2 + (half ^ 1)) * 128 + r];
            okl = __all_sync(0xffffffffu, okl && xok[(xbuf * 2 + (half ^ 1)) * 128 + r] != 0);
            xbuf ^= 1;
            return other;
        };
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        constexpr int kH = C::kTP / 2;       // key columns per thread
        // lanes 0 .. kPPS-1: the page ids of stage j, read one stage ahead; the mask of pages the producers
        // skip (entries outside the pool) is then known without waiting for the V entry
        const int32_t* trow = p.block_tables + (int64_t)b * p.max_blocks;
        int pg_cur = lane < C::kPPS && lane < n_pages ? __ldg(trow + lane) : -1;
        for (int j = 0; j < n_st; ++j) {
            bool okl = ok;
            const uint32_t tS = tmem + (j % 3) * C::kTP + lane_addr;
            const int nxt = (j + 1) * C::kPPS + lane;
            const int pg_nxt = lane < C::kPPS && nxt < n_pages ? __ldg(trow + nxt) : -1;
            float s[kH];
            if (wait(okl, s_full(j % 3), (j / 3) & 1)) {
                tc_fence_after();
                uint32_t a[32], b2[32];
                tmem_ld32(tS + half * kH, a);
                tmem_ld32(tS + half * kH + 32, b2);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) s[i] = __uint_as_float(a[i]), s[32 + i] = __uint_as_float(b2[i]);
            }
            // keys of this stage: kbase .. kbase + 127; the V entry carries the skipped-page mask
            const int ev = vslot(j);
            const int kbase = j * C::kTP;
            const int np = min(C::kPPS, n_pages - j * C::kPPS);
            const unsigned loaded = __ballot_sync(0xffffffffu, lane < np && pg_cur >= 0 && pg_cur < p.num_pages);
            const int bad = static_cast<int>(~loaded & ((1u << np) - 1u));
            pg_cur = pg_nxt;
            // keys this row may see in the stage: [0, lim); pages skipped or not loaded are masked
            const int lim = row_valid ? min(C::kTP, pos + 1 - kbase) : 0;
            const bool full_stage = lim == C::kTP && np == C::kPPS && bad == 0;
            if (!full_stage || !okl) {
#pragma unroll
                for (int c = 0; c < kH; ++c) {
                    const int cc = half * kH + c, pgi = cc / P;
                    if (!okl || cc >= lim || pgi >= np || ((bad >> pgi) & 1)) s[c] = -INFINITY;
                }
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kH; c += 2) mx = fmax3(mx, s[c], s[c + 1]);
            mx = fmaxf(mx, meet(mx, okl));
            if (!okl) {
                ok = false;  // both halves of every row of this pair stop here
                break;
            }
            const float mx2 = mx * sl2;  // sl2 > 0: the scaled maximum of the whole row
            // reference maximum: moves only when the row's max exceeds it by more than 2^8
            const bool need = mx2 > m_ref + 8.f;
            float alpha = 1.f;
            if (need) {
                alpha = exp2f(m_ref - mx2);  // 0 while m_ref is -inf
                m_ref = mx2;
                l *= alpha;
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // O holds P.V of the earlier stages: wait for the last one, then rescale this half of the rows
                if (!wait(okl, p_empty((j - 1) % 3), ((j - 1) / 3) & 1)) {
                    ok = false;  // the next meeting stops the pair
                    continue;
                }
                tc_fence_after();
                // 32 columns at a time: the 64 scores stay live across this block
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t a[32];
                    tmem_ld32(tO + lane_addr + half * kH + q2 * 32, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * alpha);
                    tmem_st32(tO + lane_addr + half * kH + q2 * 32, a);
                }
                tmem_wait_st();
            }
            // probabilities -> P over this S buffer: hi pairs in columns 0..63, residual pairs in 64..127
            // (this thread's keys: hi columns 32 half .., lo columns 64 + 32 half ..)
            const float neg = (m_ref == -INFINITY) ? 0.f : -m_ref;
            const float2 sl2v = make_float2(sl2, sl2), negv = make_float2(neg, neg);
            float2 lsum = make_float2(0.f, 0.f);
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    // two keys at a time: one packed multiply-add for the exponents, one packed add for the sums
                    const float2 x = ffma2(make_float2(s[q2 * 32 + 2 * i], s[q2 * 32 + 2 * i + 1]), sl2v, negv);
                    const float p0 = exp2f(x.x), p1 = exp2f(x.y);  // exp2(-inf) = 0 for masked keys
                    lsum = fadd2(lsum, make_float2(p0, p1));
                    pack2_split_fast<kBF16>(p0, p1, hi[i], lo[i]);
                }
                tmem_st16(tmem + (j % 3) * C::kTP + lane_addr + half * 32 + q2 * 16, hi);
                tmem_st16(tmem + (j % 3) * C::kTP + lane_addr + C::kTP / 2 + half * 32 + q2 * 16, lo);
            }
            l += lsum.x + lsum.y;
            tmem_wait_st();
            // a key no row may see (past the tile, or on a page not loaded) may hold stale bytes: zero its V row
            // (this thread: box column `half` of V row r) once the V entry has landed; only warps with such a
            // row wait for it (the P.V issuer waits for every entry)
            {
                const int pgi = r / P;
                const bool stale = kbase + r >= key_end || pgi >= np || ((bad >> pgi) & 1);
                if (__any_sync(0xffffffffu, stale)) {
                    // the entry's previous fill (stage j - kVSlots) must have been consumed first: its P.V done
                    // means that fill landed, so the wait below cannot pass on that older phase's parity
                    const int jp = j - C::kVSlots;
                    if (jp >= 0 && !wait(okl, p_empty(jp % 3), (jp / 3) & 1)) {
                        ok = false;  // the next meeting stops the pair
                        continue;
                    }
                    if (!wait(okl, full(ev), vphase(j))) {
                        ok = false;  // the next meeting stops the pair
                        continue;
                    }
                    if (stale) {
                        const uint32_t vrow = ring + ev * C::kEntry + half * C::kBoxB + r * 128;
#pragma unroll
                        for (int c = 0; c < 8; ++c) sts128_zero(vrow + c * 16);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(j % 3));
        }
        // ---- epilogue: O row / l (this thread: dims 64 half .. 64 half + 63)
        bool okl = ok;
        if (wait(okl, o_full, 0)) tc_fence_after();
        const float l_all = l + meet(l, okl);
        if (okl) {
            float* dst = p.out + qrow * DH + half * kH;
            const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
            uint32_t a[32], b2[32];
            tmem_ld32(tO + lane_addr + half * kH, a);
            tmem_ld32(tO + lane_addr + half * kH + 32, b2);
            tmem_wait_ld();
            if (row_valid) {
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    *reinterpret_cast<float4*>(dst + i) =
                        make_float4(__uint_as_float(a[i]) * inv, __uint_as_float(a[i + 1]) * inv,
                                    __uint_as_float(a[i + 2]) * inv, __uint_as_float(a[i + 3]) * inv);
                    *reinterpret_cast<float4*>(dst + 32 + i) =
                        make_float4(__uint_as_float(b2[i]) * inv, __uint_as_float(b2[i + 1]) * inv,
                                    __uint_as_float(b2[i + 2]) * inv, __uint_as_float(b2[i + 3]) * inv);
                }
            }
        } else if (row_valid) {
            for (int d = 0; d < kH; ++d) p.out[qrow * DH + half * kH + d] = 0.f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace kvp
