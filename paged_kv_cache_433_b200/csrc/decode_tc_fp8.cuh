// Paged decode attention over E4M3 K/V pools on the fifth-generation tensor
// cores (tcgen05), sm_100a: GQA groups of 4, 8 or 16 query heads, Dh = 128.
//
// The function is that of decode_tc.cuh over K_t = code_t * k_scale and
// V_t = code_t * v_scale, the per-KV-head scales of the quantised cache (the
// KV-quantisation follow-up of "03. KV Cache：用显存换计算"); attention,
// block-table walk and online merge as "07｜KV Cache、FlashAttention与
// PagedAttention的内部过程" Q027 / Q028. A page moves half the bytes of a
// 16-bit page and is widened on the SM:
//   * every E4M3 value is an fp16 value, so the products run as kind::f16 MMAs
//     on fp16 operands with K and V unrounded; q is rounded to fp16 once per
//     item (its values must lie in fp16's range), k_scale is folded into the
//     softmax's log2 scale and v_scale into the output;
//   * a converter warpgroup widens K of stage J into tensor memory (lane =
//     token, two dims per 32-bit column), where the score MMA reads it as its
//     A operand:
//       S^T[128 x g] = K_stage[128 x Dh] . Q^T[Dh x g]       (A in tensor memory)
//     and V into an fp16 tile in shared memory with the 16-bit kernel's V
//     layout (64-dim box columns, 128-byte swizzle):
//       O^T[Dh x g] += V_stage^T[Dh x 128] . P^T[128 x g]   (A, B in shared memory)
//     writing zero rows for tokens past the item's keys or on pages not
//     loaded, so no softmax warp ever waits for V.
//
// Warps (640 threads = five warpgroups, one CTA per SM, persistent):
//   warps 0, 2   producers: E4M3 K / V boxes (P rows x 128 bytes, 128-byte
//                swizzle) into staging entries of 16 KB;
//   warp 1       tensor memory, the CTA's work list; lane 0 issues QK(J);
//   warp 3       lane 0 issues P.V(J);
//   warps 4-7    softmax, as in decode_tc.cuh, but P^T is one fp16 tile: fp16's
//                11-bit significand keeps p to 2^-11 relative (the 16-bit kernels
//                add a residual tile for bf16's 8 bits), so P.V is 8 MMAs a stage;
//   warps 8-11   epilogue: O^T over the row sums times v_scale, or the partial;
//   warps 12-15  K converters: the item's q tile, then K of every stage (they run
//                ahead of the softmax, bounded only by the two K buffers);
//   warps 16-19  V converters: V of every stage (bounded by the two fp16 tiles).
// Every wait is bounded (KV_DEV_ERR_TIMEOUT); block-table entries outside
// [0, num_pages) are never loaded (their tokens are masked).
#pragma once

#include "decode_tc.cuh"
#include "fp8.cuh"

namespace kvp {

template <int P, int G>
struct TcF8Cfg {
    static constexpr int kN = 16;                // MMA N: the group's heads, zero-padded to 16
    static constexpr int kTP = 128;              // tokens per stage = MMA rows
    static constexpr int kPPS = kTP / P;         // pages per stage
    static constexpr int kStageB = kTP * 128;    // E4M3 K (or V) of a stage: one 128-byte box column
    static constexpr int kBoxB = kTP * 128;      // one 64-dim box column of the fp16 V tile
    static constexpr int kVF = 2 * kBoxB;        // fp16 V tile of a stage
    static constexpr int kQRowsB = kN * 128;     // one 64-dim box column of the fp16 q tile
    static constexpr int kQB = 2 * kQRowsB;
    static constexpr int kPRow = kN * 2;         // bytes of one P^T row (token)
    static constexpr int kPB = kTP * kPRow;      // one P^T tile (fp16, round to nearest)
    static constexpr uint32_t kPSwz = kSwz32;
    static constexpr int kPAtom = 8 * kPRow;
    static constexpr int kOBuf = 4;              // items in flight between the softmax and the epilogue
    static constexpr int kMaxList = 96;
    // staging entries: half K, half V, as many as fit beside two fp16 V tiles, two q tiles, two P^T tiles
    // and the small arrays
    static constexpr int kRing0 = (227 * 1024 - 1024 - 2 * kVF - 2 * kQB - 2 * kPB - 6144) / kStageB;
    static constexpr int kRing = kRing0 >= 8 ? 8 : (kRing0 & ~1);
    static constexpr int kKSlots = kRing / 2, kVSlots = kRing / 2;
    static constexpr int kOffVF = kRing * kStageB;
    static constexpr int kOffQ = kOffVF + 2 * kVF;
    static constexpr int kOffP = kOffQ + 2 * kQB;
    static constexpr int kOffRed = kOffP + 2 * kPB;            // 2 x [G][4] floats
    static constexpr int kOffFlag = kOffRed + 2 * G * 4 * 4;   // 2 x 4 ints
    // ints: skipped-page mask per K staging entry, per V staging entry, per K buffer, per S^T buffer
    static constexpr int kOffMask = kOffFlag + 32;
    static constexpr int kOffStats = kOffMask + 4 * (kKSlots + kVSlots + 4);  // kOBuf x [l, m][G] floats
    static constexpr int kOffList = (kOffStats + kOBuf * 2 * G * 4 + 15) & ~15;
    static constexpr int kOffStream = kOffList + kMaxList * 32;
    static constexpr int kOffBar = kOffStream + 48;
    // full[R], empty[R], q_full[2], q_empty[2], kt_full[2], kt_empty[2], vf_full[2], vf_empty[2],
    // s_full[2], s_empty[2], p_full[2], p_empty[2], mask_full[2], done_qk, done_pv, o_full[kOBuf],
    // o_empty[kOBuf], stats_full[kOBuf], stats_empty[kOBuf]
    static constexpr int kNumBars = 2 * kRing + 24 + 4 * kOBuf;
    static constexpr int kOffTmem = kOffBar + 8 * kNumBars;
    static constexpr int kSmem = 1024 + kOffTmem + 16;
    static constexpr int kThreads = 640;
    static constexpr int kVWarp = 2, kPVWarp = 3;
    static constexpr int kFirstSoftmaxWarp = 4, kFirstEpiWarp = 8, kFirstConvWarp = 12, kFirstConvVWarp = 16;
    // registers per thread after the split: warpgroups 0 (producers, issuers), 1 (softmax), 2 (epilogue),
    // 3 (K converters), 4 (V converters); 128 x their sum must fit in the launch's 640 x (registers per
    // thread)
    static constexpr uint32_t kRegsLow = 56, kRegsSoftmax = 160, kRegsEpi = 88, kRegsConvK = 88, kRegsConvV = 88;
    // tensor-memory columns: S^T x 2 and O^T x kOBuf, each as two halves of N columns (the even and the odd
    // k-steps of its MMAs accumulate apart, so consecutive MMAs do not wait on each other's result), then
    // two K buffers of 64 columns
    static constexpr uint32_t kTmemK = 256;
    static constexpr uint32_t kTmemCols = 512;
    static_assert((2 + kOBuf) * 2 * kN <= (int)kTmemK, "S^T and O^T below the K buffers");
    static_assert(G == 4 || G == 8 || G == 16, "instances: g in {4, 8, 16}");
    static_assert(kPPS <= 32, "one TMA box per lane");
    static_assert(kRing >= 4, "two staging entries each for K and V");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

// Eight bf16 values -> eight fp16 values (round to nearest, saturating at fp16's largest finite value).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
    auto cv = [](uint32_t w) {
        return pack2_satfinite_f16(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    };
    return make_uint4(cv(v.x), cv(v.y), cv(v.z), cv(v.w));
}

template <int QT, int P, int G>
__global__ void __launch_bounds__(640, 1)
    paged_decode_tc_fp8_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                               const __grid_constant__ CUtensorMap tmap_v, int n_work) {
    using C = TcF8Cfg<P, G>;
    constexpr int DH = 128;
    constexpr int N = C::kN;
    constexpr uint32_t kIdescQK = idesc_f16(false, 128, N, false, false);
    constexpr uint32_t kIdescPV = idesc_f16(false, 128, N, true, true);
    extern __shared__ __align__(1024) unsigned char smem_raw[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    const uint32_t bar0 = sbase + C::kOffBar;
    auto full = [&](int e) { return bar0 + 8u * e; };
    auto empty = [&](int e) { return bar0 + 8u * (C::kRing + e); };
    auto kslot = [](uint32_t j) { return static_cast<int>(j % C::kKSlots); };
    auto vslot = [](uint32_t j) { return static_cast<int>(C::kKSlots + j % C::kVSlots); };
    auto kphase = [](uint32_t j) { return (j / C::kKSlots) & 1u; };
    auto vphase = [](uint32_t j) { return (j / C::kVSlots) & 1u; };
    const uint32_t bx = bar0 + 8u * (2 * C::kRing);
    auto q_full = [&](int i) { return bx + 8u * i; };          // converters -> QK issuer (4 arrivals)
    auto q_empty = [&](int i) { return bx + 16u + 8u * i; };   // last QK of the item -> converters
    auto kt_full = [&](int i) { return bx + 32u + 8u * i; };   // K of stage J in tensor memory (4 arrivals)
    auto kt_empty = [&](int i) { return bx + 48u + 8u * i; };  // QK(J) done -> converters
    auto vf_full = [&](int i) { return bx + 64u + 8u * i; };   // fp16 V tile of stage J written (4 arrivals)
    auto vf_empty = [&](int i) { return bx + 80u + 8u * i; };  // P.V(J) done -> converters
    auto s_full = [&](int i) { return bx + 96u + 8u * i; };
    auto s_empty = [&](int i) { return bx + 112u + 8u * i; };
    auto p_full = [&](int i) { return bx + 128u + 8u * i; };
    auto p_empty = [&](int i) { return bx + 144u + 8u * i; };
    auto mask_full = [&](int i) { return bx + 160u + 8u * i; };
    const uint32_t done_qk = bx + 176u;
    const uint32_t done_pv = bx + 184u;
    const uint32_t bo0 = bx + 192u;
    auto o_full = [&](int i) { return bo0 + 8u * (i % C::kOBuf); };
    auto o_empty = [&](int i) { return bo0 + 8u * (C::kOBuf + i % C::kOBuf); };
    auto stats_full = [&](int i) { return bo0 + 8u * (2 * C::kOBuf + i % C::kOBuf); };
    auto stats_empty = [&](int i) { return bo0 + 8u * (3 * C::kOBuf + i % C::kOBuf); };
    auto oph = [](int i) { return static_cast<uint32_t>((i / C::kOBuf) & 1); };
    volatile int* kmask = reinterpret_cast<volatile int*>(smem + C::kOffMask);  // [kKSlots]
    volatile int* vmask = kmask + C::kKSlots;                                   // [kVSlots]
    volatile int* ktmask = vmask + C::kVSlots;                                  // [2] per K buffer
    volatile int* smask = ktmask + 2;                                           // [2] per S^T buffer
    float* stats = reinterpret_cast<float*>(smem + C::kOffStats);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmem);

    if (threadIdx.x == 0) {
        for (int e = 0; e < C::kRing; ++e) {
            mbar_init(full(e), 1);
            mbar_init(empty(e), 4);  // the four K (or V) converter warps release a staging entry
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(q_full(i), 4);
            mbar_init(q_empty(i), 1);
            mbar_init(kt_full(i), 4);
            mbar_init(kt_empty(i), 1);
            mbar_init(vf_full(i), 4);
            mbar_init(vf_empty(i), 1);
            mbar_init(s_full(i), 1);
            mbar_init(s_empty(i), 4);
            mbar_init(p_full(i), 4);
            mbar_init(p_empty(i), 1);
            mbar_init(mask_full(i), 1);
        }
        for (int i = 0; i < C::kOBuf; ++i) {
            mbar_init(o_full(i), 1);
            mbar_init(o_empty(i), 4);
            mbar_init(stats_full(i), 4);
            mbar_init(stats_empty(i), 4);
        }
        mbar_init(done_qk, 1);
        mbar_init(done_pv, 1);
        fence_barrier_init();
    }
    int4* list_e = reinterpret_cast<int4*>(smem + C::kOffList);
    const int n_cand = n_work > (int)blockIdx.x ? (n_work - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const bool stream = tc_is_stream(p);
    TcStream* st_smem = reinterpret_cast<TcStream*>(smem + C::kOffStream);
    const TcList L{list_e, stream ? C::kMaxList : min(n_cand, C::kMaxList), n_cand, stream ? st_smem : nullptr};
    if (warp == 1) {
        tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::kTmemCols);
        tmem_relinquish();
    }
    // the setup above touches only this CTA's shared and tensor memory (programmatic launch overlap)
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    if (warp == 1) tc_list_build(p, n_work, P, list_e, L.n_list, st_smem, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem;  // S^T buffer b: halves at columns 2bN and (2b + 1)N
    auto tO = [&](int i) { return tmem + 4 * N + (i % C::kOBuf) * 2 * N; };  // O^T of item i: two halves
    auto tK = [&](uint32_t j) { return tmem + C::kTmemK + (j & 1) * 64; };  // fp16 K of stage j: 64 columns
    const uint32_t ring = sbase;
    auto sVF = [&](uint32_t j) { return sbase + C::kOffVF + (j & 1) * C::kVF; };
    auto sQ = [&](int i) { return sbase + C::kOffQ + (i & 1) * C::kQB; };
    const uint32_t sP = sbase + C::kOffP;
    auto sPt = [&](uint32_t j) { return sP + (j & 1) * C::kPB; };  // P^T of stage j

    if (warp < C::kFirstSoftmaxWarp) {
    regs_dec<C::kRegsLow>();
    if (warp == 0 || warp == C::kVWarp) {
        // ------------------------------------------------------------ producers
        // warp 0 the K boxes of every stage, warp kVWarp the V boxes; each writes its entry's skipped-page
        // mask before the entry's transaction count, so a converter that has waited for it may read it
        const int half = warp == 0 ? 0 : 1;
        bool ok = true;
        uint32_t Jp = 0;
        int fills = 0;
        for (int k = 0; ok; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0 || wk.n_local <= 0) continue;
            const int32_t* row = p.block_tables + (int64_t)wk.b * p.max_blocks + wk.first;
            int tab_cur = lane < wk.n_local ? row[lane] : -1, tab_nxt = -1;
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            for (int j = 0; j < n_st && ok; ++j, ++Jp) {
                const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                if (((j * C::kPPS) & 31) == 0) {
                    const int base = j * C::kPPS;
                    tab_cur = base == 0 ? tab_cur : tab_nxt;
                    tab_nxt = (base + 32 + lane < wk.n_local) ? row[base + 32 + lane] : -1;
                }
                const int pg_all = __shfl_sync(0xffffffffu, tab_cur, (j * C::kPPS + lane) & 31);
                const int pg = lane < np ? pg_all : -1;
                const bool good = lane < np && pg >= 0 && pg < p.num_pages;
                if (lane < np && !good) raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
                const unsigned gmask = __ballot_sync(0xffffffffu, good);
                const int e = half ? vslot(Jp) : kslot(Jp);
                const uint32_t use = half ? Jp / C::kVSlots : Jp / C::kKSlots;
                if (lane == 0) {
                    if (use > 0 && !mbar_wait_bounded(empty(e), (use - 1) & 1, kWaitLimitNs)) {
                        raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                        ok = false;
                    } else {
                        (half ? vmask[e - C::kKSlots] : kmask[e]) = static_cast<int>(~gmask & ((1u << np) - 1u));
                        mbar_arrive_expect_tx(full(e), __popc(gmask) * P * 128);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane < np && ((gmask >> lane) & 1u))
                    tma_load_2d(ring + e * C::kStageB + lane * P * 128,
                                half ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k), 0,
                                (pg * p.H_kv + wk.kvh) * P, full(e));
                fills = Jp + 1;
            }
        }
        if (lane == 0) {  // every copy in flight lands before the CTA exits
            const int slots = half ? C::kVSlots : C::kKSlots;
            for (int j = max(0, fills - slots); j < fills; ++j)
                if (!mbar_wait_bounded(full(half ? vslot(j) : kslot(j)), half ? vphase(j) : kphase(j), kWaitLimitNs))
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------------------ MMA issue
        // Warp 1: QK(J) once the converters have put K(J) in tensor memory and an S^T buffer is free;
        // warp 3: P.V(J) once the fp16 V tile and P^T(J) are written.
        const bool qk = warp == 1;
        if (lane == 0) {
            bool ok = true;
            uint32_t J = 0;
            int item_i = 0;
            auto wait = [&](uint32_t bar, uint32_t parity) {
                if (ok && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                    ok = false;
                }
                return ok;
            };
            for (int k = 0; ok; ++k) {
                TcWork wk;
                const int got = tc_get(p, L, k, P, wk);
                if (got < 0) break;
                if (got == 0 || wk.n_local <= 0) continue;
                const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
                if (qk) {
                    if (!wait(q_full(item_i & 1), (item_i >> 1) & 1)) break;
                    for (int j = 0; j < n_st; ++j, ++J) {
                        const int sb = J & 1;
                        if (!wait(kt_full(J & 1), (J >> 1) & 1)) break;
                        const int bad = ktmask[J & 1];
                        if (J >= 2 && !wait(s_empty(sb), ((J >> 1) - 1) & 1)) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk) {
                            const uint32_t qoff = (kk >> 2) * C::kQRowsB + (kk & 3) * 32;
                            umma_ts(tS + (2 * sb + (kk & 1)) * N, tK(J) + kk * 8,
                                    smem_desc(sQ(item_i) + qoff, 16, 1024, kSwz128), kIdescQK, kk >= 2 ? 1u : 0u);
                        }
                        umma_commit(s_full(sb));
                        smask[sb] = bad;  // S^T buffer sb is free (s_empty above), so is its mask word
                        mbar_arrive(mask_full(sb));
                        umma_commit(kt_empty(J & 1));
                        if (j == n_st - 1) umma_commit(q_empty(item_i & 1));
                    }
                } else {
                    for (int j = 0; j < n_st; ++j, ++J) {
                        if (!wait(vf_full(J & 1), (J >> 1) & 1)) break;
                        if (!wait(p_full(J & 1), (J >> 1) & 1)) break;
                        if (j == 0 && item_i >= C::kOBuf && !wait(o_empty(item_i), oph(item_i) ^ 1u)) break;
                        tc_fence_after();
                        const uint32_t sV = sVF(J);
#pragma unroll
                        for (int kk = 0; kk < C::kTP / 16; ++kk) {
                            const uint64_t a = smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128);
                            umma_ss(tO(item_i) + (kk & 1) * N, a,
                                    smem_desc(sPt(J) + kk * 16 * C::kPRow, C::kPB, C::kPAtom, C::kPSwz), kIdescPV,
                                    (j > 0 || kk >= 2) ? 1u : 0u);
                        }
                        umma_commit(vf_empty(J & 1));
                        umma_commit(p_empty(J & 1));
                    }
                    if (ok) umma_commit(o_full(item_i));
                }
                ++item_i;
            }
            // every MMA this thread issued has completed before tensor memory is released
            const uint32_t done = qk ? done_qk : done_pv;
            umma_commit(done);
            if (!mbar_wait_bounded(done, 0, kWaitLimitNs)) raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    }
    } else if (warp < C::kFirstEpiWarp) {
        regs_inc<C::kRegsSoftmax>();
        // ------------------------------------------------------------ softmax
        // As in decode_tc.cuh; the log2 scale of an item carries its KV head's k_scale, and V rows of
        // masked tokens are zero in the fp16 tile already (the converters write them so).
        const int sw = warp - C::kFirstSoftmaxWarp;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // token row of S^T, dimension row of O^T
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        float* red = reinterpret_cast<float*>(smem + C::kOffRed);
        volatile int* flags = reinterpret_cast<volatile int*>(smem + C::kOffFlag);
        int rbuf = 0, fbuf = 0;
        bool ok = true;
        uint32_t J = 0;
        int item_i = 0;
        auto wait = [&](bool& okl, uint32_t bar, uint32_t parity) {
            if (okl && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                okl = false;
            }
            okl = __all_sync(0xffffffffu, okl);
            return okl;
        };
        auto exchange = [&](int bits) {
            bits = __reduce_or_sync(0xffffffffu, bits);
            if (lane == 0) flags[fbuf * 4 + sw] = bits;
            named_bar_sync(1, 128);
            const int all = flags[fbuf * 4] | flags[fbuf * 4 + 1] | flags[fbuf * 4 + 2] | flags[fbuf * 4 + 3];
            fbuf ^= 1;
            return all;
        };
        for (int k = 0;; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0 || wk.n_local <= 0 || !ok) continue;  // the epilogue warps zero such rows
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            const float sl2 = p.scale_log2 * p.k_scale[wk.kvh];
            float m_ref[G], lp[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY, lp[h] = 0.f;
            const int pr = r / P;
            for (int j = 0; j < n_st; ++j) {
                bool okl = ok;
                const int sb = J & 1;
                int bad = -1;
                float s[G];
#pragma unroll
                for (int h = 0; h < G; ++h) s[h] = -INFINITY;
                if (wait(okl, s_full(sb), (J >> 1) & 1)) {
                    tc_fence_after();
                    uint32_t a[N], b2[N];
                    tmem_ld_cols<N>(tS + 2 * sb * N + lane_addr, a);
                    tmem_ld_cols<N>(tS + (2 * sb + 1) * N + lane_addr, b2);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < G; ++h) s[h] = __uint_as_float(a[h]) + __uint_as_float(b2[h]);
                    tc_fence_before();
                    if (wait(okl, mask_full(sb), (J >> 1) & 1)) bad = smask[sb];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_empty(sb));
                }
                const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                const bool valid = okl && (wk.first + j * C::kPPS) * P + r < wk.len && pr < np && !((bad >> pr) & 1);
#pragma unroll
                for (int h = 0; h < G; ++h) s[h] = valid ? s[h] * sl2 : -INFINITY;
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
                    cta_heads_reduce<G, true>(mx, red, sw, lane, rbuf);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float mn = fmaxf(m_ref[h], mx[h]);
                        alpha[h] = (mn == m_ref[h]) ? 1.f : exp2f(m_ref[h] - mn);
                        m_ref[h] = mn;
                        lp[h] *= alpha[h];
                    }
                    rescale_o = j > 0;
                }
                // P^T buffer J & 1 is free once P.V(J - 2) has finished; a rescale of O^T also needs P.V(J - 1)
                bool okw = true;
                if (J >= 2) okw = wait(okl, p_empty(J & 1), ((J >> 1) - 1) & 1);
                if (okw && rescale_o) okw = wait(okl, p_empty((J - 1) & 1), ((J - 1) >> 1) & 1);
                if (!okw) {
                    ok = false;  // the next flag exchange stops every warp
                    ++J;
                    continue;
                }
                if (rescale_o) {
                    tc_fence_after();
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t a[N];
                        tmem_ld_cols<N>(tO(item_i) + hf * N + lane_addr, a);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < G; ++h) a[h] = __float_as_uint(__uint_as_float(a[h]) * alpha[h]);
                        tmem_st_cols<N>(tO(item_i) + hf * N + lane_addr, a);
                    }
                    tmem_wait_st();
                }
                // probabilities -> P^T row r (fp16, round to nearest; padding heads are zero), swizzled rows;
                // l sums the unrounded p
                uint32_t pt[N / 2];
#pragma unroll
                for (int i = 0; i < N / 2; ++i) {
                    if (2 * i < G) {
                        const float p0 = s[2 * i] == -INFINITY ? 0.f : exp2f(s[2 * i] - m_ref[2 * i]);
                        const float p1 = s[2 * i + 1] == -INFINITY ? 0.f : exp2f(s[2 * i + 1] - m_ref[2 * i + 1]);
                        lp[2 * i] += p0;
                        lp[2 * i + 1] += p1;
                        pt[i] = pack2_satfinite_f16(p0, p1);
                    } else {
                        pt[i] = 0u;
                    }
                }
#pragma unroll
                for (int c = 0; c < N / 8; ++c) {
                    const uint32_t phys = c ^ ((r >> 2) & 1);  // 32-byte rows: the 32-byte swizzle
                    sts128(sPt(J) + r * C::kPRow + (phys << 4), pt[4 * c], pt[4 * c + 1], pt[4 * c + 2], pt[4 * c + 3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full(J & 1));
                ++J;
            }
            // ---- hand the item to the epilogue warps: row sums over the CTA and the reference maxima
            cta_heads_reduce<G, false>(lp, red, sw, lane, rbuf);
            bool oks = ok;
            if (item_i >= C::kOBuf) wait(oks, stats_empty(item_i), oph(item_i) ^ 1u);
            if (exchange(oks ? 0 : 2) & 2) {
                ok = false;
                continue;
            }
            if (r == 0) {
                float* stl = stats + (item_i % C::kOBuf) * 2 * G;
#pragma unroll
                for (int h = 0; h < G; ++h) stl[h] = lp[h], stl[G + h] = m_ref[h];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(stats_full(item_i));
            ++item_i;
        }
    } else if (warp < C::kFirstConvWarp) {
        regs_dec<C::kRegsEpi>();
        // ------------------------------------------------------------ epilogue
        // Row r of O^T of each item over the CTA's row sums, times v_scale; or the partial (u, m, l).
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // dimension row of O^T
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        bool ok = true;
        int item_i = 0;
        auto wait = [&](bool& okl, uint32_t bar, uint32_t parity) {
            if (okl && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                okl = false;
            }
            okl = __all_sync(0xffffffffu, okl);
            return okl;
        };
        auto zero_rows = [&](const TcWork& wk) {
            if (!wk.split_mode)
                for (int h = 0; h < G; ++h) p.out[((int64_t)wk.b * p.H_q + wk.kvh * G + h) * DH + r] = 0.f;
        };
        for (int k = 0;; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0) continue;
            if (wk.bad_len && r == 0 && wk.split == 0 && p.items == nullptr) raise_err(p.err, KV_DEV_ERR_SEQ_LEN);
            if (wk.n_local <= 0 || !ok) {
                zero_rows(wk);
                continue;
            }
            bool okl = ok;
            wait(okl, stats_full(item_i), oph(item_i));
            wait(okl, o_full(item_i), oph(item_i));
            if (!okl) {
                ok = false;
                zero_rows(wk);
                continue;
            }
            tc_fence_after();
            float o[G];
            {
                uint32_t a[N], b2[N];
                tmem_ld_cols<N>(tO(item_i) + lane_addr, a);
                tmem_ld_cols<N>(tO(item_i) + N + lane_addr, b2);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < G; ++h) o[h] = __uint_as_float(a[h]) + __uint_as_float(b2[h]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_empty(item_i));
            float l[G], m[G];
            {
                const float* stl = stats + (item_i % C::kOBuf) * 2 * G;
#pragma unroll
                for (int h = 0; h < G; ++h) l[h] = stl[h], m[h] = stl[G + h];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(stats_empty(item_i));
            ++item_i;
            const float vs = p.v_scale[wk.kvh];
            const int64_t hq0 = (int64_t)wk.b * p.H_q + (int64_t)wk.kvh * G;
            if (!wk.split_mode) {
#pragma unroll
                for (int h = 0; h < G; ++h) p.out[(hq0 + h) * DH + r] = l[h] > 0.f ? o[h] * vs / l[h] : 0.f;
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const int64_t ps = wk.planned ? (int64_t)wk.item * G + h : (hq0 + h) * p.num_splits + wk.split;
                    p.part_u[ps * DH + r] = o[h] * vs;
                    if (r == 0) p.part_ml[ps] = make_float2(m[h], l[h]);
                }
            }
        }
    } else if (warp < C::kFirstConvVWarp) {
        regs_dec<C::kRegsConvK>();
        // ------------------------------------------------------------ K converters
        // Thread r widens token row r of every stage's K into tensor-memory lane r of the stage's K buffer
        // (32-bit column c = dims 2c, 2c + 1). Before an item's stages, the four warps write its q tile.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        bool ok = true;
        uint32_t J = 0;
        int item_i = 0;
        auto wait = [&](uint32_t bar, uint32_t parity) {
            bool w = ok;
            if (w && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                w = false;
            }
            ok = __all_sync(0xffffffffu, w);
            return ok;
        };
        for (int k = 0; ok; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0 || wk.n_local <= 0) continue;
            // q tile of the item, fp16, K-major with the 128-byte swizzle: head rows (G of them, the rest
            // zero) x 16 chunks of 8 dims; buffer item_i & 1 is free once the last QK of item i - 2 has run
            if (item_i >= 2 && !wait(q_empty(item_i & 1), ((item_i >> 1) - 1) & 1)) break;
            {
                const int64_t qrow0 = (int64_t)wk.b * p.H_q + (int64_t)wk.kvh * G;
                const uint4* qsrc = static_cast<const uint4*>(p.q);
                for (int i = r; i < N * 16; i += 128) {
                    const int h = i >> 4, c = i & 15;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (h < G) {
                        v = qsrc[(qrow0 + h) * (DH / 8) + c];
                        if constexpr (QT == KV_DTYPE_BF16) v = bf16x8_to_f16x8(v);
                    }
                    const int cc = c & 7;
                    sts128(sQ(item_i) + (c >> 3) * C::kQRowsB + h * 128 + ((cc ^ (h & 7)) << 4), v.x, v.y, v.z, v.w);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(q_full(item_i & 1));
            }
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            for (int j = 0; j < n_st; ++j, ++J) {
                const int ke = kslot(J);
                // K(J) -> registers (the staging entry is released at once) -> tensor memory, whose K buffer
                // is free once QK(J - 2) has run
                if (!wait(full(ke), kphase(J))) break;
                const uint32_t src = ring + ke * C::kStageB + r * 128;
                uint32_t w[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x = lds128(src + ((c ^ (r & 7)) << 4));  // dims 16c .. 16c + 15
                    w[4 * c] = x.x, w[4 * c + 1] = x.y, w[4 * c + 2] = x.z, w[4 * c + 3] = x.w;
                }
                if (warp == C::kFirstConvWarp && lane == 0) ktmask[J & 1] = kmask[ke];
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(ke));  // the entry's bytes are in registers
                if (J >= 2 && !wait(kt_empty(J & 1), ((J >> 1) - 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int hcol = 0; hcol < 2; ++hcol) {
                    uint32_t f[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) e4m3x4_to_f16x2x2(w[16 * hcol + i], f[2 * i], f[2 * i + 1]);
                    tmem_st32(tK(J) + lane_addr + 32 * hcol, f);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(kt_full(J & 1));
            }
            ++item_i;
        }
    } else {
        regs_dec<C::kRegsConvV>();
        // ------------------------------------------------------------ V converters
        // Thread r widens token row r of every stage's V into row r of the stage's fp16 tile: zero for a
        // token past the item's keys or on a page not loaded.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        bool ok = true;
        uint32_t J = 0;
        auto wait = [&](uint32_t bar, uint32_t parity) {
            bool w = ok;
            if (w && !mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                w = false;
            }
            ok = __all_sync(0xffffffffu, w);
            return ok;
        };
        for (int k = 0; ok; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0 || wk.n_local <= 0) continue;
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            const int pr = r / P;
            for (int j = 0; j < n_st; ++j, ++J) {
                const int ve = vslot(J);
                // V(J) -> fp16 tile J & 1, free once P.V(J - 2) has run
                if (!wait(full(ve), vphase(J))) break;
                if (J >= 2 && !wait(vf_empty(J & 1), ((J >> 1) - 1) & 1)) break;
                const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                const int bad = vmask[ve - C::kKSlots];
                const bool valid = (wk.first + j * C::kPPS) * P + r < wk.len && pr < np && !((bad >> pr) & 1);
                const uint32_t dst = sVF(J) + r * 128;
                if (valid) {
                    const uint32_t src = ring + ve * C::kStageB + r * 128;
                    uint4 x[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) x[c] = lds128(src + ((c ^ (r & 7)) << 4));  // dims 16c .. 16c + 15
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t f[8];
                        e4m3x4_to_f16x2x2(x[c].x, f[0], f[1]);
                        e4m3x4_to_f16x2x2(x[c].y, f[2], f[3]);
                        e4m3x4_to_f16x2x2(x[c].z, f[4], f[5]);
                        e4m3x4_to_f16x2x2(x[c].w, f[6], f[7]);
                        // dims 16c .. 16c + 7 and 16c + 8 .. 16c + 15: box column c / 4, chunks 2 (c % 4) (+1)
                        const uint32_t col = dst + (c >> 2) * C::kBoxB;
                        const uint32_t c0 = 2u * (c & 3);
                        sts128(col + ((c0 ^ (r & 7)) << 4), f[0], f[1], f[2], f[3]);
                        sts128(col + (((c0 + 1) ^ (r & 7)) << 4), f[4], f[5], f[6], f[7]);
                    }
                } else {
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb)
#pragma unroll
                        for (int c = 0; c < 8; ++c) sts128_zero(dst + bb * C::kBoxB + c * 16);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(vf_full(J & 1));
                    mbar_arrive(empty(ve));
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
