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
// row t of O^T. P^T goes to shared memory as a 16-bit pair hi + lo (bf16:
// hi = p truncated, lo = p - hi truncated, integer operations only; fp16: both
// rounded to nearest); the second P.V MMA on lo carries p to ~2^-14 relative,
// so short rows keep the accuracy of the fp32 softmax.
//
// Reference maximum (log2 units, per head, shared by the whole CTA): it moves
// only when some score of a stage exceeds it by more than 2^8; then the stage
// maximum is reduced over the CTA, and O^T and the partial row sums are
// rescaled (o = u / l holds for any common reference).
//
// Warp roles (384 threads = three warpgroups, one CTA per SM, persistent over
// work items):
//   warps 0, 2 producers: warp 0 the Q tile (2-D TMA, 128-byte swizzle) and
//              the K boxes of each stage, warp 2 the V boxes (P rows x 128
//              bytes each), into K and V entries of 32 KB; each writes its
//              half of the fused append when the item owns the last page.
//   warp 1     allocates tensor memory and resolves the CTA's work items
//              into shared memory; its lane 0 issues the QK(j).
//   warp 3     lane 0 issues the P.V(j). The two issuers sit in different
//              warps so that neither one's wait holds up the other (two
//              lanes of one warp would take turns).
//   warps 4-7  softmax (tensor-memory lane quarter = warp % 4); at the end of
//              an item they hand its row sums and maxima to
//   warps 8-11 the epilogue: O^T of the item over the sums, or its partial,
//              while the softmax warps already work on the next item.
// The first and last warpgroups give registers (setmaxnreg) to the softmax
// warpgroup, whose threads hold G scores, maxima and sums each.
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
#include "plan_layout.cuh"
#include "tc05.cuh"

namespace kvp {

template <int DH, int P, int G>
struct TcCfg {
    static constexpr int kN = G < 16 ? 16 : G;   // MMA N (head columns; heads >= G are zero padding)
    static constexpr int kTP = 128;              // tokens per stage = MMA rows
    static constexpr int kPPS = kTP / P;         // pages per stage
    static constexpr int kBoxCols = DH / 64;     // 128-byte box columns per token row
    static constexpr int kBoxB = kTP * 128;      // one box column of an entry
    static constexpr int kEntry = kBoxCols * kBoxB;  // K (or V) of one stage
    static constexpr int kPB0 = kTP * kN * 2;    // one P^T tile (hi or lo)
    // ring entries (K or V of a stage) that fit beside two Q tiles, two P^T buffers (hi + lo each), the
    // work list (3 KB) and the small arrays
    static constexpr int kRing0 = (227 * 1024 - 1024 - 2048 - 3120 - 2 * kBoxCols * kN * 128 - 4 * kPB0) / kEntry;
    static constexpr int kRing = kRing0 > 6 ? 6 : kRing0;
    // K of global stage J in entry J % kKSlots, V in kKSlots + J % kVSlots: a K entry is refilled as soon as
    // its QK has run, whatever the P.V of older stages
    static constexpr int kKSlots = (kRing + 1) / 2, kVSlots = kRing / 2;
    static constexpr int kQRowsB = kN * 128;     // one box column of the Q tile
    static constexpr int kQB = kBoxCols * kQRowsB;
    // At g = 32 the P^T of a stage is one tile whose token rows hold the N hi probabilities, then their N
    // residuals: the P.V MMA has 2N columns and accumulates hi into O^T columns [0, N) and lo into [N, 2N)
    // (summed in the epilogue), 8 MMAs a stage instead of 16 (the tensor pipe's cost per small MMA bounds
    // the MQA stage). Smaller groups, bound by HBM, keep separate hi and lo tiles.
    static constexpr bool kStackP = G == 32;
    static constexpr int kPRow = kN * (kStackP ? 4 : 2);  // bytes of one P^T row (token)
    static constexpr int kPB = kTP * kPRow;      // one P^T tile (stacked, or hi or lo)
    static constexpr int kPTiles = kStackP ? 2 : 4;  // P^T tiles of the two stage buffers
    static constexpr int kPVN = kStackP ? 2 * kN : kN;  // columns of the P.V MMA and of an item's O^T
    // P^T rows of 32 / 64 bytes: MN-major with the 32- / 64-byte swizzle; 8-row atoms
    static constexpr uint32_t kPSwz = kPRow == 32 ? kSwz32 : (kPRow == 64 ? kSwz64 : kSwz128);
    static constexpr int kPAtom = 8 * kPRow;
    static constexpr int kOffQ = kRing * kEntry;
    static constexpr int kOffP = kOffQ + 2 * kQB;  // two Q tiles (item parity)
    static constexpr int kOffRed = kOffP + kPTiles * kPB;    // 2 x [G][4] floats (after the P^T tiles)
    static constexpr int kOffFlag = kOffRed + 2 * G * 4 * 4;  // 2 x 4 ints
    static constexpr int kMaxList = 96;          // work items of a CTA resolved once into shared memory
    static constexpr int kOffMask = kOffFlag + 32;            // ints: skipped-page mask per K entry, per S^T buffer
    static constexpr int kOBuf = 4;              // items in flight between the softmax and the epilogue
    static constexpr int kOffStats = kOffMask + 32;           // kOBuf x [l, m][G] floats: an item's sums, maxima
    static constexpr int kOffList = kOffStats + kOBuf * 2 * G * 4;  // int4 x 2 per item
    static constexpr int kOffStream = kOffList + kMaxList * 32;   // TcStream of a balanced plan (48 bytes)
    static constexpr int kOffBar = kOffStream + 48;
    // full[R], empty[R], q_full[2], q_empty[2], s_full[2], s_empty[2], p_full[2], p_empty[2], done (QK
    // issuer), done (PV issuer), mask_full[2], o_full[kOBuf], o_empty[kOBuf], stats_full[kOBuf],
    // stats_empty[kOBuf]
    static constexpr int kNumBars = 2 * kRing + 4 + 8 + 2 + 2 + 4 * kOBuf;
    static constexpr int kOffTmem = kOffBar + 8 * kNumBars;
    static constexpr int kSmem = 1024 + kOffTmem + 16;
    static constexpr int kThreads = 384;         // three warpgroups
    static constexpr int kVWarp = 2;             // the V producer (warp 0 produces Q and K)
    static constexpr int kPVWarp = 3;            // issues P.V (warp 1 issues QK)
    static constexpr int kFirstSoftmaxWarp = 4;  // warps 4-7: softmax
    static constexpr int kFirstEpiWarp = 8;      // warps 8-11: epilogue
    // registers per thread after the split (setmaxnreg) of warpgroup 0 (producers, issuers), 1 (softmax,
    // G scores per thread) and 2 (epilogue): 128 x their sum must fit in the launch's 384 x (registers per
    // thread), which the host checks before the first launch
    static constexpr uint32_t kRegsLow = 64, kRegsSoftmax = 248, kRegsEpi = 136;
    // S^T x 2 + O^T x kOBuf, N columns each, rounded up to a power of two
    // S^T x 2 (N columns each) + O^T x kOBuf (kPVN each), rounded up to a power of two
    static constexpr int kTmemNeed = 2 * kN + kOBuf * kPVN;
    static constexpr uint32_t kTmemCols = kTmemNeed <= 64 ? 64 : (kTmemNeed <= 128 ? 128 : (kTmemNeed <= 256 ? 256 : 512));
    static_assert((G == 4 || G == 8 || G == 16 || G == 32) && DH == 128, "instances: g in {4, 8, 16, 32}, Dh = 128");
    static_assert(kPPS * kBoxCols <= 32, "one TMA box per lane");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

struct TcWork {
    int b, kvh, split, item, first, n_local, len, n_pages;
    int n_pieces;  // balanced plan: pieces of the row (CTAs split .. split + n_pieces - 1)
    bool split_mode, bad_len;
    bool planned;  // partial at slot `item` ([item][g][Dh]); else at (row, split) of the grid layout
};

// This CTA's share of a balanced plan (paged_plan_stream_kernel): positions [lo, hi) of the line of
// (sequence, KV head) row spans, the first of which, row0 = b * H_kv + kvh, holds position lo; a row's
// span is its v virtual pages (the fixed cost of a work item), then its real pages.
struct TcStream {
    long long lo, hi, row0, T;
    int G, v;
    int active;  // a balanced plan with positions for this CTA
    int pad;
};

static_assert(sizeof(TcStream) == 48, "shared-memory slot of the stream range");

// (a launch parameter: known before the plan kernel this one depends on has finished)
__device__ __forceinline__ bool tc_is_stream(const DecodeParams& p) { return p.stream_plan != 0; }

__device__ __forceinline__ TcStream tc_stream_range(const DecodeParams& p) {
    TcStream r{0, 0, 0, 0, 0, 0, 0, 0};
    const int G = plan_stream_G(p.plan);
    const int c = blockIdx.x;
    if (c >= G) return r;
    const long long T = plan_stream_T(p.plan);
    const int64_t* pre = plan_stream_prefix(p.plan);
    const int b0 = p.plan[kPlanHdr + 2 * (p.B + 1) + c];
    r.T = T;
    r.G = G;
    r.v = plan_stream_v(p.plan);
    r.lo = T * c / G;
    r.hi = T * (c + 1) / G;
    const long long s0 = pre[b0], d0 = pre[b0 + 1] - s0;
    if (r.hi <= r.lo || d0 <= 0) return r;
    r.row0 = static_cast<long long>(b0) * p.H_kv + (r.lo - p.H_kv * s0) / d0;
    r.active = 1;
    return r;
}

// Piece k of the CTA's range: the real pages of row row0 + k inside [lo, hi). 1: work, 0: none (an empty
// row, or only its virtual pages in range), -1: past the range. A row cut by a range boundary records its
// first CTA (split) and its number of pieces.
__device__ __forceinline__ int tc_stream_piece(const DecodeParams& p, const TcStream& st, int k, int P, TcWork& wk) {
    if (!st.active) return -1;
    const long long row = st.row0 + k;
    const int b = static_cast<int>(row / p.H_kv), kvh = static_cast<int>(row % p.H_kv);
    if (b >= p.B) return -1;
    const int64_t* pre = plan_stream_prefix(p.plan);
    const long long s0 = pre[b], d = pre[b + 1] - s0;
    const long long rs = p.H_kv * s0 + kvh * d;  // the row's span
    if (rs >= st.hi) return -1;
    if (d <= 0) return 0;
    const long long n = d - st.v, r0 = rs + st.v;  // its real pages
    const long long x0 = r0 > st.lo ? r0 : st.lo, x1 = r0 + n < st.hi ? r0 + n : st.hi;
    if (x1 <= x0) return 0;
    wk.b = b;
    wk.kvh = kvh;
    wk.item = 2 * static_cast<int>(blockIdx.x) + (r0 >= st.lo ? 1 : 0);
    wk.first = static_cast<int>(x0 - r0);
    wk.n_local = static_cast<int>(x1 - x0);
    wk.len = p.seq_lens[b];
    wk.n_pages = static_cast<int>(n);
    wk.split_mode = !(x0 == r0 && x1 == r0 + n);
    const int c0 = plan_stream_cta(r0, st.T, st.G);
    wk.split = c0;
    wk.n_pieces = plan_stream_cta(r0 + n - 1, st.T, st.G) - c0 + 1;
    wk.bad_len = false;  // the plan raised it and gave the row no pages
    wk.planned = true;
    return 1;
}

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
    k.planned = p.items != nullptr;
    k.n_pieces = 0;
    return true;
}

__host__ __device__ constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n / 2); }

// A CTA's candidate work items (w = blockIdx.x + k gridDim.x) resolved once by
// one warp into shared memory, so the roles walk them without the dependent
// global loads of tc_work; candidates past the list are resolved on the fly.
struct TcList {
    int4* e;            // [kMaxList][2]: {b, kvh, split, item}, {first, n_local, len, flags}
    int n_list;         // entries held
    int n_cand;         // candidates of a grid or chunked launch (a balanced plan ends at its range)
    const TcStream* st;  // balanced plan: this CTA's range (shared memory), else nullptr
};

// list entry flags (bits 0-4; the row's number of pieces from bit 8)
constexpr int kTcSplit = 1, kTcBad = 2, kTcWork = 4, kTcPlanned = 8, kTcEnd = 16;

__device__ __forceinline__ void tc_list_put(int4* e, int k, const TcWork& wk, int flags) {
    e[2 * k] = make_int4(wk.b, wk.kvh, wk.split, wk.item);
    e[2 * k + 1] = make_int4(wk.first, wk.n_local, wk.len,
                             flags | (wk.split_mode ? kTcSplit : 0) | (wk.bad_len ? kTcBad : 0) |
                                 (wk.planned ? kTcPlanned : 0) | (wk.n_pieces << 8));
}

// One warp: the stream range (balanced plan) and the first candidates, into shared memory.
__device__ __forceinline__ void tc_list_build(const DecodeParams& p, int n_work, int P, int4* e, int max_list,
                                              TcStream* st_out, int lane) {
    const bool stream = tc_is_stream(p);
    TcStream st{0, 0, 0, 0, 0, 0, 0, 0};
    if (stream) st = tc_stream_range(p);  // the same loads in every lane
    if (lane == 0) *st_out = st;
    for (int k = lane; k < max_list; k += 32) {
        TcWork wk{0, 0, 0, 0, 0, 0, 0, 0, 0, false, false, false};
        int flags = 0;
        if (stream) {
            const int got = tc_stream_piece(p, st, k, P, wk);
            flags = got > 0 ? kTcWork : (got < 0 ? kTcEnd : 0);
        } else {
            const int w = blockIdx.x + k * gridDim.x;
            if (w >= n_work) flags = kTcEnd;
            else if (tc_work(p, w, P, wk)) flags = kTcWork;
        }
        tc_list_put(e, k, wk, flags);
    }
}

// Candidate k of this CTA: 1 a work item, 0 none (skip it), -1 past the CTA's last candidate.
__device__ __forceinline__ int tc_get(const DecodeParams& p, const TcList& L, int k, int P, TcWork& wk) {
    if (k < L.n_list) {
        const int4 a = L.e[2 * k], c = L.e[2 * k + 1];
        if (c.w & kTcEnd) return -1;
        if (!(c.w & kTcWork)) return 0;
        wk.b = a.x, wk.kvh = a.y, wk.split = a.z, wk.item = a.w;
        wk.first = c.x, wk.n_local = c.y, wk.len = c.z;
        wk.split_mode = (c.w & kTcSplit) != 0, wk.bad_len = (c.w & kTcBad) != 0, wk.planned = (c.w & kTcPlanned) != 0;
        wk.n_pieces = c.w >> 8;
        wk.n_pages = (wk.len + P - 1) / P;
        return 1;
    }
    if (L.n_list > 0 && (L.e[2 * (L.n_list - 1) + 1].w & kTcEnd)) return -1;
    if (L.st != nullptr) return tc_stream_piece(p, *L.st, k, P, wk);
    if (k >= L.n_cand) return -1;
    return tc_work(p, blockIdx.x + k * gridDim.x, P, wk) ? 1 : 0;
}

// Fused append of the new token (position len - 1) for one of the pools: part 0
// writes the K row, part 1 the V row (each producer warp writes the rows its own
// TMA boxes will read, then fences them against the async proxy).
__device__ __forceinline__ void append_new_token_part(const DecodeParams& p, int b, int kvh, int len, int P,
                                                      int row_bytes, int lane, int part) {
    const int pos = len - 1;
    const int32_t page = p.block_tables[(int64_t)b * p.max_blocks + pos / P];
    if (page >= 0 && page < p.num_pages) {
        const int nch = row_bytes / 16;
        const int64_t dst_row = ((int64_t)page * p.H_kv + kvh) * P + pos % P;
        const int64_t src_row = (int64_t)b * p.H_kv + kvh;
        const uint4* src = static_cast<const uint4*>(part ? p.v_new : p.k_new) + src_row * nch;
        uint4* dst = static_cast<uint4*>(const_cast<void*>(part ? p.v_pages : p.k_pages)) + dst_row * nch;
        for (int c = lane; c < nch; c += 32) dst[c] = src[c];
        fence_proxy_async_global();
    } else if (lane == 0 && part == 0) {
        raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
    }
    __syncwarp();
}

// Per-head reduction over the 32 lanes of a warp of NV values per lane (NV a
// power of two <= 32): halving exchanges (each step ships half of the values)
// until one value is left, then a butterfly. Afterwards the lanes of group
// lane >> (5 - log2 NV) hold the reduction of that head.
template <int NV, bool MAX>
__device__ __forceinline__ float warp_heads_reduce(float (&x)[NV], int lane) {
    constexpr int kL = ilog2(NV);
#pragma unroll
    for (int k = 0; k < kL; ++k) {
        const int off = 16 >> k;
        const int half = NV >> (k + 1);
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? x[i] : x[i + half];
            const float keep = up ? x[i + half] : x[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            x[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    float v = x[0];
#pragma unroll
    for (int off = 16 >> kL; off >= 1; off >>= 1) {
        const float got = __shfl_xor_sync(0xffffffffu, v, off);
        v = MAX ? fmaxf(v, got) : v + got;
    }
    return v;
}

// The same reduction over the four softmax warps (128 threads, named barrier
// 1); every thread receives all NV results. `buf` alternates between calls.
template <int NV, bool MAX>
__device__ __forceinline__ void cta_heads_reduce(float (&x)[NV], float* red, int sw, int lane, int& buf) {
    constexpr int kShift = 5 - ilog2(NV);
    const float v = warp_heads_reduce<NV, MAX>(x, lane);
    float* r = red + buf * NV * 4;
    if ((lane & ((1 << kShift) - 1)) == 0) r[(lane >> kShift) * 4 + sw] = v;
    named_bar_sync(1, 128);
    const float4* r4 = reinterpret_cast<const float4*>(r);
#pragma unroll
    for (int h = 0; h < NV; ++h) {
        const float4 a = r4[h];
        x[h] = MAX ? fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)) : (a.x + a.y) + (a.z + a.w);
    }
    buf ^= 1;
}

// kN consecutive fp32 columns of this thread's lane (16 or 32).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&a)[N]) {
    if constexpr (N == 16) {
        tmem_ld16(taddr, a);
    } else {
        uint32_t lo[16], hi[16];
        tmem_ld16(taddr, lo);
        tmem_ld16(taddr + 16, hi);
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = lo[i], a[16 + i] = hi[i];
    }
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&a)[N]) {
    if constexpr (N == 16) {
        tmem_st16(taddr, a);
    } else {
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) lo[i] = a[i], hi[i] = a[16 + i];
        tmem_st16(taddr, lo);
        tmem_st16(taddr + 16, hi);
    }
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

template <int KT, int DH, int P, int G>
__global__ void __launch_bounds__(384, 1)
    paged_decode_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_q,
                           int n_work) {
    using C = TcCfg<DH, P, G>;
    constexpr bool kBF16 = KT == KV_DTYPE_BF16;
    constexpr int N = C::kN;
    constexpr uint32_t kIdescQK = idesc_f16(kBF16, 128, N, false, false);
    constexpr uint32_t kIdescPV = idesc_f16(kBF16, 128, C::kPVN, true, true);
    extern __shared__ __align__(1024) unsigned char smem_raw[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
        prefetch_tmap(&tmap_q);
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
    // Q tile, its barriers and the O^T accumulator are double-buffered by item parity, so the producer
    // loads the next item's Q and pages, and its first P.V starts, while this item finishes
    const uint32_t bq0 = bar0 + 8u * (2 * C::kRing);
    auto q_full = [&](int i) { return bq0 + 8u * i; };
    auto q_empty = [&](int i) { return bq0 + 16u + 8u * i; };
    const uint32_t bs0 = bq0 + 32u;
    auto s_full = [&](int i) { return bs0 + 8u * i; };
    auto s_empty = [&](int i) { return bs0 + 16u + 8u * i; };
    // P^T is double-buffered (stage J in buffer J & 1): the softmax of stage J writes while P.V(J - 1) runs
    auto p_full = [&](int i) { return bs0 + 32u + 8u * i; };
    auto p_empty = [&](int i) { return bs0 + 48u + 8u * i; };
    const uint32_t done_qk = bs0 + 64u;
    const uint32_t done_pv = bs0 + 72u;
    // the skipped-page mask of a stage travels producer -> K entry word -> QK issuer -> S^T buffer word, the
    // last hop announced on mask_full (the softmax needs it before the V entry lands)
    auto mask_full = [&](int i) { return bs0 + 80u + 8u * i; };
    // O^T and the item's row sums and reference maxima (softmax -> epilogue warps) rotate over kOBuf items,
    // so a run of short items does not wait for the epilogue of the one before last
    const uint32_t bo0 = bs0 + 96u;
    auto o_full = [&](int i) { return bo0 + 8u * (i % C::kOBuf); };
    auto o_empty = [&](int i) { return bo0 + 8u * (C::kOBuf + i % C::kOBuf); };
    auto stats_full = [&](int i) { return bo0 + 8u * (2 * C::kOBuf + i % C::kOBuf); };
    auto stats_empty = [&](int i) { return bo0 + 8u * (3 * C::kOBuf + i % C::kOBuf); };
    auto oph = [](int i) { return static_cast<uint32_t>((i / C::kOBuf) & 1); };  // phase of item i's slot
    volatile int* kmask = reinterpret_cast<volatile int*>(smem + C::kOffMask);      // [kKSlots]
    volatile int* smask = reinterpret_cast<volatile int*>(smem + C::kOffMask + 16);  // [2]
    float* stats = reinterpret_cast<float*>(smem + C::kOffStats);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmem);

    if (threadIdx.x == 0) {
        for (int e = 0; e < C::kRing; ++e) {
            mbar_init(full(e), 1);
            mbar_init(empty(e), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(q_full(i), 1);
            mbar_init(q_empty(i), 1);
        }
        for (int i = 0; i < C::kOBuf; ++i) {
            mbar_init(o_full(i), 1);
            mbar_init(o_empty(i), 4);
            mbar_init(stats_full(i), 4);
            mbar_init(stats_empty(i), 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(s_full(i), 1);
            mbar_init(s_empty(i), 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(p_full(i), 4);
            mbar_init(p_empty(i), 1);
        }
        mbar_init(done_qk, 1);
        mbar_init(done_pv, 1);
        for (int i = 0; i < 2; ++i) mbar_init(mask_full(i), 1);
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
    if constexpr (G < N) {
        // Q rows G .. N-1 are MMA padding: zero once (the TMA box writes rows 0 .. G-1 only)
        for (int i = threadIdx.x; i < C::kBoxCols * (N - G) * 8; i += blockDim.x) {
            const int bb = i / ((N - G) * 8), rest = i % ((N - G) * 8);
            sts128_zero(sbase + C::kOffQ + bb * C::kQRowsB + (G + rest / 8) * 128 + (rest % 8) * 16);
        }
        fence_proxy_async_smem();
    }
    // the setup above touches only this CTA's shared and tensor memory, so it overlaps the kernel this
    // one depends on (programmatic launch); everything below may read what that kernel wrote
    grid_dependency_wait();
    if (threadIdx.x == 0) grid_launch_dependents();
    if (warp == 1) tc_list_build(p, n_work, P, list_e, L.n_list, st_smem, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem;           // S^T buffers: columns [0, 2N)
    auto tO = [&](int i) { return tmem + 2 * N + (i % C::kOBuf) * C::kPVN; };  // O^T of item i
    const uint32_t ring = sbase;
    auto sQ = [&](int i) { return sbase + C::kOffQ + i * C::kQB; };
    const uint32_t sP = sbase + C::kOffP;
    // P^T of stage j: the stacked tile, or the hi tile with the lo tile right after it
    auto sPt = [&](uint32_t j) { return sP + (j & 1) * (C::kPTiles / 2) * C::kPB; };

    // the register split sits at the top of each warpgroup's branch, so every code path after it is
    // compiled for its own budget
    if (warp < C::kFirstSoftmaxWarp) {
    regs_dec<C::kRegsLow>();
    if (warp == 0 || warp == C::kVWarp) {
        // ------------------------------------------------------------ producers
        // Two warps issue the TMA boxes, one the K entries (and Q), the other the V entries: each
        // producer's boxes are handled in order, so two streams keep more of them moving.
        const int half = warp == 0 ? 0 : 1;
        bool ok = true;
        uint32_t Jp = 0;  // stages issued (all items)
        int fills = 0;
        int item_i = 0;
        for (int k = 0; ok; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0 || wk.n_local <= 0) continue;
            if (p.k_new != nullptr && wk.first + wk.n_local == wk.n_pages)
                append_new_token_part(p, wk.b, wk.kvh, wk.len, P, DH * 2, lane, half);
            if (half == 0 && lane == 0) {
                if (item_i > 1 && !mbar_wait_bounded(q_empty(item_i & 1), ((item_i >> 1) - 1) & 1, kWaitLimitNs)) {
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                    ok = false;
                } else {
                    mbar_arrive_expect_tx(q_full(item_i & 1), C::kBoxCols * G * 128);
#pragma unroll
                    for (int bb = 0; bb < C::kBoxCols; ++bb)
                        tma_load_2d(sQ(item_i & 1) + bb * C::kQRowsB, &tmap_q, bb * 64, wk.b * p.H_q + wk.kvh * G,
                                    q_full(item_i & 1));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            ++item_i;
            const int32_t* row = p.block_tables + (int64_t)wk.b * p.max_blocks + wk.first;
            int tab_cur = lane < wk.n_local ? row[lane] : -1, tab_nxt = -1;
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            for (int j = 0; j < n_st && ok; ++j, ++Jp) {
                const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                // block-table entries come 32 at a time, one per lane, the next 32 fetched while these are used
                // (stages never straddle a group: 32 is a multiple of the pages per stage)
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
                const int box_page = lane / C::kBoxCols, bb = lane % C::kBoxCols;
                const int pgl = __shfl_sync(0xffffffffu, pg, box_page & 31);
                {
                    const int e = half ? vslot(Jp) : kslot(Jp);
                    const uint32_t use = half ? Jp / C::kVSlots : Jp / C::kKSlots;  // earlier fills of the entry
                    if (lane == 0) {
                        if (use > 0 && !mbar_wait_bounded(empty(e), (use - 1) & 1, kWaitLimitNs)) {
                            raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                            ok = false;
                        } else {
                            if (half == 0) kmask[e] = static_cast<int>(~gmask & ((1u << np) - 1u));
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
                    fills = Jp + 1;
                }
            }
        }
        if (lane == 0) {  // let every copy in flight land before the CTA exits
            const int slots = half ? C::kVSlots : C::kKSlots;
            for (int j = max(0, fills - slots); j < fills; ++j)
                if (!mbar_wait_bounded(full(half ? vslot(j) : kslot(j)), half ? vphase(j) : kphase(j), kWaitLimitNs))
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
            if (half == 0)
                for (int i = item_i > 2 ? item_i - 2 : 0; i < item_i; ++i)
                    if (!mbar_wait_bounded(q_full(i & 1), (i >> 1) & 1, kWaitLimitNs))
                        raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------------------ MMA issue
        // Warp 1 issues the score products QK(j) as soon as K(j) has landed and an S^T buffer is free;
        // the P.V warp issues P.V(j) once the softmax has written P^T(j). Neither waits on the other's
        // barriers, so QK runs up to two stages ahead of the softmax.
        const bool qk = warp == 1;
        if (lane == 0) {
            bool ok = true;
            uint32_t J = 0;      // stages of the earlier items and this one
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
                        const int e = kslot(J);
                        const int sb = J & 1;
                        if (!wait(full(e), kphase(J))) break;
                        const int bad = kmask[e];
                        if (J >= 2 && !wait(s_empty(sb), ((J >> 1) - 1) & 1)) break;
                        tc_fence_after();
                        const uint32_t sK = ring + e * C::kEntry;
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk) {
                            const uint32_t koff = (kk >> 2) * C::kBoxB + (kk & 3) * 32;
                            const uint32_t qoff = (kk >> 2) * C::kQRowsB + (kk & 3) * 32;
                            umma_ss(tS + sb * N, smem_desc(sK + koff, 16, 1024, kSwz128),
                                    smem_desc(sQ(item_i & 1) + qoff, 16, 1024, kSwz128), kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(s_full(sb));
                        smask[sb] = bad;  // S^T buffer sb is free (s_empty above), so is its mask word
                        mbar_arrive(mask_full(sb));
                        umma_commit(empty(e));
                        if (j == n_st - 1) umma_commit(q_empty(item_i & 1));
                    }
                } else {
                    for (int j = 0; j < n_st; ++j, ++J) {
                        const int e = vslot(J);
                        if (!wait(full(e), vphase(J))) break;
                        if (!wait(p_full(J & 1), (J >> 1) & 1)) break;
                        if (j == 0 && item_i >= C::kOBuf && !wait(o_empty(item_i), oph(item_i) ^ 1u)) break;
                        tc_fence_after();
                        const uint32_t sV = ring + e * C::kEntry;
#pragma unroll
                        for (int kk = 0; kk < C::kTP / 16; ++kk) {
                            const uint64_t a = smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128);
                            umma_ss(tO(item_i), a, smem_desc(sPt(J) + kk * 16 * C::kPRow, C::kPB, C::kPAtom, C::kPSwz),
                                    kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                        }
                        if constexpr (!C::kStackP) {
#pragma unroll
                            for (int kk = 0; kk < C::kTP / 16; ++kk) {
                                const uint64_t a = smem_desc(sV + kk * 16 * 128, C::kBoxB, 1024, kSwz128);
                                umma_ss(tO(item_i), a,
                                        smem_desc(sPt(J) + C::kPB + kk * 16 * C::kPRow, C::kPB, C::kPAtom, C::kPSwz),
                                        kIdescPV, 1u);
                            }
                        }
                        umma_commit(empty(e));
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
        // Named barrier 1 (these 128 threads) is only ever reached by all four warps together: a
        // failed wait is shared at the next flag exchange and every warp then stops at once.
        const int sw = warp - C::kFirstSoftmaxWarp;  // softmax warp 0..3
        const int quarter = warp & 3;      // tensor-memory lane quarter of this warp
        const int r = quarter * 32 + lane;  // token row of S^T, dimension row of O^T
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        float* red = reinterpret_cast<float*>(smem + C::kOffRed);
        volatile int* flags = reinterpret_cast<volatile int*>(smem + C::kOffFlag);
        int rbuf = 0, fbuf = 0;
        bool ok = true;  // equal in the four warps at every flag exchange
        uint32_t J = 0;
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
        for (int k = 0;; ++k) {
            TcWork wk;
            const int got = tc_get(p, L, k, P, wk);
            if (got < 0) break;
            if (got == 0 || wk.n_local <= 0 || !ok) continue;  // the epilogue warps zero such rows
            const int n_st = (wk.n_local + C::kPPS - 1) / C::kPPS;
            float m_ref[G], lp[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY, lp[h] = 0.f;
            const int pr = r / P;  // page of row r within a stage
            for (int j = 0; j < n_st; ++j) {
                bool okl = ok;
                const int sb = J & 1;
                int bad = -1;
                float s[G];
#pragma unroll
                for (int h = 0; h < G; ++h) s[h] = -INFINITY;
                if (wait(okl, s_full(sb), (J >> 1) & 1)) {
                    tc_fence_after();
                    uint32_t a[N];
                    tmem_ld_cols<N>(tS + sb * N + lane_addr, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < G; ++h) s[h] = __uint_as_float(a[h]);
                    tc_fence_before();
                    // the stage's skipped-page mask, read before S^T buffer sb (and its mask word) is released
                    if (wait(okl, mask_full(sb), (J >> 1) & 1)) bad = smask[sb];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(s_empty(sb));
                }
                // token row r of the stage: inside the sequence, on a page of this stage that was loaded
                const int ev = vslot(J);
                const int np = min(C::kPPS, wk.n_local - j * C::kPPS);
                const bool valid = okl && (wk.first + j * C::kPPS) * P + r < wk.len && pr < np && !((bad >> pr) & 1);
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
                    for (int hf = 0; hf < C::kPVN / N; ++hf) {  // (stacked: the hi and the residual parts)
                        uint32_t a[N];
                        tmem_ld_cols<N>(tO(item_i) + hf * N + lane_addr, a);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < G; ++h) a[h] = __float_as_uint(__uint_as_float(a[h]) * alpha[h]);
                        tmem_st_cols<N>(tO(item_i) + hf * N + lane_addr, a);
                    }
                    tmem_wait_st();
                }
                // probabilities -> P^T row r (hi and residual lo; padding heads are zero), swizzled rows
                uint32_t hi[N / 2], lo[N / 2];
#pragma unroll
                for (int i = 0; i < N / 2; ++i) {
                    if (2 * i < G) {
                        const float p0 = s[2 * i] == -INFINITY ? 0.f : exp2f(s[2 * i] - m_ref[2 * i]);
                        const float p1 = s[2 * i + 1] == -INFINITY ? 0.f : exp2f(s[2 * i + 1] - m_ref[2 * i + 1]);
                        lp[2 * i] += p0;
                        lp[2 * i + 1] += p1;
                        pack2_split_fast<kBF16>(p0, p1, hi[i], lo[i]);
                    } else {
                        hi[i] = lo[i] = 0u;
                    }
                }
#pragma unroll
                for (int c = 0; c < N / 8; ++c) {
                    // 16-byte chunks of the row (stacked: c hi, c + N / 8 lo; else chunk c of each tile),
                    // placed as the MN-major swizzle of rows of kPRow bytes expects
                    const uint32_t sw = C::kPRow == 32 ? ((r >> 2) & 1) : (C::kPRow == 64 ? ((r >> 1) & 3) : (r & 7));
                    const uint32_t row = sPt(J) + r * C::kPRow;
                    const uint32_t lo_at = C::kStackP ? row + ((((uint32_t)c + N / 8) ^ sw) << 4)
                                                      : row + C::kPB + (((uint32_t)c ^ sw) << 4);
                    sts128(row + (((uint32_t)c ^ sw) << 4), hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                    sts128(lo_at, lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                }
                // a masked token's V row may hold stale bytes (even NaN): zero it before P.V, once the V entry
                // has landed (only warps with such a row wait for it; the P.V issuer waits for every entry)
                if (__any_sync(0xffffffffu, !valid)) {
                    if (!wait(okl, full(ev), vphase(J))) {
                        ok = false;  // the next flag exchange stops every warp
                        ++J;
                        continue;
                    }
                    if (!valid) {
                        const uint32_t vrow = ring + ev * C::kEntry + r * 128;
#pragma unroll
                        for (int bb = 0; bb < C::kBoxCols; ++bb)
#pragma unroll
                            for (int c = 0; c < 8; ++c) sts128_zero(vrow + bb * C::kBoxB + c * 16);
                    }
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
    } else {
        regs_dec<C::kRegsEpi>();
        // ------------------------------------------------------------ epilogue
        // Row r of O^T of each item (once its last P.V has completed) over the CTA's row sums, or kept
        // as a partial (u, m, l) for the combine kernel; the softmax warps meanwhile go on with the next
        // item. Frees O^T and the statistics slot for item i + 2.
        const int quarter = warp & 3;       // tensor-memory lane quarter of this warp
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
                ok = false;  // an earlier stage failed: this and the later rows are zeroed
                zero_rows(wk);
                continue;
            }
            tc_fence_after();
            float o[G];
            {
                uint32_t a[N];
                tmem_ld_cols<N>(tO(item_i) + lane_addr, a);
                if constexpr (C::kStackP) {
                    uint32_t b2[N];
                    tmem_ld_cols<N>(tO(item_i) + N + lane_addr, b2);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < G; ++h) o[h] = __uint_as_float(a[h]) + __uint_as_float(b2[h]);
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < G; ++h) o[h] = __uint_as_float(a[h]);
                }
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
            const int64_t hq0 = (int64_t)wk.b * p.H_q + (int64_t)wk.kvh * G;
            if (!wk.split_mode) {
#pragma unroll
                for (int h = 0; h < G; ++h) p.out[(hq0 + h) * DH + r] = l[h] > 0.f ? o[h] / l[h] : 0.f;
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const int64_t ps = wk.planned ? (int64_t)wk.item * G + h : (hq0 + h) * p.num_splits + wk.split;
                    p.part_u[ps * DH + r] = o[h];
                    if (r == 0) p.part_ml[ps] = make_float2(m[h], l[h]);
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
