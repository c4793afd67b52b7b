// Paged decode attention on the tensor cores (bf16 / fp16 / E4M3 K/V), sm_100a.
// One kernel template serves four uses: single-token decode (the default),
// E4M3 K/V (codes converted to f16 pairs in registers, two pages per stage),
// multi-token query (chunked prefill: MMA rows are (token, head) pairs with a
// per-row causal limit), and the fused rotate + append + decode step.
//
// Same contract and the same online (m, l, u) merge as decode_kernel.cuh
// ("07｜KV Cache、FlashAttention与PagedAttention的内部过程", Q027; attention
// formula of "04. 注意力与 KV 缓存" / "03. KV Cache：用显存换计算"), with the
// two small contractions of every page done by warp-level MMA so each
// (page, head) chunk costs ~100 instructions instead of ~800 on the CUDA
// cores:
//   S[16 x P]  = Q[16 heads x Dh] . K_page^T      (m16n8k16, k over Dh)
//   O[16 x Dh] += P[16 x P] . V_page               (m16n8k16, k over tokens;
//                                                   P as a 16-bit pair + residual)
// The GQA group is the M dimension (rows >= g are zero padding), so the S
// accumulator fragment is, element for element, the A fragment of the second
// product: probabilities never leave registers.
//
// Data movement: the producer warp issues 2-D TMA tile loads (no multicast)
// of each (page, head) chunk of K and V, Dh/64 boxes of P rows x 128 bytes
// with 128-byte swizzle, into a ring of NS stages; ldmatrix then reads rows
// of 8 tokens without bank conflicts. Row max uses 2 shuffles; the output
// rescale is lazy: the reference max of a row moves only when a score exceeds
// it by more than 2^8 (exact: o = u / l for any common reference).
// Masked tail tokens (t >= len) get p = 0 and their V rows are zeroed in
// shared memory first, so stale values (even NaN) in unused slots never reach
// the output.
#pragma once

#include <cuda.h>

#include "decode_kernel.cuh"
#include "fp8.cuh"
#include "rope.cuh"

#ifndef KVP_MMA_STAGE_BUDGET
#define KVP_MMA_STAGE_BUDGET (96 * 1024)
#endif

namespace kvp {

// Fused rotary embedding + append of the new token (position len - 1): the
// rotated k row and the v row go to their slot exactly as kv_rope_append
// writes them (same fp32 operations, same rounding). Lane l < Dh/16 rotates
// the vector pair (l, l + Dh/16) (split halves) or (2l, 2l + 1)
// (interleaved) of the k row; the next Dh/8 lanes copy the v row. Called by
// one whole warp before it loads the page.
template <int DT>
__device__ __forceinline__ void append_new_token_rope(const DecodeParams& p, int b, int kvh, int len, int P, int DH,
                                                      int lane) {
    using V = RopeVec<DT>;
    constexpr int N = V::kN;
    const int pos = len - 1;
    const int32_t page = p.block_tables[(int64_t)b * p.max_blocks + pos / P];
    if (pos < 0 || pos >= p.max_pos) {
        if (lane == 0) raise_err(p.err, KV_DEV_ERR_POSITION);
    } else if (page >= 0 && page < p.num_pages) {
        const int vpr = DH / N, upr = vpr / 2;
        const int64_t dst_row = ((int64_t)page * p.H_kv + kvh) * P + pos % P;
        const int64_t src_row = (int64_t)b * p.H_kv + kvh;
        if (lane < upr) {
            const uint4* src = static_cast<const uint4*>(p.k_new) + src_row * vpr;
            uint4* dst = static_cast<uint4*>(const_cast<void*>(p.k_pages)) + dst_row * vpr;
            const int va = p.rope_style == KV_ROPE_HALF ? lane : 2 * lane;
            const int vb = p.rope_style == KV_ROPE_HALF ? lane + upr : 2 * lane + 1;
            float xa[N], xb[N];
            V::load(src[va], xa);
            V::load(src[vb], xb);
            const float* crow = p.cos_sin + (int64_t)pos * DH;
            const int k0 = lane * N;
#pragma unroll
            for (int i = 0; i < N; ++i) {
                if (p.rope_style == KV_ROPE_HALF) {
                    rotate_pair(xa[i], xb[i], crow[k0 + i], crow[DH / 2 + k0 + i]);
                } else if (i < N / 2) {
                    rotate_pair(xa[2 * i], xa[2 * i + 1], crow[k0 + i], crow[DH / 2 + k0 + i]);
                    rotate_pair(xb[2 * i], xb[2 * i + 1], crow[k0 + N / 2 + i], crow[DH / 2 + k0 + N / 2 + i]);
                }
            }
            dst[va] = V::store(xa);
            dst[vb] = V::store(xb);
        } else if (lane < upr + vpr) {
            const int c = lane - upr;
            static_cast<uint4*>(const_cast<void*>(p.v_pages))[dst_row * vpr + c] =
                static_cast<const uint4*>(p.v_new)[src_row * vpr + c];
        }
        fence_proxy_async_global();
    } else if (lane == 0) {
        raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
    }
    __syncwarp();
}

// EB: bytes per K/V element (2: bf16 / fp16; 1: E4M3). A token row of Dh
// elements is loaded as boxes of at most 128 bytes (rows of 128 bytes use the
// 128-byte swizzle, rows of 64 bytes -- E4M3 at Dh = 64 -- the 64-byte one).
// PPS pages share one pipeline stage (tokens per stage TP = P * PPS): the
// consumer then works on TP tokens per barrier round trip.
template <int DH, int P, int NW, int EB, int PPS>
struct MmaCfg {
    static constexpr int kTP = P * PPS;                          // tokens per stage
    static constexpr int kRowB = DH * EB;                        // bytes per token row
    static constexpr int kBoxInner = kRowB < 128 ? kRowB : 128;  // bytes per box row
    static constexpr int kBoxElems = kBoxInner / EB;
    static constexpr int kBoxes = kRowB / kBoxInner;             // boxes per token row
    static constexpr int kPageB = P * kBoxInner;                 // bytes of one page's box (P rows)
    static constexpr int kBoxB = kTP * kBoxInner;                // bytes per box column of a stage
    static constexpr int kChunk = kTP * kRowB;                   // K (or V) of one stage
    static constexpr int kStage = 2 * kChunk;                    // K + V
    static constexpr int kKSteps = DH / 16;                      // QK k-steps
    static constexpr int kNT = kTP / 8;                          // token n-tiles of S
    static constexpr int kPK = kTP / 16;                         // PV k-steps
    static constexpr int kOT = DH / 8;                           // dim n-tiles of O
    static constexpr int kStageBudget = KVP_MMA_STAGE_BUDGET;
    // Stage i % NS is drained by page-warp i % WP (WP divides NW): NS must be
    // a multiple of NW so each stage always goes to the same warp.
    static constexpr int kNS0 = (kStageBudget / kStage) / NW * NW;
    static constexpr int kNS = kNS0 > 16 ? 16 : (kNS0 < NW ? NW : kNS0);
    static constexpr int kMergeB = NW * 16 * (DH + 2) * 4;  // per-warp (m, l, O) rows, aliased on the stages
    static constexpr int kRing = kNS * kStage;
    static constexpr int kOffBars = kRing > kMergeB ? kRing : kMergeB;
    static constexpr int kOffTag = kOffBars + 16 * kNS;
    static constexpr int kSmem = 1024 + kOffTag + 4 * kNS;  // + slack to align the ring to 1024 bytes
    static constexpr int kThreads = 32 * (NW + 1);
    static_assert(DH % 64 == 0 && P % 16 == 0, "shape");
    static_assert(kRowB % kBoxInner == 0 && (kBoxInner == 128 || kBoxInner == 64), "box rows");
    static_assert(kNS % NW == 0, "stage ring must be a multiple of the page-warps");
};

// Byte offset of 16-byte chunk c of row t in a box whose rows are kBoxInner
// bytes, as the TMA swizzle placed it (128-byte: chunk ^ row % 8; 64-byte:
// chunk ^ (row / 2) % 4).
template <int kBoxInner>
__device__ __forceinline__ uint32_t swz(int t, int c) {
    if constexpr (kBoxInner == 128)
        return t * 128 + (((c & 7) ^ (t & 7)) << 4);
    else
        return t * 64 + (((c & 3) ^ ((t >> 1) & 3)) << 4);
}

// KT: K/V storage type (bf16, fp16 or E4M3); QT: q's type (equal to KT for
// 16-bit K/V; bf16 or fp16 for E4M3, whose products run in f16). LO: the GQA
// group has at most 8 heads (one head slice, rows 8..15 are padding), so each
// row's probability residual rides in row r + 8. QM: multi-token query (a
// chunk of new tokens per sequence): the MMA rows are (token, head) pairs of
// q_tile chunk tokens, and row i of the chunk sees keys up to its own
// position (causal within the chunk).
template <int KT, int QT, int DH, int P, int NW, bool LO, int PPS, bool QM>
__global__ void __launch_bounds__(32 * (NW + 1), 2)
    paged_decode_mma_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                            const __grid_constant__ CUtensorMap tmap_v) {
    constexpr bool kFP8 = KT == KV_DTYPE_FP8_E4M3;
    using C = MmaCfg<DH, P, NW, kFP8 ? 1 : 2, PPS>;
    constexpr bool kBF16 = KT == KV_DTYPE_BF16;  // MMA operand type: bf16, else f16
    extern __shared__ __align__(1024) unsigned char smem_raw[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    grid_dependency_wait();  // inputs (and a plan) may come from the previous kernel in the stream
    if (threadIdx.x == 0) grid_launch_dependents();

    // Work of this CTA: (split, kvh, b) from the grid, or a planned chunk; for a
    // multi-token query (tile, kvh, b) with the tile's chunk tokens t0 .. t0 + nt - 1.
    int split, kvh, b, item = 0, chunk_pages;
    int qs0 = 0, n_q = 1, t0 = 0, nt = 1;
    if constexpr (QM) {
        split = 0;
        kvh = blockIdx.y;
        b = blockIdx.z;
        chunk_pages = 0;
        qs0 = p.q_start[b];
        n_q = p.q_start[b + 1] - qs0;
        t0 = blockIdx.x * p.q_tile;
        if (t0 >= n_q) return;
        nt = min(p.q_tile, n_q - t0);
    } else if (p.items != nullptr) {
        const int4 it = p.items[blockIdx.x];
        if (it.x < 0) return;
        b = it.x;
        kvh = it.y;
        split = it.z;
        item = it.w;
        chunk_pages = p.plan[0];
    } else {
        split = blockIdx.x;
        kvh = blockIdx.y;
        b = blockIdx.z;
        chunk_pages = p.pages_per_split;
    }
    const bool chunked = !QM && (p.items != nullptr || p.num_splits > 1);
    // The producer's first 32 block-table entries do not depend on the length:
    // load them alongside it.
    const int first = chunked ? split * chunk_pages : 0;
    int tab0 = 0;
    if (warp == 0 && first + lane < p.max_blocks) tab0 = p.block_tables[(int64_t)b * p.max_blocks + first + lane];
    int len = p.seq_lens[b];
    if (len < 0 || len > p.max_blocks * P || (QM && n_q > len)) {
        if (threadIdx.x == 0 && split == 0 && p.items == nullptr && t0 == 0) raise_err(p.err, KV_DEV_ERR_SEQ_LEN);
        len = 0;
    }
    // keys of this CTA: the whole sequence, or (multi-token) up to the tile's last position
    const int key_end = QM ? (len > 0 ? len - n_q + t0 + nt : 0) : len;
    const int n_pages = (key_end + P - 1) / P;
    const int n_local = chunked ? min(chunk_pages, n_pages - first) : n_pages;
    // Partials are needed when the row has more than one chunk.
    const bool split_mode = p.items != nullptr ? n_pages > chunk_pages : p.num_splits > 1;
    if (n_local <= 0) {
        if constexpr (QM) {
            for (int e = threadIdx.x; e < nt * p.g * DH; e += blockDim.x) {
                const int rr = e / DH;
                p.out[((int64_t)(qs0 + t0 + rr / p.g) * p.H_q + (int64_t)kvh * p.g + rr % p.g) * DH + e % DH] = 0.f;
            }
        } else if (!split_mode) {
            for (int e = threadIdx.x; e < p.g * DH; e += blockDim.x)
                p.out[((int64_t)b * p.H_q + (int64_t)kvh * p.g) * DH + e] = 0.f;
        }
        return;
    }

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    const uint32_t full_bar = sbase + C::kOffBars;
    const uint32_t empty_bar = full_bar + 8 * C::kNS;
    volatile int* stage_tag = reinterpret_cast<volatile int*>(smem + C::kOffTag);

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
        if constexpr (!kFP8 && !QM) {
            if (p.k_new != nullptr && first + n_local == n_pages) {
                if (p.cos_sin != nullptr)
                    append_new_token_rope<KT>(p, b, kvh, len, P, DH, lane);
                else
                    append_new_token(p, b, kvh, len, P, DH * 2, lane);
            }
        }
        const int32_t* row = p.block_tables + (int64_t)b * p.max_blocks + first;
        const int n_st = (n_local + PPS - 1) / PPS;  // stages of this CTA
        bool ok = true;
        int issued = 0;
        // A group of kGrp stages per step: lane l < kGrp claims stage base + l
        // (bounded wait on its empty barrier, tag, expect_tx for its pages),
        // then every lane issues one TMA box: box l % kBPS of stage l / kBPS.
        constexpr int kBPS = PPS * 2 * C::kBoxes;  // boxes per stage (K and V of each page)
        constexpr int kGrp0 = 32 / kBPS;
        // groups of at most 4 stages: a group is issued only once all of its
        // stages are free, so large groups leave the ring partly idle (8B-shaped
        // layer: 4 -> 0.85 of peak, 8 -> 0.82, 2 -> 0.80; E4M3: 0.62 / 0.59 / 0.57)
        constexpr int kGrpMax = kGrp0 < 4 ? kGrp0 : 4;
        constexpr int kGrp = kGrpMax >= 16 ? 16 : kGrpMax >= 8 ? 8 : kGrpMax >= 4 ? 4 : kGrpMax >= 2 ? 2 : 1;
        static_assert(32 % (kGrp * PPS) == 0, "page groups must tile the 32-entry table window");
        int tab = 0;  // block-table entry of page (first page of the group & ~31) + lane
        for (int base = 0; base < n_st; base += kGrp) {
            const int pbase = base * PPS;
            if ((pbase & 31) == 0) tab = pbase == 0 ? tab0 : ((pbase + lane < n_local) ? row[pbase + lane] : 0);
            const int cnt = min(kGrp, n_st - base);
            int pg[PPS];
#pragma unroll
            for (int j = 0; j < PPS; ++j) pg[j] = __shfl_sync(0xffffffffu, tab, ((base + lane) * PPS + j) & 31);
            bool valid = false;
            if (lane < cnt) {
                const int i = base + lane;
                const int s = i % C::kNS;
                const int np = min(PPS, n_local - i * PPS);  // pages in this stage
                bool in_range = true;
#pragma unroll
                for (int j = 0; j < PPS; ++j)
                    if (j < np) in_range = in_range && pg[j] >= 0 && pg[j] < p.num_pages;
                if (i >= C::kNS && !mbar_wait_bounded(empty_bar + 8 * s, ((i / C::kNS) - 1) & 1, kWaitLimitNs)) {
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                    ok = false;
                } else if (in_range) {
                    valid = true;
                    stage_tag[s] = i;
                    mbar_arrive_expect_tx(full_bar + 8 * s, np * 2 * C::kBoxes * C::kPageB);
                } else {
                    raise_err(p.err, KV_DEV_ERR_PAGE_RANGE);
                    stage_tag[s] = -1 - i;
                    mbar_arrive(full_bar + 8 * s);
                }
            }
            if (!__all_sync(0xffffffffu, ok)) break;
            const unsigned vmask = __ballot_sync(0xffffffffu, valid);
            const int pl = lane / kBPS, bx = lane % kBPS;
            const int j = bx / (2 * C::kBoxes);          // page of the stage
            const bool is_v = ((bx / C::kBoxes) & 1) != 0;
            const int bb = bx % C::kBoxes;               // box of the token row
            const int page_idx = (base + pl) * PPS + j;  // page of this CTA's range
            const int pgl = __shfl_sync(0xffffffffu, tab, page_idx & 31);
            if (pl < cnt && ((vmask >> pl) & 1u) && page_idx < n_local) {
                const int s = (base + pl) % C::kNS;
                const uint32_t dst =
                    sbase + s * C::kStage + (is_v ? C::kChunk : 0) + bb * C::kBoxB + j * C::kPageB;
                tma_load_2d(dst, is_v ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k),
                            bb * C::kBoxElems, (pgl * p.H_kv + kvh) * P, full_bar + 8 * s);
            }
            issued = base + cnt;
        }
        if (lane == 0) {
            for (int i = max(0, issued - C::kNS); i < issued; ++i)
                if (!mbar_wait_bounded(full_bar + 8 * (i % C::kNS), (i / C::kNS) & 1, kWaitLimitNs))
                    raise_err(p.err, KV_DEV_ERR_TIMEOUT);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int cw = warp - 1;
    const int hs = cw % p.HS;  // 16-row head slice
    const int wp = cw / p.HS;
    const bool active = wp < p.WP;
    const int quad = lane & 3;   // column pair within a fragment
    const int r0 = lane >> 2;    // fragment rows r0 and r0 + 8
    const int rows = min(16, nt * p.g - hs * 16);  // real rows (heads, or token-head pairs) in this slice
    constexpr bool lo_rows = LO;                    // padding rows 8..15 carry the P residual
    const int hbase = kvh * p.g + hs * 16;         // query head of row 0 (single-token query)
    // Global q row of slice row r, and (multi-token) the first key position row r may not see.
    auto q_row = [&](int r) -> int64_t {
        if constexpr (QM) {
            const int rr = hs * 16 + r;
            return (int64_t)(qs0 + t0 + rr / p.g) * p.H_q + (int64_t)kvh * p.g + rr % p.g;
        } else {
            return (int64_t)b * p.H_q + hbase + r;
        }
    };
    int key_lim[2] = {0x7fffffff, 0x7fffffff};
    if constexpr (QM) {
#pragma unroll
        for (int h = 0; h < 2; ++h) key_lim[h] = len - n_q + t0 + (hs * 16 + r0 + 8 * h) / p.g + 1;
    }

    // Q as the A operand of S = Q K^T: rows = heads, k = dims (pairs of elements per register).
    uint32_t qa[C::kKSteps][4];
    {
        const uint32_t* q32 = static_cast<const uint32_t*>(p.q);
#pragma unroll
        for (int kk = 0; kk < C::kKSteps; ++kk) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = r0 + 8 * rr;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    // 16-bit K/V: k-step kk covers dims kk*16 .. +15 in ldmatrix order. E4M3: the
                    // thread's K words hold dims quad*Dh/4 + 4*kk .. +3, so its q pairs follow them.
                    const int d = kFP8 ? quad * (DH / 4) + 4 * kk + 2 * ch : kk * 16 + ch * 8 + 2 * quad;
                    uint32_t v = (r < rows) ? q32[(q_row(r) * DH + d) >> 1] : 0u;
                    if constexpr (kFP8 && QT == KV_DTYPE_BF16)  // bf16 q -> f16 operands (exact in f16's range)
                        v = pack2_satfinite_f16(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
                    qa[kk][rr + 2 * ch] = v;
                }
            }
        }
    }

    // Fused rotary embedding of q at position len - 1, with the same fp32 operations and rounding as
    // kv_rope_append. In the fragment a register holds dims (d, d + 1), d = kk*16 + ch*8 + 2*quad; the
    // split-halves partner d + Dh/2 sits in k-step kk + Dh/32 of the same thread.
    if constexpr (!kFP8 && !QM) {
        const int pos = len - 1;
        if (p.cos_sin != nullptr && pos >= 0 && pos < p.max_pos) {
            const float* crow = p.cos_sin + (int64_t)pos * DH;
            auto unpack = [](uint32_t w, float& lo, float& hi) {
                if constexpr (kBF16) {
                    lo = __uint_as_float(w << 16);
                    hi = __uint_as_float(w & 0xffff0000u);
                } else {
                    lo = __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
                    hi = __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
                }
            };
#pragma unroll
            for (int kk = 0; kk < C::kKSteps; ++kk)
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    const int d = kk * 16 + ch * 8 + 2 * quad;
                    if (p.rope_style == KV_ROPE_HALF) {
                        if (kk >= C::kKSteps / 2) continue;
                        const float c0 = crow[d], c1 = crow[d + 1], s0 = crow[DH / 2 + d], s1 = crow[DH / 2 + d + 1];
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            float x0, x1, y0, y1;
                            unpack(qa[kk][rr + 2 * ch], x0, x1);
                            unpack(qa[kk + C::kKSteps / 2][rr + 2 * ch], y0, y1);
                            rotate_pair(x0, y0, c0, s0);
                            rotate_pair(x1, y1, c1, s1);
                            qa[kk][rr + 2 * ch] = pack2<kBF16>(x0, x1);
                            qa[kk + C::kKSteps / 2][rr + 2 * ch] = pack2<kBF16>(y0, y1);
                        }
                    } else {
                        const float c = crow[d / 2], s = crow[DH / 2 + d / 2];
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr) {
                            float x0, x1;
                            unpack(qa[kk][rr + 2 * ch], x0, x1);
                            rotate_pair(x0, x1, c, s);
                            qa[kk][rr + 2 * ch] = pack2<kBF16>(x0, x1);
                        }
                    }
                }
        }
    }

    float o[C::kOT][4];
#pragma unroll
    for (int n = 0; n < C::kOT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_ref[2] = {-INFINITY, -INFINITY};  // reference max (log2 units) of rows r0, r0 + 8
    float l_part[2] = {0.f, 0.f};             // this lane's share of the row sums
    const float sl2 = kFP8 ? p.scale_log2 * p.k_scale[kvh] : p.scale_log2;
    bool ok = true;

    if (active) {
        const int n_st = (n_local + PPS - 1) / PPS;
        for (int i = wp; i < n_st; i += p.WP) {
            const int s = i % C::kNS;
            if (!mbar_wait_bounded(full_bar + 8 * s, (i / C::kNS) & 1, kWaitLimitNs)) {
                raise_err(p.err, KV_DEV_ERR_TIMEOUT);
                ok = false;
            }
            if (!__all_sync(0xffffffffu, ok)) break;
            const int tag = stage_tag[s];
            if (tag != i && tag != -1 - i) {
                if (lane == 0) raise_err(p.err, KV_DEV_ERR_PIPELINE);
                break;
            }
            const uint32_t sK = sbase + s * C::kStage;
            const uint32_t sV = sK + C::kChunk;
            if (tag == i) {
                // tokens of this stage: its pages (the last stage of a range may hold fewer than PPS)
                const int nvalid = min(min(PPS, n_local - i * PPS) * P, len - (first + i * PPS) * P);

                // ---- S = Q K^T (fp32 accumulators; rows = heads, cols = tokens)
                float sc[C::kNT][4];
#pragma unroll
                for (int n = 0; n < C::kNT; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
                const int mi = lane >> 3, rr8 = lane & 7;
                if constexpr (kFP8) {
                    // token r0 of each n-tile: the thread's Dh/4 bytes of that row (E4M3 -> f16 pairs)
#pragma unroll
                    for (int n = 0; n < C::kNT; ++n) {
                        const int t = n * 8 + r0;
                        uint32_t w[DH / 16];
#pragma unroll
                        for (int c = 0; c < DH / 64; ++c) {
                            const uint4 x = lds128(sK + swz<C::kBoxInner>(t, quad * (DH / 64) + c));
                            w[4 * c] = x.x, w[4 * c + 1] = x.y, w[4 * c + 2] = x.z, w[4 * c + 3] = x.w;
                        }
#pragma unroll
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            uint32_t b0, b1;
                            e4m3x4_to_f16x2x2(w[kk], b0, b1);
                            mma_16816<false>(sc[n], qa[kk], b0, b1);
                        }
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < C::kKSteps; ++kk) {
                        const int c = kk * 2 + (mi & 1);  // 16-byte chunk of the row (8 dims)
                        const uint32_t boxb = sK + (c >> 3) * C::kBoxB;
#pragma unroll
                        for (int np = 0; np < C::kNT / 2; ++np) {
                            const int t = np * 16 + (mi >> 1) * 8 + rr8;
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4(boxb + t * 128 + (((c & 7) ^ (t & 7)) << 4), b0, b1, b2, b3);
                            mma_16816<kBF16>(sc[2 * np], qa[kk], b0, b1);
                            mma_16816<kBF16>(sc[2 * np + 1], qa[kk], b2, b3);
                        }
                    }
                }

                // ---- scale, mask, row max (4 lanes of a quad share a row)
                float mx[2] = {-INFINITY, -INFINITY};
                int tlim[2] = {nvalid, nvalid};  // first masked token of the stage per row
                if constexpr (QM) {
                    const int kbase = (first + i * PPS) * P;
                    tlim[0] = min(nvalid, key_lim[0] - kbase);
                    tlim[1] = min(nvalid, key_lim[1] - kbase);
                }
#pragma unroll
                for (int n = 0; n < C::kNT; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = n * 8 + 2 * quad + (e & 1);
                        const float v = (t < tlim[e >> 1]) ? sc[n][e] * sl2 : -INFINITY;
                        sc[n][e] = v;
                        mx[e >> 1] = fmaxf(mx[e >> 1], v);
                    }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                }
                // lazy reference update: only when a row's max grows by more than 2^8
                const bool grow = (mx[0] > m_ref[0] + 8.f) || (!lo_rows && mx[1] > m_ref[1] + 8.f);
                if (__any_sync(0xffffffffu, grow)) {
                    float a[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float mn = fmaxf(m_ref[h], mx[h]);
                        a[h] = (mn == m_ref[h]) ? 1.f : exp2f(m_ref[h] - mn);
                        m_ref[h] = mn;
                        l_part[h] *= a[h];
                    }
                    if constexpr (lo_rows) a[1] = a[0];  // rows r0 + 8 hold row r0's residual sums
#pragma unroll
                    for (int n = 0; n < C::kOT; ++n) {
                        o[n][0] *= a[0];
                        o[n][1] *= a[0];
                        o[n][2] *= a[1];
                        o[n][3] *= a[1];
                    }
                }
                // ---- probabilities straight into the A fragments of P V, as a
                // 16-bit pair plus its residual: one rounding of p to bf16
                // (2^-9 relative) alone can move a short row's output by
                // 2^-9 * max|v|, beyond the accuracy this kernel keeps. With
                // at most 8 real heads the residual of row r rides in padding
                // row r + 8 of the same MMA (summed at the end); otherwise it
                // takes a second MMA.
                uint32_t pa[C::kPK][4], pr[C::kPK][4];
#pragma unroll
                for (int n = 0; n < C::kNT; ++n) {
                    float pv[4];
#pragma unroll
                    for (int e = 0; e < (lo_rows ? 2 : 4); ++e) {
                        const float mr = m_ref[e >> 1];
                        pv[e] = (sc[n][e] == -INFINITY) ? 0.f : exp2f(sc[n][e] - mr);
                        l_part[e >> 1] += pv[e];
                    }
                    if constexpr (lo_rows) {
                        pack2_split<kBF16>(pv[0], pv[1], pa[n >> 1][(n & 1) * 2 + 0], pa[n >> 1][(n & 1) * 2 + 1]);
                    } else {
                        pack2_split<kBF16>(pv[0], pv[1], pa[n >> 1][(n & 1) * 2 + 0], pr[n >> 1][(n & 1) * 2 + 0]);
                        pack2_split<kBF16>(pv[2], pv[3], pa[n >> 1][(n & 1) * 2 + 1], pr[n >> 1][(n & 1) * 2 + 1]);
                    }
                }
                // ---- tail page: zero V rows past the length (they may hold stale data)
                if (nvalid < C::kTP) {
                    constexpr int kCPR = C::kBoxInner / 16;  // 16-byte chunks per box row
                    for (int idx = lane; idx < (C::kTP - nvalid) * C::kBoxes * kCPR; idx += 32) {
                        const int t = nvalid + idx / (C::kBoxes * kCPR);
                        const int rem = idx % (C::kBoxes * kCPR);
                        sts128_zero(sV + (rem / kCPR) * C::kBoxB + t * C::kBoxInner + ((rem % kCPR) << 4));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                // ---- O += P V (k = tokens, n = dims)
                if constexpr (kFP8) {
                    // Dim n-tile j, column r0 is dim r0 * Dh/8 + j: the thread reads its Dh/8 bytes of
                    // tokens 2q, 2q + 1, 2q + 8, 2q + 9 and pairs the two tokens' bytes per dim.
                    constexpr int kW = DH / 32;  // words per token row per thread
#pragma unroll
                    for (int ks = 0; ks < C::kPK; ++ks) {
                        uint32_t wv[4][kW];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int t = ks * 16 + 2 * quad + (e & 1) + 8 * (e >> 1);
                            if constexpr (DH == 128) {
                                const uint4 x = lds128(sV + swz<C::kBoxInner>(t, r0));
                                wv[e][0] = x.x, wv[e][1] = x.y, wv[e][2] = x.z, wv[e][3] = x.w;
                            } else {
                                const uint2 x = lds64(sV + swz<C::kBoxInner>(t, r0 >> 1) + (r0 & 1) * 8);
                                wv[e][0] = x.x, wv[e][1] = x.y;
                            }
                        }
#pragma unroll
                        for (int m = 0; m < kW; ++m) {
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {  // bytes 0-1 or 2-3 of word m
                                const uint32_t sel = hh ? 0x7362u : 0x5140u;
                                uint32_t b0[2], b1[2];  // [dim n-tile 4m + 2hh + e]
                                e4m3x4_to_f16x2x2(byte_perm(wv[0][m], wv[1][m], sel), b0[0], b0[1]);  // tokens 2q, 2q + 1
                                e4m3x4_to_f16x2x2(byte_perm(wv[2][m], wv[3][m], sel), b1[0], b1[1]);  // tokens 2q + 8, + 9
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int j = 4 * m + 2 * hh + e;
                                    mma_16816<false>(o[j], pa[ks], b0[e], b1[e]);
                                    if constexpr (!lo_rows) mma_16816<false>(o[j], pr[ks], b0[e], b1[e]);
                                }
                            }
                        }
                    }
                } else {
#pragma unroll
                for (int ks = 0; ks < C::kPK; ++ks) {
                    const int t = ks * 16 + (mi & 1) * 8 + rr8;
#pragma unroll
                    for (int op = 0; op < C::kOT / 2; ++op) {
                        const int c = op * 2 + (mi >> 1);
                        uint32_t v0, v1, v2, v3;
                        ldsm_x4_trans(sV + (c >> 3) * C::kBoxB + t * 128 + (((c & 7) ^ (t & 7)) << 4), v0, v1, v2, v3);
                        mma_16816<kBF16>(o[2 * op], pa[ks], v0, v1);
                        mma_16816<kBF16>(o[2 * op + 1], pa[ks], v2, v3);
                        if constexpr (!lo_rows) {
                            mma_16816<kBF16>(o[2 * op], pr[ks], v0, v1);
                            mma_16816<kBF16>(o[2 * op + 1], pr[ks], v2, v3);
                        }
                    }
                }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar + 8 * s);
        }
    }

    // ---- finalize: row sums over the quad, then merge page-warps in shared memory
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_part[h] += __shfl_xor_sync(0xffffffffu, l_part[h], 1);
        l_part[h] += __shfl_xor_sync(0xffffffffu, l_part[h], 2);
    }
    named_bar_sync(1, 32 * NW);  // every consumer is done with the stages (merge rows alias them)
    float* merge = reinterpret_cast<float*>(smem);  // [NW][16][DH + 2]
    if (active) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = r0 + 8 * h;
            if (r < rows) {
                float* dst = merge + (cw * 16 + r) * (DH + 2);
                const float vs = kFP8 ? p.v_scale[kvh] : 1.f;
#pragma unroll
                for (int n = 0; n < C::kOT; ++n) {
                    // column 2q (+1) of dim n-tile n: dim n*8 + 2q (+1); E4M3: dim (2q (+1)) * Dh/8 + n
                    const int d0 = kFP8 ? (2 * quad) * (DH / 8) + n : n * 8 + 2 * quad;
                    const int d1 = kFP8 ? (2 * quad + 1) * (DH / 8) + n : n * 8 + 2 * quad + 1;
                    dst[d0] = (o[n][2 * h] + (lo_rows ? o[n][2] : 0.f)) * vs;
                    dst[d1] = (o[n][2 * h + 1] + (lo_rows ? o[n][3] : 0.f)) * vs;
                }
                if (quad == 0) {
                    dst[DH] = m_ref[h];
                    dst[DH + 1] = l_part[h];
                }
            }
        }
    }
    named_bar_sync(1, 32 * NW);

    const int tid = threadIdx.x - 32;
    for (int e = tid; e < nt * p.g * DH; e += 32 * NW) {
        const int hh = e / DH;
        const int d = e % DH;
        const int slice = hh >> 4, r = hh & 15;
        float mstar = -INFINITY;
        for (int w = 0; w < p.WP; ++w) mstar = fmaxf(mstar, merge[((w * p.HS + slice) * 16 + r) * (DH + 2) + DH]);
        float L = 0.f, U = 0.f;
        if (mstar != -INFINITY) {
            for (int w = 0; w < p.WP; ++w) {
                const float* src = merge + ((w * p.HS + slice) * 16 + r) * (DH + 2);
                const float mw = src[DH];
                if (mw == -INFINITY) continue;
                const float sw = exp2f(mw - mstar);
                L += sw * src[DH + 1];
                U += sw * src[d];
            }
        }
        const int64_t hq = QM ? (int64_t)(qs0 + t0 + hh / p.g) * p.H_q + (int64_t)kvh * p.g + hh % p.g
                              : (int64_t)b * p.H_q + (int64_t)kvh * p.g + hh;
        if (!split_mode) {
            p.out[hq * DH + d] = (L > 0.f) ? U / L : 0.f;
        } else {
            const int64_t ps = p.items != nullptr ? (int64_t)item * p.g + hh : hq * p.num_splits + split;
            p.part_u[ps * DH + d] = U;
            if (d == 0) p.part_ml[ps] = make_float2(mstar, L);
        }
    }
}

}  // namespace kvp
