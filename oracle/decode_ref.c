/*
 * CPU ORACLE -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 reference for single-token decode attention over a paged
 * KV cache. Only tests/, the smoke check and the CPU-baseline leg of the
 * benchmark may load it; the product path never does. It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition; no blocking, no online softmax):
 *   Attention(Q,K,V) = softmax(Q K^T / sqrt(d) + causal_mask) V
 *   -- "04. 注意力与 KV 缓存", section "深入：注意力公式与缓存成立条件", and
 *   "03. KV Cache：用显存换计算", section "注意力的公式".
 * For one decode query the causal mask admits every cached position, so for
 * each (sequence b, query head h):
 *   1. walk the block table: position t lives in logical block t / P at offset
 *      t % P, i.e. physical page table[b][t / P]
 *      ("07｜KV Cache、FlashAttention与PagedAttention的内部过程", Q028,
 *      block-size-4 example table);
 *   2. upcast the stored K, V and q values to fp64;
 *   3. materialise the whole score row s_t = scale * <q, K_t> for t < len;
 *   4. softmax with the row maximum subtracted, o = sum_t p_t V_t.
 * Query head h reads KV head h / (H_q / H_kv) (contiguous GQA grouping: the
 * course-notes page "06 KV Cache、Prefix Cache、PagedAttention 与 vLLM",
 * section 6.3, does not fix the mapping; this is the reading taken).
 *
 * Physical layout read here: k_pages/v_pages [num_pages][H_kv][P][Dh] of the
 * storage dtype (the pages leave the layout open: HB-07 Q025 says kernels may
 * use other layouts as long as the semantic axes stay the same).
 *
 * Storage dtypes are decoded from their published bit-level definitions:
 *   fp32: IEEE 754 binary32; bf16: the upper 16 bits of a binary32;
 *   fp16: IEEE 754 binary16 (1 sign, 5 exponent bits with bias 15, 10 fraction
 *   bits; exponent 0 = subnormal, 31 = inf/NaN).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_FP32 = 0, OR_BF16 = 1, OR_FP16 = 2 };

double oracle_fp16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);              /* subnormal: f * 2^-14 * 2^-10 */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);  /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double elem(const void* base, int64_t i, int dtype) {
    if (dtype == OR_FP32) return (double)((const float*)base)[i];
    uint16_t h = ((const uint16_t*)base)[i];
    return dtype == OR_BF16 ? oracle_bf16_to_double(h) : oracle_fp16_to_double(h);
}

/* Decode a storage array to fp64 (used by tests to read inputs as numbers). */
void oracle_decode_storage(double* out, const void* src, int64_t n, int32_t dtype) {
    for (int64_t i = 0; i < n; ++i) out[i] = elem(src, i, dtype);
}

/*
 * out:   fp64 [B][H_q][Dh]; only rows named in `pairs` are written when
 *        pairs != NULL (pairs = n_pairs (b, h) int32 pairs), else all rows.
 * Returns 0, or -1 if a block-table entry needed for some row is out of
 * range / a length exceeds the table, or -2 on bad shapes.
 */
int oracle_paged_decode(double* out, const void* q, const void* k_pages, const void* v_pages,
                        const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens,
                        int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t P, int32_t num_pages,
                        double scale, int32_t dtype, const int32_t* pairs, int32_t n_pairs,
                        int32_t nthreads) {
    if (B < 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0 || Dh <= 0 || P <= 0) return -2;
    const int32_t g = H_q / H_kv;
    const int64_t n_items = pairs ? (int64_t)n_pairs : (int64_t)B * H_q;
    int status = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t it = 0; it < n_items; ++it) {
        int32_t b = pairs ? pairs[2 * it] : (int32_t)(it / H_q);
        int32_t h = pairs ? pairs[2 * it + 1] : (int32_t)(it % H_q);
        int32_t kvh = h / g;
        int32_t len = seq_lens[b];
        double* o = out + ((int64_t)b * H_q + h) * Dh;
        for (int32_t d = 0; d < Dh; ++d) o[d] = 0.0;
        if (len <= 0) continue;
        if ((int64_t)len > (int64_t)max_blocks * P) {
#pragma omp atomic write
            status = -1;
            continue;
        }
        /* step 1-3: gather K through the block table, full score row */
        double* s = (double*)malloc(sizeof(double) * (size_t)len);
        int bad = 0;
        for (int32_t t = 0; t < len && !bad; ++t) {
            int32_t page = block_tables[(int64_t)b * max_blocks + t / P];
            if (page < 0 || page >= num_pages) { bad = 1; break; }
            int64_t row = (((int64_t)page * H_kv + kvh) * P + (t % P)) * Dh;
            double acc = 0.0;
            for (int32_t d = 0; d < Dh; ++d)
                acc += elem(q, ((int64_t)b * H_q + h) * Dh + d, dtype) * elem(k_pages, row + d, dtype);
            s[t] = scale * acc;
        }
        if (bad) {
            free(s);
#pragma omp atomic write
            status = -1;
            continue;
        }
        /* step 4: softmax with the maximum subtracted, then weighted sum of V */
        double m = s[0];
        for (int32_t t = 1; t < len; ++t) if (s[t] > m) m = s[t];
        double l = 0.0;
        for (int32_t t = 0; t < len; ++t) { s[t] = exp(s[t] - m); l += s[t]; }
        for (int32_t t = 0; t < len; ++t) {
            int32_t page = block_tables[(int64_t)b * max_blocks + t / P];
            int64_t row = (((int64_t)page * H_kv + kvh) * P + (t % P)) * Dh;
            double p = s[t] / l;
            for (int32_t d = 0; d < Dh; ++d) o[d] += p * elem(v_pages, row + d, dtype);
        }
        free(s);
    }
    return status;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
