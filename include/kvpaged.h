/*
 * kvpaged.h -- C ABI of the paged KV-cache decode library (B200, sm_100a).
 *
 * Pages cited by title and section:
 *   [KV-04] "04. 注意力与 KV 缓存" (inference series)
 *   [HB-07] "07｜KV Cache、FlashAttention与PagedAttention的内部过程"
 *           (AI engineering handbook, chapter 07, questions Q025-Q028)
 *   [CN-06] "06 KV Cache、Prefix Cache、PagedAttention 与 vLLM" (course notes)
 *   [KV-03] "03. KV Cache：用显存换计算" (llm-inference series)
 *
 * Conventions for every entry point:
 *   - Returns an int status: KV_OK (0) or a negative KV_ERR_* code. No C++
 *     exception crosses the ABI. On error nothing is launched and host state
 *     is unchanged unless stated otherwise.
 *   - Device pointers are owned by the caller (e.g. PyTorch tensors) and must
 *     be 16-byte aligned. No entry point allocates device memory when it is
 *     called; kernels needing scratch take a caller-provided workspace. The
 *     one piece of device memory the library holds is a fixed module array of
 *     KV_NOALLOC_SCRATCH_BYTES per GPU (the scratch of
 *     paged_decode_attention_noalloc), present from module load until exit.
 *   - Host handles (kv_pool_t, kv_prefix_t) are owned by the library and
 *     released with their _destroy call. They are not thread-safe.
 *   - Launches are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). A launch failure is reported as KV_ERR_CUDA.
 *   - `err_flag` (nullable) is a device int that kernels OR KV_DEV_ERR_* bits
 *     into when they meet bad data (out-of-range page id or slot, bad length,
 *     a bounded wait that gave up). Kernels never trap; the caller reads the
 *     flag when it wants to know.
 *
 * Physical layout (the pages leave it open, [HB-07] Q025: "kernels may use a
 * different memory layout"): per layer, K and V pools of shape
 *   [num_pages][H_kv][page_size][Dh]
 * of the storage dtype, so one (page, head) chunk of page_size x Dh values is
 * contiguous. Block tables are int32 [B][max_blocks] (row b lists the
 * physical pages of sequence b in logical order). seq_lens are int32 [B] and
 * count the token appended in this step. Slots are int64: page * page_size +
 * offset. Query head h uses KV head h / (H_q / H_kv).
 */
#ifndef KVPAGED_H
#define KVPAGED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define KV_OK 0
#define KV_ERR_ARG (-1)          /* bad argument, shape or alignment */
#define KV_ERR_OOM (-2)          /* pool has fewer free pages than asked */
#define KV_ERR_BAD_ID (-3)       /* page id out of range, or not held */
#define KV_ERR_DOUBLE_FREE (-4)  /* free of a page more times than it is held */
#define KV_ERR_SHARED_TAIL (-5)  /* append into a partial page another sequence holds */
#define KV_ERR_CUDA (-6)         /* a CUDA launch or query failed */
#define KV_ERR_WORKSPACE (-7)    /* workspace missing or too small */
#define KV_ERR_UNSUPPORTED (-8)  /* shape outside the compiled kernel set */

/* ---- storage dtypes ----------------------------------------------------- */
#define KV_DTYPE_F32 0
#define KV_DTYPE_BF16 1
#define KV_DTYPE_F16 2
#define KV_DTYPE_FP8_E4M3 3  /* K/V pools only: 8-bit E4M3 codes with per-KV-head scales */

/* ---- device error bits (OR-ed into *err_flag) --------------------------- */
#define KV_DEV_ERR_PAGE_RANGE 1  /* a block-table entry outside [0, num_pages); that page is skipped */
#define KV_DEV_ERR_SEQ_LEN 2     /* seq_len < 0 or > max_blocks * page_size; the row is zeroed */
#define KV_DEV_ERR_SLOT 4        /* kv_append slot >= num_pages * page_size; that row is skipped */
#define KV_DEV_ERR_TIMEOUT 8     /* a bounded pipeline wait gave up; outputs of that CTA are invalid */
#define KV_DEV_ERR_PIPELINE 16   /* a pipeline stage held another page than expected; outputs invalid */
#define KV_DEV_ERR_POSITION 32   /* kv_rope_append position outside [0, max_pos); that token is skipped */

const char* kv_status_string(int status);
int kv_version(void);

/* =========================================================================
 * Page pool -- [HB-07] Q028 (fixed-size blocks in a physical pool, allocated
 * on demand, returned when a request ends); [CN-06] 6.5 (the allocation flow
 * and copy-on-write with reference counts for shared blocks); [KV-04]
 * "深入：引擎怎样找状态" (a page still used by another request is never
 * reclaimed).
 * The free list is FIFO: it starts as `init_free_order` (a permutation of
 * 0..num_pages-1; NULL = ascending), alloc pops from the head, and a page whose
 * count drops to 0 is pushed to the tail.
 * ======================================================================= */
typedef struct kv_pool kv_pool_t;

/* Create a pool of num_pages pages of page_size tokens. KV_ERR_ARG if sizes
 * are not positive or init_free_order is not a permutation. */
int kv_pool_create(int32_t num_pages, int32_t page_size, const int32_t* init_free_order, kv_pool_t** out);
int kv_pool_destroy(kv_pool_t* pool);

/* Allocate n pages (refcount 1 each) into out_ids[n], all-or-nothing:
 * KV_ERR_OOM leaves the pool unchanged. A page that a prefix index still
 * lists as reusable is dropped from that index when it is handed out. */
int kv_pool_alloc(kv_pool_t* pool, int32_t n, int32_t* out_ids);

/* Drop one reference per listed id (an id may repeat). All-or-nothing:
 * KV_ERR_BAD_ID for an id out of range, KV_ERR_DOUBLE_FREE if an id is
 * listed more times than it is held. */
int kv_pool_free(kv_pool_t* pool, int32_t n, const int32_t* ids);

/* Add one reference per listed id (sharing, e.g. after a prefix hit). A page
 * with count 0 may be revived only while a prefix index lists it (it leaves
 * the free list); otherwise KV_ERR_BAD_ID. All-or-nothing. */
int kv_pool_incref(kv_pool_t* pool, int32_t n, const int32_t* ids);
int kv_pool_refcount(const kv_pool_t* pool, int32_t id, int32_t* out);
int kv_pool_num_free(const kv_pool_t* pool, int32_t* out);
int kv_pool_page_size(const kv_pool_t* pool, int32_t* out);

/* Block accounting for one sequence of `len` tokens: pages = ceil(len / P),
 * slots = pages * P, wasted = slots - len ([CN-06] 6.5: 35 @ 16 -> 3, 48, 13). */
int kv_blocks_for_len(int32_t len, int32_t page_size, int32_t* pages, int32_t* slots, int32_t* wasted);

/* KV bytes = 2 * L * B * T * H_kv * Dh * bytes_per_elem ([HB-07] Q026;
 * [CN-06] 6.3). */
int kv_cache_bytes(int64_t L, int64_t B, int64_t T, int64_t H_kv, int64_t Dh, int64_t bytes_per_elem, int64_t* out);

/* Slot of logical position `pos` through one block-table row:
 * table_row[pos / P] * P + pos % P ([HB-07] Q028, block-size-4 table).
 * KV_ERR_ARG if pos / P >= n_blocks; KV_ERR_BAD_ID if the entry is negative. */
int kv_slot_for_pos(const int32_t* table_row, int32_t n_blocks, int32_t page_size, int64_t pos, int64_t* out);

/* Slots of `n` consecutive positions start..start+n-1 of one sequence
 * (e.g. to write a prefill or a prefix with kv_append). Same errors. */
int kv_slots_for_range(const int32_t* table_row, int32_t n_blocks, int32_t page_size, int64_t start, int64_t n,
                       int64_t* out_slots);

/* One decode step's host bookkeeping for B sequences (host arrays):
 * for each b, the new token goes to position seq_lens[b]; when
 * seq_lens[b] % P == 0 a page is allocated first and written to
 * block_tables[b][seq_lens[b] / P] ([HB-07] Q028: positions 10 and 11 fill
 * block 19, position 12 is the first that needs a new block).
 * slot_mapping[b] receives the slot and seq_lens[b] is incremented.
 * Pages are allocated together in order of b, all-or-nothing (KV_ERR_OOM).
 * KV_ERR_SHARED_TAIL if the partial tail page is held by more than one
 * sequence (it needs copy-on-write first, [HB-07] Q028 table step 6);
 * KV_ERR_ARG if a table row is full. On error nothing is changed. */
int kv_append_slots(kv_pool_t* pool, int32_t B, int32_t* block_tables, int32_t max_blocks, int32_t* seq_lens,
                    int64_t* slot_mapping);

/* Copy-on-write of shared partial tail pages ([HB-07] Q028: a partial last
 * block shared by two sequences must be copied, or kept apart, before either
 * writes to it -- table step 6; [CN-06] 6.5: shared blocks are read-only and
 * copied on write, with reference counts). Sequences are taken in order of
 * b; when the page that sequence b's next token goes to (position
 * seq_lens[b], with seq_lens[b] % P != 0) still has refcount > 1, a fresh
 * page replaces it in block_tables[b], one reference to the old page is
 * dropped, and the pair is reported in src_pages[k], dst_pages[k] for
 * k < *n_copies (host arrays with room for B entries). The last holder keeps
 * the original. Fresh pages are allocated together, all-or-nothing
 * (KV_ERR_OOM leaves everything unchanged); KV_ERR_BAD_ID for a tail entry
 * out of range; KV_ERR_ARG for a full table row. The caller copies the page
 * contents with kv_copy_pages before the next append. */
int kv_pool_cow_tails(kv_pool_t* pool, int32_t B, int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens,
                      int32_t* src_pages, int32_t* dst_pages, int32_t* n_copies);

/* =========================================================================
 * Prefix index -- [CN-06] 6.4: full cached blocks are keyed by a chained
 * hash of the parent block's key and this block's tokens; the first block
 * that differs stops the match; whether partial blocks are reused is left to
 * the implementation (here: never). [HB-07] Q028: the key must also carry the
 * identity (model, adapter, template...) -> `salt`. [KV-04] prefix demo: a
 * difference early in the prompt invalidates every later block even where
 * tokens agree again.
 * Key of block i: h_0 = salt, h_{i+1} = FNV-1a-64(h_i as 8 little-endian
 * bytes, then the block's P tokens as 4 little-endian bytes each). A hit is
 * confirmed by comparing the stored tokens and the parent entry, so results
 * never depend on hash collisions.
 * A registered page whose refcount reaches 0 stays matchable while it sits in
 * the free list (kv_pool_incref revives it); when kv_pool_alloc hands it out
 * again its entry and every entry registered below it are dropped.
 * Registering a prefix block that is already registered keeps the first page.
 * ======================================================================= */
typedef struct kv_prefix kv_prefix_t;

int kv_prefix_index_create(int32_t page_size, uint64_t salt, kv_prefix_t** out);
int kv_prefix_index_destroy(kv_prefix_t* index);

/* Register the full pages of a sequence: tokens[0..n) live in page_ids[i]
 * for block i (only the first n / P blocks are registered). Binds the index
 * to `pool` on first use (one pool per index). KV_ERR_BAD_ID if a page is not
 * currently allocated; KV_ERR_ARG if a page is already registered for a
 * different prefix, or the pool's page size differs. All-or-nothing. */
int kv_prefix_register(kv_prefix_t* index, kv_pool_t* pool, const int32_t* tokens, int32_t n, const int32_t* page_ids);

/* Number of leading FULL pages of tokens[0..n) already cached
 * (*out_num_pages), and their ids in out_page_ids (nullable; room for n / P).
 * page_size must equal the index's. Read-only: the caller takes references
 * with kv_pool_incref before using the pages. */
int kv_prefix_match(const kv_prefix_t* index, const int32_t* tokens, int32_t n, int32_t page_size,
                    int32_t* out_page_ids, int32_t* out_num_pages);

/* Number of registered pages. */
int kv_prefix_num_entries(const kv_prefix_t* index, int32_t* out);

/* =========================================================================
 * Device kernels
 * ======================================================================= */

/* KV append -- [HB-07] Q025 (each layer appends the new token's K/V to its
 * own cache before attending); [CN-06] 6.1-6.2; [KV-03] lifecycle section, fill step.
 * For every b in [0, B) with slot_mapping[b] >= 0 and every head h:
 *   k_pages[slot / P][h][slot % P][:] = k_new[b][h][:], same for V.
 * k_new, v_new: [B][H_kv][Dh] contiguous, same dtype as the pools.
 * slot_mapping: device int64 [B]; -1 skips the row. A slot >= num_pages * P
 * sets KV_DEV_ERR_SLOT and the row is skipped. B may be any size (a prefill
 * writes many tokens in one call). Rows must not share a slot. */
int kv_append(void* k_pages, void* v_pages, const void* k_new, const void* v_new, const int64_t* slot_mapping,
              int32_t B, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, int32_t dtype,
              int* err_flag, void* stream);

/* Rotary position embedding fused with the KV append -- [CN-06] 6.1 (for a
 * new token: rotate q and k by its position, append k and v, then attend).
 * The pages name the rotation without defining it; this is the usual rotary
 * embedding. For token b at position pos = positions[b] and pair k of a row
 * (k = 0 .. Dh/2 - 1), with c = cos_sin[pos][k], s = cos_sin[pos][Dh/2 + k]:
 *   x_i' = x_i c - x_j s,   x_j' = x_j c + x_i s,
 * where (i, j) = (k, k + Dh/2) for KV_ROPE_HALF (split halves, Llama-family
 * layout) or (2k, 2k + 1) for KV_ROPE_INTERLEAVED. Every product and sum is
 * rounded to fp32 on its own (no fused multiply-add), then x' is rounded to
 * the storage dtype with round-to-nearest-even: results are bit-reproducible.
 * Writes, per token: the rotated k_new rows to k_pages and the v_new rows
 * (unrotated) to v_pages at slot_mapping[b] (as kv_append: -1 skips the
 * cache write; a slot past the pool sets KV_DEV_ERR_SLOT); and, when q is not
 * NULL, the rotated q rows to q_out (q_out may equal q; in-place is safe).
 *   q, q_out: [B][H_q][Dh] (both NULL, or both set with H_q > 0).
 *   k_new, v_new: [B][H_kv][Dh]; all of the pools' dtype.
 *   positions: device int32 [B]; outside [0, max_pos) sets
 *   KV_DEV_ERR_POSITION and nothing is written for that token.
 *   cos_sin: device fp32 [max_pos][Dh] (cos then sin per row), owned by the
 *   caller (typically cos / sin of pos * base^(-2k/Dh), computed once).
 *   Dh * sizeof(dtype) must be a multiple of 32 (KV_ERR_UNSUPPORTED); all
 *   row pointers 16-byte aligned (KV_ERR_ARG). */
#define KV_ROPE_HALF 0
#define KV_ROPE_INTERLEAVED 1
int kv_rope_append(void* k_pages, void* v_pages, void* q_out, const void* q, const void* k_new, const void* v_new,
                   const int64_t* slot_mapping, const int32_t* positions, const float* cos_sin, int32_t max_pos,
                   int32_t rope_style, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size,
                   int32_t num_pages, int32_t dtype, int* err_flag, void* stream);

/* One launch for a layer's whole decode step ([CN-06] 6.1 order: rotate q
 * and k by the new token's position, append k and v, attend): as
 * paged_decode_attention_append, with the new token's k row and every query
 * head rotated at position seq_lens[b] - 1 exactly as kv_rope_append does it
 * (same cos_sin table, max_pos, rope_style; the stored k bits and the
 * rotated q bits are the same), and q read unrotated from `q`.
 * bf16 / fp16 K/V on the tensor-core kernel only (KV_ERR_UNSUPPORTED
 * otherwise). A position outside [0, max_pos) sets KV_DEV_ERR_POSITION; that
 * row's output is then undefined. */
int paged_decode_attention_rope_append(float* out, const void* q, const void* k_new, const void* v_new,
                                       void* k_pages, void* v_pages, const int32_t* block_tables, int32_t max_blocks,
                                       const int32_t* seq_lens, const float* cos_sin, int32_t max_pos,
                                       int32_t rope_style, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh,
                                       int32_t page_size, int32_t num_pages, float scale, int32_t dtype,
                                       int32_t num_splits, void* workspace, size_t ws_bytes, int* err_flag,
                                       void* stream);

/* Copy whole pages of both pools: for i < n, page src_pages[i] -> page
 * dst_pages[i] (all H_kv heads and page_size slots; src/dst are device int32
 * arrays), e.g. after kv_pool_cow_tails. A page id outside [0, num_pages)
 * sets KV_DEV_ERR_PAGE_RANGE and that pair is skipped. Destinations must be
 * distinct and must not be sources. */
int kv_copy_pages(void* k_pages, void* v_pages, const int32_t* src_pages, const int32_t* dst_pages, int32_t n,
                  int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, int32_t dtype, int* err_flag,
                  void* stream);

/* Paged decode attention -- one new query per sequence:
 *   out[b][h][:] = softmax(scale * q[b][h] . K_t) V_t  over t < seq_lens[b]
 * with K_t, V_t of KV head h / (H_q / H_kv) found through block_tables
 * ([KV-04] / [KV-03] attention formula; [HB-07] Q028 block-table walk).
 * Each CTA walks its pages and folds them with the online (m, l, u) merge of
 * [HB-07] Q027; the result equals the full softmax up to rounding order.
 *   out: fp32 [B][H_q][Dh].   q: [B][H_q][Dh] of `dtype` (same as K/V).
 *   block_tables: int32 [B][max_blocks]; seq_lens: int32 [B] (0 -> zeros).
 *   Supported: Dh in {64, 128}; page_size in {16, 32}; H_q % H_kv == 0 with
 *   H_q / H_kv <= 64 for bf16/fp16 on the tensor-core kernel, <= 32 for fp32
 *   or the CUDA-core kernel; dtype F32/BF16/F16 (E4M3 pools go through
 *   paged_decode_attention_fp8). Else KV_ERR_UNSUPPORTED/KV_ERR_ARG.
 *   num_splits: 1 = single pass; >1 = split each sequence's pages into that
 *   many contiguous ranges (split-KV) merged by a second combine kernel;
 *   0 = choose automatically from B, H_kv, max_blocks and the SM count;
 *   for bf16/fp16 K/V on the warp-MMA kernel with more (sequence, KV head)
 *   rows than 4 x the SM count (and B <= 8192), a planned launch is used
 *   instead: a one-CTA plan kernel reads seq_lens and cuts every row into
 *   chunks of C pages chosen from the actual lengths (full chunks at the
 *   front of the grid, short tail chunks at the back), then the decode and
 *   combine kernels follow that plan (three launches). On the tcgen05 kernel
 *   (see paged_decode_set_kernel) num_splits = 0 with B > 1 (B <= 8192) is
 *   always planned: the plan kernel lays the rows end to end, each counted
 *   with one stage (128 keys) of extra cost, and gives each of the SM-count
 *   persistent CTAs an equal range; rows cut between two CTAs leave
 *   partials that a combine kernel merges (one CTA per range boundary).
 *   workspace / ws_bytes: device scratch for split partials, at least
 *   paged_decode_workspace_bytes(...) for the same arguments (NULL/0 is fine
 *   when no split is used); KV_ERR_WORKSPACE if too small. Calls sharing one
 *   workspace must be ordered on the GPU (e.g. one stream). */
int paged_decode_attention(float* out, const void* q, const void* k_pages, const void* v_pages,
                           const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t B,
                           int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages, float scale,
                           int32_t dtype, int32_t num_splits, void* workspace, size_t ws_bytes, int* err_flag,
                           void* stream);

/* kv_append and paged_decode_attention in one launch. The new token of each
 * sequence is at position seq_lens[b] - 1 (seq_lens counts it, as for
 * paged_decode_attention); its K and V rows k_new[b][h][:], v_new[b][h][:]
 * ([B][H_kv][Dh], pool dtype) are written to slot
 * block_tables[b][(len-1)/P] * P + (len-1) % P of k_pages / v_pages by the
 * CTA that reads that page, before it reads it; then attention proceeds as in
 * paged_decode_attention ([HB-07] Q025: append, then q_new @ K_all^T). The
 * slot's page must already be in the block table (kv_append_slots allocates
 * it). Same arguments, errors and workspace otherwise; KV_ERR_ARG if k_new or
 * v_new is NULL or not 16-byte aligned. */
int paged_decode_attention_append(float* out, const void* q, const void* k_new, const void* v_new, void* k_pages,
                                  void* v_pages, const int32_t* block_tables, int32_t max_blocks,
                                  const int32_t* seq_lens, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh,
                                  int32_t page_size, int32_t num_pages, float scale, int32_t dtype, int32_t num_splits,
                                  void* workspace, size_t ws_bytes, int* err_flag, void* stream);

/* Multi-token query over the paged cache (chunked prefill / prompt
 * extension) -- [CN-06] 6.2 and 6.6 (a prompt processed in chunks after the
 * part already cached); causal rule of [KV-04] / [HB-07] Q025 (a token sees
 * itself and every earlier position). The chunk's K/V must already be in the
 * cache (kv_append / kv_rope_append of its rows). For sequence b its chunk is
 * the last n_b = q_start[b+1] - q_start[b] of its seq_lens[b] tokens; chunk
 * row i (q row q_start[b] + i) sits at position pos = seq_lens[b] - n_b + i
 * and
 *   out[row][h][:] = softmax(scale * q[row][h] . K_t) V_t over t <= pos.
 *   q: [q_start[B]][H_q][Dh] of `dtype` (bf16 / fp16); out: fp32, same rows.
 *   q_start: device int32 [B + 1], non-decreasing from 0; max_q_len >= every
 *   n_b (it sizes the grid: rows past max_q_len are not computed).
 *   n_b > seq_lens[b] sets KV_DEV_ERR_SEQ_LEN and zeroes those rows.
 *   Tensor cores only: H_q / H_kv <= 64, Dh in {64, 128}, page_size in
 *   {16, 32}; fp32 K/V -> KV_ERR_UNSUPPORTED. No workspace. */
int paged_prefill_attention(float* out, const void* q, const int32_t* q_start, int32_t max_q_len,
                            const void* k_pages, const void* v_pages, const int32_t* block_tables, int32_t max_blocks,
                            const int32_t* seq_lens, int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh,
                            int32_t page_size, int32_t num_pages, float scale, int32_t dtype, int* err_flag,
                            void* stream);

/* ---- FP8 (E4M3) K/V cache ---------------------------------------------
 * "03. KV Cache：用显存换计算" (KV quantisation follow-up) and [CN-06]'s
 * KV-size table name storing K / V in 8 bits without fixing a format. Here:
 * pools of E4M3 codes (1 byte per element; same [num_pages][H_kv][P][Dh]
 * layout) and one fp32 scale per KV head and pool, read value = E4M3 value *
 * scale. The scales are the caller's (device fp32 [H_kv], e.g. calibrated as
 * max|x| / 448); they must not change while codes written with them live.
 * kv_copy_pages and kv_append (raw codes) accept KV_DTYPE_FP8_E4M3. */

/* Quantising append: for each b with slot_mapping[b] >= 0 and head h,
 *   k_pages[slot][h][:] = E4M3(k_new[b][h][:] / k_scale[h]), same for V,
 * where x / scale is an IEEE fp32 division and E4M3() rounds to nearest even,
 * saturating at +-448 (NaN stays NaN). k_new, v_new: [B][H_kv][Dh] of
 * src_dtype (bf16, fp16 or fp32). Dh % 16 == 0 (else KV_ERR_UNSUPPORTED).
 * Slots as kv_append (-1 skips; past the pool: KV_DEV_ERR_SLOT). */
int kv_append_fp8(void* k_pages, void* v_pages, const void* k_new, const void* v_new, int32_t src_dtype,
                  const float* k_scale, const float* v_scale, const int64_t* slot_mapping, int32_t B, int32_t H_kv,
                  int32_t Dh, int32_t page_size, int32_t num_pages, int* err_flag, void* stream);

/* Decode attention over E4M3 pools: as paged_decode_attention with
 *   K_t = code_t * k_scale[kv head], V_t = code_t * v_scale[kv head],
 * q of q_dtype (KV_DTYPE_BF16 or KV_DTYPE_F16; its values must lie within
 * fp16's range, +-65504, as the products run on the tensor cores in fp16 --
 * E4M3 values are exact in fp16). Tensor-core kernels only (H_q / H_kv <= 64,
 * Dh in {64, 128}, page_size in {16, 32}): the warp-MMA kernel, or, when
 * KV_DECODE_KERNEL_TCGEN05 is selected and H_q / H_kv is 4, 8 or 16 with
 * Dh = 128, the tcgen05 kernel, which widens each stage's pages to fp16 on the
 * SM (K into tensor memory, V into shared memory) and keeps the probabilities
 * as one fp16 operand; num_splits, workspace (same size
 * as paged_decode_workspace_bytes), errors and output as
 * paged_decode_attention, except that the automatic split count
 * (num_splits = 0, B > 1) aims at half as many CTAs per SM, each moving half
 * the bytes of a 16-bit page: paged_decode_num_splits reports the 16-bit
 * count, an upper bound. */
int paged_decode_attention_fp8(float* out, const void* q, int32_t q_dtype, const void* k_pages, const void* v_pages,
                               const float* k_scale, const float* v_scale, const int32_t* block_tables,
                               int32_t max_blocks, const int32_t* seq_lens, int32_t B, int32_t H_q, int32_t H_kv,
                               int32_t Dh, int32_t page_size, int32_t num_pages, float scale, int32_t num_splits,
                               void* workspace, size_t ws_bytes, int* err_flag, void* stream);

/* Which decode kernel paged_decode_attention uses (process-wide; default AUTO):
 *   KV_DECODE_KERNEL_AUTO  bf16/fp16 K/V, Dh = 128, no fused rotation, and
 *                          either H_q / H_kv = 32 (MQA-shaped groups) or
 *                          H_q / H_kv in {4, 8, 16} with num_splits = 0 and
 *                          B * H_kv above four per SM: the fifth-generation
 *                          tensor-core kernel (tcgen05; the 128 tokens of a
 *                          stage are the MMA rows, scores and output accumulate
 *                          in tensor memory; persistent, one CTA per SM; with
 *                          num_splits = 0 and B > 1 a device plan gives every
 *                          CTA the same share of the batch's pages, each work
 *                          item counted one stage extra, three at g = 32).
 *                          Other bf16/fp16 shapes with
 *                          H_q / H_kv <= 64: warp MMA on TMA-staged swizzled
 *                          tiles. fp32 K/V: CUDA cores (packed f32x2 FMA);
 *   KV_DECODE_KERNEL_SIMT  CUDA cores for every dtype (H_q / H_kv <= 32);
 *   KV_DECODE_KERNEL_MMA   warp MMA for every bf16/fp16 shape (never the
 *                          tcgen05 kernel; fp32 K/V still use CUDA cores);
 *   KV_DECODE_KERNEL_TCGEN05  the tcgen05 kernels wherever they apply: bf16/fp16
 *                          K/V, Dh = 128, H_q / H_kv in {4, 8, 16, 32}, no
 *                          fused rotation; E4M3 K/V, Dh = 128, H_q / H_kv in
 *                          {4, 8, 16} (else as AUTO).
 * All kernels compute the same function; this exists to compare them.
 * KV_ERR_ARG for an unknown kind. The multi-token query
 * (paged_prefill_attention) takes its tcgen05 kernel under AUTO and TCGEN05
 * for Dh = 128 and groups that divide 128, its warp-MMA kernel otherwise. */
#define KV_DECODE_KERNEL_AUTO 0
#define KV_DECODE_KERNEL_SIMT 1
#define KV_DECODE_KERNEL_MMA 2
#define KV_DECODE_KERNEL_TCGEN05 3
int paged_decode_set_kernel(int32_t kind);

/* How paged_decode_attention (dtype = the K/V type) would launch for these
 * arguments under the current kernel selection: *splits = the split count
 * (0 = planned on the device), *kernel = KV_DECODE_KERNEL_SIMT, _MMA or
 * _TCGEN05. KV_ERR_ARG for bad shapes. */
int paged_decode_launch_info(int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t max_blocks, int32_t page_size,
                             int32_t dtype, int32_t num_splits, int32_t* splits, int32_t* kernel);

/* The split count the warp-MMA kernel uses for these arguments (resolves
 * num_splits = 0 on the current device). 0 means the launch is planned on
 * the device (see paged_decode_attention); fp32 K/V and the CUDA-core kernel
 * use the grid rule's split count even then. paged_decode_launch_info also
 * covers the tcgen05 kernel. */
int paged_decode_num_splits(int32_t B, int32_t H_kv, int32_t max_blocks, int32_t page_size, int32_t num_splits,
                            int32_t* out);

/* Workspace bytes needed by paged_decode_attention for the same arguments
 * (0 when no split is used), for 16-bit K/V under the current kernel
 * selection (an upper bound for the other types). */
int paged_decode_workspace_bytes(int32_t B, int32_t H_q, int32_t H_kv, int32_t Dh, int32_t max_blocks,
                                 int32_t page_size, int32_t num_splits, size_t* out);

/* Same computation as paged_decode_attention, for callers that cannot
 * allocate device memory -- for example a plug-in whose host framework owns
 * every device allocation and passes in only input and output tensors, or a
 * latency-critical path that must not allocate. Instead of a workspace, the
 * split partials use a fixed array of KV_NOALLOC_SCRATCH_BYTES in the
 * library's own device memory (held on every GPU that loads the library until
 * the process exits). No allocation of any kind happens in the call.
 * The pages describe nothing of this kind: it has no counterpart there.
 *   - The first call on a device looks up that array's device address
 *     (cudaGetSymbolAddress, which may load the module): make it before any
 *     stream capture on that device.
 *   - All calls share the array and it keeps the last call's contents; calls
 *     whose kernels may overlap on the GPU (unordered streams) race on it.
 *   - The address is kept for the life of the process: it does not survive
 *     cudaDeviceReset of that device, after which this entry point must not
 *     be called on it.
 *   - num_splits = 0: the automatic choice, or, when its partials would not
 *     fit the array, the largest explicit split count whose partials do
 *     (down to 1, which needs none). An explicit num_splits whose partials
 *     (paged_decode_workspace_bytes) exceed KV_NOALLOC_SCRATCH_BYTES returns
 *     KV_ERR_WORKSPACE; use fewer splits or the workspace entry point then.
 * Other arguments, errors and results: as paged_decode_attention. */
#define KV_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
int paged_decode_attention_noalloc(float* out, const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t B,
                                   int32_t H_q, int32_t H_kv, int32_t Dh, int32_t page_size, int32_t num_pages,
                                   float scale, int32_t dtype, int32_t num_splits, int* err_flag, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVPAGED_H */
