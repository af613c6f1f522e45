/*
 * kvb.h -- C ABI of libkvb: decode-step attention over a memory-bounded KV
 * cache, for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every data pointer is a DEVICE pointer owned by the caller. The library
 *   allocates nothing, keeps no pointer after a call returns and holds no
 *   state except one device error word per GPU (see kvb_get_error) and the
 *   fixed scratch array of kvb_decode_attn_noalloc.
 * - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream). Results are valid once the stream has reached the call.
 * - Host-side argument checks run before any launch; a failed check returns
 *   KVB_EINVAL and launches nothing. A launch failure returns KVB_ECUDA.
 *   Inconsistent device data (a length above the capacity, a removal range
 *   outside the cache, ...) cannot be seen on the host: the kernels skip the
 *   offending row, leave it in a defined state and set a bit in the device
 *   error word, which kvb_get_error reports as KVB_EDEVICE. No kernel traps,
 *   asserts or spins without a bound.
 * - "len" is the number of valid slots of a (sequence, kv head); slots
 *   [0, len) hold the cache in slot order, slots beyond len are never read.
 * - t[b] is the position of sequence b's current token. t[b] < 0 marks an
 *   inactive sequence: nothing is inserted and its attention is empty.
 *
 * Sources (web pages) the operations follow:
 *   [TRIM] "Cache What Lasts: Token Retention for Memory-Bounded KV Cache in
 *          LLMs" (ICLR 2026), section 2.1.
 *   [ASM]  "Context Memorization for Efficient Long Context Generation",
 *          background (online-softmax identity, GQA) and core method steps 1-4.
 *   [MEM]  "MEMENTO: Teaching LLMs to Manage Their Own Context", sections on
 *          chunking/compression, the dual information stream and the
 *          systems implementation.
 */
#ifndef KVB_H
#define KVB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvb_status {
    KVB_OK = 0,
    KVB_EINVAL = 1,  /* bad argument, detected on the host; nothing launched */
    KVB_ECUDA = 2,   /* a CUDA runtime call or a launch failed */
    KVB_EDEVICE = 3  /* a kernel met inconsistent device data (kvb_get_error) */
} kvb_status;

typedef void* kvb_stream; /* cudaStream_t */

enum kvb_out_dtype { KVB_OUT_F32 = 0, KVB_OUT_BF16 = 1 };

/* bits of the device error word */
enum kvb_device_error {
    KVB_DERR_LEN = 1u << 0,       /* len < 0 or len > cap */
    KVB_DERR_SPLIT = 1u << 1,     /* split_len * num_splits < len */
    KVB_DERR_RANGE = 1u << 2,     /* compaction range outside [0, len) */
    KVB_DERR_TIMEOUT = 1u << 3,   /* a bounded wait on a copy gave up */
    KVB_DERR_PAGES = 1u << 4,     /* a paged cache needed a page and its free stack was empty */
    KVB_DERR_STEP = 1u << 5       /* kvb_decode_step: a row below its budget (len != M) */
};

/* ------------------------------------------------------------------------
 * kvb_decode_attn -- split-K GQA decode attention with retention bias
 *
 * [TRIM] 2.1: the weight of cached token i in the attention of the token at
 * position t is proportional to exp(q.k_i + (t - i) log beta_i); [ASM] step
 * 1 adds the 1/sqrt(d_h) scale and defines the attention state (a, Z),
 * a = softmax-weighted mean of the values, Z = sum of exp(logit). For query
 * head h of sequence b (kv head g = h / (Hq / Hkv)) and slot s < len[b, g]:
 *
 *     logit_s = scale * (q . k_s) + bias_s,
 *     bias_s  = (float)(t[b] - pos_s) * log_beta_s   (0 when log_beta == NULL)
 *
 * The output state is (o, lse) with o = sum_s softmax(logit)_s v_s and
 * lse = ln sum_s exp(logit_s); an empty state is (o = 0, lse = -inf).
 * Split j covers slots [j*C, min((j+1)*C, len)), C = split_len if
 * split_len > 0, else ceil(len / num_splits). The splits' states are
 * combined with the merge operator of [ASM] step 2 (see kvb_merge_states);
 * by the online-softmax identity ([ASM] background) the result equals
 * attention over all len slots.
 *
 * Layouts (element strides; the innermost dimension d is contiguous):
 *   q        [B, Hq, d]          bf16, strides q_stride_b, q_stride_h
 *   k, v     [B, Hkv, cap, d]    bf16, strides kv_stride_b, kv_stride_h,
 *                                slot stride d; kv_stride_b may be 0 (one
 *                                cache read by every row b)
 *   log_beta [B, Hkv, cap] f32 and pos [B, Hkv, cap] int32, strides
 *            meta_stride_b, meta_stride_h (slot stride 1); log_beta may be
 *            NULL (beta = 1: plain attention), then pos and t may be NULL
 *   len      [B, Hkv] int32, contiguous
 *   t        [B] int32 (NULL: every row active, only allowed without bias)
 *   o        [B, Hq, d] f32 or bf16 (o_dtype), contiguous
 *   lse      [B, Hq] f32, contiguous, may be NULL
 *   o_part   [B, Hq, num_splits, d] f32, lse_part [B, Hq, num_splits] f32:
 *            every split's state; an empty split gets lse = -inf and its o_part
 *            row is left as it was (no merge reads the o of an empty state,
 *            kvb_merge_states included); required when
 *            num_splits > 1, may be NULL when num_splits == 1. With
 *            num_splits > 1 the call launches the attention kernel, which
 *            writes every split's state, and a merge kernel that combines
 *            them into o and lse.
 *   counters reserved: no longer read; pass NULL (kept so that the
 *            struct layout does not change).
 *   evict_cand  [B, Hkv, num_splits] kvb_evict_cand records, may be NULL.
 *            When given, the kernel also writes, for every split, the slot
 *            that budget enforcement at the NEXT position t[b] + 1 would pick
 *            within the split (the smallest (score, pos) with score =
 *            (float)(t[b] + 1 - pos) * log_beta, or 0 when log_beta is NULL;
 *            slot -1 for an empty split), stamped with that position t[b] + 1.
 *            It reads those fields anyway, so kvb_evict_insert can then skip
 *            its scan of the whole cache. Needs pos and t (and meta strides
 *            describing pos), 16-byte alignment; else KVB_EINVAL.
 *
 * Requirements (else KVB_EINVAL): d in {64, 128}; Hq % Hkv == 0 and
 * Hq / Hkv in {1, 2, 4, 8}; B, Hkv, cap >= 1; B * Hq < 2^31;
 * 1 <= num_splits <= 1024;
 * split_len >= 0; q, k, v, o and o_part 16-byte aligned (the outputs are
 * written 16 bytes at a time) and every q/kv stride a multiple
 * of 8 elements; kv_stride_h > 0 when Hkv > 1; scale finite (0 selects
 * 1/sqrt(d)). K and V are read with TMA tensor copies, so a layout the
 * tensor-map encoder refuses also returns KVB_EINVAL.
 * Device-side checks: len in [0, cap] and len <= num_splits * split_len
 * (when split_len > 0); a row that fails gets the empty state. Every wait
 * of a CTA on its copies is bounded (1 s); a CTA that gives up sets
 * KVB_DERR_TIMEOUT, waits (bounded) for the copies it issued and writes the
 * empty state for every split it owns (lse_part = -inf, and with
 * num_splits == 1 o = 0, lse = -inf; its candidate records get slot -1).
 * Preconditions (not checked): log beta finite and <= 0, positions unique
 * per (b, g), pos <= t.
 * ---------------------------------------------------------------------- */
typedef struct kvb_attn_args {
    const uint16_t* q;
    int64_t q_stride_b, q_stride_h;
    const uint16_t* k;
    const uint16_t* v;
    int64_t kv_stride_b, kv_stride_h;
    const float* log_beta;
    const int32_t* pos;
    int64_t meta_stride_b, meta_stride_h;
    const int32_t* len;
    const int32_t* t;
    int32_t B, Hq, Hkv, d, cap;
    float scale;
    int32_t num_splits, split_len;
    float* o_part;
    float* lse_part;
    uint32_t* counters;
    void* o;
    int32_t o_dtype;
    float* lse;
    void* evict_cand;
} kvb_attn_args;

/* Eviction candidate of one split (see evict_cand / kvb_evict_insert). */
typedef struct kvb_evict_cand {
    uint64_t key;   /* order-preserving key of (score, pos) */
    int32_t slot;   /* -1 for an empty split */
    int32_t t;      /* the position the record was scored for (t[b] + 1 of the attention) */
} kvb_evict_cand;

kvb_status kvb_decode_attn(const kvb_attn_args* args, kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_decode_step -- budget enforcement, insertion and attention in one launch
 *
 * [TRIM] 2.1 at inference: a decode step of a cache that holds its budget
 * evicts the slot with the lowest beta_i^(t-i) (kvb_evict_insert), writes the
 * new token there, then attends (kvb_decode_attn). This call does both in the
 * attention's launch, for caches that are full: the previous step's attention
 * already scored every slot for this position and left per-split records
 * (evict_cand), so the victim of row (b, g) is the best of its records; the
 * CTA that reads the victim's tile replaces the staged row with the new token
 * and writes it to the cache. Results equal kvb_evict_insert followed by
 * kvb_decode_attn on the same arguments.
 *
 * - args: as kvb_decode_attn. k, v, log_beta and pos are WRITTEN at the
 *   victim slots (the const qualifiers of kvb_attn_args do not apply here).
 *   args->evict_cand is required: the records for position t[b] + 1 that this
 *   step leaves for the next one.
 * - k_new, v_new [B, Hkv, d] bf16 contiguous, 16-byte aligned; log_beta_new
 *   [B, Hkv] f32, required exactly when args->log_beta is (else KVB_EINVAL).
 * - M: the budget, 1 <= M <= cap. Every active row must hold M slots.
 * - cand_in [B, Hkv, num_splits] kvb_evict_cand: the records the previous
 *   attention left (stamped t[b]); a different array from args->evict_cand
 *   (callers alternate two), 16-byte aligned.
 * - victim [B, Hkv] int32, may be NULL: the slot each row's new token took,
 *   -1 for an inactive row (t < 0).
 * - Rows with t < 0 are inactive (nothing inserted, empty state). When a row's
 *   records were not all scored for t[b] (a skipped position) or name no
 *   slot, the victim comes from a scan of the row's slots, as in
 *   kvb_evict_insert (slower: every CTA reading the row scans it). A row that
 *   is not full (len != M) is not changed: it gets the empty state, victim
 *   -1, and the device error word KVB_DERR_STEP (use kvb_evict_insert +
 *   kvb_decode_attn for such a step). Needs pos and t; no batch stride 0
 *   (kv or meta).
 * ---------------------------------------------------------------------- */
kvb_status kvb_decode_step(const kvb_attn_args* args, const uint16_t* k_new, const uint16_t* v_new,
                           const float* log_beta_new, int32_t M, const kvb_evict_cand* cand_in, int32_t* victim,
                           kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_decode_attn_noalloc -- kvb_decode_attn without caller scratch
 *
 * No counterpart in the pages: this is a deployment convenience. Some
 * callers cannot hand the library temporary device memory: a plugin inside
 * a serving process whose memory pool belongs to someone else, or code that
 * must not call cudaMalloc on the decode path because it synchronizes the
 * device and can stall or fail when memory is fully reserved. For them this
 * entry point computes exactly what kvb_decode_attn computes, with the same
 * arguments, but keeps the split states in one fixed array of
 * KVB_NOALLOC_SCRATCH_BYTES in the library's own device memory (every GPU
 * that loads the library holds it until the process exits).
 *
 * - o_part, lse_part and counters must be NULL (else KVB_EINVAL); o and lse
 *   are the outputs, as for kvb_decode_attn.
 * - A call whose split states would need more than the array, i.e.
 *   256-rounded B*Hq*S*4 + B*Hq*S*d*4 bytes with S = num_splits > 1,
 *   returns KVB_EINVAL and launches nothing. With num_splits == 1 no
 *   scratch is used.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress with that device current); make that first call
 *   before any stream capture.
 * - Every call writes all the split states it reads back, so the array's
 *   previous contents never matter; it calls no cudaMalloc/cudaFree.
 * - All calls share the one array: calls whose execution overlaps on the GPU
 *   (different streams, or different threads with no ordering) race and
 *   corrupt each other's results. Serialize them on one stream.
 * ---------------------------------------------------------------------- */
#define KVB_NOALLOC_SCRATCH_BYTES (16u << 20)

kvb_status kvb_decode_attn_noalloc(const kvb_attn_args* args, kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_merge_states -- n-way merge of attention states
 *
 * [ASM] step 2: merge((a_A, Z_A), (a_B, Z_B)) = ((Z_A a_A + Z_B a_B) /
 * (Z_A + Z_B), Z_A + Z_B), applied across the n states of each row with Z
 * carried as lse = ln Z:
 *     m = max_j lse_j,  lse = m + ln sum_j exp(lse_j - m),
 *     o = sum_j exp(lse_j - lse) o_j;
 * rows whose states are all empty get (0, -inf). The identity element is
 * (0, -inf), so external states (e.g. a stored prefix state) merge the same
 * way. The o of a state with lse = -inf is never read.
 *
 * State j of row r: o_in[j*o_stride_n + r*o_stride_r + e] (e < d, f32) and
 * lse_in[j*lse_stride_n + r*lse_stride_r]. Outputs o_out [R, d] and
 * lse_out [R] (may be NULL), contiguous.
 * Requirements: n >= 1, R >= 0, 1 <= d <= 1024, o_in/o_out 16-byte aligned
 * and o strides multiples of 4 when d % 4 == 0 (else any alignment).
 * ---------------------------------------------------------------------- */
kvb_status kvb_merge_states(const float* o_in, const float* lse_in,
                            int64_t o_stride_n, int64_t o_stride_r,
                            int64_t lse_stride_n, int64_t lse_stride_r,
                            int32_t n, int32_t R, int32_t d,
                            float* o_out, float* lse_out, kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_evict_insert -- budget enforcement and insertion of the new token
 *
 * [TRIM] 2.1, inference: when the cache exceeds the budget M the token with
 * the lowest beta_i^(t-i) is evicted. Per (b, g), for the token at t[b]:
 *   t[b] < 0      nothing changes, victim = -1;
 *   len < M       the token goes to slot len, len += 1, victim = -1;
 *   len >= M      victim = the slot with the smallest (score, pos), compared
 *                 lexicographically, where score = (float)(t - pos) *
 *                 log_beta as ONE float32 multiply rounded to nearest even
 *                 (-0 counts as +0; score = 0 when log_beta is NULL, which
 *                 makes eviction FIFO); the token overwrites that slot and
 *                 len is unchanged.
 * The written slot receives k_new/v_new [B, Hkv, d] (both NULL: K/V are not
 * written, only log_beta and pos), log_beta_new [B, Hkv] (ignored when
 * log_beta is NULL) and pos = t[b].
 * Cache layout: k, v [B, Hkv, cap, d], log_beta, pos [B, Hkv, cap], len
 * [B, Hkv], all contiguous. victim [B, Hkv] int32 (may be NULL).
 * cand, cand_n: optional [B, Hkv, cand_n] kvb_evict_cand records written by
 * the kvb_decode_attn call that immediately preceded this one on the same
 * cache (same scoring: both with or both without log_beta). A (b, g) uses
 * its records only when every one of them is stamped with t[b] (the
 * attention ran at t[b] - 1); when len >= M the victim is then the best
 * record -- the same slot a full scan picks, because the splits partition
 * the slots -- and the scan is skipped. Records stamped for another
 * position (the caller skipped a position, or attended elsewhere in
 * between) or with no usable slot fall back to the scan. 16-byte aligned,
 * 1 <= cand_n <= 1024. NULL: always scan.
 * Requirements: d in [1, 1024] with d % 8 == 0 and k/v/k_new/v_new 16-byte
 * aligned; 1 <= M <= cap. Device-side check: len in [0, cap].
 * ---------------------------------------------------------------------- */
kvb_status kvb_evict_insert(uint16_t* k, uint16_t* v, float* log_beta, int32_t* pos,
                            int32_t* len, const uint16_t* k_new, const uint16_t* v_new,
                            const float* log_beta_new, const int32_t* t,
                            int32_t B, int32_t Hkv, int32_t d, int32_t cap, int32_t M,
                            int32_t* victim, const void* cand, int32_t cand_n, kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_compact_blocks -- in-place removal of a slot range
 *
 * [MEM]: once a thinking block's memento is written, the block's KV entries
 * are physically removed in place and later entries (the memento) are kept
 * bit for bit. For every sequence b with rm_len[b] > 0 and every kv head g:
 * slots [r0, r0 + rl) (r0 = rm_start[b], rl = rm_len[b]) are removed,
 * slots r0 + rl .. len - 1 move to r0 .. len - rl - 1 in order with their
 * K, V, pos (and log_beta, when not NULL) bytes unchanged, and len -= rl.
 * Overlapping moves (more than rl slots after the range) are handled.
 * Layout as kvb_evict_insert. A range outside [0, len) leaves that head
 * untouched and sets KVB_DERR_RANGE.
 * Requirements: d % 8 == 0, k/v 16-byte aligned, cap >= 1.
 * ---------------------------------------------------------------------- */
kvb_status kvb_compact_blocks(uint16_t* k, uint16_t* v, int32_t* pos, float* log_beta,
                              int32_t* len, const int32_t* rm_start, const int32_t* rm_len,
                              int32_t B, int32_t Hkv, int32_t d, int32_t cap,
                              kvb_stream stream);

/* ------------------------------------------------------------------------
 * Paged cache: kvb_paged_reset, kvb_paged_evict_insert,
 * kvb_paged_decode_attn, kvb_paged_compact_blocks
 *
 * [MEM] systems: the engine removes KV entries physically inside generation,
 * and the cache is a sawtooth (chunking and compression) -- a flat cache must
 * reserve the peak length for every sequence, a paged one holds the pages in
 * use. The logical cache of each (sequence b, kv head g) is the flat cache of
 * the calls above (slots [0, len) in slot order); its slots live in pages of
 * KVB_PAGE_SLOTS slots taken from one pool: logical slot s is row
 * s % KVB_PAGE_SLOTS of page table[b, g, s / KVB_PAGE_SLOTS], and pages
 * 0 .. ceil(len / KVB_PAGE_SLOTS) - 1 of the table are set (the last one
 * partly used). Free pages are a stack on the device: free_pages[0 ..
 * *free_count). Each operation computes exactly what its flat counterpart
 * computes on the logical cache:
 *   kvb_paged_evict_insert   = kvb_evict_insert; an append at a page
 *       boundary pops a page from the free stack (none left: the token is not
 *       inserted, victim = -1, KVB_DERR_PAGES);
 *   kvb_paged_decode_attn    = kvb_decode_attn over the logical cache (bias
 *       when log_beta_pages != NULL); every split starts on a page: one split,
 *       or split_len a multiple of KVB_PAGE_SLOTS (else KVB_EINVAL); q is
 *       [B, Hq, d] contiguous, the outputs and evict_cand as kvb_decode_attn;
 *   kvb_paged_compact_blocks = kvb_compact_blocks; the slots after the range
 *       move down through the table (their bytes unchanged) and the pages past
 *       the new length go back on the free stack (their table entries -1);
 *   kvb_paged_reset: every page free (free_pages = 0 .. num_pages - 1 in
 *       order, *free_count = num_pages), every table entry -1, len = 0.
 * Which physical page a logical page gets depends on the order in which
 * CTAs pop the stack; only the logical cache is deterministic.
 * Layouts (contiguous): k_pages, v_pages [num_pages, KVB_PAGE_SLOTS, d] bf16;
 * log_beta_pages (nullable), pos_pages [num_pages, KVB_PAGE_SLOTS]; table
 * [B, Hkv, max_pages] int32; len [B, Hkv]; free_pages [num_pages];
 * free_count [1]. Capacity per (b, g): max_pages * KVB_PAGE_SLOTS slots.
 * Requirements: B, Hkv, max_pages, num_pages >= 1; d % 8 == 0 (d in {64,
 * 128} for the attention); k_pages, v_pages, pos_pages, log_beta_pages
 * 16-byte aligned. A table entry outside [0, num_pages) met on the device
 * sets KVB_DERR_RANGE (the insertion or removal of that head is skipped; the
 * attention reads page 0 in its place).
 * ---------------------------------------------------------------------- */
#define KVB_PAGE_SLOTS 64

typedef struct kvb_paged_cache {
    uint16_t* k_pages;
    uint16_t* v_pages;
    float* log_beta_pages;
    int32_t* pos_pages;
    int32_t* table;
    int32_t* len;
    int32_t* free_pages;
    int32_t* free_count;
    int32_t B, Hkv, d, max_pages, num_pages;
} kvb_paged_cache;

kvb_status kvb_paged_reset(const kvb_paged_cache* cache, kvb_stream stream);

kvb_status kvb_paged_evict_insert(const kvb_paged_cache* cache, const uint16_t* k_new, const uint16_t* v_new,
                                  const float* log_beta_new, const int32_t* t, int32_t M, int32_t* victim,
                                  const void* cand, int32_t cand_n, kvb_stream stream);

kvb_status kvb_paged_decode_attn(const kvb_paged_cache* cache, const uint16_t* q, const int32_t* t, int32_t Hq,
                                 float scale, int32_t num_splits, int32_t split_len, float* o_part,
                                 float* lse_part, void* o, int32_t o_dtype, float* lse, void* evict_cand,
                                 kvb_stream stream);

kvb_status kvb_paged_compact_blocks(const kvb_paged_cache* cache, const int32_t* rm_start, const int32_t* rm_len,
                                    kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_asm_lookup_merge -- attention-state-memory lookup and merge
 *
 * [ASM] steps 3-4. For query token n and head h:
 *   c* = argmax_k cos(q[n,h], qbar[h,k]) (the lowest k among equal values;
 *        cos = 0 when either vector has zero norm);
 *   (o, lse) = merge((o_self, lse_self), (abar[h, c*], log_zbar[h, c*]))
 * with the merge of kvb_merge_states; o_self/lse_self is the query's own
 * attention state (e.g. from kvb_decode_attn).
 * Layouts (contiguous): q [N, H, d] bf16; qbar [H, K, d] f32; abar [H, K, d]
 * bf16; log_zbar [H, K] f32; o_self [N, H, d] f32; lse_self [N, H] f32 ->
 * idx [N, H] int32 (may be NULL), o [N, H, d] f32, lse [N, H] f32 (may be
 * NULL).
 * workspace: device scratch of kvb_asm_workspace_bytes(N, H, K) bytes,
 * 16-byte aligned, contents irrelevant on entry.
 * Requirements: d == 128; N, H, K >= 1; all pointers 16-byte aligned.
 * A (query, head) whose every cosine is NaN retrieves nothing: idx = -1 and
 * (o, lse) = (o_self, lse_self).
 * o == NULL: only idx is computed (it must then be non-NULL; abar, log_zbar,
 * o_self, lse_self and lse may be NULL) -- the assignment step of clustering
 * the calibration queries under the cosine.
 * ---------------------------------------------------------------------- */
size_t kvb_asm_workspace_bytes(int32_t N, int32_t H, int32_t K);

kvb_status kvb_asm_lookup_merge(const uint16_t* q, const float* qbar, const uint16_t* abar,
                                const float* log_zbar, const float* o_self,
                                const float* lse_self, int32_t N, int32_t H, int32_t K,
                                int32_t d, int32_t* idx, float* o, float* lse,
                                void* workspace, size_t workspace_bytes, kvb_stream stream);

/* ------------------------------------------------------------------------
 * Prepared memory: kvb_asm_prepare, kvb_asm_lookup_merge_planes
 *
 * [ASM] steps 3-4 over a memory built once offline. kvb_asm_prepare does the
 * per-centroid work of the lookup once: every centroid row qbar[t, k] is
 * normalised in f32 (x / sqrt(sum x^2); a zero row stays zero) and split
 * exactly into three bf16 parts (hi = rn(x), mid = rn(x - hi), lo = x - hi -
 * mid), written as `planes`, an opaque device buffer of
 * kvb_asm_planes_bytes(H_tables, K) bytes (16-byte aligned) laid out for the
 * lookup's tensor-core tiles (64 centroids per tile, K rounded up to a
 * multiple of 64 with zero rows). qbar [H_tables, K, d] f32, d == 128.
 * kvb_asm_lookup_merge_planes computes exactly what kvb_asm_lookup_merge_grouped
 * computes (same arguments, with planes in place of qbar: the index, the
 * merged state, the assignment-only form with o == NULL, the same workspace).
 * The planes must have been prepared from the same qbar, H_tables and K; they
 * stay valid while qbar is unchanged.
 * ---------------------------------------------------------------------- */
size_t kvb_asm_planes_bytes(int32_t H_tables, int32_t K);

kvb_status kvb_asm_prepare(const float* qbar, int32_t H_tables, int32_t K, int32_t d, void* planes,
                           size_t planes_bytes, kvb_stream stream);

kvb_status kvb_asm_lookup_merge_planes(const uint16_t* q, const void* planes, size_t planes_bytes,
                                       const uint16_t* abar, const float* log_zbar, const float* o_self,
                                       const float* lse_self, int32_t N, int32_t H, int32_t H_tables, int32_t K,
                                       int32_t d, int32_t* idx, float* o, float* lse, void* workspace,
                                       size_t workspace_bytes, kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_asm_hier_lookup_merge -- two-level attention-state-memory lookup
 *
 * [ASM] hierarchical lookup index (technical novelty: retrieval in
 * O(log K) instead of O(K); expanding the top-16 first-level centroids
 * matches the linear top-1). The index is an input, like qbar: per head h,
 * C first-level centroids qhat[h, c] and a partition of the K entries into
 * clusters, listed cluster by cluster: cluster c holds the entries
 * members[h, i] for offsets[h, c] <= i < offsets[h, c + 1]. For query token
 * n and head h:
 *   S  = the m clusters with the largest cos(q[n,h], qhat[h,c]) (the lower c
 *        among equal values; all C when m >= C);
 *   c* = argmax of cos(q[n,h], qbar[h,k]) over the members k of the clusters
 *        in S (the lowest k among equal values);
 *   (o, lse) = merge((o_self, lse_self), (abar[h, c*], log_zbar[h, c*]))
 *        as kvb_asm_lookup_merge; when the clusters in S hold no entry,
 *        idx = -1 and (o, lse) = (o_self, lse_self).
 * Layouts (contiguous): q [N, H, d] bf16; qhat [H, C, d] f32; offsets
 * [H, C + 1] int32 (0 <= offsets[h, c] <= offsets[h, c + 1] <= K); members
 * [H, K] int32 in [0, K); qbar, abar, log_zbar, o_self, lse_self, idx, o,
 * lse as kvb_asm_lookup_merge (idx may be NULL, lse may be NULL).
 * workspace: device scratch of kvb_asm_hier_workspace_bytes(N, H, m) bytes,
 * 16-byte aligned, contents irrelevant on entry. Three launches on
 * `stream`: first-level scores and selection, member scores per selected
 * cluster, reduction + merge.
 * Requirements: d == 128; N, H, K >= 1; 1 <= C <= 1024; 1 <= m <= 64;
 * q, qhat, qbar, abar, o_self, o 16-byte aligned. Offsets out of order or
 * member ids outside [0, K) found on the device are skipped and set
 * KVB_DERR_RANGE.
 * ---------------------------------------------------------------------- */
size_t kvb_asm_hier_workspace_bytes(int32_t N, int32_t H, int32_t m);

kvb_status kvb_asm_hier_lookup_merge(const uint16_t* q, const float* qhat, const int32_t* offsets,
                                     const int32_t* members, const float* qbar, const uint16_t* abar,
                                     const float* log_zbar, const float* o_self, const float* lse_self,
                                     int32_t N, int32_t H, int32_t K, int32_t C, int32_t m, int32_t d,
                                     int32_t* idx, float* o, float* lse,
                                     void* workspace, size_t workspace_bytes, kvb_stream stream);

/* ------------------------------------------------------------------------
 * kvb_asm_aggregate -- attention-aware aggregation (offline memory build)
 *
 * [ASM] core method step 2. For head h and cluster k, over the calibration
 * queries i with idx[i, h] == k (idx < 0: the query is in no cluster):
 *   qbar[h, k]     = mean of q[i, h]
 *   abar[h, k]     = sum Z_i a[i, h] / sum Z_i, with Z_i = exp(lse[i, h])
 *   log_zbar[h, k] = ln sum Z_i (the page's merge operator sums Z); with
 *                    z_mean != 0, ln of the mean of the Z_i
 *   count[h, k]    = number of members
 * An empty cluster gets qbar = 0, abar = 0, log_zbar = -inf, count = 0.
 * Layouts (contiguous): q [M, H, d] bf16; a [M, H, d] f32; lse [M, H] f32;
 * idx [M, H] int32 -> qbar [H, K, d] f32; abar [H, K, d] bf16 (round to
 * nearest even), the format kvb_asm_lookup_merge reads; log_zbar [H, K] f32;
 * count [H, K] int32 (may be NULL). a and lse NULL together: only qbar and
 * count are computed (abar, log_zbar may then be NULL) -- the centroid update
 * of the clustering.
 * workspace: device memory of kvb_asm_aggregate_workspace_bytes(H, K) bytes,
 * 16-byte aligned, contents irrelevant on entry. The sums are fp32 atomics:
 * their rounding order varies between runs.
 * Requirements: d == 128; M, H, K >= 1; q, a, qbar, abar, workspace 16-byte
 * aligned. idx >= K found on the device is skipped and sets KVB_DERR_RANGE.
 * ---------------------------------------------------------------------- */
size_t kvb_asm_aggregate_workspace_bytes(int32_t H, int32_t K);

kvb_status kvb_asm_aggregate(const uint16_t* q, const float* a, const float* lse, const int32_t* idx,
                             int32_t M, int32_t H, int32_t K, int32_t d, int32_t z_mean,
                             float* qbar, uint16_t* abar, float* log_zbar, int32_t* count,
                             void* workspace, size_t workspace_bytes, kvb_stream stream);

/* ------------------------------------------------------------------------
 * Two-level index of a memory (for kvb_asm_hier_lookup_merge)
 *
 * [ASM] hierarchical lookup index, built the way the memory is built: the
 * entries are clustered (kvb_asm_lookup_merge with o = NULL assigns, the
 * query part of kvb_asm_aggregate moves the centroids), which needs them as
 * bf16 queries first:
 * kvb_asm_entries_bf16: qbar [H, K, d] f32 -> q [K, H, d] bf16 (round to
 *   nearest even). d == 128; both 16-byte aligned.
 * kvb_asm_index_csr: from an assignment idx [K, H] int32 (entry k of head h
 *   in cluster idx[k, h]; values outside [0, C) are listed nowhere), writes
 *   offsets [H, C + 1] and members [H, K] int32 in the layout
 *   kvb_asm_hier_lookup_merge reads, every cluster's entries in increasing
 *   order (deterministic). workspace: kvb_asm_index_workspace_bytes(H, C)
 *   bytes, 16-byte aligned. 1 <= C <= 65536.
 * ---------------------------------------------------------------------- */
kvb_status kvb_asm_entries_bf16(const float* qbar, int32_t H, int32_t K, int32_t d, uint16_t* q,
                                kvb_stream stream);

size_t kvb_asm_index_workspace_bytes(int32_t H, int32_t C);

kvb_status kvb_asm_index_csr(const int32_t* idx, int32_t K, int32_t H, int32_t C, int32_t* offsets,
                             int32_t* members, void* workspace, size_t workspace_bytes, kvb_stream stream);

/* ------------------------------------------------------------------------
 * GQA-grouped memory tables ([ASM] GQA extension: a group's queries are
 * aggregated and the centroids stored per KV head)
 *
 * kvb_asm_lookup_merge_grouped / kvb_asm_aggregate_grouped: as
 * kvb_asm_lookup_merge / kvb_asm_aggregate with H_tables tables shared by
 * the H query heads: head h reads (lookup) or feeds (aggregation) table
 * h / (H / H_tables); qbar, abar, log_zbar, count have H_tables rows instead
 * of H. The aggregation folds the calibration rows of all heads of a table
 * together; its workspace is kvb_asm_aggregate_workspace_bytes(H_tables, K).
 * H_tables must divide H. kvb_asm_lookup_merge and kvb_asm_aggregate are the
 * case H_tables == H.
 * ---------------------------------------------------------------------- */
kvb_status kvb_asm_lookup_merge_grouped(const uint16_t* q, const float* qbar, const uint16_t* abar,
                                        const float* log_zbar, const float* o_self, const float* lse_self,
                                        int32_t N, int32_t H, int32_t H_tables, int32_t K, int32_t d,
                                        int32_t* idx, float* o, float* lse, void* workspace,
                                        size_t workspace_bytes, kvb_stream stream);

kvb_status kvb_asm_aggregate_grouped(const uint16_t* q, const float* a, const float* lse, const int32_t* idx,
                                     int32_t M, int32_t H, int32_t H_tables, int32_t K, int32_t d,
                                     int32_t z_mean, float* qbar, uint16_t* abar, float* log_zbar,
                                     int32_t* count, void* workspace, size_t workspace_bytes,
                                     kvb_stream stream);

/* ------------------------------------------------------------------------
 * Errors and diagnostics
 * ---------------------------------------------------------------------- */

/* Synchronizes `stream`, then reads and clears the current GPU's device
 * error word. Returns KVB_OK, KVB_EDEVICE (with the word's bits in *bits
 * when bits != NULL) or KVB_ECUDA. */
kvb_status kvb_get_error(kvb_stream stream, uint32_t* bits);

/* Static text for a status code. */
const char* kvb_status_str(kvb_status s);

/* Version of the ABI described by this header. */
int32_t kvb_abi_version(void);

/* ------------------------------------------------------------------------
 * Testing hook (failure detection without faulting a GPU)
 *
 * kvb_test_withhold_next_decode: the next kvb_decode_attn (or
 * kvb_decode_attn_noalloc) call in this process launches its attention
 * kernel with every producer warp withholding its copies: no copy is issued
 * and no tile is ever signalled, so each CTA's first bounded wait runs out
 * after wait_limit_ns nanoseconds. The kernel then takes its timeout path:
 * KVB_DERR_TIMEOUT in the device error word and the empty state for every
 * split (see kvb_decode_attn). The call returns normally and the context
 * stays usable. One call arms one launch; 1000 <= wait_limit_ns <= 1e9, else
 * KVB_EINVAL. Not for production use.
 * ---------------------------------------------------------------------- */
kvb_status kvb_test_withhold_next_decode(uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* KVB_H */
