/*
 * csa2.h -- C ABI of the CSA2 compressed-sparse-attention library (sm_100a).
 *
 * The operations follow the CSA2 step described on the page
 * [V41] "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression"
 * (fupanwang summary), sections "后 20 层干脆共用一份 KV" and
 * "三个方向一起压小缓存", with the mode semantics corroborated by
 * [NOTES] "DeepSeek-V4.1" (dreamax reading notes).  In short:
 *   - Full layers compute their own main KV and indexer K; the first Full
 *     layer scans the whole visible context, reduces every 8 positions to
 *     their maximum score and keeps the best <= 2048 blocks as the candidate
 *     pool (<= 16384 positions); every layer finally reads 512 entries;
 *   - Reindex layers reuse the nearest Full layer's main KV and indexer K and
 *     select again, only inside the pool;
 *   - Reuse layers take the most recent Top-512 unchanged (no call here);
 *   - main KV is OCP MXFP4, the indexer q/k are FP4, the 128-token sliding
 *     window stays FP8; every m tokens (m = 2 in the encoder, 1 in the
 *     decoder) become one cache entry with no overlap between entries.
 *
 * Conventions for every call
 *   - All array arguments are DEVICE pointers into caller-owned memory unless
 *     a comment says "host".  The library never allocates, never frees and
 *     never synchronises (except csa2_device_status).  Every launch goes to
 *     `stream` (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - Fixed dimensions: main latent D = 512, query heads Hq = 16, indexer
 *     heads Hi = 4, indexer dim Di = 128, block S = 8, window W = 128.
 *   - MXFP4 row of n elements: n/2 bytes of packed E2M1 codes (element 2j in
 *     the low nibble of byte j, sign in bit 3 of the nibble) in the `codes`
 *     plane, and n/32 E8M0 block-scale bytes (scale = 2^(byte-127)) in the
 *     `scales` plane.  Row r starts at codes + r*n/2 and scales + r*n/32.
 *   - Sequence b of a cache occupies rows seq_row_off[b] .. +seq_len[b]-1;
 *     seq_row_off[b] must be a multiple of 8 (one indexer block) and the
 *     cache's `rows` (its capacity) a multiple of 8.
 *   - Scores are ranked by (score descending, position ascending); outputs
 *     holding positions or block ids are sorted ascending and padded with -1.
 *   - workspace: device scratch of at least the size the matching
 *     *_workspace_bytes() function returns, 256-byte aligned, ZERO-FILLED
 *     before its first use.  Its first 256 bytes hold a device status word
 *     that kernels OR flags into (see CSA2_DEV_*); read and clear it with
 *     csa2_device_status().  One workspace must not be used by two calls that
 *     may run concurrently.  Calls keep internal counters and histograms in
 *     the workspace and leave them zero when they finish; after a call that
 *     set a device flag, zero-fill the workspace again before reusing it.
 *     Words 2 and 3 (int32) of the status block are test controls, zero (off)
 *     in a zero-filled workspace: word 2, if nonzero, replaces the pipeline
 *     wait limit of the tensor-core scans (microseconds; built in: 2 s);
 *     word 3, if nonzero, makes each scan CTA's producer withhold the copies
 *     of its first work item so that a wait runs out (CSA2_DEV_TIMEOUT).
 *     They exist to test the timeout path; leave them zero otherwise.
 *     Word 4 is a diagnostic count of selections whose threshold bucket held
 *     more than 12288 keys (they then fall back to global radix passes).
 *   - Return value: CSA2_OK, or a negative error; on an error nothing was
 *     launched, except CSA2_ERR_CUDA (a launch failed; see csa2_last_error()).
 *     Arguments are validated on the host before the first launch.
 *   - Stream order: every call runs after the work enqueued before it on
 *     `stream`, with one refinement.  The kernels here let the stream's next
 *     kernel start early and wait for their results themselves, and the
 *     attention calls read their queries (q) before that wait, so while the
 *     preceding kernel may still run.  No kernel of this library writes a
 *     query; a query written by other earlier work (a copy, or a kernel that
 *     does not trigger the early launch of its dependents) is complete before
 *     it is read.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA2_MAIN_DIM 512
#define CSA2_Q_HEADS 16
#define CSA2_IDX_HEADS 4
#define CSA2_IDX_DIM 128
#define CSA2_BLOCK 8
#define CSA2_WINDOW 128
#define CSA2_MAX_POOL_BLOCKS 2048
#define CSA2_MAX_TOPK 2048

typedef int csa2_status;
#define CSA2_OK 0
#define CSA2_ERR_INVALID_ARG (-1)  /* null pointer, bad size, misaligned pointer */
#define CSA2_ERR_UNSUPPORTED (-2)  /* valid but outside what the kernels handle */
#define CSA2_ERR_WORKSPACE (-3)    /* workspace smaller than *_workspace_bytes() */
#define CSA2_ERR_CUDA (-4)         /* a CUDA launch or runtime call failed */
#define CSA2_ERR_DEVICE_CHECK (-5) /* returned by csa2_device_status() only */

/* Flags of the device status word (OR-ed by kernels, never cleared by them). */
#define CSA2_DEV_INDEX_RANGE 1u    /* a selected index was >= the visible length; it was skipped */
#define CSA2_DEV_ROW_LAYOUT 2u     /* seq_row_off not a multiple of 8, or rows past the capacity; sequence skipped */
#define CSA2_DEV_FP16_RANGE 4u     /* an attention operand lies outside the fp16-exact range; output invalid */
#define CSA2_DEV_LENGTH 8u         /* a device length exceeded the host bound (max_len / n_entries); clamped */
#define CSA2_DEV_TIMEOUT 16u       /* a pipeline wait inside a kernel gave up after its time limit; output invalid */

/* One MXFP4 cache (main KV: n = 512, indexer K: n = 128).  `rows` is the
 * capacity in rows (multiple of 8).  Pointers must be 16-byte aligned. */
typedef struct {
  uint8_t* codes;  /* [rows][n/2]  */
  uint8_t* scales; /* [rows][n/32] */
  int64_t rows;
} csa2_mxfp4_cache;

/* ---------------------------------------------------------------------------
 * csa2_index_full -- Full-mode decode indexer, one query token per sequence.
 * Source: [V41] section "三个方向一起压小缓存", the hierarchical sparse indexer
 * (the first Full layer scores everything, ranks 8-position blocks by their
 * best score and keeps at most 2048 of them as the pool) and its figure.
 * Scores every visible position t < seq_len[b] of sequence b:
 *   s_t = sum_h w_h * (q_h . k_t), computed exactly from the FP4 codes (each
 *   32-block dot product is an exact integer times a power of two; per head the
 *   four block terms are summed in double and rounded once to float; the heads
 *   are combined as s = w0*d0, then fmaf(w_h, d_h, s)); -0 counts as +0.
 * Block maxima over positions [8j, 8j+8) form the ranking of blocks; the pool
 * is the best `pool_blocks` blocks; topk_out is the layer's own Top-k over ALL
 * visible positions.
 *   idx_k       indexer-K cache (n = 128), read only
 *   q_codes     [B][4][64] E2M1 codes of the indexer query (4 heads x 128)
 *   q_scales    [B][4][4]  E8M0 scales of the indexer query
 *   w           [B][4]     fp32 head weights
 *   seq_row_off [B] int64, seq_len [B] int32 (0 <= seq_len <= max_len)
 *   max_len     host: upper bound of seq_len (grid sizing, scores_out stride)
 *   pool_blocks host: P, 1..2048;   k  host: 1..2048
 *   pool_out    [B][P] int32: pool block ids (block j = positions 8j..8j+7)
 *   topk_out    [B][k] int32: selected positions
 *   scores_out  [B][max_len] fp32 or NULL: every visible score
 * ------------------------------------------------------------------------- */
size_t csa2_index_full_workspace_bytes(int B, int max_len, int pool_blocks, int k);
csa2_status csa2_index_full(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                            const float* w, const int64_t* seq_row_off, const int32_t* seq_len, int B,
                            int max_len, int pool_blocks, int k, int32_t* pool_out, int32_t* topk_out,
                            float* scores_out, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * csa2_index_reindex -- Reindex-mode selection inside the pool.
 * Source: [V41] section "三个方向一起压小缓存" (later layers score only inside
 * the pool) and [NOTES] on the modes (Reindex keeps the main KV and selects
 * again).  Scores the positions 8*pool[b][i] + j (j < 8, only
 * those < seq_len[b]; pool entries < 0 are skipped) with THIS layer's indexer
 * query against the nearest Full layer's indexer K, and returns their Top-k.
 * Same score definition and tie rule as csa2_index_full.
 *   pool        [B][P] int32: strictly ascending block ids, then -1 padding,
 *               as csa2_index_full writes them (ties resolve in this order)
 *   topk_out    [B][k] int32
 * ------------------------------------------------------------------------- */
size_t csa2_index_reindex_workspace_bytes(int B, int pool_blocks, int k);
csa2_status csa2_index_reindex(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                               const float* w, const int64_t* seq_row_off, const int32_t* seq_len,
                               const int32_t* pool, int B, int pool_blocks, int k, int32_t* topk_out,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * csa2_sparse_attn_decode -- MXFP4 + FP8 sparse attention, one softmax.
 * Source: [V41] sections "三个方向一起压小缓存" (each layer reads 512 entries;
 * MXFP4 main KV; FP8 window) and "后 20 层干脆共用一份 KV" (128-token window
 * per layer); [NOTES] on the sliding-window branch.  For each sequence b and head h: one softmax over the
 * keys  {dequantised main row seq_row_off[b] + topk[b][j] : topk[b][j] >= 0}
 * followed by the first win_len[b] rows of the FP8 window, each E4M3 value
 * times win_scale[b].  Keys are also the values (shared latent).
 *   logit = sm_scale * (q_h . key);  out = softmax-weighted sum of keys;
 *   lse = log(sum(exp(logit))) (= -inf and out = 0 when there is no key).
 *   q          [B][16][512] bf16 (uint16 bit patterns)
 *   main_kv    main-KV cache (n = 512), read only
 *   topk       [B][k] int32 (-1 = empty slot); k host, 1..2048
 *   win        [B][128][512] E4M3 bytes;  win_scale [B] fp32;  win_len [B] int32 (0..128)
 *   out        [B][16][512] fp32;  lse [B][16] fp32 or NULL
 * Accuracy: max-abs error <= 2e-3 and relative-L2 error <= 1e-3 against exact
 * arithmetic for inputs whose dequantised values are exact in fp16.
 * The workspace size depends on B, k and the current device (how many CTAs
 * share a sequence follows its SM count): query it with the device current on
 * which the call will run.
 * ------------------------------------------------------------------------- */
size_t csa2_sparse_attn_decode_workspace_bytes(int B, int k);
csa2_status csa2_sparse_attn_decode(const uint16_t* q, csa2_mxfp4_cache main_kv, const int64_t* seq_row_off,
                                    const int32_t* seq_len, const int32_t* topk, int k, const uint8_t* win,
                                    const float* win_scale, const int32_t* win_len, float sm_scale, float* out,
                                    float* lse, int B, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * csa2_compress_append -- pair compression + MXFP4 quantisation of new entries.
 * Source: [V41] architecture figure caption (ratio 2 in the encoder, 1 in the
 * decoder), section "三个方向一起压小缓存" (entries have disjoint sources and no
 * absolute position encoding; the indexer K is a projection of the main KV;
 * quantisation comes after positional encoding) and section
 * "后 20 层干脆共用一份 KV" (each layer also projects compression weights).
 * Sequence b contributes raw tokens tok_off[b] .. tok_off[b+1]-1 and appends
 * n_b = (tok_off[b+1]-tok_off[b]) / ratio entries (an odd trailing token of a
 * ratio-2 append is not emitted; resend it with the next call) at cache rows
 * seq_row_off[b] + seq_len_in[b] + j.  seq_len_out[b] = seq_len_in[b] + n_b.
 *   ratio 1: c = x.   ratio 2: entry j merges tokens 2j, 2j+1 with weights
 *     w = softmax(z_2j, z_2j+1) in double (an exp of this library's own), and
 *     c_i = float(fma(w0, x0_i, w1 * x1_i)) in double.
 *   indexer row: w_idx != NULL -> r_o = float(sum_i c_i * w_idx[i][o]) by a
 *     double fma chain in order i = 0..511; else idx_raw merged like x.
 *   Both rows are MXFP4-encoded per OCP MX v1.0: X = floor(log2 amax) - 2,
 *   nearest E2M1 with ties to even, saturating at 6, sign kept.
 *   raw        [n_tok][512] bf16;  logits [n_tok] fp32 (ratio 2; may be NULL for ratio 1)
 *   w_idx      [512][128] fp32 (8-byte aligned) or NULL;  idx_raw [n_tok][128] bf16 or NULL
 *              (exactly one given)
 *   tok_off    [B+1] int64;  seq_row_off [B] int64;  seq_len_in [B], seq_len_out [B] int32
 *   n_tok      host: tok_off[B];  max_new host: upper bound of n_b (grid sizing;
 *              entries beyond it are not written and CSA2_DEV_LENGTH is flagged)
 *   workspace  csa2_compress_append_workspace_bytes(B) bytes (the status word),
 *              256-byte aligned
 * ------------------------------------------------------------------------- */
size_t csa2_compress_append_workspace_bytes(int B);
csa2_status csa2_compress_append(csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k, const uint16_t* raw,
                                 const float* logits, const float* w_idx, const uint16_t* idx_raw,
                                 const int64_t* tok_off, const int64_t* seq_row_off, const int32_t* seq_len_in,
                                 int32_t* seq_len_out, int B, int ratio, int64_t n_tok, int64_t max_new,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * csa2_compress_stream -- ratio-2 append that keeps an odd trailing token on
 * the device (decode: one raw token per sequence per step, and every second
 * token completes an entry).
 * Source: as csa2_compress_append; [V41] architecture figure caption (the
 * compressor merges disjoint pairs of consecutive tokens) applied while
 * generating.
 * Sequence b's token stream is its pending token (if pend_n[b] == 1)
 * followed by raw tokens tok_off[b] .. tok_off[b+1]-1 of this call.  Entries
 * are the stream's pairs (0,1), (2,3), ..., merged, projected and encoded
 * exactly as csa2_compress_append with ratio 2, and written at cache rows
 * seq_row_off[b] + seq_len_in[b] + j.  If the stream has odd length, its last
 * token (bf16 row, logit, idx_raw row) is kept in pend_raw[b], pend_logit[b],
 * pend_idx[b] and pend_n[b] = 1; otherwise pend_n[b] = 0.  Appending a
 * sequence's tokens over any number of calls gives the same cache bytes as
 * one csa2_compress_append of all of them.
 *   pend_n     [B] int32 (0 or 1), read and written in place
 *   pend_raw   [B][512] bf16 (16-byte aligned), pend_logit [B] fp32
 *   pend_idx   [B][128] bf16 (8-byte aligned) when idx_raw is used; NULL with w_idx
 *   seq_len_out [B] receives seq_len_in + entries; it may be seq_len_in
 *              itself (updated in place) or NULL (not written)
 *   logits     required; raw / idx_raw may be NULL when n_tok == 0
 *   max_new    host: upper bound of (pend_n[b] + tokens of b) / 2 (grid sizing)
 *   workspace  csa2_compress_stream_workspace_bytes(B), zero-filled before the
 *              first call (its counters return to zero after each call)
 * Everything else as csa2_compress_append.
 * ------------------------------------------------------------------------- */
size_t csa2_compress_stream_workspace_bytes(int B);
csa2_status csa2_compress_stream(csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k, const uint16_t* raw,
                                 const float* logits, const float* w_idx, const uint16_t* idx_raw,
                                 const int64_t* tok_off, const int64_t* seq_row_off, const int32_t* seq_len_in,
                                 int32_t* seq_len_out, int32_t* pend_n, uint16_t* pend_raw, float* pend_logit,
                                 uint16_t* pend_idx, int B, int64_t n_tok, int64_t max_new, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * csa2_index_prefill -- causal Full-mode indexer for a prefill chunk.
 * Source: [V41] hierarchical indexer (as csa2_index_full), applied to every
 * query of a causal prefill chunk.
 * Query i sits at raw position q_pos[i]; it sees the entries j with
 * (j+1)*ratio - 1 <= q_pos[i] (entry j covers raw tokens ratio*j ..
 * ratio*j+ratio-1), at most n_entries, of the single sequence stored at cache
 * rows row0 .. row0+n_entries-1.  Per query: the same score, block pool and
 * Top-k over all visible entries as csa2_index_full.
 *   q_codes [T][4][64], q_scales [T][4][4], w [T][4], q_pos [T] int32 (>= 0)
 *   row0, n_entries host; ratio 1 or 2; pool_out [T][P]; topk_out [T][k]
 * ------------------------------------------------------------------------- */
size_t csa2_index_prefill_workspace_bytes(int T, int64_t n_entries, int pool_blocks, int k);
csa2_status csa2_index_prefill(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                               const float* w, const int32_t* q_pos, int T, int64_t row0, int64_t n_entries,
                               int ratio, int pool_blocks, int k, int32_t* pool_out, int32_t* topk_out,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * csa2_index_full_pool + csa2_index_full_topk -- csa2_index_full in two
 * calls, so that work which needs only the pool (the Reindex layers) can
 * start while the Full layer's own Top-k is still being selected.
 * Source: as csa2_index_full (the pool and the Full layer's own Top-k are
 * two outputs of the one indexer step there); the split into two calls is
 * this library's scheduling choice.
 * csa2_index_full_pool runs the scan and writes pool_out; a later
 * csa2_index_full_topk on the same stream, with the same arguments, the
 * same workspace (untouched in between) and that pool, writes topk_out.
 * Together they give exactly csa2_index_full's results.
 * ------------------------------------------------------------------------- */
csa2_status csa2_index_full_pool(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const float* w, const int64_t* seq_row_off, const int32_t* seq_len, int B,
                                 int max_len, int pool_blocks, int k, int32_t* pool_out, float* scores_out,
                                 void* workspace, size_t workspace_bytes, void* stream);
csa2_status csa2_index_full_topk(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const float* w, const int64_t* seq_row_off, const int32_t* seq_len, int B,
                                 int max_len, int pool_blocks, int k, const int32_t* pool, int32_t* topk_out,
                                 float* scores_out, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Paged caches: csa2_index_full_paged, csa2_index_reindex_paged,
 * csa2_sparse_attn_decode_paged, csa2_compress_stream_paged.
 * Source: the operations are those of the calls without the suffix and cite
 * the same sections; the pages have no counterpart of the paged layout,
 * which is how serving engines keep KV caches.
 * The same operations, results and errors as the calls without the suffix,
 * for caches kept as fixed-size pages (a serving engine's block tables)
 * instead of one contiguous row range per sequence.  Position t of sequence
 * b lives at cache row
 *     pages[b * max_pages + t / page_rows] * page_rows + t % page_rows
 * (in every cache the call touches, all sharing the page table).
 *   pages      [B][max_pages] int32 physical page ids (4-byte aligned); the
 *              entries for positions >= the sequence's length are not read
 *   page_rows  host: rows per page, a power of two in [512, 2^24] (one scan
 *              work item of 512 rows never crosses a page)
 *   max_pages  host: row stride of `pages` (>= 1); a length above
 *              max_pages * page_rows empties the sequence and sets
 *              CSA2_DEV_ROW_LAYOUT
 * Every cache's `rows` must be a multiple of page_rows.  A page id outside
 * the cache sets CSA2_DEV_ROW_LAYOUT and reads (or writes) page 0 instead,
 * so no access leaves the cache.
 * ------------------------------------------------------------------------- */
csa2_status csa2_index_full_paged(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                  const float* w, const int32_t* pages, int page_rows, int max_pages,
                                  const int32_t* seq_len, int B, int max_len, int pool_blocks, int k,
                                  int32_t* pool_out, int32_t* topk_out, float* scores_out, void* workspace,
                                  size_t workspace_bytes, void* stream);
csa2_status csa2_index_reindex_paged(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                     const float* w, const int32_t* pages, int page_rows, int max_pages,
                                     const int32_t* seq_len, const int32_t* pool, int B, int pool_blocks, int k,
                                     int32_t* topk_out, void* workspace, size_t workspace_bytes, void* stream);
csa2_status csa2_sparse_attn_decode_paged(const uint16_t* q, csa2_mxfp4_cache main_kv, const int32_t* pages,
                                          int page_rows, int max_pages, const int32_t* seq_len, const int32_t* topk,
                                          int k, const uint8_t* win, const float* win_scale, const int32_t* win_len,
                                          float sm_scale, float* out, float* lse, int B, void* workspace,
                                          size_t workspace_bytes, void* stream);
csa2_status csa2_compress_stream_paged(csa2_mxfp4_cache main_kv, csa2_mxfp4_cache idx_k, const uint16_t* raw,
                                       const float* logits, const float* w_idx, const uint16_t* idx_raw,
                                       const int64_t* tok_off, const int32_t* pages, int page_rows, int max_pages,
                                       const int32_t* seq_len_in, int32_t* seq_len_out, int32_t* pend_n,
                                       uint16_t* pend_raw, float* pend_logit, uint16_t* pend_idx, int B,
                                       int64_t n_tok, int64_t max_new, void* workspace, size_t workspace_bytes,
                                       void* stream);

/* ---------------------------------------------------------------------------
 * Context parallelism: one long sequence split over G shards (GPUs), shard g
 * holding entries [lo_g, hi_g) (lo_g a multiple of 8) in its own caches.
 * Source: [V41] hierarchical indexer: the block pool and every Top-k are
 * best-first selections by (score desc, position asc), so the global winners
 * lie in the union of every shard's own winners, ranked by the same keys;
 * attention over disjoint key sets combines through their log-sum-exps.
 * A step: each shard runs csa2_index_full on its range, ranks its pool and
 * Top-k with csa2_score_positions, the shards exchange (key, id) lists (an
 * all-gather), csa2_topk_merge picks the global pool / Top-k and hands each
 * shard its own part; Reindex layers score their shard's part of the pool
 * (csa2_index_reindex + csa2_score_positions + csa2_topk_merge); attention
 * runs per shard on its selected entries (the window on the shard holding
 * the newest tokens), and csa2_attn_combine mixes the partial outputs.
 *
 * csa2_score_positions: the rank key (order-preserving uint32 of the exact
 * score, 0 = absent) of listed positions (block 1) or of listed 8-position
 * blocks (block 8: the maximum over the block's visible positions), for the
 * same query inputs as csa2_index_full.  The keys are bit-identical to the
 * ones the indexer ranks by.
 *   ids [B][n] int32 positions or block ids (< 0: key 0; beyond the visible
 *   length: key 0 and CSA2_DEV_INDEX_RANGE); keys_out [B][n] uint32
 *   workspace: csa2_score_positions_workspace_bytes(B)
 * csa2_topk_merge: per sequence b the k best of the G*n candidates
 * (keys[g][b][i], ids[g][b][i] + src_off[g][b]) by (key desc, id asc), key 0
 * never chosen, written ascending to out [B][k] (-1 padded).  Within a
 * sequence the global ids must ascend with (g, i) (each shard's list
 * ascending, shards in position order), which the lists from
 * csa2_index_full / csa2_index_reindex with src_off = lo_g (or lo_g / 8 for
 * block ids) satisfy.  src_off [G][B] int64 or NULL (ids already global).
 * out_local [B][k] or NULL: out[b][j] - lo[b] where lo[b] <= out[b][j] <
 * hi[b], else -1 (this shard's part, in its own coordinates).
 *   workspace: csa2_topk_merge_workspace_bytes(G, B, n); G*n <= 2^24
 * csa2_attn_combine: out_parts [G][B][16][512] and lse_parts [G][B][16] (from
 * csa2_sparse_attn_decode per shard; a shard with nothing selected has lse
 * -inf) -> out [B][16][512] = sum_g e^(lse_g - M) out_g / sum_g e^(lse_g - M)
 * and lse [B][16] = M + log(sum) (lse may be NULL), M = max_g lse_g.
 * ------------------------------------------------------------------------- */
size_t csa2_score_positions_workspace_bytes(int B);
csa2_status csa2_score_positions(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                                 const float* w, const int64_t* seq_row_off, const int32_t* seq_len,
                                 const int32_t* ids, int B, int n, int block, uint32_t* keys_out, void* workspace,
                                 size_t workspace_bytes, void* stream);
size_t csa2_topk_merge_workspace_bytes(int G, int B, int n);
csa2_status csa2_topk_merge(const uint32_t* keys, const int32_t* ids, const int64_t* src_off, int G, int B, int n,
                            int k, const int64_t* lo, const int64_t* hi, int32_t* out, int32_t* out_local,
                            void* workspace, size_t workspace_bytes, void* stream);
csa2_status csa2_attn_combine(const float* out_parts, const float* lse_parts, int G, int B, float* out, float* lse,
                              void* stream);

/* ---------------------------------------------------------------------------
 * csa2_index_multi -- Full-mode indexer for a batch of sequences with several
 * queries each (the candidate tokens of a speculative-decoding verification
 * step), reading every sequence's indexer K once for all of its queries.
 * Source: [V41] hierarchical indexer (as csa2_index_full) and section
 * "DSpark" (several draft positions per request verified in one forward,
 * the verification length chosen per request).
 * Sequence b owns queries q_off[b] .. q_off[b+1]-1 (ascending offsets within
 * [0, Q]); query i sees the first q_vis[i] entries of its sequence (cache
 * rows seq_row_off[b] ..).  Per query: the same score, block pool and Top-k
 * as csa2_index_full over its visible entries (the pool fast path, so
 * pool_blocks >= k).
 *   q_codes [Q][4][64] (16-byte aligned), q_scales [Q][4][4], w [Q][4]
 *   seq_row_off [B] int64 (multiples of 8); q_off [B+1] int32; q_vis [Q] int32
 *   max_vis    host: upper bound of q_vis (larger values are clamped and
 *              flagged CSA2_DEV_LENGTH)
 *   pool_out [Q][P], topk_out [Q][k] (queries of no sequence get -1 rows)
 *   q_row_off_out [Q] int64 or NULL: receives each query's seq_row_off, so
 *              that csa2_index_reindex and csa2_sparse_attn_decode can take
 *              the queries as Q segments (row offsets q_row_off_out, lengths
 *              q_vis)
 * ------------------------------------------------------------------------- */
size_t csa2_index_multi_workspace_bytes(int B, int Q, int64_t max_vis, int pool_blocks, int k);
csa2_status csa2_index_multi(csa2_mxfp4_cache idx_k, const uint8_t* q_codes, const uint8_t* q_scales,
                             const float* w, const int64_t* seq_row_off, const int32_t* q_off, const int32_t* q_vis,
                             int B, int Q, int64_t max_vis, int pool_blocks, int k, int32_t* pool_out,
                             int32_t* topk_out, int64_t* q_row_off_out, void* workspace, size_t workspace_bytes,
                             void* stream);

/* ---------------------------------------------------------------------------
 * csa2_sparse_attn_prefill -- causal sparse attention of a prefill chunk.
 * Source: as csa2_sparse_attn_decode ([V41] sections "三个方向一起压小缓存"
 * and "后 20 层干脆共用一份 KV"), applied to every query of a causal chunk
 * with the visibility rule of csa2_index_prefill.
 * Query i attends its selected entries (topk[i][j] >= 0, each < the visible
 * count of csa2_index_prefill) and the raw FP8 window rows
 * max(0, q_pos[i]-127) .. q_pos[i] of raw_win (one fp32 scale), in one
 * softmax; otherwise as csa2_sparse_attn_decode.
 *   q [T][16][512] bf16; topk [T][k]; raw_win [n_raw][512] E4M3 (q_pos < n_raw)
 *   out [T][16][512] fp32; lse [T][16] fp32 or NULL
 * ------------------------------------------------------------------------- */
size_t csa2_sparse_attn_prefill_workspace_bytes(int T, int k);
csa2_status csa2_sparse_attn_prefill(const uint16_t* q, const int32_t* q_pos, int T, csa2_mxfp4_cache main_kv,
                                     int64_t row0, int64_t n_entries, int ratio, const int32_t* topk, int k,
                                     const uint8_t* raw_win, int64_t n_raw, float win_scale, float sm_scale,
                                     float* out, float* lse, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* ---------------------------------------------------------------------------
 * csa2_sparse_attn_decode_noalloc -- csa2_sparse_attn_decode without a
 * workspace, for callers that may not allocate device memory while they run
 * (for example a plugin inside another inference runtime that owns all
 * allocations, or a serving loop held to a fixed memory budget).  The pages
 * have no counterpart of this call; it is a deployment convenience.
 * Same arguments, results and accuracy as csa2_sparse_attn_decode, except:
 *   - no workspace: the scratch is a fixed 8,421,888-byte array of device
 *     memory inside this library, which every GPU where the library's device
 *     code is loaded keeps until the process exits;
 *   - when that memory is committed: under CUDA's lazy module loading (the
 *     default) the array and the attention kernel are loaded on a device the
 *     first time a call touches them there, so the first call per device may
 *     allocate (once).  A call with B = 0 does exactly that set-up on the
 *     current device and launches nothing (the other pointers are not read):
 *     make it outside the region where allocation is forbidden and before any
 *     stream capture.  Every later call on that device allocates nothing;
 *   - limits: B <= 64 and k <= 512; larger problems return
 *     CSA2_ERR_UNSUPPORTED with a message, and nothing is launched;
 *   - flags_out: device uint32 that receives this call's CSA2_DEV_* flags, or
 *     NULL;
 *   - the scratch's device address is looked up once per device and kept for
 *     the life of the process: do not use the library across a
 *     cudaDeviceReset;
 *   - all calls on a device share the one scratch array: calls that may run
 *     at the same time on the GPU (different streams, or different host
 *     threads) race and corrupt each other's results.  Serialise them.
 * ------------------------------------------------------------------------- */
csa2_status csa2_sparse_attn_decode_noalloc(const uint16_t* q, csa2_mxfp4_cache main_kv, const int64_t* seq_row_off,
                                            const int32_t* seq_len, const int32_t* topk, int k, const uint8_t* win,
                                            const float* win_scale, const int32_t* win_len, float sm_scale,
                                            float* out, float* lse, uint32_t* flags_out, int B, void* stream);

/* Synchronises `stream`, returns the status word of `workspace` in *flags
 * (CSA2_DEV_* bits) and clears it.  Returns CSA2_ERR_DEVICE_CHECK when any
 * flag was set, CSA2_OK otherwise.  Test and debugging helper. */
csa2_status csa2_device_status(void* workspace, void* stream, uint32_t* flags);

/* Static text of a status code, and the message of the last CSA2_ERR_* of the
 * calling host thread ("" if none). */
const char* csa2_status_string(csa2_status s);
const char* csa2_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
