/*
 * qsa.h -- C ABI of libqsa.so, the B200 (sm_100a) hot path of Qwen Sparse
 * Attention (QSA).
 *
 * The method (pages "Qwen4 architecture: QSA, GR, PLE", section "1. QSA: not
 * looking at every token equally", and "Qwen4 in llama.cpp: Dissecting PR
 * #27742", section "QSA Is an Address-Selection Problem, Not a New Attention
 * Equation"): keys are compressed into per-block summaries, the summaries are
 * scored against the queries, the top-k most relevant contiguous token blocks
 * are selected, and exact softmax attention runs over the selected blocks
 * only.  The selector returns block addresses, not values.
 *
 * Parameterization (the pages give none): key blocks of QSA_BLOCK = 64
 * tokens, mean-pooled summaries; one selection per (query block of 64
 * tokens -- or one token in decode --, KV group), shared by all query heads of
 * the group; block 0 (sink) and the causal diagonal block are always kept
 * and count toward top-k; ties go to the lower block index.
 *
 * Layouts (all dense, row-major, no padding):
 *   Q, O    [B][Tq][Hq][d]        bf16  (query head h is in group h / (Hq/Hkv))
 *   K, V    [B][Hkv][T_kv_max][d] bf16  (cache; a 64-token block of one head
 *                                        is one contiguous 64*d run)
 *   Kc      [B][Hkv][T_kv_max/64][d] fp32 (block summaries)
 *   idx     [B][Hkv][NR][topk]     int32 (NR = ceil(Tq/qblk); ascending block
 *                                        ids, -1 padding at the end)
 *   lse     [B][Tq][Hq]            fp32  (natural-log softmax normaliser)
 * The Tq query tokens sit at absolute positions q_pos0 .. q_pos0+Tq-1 of the
 * cache; their own keys/values must already be written there.
 *
 * Supported: d in {64, 128}; Hq/Hkv in {4, 8}; 2 <= topk <= 64 (decode and
 * score/select: topk <= 64; prefill attention: topk <= 64); every pointer
 * 16-byte aligned; T_kv_max a multiple of 64.  Anything else returns
 * QSA_ERR_UNSUPPORTED (or QSA_ERR_INVALID_ARG for malformed arguments).
 *
 * Beyond the hot path the header declares, each with its own layouts:
 * bf16 summaries (qsa_*_bf16), ragged batches over paged caches
 * (qsa_*_paged, qsa_score_select_ragged*), the Walsh-Hadamard-rotated fp8
 * cache for decode (qsa_quantize_kv_fp8, qsa_decode_fp8*), and the selection
 * variants with other aggregators of the row's tokens and heads
 * (qsa_score_select_token_agg, qsa_score_select_prefill_agg).  Some of them
 * narrow the supported set (d = 128 only for the fp8 cache and the
 * prefill-row aggregators).
 *
 * Ownership and errors: the caller owns every buffer, including the
 * workspace; the library allocates no device memory, except inside the
 * host-buffer prefill pipeline object (qsa_prefill_pipeline_*), which owns
 * the device buffers it stages steps through.  All calls are
 * asynchronous on `stream` (0 = legacy default stream).  Argument checks run
 * on the host before any launch and return an error without launching.
 * A failed launch returns QSA_ERR_CUDA (text in qsa_last_error()).  Errors
 * found by a kernel (a bounded wait that timed out, an index outside the
 * cache) are recorded in a device status word read by
 * qsa_get_device_status().
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_BLOCK 64

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

/* ABI-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st *qsa_stream_t;

typedef enum {
    QSA_OK = 0,
    QSA_ERR_INVALID_ARG = 1, /* null pointer, bad shape or position        */
    QSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported set above  */
    QSA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed          */
    QSA_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out            */
    QSA_ERR_BOUNDS = 5,      /* a kernel met a block index outside its range */
    QSA_ERR_WORKSPACE = 6    /* workspace pointer null or too small        */
} qsa_status;

/*
 * Step 1: compress keys.  Writes the fp32 mean of the 64 keys of every
 * block j in [blk_begin, blk_end) of every (b, KV head):
 *     Kc[b][h][j][:] = (1/64) * sum_{r<64} K[b][h][64 j + r][:]
 * ("compress into small blocks" / "compressed-block representation").
 * The reduction order is fixed, so summaries are bit-reproducible: a
 * summary written incrementally (one block as it completes) equals the one
 * written in a whole-cache pass.  Blocks outside the range are untouched.
 * Requires 0 <= blk_begin <= blk_end <= T_kv_max/64.
 */
QSA_API qsa_status qsa_compress_keys(const void *K, float *Kc, int B, int Hkv, int T_kv_max,
                             int d, int blk_begin, int blk_end, qsa_stream_t stream);

/*
 * Step 1 with bf16 summaries (an option; the default summaries are fp32):
 * the same fp32 mean, stored rounded to the nearest bf16 (ties to even), so
 * that scoring reads half the bytes -- the selection read of a long decode
 * cache is as large as the attention's.  Kc is bf16
 * [B][Hkv][T_kv_max/64][d]; everything else as qsa_compress_keys.
 */
QSA_API qsa_status qsa_compress_keys_bf16(const void *K, void *Kc, int B, int Hkv, int T_kv_max,
                                          int d, int blk_begin, int blk_end, qsa_stream_t stream);

/*
 * Steps 2-4: pool queries, score the block summaries and select the top-k
 * blocks ("indexer scoring" -> "top-k selection").
 *
 * Selection rows: qblk = 64 (prefill; q_pos0 must be a multiple of 64) or
 * qblk = 1 (one selection per query token, e.g. decode with Tq = 1).  Row i
 * covers query tokens [i*qblk, min((i+1)*qblk, Tq)); its diagonal block is
 * D = (q_pos0 + last token of the row) / 64.  Its pooled query is the fp32
 * mean of Q over those tokens and the group's heads, and each candidate
 * block j in [1, D-1] scores s_j = sm_scale * <pooled query, Kc[b][g][j]>
 * in fp32.  The row keeps {0, D} plus the min(topk-2, D-1) best candidates
 * by (s descending, j ascending) -- only {0} when D = 0 -- written ascending
 * into idx[b][g][i][:] and padded with -1.  Summaries of blocks 1 .. D-1
 * must be present in Kc.  Scores are assumed finite.
 *
 * Workspace: qsa_score_select_workspace() bytes, caller-owned, no
 * initialisation needed, must not be shared by concurrent calls.
 */
QSA_API size_t qsa_score_select_workspace(int B, int Hq, int Hkv, int Tq, int q_pos0, int qblk,
                                  int d, int topk);
QSA_API qsa_status qsa_score_select(const void *Q, const float *Kc, int32_t *idx, int B, int Hq,
                            int Hkv, int Tq, int q_pos0, int qblk, int T_kv_max, int d,
                            int topk, float sm_scale, void *workspace,
                            size_t workspace_bytes, qsa_stream_t stream);

/*
 * qsa_score_select over bf16 summaries (as written by qsa_compress_keys_bf16):
 * Kc is bf16 [B][Hkv][T_kv_max/64][d]; each component is widened to fp32
 * exactly and the scores are computed in fp32 as above.  Same workspace
 * (qsa_score_select_workspace), rows, ordering, outputs and errors.
 */
QSA_API qsa_status qsa_score_select_bf16(const void *Q, const void *Kc, int32_t *idx, int B, int Hq,
                                         int Hkv, int Tq, int q_pos0, int qblk, int T_kv_max, int d,
                                         int topk, float sm_scale, void *workspace,
                                         size_t workspace_bytes, qsa_stream_t stream);

/*
 * Allocation-free variant of qsa_score_select.  The pages have no
 * counterpart: it exists for callers that cannot allocate device memory
 * themselves -- e.g. a plug-in or custom operator inside a host engine whose
 * memory planner owns the whole device and forbids side allocations, or a
 * runtime that has no handle on an allocator at the call site.  Same inputs,
 * outputs and results as qsa_score_select, but the workspace is a
 * static device array of QSA_SELECT_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits.  Shapes
 * whose workspace (qsa_score_select_workspace) exceeds that size return
 * QSA_ERR_WORKSPACE without launching.  The function calls no cudaMalloc,
 * cudaFree or other allocating routine.
 * The first call on each device looks up the buffer's device address (with
 * that device current) and caches it; make that first call before any
 * stream capture.  The cached address lives as long as the process's
 * context on that device: after cudaDeviceReset() the library's device
 * memory is gone and this entry point must not be called again in the
 * process.  Every call shares the one buffer and it keeps the last
 * call's contents (nothing in it needs to start at zero), so calls that
 * overlap on the GPU -- on different streams, or from different host
 * threads on the same device -- race with each other: serialise them.
 */
#define QSA_SELECT_SCRATCH_BYTES ((size_t)4 << 20)
QSA_API qsa_status qsa_score_select_noalloc(const void *Q, const float *Kc, int32_t *idx, int B,
                                            int Hq, int Hkv, int Tq, int q_pos0, int qblk,
                                            int T_kv_max, int d, int topk, float sm_scale,
                                            qsa_stream_t stream);

/*
 * Step 5 (prefill): exact softmax attention over the selected blocks
 * ("attention over those cells").  Query token t (position p = q_pos0 + t,
 * selection row t/64) of head h sees the keys u <= p of the blocks listed in
 * idx[b][h/(Hq/Hkv)][t/64][:]:
 *     O[b][t][h][:] = sum_u softmax_u(sm_scale * <q, k_u>) v_u
 * computed flash-style (online softmax, fp32 accumulation in tensor memory,
 * bf16 tensor-core MMA).  Requires q_pos0 % 64 == 0 and q_pos0 + Tq <=
 * T_kv_max; every listed block must satisfy 0 <= j <= D of its row (a
 * violation sets QSA_ERR_BOUNDS in the device status and the row's blocks
 * past the violation are skipped).  lse may be NULL.  No workspace.
 */
QSA_API qsa_status qsa_sparse_attn_prefill(const void *Q, const void *K, const void *V,
                                   const int32_t *idx, void *O, float *lse, int B, int Hq,
                                   int Hkv, int Tq, int q_pos0, int T_kv_max, int d,
                                   int topk, float sm_scale, qsa_stream_t stream);

/*
 * Step 5 (decode): one query token per sequence at position L-1 of its
 * cache (cache length L includes the token itself), attending to the
 * blocks listed in idx[b][g][0][:] (as produced by qsa_score_select with
 * Tq = 1, qblk = 1, q_pos0 = L-1).  q and o are [B][Hq][d] bf16.  Split-K
 * over the selected blocks: up to 8 CTAs per (b, g) form a thread-block
 * cluster and merge their partial softmax states through distributed
 * shared memory.  Needs no workspace: qsa_decode_workspace() returns 0 and
 * `workspace` may be NULL.  B*Hkv <= 65535.
 */
QSA_API size_t qsa_decode_workspace(int B, int Hq, int Hkv, int d, int topk);
QSA_API qsa_status qsa_decode(const void *q, const void *K_cache, const void *V_cache,
                      const int32_t *idx, void *o, int B, int Hq, int Hkv, int L,
                      int T_kv_max, int d, int topk, float sm_scale, void *workspace,
                      size_t workspace_bytes, qsa_stream_t stream);

/*
 * Ragged batches over paged caches (serving).  The selector hands the
 * attention the addresses of the cache cells it may see, and attention runs
 * over those cells only (page "Qwen4 in llama.cpp: Dissecting PR #27742",
 * section "QSA Is an Address-Selection Problem, Not a New Attention
 * Equation"); here a cell is a 64-token page:
 *   K_pages, V_pages  bf16 [num_pages][Hkv][64][d] (page p holds one block of
 *                     one sequence for all KV heads);
 *   block_table       int32 [B][max_blocks] device array: logical block j of
 *                     sequence b lives in page block_table[b][j];
 *   seq_lens          int32 [B] device array: sequence b's cache length,
 *                     1 <= seq_lens[b] <= 64 * max_blocks, its current token
 *                     at position seq_lens[b] - 1;
 *   Kc                fp32 [B][Hkv][max_blocks][d], summaries in logical order.
 * The kernels read lengths, pages and indices on the device and check them
 * before any access: an invalid one sets QSA_ERR_BOUNDS in the device status
 * word and its block is skipped (a sequence with an invalid length outputs
 * zeros).  Host-side checks return errors before any launch as elsewhere.
 *
 * qsa_compress_keys_paged: summaries of the complete blocks
 * (64 (j+1) <= seq_lens[b]) among logical blocks [blk_begin, blk_end) of
 * every sequence; other entries of Kc are untouched.
 * qsa_score_select_ragged: the per-token selection of qsa_score_select
 * (qblk = 1) for one token per sequence, Q [B][1][Hq][d], each at its own
 * position; idx [B][Hkv][1][topk].  max_len >= every seq_lens[b] sizes the
 * launch.  No workspace (UNSUPPORTED past 8 x 8192 candidates).
 * qsa_decode_paged: qsa_decode with each sequence's own length and pages.
 *
 * Chunked prefill of a ragged batch (B requests, Tq new tokens each):
 * sequence b's chunk occupies positions q_pos[b] .. q_pos[b] + Tq - 1
 * (int32 [B] device array; each a multiple of 64 with
 * q_pos[b] + Tq <= 64 * max_blocks), its K/V (cache and chunk) already in
 * its pages and its summaries in Kc (complete blocks; see
 * qsa_compress_keys_paged with seq_lens = q_pos + Tq).
 * qsa_score_select_ragged_prefill: qsa_score_select with qblk = 64 and each
 * sequence at its own position; max_pos (a multiple of 64, >= every
 * q_pos[b]) sizes the launch and the workspace
 * (qsa_score_select_workspace(B, Hq, Hkv, Tq, max_pos, 64, d, topk)); a
 * q_pos[b] above max_pos is an invalid position (QSA_ERR_BOUNDS, the
 * sequence treated as starting at 0).
 * qsa_sparse_attn_prefill_paged: qsa_sparse_attn_prefill over the pages,
 * each sequence at its own position.
 */
QSA_API qsa_status qsa_compress_keys_paged(const void *K_pages, const int32_t *block_table,
                                           const int32_t *seq_lens, float *Kc, int B, int Hkv,
                                           int max_blocks, int num_pages, int d, int blk_begin,
                                           int blk_end, qsa_stream_t stream);
QSA_API qsa_status qsa_score_select_ragged(const void *Q, const float *Kc, const int32_t *seq_lens,
                                           int32_t *idx, int B, int Hq, int Hkv, int max_blocks,
                                           int max_len, int d, int topk, float sm_scale,
                                           qsa_stream_t stream);
QSA_API qsa_status qsa_score_select_ragged_prefill(const void *Q, const float *Kc, const int32_t *q_pos,
                                                   int32_t *idx, int B, int Hq, int Hkv, int Tq,
                                                   int max_blocks, int max_pos, int d, int topk,
                                                   float sm_scale, void *workspace,
                                                   size_t workspace_bytes, qsa_stream_t stream);
QSA_API qsa_status qsa_sparse_attn_prefill_paged(const void *Q, const void *K_pages,
                                                 const void *V_pages, const int32_t *block_table,
                                                 const int32_t *q_pos, const int32_t *idx, void *O,
                                                 float *lse, int B, int Hq, int Hkv, int Tq,
                                                 int max_blocks, int num_pages, int d, int topk,
                                                 float sm_scale, qsa_stream_t stream);
QSA_API qsa_status qsa_decode_paged(const void *q, const void *K_pages, const void *V_pages,
                                    const int32_t *block_table, const int32_t *seq_lens,
                                    const int32_t *idx, void *o, int B, int Hq, int Hkv,
                                    int max_blocks, int num_pages, int d, int topk, float sm_scale,
                                    qsa_stream_t stream);

/*
 * Per-token selection (decode rows: one query token per row) with another
 * way of combining the group's heads than the pooled query.  The pages have
 * the selector score compressed keys against the queries (page "Qwen4 in
 * llama.cpp: Dissecting PR #27742", section "QSA Is an Address-Selection
 * Problem, Not a New Attention Equation") and leave the combination open.
 * With z_h(j) = sm_scale * <q_h, Kc_j> for the group's heads h and the
 * complete blocks j < D before the token's diagonal block D:
 *   QSA_AGG_MEAN         s_j = mean over h of z_h(j) (= qsa_score_select)
 *   QSA_AGG_MAX          s_j = max over the row's tokens of the head mean;
 *                        with one token per row it equals QSA_AGG_MEAN
 *   QSA_AGG_SOFTMAX_SUM  s_j = sum over h of exp(z_h(j)) / sum over j' < D
 *                        of exp(z_h(j')) (block 0 is in the normalisation,
 *                        not among the candidates)
 * then the usual rule: block 0 and D forced, the top (topk - forced) of the
 * candidates 1 .. D-1 by (s descending, index ascending), ascending, -1
 * padded.  Q bf16 [B][Tq][Hq][d] at positions q_pos0 .. q_pos0 + Tq - 1, or
 * with seq_lens (int32 [B], Tq = 1) at seq_lens[b] - 1 with q_pos0 the
 * largest of them (planning); Kc fp32 [B][Hkv][max_blocks][d]; idx int32
 * [B][Hkv][Tq][topk].  Errors: null pointer, bad shape, unknown aggregator
 * or misaligned pointer -> QSA_ERR_INVALID_ARG; d not 64/128, Hq/Hkv > 8,
 * topk outside 2..64 or a row longer than one cluster of chunks holds ->
 * QSA_ERR_UNSUPPORTED; an invalid seq_lens entry -> QSA_ERR_BOUNDS on the
 * device.  Prefill rows (64-token query blocks) with the max or softmax-sum
 * aggregators are not provided.
 */
enum { QSA_AGG_MEAN = 0, QSA_AGG_MAX = 1, QSA_AGG_SOFTMAX_SUM = 2 };
QSA_API qsa_status qsa_score_select_token_agg(const void *Q, const float *Kc, const int32_t *seq_lens,
                                              int32_t *idx, int B, int Hq, int Hkv, int Tq, int q_pos0,
                                              int max_blocks, int d, int topk, float sm_scale, int aggregator,
                                              qsa_stream_t stream);

/*
 * Selection for prefill rows (64-token query blocks) under the max-over-
 * tokens or the softmax-sum aggregator (QSA_AGG_MAX, QSA_AGG_SOFTMAX_SUM; the
 * mean is qsa_score_select_bf16).  With z_{h,t}(j) = sm_scale *
 * <Q[b][t][h], Kc[b][g][j]> over the group's heads h, the block's valid
 * tokens t and the complete blocks j < D before the row's diagonal block D:
 *   QSA_AGG_MAX          s_j = max over t of (mean over h of z_{h,t}(j))
 *   QSA_AGG_SOFTMAX_SUM  s_j = sum over (h, t) of exp(z_{h,t}(j)) / sum over
 *                        j' < D of exp(z_{h,t}(j'))
 * then the usual rule (sink and diagonal forced, top (topk - forced) of the
 * candidates 1 .. D-1 by (s descending, index ascending), ascending, -1
 * padded).  The per-(head, token) logits are a dense contraction and run on
 * the tensor cores, so the summaries are the bf16 option's (Kc bf16
 * [B][Hkv][T_kv_max/64][128] from qsa_compress_keys_bf16: exact products,
 * fp32 sums).  Q bf16 [B][Tq][Hq][128] at positions q_pos0 .. q_pos0+Tq-1
 * (q_pos0 a multiple of 64); idx int32 [B][Hkv][ceil(Tq/64)][topk].  The
 * caller's workspace (16-byte aligned, qsa_score_select_prefill_agg_workspace
 * bytes) holds the score table, the softmax statistics and the chunk lists.
 * Errors: null pointer, unknown aggregator, bad shape or misaligned pointer
 * -> QSA_ERR_INVALID_ARG; the mean, d != 128, Hq/Hkv not 4 or 8, topk
 * outside 2..64 or too large a problem -> QSA_ERR_UNSUPPORTED; a short
 * workspace -> QSA_ERR_WORKSPACE.
 */
QSA_API size_t qsa_score_select_prefill_agg_workspace(int B, int Hq, int Hkv, int Tq, int q_pos0,
                                                      int T_kv_max, int d, int topk, int aggregator);
QSA_API qsa_status qsa_score_select_prefill_agg(const void *Q, const void *Kc, int32_t *idx, int B, int Hq,
                                                int Hkv, int Tq, int q_pos0, int T_kv_max, int d, int topk,
                                                float sm_scale, int aggregator, void *workspace,
                                                size_t workspace_bytes, qsa_stream_t stream);

/*
 * Quantized-KV option for decode (page "Qwen4 in llama.cpp: Dissecting PR
 * #27742", section "Quantized KV Exposed a Backend Storage Invariant"): the
 * cache holds K and V in a Walsh-Hadamard-rotated basis as fp8 e4m3 codes
 * with one fp32 scale per (token, head) row; attention runs in that basis
 * and the output is rotated back.  d = 128.  The selection keeps reading the
 * summaries of the unrotated keys (qsa_compress_keys on the bf16 K): it
 * returns cell addresses, which the rotation does not change.
 *
 * qsa_quantize_kv_fp8: for each of `rows` rows of 128 bf16 values x (row r
 * at X + 128 r): u = WHT(x), the unnormalised 128-point Walsh-Hadamard
 * transform in fp32 (butterfly stages len = 1, 2, ..., 64, each pair
 * becoming (a + b, a - b)); scales[r] = max|u| / 448; codes (row r at
 * codes + 128 r) = e4m3(u / scales[r]), nearest with ties to even,
 * saturating (zeros when the row is zero).  Rows [B][Hkv][T_kv_max] of a
 * cache are rows = B*Hkv*T_kv_max; a single new token's rows can be written
 * alone.
 * qsa_decode_fp8: qsa_decode over such a cache (codes uint8
 * [B][Hkv][T_kv_max][128], scales fp32 [B][Hkv][T_kv_max]); q and o bf16 in
 * the original basis.  Scores are (WHT(q) . u) / 128 = q . k up to the
 * quantization; o = WHT(o') / 128.  idx, L, topk and sm_scale as for
 * qsa_decode (an index past the token's block sets QSA_ERR_BOUNDS on the
 * device and is skipped).  All buffers are the caller's device memory.
 * Errors, before any launch: a null pointer, a bad shape (L > T_kv_max,
 * T_kv_max not a multiple of 64, Hq not a multiple of Hkv) or a pointer not
 * 16-byte aligned (X, codes, q, o, idx, both scale arrays of the decode;
 * the quantizer's scales need 4 bytes) -> QSA_ERR_INVALID_ARG; d != 128,
 * Hq/Hkv not 4 or 8, topk outside 2..64 or a cache of 2^31 rows or more ->
 * QSA_ERR_UNSUPPORTED.  rows == 0 is a no-op.
 */
QSA_API qsa_status qsa_quantize_kv_fp8(const void *X, void *codes, float *scales, int64_t rows, int d,
                                       qsa_stream_t stream);
QSA_API qsa_status qsa_decode_fp8(const void *q, const void *K_codes, const float *K_scales,
                                  const void *V_codes, const float *V_scales, const int32_t *idx,
                                  void *o, int B, int Hq, int Hkv, int L, int T_kv_max, int d,
                                  int topk, float sm_scale, qsa_stream_t stream);

/*
 * qsa_decode_fp8_paged: qsa_decode_paged over a rotated fp8 cache in pages
 * -- codes uint8 [num_pages][Hkv][64][128] and scales fp32
 * [num_pages][Hkv][64] (a page's rows quantized by qsa_quantize_kv_fp8 like
 * any other rows), block_table, seq_lens and idx as for qsa_decode_paged.
 * Device-side checks and errors as for qsa_decode_paged; the argument
 * checks as for qsa_decode_fp8.
 */
QSA_API qsa_status qsa_decode_fp8_paged(const void *q, const void *K_codes, const float *K_scales,
                                        const void *V_codes, const float *V_scales,
                                        const int32_t *block_table, const int32_t *seq_lens,
                                        const int32_t *idx, void *o, int B, int Hq, int Hkv,
                                        int max_blocks, int num_pages, int d, int topk, float sm_scale,
                                        qsa_stream_t stream);

/*
 * One long sequence whose cache is split across GPUs (contiguous block
 * ranges, one per rank).  The pages set the regime -- contexts from 262K
 * tokens up (page "Qwen4 in llama.cpp: Dissecting PR #27742", section "Why
 * Short-Context Tests Can Lie"; the cache of page "Qwen3.8 Flash Next
 * VRAM", section "What It Needs") -- and the selection's two-part cost, so
 * both the scoring and the attention are split by block range and only
 * small lists cross between GPUs.  A chunk of Tq new query tokens at
 * positions q_pos0 .. q_pos0 + Tq - 1 (q_pos0 a multiple of 64; prefill
 * rows of 64 tokens) is processed by every rank r, which holds the blocks
 * [blk_lo, blk_hi) of the sequence (the rank with the chunk's own blocks
 * holds them at the end of its range) and the whole Q:
 *   1. qsa_score_select_local: pooled queries, scores of the rank's own
 *      candidates (blocks j in [blk_lo, blk_hi) with 1 <= j < D of the row;
 *      Kc_local fp32 [B][Hkv][blk_hi - blk_lo][d] holds their summaries),
 *      and per row nlists lists of 62 keys (lists uint64
 *      [B][Hkv][ceil(Tq/64)][nlists][62]): chunk c's top m candidates as
 *      (order-preserving score bits << 32 | ~j), in block order, padded with
 *      0.  nlists >= qsa_select_local_lists(Tq, q_pos0, blk_lo, blk_hi) and
 *      the same on every rank; the workspace is
 *      qsa_score_select_local_workspace() bytes.
 *   2. all ranks' lists gathered in rank order (ranges ascending) as an
 *      all-gather leaves them: [R][B][Hkv][NR][nlists][62];
 *   3. qsa_merge_select_lists (nranks = R): the row's top m of the gathered
 *      keys by
 *      (score descending, block ascending) plus blocks 0 and D -- exactly
 *      qsa_score_select's indices of the whole cache, on every rank;
 *   4. qsa_sparse_attn_prefill_local: attention over the listed blocks the
 *      rank holds (K_local, V_local bf16 [B][Hkv][T_local][d], block j at row
 *      64 (j - blk_lo); T_local >= 64 (blk_hi - blk_lo)), other listed
 *      blocks skipped; O bf16 [B][Tq][Hq][d] normalised over the rank's
 *      keys and lse fp32 [B][Tq][Hq] (required) their natural-log
 *      normaliser, O = 0 and lse = -inf for a row none of whose blocks the
 *      rank holds;
 *   5. the ranks' (O, lse) gathered as O_parts bf16 [R][rows][d] and
 *      lse_parts fp32 [R][rows] (rows = B * Tq * Hq), and qsa_merge_partials:
 *      O = sum_r exp(lse_r - L) O_r, L = log sum_r exp(lse_r) (lse may be
 *      NULL).
 * The gathers are the caller's collectives (e.g. NCCL all-gather).
 * Errors: null pointers, a bad range or shape, nlists below what the range
 * needs or above 64, misaligned pointers -> QSA_ERR_INVALID_ARG; d, topk
 * or group size outside the supported set -> QSA_ERR_UNSUPPORTED; a short
 * workspace -> QSA_ERR_WORKSPACE.  Device-side checks as for
 * qsa_sparse_attn_prefill.
 */
QSA_API int qsa_select_local_lists(int Tq, int q_pos0, int blk_lo, int blk_hi);
QSA_API size_t qsa_score_select_local_workspace(int B, int Hq, int Hkv, int Tq, int q_pos0, int d, int blk_lo,
                                                int blk_hi);
QSA_API qsa_status qsa_score_select_local(const void *Q, const float *Kc_local, uint64_t *lists, int B, int Hq,
                                          int Hkv, int Tq, int q_pos0, int blk_lo, int blk_hi, int nlists, int d,
                                          int topk, float sm_scale, void *workspace, size_t workspace_bytes,
                                          qsa_stream_t stream);
QSA_API qsa_status qsa_merge_select_lists(const uint64_t *lists, int32_t *idx, int B, int Hkv, int Tq, int q_pos0,
                                          int nranks, int nlists, int topk, qsa_stream_t stream);
QSA_API qsa_status qsa_sparse_attn_prefill_local(const void *Q, const void *K_local, const void *V_local,
                                                 const int32_t *idx, void *O, float *lse, int B, int Hq, int Hkv,
                                                 int Tq, int q_pos0, int T_local, int blk_lo, int blk_hi, int d,
                                                 int topk, float sm_scale, qsa_stream_t stream);
QSA_API qsa_status qsa_merge_partials(const void *O_parts, const float *lse_parts, void *O, float *lse, int nparts,
                                      int64_t rows, int d, qsa_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status word
 * (QSA_OK if no kernel recorded an error since the last call).  If detail
 * is not NULL it receives a kernel-specific code (0 if none).  The word
 * keeps the first error until it is read here; a recorded timeout does not
 * cut short the bounded waits of kernels launched after it (they give up
 * early only on a timeout recorded while they wait), but read and clear
 * the word after any error so that later errors are seen.
 */
QSA_API qsa_status qsa_get_device_status(qsa_stream_t stream, int *detail);

/* Test hook for the bounded waits: launches one CTA that waits on an
 * mbarrier nothing will ever complete, with the given limit in
 * nanoseconds, and records QSA_ERR_TIMEOUT in the device status word.
 * The kernel returns normally; the context stays usable. */
QSA_API qsa_status qsa_selftest_wait_timeout(uint64_t timeout_ns, qsa_stream_t stream);

/* Test hook for the FMA-pipe exponential used by the prefill softmax:
 * y[i] = 2^x[i] for n device floats with x <= 8 (Cody-Waite reduction plus a
 * degree-3 polynomial; inputs below -126 are clamped to -126).  Lets a test
 * compare it with the CUDA exp2 on the same device. */
QSA_API qsa_status qsa_selftest_exp2(const float *x, float *y, int n, qsa_stream_t stream);

/* Test hook for the FMA-pipe exponential used by the softmax-sum selection
 * passes: y[i] = 2^x[i] for n device floats with x <= 0 (the same reduction
 * plus a degree-5 polynomial; inputs below -126 are clamped to -126). */
QSA_API qsa_status qsa_selftest_exp2_weight(const float *x, float *y, int n, qsa_stream_t stream);

/*
 * Host-buffer prefill pipeline: the whole prefill step (steps 1-5 as
 * qsa_compress_keys over blocks [0, (q_pos0+Tq)/64), qsa_score_select with
 * qblk = 64 and qsa_sparse_attn_prefill) fed from host memory, the way a
 * serving loop feeds it.  The object owns two device buffer sets (Q, K, V,
 * O, summaries, indices, selection workspace) and three non-blocking
 * streams; each submitted step uploads its Q, K, V on the copy-in stream,
 * runs on the compute stream and downloads its O on the copy-out stream,
 * with events ordering them, so that step k's upload, step k-1's compute
 * and step k-2's download overlap.  Host buffers use the layouts above
 * (Q [B][Tq][Hq][d], K and V [B][Hkv][T_kv_max][d], O [B][Tq][Hq][d], all
 * bf16); they must be page-locked (cudaHostAlloc / cudaHostRegister) for
 * the copies to overlap, and must stay valid and unmodified until the step
 * has completed (qsa_prefill_pipeline_synchronize).
 *
 * create: checks the shape (as the step's entry points would, plus
 * 0 <= q_pos0, q_pos0 % 64 == 0, q_pos0 + Tq <= T_kv_max) before touching
 * the device -- QSA_ERR_INVALID_ARG / QSA_ERR_UNSUPPORTED with *out left
 * NULL -- then allocates on the current device (QSA_ERR_CUDA if that
 * fails, nothing left allocated).  submit: returns once the step is queued;
 * errors of the launches it makes are returned as by the entry points.
 * synchronize: waits for every queued step.  streams: the copy-in, compute
 * and copy-out streams (owned by the object; e.g. to record timing events
 * on).  destroy: waits, then frees everything; NULL is accepted.  After a
 * submit that returned an error the order of the object's buffer reuse is
 * no longer guaranteed: synchronize and destroy it.  One object is not to
 * be used from several host threads at once.
 */
typedef struct qsa_prefill_pipeline qsa_prefill_pipeline;
QSA_API qsa_status qsa_prefill_pipeline_create(qsa_prefill_pipeline **out, int B, int Hq, int Hkv, int Tq,
                                               int q_pos0, int T_kv_max, int d, int topk, float sm_scale);
QSA_API qsa_status qsa_prefill_pipeline_submit(qsa_prefill_pipeline *p, const void *hQ, const void *hK,
                                               const void *hV, void *hO);
QSA_API qsa_status qsa_prefill_pipeline_synchronize(qsa_prefill_pipeline *p);
QSA_API qsa_status qsa_prefill_pipeline_streams(qsa_prefill_pipeline *p, qsa_stream_t *copy_in,
                                                qsa_stream_t *compute, qsa_stream_t *copy_out);
QSA_API qsa_status qsa_prefill_pipeline_destroy(qsa_prefill_pipeline *p);

/* Human-readable name of a status code (static storage). */
QSA_API const char *qsa_status_string(qsa_status s);

/* Number of kernels this library has launched in this process (all
 * threads, all devices); for accounting in benchmarks. */
QSA_API unsigned long long qsa_launch_count(void);

/* Text of the last QSA_ERR_* returned on this host thread (static per
 * thread; empty string if none). */
QSA_API const char *qsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
