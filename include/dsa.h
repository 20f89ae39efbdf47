/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention (DSA) forward library, libdsa.so.
 *
 * The method ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models", velog.io summary,
 * DeepSeek Sparse Attention section):
 *   1. lightning indexer (section 1.1):  I[t,s] = sum_{j<H_I} w[t,j] * ReLU(q_I[t,j] . k_I[s]),  s <= t;
 *   2. fine-grained token selection (section 1.2): S_t = the k positions s with the largest I[t,s]
 *      (ties broken by the smaller s; every s <= t when t + 1 <= k);
 *   3. MLA in MQA mode (section 1.3): u_t[h] = softmax_{s in S_t}(scale * q[t,h] . c_s) . c_s[:D_v], with
 *      one shared latent entry c_s per token for all query heads.
 *
 * Conventions common to every entry point:
 *   - Pointers are DEVICE pointers owned by the caller, row-major and contiguous.  FP8 tensors are e4m3fn
 *     bit patterns (uint8_t), bf16 tensors are bf16 bit patterns (uint16_t).  Tensors read by TMA (q_idx,
 *     k_idx, q, c and the caches) must start on a 16-byte boundary.
 *   - `stream` is a cudaStream_t passed as void*; every call is asynchronous on it and never synchronises
 *     the device, except dsa_get_device_status().
 *   - Arguments are checked on the host before anything is launched; a failed check returns an error code
 *     and launches nothing.  Errors found while kernels run (an index out of range, a pipeline wait that ran
 *     out of time) are recorded in a device status word read by dsa_get_device_status().
 *   - Nothing is allocated inside a call: scratch memory is a caller-provided workspace whose size the
 *     matching *_workspace_size() function returns.  The one exception is dsa_forward_decode_noalloc, whose
 *     scratch is a fixed array inside the library (no workspace argument, and still no allocation).
 *   - Supported shapes: H_I in {4, 64} with d_I = 64 / 128 respectively, H <= 128 query heads, D = 576 latent
 *     dims of which the first D_v = 512 are the value, k a multiple of 64 from 128 to 2048.  Other shapes
 *     return DSA_ERR_UNSUPPORTED_SHAPE.
 *   - Results are bitwise deterministic for fixed inputs and launch configuration.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,        /* null pointer, negative size, ... */
  DSA_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside the compiled set */
  DSA_ERR_ALIGNMENT = 3,          /* a TMA-read tensor is not 16-byte aligned */
  DSA_ERR_CUDA = 4,               /* a CUDA runtime / driver call failed */
  DSA_ERR_TIMEOUT = 5,            /* device: a pipeline wait ran out of its clock budget */
  DSA_ERR_BAD_INDEX = 6,          /* device: a selected index was outside [-1, S) (treated as -1) */
  DSA_ERR_WORKSPACE = 7,          /* workspace missing or smaller than *_workspace_size() */
  DSA_ERR_CHECK = 8               /* device, DSA_CHECKS builds only: pipeline bookkeeping or a result invariant
                                     failed (see dsa_checks_enabled) */
} dsa_status_t;

/* Human-readable name of a status code (static storage). */
DSA_API const char* dsa_status_string(dsa_status_t status);

/* Synchronises `stream`, then reads and clears the device status word of the current device.
 * *device_status receives DSA_OK or the first device-side error since the last call. */
DSA_API dsa_status_t dsa_get_device_status(void* stream, int* device_status);

/* Self-check of failure detection: launches one small kernel whose two warps run the library's bounded
 * pipeline wait on barriers that nothing arrives on.  Warp 0 runs out of its clock budget (about a second),
 * which records DSA_ERR_TIMEOUT in the device status word and raises the block's abort flag; warp 1 starts
 * waiting half a budget later and must leave on that flag.  The kernel then returns normally and the context
 * stays usable.  result: caller-owned device array of 4 int32 (16-byte aligned), written as
 * [warp 0 succeeded (0/1), warp 0's wait in 2^20 cycles, warp 1 succeeded, warp 1's wait in 2^20 cycles].
 * Asynchronous on `stream`; read the status with dsa_get_device_status afterwards.  Returns
 * DSA_ERR_INVALID_ARG for a null result, DSA_ERR_ALIGNMENT for a misaligned one, DSA_ERR_CUDA if the launch
 * fails.  This entry point has no counterpart in the paper. */
DSA_API dsa_status_t dsa_check_bounded_wait(int32_t* result, void* stream);

/* Number of SMs the launches of the current device are sized for (148 on a B200). */
DSA_API int dsa_num_sms(void);

/* 1 in a library built with -DDSA_CHECKS (libdsa_checks.so), 0 otherwise.  That debug build runs the same
 * kernels with checks that record DSA_ERR_CHECK or DSA_ERR_BAD_INDEX in the device status word (read it with
 * dsa_get_device_status), and otherwise leave every result as the normal build computes it:
 *   - indexer: the TMA producer, the MMA issuer and the epilogue count the key tiles and accumulator stages they
 *     pass through, and the counts must agree when the kernel ends; every key tile and query group it loads
 *     starts inside its tensor;
 *   - top-k: a check kernel after each top-k launch verifies every output row: min(k, n) entries, strictly
 *     ascending, each in [0, n) for the row's n keys, then -1 (the selection rule of the velog.io DSA page,
 *     §1.2, leaves exactly that many);
 *   - attention: wherever a token's key count is known (the prefill and decode paths, not dsa_sparse_mla_attn),
 *     a selected entry must lie below it (causality), else DSA_ERR_BAD_INDEX; every warp that walks the
 *     tokens' key tiles counts them, and the counts of a CTA's warps must agree.
 * The checks cost time; the normal build compiles none of them. */
DSA_API int dsa_checks_enabled(void);

/* Self-test of the DSA_CHECKS build: plants one violation the checks must catch, on `stream`.
 *   which = 0: a top-k output row that is not ascending -> the device status becomes DSA_ERR_CHECK;
 *   which = 1: a selected entry beyond its token's key count (inside the latent) -> DSA_ERR_BAD_INDEX.
 * scratch: caller-owned device buffer of dsa_checks_selftest_bytes() bytes (16-byte aligned), overwritten.
 * Read the outcome with dsa_get_device_status.  Returns DSA_ERR_UNSUPPORTED_SHAPE in the normal build (nothing
 * launched), DSA_ERR_INVALID_ARG for a null scratch or another `which`.  No counterpart in the paper. */
DSA_API size_t dsa_checks_selftest_bytes(void);
DSA_API dsa_status_t dsa_checks_selftest(int which, void* scratch, void* stream);

/*
 * Lightning-indexer scores, materialised for T query rows (velog.io section 1.1).
 *   q_idx   [T, H_I, d_I] e4m3   indexer queries of rows 0..T-1, whose absolute positions are pos0..pos0+T-1
 *   q_scale [T] fp32 or NULL     per-token dequantisation scale of q_idx (NULL: 1)
 *   k_idx   [S, d_I] e4m3        indexer keys of positions 0..S-1
 *   k_scale [S] fp32 or NULL     per-token dequantisation scale of k_idx (NULL: 1)
 *   w       [T, H_I] fp32        indexer head weights
 *   scores  [T, S] fp32 (out)    I[pos0 + r, s] for s <= pos0 + r, -INFINITY for s > pos0 + r
 * Scores are accumulated in fp32 from exact e4m3 x e4m3 products, so integer-valued inputs with |I| < 2^24
 * give exact scores.  Needs no workspace.
 */
DSA_API dsa_status_t dsa_indexer_scores(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                const float* k_scale, const float* w, int T, int S, int H_I, int d_I,
                                int pos0, float* scores, void* stream);

/*
 * Row-wise top-k selection (velog.io section 1.2) over materialised scores.
 *   scores  [rows, ld] fp32      row r holds n_r valid scores in columns 0..n_r-1
 *   row_len [rows] int32 or NULL n_r (device array); NULL means n_r = min(ld, pos0 + r + 1) (causal rows)
 *   idx     [rows, k] int32 (out) the min(k, n_r) columns with the largest scores, ties to the smaller
 *                                column, in ascending column order, padded with -1
 * -0.0 and +0.0 compare equal; NaN ranks below every number.  Needs no workspace.
 */
DSA_API dsa_status_t dsa_topk(const float* scores, int rows, int64_t ld, const int32_t* row_len, int pos0, int k,
                      int32_t* idx, void* stream);

/*
 * Sparse MLA attention in MQA mode over selected latent entries (velog.io sections 1.2 and 1.3).
 * k is a multiple of 64 between 128 and 2048; idx must be 16-byte aligned.
 *   q     [T, H, 576] bf16    queries (H <= 128)
 *   c     [S, 576] bf16       shared latent entries; the value of an entry is its first 512 dims
 *   idx   [T, k] int32        selected entries of each row, in [0, S) or -1 (= nothing), any order
 *   out   [T, H, 512] bf16 (out)  softmax(scale * q . c_s) . c_s[:512] over the selected s
 *   lse   [T, H] fp32 or NULL (out)  natural-log log-sum-exp of the scaled logits (-INF for an empty row)
 * A row with no selected entry gets out = 0.  Indices outside [-1, S) are treated as -1 and recorded as
 * DSA_ERR_BAD_INDEX.  Needs no workspace.
 */
DSA_API dsa_status_t dsa_sparse_mla_attn(const uint16_t* q, const uint16_t* c, int S, const int32_t* idx, int T,
                                 int H, int k, float scale, uint16_t* out, float* lse, void* stream);

/*
 * The indexer's training objective (velog.io page, Stage 1 Dense Warm-up): for each query token t,
 *   kl[t] = KL(p_t || Softmax(I_t)),  p_t = the heads' attention probabilities summed and L1-normalised,
 * both distributions taken over the token's selected entries (all s <= t in the dense warm-up, where the selection
 * is every earlier token; the selected set S_t in sparse training, a reading of the page, which does not say it).
 *   q [T, H, 576] bf16, c [S, 576] bf16, idx [T, k] int32: as in dsa_sparse_mla_attn;
 *   sel_scores [T, k] fp32: the index score I[t, idx[t][i]] of each selected entry (ignored where idx is -1);
 *   lse [T, H] fp32: the attention's natural-log log-sum-exp per head over the same entries (dsa_sparse_mla_attn's
 *     lse output), from which the probabilities are formed;
 *   kl [T] fp32 (out): the divergence in nats (0 for a token without entries).
 * The logits are recomputed on the tensor cores as in the attention.  Needs no workspace.
 */
DSA_API dsa_status_t dsa_indexer_kl(const uint16_t* q, const uint16_t* c, int S, const int32_t* idx,
                                    const float* sel_scores, const float* lse, int T, int H, int k, float scale,
                                    float* kl, void* stream);

/* Workspace bytes of dsa_forward_prefill_kl. */
DSA_API size_t dsa_prefill_kl_workspace_size(int L, int H_I, int d_I, int H, int k);

/*
 * dsa_forward_prefill plus the indexer objective of every row: the selection also scores the rows t < k (the
 * objective needs their index scores), the attention writes out and lse, and kl [L] fp32 (out) receives
 * KL(p_t || Softmax(I_t)) over each row's selected entries, as dsa_indexer_kl.  L_I is the sum of kl over the
 * rows.  Other arguments as in dsa_forward_prefill (lse may be NULL: the workspace then holds it).
 */
DSA_API dsa_status_t dsa_forward_prefill_kl(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                            const float* k_scale, const float* w, const uint16_t* q,
                                            const uint16_t* c, int L, int H_I, int d_I, int H, int k, float scale,
                                            int32_t* idx_out, uint16_t* out, float* lse, float* kl, void* ws,
                                            size_t ws_bytes, void* stream);

/* Number of kernels this library has launched in this process (all devices, all entry points). */
DSA_API uint64_t dsa_launch_count(void);

/* Rows of the score block that dsa_prefill_select (and dsa_forward_prefill) processes next, starting at row r0
 * of an L-row prefill with selection size k: rows r0 < k form one block (their selection needs no scores);
 * later blocks hold the workspace's row count (about 1 GiB of fp32 scores at L keys, at least 256 rows).
 * 0 when r0 is outside [0, L) or L, k <= 0.  Host function, no GPU. */
DSA_API int dsa_prefill_block_rows(int L, int k, int r0);

/* Workspace bytes of dsa_prefill_select and dsa_forward_prefill for these shapes. */
DSA_API size_t dsa_prefill_workspace_size(int L, int H_I, int d_I, int H, int k);

/*
 * Steps 1-2 for one causal prefill sequence of L tokens: the lightning-indexer scores of every row (s <= t)
 * and their top-k selection (velog.io sections 1.1-1.2).
 *   q_idx [L, H_I, d_I] e4m3, q_scale [L] or NULL, k_idx [L, d_I] e4m3, k_scale [L] or NULL, w [L, H_I] fp32;
 *   idx_out [L, k] int32 (out): the selected positions of each row, ascending, padded with -1.
 * The L x L score matrix is never stored (the workspace holds a bounded block of rows).  A block whose rows all
 * have t + 1 <= k (every prefill with L <= k) needs no scores: each of its rows selects all of 0..t, and the
 * indexer is not launched for it.
 */
DSA_API dsa_status_t dsa_prefill_select(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                        const float* k_scale, const float* w, int L, int H_I, int d_I, int k,
                                        int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Whole DSA forward for one causal prefill sequence of L tokens (steps 1-3 above, s <= t).
 *   q_idx [L, H_I, d_I] e4m3, q_scale [L] or NULL, k_idx [L, d_I] e4m3, k_scale [L] or NULL, w [L, H_I] fp32,
 *   q [L, H, 576] bf16, c [L, 576] bf16;
 *   idx_out [L, k] int32 (out, may be NULL): the selected positions of each row (ascending, -1 padded);
 *   out [L, H, 512] bf16 (out); lse [L, H] fp32 (out, may be NULL).
 * The L x L score matrix is never stored.
 */
DSA_API dsa_status_t dsa_forward_prefill(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                 const float* k_scale, const float* w, const uint16_t* q, const uint16_t* c,
                                 int L, int H_I, int d_I, int H, int k, float scale, int32_t* idx_out,
                                 uint16_t* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Device workspace bytes of dsa_forward_prefill_host: the prefill's workspace plus device copies of every input and
 * output. */
DSA_API size_t dsa_prefill_host_workspace_size(int L, int H_I, int d_I, int H, int k);

/*
 * dsa_forward_prefill with every input and output in HOST memory (steps 1-3 for one causal sequence, as
 * dsa_forward_prefill; same arguments, HOST pointers; lse and idx_out may be NULL).  The call moves the data
 * itself and overlaps the transfers with the kernels: the indexer's inputs are copied first; then, in
 * 16 chunks of rows, each chunk's selection runs while later queries are still arriving, each chunk's attention
 * starts once its queries have landed, and its results go back while the next chunk computes.  Host-to-device
 * and device-to-host copies run on two copy streams of the library's own (created once per device on first
 * use), so both directions of the host link are busy at once.  For the copies to be asynchronous the host
 * buffers must be page-locked (cudaHostAlloc / cudaHostRegister); pageable buffers work but serialise.
 *   ws: DEVICE workspace of dsa_prefill_host_workspace_size() bytes (it holds the device copies).
 * Everything is enqueued on `stream`: when `stream` reaches the end of the call's work, the host outputs hold the
 * results.  The host inputs must stay unchanged and the host outputs unread until then.
 */
DSA_API dsa_status_t dsa_forward_prefill_host(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                              const float* k_scale, const float* w, const uint16_t* q,
                                              const uint16_t* c, int L, int H_I, int d_I, int H, int k, float scale,
                                              int32_t* idx_out, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                                              void* stream);

/* Workspace bytes of dsa_forward_prefill_rows for the rows [row0, row0 + nrows) of a sequence. */
DSA_API size_t dsa_prefill_rows_workspace_size(int row0, int nrows, int H_I, int d_I, int H, int k);

/*
 * Steps 1-3 for the rows [row0, row0 + nrows) of one causal sequence: a block of query rows that attends to all of
 * the sequence's keys up to its own positions.  With the sequence's rows split over several GPUs (each GPU
 * computes the query-side tensors of its own rows and receives every key-side tensor), each GPU calls this for
 * each of its blocks.  The pages describe the computation of one sequence; this is that computation for a
 * subset of its rows.  Results are bitwise identical to the same rows of dsa_forward_prefill.
 *   q_idx [nrows, H_I, d_I] e4m3, q_scale [nrows] or NULL, w [nrows, H_I] fp32, q [nrows, H, 576] bf16: the
 *     block's query-side tensors (row i is position row0 + i);
 *   k_idx [>= row0 + nrows, d_I] e4m3, k_scale [>= row0 + nrows] or NULL, c [>= row0 + nrows, 576] bf16: the
 *     sequence's key-side tensors from position 0 (rows past row0 + nrows - 1 are not read);
 *   idx_out [nrows, k] int32 (out, may be NULL), out [nrows, H, 512] bf16 (out), lse [nrows, H] fp32 (out, may be
 *     NULL), as in dsa_forward_prefill.
 */
DSA_API dsa_status_t dsa_forward_prefill_rows(const uint8_t* q_idx, const float* q_scale, const uint8_t* k_idx,
                                              const float* k_scale, const float* w, const uint16_t* q,
                                              const uint16_t* c, int row0, int nrows, int H_I, int d_I, int H, int k,
                                              float scale, int32_t* idx_out, uint16_t* out, float* lse, void* ws,
                                              size_t ws_bytes, void* stream);

/* Workspace bytes of dsa_forward_prefill_varlen: nseq sequences of `total` rows in all, the longest max_len. */
DSA_API size_t dsa_prefill_varlen_workspace_size(int nseq, int64_t total, int max_len, int H_I, int d_I, int H,
                                                 int k);

/*
 * Steps 1-3 for a batch of independent causal prefill sequences packed one after another ("varlen").  The
 * pages describe one sequence; this is that computation for each sequence of the batch.
 * Sequence b holds rows [cu_seqlens[b], cu_seqlens[b + 1]) of every per-row array.  Its positions and its
 * selected indices count from its first row, and it attends only to its own rows.
 *   cu_seqlens: HOST array of nseq + 1 int64; cu_seqlens[0] = 0, non-decreasing (empty sequences allowed),
 *     total = cu_seqlens[nseq] rows in all, at most INT32_MAX.
 *   q_idx [total, H_I, d_I] e4m3, q_scale [total] or NULL, k_idx [total, d_I] e4m3, k_scale [total] or NULL,
 *     w [total, H_I] fp32, q [total, H, 576] bf16, c [total, 576] bf16 (device arrays);
 *   idx_out [total, k] int32 (out, may be NULL): each row's selection within its own sequence;
 *   out [total, H, 512] bf16 (out), lse [total, H] fp32 (out, may be NULL).
 * Steps 1-2 run per sequence, as dsa_prefill_select.  Step 3 runs once for every row of the batch: each row
 * reads c from its own sequence's first row.  cu_seqlens is read on the host during the call and copied into
 * the workspace, so the caller may reuse it when the call returns.
 * Returns DSA_ERR_INVALID_ARG for a malformed cu_seqlens and the errors of dsa_forward_prefill otherwise.
 */
DSA_API dsa_status_t dsa_forward_prefill_varlen(int nseq, const int64_t* cu_seqlens, const uint8_t* q_idx,
                                                const float* q_scale, const uint8_t* k_idx, const float* k_scale,
                                                const float* w, const uint16_t* q, const uint16_t* c, int H_I,
                                                int d_I, int H, int k, float scale, int32_t* idx_out,
                                                uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                                                void* stream);

/* Workspace bytes of dsa_forward_decode for a batch of B sequences over caches of cache_rows rows. */
DSA_API size_t dsa_decode_workspace_size(int B, int64_t cache_rows, int H_I, int d_I, int H, int k);

/*
 * One DSA decode step for a batch of B sequences, each with one new token.
 * Sequence b owns cache rows [cache_off[b], cache_off[b] + capacity); before the call it holds ctx_len[b]
 * entries.  The call appends the new token's entries at position ctx_len[b] and then runs steps 1-3 for the
 * new token (position ctx_len[b]) over positions 0..ctx_len[b].  ctx_len is not modified: the caller
 * advances it.
 *   cache_off [B] int64, ctx_len [B] int32                            (device arrays)
 *   q_idx [B, H_I, d_I] e4m3, q_scale [B] or NULL, w [B, H_I] fp32, q [B, H, 576] bf16   new-token queries
 *   k_new [B, d_I] e4m3, k_scale_new [B] fp32, c_new [B, 576] bf16                          new-token entries
 *   k_cache [cache_rows, d_I] e4m3, k_scale_cache [cache_rows] fp32, c_cache [cache_rows, 576] bf16 (in/out)
 *   idx_out [B, k] int32 (out, may be NULL): selected positions within each sequence (ascending, -1 padded)
 *   out [B, H, 512] bf16 (out), lse [B, H] fp32 (out, may be NULL)
 * k_scale_new / k_scale_cache are always stored; pass 1.0 for unscaled (integer-valued) keys, and
 * q_scale = NULL.
 * Sequences must own disjoint cache ranges.  A sequence with cache_off[b] < 0, ctx_len[b] < 0 or
 * cache_off[b] + ctx_len[b] >= cache_rows sets the device status to DSA_ERR_BAD_INDEX (read it with
 * dsa_get_device_status); nothing of its cache is read or written, its idx_out row is all -1, and the other
 * sequences of the batch are computed as usual.
 */
DSA_API dsa_status_t dsa_forward_decode(int B, const int64_t* cache_off, const int32_t* ctx_len, const uint8_t* q_idx,
                                const float* q_scale, const float* w, const uint16_t* q, const uint8_t* k_new,
                                const float* k_scale_new, const uint16_t* c_new, uint8_t* k_cache,
                                float* k_scale_cache, uint16_t* c_cache, int64_t cache_rows, int H_I, int d_I,
                                int H, int k, float scale, int32_t* idx_out, uint16_t* out, float* lse, void* ws,
                                size_t ws_bytes, void* stream);

/* Workspace bytes of dsa_forward_decode_paged for a batch of B sequences whose page tables hold max_pages
 * entries of page_rows positions. */
DSA_API size_t dsa_decode_paged_workspace_size(int B, int max_pages, int page_rows, int H_I, int d_I, int H, int k);

/*
 * dsa_forward_decode over paged caches.  The pages describe one cache per sequence; a serving system keeps the
 * caches of many sequences in pools of fixed-size pages (macaron.im page, decode cost at 128K: the decode reads
 * the indexer keys and the selected latent entries of every sequence of the batch), and this is the same decode
 * step with the positions of each sequence mapped through a page table.
 *   page_table [B, max_pages] int32 (device): position p of sequence b is row
 *     page_table[b][p / page_rows] * page_rows + p % page_rows of the pools;
 *   page_rows: positions per page, a positive multiple of 128 (a 128-key indexer tile lies in one page);
 *   k_cache [num_pages * page_rows, d_I] e4m3, k_scale_cache [num_pages * page_rows] fp32,
 *   c_cache [num_pages * page_rows, 576] bf16: the page pools (in/out), at most INT32_MAX rows;
 *   every other argument as in dsa_forward_decode (ctx_len[b] positions before the call; the new entries go to
 *   position ctx_len[b]).
 * Pages may be shared between sequences (a common prefix) except the page that receives the new entry.  A
 * sequence whose new position falls outside its table (ctx_len[b] / page_rows >= max_pages) or whose table names
 * a page outside [0, num_pages) among the pages 0 .. ctx_len[b] / page_rows sets DSA_ERR_BAD_INDEX, and nothing
 * of it is read or written, as in dsa_forward_decode.  Results are bitwise identical to dsa_forward_decode's over
 * flat caches holding the same entries.  Returns DSA_ERR_UNSUPPORTED_SHAPE for a page_rows that is not a
 * multiple of 128 and the errors of dsa_forward_decode otherwise.
 */
DSA_API dsa_status_t dsa_forward_decode_paged(int B, const int32_t* page_table, int max_pages, int page_rows,
                                              const int32_t* ctx_len, const uint8_t* q_idx, const float* q_scale,
                                              const float* w, const uint16_t* q, const uint8_t* k_new,
                                              const float* k_scale_new, const uint16_t* c_new, uint8_t* k_cache,
                                              float* k_scale_cache, uint16_t* c_cache, int num_pages, int H_I,
                                              int d_I, int H, int k, float scale, int32_t* idx_out, uint16_t* out,
                                              float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * dsa_forward_decode without a caller-provided workspace, for callers that cannot allocate device memory
 * (for example a serving loop that runs under a memory pool it may not grow, or code that only receives
 * borrowed buffers).  This entry point has no counterpart in the paper: it is the decode step above with its
 * scratch (the packed score rows, per-sequence lengths, offsets and score histograms and, when idx_out is NULL,
 * the selected indices) held in a fixed device array inside the library, of dsa_decode_noalloc_scratch_bytes() bytes
 * (32 MiB).  Every GPU that loads the library keeps that array until the process exits.
 *   - Arguments and results are those of dsa_forward_decode; shapes whose dsa_decode_workspace_size()
 *     exceeds the array return DSA_ERR_WORKSPACE and launch nothing.
 *   - The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - Argument and shape checks are those of dsa_forward_decode and come first, with its error codes; the
 *     size check against the array comes after them.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that device
 *     current; make that first call before any stream capture on the device.  The address is kept with the
 *     context it was looked up in and looked up again when the device's current context changes (after a
 *     cudaDeviceReset, for instance); a first call in a new context must also come before any capture.
 *   - All calls share the one array and it keeps the last call's contents: calls that may overlap on the GPU
 *     (different streams, or graph replays in flight together) race on it and must be serialised by the
 *     caller.
 */
DSA_API size_t dsa_decode_noalloc_scratch_bytes(void);
DSA_API dsa_status_t dsa_forward_decode_noalloc(int B, const int64_t* cache_off, const int32_t* ctx_len,
                                                const uint8_t* q_idx, const float* q_scale, const float* w,
                                                const uint16_t* q, const uint8_t* k_new, const float* k_scale_new,
                                                const uint16_t* c_new, uint8_t* k_cache, float* k_scale_cache,
                                                uint16_t* c_cache, int64_t cache_rows, int H_I, int d_I, int H,
                                                int k, float scale, int32_t* idx_out, uint16_t* out, float* lse,
                                                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
