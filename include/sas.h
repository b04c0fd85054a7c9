/*
 * sas.h - C ABI of libsas.so: SAS gated block-sparse causal attention on B200.
 *
 * The method (SAS review (paper.oopus.info), §2.1-§2.6):
 *   - the context is cut into blocks of b = 64 tokens (§2.1);
 *   - per query block (prefill/training) or per query token (decode), the
 *     history blocks are ranked by selector scores s and the Top-K kept; the
 *     block holding the query is always kept (§2.1, §2.2);
 *   - every kept history block m gets log g_m = s_m - LSE(s), the LSE over
 *     ALL history blocks; the current block gets log g = 0 (§2.4, eq. log g);
 *   - o = softmax(q K_S^T + log g_S) V_S, the gate inside the softmax (§2.3,
 *     eq. o_SAS), computed tile by tile without the full matrix (§2.6);
 *   - the backward gives dq/dk/dv and, for the selector, ds: the gate
 *     gradient of a block is the sum of its logit gradients (§2.6), carried
 *     to s through the Jacobian of s - LSE(s) (§2.4).
 *
 * Conventions shared by every entry point:
 *   - Pointers marked "device" are CUDA device pointers owned by the caller;
 *     the library never frees or keeps them. Workspaces are caller-allocated;
 *     their size is queried first. Except where an entry point says so, the
 *     library allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Every call only enqueues work on it; none synchronises,
 *     except sas_get_error_flag.
 *   - Arguments are validated on the host before anything is launched. A
 *     bad argument returns SAS_ERR_INVALID_ARG, a valid but unimplemented
 *     case SAS_ERR_UNSUPPORTED; in both cases nothing is launched. A failed
 *     launch returns SAS_ERR_CUDA. sas_last_error() gives the message.
 *   - Kernels check the values they read from device memory (indices, page
 *     ids, lengths) and skip what is out of range instead of touching it;
 *     they record the first problem in a per-device status word that
 *     sas_get_error_flag() reports and clears (SAS_ERR_INVALID_ARG for bad
 *     device-side data, SAS_ERR_TIMEOUT when a bounded wait gave up).
 *   - Scores must be finite. A selection row whose history holds a NaN or
 *     +-inf score is flagged (SAS_ERR_INVALID_ARG from sas_get_error_flag)
 *     and gets the empty selection (cnt 0, idx -1, log_gate -inf) with
 *     lse_s = NaN; the other rows are unaffected.
 *   - Prefill sequences may have any length: a length that is not a multiple
 *     of 64 ends in a partial block, which is a query block like the others
 *     and (having no later block) is never selected as history. Batches of
 *     different lengths use the _varlen entry points: q/k/v packed along the
 *     token axis, sequence b at token rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 *     (device int32 [B + 1], non-decreasing, cu_seqlens[B] <= total_tokens,
 *     each length <= max_seqlen; a sequence that breaks this is flagged and
 *     treated as empty), per-block tensors padded to ceil(max_seqlen / 64)
 *     rows per sequence and the row LSE to max_seqlen.
 *   - Tensor layouts are row-major with the last named dimension contiguous.
 *     GQA: query head hq reads KV head hq / (Hq / Hkv).
 *   - Logits are sm_scale * q.k + log g: sm_scale multiplies q.k only.
 *   - block_size (= page_size for decode) must be 64.
 */
#ifndef SAS_H
#define SAS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAS_OK = 0,
    SAS_ERR_INVALID_ARG = 1,
    SAS_ERR_UNSUPPORTED = 2,
    SAS_ERR_CUDA = 3,
    SAS_ERR_TIMEOUT = 4
} sas_status;

typedef enum { SAS_F32 = 0, SAS_BF16 = 1 } sas_dtype;

/* Message of the last failed call on this host thread ("" if none). */
const char *sas_last_error(void);

/* Number of kernels this library has enqueued in this process so far
 * (diagnostics: lets a caller count the launches inside a timed region). */
uint64_t sas_kernel_launches(void);

/* Synchronises `stream`, then returns and clears the status word of the
 * current device: SAS_OK, SAS_ERR_INVALID_ARG (a kernel met an out-of-range
 * index, page id or length and skipped it) or SAS_ERR_TIMEOUT. */
sas_status sas_get_error_flag(void *stream);

/*
 * sas_select - Top-K history blocks and their normalised log-gates.
 * SAS review §2.2 (Top-K of the selector scores over history blocks) and
 * §2.4, eq. log g (log g_m = s_m - LSE(s) over all history blocks).
 *
 * s        device fp32 [B, Hkv, n_rows, ld_s]; row (b,h,r) reads entries
 *          0..nh-1 only (others may hold anything, NaN included).
 * kv_len   NULL for prefill: row r is query block r and has nh = r history
 *          blocks (requires ld_s >= n_rows).
 *          Else decode: device int32 [B]; every row of batch entry b has
 *          nh = (kv_len[b] - 1) / block_size history blocks (kv_len[b] >= 1;
 *          nh > ld_s is flagged and clamped to ld_s).
 *          Rows hold at most 16384 history blocks (1M tokens); longer rows
 *          return SAS_ERR_UNSUPPORTED.
 * K        budget in blocks, K >= 0. A row keeps min(K, nh) blocks.
 * idx      device int32 [B, Hkv, n_rows, K]: kept block indices, ascending,
 *          padded with -1. Order of the Top-K: score descending, then block
 *          index ascending (the lower index wins a tie; -0.0 == +0.0).
 * cnt      device int32 [B, Hkv, n_rows]: min(K, nh).
 * log_gate device fp32 [B, Hkv, n_rows, K]: s[idx] - lse_s, padded with -inf.
 * lse_s    device fp32 [B, Hkv, n_rows]: natural-log LSE of the nh scores
 *          (-inf when nh = 0).
 */
sas_status sas_select(const float *s, int B, int Hkv, int n_rows, int ld_s,
                      const int32_t *kv_len, int block_size, int K,
                      int32_t *idx, int32_t *cnt, float *log_gate, float *lse_s,
                      void *stream);

/*
 * sas_select_varlen - sas_select (prefill) for a packed batch of sequences of
 * different lengths (the same method applied to each sequence, SAS review
 * §2.2, §2.4). cu_seqlens: device int32 [B + 1] (see the conventions above).
 * Row (b, h, r) is query block r of sequence b when r < ceil(len_b / 64);
 * later rows are padding: cnt 0, idx -1, log_gate -inf, lse_s -inf, and their
 * scores are not read. n_rows >= ceil(max_seqlen / 64), ld_s >= n_rows.
 */
sas_status sas_select_varlen(const float *s, int B, int Hkv, int n_rows, int ld_s,
                             const int32_t *cu_seqlens, int block_size, int K,
                             int32_t *idx, int32_t *cnt, float *log_gate, float *lse_s,
                             void *stream);

/*
 * sas_attn_fwd - gated block-sparse causal attention, forward.
 * SAS review §2.3, eq. o_SAS, with the current block kept at gate 1 (§2.4)
 * under a causal mask, tiled over the kept key blocks only (§2.6).
 *
 * dtype    SAS_BF16 (tensor cores, fp32 accumulation) or SAS_F32 (fp32
 *          FMA throughout). bf16 with D = 128 runs on the tcgen05 tensor
 *          cores; fp32, and bf16 with D = 64, run on the CUDA cores (an
 *          untuned path: fp32 keeps full fp32 arithmetic, D = 64 is a
 *          secondary head size).
 * q        device [B, S, Hq, D]; k, v device [B, S, Hkv, D]; all of dtype,
 *          16-byte aligned. S >= 1 (the last block may be partial),
 *          Hq % Hkv == 0, D in {64, 128}.
 * idx, cnt, log_gate   as written by sas_select with n_rows = ceil(S/64) and
 *          the same K; an index outside 0..i-1 for query block i is flagged
 *          and skipped.
 * o        device [B, S, Hq, D] of dtype (output).
 * lse      device fp32 [B, Hq, S] (output): natural-log LSE of each row's
 *          logits, kept for the backward.
 */
sas_status sas_attn_fwd(sas_dtype dtype, const void *q, const void *k, const void *v,
                        int B, int S, int Hq, int Hkv, int D, int block_size, int K,
                        const int32_t *idx, const int32_t *cnt, const float *log_gate,
                        float sm_scale, void *o, float *lse, void *stream);

/*
 * sas_attn_fwd_varlen - sas_attn_fwd for a packed batch of sequences of
 * different lengths (the method applied to each sequence on its own).
 * q        device [total_tokens, Hq, D]; k, v [total_tokens, Hkv, D].
 * cu_seqlens, max_seqlen   see the conventions above.
 * idx, cnt, log_gate   from sas_select_varlen with n_rows = ceil(max_seqlen/64).
 * o        device [total_tokens, Hq, D]; rows of no sequence are not written.
 * lse      device fp32 [B, Hq, max_seqlen]; entries past a sequence's length
 *          are not written.
 */
sas_status sas_attn_fwd_varlen(sas_dtype dtype, const void *q, const void *k, const void *v,
                               const int32_t *cu_seqlens, int B, int max_seqlen, int total_tokens,
                               int Hq, int Hkv, int D, int block_size, int K,
                               const int32_t *idx, const int32_t *cnt, const float *log_gate,
                               float sm_scale, void *o, float *lse, void *stream);

/* Bytes of device workspace sas_attn_bwd needs for these sizes (0 on a bad
 * argument). */
size_t sas_attn_bwd_workspace_size(sas_dtype dtype, int B, int S, int Hq, int Hkv, int D, int K);

/* Bytes of device workspace sas_attn_bwd_varlen needs (0 on a bad argument). */
size_t sas_attn_bwd_varlen_workspace_size(sas_dtype dtype, int B, int max_seqlen, int total_tokens,
                                          int Hq, int Hkv, int D, int K);

/*
 * sas_attn_bwd - gradients of the forward with respect to q, k, v and s.
 * SAS review §2.6 (probabilities recomputed tile by tile; the gradient of a
 * block's gate is the sum of the logit gradients inside it) and §2.4, eq.
 * log g (its Jacobian): for query block i, history block j < i,
 *   ds[i][j] = Gsum[i][j] * [j kept] - softmax(s_i)[j] * sum_{m kept} Gsum[i][m],
 * where Gsum[i][m] sums the logit gradients of key block m over the rows of
 * block i and the query heads of the KV head. ds[i][j] = 0 for j >= i.
 *
 * q, k, v, o, lse, idx, cnt, log_gate   as passed to / written by the forward.
 * dout     device [B, S, Hq, D] of dtype: upstream gradient of o.
 * s, ld_s  the scores given to sas_select; lse_s its output.
 * dq       device [B, S, Hq, D] of dtype (output).
 * dk, dv   device [B, S, Hkv, D] of dtype (output).
 * ds       device fp32 [B, Hkv, ceil(S/64), ld_s] (output; every entry of
 *          each row 0..ld_s-1 is written).
 * workspace device, ws_bytes >= sas_attn_bwd_workspace_size(...), 256-byte
 *          aligned; contents on entry do not matter.
 * The bf16 D = 128 path writes dq, dk and dv once each (deterministic); the
 * CUDA-core path accumulates dk/dv with fp32 atomics, whose summation order
 * may vary between runs. The bf16 D = 128 path handles at most 32767 query
 * blocks per sequence (S <= 2,097,088; SAS_ERR_UNSUPPORTED beyond).
 */
sas_status sas_attn_bwd(sas_dtype dtype, const void *q, const void *k, const void *v,
                        const void *o, const void *dout, const float *lse,
                        const float *s, int ld_s, const float *lse_s,
                        const int32_t *idx, const int32_t *cnt, const float *log_gate,
                        int B, int S, int Hq, int Hkv, int D, int block_size, int K,
                        float sm_scale, void *dq, void *dk, void *dv, float *ds,
                        void *workspace, size_t ws_bytes, void *stream);

/*
 * sas_attn_bwd_varlen - sas_attn_bwd for a packed batch (layouts as in
 * sas_attn_fwd_varlen; s and ds [B, Hkv, ceil(max_seqlen/64), ld_s], whose
 * padding rows of ds are written as zero). dk/dv rows of no sequence are not
 * written.
 */
sas_status sas_attn_bwd_varlen(sas_dtype dtype, const void *q, const void *k, const void *v,
                               const void *o, const void *dout, const float *lse,
                               const float *s, int ld_s, const float *lse_s,
                               const int32_t *idx, const int32_t *cnt, const float *log_gate,
                               const int32_t *cu_seqlens, int B, int max_seqlen, int total_tokens,
                               int Hq, int Hkv, int D, int block_size, int K, float sm_scale,
                               void *dq, void *dk, void *dv, float *ds,
                               void *workspace, size_t ws_bytes, void *stream);

/* Bytes of device workspace sas_score_select needs (0 on a bad argument). */
size_t sas_score_select_workspace_size(int B, int S, int Hq, int Hkv, int D);

/*
 * sas_score_select - block-pooled stand-in selector scores, followed in the
 * same call by the Top-K selection and the log-gates of sas_select (prefill).
 * SAS review §2.2: the selector scores each history block of a query block,
 * s = R_theta(q, {K_Bm}), and the Top-K are kept; §2.4, eq. log g. The
 * trained selector (AttnGate) is not part of this library; its stand-in is
 *   s[b,h,i,j] = mean over the 64 rows of block i and the G query heads of
 *                KV head h of q, dotted with the mean over the 64 rows of
 *                block j of k[:, :, h], divided by sqrt(D), plus noise[b,h,i,j]
 * for j < i (fp32 sums of the bf16 inputs).
 *
 * q, k     device bf16 [B, S, Hq, D], [B, S, Hkv, D]; S % 64 == 0, D in
 *          {64, 128}, 16-byte aligned.
 * noise    device fp32 [B, Hkv, S/64, ld_noise] added to the scores, or NULL.
 * s        device fp32 [B, Hkv, S/64, ld_s] (output): entries j < i of row
 *          (b, h, i) are written, the others are left as they are. These are
 *          the scores the backward's Jacobian needs.
 * idx, cnt, log_gate, lse_s   as sas_select writes them for these scores.
 * workspace device, 256-byte aligned, ws_bytes >= sas_score_select_workspace_size
 *          (it holds the pooled queries and keys).
 * SAS_ERR_UNSUPPORTED for rows of more than 16384 history blocks, for
 * B * Hkv > 65535, and when (Hq + Hkv) * D fp32 values exceed 200 KiB.
 */
sas_status sas_score_select(const void *q, const void *k, const float *noise, int ld_noise,
                            int B, int S, int Hq, int Hkv, int D, int block_size, int K,
                            float *s, int ld_s, int32_t *idx, int32_t *cnt, float *log_gate,
                            float *lse_s, void *workspace, size_t ws_bytes, void *stream);

/*
 * sas_pool_pages - the pooled-key cache of a paged KV cache, for the decode
 * stand-in scorer: kpool[p, h, :] = the mean of the 64 key rows of page p and
 * KV head h (fp32 sums of the bf16 keys). The stand-in for the selector of
 * SAS review §2.2 scores a history block by its mean key; a serving engine
 * computes it once, when a page fills, instead of at every decode step.
 *
 * k_cache  device bf16 [num_pages, Hkv, 64, D], D in {64, 128}, 16-byte aligned.
 * pages    device int32 [n_pages] page ids to pool, or NULL for all pages.
 *          An id outside [0, num_pages) is flagged and skipped.
 * kpool    device fp32 [num_pages, Hkv, D] (output; only the listed pages are
 *          written), 16-byte aligned.
 */
sas_status sas_pool_pages(const void *k_cache, int num_pages, int Hkv, int D, int page_size,
                          const int32_t *pages, int n_pages, float *kpool, void *stream);

/*
 * sas_score_select_decode - decode stand-in scores from the pooled-key cache,
 * then the decode selection (SAS review §2.2, §2.4). For sequence n (query at
 * kv_len[n]-1, history blocks j < (kv_len[n]-1)/64) and KV head h:
 *   s[n, h, j] = mean over the G query heads of h of q[n] . kpool[page_table[n, j], h]
 *                / sqrt(D) + noise[n, h, j]
 * then idx, cnt, log_gate, lse_s exactly as sas_select in decode mode.
 *
 * q          device bf16 [N, Hq, D]; kpool from sas_pool_pages.
 * page_table device int32 [N, max_pages]; a bad page id is flagged and the
 *            row gets a NaN score (so the selection flags it and keeps nothing).
 * noise      device fp32 [N, Hkv, ld_noise] or NULL.
 * s          device fp32 [N, Hkv, ld_s] (output; entries j < nh written),
 *            ld_s >= the longest history (<= 16384 blocks).
 * idx, cnt, log_gate, lse_s   device [N, Hkv, K], [N, Hkv], [N, Hkv, K], [N, Hkv].
 * SAS_ERR_UNSUPPORTED for N * Hkv > 65535.
 */
sas_status sas_score_select_decode(const void *q, const float *kpool, int num_pages,
                                   const int32_t *page_table, int max_pages, const int32_t *kv_len,
                                   int N, int Hq, int Hkv, int D, int page_size,
                                   const float *noise, int ld_noise, int K, float *s, int ld_s,
                                   int32_t *idx, int32_t *cnt, float *log_gate, float *lse_s,
                                   void *stream);

/* Bytes of device workspace sas_decode_paged needs (0 on a bad argument). */
size_t sas_decode_workspace_size(int N, int Hq, int Hkv, int D, int K);

/*
 * sas_decode_paged - one decode step over a paged KV cache.
 * The same gated softmax (SAS review §2.3, eq. o_SAS; §2.4) for one query
 * token per sequence, reading only the kept pages of the paged cache the
 * serving side keeps (§2.6). Sequence n's query sits at position
 * kv_len[n]-1; its current block c = (kv_len[n]-1)/64 holds tokens
 * 64c..kv_len[n]-1 (all attended, gate 1); its history is blocks 0..c-1,
 * selected by sas_select in decode mode (n_rows = 1).
 *
 * q          device bf16 [N, Hq, D], D = 128.
 * k_cache, v_cache  device bf16 [num_pages, Hkv, 64, D]: page p holds 64
 *            consecutive tokens; (page, head) is one contiguous 16 KiB tile.
 * page_table device int32 [N, max_pages]: logical block -> page id. Entries
 *            0..ceil(kv_len[n]/64)-1 must lie in [0, num_pages); a bad id is
 *            flagged and its block skipped.
 * kv_len     device int32 [N], 1 <= kv_len[n] <= 64*max_pages.
 * idx, cnt, log_gate   device [N, Hkv, K], [N, Hkv], [N, Hkv, K] from
 *            sas_select (decode mode).
 * o          device bf16 [N, Hq, D] (output). lse: device fp32 [N, Hq] or NULL.
 * workspace  device, ws_bytes >= sas_decode_workspace_size(...), 256-byte
 *            aligned; contents on entry do not matter.
 * SAS_ERR_UNSUPPORTED unless D = 128, page_size = 64 and the GQA group size
 * Hq/Hkv is 1, 2, 4, 5 or 8.
 */
sas_status sas_decode_paged(const void *q, const void *k_cache, const void *v_cache,
                            int num_pages, const int32_t *page_table, int max_pages,
                            const int32_t *kv_len, int N, int Hq, int Hkv, int D,
                            int page_size, int K, const int32_t *idx, const int32_t *cnt,
                            const float *log_gate, float sm_scale, void *o, float *lse,
                            void *workspace, size_t ws_bytes, void *stream);

/*
 * sas_decode_paged_noalloc - sas_decode_paged for callers that cannot
 * allocate device memory. The SAS pages have no counterpart to this call: it
 * exists for callers such as a serving engine that gives nearly all of the
 * GPU to its KV-cache pool at start-up, or a plain C host that holds only
 * its input and output buffers and no device allocator.
 *
 * Arguments, outputs and errors are those of sas_decode_paged, without the
 * workspace: the split-KV partials go to a 16 MiB array that the library
 * reserves in device memory when it is loaded (every GPU that loads the
 * library holds it until the process exits). Sizes whose partials need more
 * than 16 MiB (sas_decode_workspace_size(N, Hq, Hkv, D, K) > 16 MiB) are
 * rejected with SAS_ERR_INVALID_ARG before anything runs. No device memory
 * is allocated or freed by the call.
 * All calls on one device share that array, which keeps the last call's
 * contents; nothing in it needs to start at zero. Calls that overlap on the
 * GPU (on different streams, or from threads without ordering) race on it.
 * The first call on a device looks up the array's device address with that
 * device current and caches it with the current context's id; the lookup is
 * repeated when another context is current (after cudaDeviceReset). Make the
 * first call on a device, and the first after a reset, before any stream
 * capture.
 */
sas_status sas_decode_paged_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                    int num_pages, const int32_t *page_table, int max_pages,
                                    const int32_t *kv_len, int N, int Hq, int Hkv, int D,
                                    int page_size, int K, const int32_t *idx, const int32_t *cnt,
                                    const float *log_gate, float sm_scale, void *o, float *lse,
                                    void *stream);

/*
 * sas_selftest_bounded_wait - fault injection for the bounded waits, with no
 * GPU fault (no counterpart on the SAS pages: it tests this library's failure
 * detection). Enqueues on `stream` one single-warp kernel that waits, with
 * the bounded mbarrier wait every kernel of the library uses, on a barrier
 * that nothing ever arrives on. The wait gives up after its budget (about 2 s
 * of SM clocks), records a timeout in the device status word and the kernel
 * returns; the next sas_get_error_flag on the device reports (and clears)
 * SAS_ERR_TIMEOUT, and the context stays usable.
 * Returns SAS_OK once the kernel is enqueued, SAS_ERR_CUDA if it is not.
 */
sas_status sas_selftest_bounded_wait(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SAS_H */
