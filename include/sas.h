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
 *   - Scores must be finite; NaN rows have no defined Top-K.
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
 * sas_attn_fwd - gated block-sparse causal attention, forward.
 * SAS review §2.3, eq. o_SAS, with the current block kept at gate 1 (§2.4)
 * under a causal mask, tiled over the kept key blocks only (§2.6).
 *
 * dtype    SAS_BF16 (tensor cores, fp32 accumulation) or SAS_F32 (fp32
 *          FMA throughout).
 * q        device [B, S, Hq, D]; k, v device [B, S, Hkv, D]; all of dtype,
 *          16-byte aligned. S % 64 == 0, Hq % Hkv == 0, D in {64, 128}.
 * idx, cnt, log_gate   as written by sas_select with n_rows = S/64 and the
 *          same K; an index outside 0..i-1 for query block i is flagged and
 *          skipped.
 * o        device [B, S, Hq, D] of dtype (output).
 * lse      device fp32 [B, Hq, S] (output): natural-log LSE of each row's
 *          logits, kept for the backward.
 */
sas_status sas_attn_fwd(sas_dtype dtype, const void *q, const void *k, const void *v,
                        int B, int S, int Hq, int Hkv, int D, int block_size, int K,
                        const int32_t *idx, const int32_t *cnt, const float *log_gate,
                        float sm_scale, void *o, float *lse, void *stream);

/* Bytes of device workspace sas_attn_bwd needs for these sizes (0 on a bad
 * argument). */
size_t sas_attn_bwd_workspace_size(sas_dtype dtype, int B, int S, int Hq, int Hkv, int D, int K);

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
 * ds       device fp32 [B, Hkv, S/64, ld_s] (output; every entry of each
 *          row 0..ld_s-1 is written).
 * workspace device, ws_bytes >= sas_attn_bwd_workspace_size(...), 256-byte
 *          aligned; contents on entry do not matter.
 * Summation order inside dk/dv may vary between runs (fp32 atomics).
 */
sas_status sas_attn_bwd(sas_dtype dtype, const void *q, const void *k, const void *v,
                        const void *o, const void *dout, const float *lse,
                        const float *s, int ld_s, const float *lse_s,
                        const int32_t *idx, const int32_t *cnt, const float *log_gate,
                        int B, int S, int Hq, int Hkv, int D, int block_size, int K,
                        float sm_scale, void *dq, void *dk, void *dv, float *ds,
                        void *workspace, size_t ws_bytes, void *stream);

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
 * workspace  device, ws_bytes >= sas_decode_workspace_size(...).
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
 * device current; make that first call before any stream capture.
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
