// Internal host-side launchers, one per kernel family. Arguments are already
// validated by sas_api.cu; each launcher only picks a configuration, enqueues
// on `stream` and returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

namespace sas {

// Process-wide count of kernels enqueued by the launchers below.
void count_launches(int n);

// Sets the message sas_last_error() returns on this host thread.
void set_last_error(const char* msg);

// Identifier of the CUDA context current on this host thread (0 if unknown).
unsigned long long current_context_id();

// Device address of a module variable on device `dev` (which must be
// current) into *out, from `lookup` (a cudaGetSymbolAddress call) whose
// return code is passed on. The address is cached per device with the id of
// the context it was taken in, and looked up again when another context is
// current (after cudaDeviceReset, a variable's address may change).
cudaError_t cached_symbol_address(int dev, std::mutex* mu, unsigned long long* ctx_ids, void** ptrs,
                                  cudaError_t (*lookup)(void**), void** out);

// kv_len: decode rows (else prefill); cu: per-sequence lengths of a packed
// prefill batch (rows past a sequence's last block are padding), or nullptr.
cudaError_t launch_select(const float* s, int B, int Hkv, int n_rows, int ld_s,
                          const int32_t* kv_len, const int32_t* cu, int K, int max_hist,
                          int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s,
                          int* status, cudaStream_t stream);

// q/k/v rows: T token rows; sequence b at rows b*S.. (cu == nullptr, T = B*S)
// or cu[b]..cu[b+1]-1 (packed, S = the longest length). Per-block tensors are
// [B, Hkv, ceil(S/64), ...], row LSEs [B, Hq, S].
struct AttnArgs {
    const void* q; const void* k; const void* v;
    int B, S, Hq, Hkv, D, K;
    const int32_t* cu; long long T;
    const int32_t* idx; const int32_t* cnt; const float* log_gate;
    float sm_scale;
    int* status;
};

// fp32 (and reference-grade generic) CUDA-core path.
cudaError_t launch_fwd_simt(const AttnArgs& a, bool bf16, void* o, float* lse, cudaStream_t st);
// bf16, D = 128: tcgen05 tensor-core path.
cudaError_t launch_fwd_sm100(const AttnArgs& a, void* o, float* lse, cudaStream_t st);

struct BwdArgs {
    AttnArgs a;
    const void* o; const void* dout; const float* lse;
    const float* s; int ld_s; const float* lse_s;
    void* dq; void* dk; void* dv; float* ds;
    void* workspace; size_t ws_bytes;
};
size_t bwd_simt_workspace(int B, int S, long long T, int Hq, int Hkv, int D, int K);
cudaError_t launch_bwd_simt(const BwdArgs& b, bool bf16, cudaStream_t st);
// bf16, D = 128: tcgen05 tensor-core path.
size_t bwd_sm100_workspace(int B, int S, int Hq, int Hkv, int K);
cudaError_t launch_bwd_sm100(const BwdArgs& b, cudaStream_t st);
// ds from the per-block gate gradients gsum [B, Hkv, NQB, K]; rows past a
// sequence's last block (packed batches) are zero.
cudaError_t launch_ds_finalize(const float* s, int ld_s, const float* lse_s, const int32_t* idx,
                               const int32_t* cnt, const float* gsum, int B, int Hkv, int NQB, int K,
                               const int32_t* cu, int S, long long T, float* ds, cudaStream_t st);

// Stand-in selector scores (block-pooled q . k / sqrt(D) + noise) fused with
// the selection; q/k bf16 [B, S, H, D] with S % 64 == 0.
struct ScoreArgs {
    const void* q; const void* k; const float* noise; int ld_noise;
    int B, S, Hq, Hkv, D, K;
    float* s; int ld_s;
    int32_t* idx; int32_t* cnt; float* log_gate; float* lse_s;
    void* workspace; int* status;
};
size_t score_workspace(int B, int S, int Hkv, int D);
cudaError_t launch_score_select(const ScoreArgs& a, cudaStream_t st);

// Pooled-key cache of a paged KV cache: kpool[p, h, :] = mean of the 64 rows
// of page p (all pages when `pages` is null, else the n_pages listed).
cudaError_t launch_pool_pages(const void* k_cache, int num_pages, int Hkv, int D, const int32_t* pages, int n_pages,
                              float* kpool, int* status, cudaStream_t st);
// Decode stand-in scores from the pooled-key cache, then the decode selection.
struct DecodeScoreArgs {
    const void* q; const float* kpool; int num_pages;
    const int32_t* page_table; int max_pages; const int32_t* kv_len;
    int N, Hq, Hkv, D, K;
    const float* noise; int ld_noise;
    float* s; int ld_s;
    int32_t* idx; int32_t* cnt; float* log_gate; float* lse_s;
    int* status;
};
cudaError_t launch_score_select_decode(const DecodeScoreArgs& a, cudaStream_t st);

// Decode.
struct DecodeArgs {
    const void* q; const void* k_cache; const void* v_cache;
    int num_pages; const int32_t* page_table; int max_pages; const int32_t* kv_len;
    int N, Hq, Hkv, D, K;
    const int32_t* idx; const int32_t* cnt; const float* log_gate;
    float sm_scale; void* o; float* lse;
    int* status;
};
size_t decode_workspace(int N, int Hq, int Hkv, int D, int K);
cudaError_t launch_decode(const DecodeArgs& d, void* workspace, cudaStream_t st);

// One warp waiting (bounded) on a barrier nothing arrives on: records a timeout in *status.
cudaError_t launch_bounded_wait_selftest(int* status, cudaStream_t st);

}  // namespace sas
