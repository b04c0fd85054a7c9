// Internal host-side launchers, one per kernel family. Arguments are already
// validated by sas_api.cu; each launcher only picks a configuration, enqueues
// on `stream` and returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sas {

// Process-wide count of kernels enqueued by the launchers below.
void count_launches(int n);

// Sets the message sas_last_error() returns on this host thread.
void set_last_error(const char* msg);

cudaError_t launch_select(const float* s, int B, int Hkv, int n_rows, int ld_s,
                          const int32_t* kv_len, int K, int max_hist,
                          int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s,
                          int* status, cudaStream_t stream);

struct AttnArgs {
    const void* q; const void* k; const void* v;
    int B, S, Hq, Hkv, D, K;
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
size_t bwd_simt_workspace(int B, int S, int Hq, int Hkv, int D, int K);
cudaError_t launch_bwd_simt(const BwdArgs& b, bool bf16, cudaStream_t st);
// bf16, D = 128: tcgen05 tensor-core path.
size_t bwd_sm100_workspace(int B, int S, int Hq, int Hkv, int K);
cudaError_t launch_bwd_sm100(const BwdArgs& b, cudaStream_t st);
// ds from the per-block gate gradients gsum [B, Hkv, NQB, K].
cudaError_t launch_ds_finalize(const float* s, int ld_s, const float* lse_s, const int32_t* idx,
                               const int32_t* cnt, const float* gsum, int B, int Hkv, int NQB, int K,
                               float* ds, cudaStream_t st);

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
