// C ABI of libsas.so (declared in include/sas.h): host-side validation,
// per-device status word, and dispatch to the kernel launchers.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/sas.h"
#include "launch.h"

namespace {

thread_local char g_msg[512] = "";

sas_status fail(sas_status code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return code;
}

sas_status ok() {
    g_msg[0] = '\0';
    return SAS_OK;
}

sas_status cuda_fail(cudaError_t e, const char* where) {
    return fail(SAS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Per-device status word written by kernels (first problem wins).
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};

int* status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (g_status_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sas_status check_attn_shape(sas_dtype dtype, const void* q, const void* k, const void* v, int B, int S,
                            int Hq, int Hkv, int D, int block_size, int K, const int32_t* idx,
                            const int32_t* cnt, const float* log_gate) {
    if (dtype != SAS_F32 && dtype != SAS_BF16) return fail(SAS_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (!q || !k || !v || !cnt) return fail(SAS_ERR_INVALID_ARG, "null tensor pointer");
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "null idx/log_gate with K > 0");
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "non-positive size (B=%d S=%d Hq=%d Hkv=%d D=%d K=%d)", B, S, Hq, Hkv, D, K);
    if (Hq % Hkv) return fail(SAS_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
    if (block_size != 64) return fail(SAS_ERR_UNSUPPORTED, "block_size=%d (only 64)", block_size);
    if (S % 64) return fail(SAS_ERR_INVALID_ARG, "S=%d is not a multiple of 64", S);
    if (D != 64 && D != 128) return fail(SAS_ERR_UNSUPPORTED, "D=%d (only 64 or 128)", D);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return fail(SAS_ERR_INVALID_ARG, "q/k/v not 16-byte aligned");
    if ((long long)B * S * Hq > (1LL << 31) - 1) return fail(SAS_ERR_UNSUPPORTED, "B*S*Hq too large");
    return SAS_OK;
}

}  // namespace

namespace sas {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
void set_last_error(const char* msg) { snprintf(g_msg, sizeof g_msg, "%s", msg); }
}  // namespace sas

extern "C" {

uint64_t sas_kernel_launches(void) { return (uint64_t)sas::g_launches.load(std::memory_order_relaxed); }

const char* sas_last_error(void) { return g_msg; }

sas_status sas_get_error_flag(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "sas_get_error_flag: stream sync");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "sas_get_error_flag: read");
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "sas_get_error_flag: clear");
    if (v == 0) return ok();
    if (v == SAS_ERR_TIMEOUT) return fail(SAS_ERR_TIMEOUT, "a kernel's bounded wait expired");
    return fail(SAS_ERR_INVALID_ARG, "a kernel met out-of-range device data (index, page id or length)");
}

sas_status sas_select(const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* kv_len,
                      int block_size, int K, int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s,
                      void* stream) {
    if (!s || !cnt || !lse_s) return fail(SAS_ERR_INVALID_ARG, "sas_select: null pointer");
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "sas_select: null idx/log_gate with K > 0");
    if (B <= 0 || Hkv <= 0 || n_rows <= 0 || ld_s <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "sas_select: bad size (B=%d Hkv=%d n_rows=%d ld_s=%d K=%d)", B, Hkv, n_rows, ld_s, K);
    if (block_size != 64) return fail(SAS_ERR_UNSUPPORTED, "sas_select: block_size=%d (only 64)", block_size);
    if (!kv_len && ld_s < n_rows) return fail(SAS_ERR_INVALID_ARG, "sas_select: prefill needs ld_s >= n_rows");
    const int max_hist = kv_len ? ld_s : n_rows - 1;
    if (max_hist > 1024) return fail(SAS_ERR_UNSUPPORTED, "sas_select: rows of more than 1024 history blocks");
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "sas_select: no CUDA device");
    cudaError_t e = sas::launch_select(s, B, Hkv, n_rows, ld_s, kv_len, K, max_hist, idx, cnt, log_gate, lse_s, st,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sas_select");
}

sas_status sas_attn_fwd(sas_dtype dtype, const void* q, const void* k, const void* v, int B, int S, int Hq,
                        int Hkv, int D, int block_size, int K, const int32_t* idx, const int32_t* cnt,
                        const float* log_gate, float sm_scale, void* o, float* lse, void* stream) {
    sas_status r = check_attn_shape(dtype, q, k, v, B, S, Hq, Hkv, D, block_size, K, idx, cnt, log_gate);
    if (r != SAS_OK) return r;
    if (!o || !lse) return fail(SAS_ERR_INVALID_ARG, "sas_attn_fwd: null output");
    if (!aligned16(o)) return fail(SAS_ERR_INVALID_ARG, "sas_attn_fwd: o not 16-byte aligned");
    if (!std::isfinite(sm_scale)) return fail(SAS_ERR_INVALID_ARG, "sas_attn_fwd: sm_scale not finite");
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "sas_attn_fwd: no CUDA device");
    sas::AttnArgs a{q, k, v, B, S, Hq, Hkv, D, K, idx, cnt, log_gate, sm_scale, st};
    cudaError_t e = (dtype == SAS_BF16 && D == 128)
                        ? sas::launch_fwd_sm100(a, o, lse, static_cast<cudaStream_t>(stream))
                        : sas::launch_fwd_simt(a, dtype == SAS_BF16, o, lse, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sas_attn_fwd");
}

size_t sas_attn_bwd_workspace_size(sas_dtype dtype, int B, int S, int Hq, int Hkv, int D, int K) {
    if ((dtype != SAS_F32 && dtype != SAS_BF16) || B <= 0 || S <= 0 || S % 64 || Hq <= 0 || Hkv <= 0 ||
        Hq % Hkv || (D != 64 && D != 128) || K < 0)
        return 0;
    if (dtype == SAS_BF16 && D == 128) return sas::bwd_sm100_workspace(B, S, Hq, Hkv, K);
    return sas::bwd_simt_workspace(B, S, Hq, Hkv, D, K);
}

sas_status sas_attn_bwd(sas_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, const float* s, int ld_s, const float* lse_s,
                        const int32_t* idx, const int32_t* cnt, const float* log_gate, int B, int S, int Hq,
                        int Hkv, int D, int block_size, int K, float sm_scale, void* dq, void* dk, void* dv,
                        float* ds, void* workspace, size_t ws_bytes, void* stream) {
    sas_status r = check_attn_shape(dtype, q, k, v, B, S, Hq, Hkv, D, block_size, K, idx, cnt, log_gate);
    if (r != SAS_OK) return r;
    if (!o || !dout || !lse || !s || !lse_s || !dq || !dk || !dv || !ds || !workspace)
        return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd: null pointer");
    if (ld_s < S / 64) return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd: ld_s=%d < S/64", ld_s);
    if (!aligned16(o) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd: tensors not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd: workspace not 256-byte aligned");
    const size_t need = sas_attn_bwd_workspace_size(dtype, B, S, Hq, Hkv, D, K);
    if (ws_bytes < need) return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd: workspace %zu < %zu bytes", ws_bytes, need);
    if (!std::isfinite(sm_scale)) return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd: sm_scale not finite");
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "sas_attn_bwd: no CUDA device");
    sas::BwdArgs b{{q, k, v, B, S, Hq, Hkv, D, K, idx, cnt, log_gate, sm_scale, st},
                   o, dout, lse, s, ld_s, lse_s, dq, dk, dv, ds, workspace, ws_bytes};
    cudaError_t e = (dtype == SAS_BF16 && D == 128)
                        ? sas::launch_bwd_sm100(b, static_cast<cudaStream_t>(stream))
                        : sas::launch_bwd_simt(b, dtype == SAS_BF16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sas_attn_bwd");
}

size_t sas_decode_workspace_size(int N, int Hq, int Hkv, int D, int K) {
    if (N <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D != 128 || K < 0) return 0;
    return sas::decode_workspace(N, Hq, Hkv, D, K);
}

sas_status sas_decode_paged(const void* q, const void* k_cache, const void* v_cache, int num_pages,
                            const int32_t* page_table, int max_pages, const int32_t* kv_len, int N, int Hq,
                            int Hkv, int D, int page_size, int K, const int32_t* idx, const int32_t* cnt,
                            const float* log_gate, float sm_scale, void* o, float* lse, void* workspace,
                            size_t ws_bytes, void* stream) {
    if (!q || !k_cache || !v_cache || !page_table || !kv_len || !cnt || !o || !workspace)
        return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: null pointer");
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: null idx/log_gate with K > 0");
    if (N <= 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || max_pages <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: bad size");
    if (Hq % Hkv) return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: Hq %% Hkv != 0");
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 5 && G != 8)
        return fail(SAS_ERR_UNSUPPORTED, "sas_decode_paged: group size %d (1, 2, 4, 5 or 8)", G);
    if (page_size != 64) return fail(SAS_ERR_UNSUPPORTED, "sas_decode_paged: page_size=%d (only 64)", page_size);
    if (D != 128) return fail(SAS_ERR_UNSUPPORTED, "sas_decode_paged: D=%d (only 128)", D);
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: tensors not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: workspace not 256-byte aligned");
    const size_t need = sas_decode_workspace_size(N, Hq, Hkv, D, K);
    if (ws_bytes < need) return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: workspace %zu < %zu bytes", ws_bytes, need);
    if (!std::isfinite(sm_scale)) return fail(SAS_ERR_INVALID_ARG, "sas_decode_paged: sm_scale not finite");
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "sas_decode_paged: no CUDA device");
    sas::DecodeArgs a{q, k_cache, v_cache, num_pages, page_table, max_pages, kv_len, N, Hq, Hkv, D, K,
                      idx, cnt, log_gate, sm_scale, o, lse, st};
    cudaError_t e = sas::launch_decode(a, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sas_decode_paged");
}

sas_status sas_selftest_bounded_wait(void* stream) {
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "sas_selftest_bounded_wait: no CUDA device");
    cudaError_t e = sas::launch_bounded_wait_selftest(st, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "sas_selftest_bounded_wait");
}

}  // extern "C"
