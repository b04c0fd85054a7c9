// C ABI of libsas.so (declared in include/sas.h): host-side validation,
// per-device status word, and dispatch to the kernel launchers.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

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

// Device address of g_status_word, cached per device together with the
// context it was looked up in: a module variable gets a new address when the
// device's context is destroyed and created again (cudaDeviceReset), so a
// cached address is only reused while the same context is current.
struct SymbolCache {
    std::mutex mu;
    unsigned long long ctx[kMaxDevices] = {};
    void* ptr[kMaxDevices] = {};
};
SymbolCache g_status_cache;

int* status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = nullptr;
    if (sas::cached_symbol_address(dev, &g_status_cache.mu, g_status_cache.ctx, g_status_cache.ptr,
                                   [](void** out) { return cudaGetSymbolAddress(out, g_status_word); },
                                   &p) != cudaSuccess)
        return nullptr;
    return static_cast<int*>(p);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shapes shared by the dense and packed entry points: B sequences of at most
// S tokens in T token rows (dense: T = B * S).
sas_status check_attn_shape(const char* fn, sas_dtype dtype, const void* q, const void* k, const void* v, int B,
                            int S, long long T, int Hq, int Hkv, int D, int block_size, int K, const int32_t* idx,
                            const int32_t* cnt, const float* log_gate) {
    if (dtype != SAS_F32 && dtype != SAS_BF16) return fail(SAS_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
    if (!q || !k || !v || !cnt) return fail(SAS_ERR_INVALID_ARG, "%s: null tensor pointer", fn);
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "%s: null idx/log_gate with K > 0", fn);
    if (B <= 0 || S <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "%s: non-positive size (B=%d S=%d T=%lld Hq=%d Hkv=%d D=%d K=%d)", fn, B, S,
                    T, Hq, Hkv, D, K);
    if (Hq % Hkv) return fail(SAS_ERR_INVALID_ARG, "%s: Hq=%d is not a multiple of Hkv=%d", fn, Hq, Hkv);
    if (block_size != 64) return fail(SAS_ERR_UNSUPPORTED, "%s: block_size=%d (only 64)", fn, block_size);
    if (D != 64 && D != 128) return fail(SAS_ERR_UNSUPPORTED, "%s: D=%d (only 64 or 128)", fn, D);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v))
        return fail(SAS_ERR_INVALID_ARG, "%s: q/k/v not 16-byte aligned", fn);
    if (T * Hq > (1LL << 31) - 1 || (long long)B * S * Hq > (1LL << 31) - 1)
        return fail(SAS_ERR_UNSUPPORTED, "%s: token rows x query heads beyond 2^31", fn);
    return SAS_OK;
}

// Query blocks per sequence above which the backward's reverse index (block
// and slot packed into 16 bits each) does not fit.
constexpr int kMaxBwdBlocks = 32767;

sas_status attn_fwd_impl(const char* fn, sas_dtype dtype, const void* q, const void* k, const void* v,
                         const int32_t* cu, int B, int S, long long T, int Hq, int Hkv, int D, int block_size, int K,
                         const int32_t* idx, const int32_t* cnt, const float* log_gate, float sm_scale, void* o,
                         float* lse, void* stream) {
    sas_status r = check_attn_shape(fn, dtype, q, k, v, B, S, T, Hq, Hkv, D, block_size, K, idx, cnt, log_gate);
    if (r != SAS_OK) return r;
    if (!o || !lse) return fail(SAS_ERR_INVALID_ARG, "%s: null output", fn);
    if (!aligned16(o)) return fail(SAS_ERR_INVALID_ARG, "%s: o not 16-byte aligned", fn);
    if (!std::isfinite(sm_scale)) return fail(SAS_ERR_INVALID_ARG, "%s: sm_scale not finite", fn);
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "%s: no CUDA device", fn);
    sas::AttnArgs a{q, k, v, B, S, Hq, Hkv, D, K, cu, T, idx, cnt, log_gate, sm_scale, st};
    cudaError_t e = (dtype == SAS_BF16 && D == 128)
                        ? sas::launch_fwd_sm100(a, o, lse, static_cast<cudaStream_t>(stream))
                        : sas::launch_fwd_simt(a, dtype == SAS_BF16, o, lse, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

size_t bwd_workspace(sas_dtype dtype, int B, int S, long long T, int Hq, int Hkv, int D, int K) {
    if ((dtype != SAS_F32 && dtype != SAS_BF16) || B <= 0 || S <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv ||
        (D != 64 && D != 128) || K < 0)
        return 0;
    if (dtype == SAS_BF16 && D == 128) {
        if ((S + 63) / 64 > kMaxBwdBlocks) return 0;
        return sas::bwd_sm100_workspace(B, S, Hq, Hkv, K);
    }
    return sas::bwd_simt_workspace(B, S, T, Hq, Hkv, D, K);
}

sas_status attn_bwd_impl(const char* fn, sas_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, const float* s, int ld_s, const float* lse_s,
                         const int32_t* idx, const int32_t* cnt, const float* log_gate, const int32_t* cu, int B,
                         int S, long long T, int Hq, int Hkv, int D, int block_size, int K, float sm_scale, void* dq,
                         void* dk, void* dv, float* ds, void* workspace, size_t ws_bytes, void* stream) {
    sas_status r = check_attn_shape(fn, dtype, q, k, v, B, S, T, Hq, Hkv, D, block_size, K, idx, cnt, log_gate);
    if (r != SAS_OK) return r;
    if (!o || !dout || !lse || !s || !lse_s || !dq || !dk || !dv || !ds || !workspace)
        return fail(SAS_ERR_INVALID_ARG, "%s: null pointer", fn);
    const int nqb = (S + 63) / 64;
    if (ld_s < nqb) return fail(SAS_ERR_INVALID_ARG, "%s: ld_s=%d < %d blocks", fn, ld_s, nqb);
    if (dtype == SAS_BF16 && D == 128 && nqb > kMaxBwdBlocks)
        return fail(SAS_ERR_UNSUPPORTED, "%s: %d query blocks per sequence (at most %d)", fn, nqb, kMaxBwdBlocks);
    if (!aligned16(o) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return fail(SAS_ERR_INVALID_ARG, "%s: tensors not 16-byte aligned", fn);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SAS_ERR_INVALID_ARG, "%s: workspace not 256-byte aligned", fn);
    const size_t need = bwd_workspace(dtype, B, S, T, Hq, Hkv, D, K);
    if (ws_bytes < need) return fail(SAS_ERR_INVALID_ARG, "%s: workspace %zu < %zu bytes", fn, ws_bytes, need);
    if (!std::isfinite(sm_scale)) return fail(SAS_ERR_INVALID_ARG, "%s: sm_scale not finite", fn);
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "%s: no CUDA device", fn);
    sas::BwdArgs b{{q, k, v, B, S, Hq, Hkv, D, K, cu, T, idx, cnt, log_gate, sm_scale, st},
                   o, dout, lse, s, ld_s, lse_s, dq, dk, dv, ds, workspace, ws_bytes};
    cudaError_t e = (dtype == SAS_BF16 && D == 128)
                        ? sas::launch_bwd_sm100(b, static_cast<cudaStream_t>(stream))
                        : sas::launch_bwd_simt(b, dtype == SAS_BF16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

// Longest row sas_select handles (history blocks), = 1M tokens of context.
constexpr int kMaxHistory = 16384;

sas_status select_impl(const char* fn, const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* kv_len,
                       const int32_t* cu, int block_size, int K, int32_t* idx, int32_t* cnt, float* log_gate,
                       float* lse_s, void* stream) {
    if (!s || !cnt || !lse_s) return fail(SAS_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "%s: null idx/log_gate with K > 0", fn);
    if (B <= 0 || Hkv <= 0 || n_rows <= 0 || ld_s <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "%s: bad size (B=%d Hkv=%d n_rows=%d ld_s=%d K=%d)", fn, B, Hkv, n_rows, ld_s, K);
    if (block_size != 64) return fail(SAS_ERR_UNSUPPORTED, "%s: block_size=%d (only 64)", fn, block_size);
    if (!kv_len && ld_s < n_rows) return fail(SAS_ERR_INVALID_ARG, "%s: prefill needs ld_s >= n_rows", fn);
    const int max_hist = kv_len ? ld_s : n_rows - 1;
    if (max_hist > kMaxHistory)
        return fail(SAS_ERR_UNSUPPORTED, "%s: rows of more than %d history blocks", fn, kMaxHistory);
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "%s: no CUDA device", fn);
    cudaError_t e = sas::launch_select(s, B, Hkv, n_rows, ld_s, kv_len, cu, K, max_hist, idx, cnt, log_gate, lse_s,
                                       st, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

}  // namespace

namespace sas {

unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (get_cur == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    unsigned long long id = 0;
    return get_id(ctx, &id) == CUDA_SUCCESS ? id + 1 : 0;   // +1: 0 means "unknown"
}

cudaError_t cached_symbol_address(int dev, std::mutex* mu, unsigned long long* ctx_ids, void** ptrs,
                                  cudaError_t (*lookup)(void**), void** out) {
    *out = nullptr;
    std::lock_guard<std::mutex> lock(*mu);
    const unsigned long long id = current_context_id();     // 0 before the runtime made its context
    if (id != 0 && ctx_ids[dev] == id && ptrs[dev] != nullptr) {
        *out = ptrs[dev];
        return cudaSuccess;
    }
    void* p = nullptr;
    const cudaError_t e = lookup(&p);                       // creates the context if needed
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    ctx_ids[dev] = current_context_id();   // 0 (unknown) never matches: looked up again next call
    ptrs[dev] = p;
    *out = p;
    return cudaSuccess;
}

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
    return select_impl("sas_select", s, B, Hkv, n_rows, ld_s, kv_len, nullptr, block_size, K, idx, cnt, log_gate,
                       lse_s, stream);
}

sas_status sas_select_varlen(const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* cu_seqlens,
                             int block_size, int K, int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s,
                             void* stream) {
    if (!cu_seqlens) return fail(SAS_ERR_INVALID_ARG, "sas_select_varlen: null cu_seqlens");
    return select_impl("sas_select_varlen", s, B, Hkv, n_rows, ld_s, nullptr, cu_seqlens, block_size, K, idx, cnt,
                       log_gate, lse_s, stream);
}

sas_status sas_attn_fwd(sas_dtype dtype, const void* q, const void* k, const void* v, int B, int S, int Hq,
                        int Hkv, int D, int block_size, int K, const int32_t* idx, const int32_t* cnt,
                        const float* log_gate, float sm_scale, void* o, float* lse, void* stream) {
    return attn_fwd_impl("sas_attn_fwd", dtype, q, k, v, nullptr, B, S, (long long)B * S, Hq, Hkv, D, block_size, K,
                         idx, cnt, log_gate, sm_scale, o, lse, stream);
}

sas_status sas_attn_fwd_varlen(sas_dtype dtype, const void* q, const void* k, const void* v,
                               const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq, int Hkv,
                               int D, int block_size, int K, const int32_t* idx, const int32_t* cnt,
                               const float* log_gate, float sm_scale, void* o, float* lse, void* stream) {
    if (!cu_seqlens) return fail(SAS_ERR_INVALID_ARG, "sas_attn_fwd_varlen: null cu_seqlens");
    return attn_fwd_impl("sas_attn_fwd_varlen", dtype, q, k, v, cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv, D,
                         block_size, K, idx, cnt, log_gate, sm_scale, o, lse, stream);
}

size_t sas_attn_bwd_workspace_size(sas_dtype dtype, int B, int S, int Hq, int Hkv, int D, int K) {
    return bwd_workspace(dtype, B, S, (long long)B * S, Hq, Hkv, D, K);
}

size_t sas_attn_bwd_varlen_workspace_size(sas_dtype dtype, int B, int max_seqlen, int total_tokens, int Hq, int Hkv,
                                          int D, int K) {
    return bwd_workspace(dtype, B, max_seqlen, total_tokens, Hq, Hkv, D, K);
}

sas_status sas_attn_bwd(sas_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, const float* s, int ld_s, const float* lse_s,
                        const int32_t* idx, const int32_t* cnt, const float* log_gate, int B, int S, int Hq,
                        int Hkv, int D, int block_size, int K, float sm_scale, void* dq, void* dk, void* dv,
                        float* ds, void* workspace, size_t ws_bytes, void* stream) {
    return attn_bwd_impl("sas_attn_bwd", dtype, q, k, v, o, dout, lse, s, ld_s, lse_s, idx, cnt, log_gate, nullptr, B,
                         S, (long long)B * S, Hq, Hkv, D, block_size, K, sm_scale, dq, dk, dv, ds, workspace,
                         ws_bytes, stream);
}

sas_status sas_attn_bwd_varlen(sas_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                               const void* dout, const float* lse, const float* s, int ld_s, const float* lse_s,
                               const int32_t* idx, const int32_t* cnt, const float* log_gate,
                               const int32_t* cu_seqlens, int B, int max_seqlen, int total_tokens, int Hq, int Hkv,
                               int D, int block_size, int K, float sm_scale, void* dq, void* dk, void* dv, float* ds,
                               void* workspace, size_t ws_bytes, void* stream) {
    if (!cu_seqlens) return fail(SAS_ERR_INVALID_ARG, "sas_attn_bwd_varlen: null cu_seqlens");
    return attn_bwd_impl("sas_attn_bwd_varlen", dtype, q, k, v, o, dout, lse, s, ld_s, lse_s, idx, cnt, log_gate,
                         cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv, D, block_size, K, sm_scale, dq, dk, dv, ds,
                         workspace, ws_bytes, stream);
}

size_t sas_score_select_workspace_size(int B, int S, int Hq, int Hkv, int D) {
    if (B <= 0 || S <= 0 || S % 64 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || (D != 64 && D != 128)) return 0;
    return sas::score_workspace(B, S, Hkv, D);
}

sas_status sas_score_select(const void* q, const void* k, const float* noise, int ld_noise, int B, int S, int Hq,
                            int Hkv, int D, int block_size, int K, float* s, int ld_s, int32_t* idx, int32_t* cnt,
                            float* log_gate, float* lse_s, void* workspace, size_t ws_bytes, void* stream) {
    const char* fn = "sas_score_select";
    if (!q || !k || !s || !cnt || !lse_s || !workspace) return fail(SAS_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "%s: null idx/log_gate with K > 0", fn);
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "%s: bad size (B=%d S=%d Hq=%d Hkv=%d K=%d)", fn, B, S, Hq, Hkv, K);
    if (Hq % Hkv) return fail(SAS_ERR_INVALID_ARG, "%s: Hq=%d is not a multiple of Hkv=%d", fn, Hq, Hkv);
    if (block_size != 64) return fail(SAS_ERR_UNSUPPORTED, "%s: block_size=%d (only 64)", fn, block_size);
    if (S % 64) return fail(SAS_ERR_UNSUPPORTED, "%s: S=%d is not a multiple of 64 (pooling needs full blocks)", fn, S);
    if (D != 64 && D != 128) return fail(SAS_ERR_UNSUPPORTED, "%s: D=%d (only 64 or 128)", fn, D);
    const int nqb = S / 64;
    if (ld_s < nqb || (noise && ld_noise < nqb))
        return fail(SAS_ERR_INVALID_ARG, "%s: row strides (ld_s=%d, ld_noise=%d) below %d blocks", fn, ld_s, ld_noise, nqb);
    if (nqb - 1 > kMaxHistory)
        return fail(SAS_ERR_UNSUPPORTED, "%s: rows of more than %d history blocks", fn, kMaxHistory);
    if ((long long)B * Hkv > 65535)     // grid dimension of the score tiles
        return fail(SAS_ERR_UNSUPPORTED, "%s: B*Hkv=%lld above 65535", fn, (long long)B * Hkv);
    if ((size_t)(Hq + Hkv) * D * sizeof(float) > 200 * 1024)
        return fail(SAS_ERR_UNSUPPORTED, "%s: %d + %d heads of %d dims exceed the pooling CTA's shared memory", fn,
                    Hq, Hkv, D);
    if ((long long)B * S * Hq > (1LL << 31) - 1) return fail(SAS_ERR_UNSUPPORTED, "%s: B*S*Hq too large", fn);
    if (!aligned16(q) || !aligned16(k)) return fail(SAS_ERR_INVALID_ARG, "%s: q/k not 16-byte aligned", fn);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(SAS_ERR_INVALID_ARG, "%s: workspace not 256-byte aligned", fn);
    const size_t need = sas::score_workspace(B, S, Hkv, D);
    if (ws_bytes < need) return fail(SAS_ERR_INVALID_ARG, "%s: workspace %zu < %zu bytes", fn, ws_bytes, need);
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "%s: no CUDA device", fn);
    sas::ScoreArgs a{q, k, noise, ld_noise, B, S, Hq, Hkv, D, K, s, ld_s, idx, cnt, log_gate, lse_s, workspace, st};
    cudaError_t e = sas::launch_score_select(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

sas_status sas_pool_pages(const void* k_cache, int num_pages, int Hkv, int D, int page_size, const int32_t* pages,
                          int n_pages, float* kpool, void* stream) {
    const char* fn = "sas_pool_pages";
    if (!k_cache || !kpool) return fail(SAS_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (num_pages <= 0 || Hkv <= 0 || (pages && n_pages < 0)) return fail(SAS_ERR_INVALID_ARG, "%s: bad size", fn);
    if (page_size != 64) return fail(SAS_ERR_UNSUPPORTED, "%s: page_size=%d (only 64)", fn, page_size);
    if (D != 64 && D != 128) return fail(SAS_ERR_UNSUPPORTED, "%s: D=%d (only 64 or 128)", fn, D);
    if (!aligned16(k_cache) || !aligned16(kpool)) return fail(SAS_ERR_INVALID_ARG, "%s: not 16-byte aligned", fn);
    const int n = pages ? n_pages : num_pages;
    if (n == 0) return ok();
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "%s: no CUDA device", fn);
    cudaError_t e = sas::launch_pool_pages(k_cache, num_pages, Hkv, D, pages, n, kpool, st,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
}

sas_status sas_score_select_decode(const void* q, const float* kpool, int num_pages, const int32_t* page_table,
                                   int max_pages, const int32_t* kv_len, int N, int Hq, int Hkv, int D,
                                   int page_size, const float* noise, int ld_noise, int K, float* s, int ld_s,
                                   int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s, void* stream) {
    const char* fn = "sas_score_select_decode";
    if (!q || !kpool || !page_table || !kv_len || !s || !cnt || !lse_s)
        return fail(SAS_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (K > 0 && (!idx || !log_gate)) return fail(SAS_ERR_INVALID_ARG, "%s: null idx/log_gate with K > 0", fn);
    if (N <= 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || max_pages <= 0 || ld_s <= 0 || K < 0)
        return fail(SAS_ERR_INVALID_ARG, "%s: bad size", fn);
    if (Hq % Hkv) return fail(SAS_ERR_INVALID_ARG, "%s: Hq %% Hkv != 0", fn);
    if (page_size != 64) return fail(SAS_ERR_UNSUPPORTED, "%s: page_size=%d (only 64)", fn, page_size);
    if (D != 64 && D != 128) return fail(SAS_ERR_UNSUPPORTED, "%s: D=%d (only 64 or 128)", fn, D);
    if (noise && ld_noise < ld_s) return fail(SAS_ERR_INVALID_ARG, "%s: ld_noise=%d < ld_s=%d", fn, ld_noise, ld_s);
    if (ld_s > kMaxHistory) return fail(SAS_ERR_UNSUPPORTED, "%s: rows of more than %d history blocks", fn, kMaxHistory);
    if ((long long)N * Hkv > 65535)     // grid dimension of the scoring kernel
        return fail(SAS_ERR_UNSUPPORTED, "%s: N*Hkv=%lld above 65535", fn, (long long)N * Hkv);
    if (!aligned16(kpool)) return fail(SAS_ERR_INVALID_ARG, "%s: kpool not 16-byte aligned", fn);
    int* st = status_ptr();
    if (!st) return fail(SAS_ERR_CUDA, "%s: no CUDA device", fn);
    sas::DecodeScoreArgs a{q, kpool, num_pages, page_table, max_pages, kv_len, N, Hq, Hkv, D, K, noise, ld_noise,
                           s, ld_s, idx, cnt, log_gate, lse_s, st};
    cudaError_t e = sas::launch_score_select_decode(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, fn);
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
