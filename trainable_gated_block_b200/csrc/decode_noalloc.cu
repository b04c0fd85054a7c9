// sas_decode_paged_noalloc: paged decode that needs no workspace from the caller.
//
// sas_decode_paged keeps its split-KV partial results in a workspace the
// caller allocates. Some callers cannot allocate device memory when they
// decode: a serving engine that hands nearly all of the GPU's memory to its
// KV-cache pool at start-up and has nothing left to give, or a plain C host
// that holds device pointers to its inputs and outputs but has no device
// allocator of its own. This entry point serves them: the partials live in
// one file-scope device array that the library reserves when it is loaded.
//
// Limits and sharing rules (also stated in include/sas.h):
//   * the array holds kScratchBytes; a call whose partials need more is
//     rejected on the host with SAS_ERR_INVALID_ARG before anything runs;
//   * every GPU that loads the library keeps the array until the process exits;
//   * all calls on a device share the one array and it keeps what the last
//     call wrote. Nothing in it has to start at zero: each split writes its
//     whole partial before the combine step reads it. Calls that overlap on
//     the GPU (different streams, or threads without ordering) race on it.
//   * the first call on a device looks up the array's device address (with
//     that device current) and caches it with the id of the current context;
//     it is looked up again only when another context is current (after a
//     cudaDeviceReset). Make the first call on a device, and the first call
//     after a reset, before any stream capture.
// No cudaMalloc, cudaFree or allocating library routine is called here.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/sas.h"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;     // 16 MiB

// Host code must not use this name as an address: on the host it is only a
// stand-in symbol. Its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
unsigned long long g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_addr[kMaxDevices] = {};

cudaError_t scratch_lookup(void** out) { return cudaGetSymbolAddress(out, g_decode_scratch); }

}  // namespace

extern "C" sas_status sas_decode_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                               int num_pages, const int32_t* page_table, int max_pages,
                                               const int32_t* kv_len, int N, int Hq, int Hkv, int D,
                                               int page_size, int K, const int32_t* idx, const int32_t* cnt,
                                               const float* log_gate, float sm_scale, void* o, float* lse,
                                               void* stream) {
    const size_t need = sas_decode_workspace_size(N, Hq, Hkv, D, K);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "sas_decode_paged_noalloc: these sizes need %zu bytes of scratch; the library's static "
                 "scratch holds %zu bytes (use sas_decode_paged with a workspace)", need, kScratchBytes);
        sas::set_last_error(msg);
        return SAS_ERR_INVALID_ARG;
    }
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        sas::set_last_error("sas_decode_paged_noalloc: no usable current CUDA device");
        return SAS_ERR_CUDA;
    }
    // Set-up: the array's device address, looked up with this device current
    // and cached together with the id of the context it belongs to (after a
    // cudaDeviceReset the device gets a new context and the array a new
    // address, so the lookup is repeated whenever the context changes).
    void* ptr = nullptr;
    e = sas::cached_symbol_address(dev, &g_scratch_mu, g_scratch_ctx, g_scratch_addr, scratch_lookup, &ptr);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "sas_decode_paged_noalloc: cudaGetSymbolAddress failed: %s",
                 cudaGetErrorString(e));
        sas::set_last_error(msg);
        return SAS_ERR_CUDA;
    }
    // Same validation and kernels as the workspace entry point, on the static scratch.
    return sas_decode_paged(q, k_cache, v_cache, num_pages, page_table, max_pages, kv_len, N, Hq, Hkv, D,
                            page_size, K, idx, cnt, log_gate, sm_scale, o, lse, ptr, kScratchBytes, stream);
}
