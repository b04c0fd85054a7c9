// Device helpers shared by the SAS kernels (no method arithmetic lives here).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sas {

constexpr int kBlock = 64;            // tokens per block (= page size)

// Codes written to the per-device status word (match sas_status).
constexpr int kStatusBadData = 1;
constexpr int kStatusTimeout = 4;

__device__ __forceinline__ void flag_status(int* status, int code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

// Token rows of sequence b of a batch. Dense batches (cu == nullptr) hold B
// sequences of S tokens, sequence b at rows b*S .. b*S+S-1; packed batches
// hold sequence b at rows cu[b] .. cu[b+1]-1, with S the longest length.
// Packed bounds that are out of range (negative, longer than S, or past the
// T rows) are flagged and the sequence is treated as empty.
struct SeqRange {
    long long start;
    int len;
};
__device__ __forceinline__ SeqRange seq_range(const int32_t* cu, int b, int S, long long T, int* status) {
    SeqRange r;
    if (cu == nullptr) {
        r.start = (long long)b * S;
        r.len = S;
        return r;
    }
    const int a = __ldg(cu + b), e = __ldg(cu + b + 1);
    r.start = a;
    r.len = e - a;
    if (a < 0 || r.len < 0 || r.len > S || (long long)e > T) {
        flag_status(status, kStatusBadData);
        r.start = 0;
        r.len = 0;
    }
    return r;
}

// Sequence and position of token row `tok` (binary search over cu for packed
// batches). Returns false for a row that belongs to no sequence.
__device__ __forceinline__ bool token_seq(const int32_t* cu, int B, int S, long long tok, int& b, int& t) {
    if (cu == nullptr) {
        b = (int)(tok / S);
        t = (int)(tok % S);
        return b < B;
    }
    int lo = 0, hi = B;                      // find the last b with cu[b] <= tok
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)__ldg(cu + mid) <= tok) lo = mid; else hi = mid;
    }
    b = lo;
    const long long st = __ldg(cu + lo), en = __ldg(cu + lo + 1);
    t = (int)(tok - st);
    return tok >= st && tok < en && t < S;
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Unpack two bf16 (low half first) from a 32-bit word to fp32 exactly.
__device__ __forceinline__ float2 bf16x2_to_f32(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace sas
