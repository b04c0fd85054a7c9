// Top-K selection and log-gates of one score row held by one warp (the
// warp-per-row kernel of sas_select).
//
// SAS review (paper.oopus.info) §2.2 (Top-K of the selector scores) and §2.4,
// eq. log g (log g_m = s_m - LSE(s) over all history blocks). Exact and
// order-independent: every score is mapped to an order-preserving 32-bit key
// (-0.0 folded onto +0.0), a 32-step bitwise search finds the K-th largest
// key T, and the row keeps every key above T plus the lowest-indexed keys
// equal to T; kept indices come out ascending by a ballot/popc compaction in
// index order.
#pragma once

#include "common.cuh"

namespace sas {

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t b = __float_as_uint(x);
    if (b == 0x80000000u) b = 0u;                       // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);  // finite x -> key > 0
}

__device__ __forceinline__ bool finite_score(float x) { return fabsf(x) <= 3.402823466e38f; }

// The row's scores are val[e] for history block j = 32 e + lane (entries at
// j >= nh are ignored). A row holding a non-finite score is flagged and gets
// the empty selection with lse_s = NaN.
template <int E>
__device__ __forceinline__ void select_warp_row(const float (&val)[E], int nh, int K, long long row,
                                                int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                                                float* __restrict__ log_gate, float* __restrict__ lse_s, int* status) {
    const int lane = threadIdx.x & 31;
    uint32_t key[E];
    float m = -INFINITY;
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const bool in = e * 32 + lane < nh;
        key[e] = in ? order_key(val[e]) : 0u;
        bad |= in && !finite_score(val[e]);
        m = fmaxf(m, in ? val[e] : -INFINITY);
    }
    const long long obase = row * (long long)K;
    if (__any_sync(0xffffffffu, bad)) {
        // a non-finite score: no defined Top-K or LSE for this row
        if (lane == 0) {
            flag_status(status, kStatusBadData);
            cnt[row] = 0;
            lse_s[row] = __int_as_float(0x7fc00000);
        }
        for (int p = lane; p < K; p += 32) {
            idx[obase + p] = -1;
            log_gate[obase + p] = -INFINITY;
        }
        return;
    }
    m = warp_max(m);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e * 32 + lane < nh) acc += expf(val[e] - m);
    acc = warp_sum(acc);
    const float lse = (nh > 0) ? m + logf(acc) : -INFINITY;

    const int kk = min(K, nh);
    uint32_t T = 0u;          // keys > T are kept; keys == T kept by index
    int need = 0;             // how many keys equal to T to keep
    if (kk > 0 && kk < nh) {
        uint32_t prefix = 0u;
#pragma unroll 1
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t cand = prefix | (1u << bit);
            unsigned c = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) c += (key[e] >= cand);
            c = __reduce_add_sync(0xffffffffu, c);
            if (c >= (unsigned)kk) prefix = cand;
        }
        T = prefix;
        unsigned gt = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) gt += (key[e] > T);
        gt = __reduce_add_sync(0xffffffffu, gt);
        need = kk - (int)gt;
    }
    // kk == nh: every valid key (> 0) is kept (T = 0, need = 0)

    const unsigned lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, out = 0;
    if (kk > 0) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const bool valid = (e * 32 + lane) < nh;
            const bool eq = valid && key[e] == T;
            const unsigned eq_ball = __ballot_sync(0xffffffffu, eq);
            const int eq_rank = eq_seen + __popc(eq_ball & lt_mask);
            const bool keep = valid && (key[e] > T || (eq && eq_rank < need));
            const unsigned keep_ball = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const int pos = out + __popc(keep_ball & lt_mask);
                idx[obase + pos] = e * 32 + lane;
                log_gate[obase + pos] = val[e] - lse;
            }
            eq_seen += __popc(eq_ball);
            out += __popc(keep_ball);
        }
    }
    for (int p = kk + lane; p < K; p += 32) {
        idx[obase + p] = -1;
        log_gate[obase + p] = -INFINITY;
    }
    if (lane == 0) {
        cnt[row] = kk;
        lse_s[row] = lse;
    }
}

}  // namespace sas
