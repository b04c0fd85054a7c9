// sas_select: Top-K history blocks fused with the normalised log-gates.
//
// SAS review (paper.oopus.info) §2.2: keep the K history blocks with the
// highest selector scores. §2.4, eq. log g: each kept block m gets
// log g_m = s_m - LSE(s), the LSE over all history blocks of the row.
//
// Rows of up to 512 history blocks: one warp per row, the row's scores in
// registers (E per lane). Longer rows: one CTA per row (select_cta_kernel).
// The Top-K is exact and order-independent: every score is mapped to an
// order-preserving 32-bit key (-0.0 folded onto +0.0), a bitwise search
// finds the K-th largest key T, and the row keeps every key above T plus
// the lowest-indexed keys equal to T. Kept indices come out ascending by a
// ballot/popc compaction in index order.
#include "common.cuh"
#include "launch.h"

namespace sas {
namespace {

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t b = __float_as_uint(x);
    if (b == 0x80000000u) b = 0u;                       // -0.0 == +0.0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);  // finite x -> key > 0
}

template <int E>
__global__ void __launch_bounds__(256)
select_kernel(const float* __restrict__ s, int B, int Hkv, int n_rows, int ld_s,
              const int32_t* __restrict__ kv_len, int K,
              int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
              float* __restrict__ log_gate, float* __restrict__ lse_s, int* status) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long n_total = (long long)B * Hkv * n_rows;
    if (row >= n_total) return;
    const int r = (int)(row % n_rows);
    const int b = (int)(row / ((long long)Hkv * n_rows));

    int nh = r;
    if (kv_len != nullptr) {
        const int L = kv_len[b];
        nh = (L >= 1) ? (L - 1) / kBlock : 0;
        if (L < 1) flag_status(status, kStatusBadData);
    }
    if (nh > ld_s || nh > 32 * E) {
        flag_status(status, kStatusBadData);
        nh = min(ld_s, 32 * E);
    }
    const float* srow = s + row * (long long)ld_s;

    float val[E];
    uint32_t key[E];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = e * 32 + lane;
        val[e] = (j < nh) ? __ldg(srow + j) : -INFINITY;
        key[e] = (j < nh) ? order_key(val[e]) : 0u;
        m = fmaxf(m, val[e]);
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
    } else if (kk == nh) {
        T = 0u;               // every valid key (> 0) is kept
        need = 0;
    }

    const long long obase = row * (long long)K;
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

// Long rows: one CTA of W warps per row, E keys per lane (rows of up to
// 32*W*E history blocks; key j held by lane j % 32 of warp (j / 32) % W as
// element j / (32 W)). Same exact selection as select_kernel; the counts of
// the bitwise search and of the compaction are summed over the warps through
// shared memory. A kept key's output position is (# keys > T before it) +
// min(need, # keys == T before it), so indices come out ascending.
template <int E, int W>
__global__ void __launch_bounds__(W * 32)
select_cta_kernel(const float* __restrict__ s, int B, int Hkv, int n_rows, int ld_s,
                  const int32_t* __restrict__ kv_len, int K,
                  int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                  float* __restrict__ log_gate, float* __restrict__ lse_s, int* status) {
    __shared__ float red_f[W];
    __shared__ unsigned red_u[2][W];
    __shared__ unsigned red_eq[2][W], red_gt[2][W];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long row = blockIdx.x;
    const int r = (int)(row % n_rows);
    const int b = (int)(row / ((long long)Hkv * n_rows));

    int nh = r;
    if (kv_len != nullptr) {
        const int L = kv_len[b];
        nh = (L >= 1) ? (L - 1) / kBlock : 0;
        if (L < 1 && threadIdx.x == 0) flag_status(status, kStatusBadData);
    }
    if (nh > ld_s || nh > 32 * W * E) {
        if (threadIdx.x == 0) flag_status(status, kStatusBadData);
        nh = min(ld_s, 32 * W * E);
    }
    const float* srow = s + row * (long long)ld_s;

    float val[E];
    uint32_t key[E];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = (e * W + warp) * 32 + lane;
        val[e] = (j < nh) ? __ldg(srow + j) : -INFINITY;
        key[e] = (j < nh) ? order_key(val[e]) : 0u;
        m = fmaxf(m, val[e]);
    }
    m = warp_max(m);
    if (lane == 0) red_f[warp] = m;
    __syncthreads();
    m = red_f[0];
#pragma unroll
    for (int w = 1; w < W; ++w) m = fmaxf(m, red_f[w]);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((e * W + warp) * 32 + lane < nh) acc += expf(val[e] - m);
    acc = warp_sum(acc);
    __syncthreads();                          // every thread has read red_f
    if (lane == 0) red_f[warp] = acc;
    __syncthreads();
    acc = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) acc += red_f[w];
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
            if (lane == 0) red_u[bit & 1][warp] = c;      // alternate buffers: one barrier per step
            __syncthreads();
            unsigned tot = 0;
#pragma unroll
            for (int w = 0; w < W; ++w) tot += red_u[bit & 1][w];
            if (tot >= (unsigned)kk) prefix = cand;
        }
        T = prefix;
        unsigned gt = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) gt += (key[e] > T);
        gt = __reduce_add_sync(0xffffffffu, gt);
        __syncthreads();                      // the last search step's buffer has been read
        if (lane == 0) red_u[0][warp] = gt;
        __syncthreads();
        unsigned tot = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) tot += red_u[0][w];
        need = kk - (int)tot;
    }
    // kk == nh: every valid key (> 0) is kept (T = 0, need = 0)

    const long long obase = row * (long long)K;
    const unsigned lt_mask = (1u << lane) - 1u;
    if (kk > 0) {
        int eq_seen = 0, gt_seen = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const bool valid = ((e * W + warp) * 32 + lane) < nh;
            const bool eq = valid && key[e] == T;
            const bool gtk = valid && key[e] > T;
            const unsigned eq_ball = __ballot_sync(0xffffffffu, eq);
            const unsigned gt_ball = __ballot_sync(0xffffffffu, gtk);
            if (lane == 0) {
                red_eq[e & 1][warp] = __popc(eq_ball);
                red_gt[e & 1][warp] = __popc(gt_ball);
            }
            __syncthreads();
            int eq_before = eq_seen, gt_before = gt_seen;
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const int ce = (int)red_eq[e & 1][w], cg = (int)red_gt[e & 1][w];
                if (w < warp) {
                    eq_before += ce;
                    gt_before += cg;
                }
                eq_seen += ce;
                gt_seen += cg;
            }
            const int eq_rank = eq_before + __popc(eq_ball & lt_mask);
            const int gt_rank = gt_before + __popc(gt_ball & lt_mask);
            if (gtk || (eq && eq_rank < need)) {
                const int pos = gt_rank + min(need, eq_rank);
                idx[obase + pos] = (e * W + warp) * 32 + lane;
                log_gate[obase + pos] = val[e] - lse;
            }
        }
    }
    for (int p = kk + (int)threadIdx.x; p < K; p += W * 32) {
        idx[obase + p] = -1;
        log_gate[obase + p] = -INFINITY;
    }
    if (threadIdx.x == 0) {
        cnt[row] = kk;
        lse_s[row] = lse;
    }
}

template <int E, int W>
cudaError_t go_cta(const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* kv_len, int K,
                   int32_t* idx, int32_t* cnt, float* lg, float* lse_s, int* status, cudaStream_t st) {
    const long long rows = (long long)B * Hkv * n_rows;
    select_cta_kernel<E, W><<<(unsigned)rows, W * 32, 0, st>>>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, lg,
                                                             lse_s, status);
    count_launches(1);
    return cudaGetLastError();
}

template <int E>
cudaError_t go(const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* kv_len, int K,
               int32_t* idx, int32_t* cnt, float* lg, float* lse_s, int* status, cudaStream_t st) {
    const long long rows = (long long)B * Hkv * n_rows;
    const int warps = 8;
    const long long grid = (rows + warps - 1) / warps;
    select_kernel<E><<<(unsigned)grid, warps * 32, 0, st>>>(s, B, Hkv, n_rows, ld_s, kv_len, K,
                                                            idx, cnt, lg, lse_s, status);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const float* s, int B, int Hkv, int n_rows, int ld_s,
                          const int32_t* kv_len, int K, int max_hist,
                          int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s,
                          int* status, cudaStream_t st) {
    if (max_hist <= 32) return go<1>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, log_gate, lse_s, status, st);
    if (max_hist <= 64) return go<2>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, log_gate, lse_s, status, st);
    if (max_hist <= 128) return go<4>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, log_gate, lse_s, status, st);
    if (max_hist <= 256) return go<8>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, log_gate, lse_s, status, st);
    if (max_hist <= 512) return go<16>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, log_gate, lse_s, status, st);
    // longer rows (decode: one row per sequence and KV head, so few rows): a CTA
    // per row, so that the 32-step search is not one warp's serial chain
    return go_cta<4, 8>(s, B, Hkv, n_rows, ld_s, kv_len, K, idx, cnt, log_gate, lse_s, status, st);
}

}  // namespace sas
