// sas_select: Top-K history blocks fused with the normalised log-gates.
//
// SAS review (paper.oopus.info) §2.2: keep the K history blocks with the
// highest selector scores. §2.4, eq. log g: each kept block m gets
// log g_m = s_m - LSE(s), the LSE over all history blocks of the row.
//
// Rows of up to 512 history blocks: one warp per row, the row's scores in
// registers (E per lane), the K-th largest key found by a 32-step bitwise
// search with warp reductions. Longer rows (decode at long context): one CTA
// per row (select_cta_kernel), the K-th largest key found by a 4-pass radix
// select over 8-bit digits with shared-memory histograms.
// The Top-K is exact and order-independent: every score is mapped to an
// order-preserving 32-bit key (-0.0 folded onto +0.0); the row keeps every
// key above the K-th largest key T plus the lowest-indexed keys equal to T.
// Kept indices come out ascending by a ballot/popc compaction in index order.
//
// Rows are checked: a row whose history holds a non-finite score (NaN or
// +-inf) is flagged in the status word and given the empty selection (cnt 0,
// indices -1, log-gates -inf) with lse_s = NaN. In prefill with per-sequence
// lengths, rows past a sequence's last block are padding: empty selection,
// lse_s = -inf, nothing read.
#include "common.cuh"
#include "launch.h"
#include "select_row.cuh"

namespace sas {
namespace {

struct RowCtx {
    int nh;          // history blocks of the row
    bool pad;        // padding row (past its sequence's last block): empty, lse -inf, nothing read
};

// History length of selection row `row` (= (b, h, r) flattened).
//  decode (kv_len != null): nh = (kv_len[b] - 1) / 64
//  prefill: nh = r; with per-sequence lengths (cu != null) rows r >= ceil(len_b / 64) are padding
__device__ __forceinline__ RowCtx row_ctx(long long row, int Hkv, int n_rows, int ld_s, int cap,
                                          const int32_t* __restrict__ kv_len, const int32_t* __restrict__ cu,
                                          int* status, bool leader) {
    RowCtx c;
    const int r = (int)(row % n_rows);
    const int b = (int)(row / ((long long)Hkv * n_rows));
    c.pad = false;
    c.nh = r;
    if (kv_len != nullptr) {
        const int L = kv_len[b];
        c.nh = (L >= 1) ? (L - 1) / kBlock : 0;
        if (L < 1 && leader) flag_status(status, kStatusBadData);
    } else if (cu != nullptr) {
        const int len = cu[b + 1] - cu[b];
        if (len < 0 && leader) flag_status(status, kStatusBadData);
        c.pad = r >= (max(len, 0) + kBlock - 1) / kBlock;
    }
    if (c.nh > ld_s || c.nh > cap) {
        if (leader) flag_status(status, kStatusBadData);
        c.nh = min(ld_s, cap);
    }
    return c;
}

template <int E>
__global__ void __launch_bounds__(256)
select_kernel(const float* __restrict__ s, int B, int Hkv, int n_rows, int ld_s,
              const int32_t* __restrict__ kv_len, const int32_t* __restrict__ cu, int K,
              int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
              float* __restrict__ log_gate, float* __restrict__ lse_s, int* status) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long n_total = (long long)B * Hkv * n_rows;
    if (row >= n_total) return;
    const RowCtx rc = row_ctx(row, Hkv, n_rows, ld_s, 32 * E, kv_len, cu, status, lane == 0);
    const int nh = rc.pad ? 0 : rc.nh;
    const float* srow = s + row * (long long)ld_s;
    float val[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = e * 32 + lane;
        val[e] = (j < nh) ? __ldg(srow + j) : -INFINITY;
    }
    select_warp_row<E>(val, nh, K, row, idx, cnt, log_gate, lse_s, status);
}

// Long rows: one CTA of W warps per row, E keys per thread (rows of up to
// 32 * W * E history blocks; key j held by thread j % (32 W) as element
// j / (32 W), so the loads are coalesced). LSE by block reductions. The K-th
// largest key T is found by a radix select: four passes over 8-bit digits,
// most significant first; each pass histograms the digit of the keys that
// still match the prefix found so far (shared-memory atomics, one per group of
// lanes of a warp holding the same digit), and one warp scans the 256 bins
// from the top to find the digit holding the K-th key.
// A kept key's output position is (# keys > T before it) + min(need,
// # keys == T before it), so indices come out ascending.
template <int E, int W>
__global__ void __launch_bounds__(W * 32)
select_cta_kernel(const float* __restrict__ s, int B, int Hkv, int n_rows, int ld_s,
                  const int32_t* __restrict__ kv_len, const int32_t* __restrict__ cu, int K,
                  int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                  float* __restrict__ log_gate, float* __restrict__ lse_s, int* status) {
    constexpr int NT = W * 32;
    __shared__ float red_f[W];
    __shared__ unsigned hist[256];
    __shared__ unsigned sel_digit, sel_need;
    __shared__ unsigned cnt_eq[E][W], cnt_gt[E][W], tot_eq[E], tot_gt[E];
    __shared__ int any_bad;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long row = blockIdx.x;
    const RowCtx rc = row_ctx(row, Hkv, n_rows, ld_s, NT * E, kv_len, cu, status, threadIdx.x == 0);
    const int nh = rc.pad ? 0 : rc.nh;
    const float* srow = s + row * (long long)ld_s;
    if (threadIdx.x == 0) any_bad = 0;

    float val[E];
    uint32_t key[E];
    float m = -INFINITY;
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = e * NT + (int)threadIdx.x;
        val[e] = (j < nh) ? __ldg(srow + j) : -INFINITY;
        key[e] = (j < nh) ? order_key(val[e]) : 0u;
        bad |= (j < nh) && !finite_score(val[e]);
        m = fmaxf(m, val[e]);
    }
    __syncthreads();                          // any_bad initialised
    if (__any_sync(0xffffffffu, bad) && lane == 0) any_bad = 1;
    m = warp_max(m);
    if (lane == 0) red_f[warp] = m;
    __syncthreads();
    const long long obase = row * (long long)K;
    if (any_bad) {
        // a non-finite score: no defined Top-K or LSE for this row
        if (threadIdx.x == 0) {
            flag_status(status, kStatusBadData);
            cnt[row] = 0;
            lse_s[row] = __int_as_float(0x7fc00000);
        }
        for (int p = threadIdx.x; p < K; p += NT) {
            idx[obase + p] = -1;
            log_gate[obase + p] = -INFINITY;
        }
        return;
    }
    m = red_f[0];
#pragma unroll
    for (int w = 1; w < W; ++w) m = fmaxf(m, red_f[w]);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e * NT + (int)threadIdx.x < nh) acc += expf(val[e] - m);
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
        uint32_t prefix = 0u, mask = 0u;
        unsigned want = (unsigned)kk;        // rank (from the top) still to locate among the matching keys
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int c = threadIdx.x; c < 256; c += NT) hist[c] = 0u;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < E; ++e) {
                // scores crowd into a few digits (most keys share their top byte), so the
                // lanes of a warp that hold the same digit add their count in one atomic
                const bool in = e * NT + (int)threadIdx.x < nh && (key[e] & mask) == prefix;
                const unsigned digit = in ? (key[e] >> shift) & 255u : 256u;
                const unsigned peers = __match_any_sync(0xffffffffu, digit);
                if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
            }
            __syncthreads();
            if (warp == 0) {
                // lane l owns bins 255 - 8l down to 248 - 8l (scanned from the top)
                unsigned h8[8], tot = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    h8[q] = hist[255 - 8 * lane - q];
                    tot += h8[q];
                }
                unsigned incl = tot;         // inclusive scan over lanes, from the top
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const unsigned t = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += t;
                }
                unsigned above = incl - tot;  // keys in the bins above this lane's chunk
                if (above < want && want <= incl) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (above < want && want <= above + h8[q]) {
                            sel_digit = 255u - 8u * lane - q;
                            sel_need = want - above;
                        }
                        above += h8[q];
                    }
                }
            }
            __syncthreads();
            prefix |= sel_digit << shift;
            mask |= 255u << shift;
            want = sel_need;
            __syncthreads();                  // sel_* read before the next pass writes them
        }
        T = prefix;
        need = (int)want;
    }
    // kk == nh: every valid key (> 0) is kept (T = 0, need = 0)

    const unsigned lt_mask = (1u << lane) - 1u;
    if (kk > 0) {
        // Output position of a kept key = (# keys > T before it) + min(need, # keys == T before
        // it), in index order j = e * NT + thread. Every warp publishes its per-chunk counts,
        // warp e scans chunk e's counts over the warps, and the chunk totals are summed in order.
        static_assert(E <= W, "one scanning warp per chunk");
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const bool valid = (e * NT + (int)threadIdx.x) < nh;
            const unsigned eb = __ballot_sync(0xffffffffu, valid && key[e] == T);
            const unsigned gb = __ballot_sync(0xffffffffu, valid && key[e] > T);
            if (lane == 0) {
                cnt_eq[e][warp] = __popc(eb);
                cnt_gt[e][warp] = __popc(gb);
            }
        }
        __syncthreads();
        if (warp < E) {                       // warp e: exclusive prefix of chunk e over the warps
            const unsigned ce = lane < W ? cnt_eq[warp][lane] : 0u, cg = lane < W ? cnt_gt[warp][lane] : 0u;
            unsigned ie = ce, ig = cg;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const unsigned te = __shfl_up_sync(0xffffffffu, ie, d), tg = __shfl_up_sync(0xffffffffu, ig, d);
                if (lane >= d) {
                    ie += te;
                    ig += tg;
                }
            }
            if (lane < W) {
                cnt_eq[warp][lane] = ie - ce;
                cnt_gt[warp][lane] = ig - cg;
            }
            if (lane == 31) {
                tot_eq[warp] = ie;
                tot_gt[warp] = ig;
            }
        }
        __syncthreads();
        int eq_base = 0, gt_base = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const bool valid = (e * NT + (int)threadIdx.x) < nh;
            const bool eq = valid && key[e] == T, gtk = valid && key[e] > T;
            const unsigned eb = __ballot_sync(0xffffffffu, eq), gb = __ballot_sync(0xffffffffu, gtk);
            const int eq_rank = eq_base + (int)cnt_eq[e][warp] + __popc(eb & lt_mask);
            const int gt_rank = gt_base + (int)cnt_gt[e][warp] + __popc(gb & lt_mask);
            if (gtk || (eq && eq_rank < need)) {
                const int pos = gt_rank + min(need, eq_rank);
                idx[obase + pos] = e * NT + (int)threadIdx.x;
                log_gate[obase + pos] = val[e] - lse;
            }
            eq_base += (int)tot_eq[e];
            gt_base += (int)tot_gt[e];
        }
    }
    for (int p = kk + (int)threadIdx.x; p < K; p += NT) {
        idx[obase + p] = -1;
        log_gate[obase + p] = -INFINITY;
    }
    if (threadIdx.x == 0) {
        cnt[row] = kk;
        lse_s[row] = lse;
    }
}

template <int E, int W>
cudaError_t go_cta(const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* kv_len, const int32_t* cu,
                   int K, int32_t* idx, int32_t* cnt, float* lg, float* lse_s, int* status, cudaStream_t st) {
    const long long rows = (long long)B * Hkv * n_rows;
    select_cta_kernel<E, W><<<(unsigned)rows, W * 32, 0, st>>>(s, B, Hkv, n_rows, ld_s, kv_len, cu, K, idx, cnt, lg,
                                                             lse_s, status);
    count_launches(1);
    return cudaGetLastError();
}

template <int E>
cudaError_t go(const float* s, int B, int Hkv, int n_rows, int ld_s, const int32_t* kv_len, const int32_t* cu, int K,
               int32_t* idx, int32_t* cnt, float* lg, float* lse_s, int* status, cudaStream_t st) {
    const long long rows = (long long)B * Hkv * n_rows;
    const int warps = 8;
    const long long grid = (rows + warps - 1) / warps;
    select_kernel<E><<<(unsigned)grid, warps * 32, 0, st>>>(s, B, Hkv, n_rows, ld_s, kv_len, cu, K,
                                                            idx, cnt, lg, lse_s, status);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const float* s, int B, int Hkv, int n_rows, int ld_s,
                          const int32_t* kv_len, const int32_t* cu, int K, int max_hist,
                          int32_t* idx, int32_t* cnt, float* log_gate, float* lse_s,
                          int* status, cudaStream_t st) {
#define SAS_SEL_ARGS s, B, Hkv, n_rows, ld_s, kv_len, cu, K, idx, cnt, log_gate, lse_s, status, st
    if (max_hist <= 32) return go<1>(SAS_SEL_ARGS);
    if (max_hist <= 64) return go<2>(SAS_SEL_ARGS);
    if (max_hist <= 128) return go<4>(SAS_SEL_ARGS);
    if (max_hist <= 256) return go<8>(SAS_SEL_ARGS);
    if (max_hist <= 512) return go<16>(SAS_SEL_ARGS);
    // longer rows (decode: one row per sequence and KV head, so few rows): a CTA
    // per row, so that the search is not one warp's serial chain
    if (max_hist <= 1024) return go_cta<4, 8>(SAS_SEL_ARGS);
    if (max_hist <= 4096) return go_cta<4, 32>(SAS_SEL_ARGS);
    if (max_hist <= 8192) return go_cta<8, 32>(SAS_SEL_ARGS);
    return go_cta<16, 32>(SAS_SEL_ARGS);
#undef SAS_SEL_ARGS
}

}  // namespace sas
