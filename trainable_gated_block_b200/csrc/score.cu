// sas_score_select: block-pooled stand-in selector scores fused with the
// Top-K selection and the log-gates.
//
// SAS review (paper.oopus.info) §2.2: the selector scores every history block
// of a query block, s = R_theta(q, {K_Bm}), and the Top-K are kept; §2.4, eq.
// log g: log g_m = s_m - LSE(s). The trained selector (AttnGate) is not part
// of this library; its stand-in is the pooled attention logit
//   s[b,h,i,j] = mean_{64 rows of block i, G query heads of h}(q)
//              . mean_{64 rows of block j}(k[h]) / sqrt(D)  (+ noise[b,h,i,j]),
// for j < i, the noise being an optional input.
//
// Two kernels:
//  * pool_kernel - one CTA per (query block, batch): sums the 64 rows of q
//    (all query heads) and of k in fp32 with 16-byte loads, then folds the G
//    heads of each KV head; writes the block means qp, kp [B, Hkv, NQB, D]
//    (fp32, in the workspace). Reads q and k once: HBM-bound.
//  * score_select_kernel - one warp per selection row (b, h, i), eight rows of
//    one (b, h) per CTA. Chunks of 32 pooled keys are staged in shared memory
//    (one row per lane, 16-byte rows padded against bank conflicts, read as
//    float4) and every lane forms
//    the dot product of its key with the warp's pooled query, so that lane l
//    holds s[i][32 e + l] - the register layout of the warp-row selection,
//    which runs next (select_row.cuh). s is written once (the backward's
//    Jacobian reads it).
// Rows of more than 512 history blocks: the scores are written by the same
// kernel without the selection, then selected by sas_select's CTA-per-row
// kernel.
//
// Decode (sas_pool_pages, sas_score_select_decode): the mean key of every
// (page, KV head) is kept in a pooled-key cache (fp32 [pages, Hkv, D]),
// filled once per page by pool_pages_kernel (one warp per 16 KiB page tile).
// A decode query's scores then read only that cache: score_decode_kernel
// gathers the pooled keys of the sequence's history pages through the page
// table (8 lanes per key, 128-byte reads) and dots them with the query
// pooled over its GQA group; the scores go to sas_select's decode path.
#include "common.cuh"
#include "launch.h"
#include "select_row.cuh"

namespace sas {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kRowsPerCta = 8;

// qp[b, h, i, :] = mean over the 64 rows of block i and the G query heads of
// KV head h; kp[b, h, i, :] = mean over the 64 rows of block i of k[:, :, h].
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int S, int Hq, int Hkv, int D,
            float* __restrict__ qp, float* __restrict__ kp) {
    extern __shared__ float acc[];                  // [Hq * D] q sums, then [Hkv * D] k sums
    const int i = blockIdx.x, b = blockIdx.y, NQB = gridDim.x;
    const int G = Hq / Hkv;
    const long long row0 = (long long)b * S + (long long)i * kBlock;
    for (int pass = 0; pass < 2; ++pass) {
        const __nv_bfloat16* src = pass == 0 ? q : k;
        const int cols = (pass == 0 ? Hq : Hkv) * D;             // bf16 per token row
        float* dst = acc + (pass == 0 ? 0 : Hq * D);
        for (int c = threadIdx.x; c < cols / 8; c += kPoolThreads) {   // 16-byte chunk c of every row
            float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const uint4* p = reinterpret_cast<const uint4*>(src + row0 * cols) + c;
#pragma unroll 8
            for (int r = 0; r < kBlock; ++r) {
                const uint4 w = __ldg(p + (long long)r * (cols / 8));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = bf16x2_to_f32(ws[e]);
                    a[2 * e] += f.x;
                    a[2 * e + 1] += f.y;
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[c * 8 + e] = a[e];
        }
    }
    __syncthreads();
    const float inv_q = 1.f / (float)(kBlock * G), inv_k = 1.f / (float)kBlock;
    for (int t = threadIdx.x; t < Hkv * D; t += kPoolThreads) {
        const int h = t / D, d = t % D;
        float sq = 0.f;
        for (int g = 0; g < G; ++g) sq += acc[(h * G + g) * D + d];
        const long long o = (((long long)b * Hkv + h) * NQB + i) * D + d;
        qp[o] = sq * inv_q;
        kp[o] = acc[Hq * D + t] * inv_k;
    }
}

// Scores of the rows of one CTA: warp w owns row i = 8 blockIdx.x + w of
// (b, h) = blockIdx.y; lane l of the warp computes j = 32 e + l for every
// chunk e below `chunks`. The pooled keys of chunk e are staged by the CTA.
template <int E, bool kSelect>
__global__ void __launch_bounds__(kRowsPerCta * 32, 3)     // three CTAs per SM: 85 registers at most
score_select_kernel(const float* __restrict__ qp, const float* __restrict__ kp, int NQB, int D, float inv_sqrt_d,
                    const float* __restrict__ noise, int ld_noise, float* __restrict__ s, int ld_s, int K,
                    int32_t* __restrict__ idx, int32_t* __restrict__ cnt, float* __restrict__ log_gate,
                    float* __restrict__ lse_s, int* status) {
    extern __shared__ float sm[];
    // two [32][D + 4] buffers of pooled keys (chunk e in buffer e & 1): rows 16-byte aligned,
    // and the +4 padding keeps the eight lanes of each quarter-warp 128-bit load on distinct
    // banks. Chunk e + 1 is loaded into registers while chunk e is used.
    const int ldk = D + 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* qrow = sm + 2 * 32 * ldk + warp * D;                // this warp's pooled query
    const long long bh = blockIdx.y;
    const int i = blockIdx.x * kRowsPerCta + warp;
    const bool live = i < NQB;
    const int i_max = min(NQB - 1, (int)blockIdx.x * kRowsPerCta + kRowsPerCta - 1);   // longest row of the CTA
    const long long row = bh * NQB + i;
    if (live)
        for (int d = lane; d < D; d += 32) qrow[d] = qp[row * D + d];
    const int chunks = kSelect ? E : (i_max + 31) / 32;
    const int used = (i_max + 31) / 32;                        // chunks holding some j < i_max
    constexpr int kPer = 32 * 128 / 4 / (kRowsPerCta * 32);    // float4 of a chunk per thread (D = 128)
    float4 nxt[kPer];
    auto fetch = [&](int e) {                                  // chunk e -> registers
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int t = threadIdx.x + u * kRowsPerCta * 32;
            const int r = t / (D / 4), d4 = t % (D / 4);
            nxt[u] = (t < 8 * D && e * 32 + r < i_max)
                         ? reinterpret_cast<const float4*>(kp + (bh * NQB + e * 32 + r) * D)[d4]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto stash = [&](int e) {                                  // registers -> buffer e & 1
        float* kc = sm + (e & 1) * 32 * ldk;
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int t = threadIdx.x + u * kRowsPerCta * 32;
            if (t < 8 * D) reinterpret_cast<float4*>(kc + (t / (D / 4)) * ldk)[t % (D / 4)] = nxt[u];
        }
    };
    float val[kSelect ? E : 1];
#pragma unroll
    for (int e = 0; e < (kSelect ? E : 1); ++e) val[e] = -INFINITY;
    if (used > 0) {
        fetch(0);
        stash(0);
    }
    for (int e = 0; e < chunks; ++e) {
        if (e < used) {                                        // the same for the whole CTA
            if (e + 1 < used) fetch(e + 1);                    // in flight while chunk e is used
            __syncthreads();                                   // chunk e is in its buffer
        }
        const int j = e * 32 + lane;
        if (live && j < i) {
            const float4* kr = reinterpret_cast<const float4*>(sm + (e & 1) * 32 * ldk + lane * ldk);
            const float4* qr = reinterpret_cast<const float4*>(qrow);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;       // four chains
            for (int d4 = 0; d4 < D / 4; ++d4) {
                const float4 kv = kr[d4], qv = qr[d4];
                a0 = fmaf(qv.x, kv.x, a0);
                a1 = fmaf(qv.y, kv.y, a1);
                a2 = fmaf(qv.z, kv.z, a2);
                a3 = fmaf(qv.w, kv.w, a3);
            }
            float v = ((a0 + a1) + (a2 + a3)) * inv_sqrt_d;
            if (noise != nullptr) v += __ldg(noise + row * (long long)ld_noise + j);
            s[row * (long long)ld_s + j] = v;
            if (kSelect) {
#pragma unroll
                for (int ee = 0; ee < (kSelect ? E : 1); ++ee)
                    if (ee == e) val[ee] = v;
            }
        }
        if (e + 1 < used) stash(e + 1);                        // the other buffer: no one reads it now
    }
    if (kSelect && live) select_warp_row<kSelect ? E : 1>(val, i, K, row, idx, cnt, log_gate, lse_s, status);
}

template <int E>
cudaError_t go_fused(const float* qp, const float* kp, int B, int Hkv, int NQB, int D, float inv, const float* noise,
                     int ld_noise, float* s, int ld_s, int K, int32_t* idx, int32_t* cnt, float* lg, float* lse_s,
                     int* status, cudaStream_t st) {
    const dim3 grid((NQB + kRowsPerCta - 1) / kRowsPerCta, B * Hkv);
    const size_t sm = sizeof(float) * (2 * 32 * (D + 4) + kRowsPerCta * D);
    score_select_kernel<E, true><<<grid, kRowsPerCta * 32, sm, st>>>(qp, kp, NQB, D, inv, noise, ld_noise, s, ld_s,
                                                                     K, idx, cnt, lg, lse_s, status);
    count_launches(1);
    return cudaGetLastError();
}

// kpool[page, h, :] = mean over the 64 rows of k_cache[page, h] (fp32 sums).
// One warp per (page, head); D/8 lanes cover a row with 16-byte loads, 32/(D/8)
// rows per load round, and the partial sums of the row groups are folded by
// shuffles.
__global__ void __launch_bounds__(256)
pool_pages_kernel(const __nv_bfloat16* __restrict__ k_cache, int num_pages, int Hkv, int D,
                  const int32_t* __restrict__ pages, int n_pages, float* __restrict__ kpool, int* status) {
    const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= (long long)n_pages * Hkv) return;
    const int h = (int)(w % Hkv);
    int page = (int)(w / Hkv);
    if (pages != nullptr) page = pages[page];
    if (page < 0 || page >= num_pages) {
        if (lane == 0) flag_status(status, kStatusBadData);
        return;
    }
    const int C = D / 8, R = 32 / C;                 // 16-byte chunks per row, rows per round
    const int c = lane % C, rsub = lane / C;
    const uint4* tile = reinterpret_cast<const uint4*>(k_cache + ((long long)page * Hkv + h) * kBlock * D);
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int r = rsub; r < kBlock; r += R) {
        const uint4 v = __ldg(tile + r * C + c);
        const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = bf16x2_to_f32(ws[e]);
            a[2 * e] += f.x;
            a[2 * e + 1] += f.y;
        }
    }
    for (int off = C; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], off);
    if (rsub == 0) {
        float4* dst = reinterpret_cast<float4*>(kpool + ((long long)page * Hkv + h) * D + 8 * c);
        const float inv = 1.f / (float)kBlock;
        dst[0] = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
        dst[1] = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
    }
}

// Decode scores: CTA (chunk, row = (n, h)) scores history blocks
// [128 chunk, 128 chunk + 128) of row (n, h); warp w takes 4 blocks per round,
// 8 lanes per block, each lane a strided quarter (D = 128) of the pooled key.
constexpr int kDecScoreBlocks = 128;
__global__ void __launch_bounds__(256)
score_decode_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ kpool, int num_pages,
                    const int32_t* __restrict__ page_table, int max_pages, const int32_t* __restrict__ kv_len,
                    int Hq, int Hkv, int D, float inv_sqrt_d, const float* __restrict__ noise, int ld_noise,
                    float* __restrict__ s, int ld_s, int* status) {
    __shared__ float qbar[128];
    const int row = blockIdx.y, n = row / Hkv, h = row % Hkv, G = Hq / Hkv;
    const int L = kv_len[n];
    int nh = L >= 1 ? (L - 1) / kBlock : 0;
    if (nh > ld_s || nh > max_pages) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_status(status, kStatusBadData);
        nh = min(ld_s, max_pages);
    }
    const int j0 = blockIdx.x * kDecScoreBlocks;
    if (j0 >= nh) return;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {     // the query pooled over its GQA group
        float acc = 0.f;
        for (int g = 0; g < G; ++g) acc += __bfloat162float(q[((long long)n * Hq + h * G + g) * D + d]);
        qbar[d] = acc / (float)G;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = lane >> 3, l8 = lane & 7;
    const int nq = D / 32;                                     // float4 loads per lane
    for (int jj = warp * 4 + sub; jj < kDecScoreBlocks; jj += 32) {
        const int j = j0 + jj;
        const bool in = j < nh;
        const int page = in ? page_table[(long long)n * max_pages + j] : 0;
        const bool ok = in && page >= 0 && page < num_pages;
        float acc = 0.f;
        if (ok) {
            const float4* kr = reinterpret_cast<const float4*>(kpool + ((long long)page * Hkv + h) * D);
            for (int k = 0; k < nq; ++k) {
                const float4 kv = __ldg(kr + l8 + 8 * k);
                const float4 qv = reinterpret_cast<const float4*>(qbar)[l8 + 8 * k];
                acc = fmaf(kv.x, qv.x, fmaf(kv.y, qv.y, fmaf(kv.z, qv.z, fmaf(kv.w, qv.w, acc))));
            }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (in && l8 == 0) {
            float v = __int_as_float(0x7fc00000);              // a bad page id: NaN, flagged by select too
            if (ok) {
                v = acc * inv_sqrt_d;
                if (noise != nullptr) v += __ldg(noise + (long long)row * ld_noise + j);
            } else {
                flag_status(status, kStatusBadData);
            }
            s[(long long)row * ld_s + j] = v;
        }
    }
}

}  // namespace

cudaError_t launch_pool_pages(const void* k_cache, int num_pages, int Hkv, int D, const int32_t* pages, int n_pages,
                              float* kpool, int* status, cudaStream_t st) {
    const long long warps = (long long)n_pages * Hkv;
    pool_pages_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>((const __nv_bfloat16*)k_cache, num_pages, Hkv, D,
                                                                   pages, n_pages, kpool, status);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_score_select_decode(const DecodeScoreArgs& a, cudaStream_t st) {
    const dim3 grid((a.ld_s + kDecScoreBlocks - 1) / kDecScoreBlocks, a.N * a.Hkv);
    score_decode_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)a.q, a.kpool, a.num_pages, a.page_table,
                                              a.max_pages, a.kv_len, a.Hq, a.Hkv, a.D, 1.f / sqrtf((float)a.D),
                                              a.noise, a.ld_noise, a.s, a.ld_s, a.status);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_select(a.s, a.N, a.Hkv, 1, a.ld_s, a.kv_len, nullptr, a.K, a.ld_s, a.idx, a.cnt, a.log_gate,
                         a.lse_s, a.status, st);
}

size_t score_workspace(int B, int S, int Hkv, int D) {
    const size_t n = (size_t)B * Hkv * ((S + 63) / 64) * D;
    return 2 * ((sizeof(float) * n + 255) & ~size_t(255));
}

cudaError_t launch_score_select(const ScoreArgs& a, cudaStream_t st) {
    const int NQB = a.S / kBlock;
    const size_t n = (size_t)a.B * a.Hkv * NQB * a.D;
    float* qp = static_cast<float*>(a.workspace);
    float* kp = qp + (((sizeof(float) * n + 255) & ~size_t(255)) / sizeof(float));
    const size_t psm = sizeof(float) * (size_t)(a.Hq + a.Hkv) * a.D;
    cudaError_t e = cudaFuncSetAttribute(pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm);
    if (e != cudaSuccess) return e;
    pool_kernel<<<dim3(NQB, a.B), kPoolThreads, psm, st>>>((const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k,
                                                             a.S, a.Hq, a.Hkv, a.D, qp, kp);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const float inv = 1.f / sqrtf((float)a.D);
    const int max_hist = NQB - 1;
#define SAS_FUSED_ARGS qp, kp, a.B, a.Hkv, NQB, a.D, inv, a.noise, a.ld_noise, a.s, a.ld_s, a.K, a.idx, a.cnt, \
                       a.log_gate, a.lse_s, a.status, st
    if (max_hist <= 32) return go_fused<1>(SAS_FUSED_ARGS);
    if (max_hist <= 64) return go_fused<2>(SAS_FUSED_ARGS);
    if (max_hist <= 128) return go_fused<4>(SAS_FUSED_ARGS);
    if (max_hist <= 256) return go_fused<8>(SAS_FUSED_ARGS);
    if (max_hist <= 512) return go_fused<16>(SAS_FUSED_ARGS);
#undef SAS_FUSED_ARGS
    // longer rows: scores first, then the CTA-per-row selection
    const dim3 grid((NQB + kRowsPerCta - 1) / kRowsPerCta, a.B * a.Hkv);
    const size_t sm = sizeof(float) * (2 * 32 * (a.D + 4) + kRowsPerCta * a.D);
    score_select_kernel<1, false><<<grid, kRowsPerCta * 32, sm, st>>>(
        qp, kp, NQB, a.D, inv, a.noise, a.ld_noise, a.s, a.ld_s, a.K, a.idx, a.cnt, a.log_gate, a.lse_s, a.status);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_select(a.s, a.B, a.Hkv, NQB, a.ld_s, nullptr, nullptr, a.K, max_hist, a.idx, a.cnt, a.log_gate,
                         a.lse_s, a.status, st);
}

}  // namespace sas
