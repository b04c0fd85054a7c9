// sas_score_select: block-pooled stand-in selector scores, then the Top-K
// selection and the log-gates.
//
// SAS review (paper.oopus.info) §2.2: the selector scores every history block
// of a query block, s = R_theta(q, {K_Bm}), and the Top-K are kept; §2.4, eq.
// log g: log g_m = s_m - LSE(s). The trained selector (AttnGate) is not part
// of this library; its stand-in is the pooled attention logit
//   s[b,h,i,j] = mean_{64 rows of block i, G query heads of h}(q)
//              . mean_{64 rows of block j}(k[h]) / sqrt(D)  (+ noise[b,h,i,j]),
// for j < i, the noise being an optional input.
//
// Prefill, three kernels:
//  * pool_kernel - one CTA per (query block, batch): sums the 64 rows of q
//    (all query heads) and of k in fp32 with 16-byte loads, then folds the G
//    heads of each KV head; writes the block means qp, kp [B, Hkv, NQB, D]
//    (fp32, in the workspace). Reads q and k once: HBM-bound.
//  * score_tile_kernel - the lower triangle of qp kp^T / sqrt(D) (+ noise) in
//    64 x 64 tiles, 4 x 4 products per thread from shared memory; s is
//    written once (the backward's Jacobian reads it).
//  * the selection of sas_select on those rows (warp per row, CTA per row
//    beyond 512 history blocks), reading s back from L2.
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

namespace sas {
namespace {

constexpr int kPoolThreads = 256;

// qp[b, h, i, :] = mean over the 64 rows of block i and the G query heads of
// KV head h; kp[b, h, i, :] = mean over the 64 rows of block i of k[:, :, h].
// One CTA per (KV head h, query block i, batch b), h fastest so that the CTAs
// running together read whole token rows of q and k: a token row of the group
// is C = (G + 1) D / 8 16-byte chunks (G query heads, contiguous in q, then
// the KV head's key row), thread t sums chunk t % C over the rows
// t / C, t / C + R, ... (R = 256 / C row groups), the R partial sums meet in
// shared memory and D threads fold them and the G heads. Small CTAs keep
// every SM's share of the bytes within one CTA of the mean.
__global__ void __launch_bounds__(kPoolThreads, 4)     // eight 16-byte loads in flight per thread
pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int S, int Hq, int Hkv, int D,
            float* __restrict__ qp, float* __restrict__ kp) {
    extern __shared__ float acc[];                  // [R][C * 8] partial sums
    const int h = blockIdx.x, i = blockIdx.y, b = blockIdx.z, NQB = gridDim.y;
    const int G = Hq / Hkv;
    const int cq = G * D / 8, C = cq + D / 8;       // chunks of the group's q row, of the whole row
    const int R = max(1, kPoolThreads / C);
    const long long row0 = (long long)b * S + (long long)i * kBlock;
    const uint4* qsrc = reinterpret_cast<const uint4*>(q + (row0 * Hq + (long long)h * G) * D);
    const uint4* ksrc = reinterpret_cast<const uint4*>(k + (row0 * Hkv + h) * D);
    const long long qstride = (long long)Hq * D / 8, kstride = (long long)Hkv * D / 8;   // chunks per token row
    for (int u = threadIdx.x; u < C * R; u += kPoolThreads) {
        const int c = u % C, rg = u / C;
        const uint4* p = c < cq ? qsrc + c : ksrc + (c - cq);
        const long long stride = c < cq ? qstride : kstride;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int r = rg; r < kBlock; r += R) {
            const uint4 w = __ldg(p + (long long)r * stride);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = bf16x2_to_f32(ws[e]);
                a[2 * e] += f.x;
                a[2 * e + 1] += f.y;
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[(size_t)rg * C * 8 + c * 8 + e] = a[e];
    }
    __syncthreads();
    const float inv_q = 1.f / (float)(kBlock * G), inv_k = 1.f / (float)kBlock;
    for (int d = threadIdx.x; d < D; d += kPoolThreads) {
        float sq = 0.f, sk = 0.f;
        for (int rg = 0; rg < R; ++rg) {
            const float* pr = acc + (size_t)rg * C * 8;
            for (int g = 0; g < G; ++g) sq += pr[g * D + d];
            sk += pr[G * D + d];
        }
        const long long o = (((long long)b * Hkv + h) * NQB + i) * D + d;
        qp[o] = sq * inv_q;
        kp[o] = sk * inv_k;
    }
}

// Scores of one 64 x 64 tile (query blocks [64 ti, 64 ti + 64) x key blocks
// [64 tj, 64 tj + 64), tj <= ti) of (b, h) = blockIdx.y: the tile's pooled
// queries and keys are staged in shared memory transposed ([d][row], rows
// padded to 68 floats), and each thread accumulates a 4 x 4 block of dot
// products over D from two 128-bit loads per d (the query load is a
// broadcast, the key loads of a half-warp cover 256 contiguous bytes), so
// every staged value feeds 4 products. Entries with j < i get noise added and
// are written; the selection then reads them back (from L2).
constexpr int kTile = 64;
constexpr int kTileLd = kTile + 4;
__global__ void __launch_bounds__(256)
score_tile_kernel(const float* __restrict__ qp, const float* __restrict__ kp, int NQB, int D, float inv_sqrt_d,
                  const float* __restrict__ noise, int ld_noise, float* __restrict__ s, int ld_s) {
    extern __shared__ __align__(16) float sm[];
    float* qs = sm;                                   // [D][kTileLd] pooled queries of the tile's rows
    float* ks = sm + (size_t)D * kTileLd;             // [D][kTileLd] pooled keys of the tile's columns
    // lower-triangle tile index -> (ti, tj): tiles of row ti are ti*(ti+1)/2 .. + ti
    const int t = blockIdx.x;
    int ti = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
    while (ti * (ti + 1) / 2 > t) --ti;
    const int tj = t - ti * (ti + 1) / 2;
    const long long bh = blockIdx.y;
    const int i0 = ti * kTile, j0 = tj * kTile;
    // lanes of a warp take consecutive rows: 16-byte global loads, conflict-free transposed stores;
    // eight loads of each operand are in flight per thread before the stores
    constexpr int kU = 8;
    const int units = kTile * (D / 4);
    for (int e0 = threadIdx.x; e0 < units; e0 += kU * blockDim.x) {
        float4 qv[kU], kv[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int e = e0 + u * blockDim.x;
            const int r = e % kTile, d4 = e / kTile;
            const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
            const bool in = e < units;
            qv[u] = (in && i0 + r < NQB) ? reinterpret_cast<const float4*>(qp + (bh * NQB + i0 + r) * D)[d4] : zero;
            kv[u] = (in && j0 + r < NQB) ? reinterpret_cast<const float4*>(kp + (bh * NQB + j0 + r) * D)[d4] : zero;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int e = e0 + u * blockDim.x;
            if (e >= units) break;
            const int r = e % kTile, d4 = e / kTile;
            float* qd = qs + (4 * d4) * kTileLd + r;
            float* kd = ks + (4 * d4) * kTileLd + r;
            qd[0] = qv[u].x; qd[kTileLd] = qv[u].y; qd[2 * kTileLd] = qv[u].z; qd[3 * kTileLd] = qv[u].w;
            kd[0] = kv[u].x; kd[kTileLd] = kv[u].y; kd[2 * kTileLd] = kv[u].z; kd[3 * kTileLd] = kv[u].w;
        }
    }
    __syncthreads();
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    float acc[4][4] = {};
#pragma unroll 2
    for (int d = 0; d < D; ++d) {
        const float4 av = *reinterpret_cast<const float4*>(qs + d * kTileLd + ty * 4);
        const float4 cv = *reinterpret_cast<const float4*>(ks + d * kTileLd + tx * 4);
        const float a[4] = {av.x, av.y, av.z, av.w}, c[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], c[w], acc[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty * 4 + u;
        if (i >= NQB) continue;
        const long long row = bh * NQB + i;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int j = j0 + tx * 4 + w;
            if (j < i) {
                float v = acc[u][w] * inv_sqrt_d;
                if (noise != nullptr) v += __ldg(noise + row * (long long)ld_noise + j);
                s[row * (long long)ld_s + j] = v;
            }
        }
    }
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
__global__ void __launch_bounds__(256, 4)
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
    const int C = (a.Hq / a.Hkv + 1) * a.D / 8;
    const size_t psm = sizeof(float) * 8 * (size_t)C * (size_t)std::max(1, kPoolThreads / C);
    cudaError_t e = cudaFuncSetAttribute(pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm);
    if (e != cudaSuccess) return e;
    pool_kernel<<<dim3(a.Hkv, NQB, a.B), kPoolThreads, psm, st>>>((const __nv_bfloat16*)a.q,
                                                                    (const __nv_bfloat16*)a.k, a.S, a.Hq, a.Hkv,
                                                                    a.D, qp, kp);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int nt = (NQB + kTile - 1) / kTile;
    const size_t tsm = sizeof(float) * 2 * (size_t)a.D * kTileLd;
    if ((e = cudaFuncSetAttribute(score_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm)) !=
        cudaSuccess)
        return e;
    score_tile_kernel<<<dim3(nt * (nt + 1) / 2, a.B * a.Hkv), 256, tsm, st>>>(
        qp, kp, NQB, a.D, 1.f / sqrtf((float)a.D), a.noise, a.ld_noise, a.s, a.ld_s);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_select(a.s, a.B, a.Hkv, NQB, a.ld_s, nullptr, nullptr, a.K, NQB - 1, a.idx, a.cnt, a.log_gate,
                         a.lse_s, a.status, st);
}

}  // namespace sas
